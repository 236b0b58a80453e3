"""Python binding of liblrkv.so: split-value-cache attention on B200.

A thin ctypes layer with the C ABI's names (include/lrkv.h).  It marshals
``torch.Tensor`` device pointers, shapes and the current CUDA stream into the
C calls; every step of the computation runs in the library's CUDA kernels.
There is no fallback: if the shared library is missing, importing the
functions raises.

Typical decode call::

    import lora_shared_kv_b200 as lrkv
    prob = lrkv.make_problem(S, N, Hq, Hkv, d, r, mode=lrkv.BASE_SHARED)
    kv = lrkv.kv_view_dense(k, v)              # k, v: [S, Hkv, L, d] bf16
    uv = lrkv.u_view(u)                         # u: [S, N_U, L, r] bf16
    ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, L), dtype=torch.uint8, device="cuda")
    lrkv.lrkv_attn_decode(prob, q, kv, seq_lens, L, uv, b, offsets, out, ws)
"""

import ctypes
import os

import torch

BASE_SHARED = 0
BASE_LR_SHARED = 1
BF16 = 0
F32 = 1

_STATUS = {
    0: "LRKV_OK",
    1: "LRKV_ERR_INVALID_ARGUMENT",
    2: "LRKV_ERR_UNSUPPORTED",
    3: "LRKV_ERR_MISALIGNED",
    4: "LRKV_ERR_WORKSPACE_TOO_SMALL",
    5: "LRKV_ERR_CUDA",
    6: "LRKV_ERR_DEVICE_FAULT",
    7: "LRKV_ERR_TIMEOUT",
}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblrkv.so")

# Every exported symbol of include/lrkv.h.
EXPORTS = (
    "lrkv_append_lr_cache",
    "lrkv_append_lr_cache_ranges",
    "lrkv_value_projection",
    "lrkv_decode_workspace_bytes",
    "lrkv_attn_decode",
    "lrkv_decode_kv_heads_workspace_bytes",
    "lrkv_attn_decode_kv_heads",
    "lrkv_attn_decode_static_scratch",
    "lrkv_query_static_scratch_status",
    "lrkv_prefill_workspace_bytes",
    "lrkv_attn_prefill_chunk",
    "lrkv_workspace_reset",
    "lrkv_query_device_status",
    "lrkv_debug_stall_next_launch",
    "lrkv_status_string",
    "lrkv_last_error_detail",
    "lrkv_version",
)


class LrkvError(RuntimeError):
    def __init__(self, status, detail):
        self.status = status
        self.name = _STATUS.get(status, str(status))
        super().__init__(f"{self.name}: {detail}")


class Problem(ctypes.Structure):
    _fields_ = [("num_sessions", ctypes.c_int32), ("num_agents", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("rank", ctypes.c_int32), ("mode", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float)]


class KVView(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("stride_session", ctypes.c_int64),
                ("stride_head", ctypes.c_int64), ("stride_token", ctypes.c_int64),
                ("page_table", ctypes.c_void_p), ("page_table_stride", ctypes.c_int64),
                ("stride_page", ctypes.c_int64), ("page_size", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


class UView(ctypes.Structure):
    _fields_ = [("u", ctypes.c_void_p), ("stride_session", ctypes.c_int64),
                ("stride_agent", ctypes.c_int64), ("stride_token", ctypes.c_int64),
                ("num_rows", ctypes.c_int32)]


_lib = None


def lib():
    """Load liblrkv.so (built in-tree by ``python -m lora_shared_kv_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m lora_shared_kv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.lrkv_append_lr_cache.argtypes = [vp, vp, i32, i32, i32, i32, P(UView), i32, i32, vp]
        L.lrkv_append_lr_cache_ranges.argtypes = [vp, i32, vp, i32, i32, i32, P(i32), P(i32), P(UView), i32, vp]
        L.lrkv_value_projection.argtypes = [P(Problem), vp, i32, i32, vp, P(KVView), i32, P(UView), i32, i32, vp, sz,
                                            vp]
        L.lrkv_decode_workspace_bytes.argtypes = [P(Problem), i32]
        L.lrkv_decode_workspace_bytes.restype = sz
        L.lrkv_attn_decode.argtypes = [P(Problem), vp, P(KVView), vp, i32, P(UView), vp, vp, vp, i32, vp, sz, vp]
        L.lrkv_decode_kv_heads_workspace_bytes.argtypes = [P(Problem), i32, i32]
        L.lrkv_decode_kv_heads_workspace_bytes.restype = sz
        L.lrkv_attn_decode_kv_heads.argtypes = [P(Problem), i32, i32, vp, P(KVView), vp, i32, P(UView), vp, vp, vp,
                                                i32, vp, sz, vp]
        L.lrkv_attn_decode_static_scratch.argtypes = [P(Problem), vp, P(KVView), vp, i32, P(UView), vp, vp, vp,
                                                      i32, vp]
        L.lrkv_prefill_workspace_bytes.argtypes = [P(Problem), i32, i32]
        L.lrkv_prefill_workspace_bytes.restype = sz
        L.lrkv_attn_prefill_chunk.argtypes = [P(Problem), vp, P(KVView), i32, i32, i32, P(UView), vp, vp, vp,
                                              i32, vp, sz, vp]
        L.lrkv_workspace_reset.argtypes = [vp, sz, vp]
        L.lrkv_query_device_status.argtypes = [vp, i32, P(ctypes.c_uint32), vp]
        L.lrkv_query_static_scratch_status.argtypes = [i32, P(ctypes.c_uint32), vp]
        L.lrkv_debug_stall_next_launch.argtypes = [ctypes.c_uint32]
        L.lrkv_status_string.argtypes = [i32]
        L.lrkv_status_string.restype = ctypes.c_char_p
        L.lrkv_last_error_detail.argtypes = []
        L.lrkv_last_error_detail.restype = ctypes.c_char_p
        L.lrkv_version.restype = i32
        for name in ("lrkv_append_lr_cache", "lrkv_attn_decode", "lrkv_attn_decode_kv_heads",
                     "lrkv_attn_decode_static_scratch",
                     "lrkv_attn_prefill_chunk",
                     "lrkv_workspace_reset", "lrkv_query_device_status", "lrkv_query_static_scratch_status",
                     "lrkv_debug_stall_next_launch"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def _check(status):
    if status != 0:
        raise LrkvError(status, lib().lrkv_last_error_detail().decode(errors="replace"))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _require(cond, msg):
    if not cond:
        raise ValueError(msg)


def _on_device(**tensors):
    """Every tensor the kernels read or write must live in the current CUDA device's memory: the GPU would
    dereference a host pointer, or another device's memory, as if it were its own.  None is skipped (an
    optional argument)."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor, got one on {t.device}")
        if dev is None:
            dev = torch.cuda.current_device()
        if t.get_device() != dev:
            raise ValueError(f"{name} is on cuda:{t.get_device()} but the current device is cuda:{dev}")


# ---------------------------------------------------------------------------
# views
# ---------------------------------------------------------------------------

def make_problem(S, N, Hq, Hkv, d, r, mode=BASE_SHARED, softmax_scale=0.0):
    return Problem(S, N, Hq, Hkv, d, r, mode, softmax_scale)


def kv_view_dense(k, v):
    """k, v: bf16 [S, Hkv, L, d] with d contiguous (same strides)."""
    _require(k.dtype == torch.bfloat16 and v.dtype == torch.bfloat16 and k.dim() == 4, "k, v: bf16 [S, Hkv, L, d]")
    _require(k.stride() == v.stride() and k.stride(3) == 1, "k, v: same strides, d contiguous")
    _on_device(k=k, v=v)
    return KVView(k.data_ptr(), v.data_ptr(), k.stride(0), k.stride(1), k.stride(2), None, 0, 0, 0, 0)


def kv_view_paged(k_pages, v_pages, page_table):
    """k_pages, v_pages: bf16 [P, Hkv, page, d]; page_table: int32 [S, n_logical_pages] on the device."""
    _require(k_pages.dtype == torch.bfloat16 and v_pages.dtype == torch.bfloat16 and k_pages.dim() == 4
             and k_pages.stride() == v_pages.stride(), "k_pages, v_pages: bf16 [P, Hkv, page, d], same strides")
    _require(page_table.dtype == torch.int32 and page_table.dim() == 2 and page_table.stride(1) == 1,
             "page_table: int32 [S, n_logical_pages], rows contiguous")
    _on_device(k_pages=k_pages, v_pages=v_pages, page_table=page_table)
    return KVView(k_pages.data_ptr(), v_pages.data_ptr(), 0, k_pages.stride(1), k_pages.stride(2),
                  page_table.data_ptr(), page_table.stride(0), k_pages.stride(0), k_pages.shape[2],
                  k_pages.shape[0])


def u_view(u):
    """u: bf16 [S, N_U, rows, r] with r contiguous."""
    _require(u.dtype == torch.bfloat16 and u.dim() == 4 and u.stride(3) == 1, "u: bf16 [S, N_U, rows, r], r contiguous")
    _on_device(u=u)
    return UView(u.data_ptr(), u.stride(0), u.stride(1), u.stride(2), u.shape[2])


# ---------------------------------------------------------------------------
# the C entry points
# ---------------------------------------------------------------------------

def lrkv_append_lr_cache(x, a, u, session, start_row, stream=None, uview=None):
    """U[session, i, start_row + t, :] = x[t] @ a[i] for every slot i of a (bit-exact fixed order)."""
    T, Dm = x.shape
    n_a, Dm2, r = a.shape
    _require(Dm == Dm2 and x.is_contiguous() and a.is_contiguous(), "x [T, Dm] and a [n_a, Dm, r], contiguous")
    _on_device(x=x, a=a)
    uv = uview if uview is not None else u_view(u)
    _check(lib().lrkv_append_lr_cache(_ptr(x), _ptr(a), n_a, T, Dm, r, ctypes.byref(uv), session, start_row,
                                      _stream(stream)))


def lrkv_append_lr_cache_ranges(x, a, u, session, row_begin, row_end, stream=None, uview=None):
    """U[session, i, t, :] = x[t] @ a[i] for t in [row_begin[i], row_end[i]) of every slot i of a:
    the per-agent catch-up append (bit-exact fixed order).  x holds the hidden states by absolute position."""
    x_rows, Dm = x.shape
    n_a, Dm2, r = a.shape
    _require(Dm == Dm2 and x.is_contiguous() and a.is_contiguous(), "x [rows, Dm] and a [n_a, Dm, r], contiguous")
    _require(len(row_begin) == n_a and len(row_end) == n_a, "one row_begin and one row_end per slot of a")
    _on_device(x=x, a=a)
    uv = uview if uview is not None else u_view(u)
    b = (ctypes.c_int32 * n_a)(*[int(v) for v in row_begin])
    e = (ctypes.c_int32 * n_a)(*[int(v) for v in row_end])
    _check(lib().lrkv_append_lr_cache_ranges(_ptr(x), x_rows, _ptr(a), n_a, Dm, r, b, e, ctypes.byref(uv),
                                             session, _stream(stream)))


def lrkv_value_projection(problem, x, w, kv, kv_rows, u, session, start_row, workspace, stream=None):
    """[V_base | U_1..U_n] = x @ w for T new tokens, written into kv.v rows and u rows
    [start_row, start_row + T) of `session` (x [T, Dm], w [Dm, Hkv*d + n_u*r])."""
    T, Dm = x.shape
    _require(x.is_contiguous() and w.is_contiguous() and w.shape[0] == Dm, "x [T, Dm] and w [Dm, cols], contiguous")
    _on_device(x=x, w=w, workspace=workspace)
    uv = u if isinstance(u, UView) else u_view(u)
    _check(lib().lrkv_value_projection(ctypes.byref(problem), _ptr(x), T, Dm, _ptr(w), ctypes.byref(kv), int(kv_rows),
                                       ctypes.byref(uv), session, start_row, _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)))


def lrkv_decode_workspace_bytes(problem, max_seq_len):
    n = lib().lrkv_decode_workspace_bytes(ctypes.byref(problem), int(max_seq_len))
    if n == 0:
        raise LrkvError(1, "invalid decode shape")
    return n


def lrkv_attn_decode(problem, q, kv, seq_lens, max_seq_len, u, b, offsets, out, workspace, stream=None):
    """out[s, i, h] = attention of q[s, i, h] over the shared cache with agent i's low-rank values."""
    _require(q.is_contiguous() and b.is_contiguous() and out.is_contiguous(), "q, b and out must be contiguous")
    _on_device(q=q, seq_lens=seq_lens, b=b, offsets=offsets, out=out, workspace=workspace)
    odt = F32 if out.dtype == torch.float32 else BF16
    uv = u if isinstance(u, UView) else u_view(u)
    _check(lib().lrkv_attn_decode(ctypes.byref(problem), _ptr(q), ctypes.byref(kv), _ptr(seq_lens),
                                  int(max_seq_len), ctypes.byref(uv), _ptr(b), _ptr(offsets), _ptr(out), odt,
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream)))


def lrkv_decode_kv_heads_workspace_bytes(problem, kv_head_count, max_seq_len):
    n = lib().lrkv_decode_kv_heads_workspace_bytes(ctypes.byref(problem), int(kv_head_count), int(max_seq_len))
    if n == 0:
        raise LrkvError(1, "invalid decode shape or KV-head count")
    return n


def lrkv_attn_decode_kv_heads(problem, kv_head_begin, kv_head_count, q, kv, seq_lens, max_seq_len, u, b, offsets,
                              out, workspace, stream=None):
    """lrkv_attn_decode for the query heads of KV heads [kv_head_begin, kv_head_begin + kv_head_count) only.
    kv holds those KV heads (its head 0 is kv_head_begin); q, b and out are the whole problem's tensors."""
    _require(q.is_contiguous() and b.is_contiguous() and out.is_contiguous(), "q, b and out must be contiguous")
    _on_device(q=q, seq_lens=seq_lens, b=b, offsets=offsets, out=out, workspace=workspace)
    odt = F32 if out.dtype == torch.float32 else BF16
    uv = u if isinstance(u, UView) else u_view(u)
    _check(lib().lrkv_attn_decode_kv_heads(ctypes.byref(problem), int(kv_head_begin), int(kv_head_count), _ptr(q),
                                           ctypes.byref(kv), _ptr(seq_lens), int(max_seq_len), ctypes.byref(uv),
                                           _ptr(b), _ptr(offsets), _ptr(out), odt, _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream)))


def lrkv_attn_decode_static_scratch(problem, q, kv, seq_lens, max_seq_len, u, b, offsets, out, stream=None):
    """lrkv_attn_decode without a workspace argument, for callers that may not allocate device memory.

    The library keeps one fixed scratch array per GPU (LRKV_STATIC_SCRATCH_BYTES); shapes that need more
    are rejected with LRKV_ERR_WORKSPACE_TOO_SMALL.  Calls share that array: keep them ordered on one stream.
    """
    _require(q.is_contiguous() and b.is_contiguous() and out.is_contiguous(), "q, b and out must be contiguous")
    _on_device(q=q, seq_lens=seq_lens, b=b, offsets=offsets, out=out)
    odt = F32 if out.dtype == torch.float32 else BF16
    uv = u if isinstance(u, UView) else u_view(u)
    _check(lib().lrkv_attn_decode_static_scratch(ctypes.byref(problem), _ptr(q), ctypes.byref(kv), _ptr(seq_lens),
                                                 int(max_seq_len), ctypes.byref(uv), _ptr(b), _ptr(offsets),
                                                 _ptr(out), odt, _stream(stream)))


def lrkv_prefill_workspace_bytes(problem, ctx_len, T):
    return lib().lrkv_prefill_workspace_bytes(ctypes.byref(problem), int(ctx_len), int(T))


def lrkv_attn_prefill_chunk(problem, q, kv, session, ctx_len, T, u, b, offsets, out, workspace, stream=None):
    """Causal chunk: row j of every agent sits at ctx_len + j and sees keys t <= ctx_len + j."""
    _require(q.is_contiguous() and b.is_contiguous() and out.is_contiguous(), "q, b and out must be contiguous")
    _on_device(q=q, b=b, offsets=offsets, out=out, workspace=workspace)
    odt = F32 if out.dtype == torch.float32 else BF16
    uv = u if isinstance(u, UView) else u_view(u)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().lrkv_attn_prefill_chunk(ctypes.byref(problem), _ptr(q), ctypes.byref(kv), int(session),
                                         int(ctx_len), int(T), ctypes.byref(uv), _ptr(b), _ptr(offsets),
                                         _ptr(out), odt, _ptr(workspace), nbytes, _stream(stream)))


def lrkv_workspace_reset(workspace, stream=None):
    _on_device(workspace=workspace)
    _check(lib().lrkv_workspace_reset(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream)))


def lrkv_query_device_status(workspace, clear=True, stream=None):
    """Synchronise and return (status_name, flags); does not raise on device-side flags."""
    _on_device(workspace=workspace)
    flags = ctypes.c_uint32(0)
    st = lib().lrkv_query_device_status(_ptr(workspace), 1 if clear else 0, ctypes.byref(flags), _stream(stream))
    if st not in (0, 6, 7):
        _check(st)
    return _STATUS[st], flags.value


def lrkv_query_static_scratch_status(clear=True, stream=None):
    """Flags of the most recent lrkv_attn_decode_static_scratch call on the current device: synchronise and
    return (status_name, flags); does not raise on device-side flags."""
    flags = ctypes.c_uint32(0)
    st = lib().lrkv_query_static_scratch_status(1 if clear else 0, ctypes.byref(flags), _stream(stream))
    if st not in (0, 6, 7):
        _check(st)
    return _STATUS[st], flags.value


def lrkv_debug_stall_next_launch(spin_cap):
    """Test hook: the next decode or prefill call from this thread issues no copies and its bounded waits give
    up after spin_cap attempts (the launch then reports LRKV_ERR_TIMEOUT).  0 disarms."""
    _check(lib().lrkv_debug_stall_next_launch(int(spin_cap)))


def version():
    return lib().lrkv_version()
