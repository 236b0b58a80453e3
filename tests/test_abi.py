"""The C ABI without a GPU: the library loads, exports every declared symbol,
and rejects bad arguments with status codes before touching the device."""

import ctypes
import os
import re

import pytest

import lora_shared_kv_b200 as lrkv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "lrkv.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lrkv_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = lrkv.lib()
    names = _declared()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert sorted(lrkv.EXPORTS) == names


def test_status_strings_and_version():
    L = lrkv.lib()
    for s in range(8):
        assert L.lrkv_status_string(s)
    assert lrkv.version() >= 100


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _problem(**kw):
    base = dict(S=2, N=3, Hq=12, Hkv=2, d=128, r=16, mode=0)
    base.update(kw)
    return lrkv.make_problem(base["S"], base["N"], base["Hq"], base["Hkv"], base["d"], base["r"], base["mode"])


def _views(misaligned=False):
    p = FAKE + (2 if misaligned else 0)
    kv = lrkv.KVView(p, FAKE, 2 * 8192 * 128, 8192 * 128, 128, None, 0, 0, 0, 0)
    uv = lrkv.UView(FAKE, 3 * 8192 * 16, 8192 * 16, 16, 8192)
    return kv, uv


def _decode(prob, kv, uv, q=FAKE, max_len=8192, ws_bytes=1 << 20):
    L = lrkv.lib()
    return L.lrkv_attn_decode(ctypes.byref(prob), ctypes.c_void_p(q), ctypes.byref(kv), ctypes.c_void_p(FAKE),
                              max_len, ctypes.byref(uv), ctypes.c_void_p(FAKE), None, ctypes.c_void_p(FAKE), 0,
                              ctypes.c_void_p(FAKE), ws_bytes, None)


def test_decode_argument_errors():
    kv, uv = _views()
    assert _decode(_problem(d=96), kv, uv) == 2            # unsupported head_dim
    assert _decode(_problem(r=12), kv, uv) == 2            # unsupported rank
    assert _decode(_problem(Hq=10, Hkv=4), kv, uv) == 2    # Hq not a multiple of Hkv
    assert _decode(_problem(S=0), kv, uv) == 1
    assert _decode(_problem(mode=5), kv, uv) == 1
    assert _decode(_problem(N=17), kv, uv) == 2            # too many agents
    assert _decode(_problem(), kv, uv, q=0) == 1           # NULL q
    assert _decode(_problem(), kv, uv, q=FAKE + 8) == 3    # misaligned q
    kvm, _ = _views(misaligned=True)
    assert _decode(_problem(), kvm, uv) == 3               # misaligned k
    assert _decode(_problem(), kv, uv, max_len=9000) == 1  # U capacity below max_seq_len
    L = lrkv.lib()
    assert L.lrkv_attn_decode(None, None, None, None, 0, None, None, None, None, 0, None, 0, None) == 1
    assert "q" in L.lrkv_last_error_detail().decode() or L.lrkv_last_error_detail()


def test_append_argument_errors():
    L = lrkv.lib()
    uv = lrkv.UView(FAKE, 0, 100 * 16, 16, 100)
    f = lambda **k: L.lrkv_append_lr_cache(ctypes.c_void_p(FAKE), ctypes.c_void_p(FAKE), k.get("n_a", 1),
                                           k.get("T", 10), k.get("Dm", 64), k.get("r", 16), ctypes.byref(uv),
                                           0, k.get("start", 0), None)
    assert f(T=-1) == 1
    assert f(r=12) == 2
    assert f(start=95) == 1          # rows past the capacity
    assert f(n_a=0) == 1
    assert f(T=0) == 0               # empty append is a no-op, no launch
    assert L.lrkv_append_lr_cache(None, None, 1, 1, 1, 16, None, 0, 0, None) == 1


def test_append_ranges_argument_errors():
    L = lrkv.lib()
    uv = lrkv.UView(FAKE, 0, 100 * 16, 16, 100)

    def f(begin, end, x_rows=100, r=16, Dm=64):
        n = len(begin)
        b = (ctypes.c_int32 * n)(*begin)
        e = (ctypes.c_int32 * n)(*end)
        return L.lrkv_append_lr_cache_ranges(ctypes.c_void_p(FAKE), x_rows, ctypes.c_void_p(FAKE), n, Dm, r, b, e,
                                             ctypes.byref(uv), 0, None)
    assert f([5, 0], [4, 10]) == 1         # begin > end
    assert f([-1], [3]) == 1               # negative begin
    assert f([0], [101]) == 1              # past the U capacity
    assert f([0], [60], x_rows=50) == 1    # past the hidden states given
    assert f([0], [10], r=12) == 2         # unsupported rank
    assert f([3, 7], [3, 7]) == 0          # all ranges empty: a no-op, no launch
    assert L.lrkv_append_lr_cache_ranges(None, 1, None, 1, 1, 16, None, None, None, 0, None) == 1


def test_value_projection_argument_errors():
    L = lrkv.lib()
    kv, uv = _views()
    prob = _problem()

    def f(T=16, Dm=64, start=0, kv_rows=8192, x=FAKE, ws=FAKE):
        return L.lrkv_value_projection(ctypes.byref(prob), ctypes.c_void_p(x), T, Dm, ctypes.c_void_p(FAKE),
                                       ctypes.byref(kv), kv_rows, ctypes.byref(uv), 0, start, ctypes.c_void_p(ws),
                                       1 << 20, None)
    assert f(Dm=60) == 3                 # rows of x not 16-byte multiples
    assert f(x=FAKE + 2) == 3            # misaligned x
    assert f(T=-1) == 1
    assert f(start=8190) == 1            # rows past the U capacity
    assert f(kv_rows=10) == 1            # rows past the value cache
    assert f(T=0) == 0                   # nothing to project: a no-op
    assert L.lrkv_value_projection(ctypes.byref(prob), None, 1, 64, None, None, 0, None, 0, 0, None, 0, None) == 1


def test_workspace_bytes_shape_rules():
    # without a device the plan falls back to 148 SMs; invalid shapes give 0
    assert lrkv.lib().lrkv_decode_workspace_bytes(ctypes.byref(_problem(d=96)), 128) == 0
    n = lrkv.lib().lrkv_decode_workspace_bytes(ctypes.byref(_problem()), 8192)
    assert n >= 256


def _decode_ws_expected(S, N, Hq, Hkv, d, r, L, sms=148):
    # the decode plan, derived here independently: the N*G rows of a KV head
    # in as few groups of at most 32 as cover them, each padded to a multiple
    # of 8; work items (session, KV head, row group) of ceil(L/64) key tiles;
    # the flattened tiles split evenly over min(tiles, SMs) CTAs, CTA c taking
    # [c W / C, (c + 1) W / C), unless whole items fit one per SM and add at
    # most 12 tiles to a CTA's share (then one CTA per item); one partial
    # record per CTA that touches an item, when more than one does
    R = N * (Hq // Hkv)
    n_rg = -(-R // 32)
    NT = -(-(-(-R // n_rg)) // 8)
    nt = max(1, -(-L // 64))
    items = S * Hkv * n_rg
    W = items * nt
    C = min(W, sms)
    if items <= sms and nt <= -(-W // C) + 12:
        C = items
    touching = [0] * items
    for c in range(C):
        lo, hi = c * W // C, (c + 1) * W // C
        for it in range(lo // nt, (hi - 1) // nt + 1):
            touching[it] += 1
    segs = max(touching)
    partials_off = 256 + -(-(4 * items) // 256) * 256
    rec = NT * 8 * (d + r + 2) * 4
    return partials_off + (items * segs * rec if segs > 1 else 0)


@pytest.mark.parametrize("S,N,Hq,Hkv,d,r,L", [
    (32, 3, 12, 2, 128, 16, 8192),   # the Qwen2.5 decode workload: items cut by CTA boundaries
    (1, 5, 8, 1, 64, 32, 300),       # 40 rows: two row groups, fewer tiles than SMs
    (16, 2, 16, 8, 128, 16, 1024),   # 4 rows per KV head
    (200, 1, 4, 4, 128, 8, 64),      # one tile per item, more items than SMs: no partials
    (1, 16, 32, 8, 128, 32, 65536),  # 64 rows: two full row groups, many CTAs per item
])
def test_decode_workspace_follows_the_stream_k_plan(S, N, Hq, Hkv, d, r, L):
    prob = lrkv.make_problem(S, N, Hq, Hkv, d, r, lrkv.BASE_SHARED)
    assert lrkv.lib().lrkv_decode_workspace_bytes(ctypes.byref(prob), L) == _decode_ws_expected(S, N, Hq, Hkv, d, r, L)


def test_kv_head_range_decode_argument_errors_and_workspace():
    L = lrkv.lib()
    kv, uv = _views()
    prob = _problem(S=2, N=3, Hq=12, Hkv=2)

    def f(g0, ng):
        return L.lrkv_attn_decode_kv_heads(ctypes.byref(prob), g0, ng, ctypes.c_void_p(FAKE), ctypes.byref(kv),
                                           ctypes.c_void_p(FAKE), 8192, ctypes.byref(uv), ctypes.c_void_p(FAKE), None,
                                           ctypes.c_void_p(FAKE), 0, ctypes.c_void_p(FAKE), 1 << 30, None)
    for g0, ng in [(-1, 1), (0, 0), (1, 2), (2, 1), (0, 3)]:
        assert f(g0, ng) == 1, (g0, ng)
    # a shard's workspace is the plan of a launch over its heads only
    for ng in (1, 2):
        got = L.lrkv_decode_kv_heads_workspace_bytes(ctypes.byref(prob), ng, 8192)
        assert got == _decode_ws_expected(2, 3, 12 // 2 * ng, ng, 128, 16, 8192)
    assert L.lrkv_decode_kv_heads_workspace_bytes(ctypes.byref(prob), 3, 8192) == 0
    assert L.lrkv_decode_kv_heads_workspace_bytes(ctypes.byref(prob), 0, 8192) == 0


def _prefill_ws_expected(T, L0, G, Hkv, N, d, sms=148):
    # the stream-K plan, derived here independently: 128-row tiles of 128/G
    # tokens, each needing the 128-key blocks its last row sees; the blocks of
    # all tiles split evenly over min(blocks, SMs) CTAs; a tile spans at most
    # ceil(blocks / fewest-per-CTA) + 1 CTAs, each keeping 128 rows of (m, l, O)
    tm = 128 // G
    n_tb = -(-T // tm)
    nbs = [-(-(L0 + tb * tm + min(tm, T - tb * tm)) // 128) for tb in range(n_tb)]
    W = sum(nbs) * Hkv * N
    C = min(W, sms)
    parts = -(-max(nbs) // (W // C)) + 1
    tiles = Hkv * N * n_tb
    partials_off = -(-(256 + 4 * tiles) // 256) * 256
    return partials_off + tiles * parts * 128 * (d + 2) * 4


@pytest.mark.parametrize("T,L0,Hq,Hkv,N,d,r", [
    (512, 16384, 16, 8, 4, 128, 32),   # the prefill workload: 2 parts per tile at most
    (100, 300, 4, 2, 2, 128, 32),      # fewer blocks than SMs: one block per CTA
    (1, 77, 8, 4, 2, 64, 16),
    (64, 8192, 12, 2, 3, 128, 16),     # Qwen2.5-Coder role header: G = 6, tiles of 21 tokens (126 rows)
    (300, 1000, 10, 2, 2, 64, 8),      # G = 5 (25 tokens per tile), rank 8
    (9, 40, 128, 1, 1, 64, 16),        # G = 128: one token per tile
])
def test_prefill_workspace_follows_the_stream_k_plan(T, L0, Hq, Hkv, N, d, r):
    prob = lrkv.make_problem(1, N, Hq, Hkv, d, r, lrkv.BASE_SHARED)
    got = lrkv.lib().lrkv_prefill_workspace_bytes(ctypes.byref(prob), L0, T)
    assert got == _prefill_ws_expected(T, L0, Hq // Hkv, Hkv, N, d)


def _prefill(prob, kv=None, uv=None, q=FAKE, session=0, L0=1000, T=64, ws=FAKE, ws_bytes=1 << 20, out_dtype=0):
    L = lrkv.lib()
    if kv is None:
        kv, uv = _views()
    return L.lrkv_attn_prefill_chunk(ctypes.byref(prob), ctypes.c_void_p(q), ctypes.byref(kv), session, L0, T,
                                     ctypes.byref(uv), ctypes.c_void_p(FAKE), None, ctypes.c_void_p(FAKE), out_dtype,
                                     ctypes.c_void_p(ws), ws_bytes, None)


def test_prefill_argument_errors():
    kv, uv = _views()
    p = _problem(S=2)
    assert _prefill(_problem(d=96), kv, uv) == 2             # unsupported head_dim
    assert _prefill(_problem(r=12), kv, uv) == 2             # unsupported rank
    assert _prefill(_problem(Hq=10, Hkv=4), kv, uv) == 2     # Hq not a multiple of Hkv
    assert _prefill(_problem(Hq=129 * 2, Hkv=2), kv, uv) == 2  # G > 128: a tile cannot hold one token
    assert _prefill(_problem(N=17), kv, uv) == 2             # too many agents
    assert _prefill(_problem(mode=3), kv, uv) == 1
    assert _prefill(p, kv, uv, q=0) == 1                     # NULL q
    assert _prefill(p, kv, uv, ws=0) == 1                    # NULL workspace
    assert _prefill(p, kv, uv, q=FAKE + 4) == 3              # misaligned q
    assert _prefill(p, kv, uv, ws=FAKE + 8) == 3             # misaligned workspace
    assert _prefill(p, kv, uv, out_dtype=7) == 1             # unknown output dtype
    assert _prefill(p, kv, uv, session=2) == 1               # session out of range
    assert _prefill(p, kv, uv, session=-1) == 1
    assert _prefill(p, kv, uv, L0=-1) == 1
    assert _prefill(p, kv, uv, T=-5) == 1
    assert _prefill(p, kv, uv, L0=8190, T=64) == 1           # rows past the U capacity (8192)
    assert _prefill(p, kv, uv, L0=0x7fffffff, T=2) == 1      # ctx_len + T overflows
    kvm, _ = _views(misaligned=True)
    assert _prefill(p, kvm, uv) == 3                         # misaligned k
    assert _prefill(p, kv, uv, ws_bytes=100) == 4            # workspace below its status header
    assert _prefill(p, kv, uv, T=0) == 0                     # an empty chunk is a no-op, no launch
    L = lrkv.lib()
    assert L.lrkv_attn_prefill_chunk(None, None, None, 0, 0, 0, None, None, None, None, 0, None, 0, None) == 1


def test_prefill_workspace_is_zero_for_refused_shapes():
    L = lrkv.lib()
    for prob, L0, T in [(_problem(d=96), 100, 10), (_problem(r=12), 100, 10), (_problem(Hq=10, Hkv=4), 100, 10),
                        (_problem(Hq=129 * 2, Hkv=2), 100, 10), (_problem(), -1, 10), (_problem(), 100, -1),
                        (_problem(), 0x7fffffff, 2)]:
        assert L.lrkv_prefill_workspace_bytes(ctypes.byref(prob), L0, T) == 0
    for r in (8, 16, 32):  # every supported rank and G = 6 get a plan
        assert L.lrkv_prefill_workspace_bytes(ctypes.byref(_problem(r=r)), 8192, 64) > 256


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(lrkv, "_lib", None)
    monkeypatch.setattr(lrkv, "LIB_PATH", str(tmp_path / "liblrkv.so"))
    with pytest.raises(ImportError):
        lrkv.lib()
