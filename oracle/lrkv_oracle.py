"""Plain, slow, fp64 CPU oracle for split-value-cache attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, the smoke check (``__graft_entry__.smoke``) and the bench's
CPU-baseline leg may call it.  It shares no code with the CUDA library.

What it computes, and where the pages define it:

* "LRAgent: Efficient KV Cache Sharing for Multi-LoRA LLM Agents" (Pith review),
  "What carries the argument", Eq. 3: the LoRA value projection splits exactly
  as  V_i = X W0 + (X A_i) B_i.  The base term X W0 is the shared base value
  cache; the adapter term is kept as the rank-r low-rank cache U_i = X A_i.
* Same page, Fig. 2-3: BaseShared keeps one U_i per agent; BaseLRShared shares
  one down-projection A, so one U is shared by all agents (B_i stays per agent).
* Same page, Fig. 7 note and "If this is right": keys are shared with no
  adapter term, so every agent attends with the base key cache.
* "RoleKV" (Devpost), "What it does": an aLoRA adapter switches on only after
  the role header, so rows before the activation offset a_i use base weights:
  U_i rows t < a_i contribute nothing.

The method itself (Eq. 12 of the LRAgent page) reaches the same result by
reordering, O = P V_base + (P U_i) B_i, which is exact up to rounding.  The
oracle is therefore the plain definition: it MATERIALISES
V_i = V_base + Umask_i B_i (the L x d_out cache the kernel avoids) and runs
textbook softmax attention over it, in float64.

Readings where the pages are silent (each also listed in the design notes):
* softmax scale 1/sqrt(head_dim); LoRA's alpha/r factor is folded into B_i;
* one U_i [L, r] per (session, agent, layer), used by every KV head; B_i is
  r x (Hkv * d) and KV head g uses columns [g d, (g+1) d);
* a_i is inclusive: rows t >= a_i are adapted; a_i >= L means no adapter term;
* decode attends to the cached positions [0, seq_len) of its session;
* a prefill-chunk row j sits at absolute position L0 + j and sees keys t <= L0 + j;
* query head h reads KV head g = h // (Hq / Hkv).

Every function here is pinned by the CPU tests (identities, closed forms,
library special cases, a 40-digit brute force and the fp32 error bound).
"""

import numpy as np

__all__ = [
    "to_f64",
    "bf16_bits_to_f64",
    "f32_to_bf16_bits_rne",
    "masked_lr_cache",
    "agent_value_cache",
    "attention_rows",
    "gather_paged",
    "decode",
    "prefill_chunk",
    "ref_append_fp32",
    "value_projection",
]

BASE_SHARED = 0
BASE_LR_SHARED = 1


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def to_f64(t) -> np.ndarray:
    """Exact float64 copy of a CPU tensor or array (bf16 and fp32 embed exactly)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64, exactly.

    bfloat16 is the upper half of an IEEE binary32, so the value is the float32
    whose top 16 bits are the pattern and whose low 16 bits are zero.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f32_to_bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even.

    Keeps the top 16 bits of the binary32 pattern after adding half an ulp of
    the kept part (0x7FFF plus the kept part's lowest bit, which breaks ties
    towards the even pattern).  NaN maps to the quiet NaN 0x7FC0.
    """
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    rounded = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    return np.where(np.isnan(f), np.uint16(0x7FC0), rounded).astype(np.uint16)


# --------------------------------------------------------------------------
# the split value cache
# --------------------------------------------------------------------------

def masked_lr_cache(u_i: np.ndarray, a_i: int) -> np.ndarray:
    """Umask_i: the low-rank cache with rows before the aLoRA offset removed.

    u_i [L, r].  Rows t < a_i are replaced by zero (a select, so that whatever
    those rows hold, NaN included, never reaches the result).  RoleKV page,
    "What it does": the adapter is off before the role header.
    """
    u_i = np.asarray(u_i, dtype=np.float64)
    L = u_i.shape[0]
    keep = (np.arange(L) >= int(a_i))[:, None]
    return np.where(keep, u_i, 0.0)


def agent_value_cache(v_base: np.ndarray, umask: np.ndarray, b_i: np.ndarray) -> np.ndarray:
    """Materialised value cache of one agent: V_i,g = V_base,g + Umask_i B_i[:, g d:(g+1) d].

    v_base [Hkv, L, d], umask [L, r], b_i [r, Hkv * d]  ->  [Hkv, L, d].
    This is Eq. 3 of the LRAgent page with the base cache X W0 and the
    low-rank cache X A_i already computed; it is exactly the L x d_out adapter
    cache that the kernel never forms.
    """
    Hkv, L, d = v_base.shape
    out = np.empty((Hkv, L, d), dtype=np.float64)
    for g in range(Hkv):
        b_g = b_i[:, g * d:(g + 1) * d]          # [r, d]
        out[g] = v_base[g] + umask @ b_g
    return out


def attention_rows(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, visible, scale: float) -> np.ndarray:
    """Textbook softmax attention, one query row at a time.

    q_rows [R, d]; k, v [L, d]; visible[j] = number of leading keys row j sees.
    o_j = sum_t p_t v_t with p = softmax(scale * q_j . k_t) over t < visible[j].
    A row that sees no key returns zeros.
    """
    R, d = q_rows.shape
    out = np.zeros((R, v.shape[1]), dtype=np.float64)
    for j in range(R):
        n = int(visible[j])
        if n <= 0:
            continue
        s = (k[:n] @ q_rows[j]) * scale
        e = np.exp(s - s.max())
        p = e / e.sum()
        out[j] = p @ v[:n]
    return out


def gather_paged(pages: np.ndarray, table_row, L: int) -> np.ndarray:
    """Logical [Hkv, L, d] view of one session's paged cache.

    pages [P, Hkv, page, d]; logical token t lives in physical page
    table_row[t // page] at slot t % page (the paged-cache route to physical
    sharing named on the reuse-study page, section 3.2).
    """
    P, Hkv, page, d = pages.shape
    out = np.empty((Hkv, L, d), dtype=np.float64)
    for t0 in range(0, L, page):
        n = min(page, L - t0)
        out[:, t0:t0 + n] = pages[int(table_row[t0 // page]), :, :n]
    return out


def _scale(d: int, scale):
    return (1.0 / np.sqrt(d)) if (scale is None or scale == 0) else float(scale)


# --------------------------------------------------------------------------
# decode and prefill chunk
# --------------------------------------------------------------------------

def decode(q, k, v, u, b, offsets, seq_lens, mode=BASE_SHARED, scale=None,
           page_table=None, sessions=None):
    """Decode attention of every agent's query over its session's shared cache.

    q [S, N, Hq, d]; k, v dense [S, Hkv, Lcap, d] or physical pages
    [P, Hkv, page, d] with page_table [S, n_logical_pages];
    u [S, N_U, Lcap, r] (N_U = N in BaseShared, 1 in BaseLRShared);
    b [N, r, Hkv * d]; offsets [S, N] (or None: all zero); seq_lens [S].
    Returns float64 [S, N, Hq, d]; rows of sessions not in ``sessions`` are NaN.

    For agent i and query head h of session s (g = h // G):
        V_i,g = V_base,g + Umask_i B_i[:, g d:(g+1) d]
        o = softmax(q K_base,g^T * scale) V_i,g     over t in [0, seq_len_s).
    """
    q = to_f64(q)
    b = to_f64(b)
    S, N, Hq, d = q.shape
    kk = to_f64(k)
    vv = to_f64(v)
    uu = to_f64(u)
    Hkv = kk.shape[1]
    G = Hq // Hkv
    sc = _scale(d, scale)
    offs = np.zeros((S, N), dtype=np.int64) if offsets is None else np.asarray(to_f64(offsets), dtype=np.int64)
    sl = np.asarray(to_f64(seq_lens), dtype=np.int64)
    out = np.full((S, N, Hq, d), np.nan)
    for s in (range(S) if sessions is None else sessions):
        L = int(sl[s])
        if page_table is not None:
            pt = np.asarray(to_f64(page_table), dtype=np.int64)
            k_s = gather_paged(kk, pt[s], L)
            v_s = gather_paged(vv, pt[s], L)
        else:
            k_s = kk[s, :, :L]
            v_s = vv[s, :, :L]
        for i in range(N):
            u_i = uu[s, i if mode == BASE_SHARED else 0, :L]
            umask = masked_lr_cache(u_i, offs[s, i])
            v_i = agent_value_cache(v_s, umask, b[i])
            for h in range(Hq):
                g = h // G
                out[s, i, h] = attention_rows(q[s, i, h][None, :], k_s[g], v_i[g], [L], sc)[0]
    return out


def prefill_chunk(q, k, v, u, b, offsets, ctx_len, mode=BASE_SHARED, scale=None, rows=None):
    """Causal attention of a chunk of T new rows per agent over one session.

    q [N, T, Hq, d]; k, v [Hkv, L0 + T, d] (the chunk's own base K/V already at
    rows [L0, L0 + T)); u [N_U, L0 + T, r] (chunk rows already appended);
    b [N, r, Hkv * d]; offsets [N] (or None); ctx_len = L0.
    Row j of agent i sits at absolute position L0 + j and sees keys t <= L0 + j.
    Returns float64 [N, T, Hq, d]; with ``rows`` (chunk row indices) only those
    rows are computed and the others are NaN.
    """
    q = to_f64(q)
    kk = to_f64(k)
    vv = to_f64(v)
    uu = to_f64(u)
    b = to_f64(b)
    N, T, Hq, d = q.shape
    Hkv = kk.shape[0]
    G = Hq // Hkv
    L0 = int(ctx_len)
    Ltot = L0 + T
    sc = _scale(d, scale)
    offs = np.zeros(N, dtype=np.int64) if offsets is None else np.asarray(to_f64(offsets), dtype=np.int64)
    sel = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    visible = L0 + sel + 1
    out = np.full((N, T, Hq, d), np.nan)
    for i in range(N):
        u_i = uu[i if mode == BASE_SHARED else 0, :Ltot]
        umask = masked_lr_cache(u_i, offs[i])
        v_i = agent_value_cache(vv[:, :Ltot], umask, b[i])
        for h in range(Hq):
            g = h // G
            out[i, sel, h] = attention_rows(q[i, sel, h], kk[g, :Ltot], v_i[g], visible, sc)
    return out


# --------------------------------------------------------------------------
# low-rank cache append, fixed summation order
# --------------------------------------------------------------------------

def ref_append_fp32(x, a) -> np.ndarray:
    """U rows of new tokens, U = X A_i, with a fixed fp32 summation order.

    x [T, Dm] and a [N_A, Dm, r] hold bf16 values.  For each (agent, t, j):
        acc = +0.0f;  for k = 0 .. Dm-1:  acc = fp32(acc + x[t,k] * a[k,j]);
        U[agent, t, j] = bf16_rne(acc).
    A bf16 x bf16 product has at most 16 significant bits, so it is exact in
    fp32 and each step rounds once: the result is fully determined.
    Returns uint16 bf16 bit patterns [N_A, T, r].  (Eq. 3 of the LRAgent page:
    the low-rank cache X A_i; Fig. 3: it is appended for tokens the agent has
    not processed yet.)
    """
    x32 = to_f64(x).astype(np.float32)
    a32 = to_f64(a).astype(np.float32)
    NA, Dm, r = a32.shape
    T = x32.shape[0]
    out = np.empty((NA, T, r), dtype=np.uint16)
    for ag in range(NA):
        acc = np.zeros((T, r), dtype=np.float32)
        for kk in range(Dm):
            prod = x32[:, kk:kk + 1] * a32[ag, kk:kk + 1, :]   # exact in fp32
            acc = (acc + prod).astype(np.float32)
        out[ag] = f32_to_bf16_bits_rne(acc)
    return out


# --------------------------------------------------------------------------
# the value projection with the adapters' down-projections side by side
# --------------------------------------------------------------------------

def value_projection(x, w, num_kv_heads: int, head_dim: int, n_u: int, rank: int):
    """[V_base | U_1 ... U_n] = X [W0_v | A_1 ... A_n], in float64.

    Eq. 3 of the LRAgent page splits the value projection of agent i as
    X W0 + (X A_i) B_i: the base value cache X W0 is shared and U_i = X A_i is
    the agent's rank-r cache.  Both come from the same hidden states, so one
    product with the weights side by side yields the base values and every
    agent's (or, with one shared A, the one) U rows.
    x [T, Dm]; w [Dm, Hkv * d + n_u * r], columns: W0_v (KV head g in
    [g d, (g + 1) d)), then A_1, ..., A_n (r columns each).
    Returns v [Hkv, T, d] and u [n_u, T, r].
    """
    x64 = to_f64(x)
    w64 = to_f64(w)
    T = x64.shape[0]
    hd = num_kv_heads * head_dim
    y = x64 @ w64
    v = y[:, :hd].reshape(T, num_kv_heads, head_dim).transpose(1, 0, 2)
    u = y[:, hd:hd + n_u * rank].reshape(T, n_u, rank).transpose(1, 0, 2)
    return v, u
