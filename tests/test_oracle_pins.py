"""Pins of the fp64 oracle against what the pages and the mathematics fix.

No test here calls the CUDA library.  Each pin checks the oracle against
something other than itself:

* the decomposition identity V_i = X (W0 + A_i B_i) = X W0 + (X A_i) B_i
  (LRAgent page, "What carries the argument", Eq. 3) - exact algebra;
* the reordering O = P V_base + (P Umask_i) B_i (same page, Eq. 12) -
  exact algebra, computed here in the other order;
* B_i = 0 (the FullShared case of the LRAgent page, Fig. 2) reduces to plain
  attention, checked against torch's fp64 scaled_dot_product_attention;
* rows before the aLoRA offset equal the base output (RoleKV page, "What it does");
* a 40-digit scalar brute force on L <= 8;
* shared-A equivalence (BaseLRShared = BaseShared with equal U_i, LRAgent Fig. 3b);
* closed forms (q = 0 gives the mean value row; L = 1; linearity in B);
* paging invariance;
* the append's fixed fp32 order against scalar float32 loops and torch's
  bf16 cast, and its error against fp64 within the fp32 summation bound.

A final test plants mistakes in the oracle (on the CPU) and checks that the
pins catch each one.
"""

import numpy as np
import pytest
import torch

import oracle.lrkv_oracle as O
from brute_decimal import brute_decode, brute_prefill


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.shape != b.shape or not np.all(np.isfinite(a)) or not np.all(np.isfinite(b)):
        return False
    den = max(1.0, float(np.max(np.abs(b))))
    return float(np.max(np.abs(a - b))) <= tol * den


# --------------------------------------------------------------------------
# tiny problems
# --------------------------------------------------------------------------

def _tiny_decode(seed, mode, S=2, N=2, Hq=4, Hkv=2, d=4, Lcap=8, r=2,
                 offsets=((0, 3), (5, 9)), seq_lens=(6, 3), b_scale=0.7):
    g = _rng(seed)
    q = g.standard_normal((S, N, Hq, d))
    k = g.standard_normal((S, Hkv, Lcap, d))
    v = g.standard_normal((S, Hkv, Lcap, d))
    nu = N if mode == O.BASE_SHARED else 1
    u = g.standard_normal((S, nu, Lcap, r))
    b = g.standard_normal((N, r, Hkv * d)) * b_scale
    return dict(q=q, k=k, v=v, u=u, b=b, offsets=np.array(offsets), seq_lens=np.array(seq_lens), mode=mode)


def _tiny_prefill(seed, mode, N=3, T=3, Hq=4, Hkv=2, d=4, L0=4, r=2, offsets=(0, 5, 2), b_scale=0.7):
    g = _rng(seed)
    q = g.standard_normal((N, T, Hq, d))
    k = g.standard_normal((Hkv, L0 + T, d))
    v = g.standard_normal((Hkv, L0 + T, d))
    nu = N if mode == O.BASE_SHARED else 1
    u = g.standard_normal((nu, L0 + T, r))
    b = g.standard_normal((N, r, Hkv * d)) * b_scale
    return dict(q=q, k=k, v=v, u=u, b=b, offsets=np.array(offsets), ctx_len=L0, mode=mode)


# --------------------------------------------------------------------------
# pin checks, each returning True when the oracle module passes
# --------------------------------------------------------------------------

def pin_decomposition(mod):
    """V_i from the split caches equals the unsplit projection X (W0 + A_i B_i)."""
    g = _rng(11)
    L, Dm, Hkv, d, r, a = 9, 6, 3, 4, 2, 4
    X = g.standard_normal((L, Dm))
    W0 = g.standard_normal((Dm, Hkv * d))
    A = g.standard_normal((Dm, r))
    B = g.standard_normal((r, Hkv * d))
    unsplit = (X @ (W0 + A @ B)).reshape(L, Hkv, d).transpose(1, 0, 2)
    base = (X @ W0).reshape(L, Hkv, d).transpose(1, 0, 2)
    v_i = mod.agent_value_cache(base, mod.masked_lr_cache(X @ A, a), B)
    ok = _close(v_i[:, a:], unsplit[:, a:], 1e-12)
    ok &= _close(v_i[:, :a], base[:, :a], 1e-12)       # adapter off before a_i
    v_0 = mod.agent_value_cache(base, mod.masked_lr_cache(X @ A, 0), B)
    ok &= _close(v_0, unsplit, 1e-12)
    return bool(ok)


def pin_reordering(mod):
    """Oracle (materialised V_i) equals P V_base + (P Umask_i) B_i,g computed here."""
    ok = True
    for mode in (O.BASE_SHARED, O.BASE_LR_SHARED):
        p = _tiny_decode(21 + mode, mode)
        out = mod.decode(p["q"], p["k"], p["v"], p["u"], p["b"], p["offsets"], p["seq_lens"], mode)
        S, N, Hq, d = p["q"].shape
        Hkv = p["k"].shape[1]
        G = Hq // Hkv
        for s in range(S):
            L = int(p["seq_lens"][s])
            for i in range(N):
                u = p["u"][s, i if mode == O.BASE_SHARED else 0, :L]
                t = np.arange(L)
                um = u * (t >= p["offsets"][s, i])[:, None]
                for h in range(Hq):
                    gg = h // G
                    logits = p["k"][s, gg, :L] @ p["q"][s, i, h] / np.sqrt(d)
                    w = np.exp(logits - logits.max())
                    P = w / w.sum()
                    ref = P @ p["v"][s, gg, :L] + (P @ um) @ p["b"][i][:, gg * d:(gg + 1) * d]
                    ok &= _close(out[s, i, h], ref, 1e-12)
    return bool(ok)


def _sdpa(q, k, v, mask):
    """torch fp64 scaled_dot_product_attention; q [H, M, d], k/v [H, L, d], mask [M, L] bool."""
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=torch.from_numpy(mask)).numpy()


def pin_sdpa_decode(mod):
    """B = 0: decode is plain attention with the repeat-interleaved (GQA) base cache."""
    p = _tiny_decode(31, O.BASE_SHARED)
    b0 = np.zeros_like(p["b"])
    out = mod.decode(p["q"], p["k"], p["v"], p["u"], b0, p["offsets"], p["seq_lens"], O.BASE_SHARED)
    S, N, Hq, d = p["q"].shape
    Hkv = p["k"].shape[1]
    G = Hq // Hkv
    ok = True
    for s in range(S):
        L = int(p["seq_lens"][s])
        kk = np.repeat(p["k"][s, :, :L], G, axis=0)
        vv = np.repeat(p["v"][s, :, :L], G, axis=0)
        for i in range(N):
            ref = _sdpa(p["q"][s, i][:, None, :], kk, vv, np.ones((1, L), dtype=bool))[:, 0]
            ok &= _close(out[s, i], ref, 1e-12)
    return bool(ok)


def pin_sdpa_prefill(mod):
    """B = 0: each chunk row j sees keys t <= L0 + j (bottom-right causal), via an explicit mask."""
    p = _tiny_prefill(41, O.BASE_SHARED)
    b0 = np.zeros_like(p["b"])
    out = mod.prefill_chunk(p["q"], p["k"], p["v"], p["u"], b0, p["offsets"], p["ctx_len"], O.BASE_SHARED)
    N, T, Hq, d = p["q"].shape
    Hkv = p["k"].shape[0]
    G = Hq // Hkv
    L0 = p["ctx_len"]
    mask = np.arange(L0 + T)[None, :] <= (L0 + np.arange(T))[:, None]
    kk = np.repeat(p["k"], G, axis=0)
    vv = np.repeat(p["v"], G, axis=0)
    ok = True
    for i in range(N):
        ref = _sdpa(p["q"][i].transpose(1, 0, 2), kk, vv, mask).transpose(1, 0, 2)
        ok &= _close(out[i], ref, 1e-12)
    return bool(ok)


def pin_rows_before_offset(mod):
    """Prefill rows whose whole visible range precedes a_i equal the base output, for every agent."""
    p = _tiny_prefill(51, O.BASE_SHARED, offsets=(6, 6, 7), L0=4, T=3)
    out = mod.prefill_chunk(p["q"], p["k"], p["v"], p["u"], p["b"], p["offsets"], p["ctx_len"], O.BASE_SHARED)
    base = mod.prefill_chunk(p["q"], p["k"], p["v"], p["u"], np.zeros_like(p["b"]), p["offsets"],
                             p["ctx_len"], O.BASE_SHARED)
    ok = True
    L0 = p["ctx_len"]
    for i in range(p["q"].shape[0]):
        for j in range(p["q"].shape[1]):
            if L0 + j < p["offsets"][i]:
                ok &= bool(np.array_equal(out[i, j], base[i, j]))
            else:
                ok &= not np.allclose(out[i, j], base[i, j], atol=1e-6)
    # decode: a session whose context ends before a_i is pure base attention
    pd = _tiny_decode(52, O.BASE_SHARED, offsets=((6, 0), (3, 9)), seq_lens=(6, 3))
    od = mod.decode(pd["q"], pd["k"], pd["v"], pd["u"], pd["b"], pd["offsets"], pd["seq_lens"], O.BASE_SHARED)
    bd = mod.decode(pd["q"], pd["k"], pd["v"], pd["u"], np.zeros_like(pd["b"]), pd["offsets"],
                    pd["seq_lens"], O.BASE_SHARED)
    ok &= bool(np.array_equal(od[0, 0], bd[0, 0]) and np.array_equal(od[1, 0], bd[1, 0])
               and np.array_equal(od[1, 1], bd[1, 1]))
    ok &= not np.allclose(od[0, 1], bd[0, 1], atol=1e-6)
    return bool(ok)


def pin_brute_decode(mod):
    ok = True
    for mode in (O.BASE_SHARED, O.BASE_LR_SHARED):
        p = _tiny_decode(61 + mode, mode)
        out = mod.decode(p["q"], p["k"], p["v"], p["u"], p["b"], p["offsets"], p["seq_lens"], mode)
        ref = brute_decode(p["q"].tolist(), p["k"].tolist(), p["v"].tolist(), p["u"].tolist(),
                           p["b"].tolist(), p["offsets"].tolist(), p["seq_lens"].tolist(), mode)
        ok &= _close(out, np.array(ref), 1e-13)
    return bool(ok)


def pin_brute_prefill(mod):
    ok = True
    for mode in (O.BASE_SHARED, O.BASE_LR_SHARED):
        p = _tiny_prefill(71 + mode, mode)
        out = mod.prefill_chunk(p["q"], p["k"], p["v"], p["u"], p["b"], p["offsets"], p["ctx_len"], mode)
        ref = brute_prefill(p["q"].tolist(), p["k"].tolist(), p["v"].tolist(), p["u"].tolist(),
                            p["b"].tolist(), p["offsets"].tolist(), p["ctx_len"], mode)
        ok &= _close(out, np.array(ref), 1e-13)
    return bool(ok)


def pin_shared_a(mod):
    """BaseLRShared with one U equals BaseShared with every U_i = U (same per-agent a_i)."""
    p = _tiny_decode(81, O.BASE_LR_SHARED)
    shared = mod.decode(p["q"], p["k"], p["v"], p["u"], p["b"], p["offsets"], p["seq_lens"], O.BASE_LR_SHARED)
    N = p["q"].shape[1]
    u_rep = np.repeat(p["u"], N, axis=1)
    per_agent = mod.decode(p["q"], p["k"], p["v"], u_rep, p["b"], p["offsets"], p["seq_lens"], O.BASE_SHARED)
    return bool(np.array_equal(shared, per_agent))


def pin_closed_forms(mod):
    ok = True
    p = _tiny_decode(91, O.BASE_SHARED)
    S, N, Hq, d = p["q"].shape
    Hkv = p["k"].shape[1]
    G = Hq // Hkv
    # q = 0: uniform weights, output = mean over t of V_base[t] + mean over t of Umask[t] B
    q0 = np.zeros_like(p["q"])
    out = mod.decode(q0, p["k"], p["v"], p["u"], p["b"], p["offsets"], p["seq_lens"], O.BASE_SHARED)
    for s in range(S):
        L = int(p["seq_lens"][s])
        for i in range(N):
            a = int(p["offsets"][s, i])
            usum = p["u"][s, i, a:L].sum(axis=0) if a < L else np.zeros(p["u"].shape[-1])
            for h in range(Hq):
                gg = h // G
                ref = p["v"][s, gg, :L].mean(axis=0) + (usum / L) @ p["b"][i][:, gg * d:(gg + 1) * d]
                ok &= _close(out[s, i, h], ref, 1e-12)
    # L = 1: output = V_i[0] whatever q is
    sl1 = np.ones_like(p["seq_lens"])
    offs0 = np.zeros_like(p["offsets"])
    out1 = mod.decode(p["q"], p["k"], p["v"], p["u"], p["b"], offs0, sl1, O.BASE_SHARED)
    for s in range(S):
        for i in range(N):
            for h in range(Hq):
                gg = h // G
                ref = p["v"][s, gg, 0] + p["u"][s, i, 0] @ p["b"][i][:, gg * d:(gg + 1) * d]
                ok &= _close(out1[s, i, h], ref, 1e-12)
    # linearity in B: the weights do not depend on B
    o0 = mod.decode(p["q"], p["k"], p["v"], p["u"], 0 * p["b"], p["offsets"], p["seq_lens"], O.BASE_SHARED)
    o1 = mod.decode(p["q"], p["k"], p["v"], p["u"], p["b"], p["offsets"], p["seq_lens"], O.BASE_SHARED)
    o2 = mod.decode(p["q"], p["k"], p["v"], p["u"], 2 * p["b"], p["offsets"], p["seq_lens"], O.BASE_SHARED)
    ok &= _close(o2 - o0, 2 * (o1 - o0), 1e-12)
    return bool(ok)


def pin_paged(mod):
    """A paged cache with a random page order gives the dense result exactly."""
    g = _rng(101)
    S, N, Hq, Hkv, d, r, page, n_lp = 2, 2, 4, 2, 4, 2, 4, 3
    L = page * n_lp
    q = g.standard_normal((S, N, Hq, d))
    kd = g.standard_normal((S, Hkv, L, d))
    vd = g.standard_normal((S, Hkv, L, d))
    u = g.standard_normal((S, N, L, r))
    b = g.standard_normal((N, r, Hkv * d))
    offs = np.array([[0, 5], [7, 2]])
    sl = np.array([L, L - 2])
    perm = g.permutation(S * n_lp)
    table = perm.reshape(S, n_lp)
    kp = np.empty((S * n_lp, Hkv, page, d))
    vp = np.empty_like(kp)
    for s in range(S):
        for lp in range(n_lp):
            kp[table[s, lp]] = kd[s, :, lp * page:(lp + 1) * page]
            vp[table[s, lp]] = vd[s, :, lp * page:(lp + 1) * page]
    dense = mod.decode(q, kd, vd, u, b, offs, sl, O.BASE_SHARED)
    paged = mod.decode(q, kp, vp, u, b, offs, sl, O.BASE_SHARED, page_table=table)
    return bool(np.array_equal(dense, paged))


def pin_nan_rows_selected_out(mod):
    """U rows before a_i or past seq_len and K/V rows past seq_len may hold NaN: never read."""
    p = _tiny_decode(111, O.BASE_SHARED, offsets=((2, 4), (1, 0)), seq_lens=(6, 3))
    u = p["u"].copy()
    for s in range(2):
        for i in range(2):
            u[s, i, :p["offsets"][s, i]] = np.nan
            u[s, i, p["seq_lens"][s]:] = np.nan
    k = p["k"].copy()
    v = p["v"].copy()
    k[0, :, 6:] = np.nan
    v[1, :, 3:] = np.nan
    out = mod.decode(p["q"], k, v, u, p["b"], p["offsets"], p["seq_lens"], O.BASE_SHARED)
    ref = mod.decode(p["q"], p["k"], p["v"], p["u"], p["b"], p["offsets"], p["seq_lens"], O.BASE_SHARED)
    return bool(np.all(np.isfinite(out)) and np.array_equal(out, ref))


def pin_value_projection(mod):
    """[V_base | U_1 .. U_n] = X [W0_v | A_1 .. A_n]: element by element on small
    integers (exact), and the split caches it yields rebuild the unsplit projection."""
    g = _rng(41)
    T, Dm, Hkv, d, n, r = 3, 5, 2, 3, 2, 2
    X = g.integers(-3, 4, (T, Dm)).astype(np.float64)
    W = g.integers(-3, 4, (Dm, Hkv * d + n * r)).astype(np.float64)
    v, u = mod.value_projection(X, W, Hkv, d, n, r)
    ok = v.shape == (Hkv, T, d) and u.shape == (n, T, r)
    for t in range(T):
        for gg in range(Hkv):
            for c in range(d):
                ok &= v[gg, t, c] == sum(X[t, k] * W[k, gg * d + c] for k in range(Dm))
        for i in range(n):
            for j in range(r):
                ok &= u[i, t, j] == sum(X[t, k] * W[k, Hkv * d + i * r + j] for k in range(Dm))
    # Eq. 3: V_base + U_i B_i = X (W0 + A_i B_i)
    Xf = g.standard_normal((6, 7))
    W0 = g.standard_normal((7, Hkv * d))
    A = [g.standard_normal((7, r)) for _ in range(n)]
    B = [g.standard_normal((r, Hkv * d)) for _ in range(n)]
    v, u = mod.value_projection(Xf, np.concatenate([W0] + A, axis=1), Hkv, d, n, r)
    for i in range(n):
        unsplit = (Xf @ (W0 + A[i] @ B[i])).reshape(6, Hkv, d).transpose(1, 0, 2)
        ok &= _close(mod.agent_value_cache(v, mod.masked_lr_cache(u[i], 0), B[i]), unsplit, 1e-12)
    return bool(ok)


ALL_PINS = [pin_decomposition, pin_reordering, pin_sdpa_decode, pin_sdpa_prefill,
            pin_rows_before_offset, pin_brute_decode, pin_brute_prefill, pin_shared_a,
            pin_closed_forms, pin_paged, pin_nan_rows_selected_out, pin_value_projection]


@pytest.mark.parametrize("pin", ALL_PINS, ids=[p.__name__ for p in ALL_PINS])
def test_oracle_pin(pin):
    assert pin(O)


# --------------------------------------------------------------------------
# number formats and the fixed-order append
# --------------------------------------------------------------------------

def test_rne_matches_torch_cast():
    g = _rng(121)
    vals = [g.standard_normal(20000).astype(np.float32),
            (g.standard_normal(2000) * 1e-39).astype(np.float32),           # subnormals
            np.array([0.0, -0.0, np.inf, -np.inf, 1.0, -1.0, 3.4e38, -3.4e38], dtype=np.float32)]
    # exact ties: bf16 value plus half an ulp, with even and odd kept parts
    base = g.standard_normal(4000).astype(np.float32)
    tb = (base.view(np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    vals.append(tb.view(np.float32))
    x = np.concatenate(vals)
    ours = O.f32_to_bf16_bits_rne(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    nan_bits = O.f32_to_bf16_bits_rne(np.array([np.nan], dtype=np.float32))
    assert (nan_bits[0] & 0x7F80) == 0x7F80 and (nan_bits[0] & 0x7F) != 0
    back = O.bf16_bits_to_f64(ours[:20000])
    assert np.array_equal(back, torch.from_numpy(x[:20000]).to(torch.bfloat16).to(torch.float64).numpy())


def _bf16_vals(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def test_append_matches_scalar_float32_loop():
    g = _rng(131)
    T, Dm, r, NA = 3, 37, 3, 2
    x = _bf16_vals(g.standard_normal((T, Dm)))
    a = _bf16_vals(g.standard_normal((NA, Dm, r)) / 6)
    got = O.ref_append_fp32(x, a)
    for ag in range(NA):
        for t in range(T):
            for j in range(r):
                acc = np.float32(0.0)
                for kk in range(Dm):
                    acc = np.float32(acc + np.float32(np.float32(x[t, kk]) * np.float32(a[ag, kk, j])))
                want = torch.tensor([float(acc)], dtype=torch.float32).to(torch.bfloat16)
                want = int(want.view(torch.int16).item()) & 0xFFFF
                assert int(got[ag, t, j]) == want


def test_append_within_fp32_summation_bound():
    g = _rng(141)
    T, Dm, r, NA = 16, 2048, 8, 2
    x = _bf16_vals(g.standard_normal((T, Dm)))
    a = _bf16_vals(g.standard_normal((NA, Dm, r)) / np.sqrt(Dm))
    got = O.bf16_bits_to_f64(O.ref_append_fp32(x, a))
    u32 = 2.0 ** -24
    gamma = Dm * u32 / (1 - Dm * u32)
    for ag in range(NA):
        exact = x @ a[ag]
        absdot = np.abs(x) @ np.abs(a[ag])
        bound = gamma * absdot * (1 + 2.0 ** -8) + np.abs(exact) * 2.0 ** -8 + 1e-30
        assert np.all(np.abs(got[ag] - exact) <= bound)


def test_append_sums_first_to_last():
    """Absorption makes the order visible: 2^25 - 2^25 + 1 = 1, but 1 - 2^25 + 2^25 = 0 in fp32."""
    x = np.ones((1, 3))
    a = np.array([[[2.0 ** 25], [-(2.0 ** 25)], [1.0]]])          # [N_A=1, Dm=3, r=1]
    assert int(O.ref_append_fp32(x, a)[0, 0, 0]) == 0x3F80        # bf16 1.0
    assert int(O.ref_append_fp32(x, a[:, ::-1].copy())[0, 0, 0]) == 0x0000


# --------------------------------------------------------------------------
# planted mistakes: every one must break at least one pin
# --------------------------------------------------------------------------

def _mut_exclusive_offset(u_i, a_i):
    u_i = np.asarray(u_i, dtype=np.float64)
    keep = (np.arange(u_i.shape[0]) > int(a_i))[:, None]
    return np.where(keep, u_i, 0.0)


def _mut_multiply_mask(u_i, a_i):
    u_i = np.asarray(u_i, dtype=np.float64)
    return u_i * (np.arange(u_i.shape[0]) >= int(a_i))[:, None]


def _mut_drop_lr_term(v_base, umask, b_i):
    return np.array(v_base, dtype=np.float64)


def _mut_wrong_head_slice(v_base, umask, b_i):
    Hkv, L, d = v_base.shape
    return np.stack([v_base[g] + umask @ b_i[:, (Hkv - 1 - g) * d:(Hkv - g) * d] for g in range(Hkv)])


def _mut_head_major_b(v_base, umask, b_i):
    Hkv, L, d = v_base.shape
    r = umask.shape[1]
    bb = np.asarray(b_i).reshape(Hkv, r, d)   # reads B as [Hkv][r][d]
    return np.stack([v_base[g] + umask @ bb[g] for g in range(Hkv)])


def _mut_exclude_diagonal(q_rows, k, v, visible, scale):
    return _ORIG_ATTN(q_rows, k, v, [max(1, int(n) - 1) for n in visible], scale)


def _mut_unnormalised(q_rows, k, v, visible, scale):
    R = q_rows.shape[0]
    out = np.zeros((R, v.shape[1]))
    for j in range(R):
        n = int(visible[j])
        s = (k[:n] @ q_rows[j]) * scale
        out[j] = np.exp(s - s.max()) @ v[:n]
    return out


def _mut_no_scale(d, scale):
    return 1.0


_ORIG_ATTN = O.attention_rows
_ORIG_VPROJ = O.value_projection


def _mut_u_from_front(x, w, Hkv, d, n, r):
    v, _ = _ORIG_VPROJ(x, w, Hkv, d, n, r)
    y = O.to_f64(x) @ O.to_f64(w)
    return v, y[:, :n * r].reshape(y.shape[0], n, r).transpose(1, 0, 2)


def _mut_dim_major_heads(x, w, Hkv, d, n, r):
    _, u = _ORIG_VPROJ(x, w, Hkv, d, n, r)
    y = O.to_f64(x) @ O.to_f64(w)
    return y[:, :Hkv * d].reshape(y.shape[0], d, Hkv).transpose(2, 0, 1), u

MUTANTS = [
    ("masked_lr_cache", _mut_exclusive_offset),
    ("masked_lr_cache", _mut_multiply_mask),
    ("agent_value_cache", _mut_drop_lr_term),
    ("agent_value_cache", _mut_wrong_head_slice),
    ("agent_value_cache", _mut_head_major_b),
    ("attention_rows", _mut_exclude_diagonal),
    ("attention_rows", _mut_unnormalised),
    ("_scale", _mut_no_scale),
    ("value_projection", _mut_u_from_front),
    ("value_projection", _mut_dim_major_heads),
]


@pytest.mark.parametrize("name,mutant", MUTANTS, ids=[m[1].__name__ for m in MUTANTS])
def test_planted_mistake_is_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(O, name, mutant)
    failed = []
    for pin in ALL_PINS:
        try:
            if not pin(O):
                failed.append(pin.__name__)
        except Exception:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {mutant.__name__}"
