"""40-digit scalar brute force of split-value-cache attention, for tiny inputs.

An implementation independent of the oracle: Python ``decimal`` arithmetic,
explicit scalar loops, no numpy in the arithmetic.  It writes out the plain
definition (LRAgent page, "What carries the argument", Eq. 3; RoleKV page,
"What it does" for the activation offset):

    V_i[t] = V_base[t] + [t >= a_i] * sum_k U_i[t, k] B_i[k, g d + e]
    o      = sum_t softmax_t(scale * q . K_base[t]) V_i[t]

Only for L <= 8 and tiny head sizes.
"""

from decimal import Decimal, getcontext

getcontext().prec = 40


def _D(x) -> Decimal:
    return Decimal(float(x))  # exact: every float64 is a finite binary fraction


def _softmax_weighted(logits, values):
    m = max(logits)
    w = [(lg - m).exp() for lg in logits]
    z = sum(w, Decimal(0))
    dim = len(values[0])
    return [sum((w[t] * values[t][e] for t in range(len(w))), Decimal(0)) / z for e in range(dim)]


def _scale(d, scale):
    if scale is None or scale == 0:
        return Decimal(1) / Decimal(d).sqrt()
    return _D(scale)


def brute_decode(q, k, v, u, b, offsets, seq_lens, mode, scale=None):
    """Nested lists / arrays of floats, same shapes as the oracle's decode (dense only)."""
    S, N, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k[0])
    G = Hq // Hkv
    r = len(b[0])
    sc = _scale(d, scale)
    out = [[[None] * Hq for _ in range(N)] for _ in range(S)]
    for s in range(S):
        L = int(seq_lens[s])
        for i in range(N):
            ui = 0 if mode == 1 else i
            a = int(offsets[s][i]) if offsets is not None else 0
            for h in range(Hq):
                g = h // G
                logits = []
                vals = []
                for t in range(L):
                    dot = sum((_D(q[s][i][h][e]) * _D(k[s][g][t][e]) for e in range(d)), Decimal(0))
                    logits.append(dot * sc)
                    row = []
                    for e in range(d):
                        val = _D(v[s][g][t][e])
                        if t >= a:
                            val += sum((_D(u[s][ui][t][kk]) * _D(b[i][kk][g * d + e]) for kk in range(r)),
                                       Decimal(0))
                        row.append(val)
                    vals.append(row)
                out[s][i][h] = [float(x) for x in _softmax_weighted(logits, vals)]
    return out


def brute_prefill(q, k, v, u, b, offsets, ctx_len, mode, scale=None):
    """Same shapes as the oracle's prefill_chunk; row j sees keys t <= ctx_len + j."""
    N, T, Hq, d = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    Hkv = len(k)
    G = Hq // Hkv
    r = len(b[0])
    sc = _scale(d, scale)
    out = [[[None] * Hq for _ in range(T)] for _ in range(N)]
    for i in range(N):
        ui = 0 if mode == 1 else i
        a = int(offsets[i]) if offsets is not None else 0
        for j in range(T):
            n = ctx_len + j + 1
            for h in range(Hq):
                g = h // G
                logits, vals = [], []
                for t in range(n):
                    dot = sum((_D(q[i][j][h][e]) * _D(k[g][t][e]) for e in range(d)), Decimal(0))
                    logits.append(dot * sc)
                    row = []
                    for e in range(d):
                        val = _D(v[g][t][e])
                        if t >= a:
                            val += sum((_D(u[ui][t][kk]) * _D(b[i][kk][g * d + e]) for kk in range(r)),
                                       Decimal(0))
                        row.append(val)
                    vals.append(row)
                out[i][j][h] = [float(x) for x in _softmax_weighted(logits, vals)]
    return out
