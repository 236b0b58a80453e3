"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare with the fp64 oracle under the stated tolerance."""

import numpy as np
import torch

import lora_shared_kv_b200 as lrkv
import oracle

# Parity bar of the floating-point path against the fp64 oracle: bf16 inputs,
# fp32 accumulation, bf16 probabilities into the value contraction, bf16 output.
MAX_ABS = 1e-2
REL_L2 = 5e-3


def errors(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    diff = g - r
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(r))
    rel = float(np.linalg.norm(diff)) / den if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_parity(gpu, ref, what=""):
    g = np.asarray(gpu, dtype=np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    max_abs, rel = errors(g, ref)
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def decode_gpu(q, k, v, u, b, offsets, seq_lens, max_seq_len, mode, page_table=None, out_dtype=torch.bfloat16,
               workspace=None, check_flags=True):
    S, N, Hq, d = q.shape
    if page_table is None:
        Hkv = k.shape[1]
        kv = lrkv.kv_view_dense(k, v)
    else:
        Hkv = k.shape[1]
        kv = lrkv.kv_view_paged(k, v, page_table)
    r = u.shape[-1]
    prob = lrkv.make_problem(S, N, Hq, Hkv, d, r, mode)
    if workspace is None:
        workspace = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, max_seq_len), dtype=torch.uint8,
                                device=q.device)
    out = torch.full((S, N, Hq, d), float("nan"), dtype=out_dtype, device=q.device)
    lrkv.lrkv_attn_decode(prob, q, kv, seq_lens, max_seq_len, u, b, offsets, out, workspace)
    torch.cuda.synchronize()
    if check_flags:
        st, flags = lrkv.lrkv_query_device_status(workspace)
        assert st == "LRKV_OK", (st, hex(flags))
    return out


def decode_oracle(q, k, v, u, b, offsets, seq_lens, mode, page_table=None, sessions=None):
    return oracle.decode(q.cpu(), k.cpu(), v.cpu(), u.cpu(), b.cpu(),
                         None if offsets is None else offsets.cpu(), seq_lens.cpu(), mode,
                         page_table=None if page_table is None else page_table.cpu(), sessions=sessions)


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)
