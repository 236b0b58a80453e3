"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every wait inside the kernels is bounded; when one gives up, the kernel records
a timeout flag, stops issuing work, lets its own copies land and returns, so
the host reads LRKV_ERR_TIMEOUT and the context stays usable.  The test hook
lrkv_debug_stall_next_launch makes the next launch's copy-issuing warps issue
nothing (a flag that nothing sets, from the waiting warps' point of view) and
caps its waits at a few attempts.  Each test checks the status, resets the
workspace, and checks that the next call on the same workspace is correct.
"""

import pytest
import torch

import lora_shared_kv_b200 as lrkv
import oracle
from gpu_util import assert_parity, decode_oracle, to_np
from workloads.gen import _normal

pytestmark = pytest.mark.gpu
DEV = "cuda"
CAP = 64  # attempts before a wait gives up in the stalled launch


def _decode_case(seed, S=3, N=3, Hq=12, Hkv=2, d=128, r=16, L=3000):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    q = _normal((S, N, Hq, d), 1.0, g, DEV)
    k = _normal((S, Hkv, L, d), 1.0, g, DEV)
    v = _normal((S, Hkv, L, d), 1.0, g, DEV)
    u = _normal((S, N, L, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), 0.05, g, DEV)
    offs = torch.tensor([[0, 1000, 2500]] * S, dtype=torch.int32, device=DEV)
    seq = torch.tensor([L, L - 5, L // 2][:S], dtype=torch.int32, device=DEV)
    return q, k, v, u, b, offs, seq


def test_decode_wait_that_runs_out_reports_timeout_and_recovers():
    q, k, v, u, b, offs, seq = _decode_case(31)
    S, N, Hq, d = q.shape
    L = k.shape[2]
    prob = lrkv.make_problem(S, N, Hq, k.shape[1], d, u.shape[-1], lrkv.BASE_SHARED)
    kv = lrkv.kv_view_dense(k, v)
    ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, L), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    lrkv.lrkv_debug_stall_next_launch(CAP)
    lrkv.lrkv_attn_decode(prob, q, kv, seq, L, u, b, offs, out, ws)
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_ERR_TIMEOUT" and flags & 0x8, (st, hex(flags))
    # the context is usable and, after a reset, the same workspace gives the right result
    lrkv.lrkv_workspace_reset(ws)
    lrkv.lrkv_attn_decode(prob, q, kv, seq, L, u, b, offs, out, ws)
    assert lrkv.lrkv_query_device_status(ws) == ("LRKV_OK", 0)
    assert_parity(to_np(out), decode_oracle(q, k, v, u, b, offs, seq, lrkv.BASE_SHARED), "after timeout")


def test_static_scratch_wait_that_runs_out_is_reported():
    q, k, v, u, b, offs, seq = _decode_case(32, L=1024)
    S, N, Hq, d = q.shape
    prob = lrkv.make_problem(S, N, Hq, k.shape[1], d, u.shape[-1], lrkv.BASE_SHARED)
    kv = lrkv.kv_view_dense(k, v)
    out = torch.empty_like(q)
    lrkv.lrkv_debug_stall_next_launch(CAP)
    lrkv.lrkv_attn_decode_static_scratch(prob, q, kv, seq, 1024, u, b, offs, out)
    st, flags = lrkv.lrkv_query_static_scratch_status()
    assert st == "LRKV_ERR_TIMEOUT" and flags & 0x8, (st, hex(flags))
    lrkv.lrkv_attn_decode_static_scratch(prob, q, kv, seq, 1024, u, b, offs, out)  # clears its own header
    assert lrkv.lrkv_query_static_scratch_status() == ("LRKV_OK", 0)
    assert_parity(to_np(out), decode_oracle(q, k, v, u, b, offs, seq, lrkv.BASE_SHARED), "after timeout")


def test_prefill_wait_that_runs_out_reports_timeout_and_recovers():
    g = torch.Generator(device=DEV)
    g.manual_seed(33)
    N, T, Hq, Hkv, d, r, L0 = 2, 200, 8, 2, 128, 32, 2000
    Ltot = L0 + T
    q = _normal((N, T, Hq, d), 1.0, g, DEV)
    k = _normal((1, Hkv, Ltot, d), 1.0, g, DEV)
    v = _normal((1, Hkv, Ltot, d), 1.0, g, DEV)
    u = _normal((1, N, Ltot, r), 1.0, g, DEV)
    b = _normal((N, r, Hkv * d), 0.05, g, DEV)
    offs = torch.tensor([0, 1500], dtype=torch.int32, device=DEV)
    prob = lrkv.make_problem(1, N, Hq, Hkv, d, r, lrkv.BASE_SHARED)
    kv = lrkv.kv_view_dense(k, v)
    ws = torch.zeros(lrkv.lrkv_prefill_workspace_bytes(prob, L0, T), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    lrkv.lrkv_debug_stall_next_launch(CAP)
    lrkv.lrkv_attn_prefill_chunk(prob, q, kv, 0, L0, T, u, b, offs, out, ws)
    st, flags = lrkv.lrkv_query_device_status(ws)
    assert st == "LRKV_ERR_TIMEOUT" and flags & 0x8, (st, hex(flags))
    lrkv.lrkv_workspace_reset(ws)
    lrkv.lrkv_attn_prefill_chunk(prob, q, kv, 0, L0, T, u, b, offs, out, ws)
    assert lrkv.lrkv_query_device_status(ws) == ("LRKV_OK", 0)
    ref = oracle.prefill_chunk(q.cpu(), k[0].cpu(), v[0].cpu(), u[0].cpu(), b.cpu(), offs.cpu(), L0, 0)
    assert_parity(to_np(out), ref, "after timeout")


def test_the_hook_arms_one_launch_only():
    q, k, v, u, b, offs, seq = _decode_case(34, L=512)
    S, N, Hq, d = q.shape
    prob = lrkv.make_problem(S, N, Hq, k.shape[1], d, u.shape[-1], lrkv.BASE_SHARED)
    kv = lrkv.kv_view_dense(k, v)
    ws = torch.zeros(lrkv.lrkv_decode_workspace_bytes(prob, 512), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(q)
    lrkv.lrkv_debug_stall_next_launch(CAP)
    lrkv.lrkv_debug_stall_next_launch(0)  # disarmed again
    lrkv.lrkv_attn_decode(prob, q, kv, seq, 512, u, b, offs, out, ws)
    assert lrkv.lrkv_query_device_status(ws) == ("LRKV_OK", 0)
