"""The Python binding refuses, before any call into the library, arguments the
kernels would dereference wrongly: tensors in host memory (the GPU would read
a host address as its own), the wrong dtypes and non-contiguous operands.
Runs without a GPU: the library is replaced by an object that fails the test
if anything reaches it."""

import pytest
import torch

import lora_shared_kv_b200 as lrkv


class _NoLibrary:
    def __getattr__(self, name):
        raise AssertionError(f"{name} was called although the arguments were invalid")


@pytest.fixture(autouse=True)
def no_library(monkeypatch):
    monkeypatch.setattr(lrkv, "_lib", _NoLibrary())


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def _i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


S, N, Hq, Hkv, d, r, L = 2, 3, 12, 2, 128, 16, 256


def test_views_reject_host_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.kv_view_dense(_bf16(S, Hkv, L, d), _bf16(S, Hkv, L, d))
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.kv_view_paged(_bf16(8, Hkv, 64, d), _bf16(8, Hkv, 64, d), _i32(S, 4))
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.u_view(_bf16(S, N, L, r))


def test_views_reject_wrong_dtypes_and_layouts():
    with pytest.raises(ValueError, match="bf16"):
        lrkv.kv_view_dense(torch.zeros(S, Hkv, L, d), _bf16(S, Hkv, L, d))
    with pytest.raises(ValueError, match="d contiguous"):
        lrkv.kv_view_dense(_bf16(S, Hkv, d, L).transpose(2, 3), _bf16(S, Hkv, d, L).transpose(2, 3))
    with pytest.raises(ValueError, match="int32"):
        lrkv.kv_view_paged(_bf16(8, Hkv, 64, d), _bf16(8, Hkv, 64, d), torch.zeros(S, 4, dtype=torch.int64))
    with pytest.raises(ValueError, match="r contiguous"):
        lrkv.u_view(_bf16(S, N, r, L).transpose(2, 3))


def test_entry_points_reject_host_tensors():
    prob = lrkv.make_problem(S, N, Hq, Hkv, d, r)
    kv = lrkv.KVView(0x1000, 0x1000, Hkv * L * d, L * d, d, None, 0, 0, 0, 0)
    uv = lrkv.UView(0x1000, N * L * r, L * r, r, L)
    q, out, b = _bf16(S, N, Hq, d), _bf16(S, N, Hq, d), _bf16(N, r, Hkv * d)
    sl, offs, ws = _i32(S), _i32(S, N), torch.zeros(4096, dtype=torch.uint8)
    with pytest.raises(ValueError, match="q must be a CUDA tensor"):
        lrkv.lrkv_attn_decode(prob, q, kv, sl, L, uv, b, offs, out, ws)
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.lrkv_attn_decode_static_scratch(prob, q, kv, sl, L, uv, b, offs, out)
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.lrkv_attn_prefill_chunk(prob, _bf16(N, 8, Hq, d), kv, 0, L - 8, 8, uv, b, _i32(N),
                                     _bf16(N, 8, Hq, d), ws)
    with pytest.raises(ValueError, match="x must be a CUDA tensor"):
        lrkv.lrkv_append_lr_cache(_bf16(8, 64), _bf16(N, 64, r), None, 0, 0, uview=uv)
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.lrkv_append_lr_cache_ranges(_bf16(8, 64), _bf16(N, 64, r), None, 0, [0] * N, [8] * N, uview=uv)
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.lrkv_value_projection(prob, _bf16(8, 64), _bf16(64, Hkv * d + N * r), kv, L, uv, 0, 0, ws)
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.lrkv_workspace_reset(ws)
    with pytest.raises(ValueError, match="CUDA"):
        lrkv.lrkv_query_device_status(ws)


def test_entry_points_reject_non_tensors_and_bad_layouts():
    prob = lrkv.make_problem(S, N, Hq, Hkv, d, r)
    kv = lrkv.KVView(0x1000, 0x1000, Hkv * L * d, L * d, d, None, 0, 0, 0, 0)
    uv = lrkv.UView(0x1000, N * L * r, L * r, r, L)
    q = _bf16(S, N, Hq, d)
    with pytest.raises(TypeError, match="seq_lens must be a torch.Tensor"):
        lrkv._on_device(seq_lens=[L] * S)
    with pytest.raises(ValueError, match="contiguous"):
        lrkv.lrkv_attn_decode(prob, _bf16(S, N, d, Hq).transpose(2, 3), kv, _i32(S), L, uv, _bf16(N, r, Hkv * d),
                              None, q, torch.zeros(64, dtype=torch.uint8))
    with pytest.raises(ValueError, match="one row_begin and one row_end"):
        lrkv.lrkv_append_lr_cache_ranges(_bf16(8, 64), _bf16(N, 64, r), None, 0, [0], [8], uview=uv)
    with pytest.raises(ValueError, match="contiguous"):
        lrkv.lrkv_append_lr_cache(_bf16(64, 8).t(), _bf16(N, 64, r), None, 0, 0, uview=uv)
