"""mla_decode_attn_noalloc, the decode entry point that allocates nothing.

It exists for callers that cannot allocate device memory: code inside a host
framework that owns all device memory (a serving-engine plugin with a fixed
budget), or a decode loop that must not call cudaMalloc because it can
synchronise the device.  Instead of a caller workspace it uses a 64 MiB device
array owned by the library, shared by every call.

These tests call it through the C ABI and compare it with mla_decode_attn (the
entry point that takes a caller workspace) on the same inputs, for two calls in a
row with different batches, so that what the first call leaves in the shared
array cannot leak into the second.  Both calls run the same kernels on the same
inputs, so the outputs must agree bit for bit.  This file is collected last on
purpose, and it also passes when run alone in a fresh process.
"""
import pytest
import torch

import head_latent_attention_07_b200 as M
import workload as W
from mla_gpu_util import GpuStep

pytestmark = pytest.mark.gpu

SHAPE = dict(d_model=512, d_c=512, d_rope=64, qk_nope=128, v_head=128)


def _prepared(batch, nq, lens, seed, n_heads=128):
    w = W.Workload(f"noalloc{seed}", batch=batch, nq=nq, n_heads=n_heads, context=None, ragged=(1, 1),
                   **SHAPE)
    g = GpuStep(W.make_decode_inputs(w, seed=seed, lens=lens))
    g.append()
    g.absorb()
    g.decode()                      # mla_decode_attn with a caller workspace: the reference
    torch.cuda.synchronize()
    assert g.device_status() == 0
    return g


def _noalloc(g):
    w = g.w
    out = torch.full_like(g.out, float("nan"))
    lse = torch.full_like(g.lse, float("nan"))
    M.mla_decode_attn_noalloc(g.dims, g.q_lat.view(w.batch, w.nq, w.n_heads, w.row), g.pool, g.page_table,
                              g.seq_lens, g.w_uv, out, lse, dev_status=g.status)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    return out, lse


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    # both fit the 64 MiB scratch: (#SMs + batch) pieces x nq*H rows x d_c floats
    first = _prepared(batch=4, nq=2, lens=[3000, 65, 2, 700], seed=7, n_heads=64)
    second = _prepared(batch=3, nq=1, lens=[129, 5000, 1], seed=8, n_heads=128)
    for g in (first, second):
        out, lse = _noalloc(g)
        assert torch.equal(out.view(torch.int16), g.out.view(torch.int16)), "out differs from the workspace call"
        assert torch.equal(lse.view(torch.int32), g.lse.view(torch.int32)), "lse differs from the workspace call"


def test_noalloc_rejects_work_beyond_its_scratch():
    dims = M.MlaDims(page_size=64, n_heads=128, **SHAPE)
    # 200 sequences of one query token at 128 heads: (#workers + 200) partials of
    # 128 rows x 512 floats exceed the 64 MiB scratch; the tensors are left
    # uninitialised, since a rejected call reads none of them
    B = 200
    need = M.mla_decode_workspace_bytes(dims, B, 1)
    assert need > (64 << 20)
    g = _prepared(batch=1, nq=1, lens=[64], seed=9)
    q_lat = torch.empty(B, 1, 128, 576, dtype=torch.bfloat16, device="cuda")
    page_table = torch.zeros(B, 1, dtype=torch.int32, device="cuda")
    seq_lens = torch.full((B,), 64, dtype=torch.int32, device="cuda")
    # sentinels: the rejected call must write neither output
    out = torch.full((B, 1, 128, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, 1, 128), -7.0, dtype=torch.float32, device="cuda")
    out_bits, lse_bits = out.view(torch.int16).clone(), lse.view(torch.int32).clone()
    with pytest.raises(M.MlaError) as err:
        M.mla_decode_attn_noalloc(dims, q_lat, g.pool, page_table, seq_lens, g.w_uv, out, lse)
    assert err.value.status == M.MLA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out_bits), "a rejected call wrote out"
    assert torch.equal(lse.view(torch.int32), lse_bits), "a rejected call wrote lse"
