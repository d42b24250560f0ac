"""mla_decode_attn_noalloc, the decode entry point that allocates nothing.

It exists for callers that cannot allocate device memory: code inside a host
framework that owns all device memory (a serving-engine plugin with a fixed
budget), or a decode loop that must not call cudaMalloc because it can
synchronise the device.  Instead of a caller workspace it uses a 64 MiB device
array owned by the library, shared by every call.

These tests call it through the C ABI and compare it with mla_decode_attn (the
entry point that takes a caller workspace) on the same inputs, for two calls in a
row with different batches, so that what the first call leaves in the shared
array cannot leak into the second.  This file is collected last on purpose, and
it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import head_latent_attention_07_b200 as M
import workload as W
from mla_gpu_util import GpuStep, assert_close, f64_of

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
        assert_close(f64_of(out), f64_of(g.out), "out (no-alloc vs workspace)")
        assert_close(f64_of(lse), f64_of(g.lse), "lse (no-alloc vs workspace)")


def test_noalloc_rejects_work_beyond_its_scratch():
    dims = M.MlaDims(page_size=64, n_heads=128, **SHAPE)
    # 1024 sequences x 16 query tokens x 128 heads need far more than 64 MiB of partials
    need = M.mla_decode_workspace_bytes(dims, 1024, 16)
    assert need > (64 << 20)
    g = _prepared(batch=1, nq=1, lens=[64], seed=9)
    one = lambda t: t.expand(1024, *t.shape[1:]).contiguous()
    q_lat = one(g.q_lat.view(1, 1, 128, 576)).expand(1024, 16, 128, 576).contiguous()
    page_table = g.page_table.expand(1024, -1).contiguous()
    seq_lens = torch.full((1024,), 64, dtype=torch.int32, device="cuda")
    out = torch.empty(1024, 16, 128, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MlaError) as err:
        M.mla_decode_attn_noalloc(dims, q_lat, g.pool, page_table, seq_lens, g.w_uv, out)
    assert err.value.status == M.MLA_ERR_WORKSPACE
    assert np.isfinite(f64_of(g.out)).all()
