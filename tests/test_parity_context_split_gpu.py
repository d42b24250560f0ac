"""GPU parity of the context split: mla_decode_attn_partial on each rank's window
of every sequence's pages, then mla_merge_ranks (log-sum-exp merge + W_UV).

The ranks are emulated on one GPU (one partial call per rank into its own
buffers; the merge reads them through their pointers, as it would read peer
memory).  Checks, on the same seeded inputs:
  * each rank's (o_lat, lse) against the oracle's latent attention over exactly
    that rank's keys: pages [P_b r / R, P_b (r+1) / R), clipped to the keys the
    query sees (an empty window gives o_lat = 0, lse = -inf);
  * the merged out / lse against the oracle over the whole cache and against the
    one-call mla_decode_attn;
  * one rank: the merge reproduces mla_decode_attn bit for bit.
Lengths include sequences with fewer pages than ranks and two query tokens per
sequence (causal within the step); the long-context workload runs at full size.
"""
import numpy as np
import pytest
import torch

import head_latent_attention_07_b200 as M
import workload as W
from mla_gpu_util import GpuStep, assert_close, f64_of
from oracle import mla as O

pytestmark = pytest.mark.gpu

SMALL = dict(n_heads=8, d_model=256, d_c=512, d_rope=64, qk_nope=128, v_head=128)


def run_partials(g, R):
    w = g.w
    ql = g.q_lat.view(w.batch, w.nq, w.n_heads, w.row)
    parts = []
    for r in range(R):
        o = torch.full((w.batch, w.nq, w.n_heads, w.d_c), float("nan"), dtype=torch.float32, device="cuda")
        l = torch.full((w.batch, w.nq, w.n_heads), float("nan"), dtype=torch.float32, device="cuda")
        M.mla_decode_attn_partial(g.dims, ql, g.pool, g.page_table, g.seq_lens, r, R, g.ws, o, l,
                                  dev_status=g.status)
        parts.append((o, l))
    return parts


def run_merge(g, parts):
    out = torch.full_like(g.out, float("nan"))
    lse = torch.full_like(g.lse, float("nan"))
    M.mla_merge_ranks(g.dims, [p[0] for p in parts], [p[1] for p in parts], g.w_uv, out, lse)
    torch.cuda.synchronize()
    return out, lse


def check_partials(x, g, parts, heads=None):
    """Rank r's partial against the oracle's latent attention over rank r's keys."""
    w = x.workload
    R = len(parts)
    P = w.page_size
    scale = O.softmax_scale(w.qk_nope, w.d_rope)
    q_lat = f64_of(g.q_lat)
    pool = W.bf16_to_f32(g.pool.view(torch.int16).cpu().numpy().view(np.uint16))
    hs = list(range(w.n_heads)) if heads is None else list(heads)
    for r, (o, l) in enumerate(parts):
        o = f64_of(o).reshape(w.tokens, w.n_heads, w.d_c)
        l = f64_of(l).reshape(w.tokens, w.n_heads)
        for t in range(w.tokens):
            b = t // w.nq
            n_vis = int(x.lens[b]) - w.nq + t % w.nq + 1
            n_pages = (int(x.lens[b]) + P - 1) // P
            k0 = P * (n_pages * r // R)
            k1 = min(P * (n_pages * (r + 1) // R), n_vis)
            cache = O.gather_cache(pool, x.page_table[b], n_vis).astype(np.float64)
            win = cache[k0:max(k0, k1)]
            o_ref, l_ref = O.attend_latent(q_lat[t, hs], win[:, :w.d_c], win[:, w.d_c:], scale)
            assert_close(o[t, hs], o_ref, f"rank {r} o_lat t={t}")
            assert_close(l[t, hs], l_ref, f"rank {r} lse t={t}")


def check_merged(x, g, out, lse, heads=None):
    w = x.workload
    hs = list(range(w.n_heads)) if heads is None else list(heads)
    pool = g.pool.view(torch.int16).cpu().numpy().view(np.uint16)
    ref_out, ref_lse = O.attend_paged_latents(q_lat=f64_of(g.q_lat), pool=W.bf16_to_f32(pool),
                                              page_table=x.page_table, lens=x.lens, nq=w.nq,
                                              w_uv=x.f64("w_uv"), scale=O.softmax_scale(w.qk_nope, w.d_rope),
                                              heads=hs)
    got_o = f64_of(out).reshape(w.tokens, w.n_heads, w.v_head)
    got_l = f64_of(lse).reshape(w.tokens, w.n_heads)
    assert_close(got_o[:, hs], ref_out[:, hs], "merged out")
    assert_close(got_l[:, hs], ref_lse[:, hs], "merged lse")
    # and against the one-call path
    assert_close(got_o, f64_of(g.out).reshape(got_o.shape), "merged out vs mla_decode_attn")
    assert_close(got_l, f64_of(g.lse).reshape(got_l.shape), "merged lse vs mla_decode_attn")


def test_one_rank_is_bitwise_the_one_call():
    w = W.Workload("cp1", batch=5, nq=1, context=None, ragged=(1, 1), **SMALL)
    x = W.make_decode_inputs(w, seed=31, lens=[1, 65, 300, 1000, 4097])
    g = GpuStep(x).run()
    out, lse = run_merge(g, run_partials(g, 1))
    assert torch.equal(out, g.out)
    assert torch.equal(lse, g.lse)
    assert g.device_status() == 0


@pytest.mark.parametrize("R", [2, 3, 4])
@pytest.mark.parametrize("nq,lens", [
    (1, [1, 64, 65, 130, 300, 1000, 4097]),
    (2, [2, 3, 65, 129, 5000]),
])
def test_ranks_small(R, nq, lens):
    w = W.Workload("cp", batch=len(lens), nq=nq, context=None, ragged=(1, 1), **SMALL)
    x = W.make_decode_inputs(w, seed=40 + R, lens=lens)
    g = GpuStep(x).run()
    parts = run_partials(g, R)
    torch.cuda.synchronize()
    assert g.device_status() == 0          # empty windows are not errors
    check_partials(x, g, parts)
    out, lse = run_merge(g, parts)
    check_merged(x, g, out, lse)


def test_long_context_four_ranks_full_size_sampled():
    x = W.make_decode_inputs(W.WORKLOADS["long"], seed=0)
    g = GpuStep(x).run()
    out, lse = run_merge(g, run_partials(g, 4))
    assert g.device_status() == 0
    check_merged(x, g, out, lse, heads=[0, 77, 127])


def test_context_split_decode_one_rank_nccl_group(tmp_path):
    # the package's plumbing on one GPU: a one-rank NCCL group, the gather of one
    # partial, the merge: bit for bit the one-call result
    import torch.distributed as dist
    from head_latent_attention_07_b200.context_split import context_split_decode
    dist.init_process_group("nccl", init_method=f"file://{tmp_path}/pg", rank=0, world_size=1)
    try:
        w = W.Workload("cp_nccl", batch=3, nq=2, context=None, ragged=(1, 1), **SMALL)
        x = W.make_decode_inputs(w, seed=77, lens=[65, 300, 1000])
        g = GpuStep(x).run()
        out = torch.full_like(g.out, float("nan"))
        lse = torch.full_like(g.lse, float("nan"))
        context_split_decode(g.dims, g.q_lat.view(w.batch, w.nq, w.n_heads, w.row), g.pool, g.page_table,
                             g.seq_lens, g.w_uv, g.ws, out, lse, dev_status=g.status)
        torch.cuda.synchronize()
        assert torch.equal(out, g.out)
        assert torch.equal(lse, g.lse)
        assert g.device_status() == 0
    finally:
        dist.destroy_process_group()
