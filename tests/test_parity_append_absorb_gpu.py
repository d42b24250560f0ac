"""GPU parity of mla_append_absorb, the decode step's append and absorb in one
call: the appended cache rows against the float64 oracle (other slots
bit-identical), q_lat bit-identical to mla_absorb_q's, and the decode on top of
them against the oracle.  Covers the one-launch path (<= 16 tokens: the V3 shape,
a shape with fewer heads than the CTAs the append needs, a single token) and
the two-launch path (more than 16 tokens)."""
import numpy as np
import pytest
import torch

import head_latent_attention_07_b200 as M
import workload as W
from oracle import mla as O
from mla_gpu_util import GpuStep, assert_close, bits_of, f64_of, oracle_inputs

pytestmark = pytest.mark.gpu

SMALL = dict(d_model=256, d_c=512, d_rope=64, qk_nope=128, v_head=128)


def fused_step(x):
    """A GpuStep whose append and absorb ran through mla_append_absorb."""
    assert np.array_equal(x.h_pos, x.pos) and np.array_equal(x.h_seq_idx, x.seq_idx)
    g = GpuStep(x)
    M.mla_append_absorb(g.dims, g.h, g.w_dkv, g.h_seq_idx, g.h_pos, g.page_table, g.pool, g.q, g.w_uk, g.q_lat,
                        dev_status=g.status)
    return g


def check(x, heads=None, queries=None):
    w = x.workload
    g = fused_step(x)
    g.decode()
    torch.cuda.synchronize()
    assert g.device_status() == 0
    # q_lat: the same arithmetic as mla_absorb_q, bit for bit
    ref_g = GpuStep(x)
    ref_g.absorb()
    torch.cuda.synchronize()
    assert torch.equal(g.q_lat.view(torch.int16), ref_g.q_lat.view(torch.int16)), "q_lat differs from mla_absorb_q"
    # appended rows against the oracle; every other slot unchanged
    rows_ref = O.kv_rows(x.f64("h"), x.f64("w_dkv"), x.h_pos, w.d_c)
    P = w.page_size
    got = bits_of(g.pool)
    before = x.bits["pool"]
    pages = x.page_table[x.h_seq_idx, x.h_pos // P]
    slots = x.h_pos % P
    assert_close(W.bf16_to_f32(got[pages, slots]).astype(np.float64), rows_ref, "appended rows")
    mask = np.ones(before.shape[:2], dtype=bool)
    mask[pages, slots] = False
    assert np.array_equal(got[mask], before[mask]), "a slot outside this step's rows changed"
    # the decode on top of them
    args = oracle_inputs(x)
    ref = O.decode_step(**args, form="absorbed", heads=heads, queries=queries)
    T, H = w.tokens, w.n_heads
    hs = list(range(H)) if heads is None else list(heads)
    qs = list(range(T)) if queries is None else list(queries)
    sel = np.ix_(qs, hs)
    assert_close(f64_of(g.out).reshape(T, H, w.v_head)[sel], ref["out"][sel], "out")
    assert_close(f64_of(g.lse).reshape(T, H)[sel], ref["lse"][sel], "lse")


def test_v3_shape_one_launch():
    w = W.Workload("v3_short", batch=16, nq=1, n_heads=128, d_model=7168, d_c=512, d_rope=64, qk_nope=128,
                   v_head=128, context=1000)
    x = W.make_decode_inputs(w, seed=21, spare_pages=2)
    check(x, heads=[0, 31, 32, 63, 64, 95, 96, 127])


@pytest.mark.parametrize("batch,heads", [(1, 8), (5, 8), (16, 4), (16, 128)])
def test_small_shapes_one_launch(batch, heads):
    # fewer heads than the CTAs the append needs (288 RoPE pairs, 4 per CTA), and a single token
    lens = [64 * (b % 3) + 1 + 17 * b for b in range(batch)]
    w = W.Workload("fused_small", batch=batch, nq=1, n_heads=heads, context=None, ragged=(1, 1), **SMALL)
    x = W.make_decode_inputs(w, seed=22 + batch, spare_pages=2, lens=lens)
    check(x)


def test_more_than_16_tokens_two_launches():
    lens = [3 + 41 * b for b in range(20)]
    w = W.Workload("fused_many", batch=20, nq=1, n_heads=8, context=None, ragged=(1, 1), **SMALL)
    x = W.make_decode_inputs(w, seed=23, spare_pages=2, lens=lens)
    check(x)
