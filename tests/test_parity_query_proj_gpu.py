"""GPU parity of the q-LoRA query path (mla_query_proj: c_Q = W_DQ h, then
q = W_UQ c_Q per head) against the float64 oracle on identical seeded inputs.

Both outputs are compared element by element (max abs <= 2e-2, relative L2 <=
1e-2), each against the oracle on the same inputs: c_Q against the oracle's
latent, q against the oracle's up-projection of the kernel's own bf16 c_Q, and
q end to end against the oracle's two maps with a bf16 latent.  Outputs start as
NaN so that an element never written fails.  Shapes cover the cluster split of
the reduction (few output rows: 2, 4 and 8 CTAs per tile), ragged row tiles and
token counts, and the V3 and ragged-serving shapes at full size.
"""
import dataclasses

import numpy as np
import pytest
import torch

import head_latent_attention_07_b200 as M
import workload as W
from mla_gpu_util import assert_close, dev_bf16, dims_of, f64_of
from oracle import mla as O

pytestmark = pytest.mark.gpu


def run_and_check(w, T, r, seed=0):
    x = W.make_query_proj_inputs(w, seed, T, r)
    nq = w.qk_nope + w.d_rope
    c_q = torch.full((T, r), float("nan"), dtype=torch.bfloat16, device="cuda")
    q = torch.full((T, w.n_heads, nq), float("nan"), dtype=torch.bfloat16, device="cuda")
    M.mla_query_proj(dims_of(w), dev_bf16(x["h"]), dev_bf16(x["w_dq"]), dev_bf16(x["w_uq"]), c_q, q)
    torch.cuda.synchronize()
    h, w_dq, w_uq = (W.bf16_to_f32(x[k]) for k in ("h", "w_dq", "w_uq"))
    c_ref, q_ref = O.query_project(h, w_dq, w_uq, w.n_heads)
    assert_close(f64_of(c_q), c_ref, "c_q")
    # the up-projection on the kernel's own latent
    _, q_on_gpu_latent = O.query_project(f64_of(c_q), np.eye(r), w_uq, w.n_heads)
    assert_close(f64_of(q), q_on_gpu_latent, "q (kernel's c_q)")
    assert_close(f64_of(q), q_ref, "q")


@pytest.mark.parametrize("H,D,r,T", [
    (2, 8192, 16, 1),      # W_DQ: one row tile, reduction split over a cluster of 8
    (4, 1000, 40, 3),      # no split; ragged row tile and a ragged 32-wide slice of W_DQ
    (8, 2048, 104, 13),    # W_DQ split over 4; ragged slices of W_UQ (K = 104)
    (4, 2048, 512, 16),    # W_DQ split over 2
    (16, 4096, 512, 40),   # W_DQ split over 8; two token blocks of 32, ragged
])
def test_shapes(H, D, r, T):
    w = dataclasses.replace(W.WORKLOADS["v2"], n_heads=H, d_model=D)
    run_and_check(w, T, r, seed=T + r)


def test_v3_full_size():
    w = W.WORKLOADS["v3"]
    run_and_check(w, w.tokens, W.Q_LORA_RANK)


def test_ragged_serving_full_size():
    w = W.WORKLOADS["ragged"]                # 128 tokens
    run_and_check(w, w.tokens, W.Q_LORA_RANK, seed=7)


def test_feeds_absorb():
    # the query path's q is mla_absorb_q's input: absorb it and compare q_lat
    w = W.WORKLOADS["v2"]
    x = W.make_query_proj_inputs(w, 11, w.tokens)
    d = dims_of(w)
    r = W.Q_LORA_RANK
    c_q = torch.empty((w.tokens, r), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((w.tokens, w.n_heads, w.qk_nope + w.d_rope), dtype=torch.bfloat16, device="cuda")
    M.mla_query_proj(d, dev_bf16(x["h"]), dev_bf16(x["w_dq"]), dev_bf16(x["w_uq"]), c_q, q)
    pos = torch.arange(w.tokens, dtype=torch.int32, device="cuda") * 37 + 5
    w_uk = W.make_decode_inputs(dataclasses.replace(w, batch=1, context=64), seed=11).bits["w_uk"]
    q_lat = torch.empty((w.tokens, w.n_heads, w.row), dtype=torch.bfloat16, device="cuda")
    M.mla_absorb_q(d, q, pos, dev_bf16(w_uk), q_lat)
    torch.cuda.synchronize()
    ref = O.absorb_queries(f64_of(q), pos.cpu().numpy(), W.bf16_to_f32(w_uk).astype(np.float64))
    assert_close(f64_of(q_lat), ref, "q_lat")
