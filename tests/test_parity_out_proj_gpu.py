"""GPU parity of the layer output projection (mla_out_proj, y = W_O concat_h(o_h))
against the float64 oracle on identical seeded inputs.

Every output element is compared (max abs <= 2e-2, relative L2 <= 1e-2); the
output starts as NaN so that an element the kernel never writes fails.  Shapes
cover a ragged 16-row tile, a reduction length that is not a multiple of the
32-wide slices, each token-tile width of the kernel (8, 16 and 32 tokens per CTA)
with ragged token counts, several token blocks, and the V3-shaped and
ragged-serving workloads at full size (the benchmark's launch configuration).
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


def run_and_check(w, T, seed=0):
    x = W.make_out_proj_inputs(w, seed, T)
    o, w_o = dev_bf16(x["o"]), dev_bf16(x["w_o"])
    y = torch.full((T, w.d_model), float("nan"), dtype=torch.bfloat16, device="cuda")
    M.mla_out_proj(dims_of(w), o, w_o, y)
    torch.cuda.synchronize()
    ref = O.out_project(W.bf16_to_f32(x["o"]), W.bf16_to_f32(x["w_o"]))
    assert_close(f64_of(y), ref, "y")


@pytest.mark.parametrize("H,v_head,D,T", [
    (2, 8, 8, 1),          # K = 16: one partial slice; 8 outputs in a 16-row tile
    (4, 32, 72, 3),        # ragged last row tile; 8 tokens per CTA
    (5, 24, 200, 13),      # K = 120 (ragged slice); 16 tokens per CTA, ragged
    (16, 128, 1000, 40),   # 32 tokens per CTA, two token blocks, ragged
    (128, 128, 520, 16),   # V3 reduction length (K = 16384) on few outputs
])
def test_shapes(H, v_head, D, T):
    w = dataclasses.replace(W.WORKLOADS["tiny"], n_heads=H, v_head=v_head, d_model=D)
    run_and_check(w, T, seed=H * 1000 + T)


def test_v3_full_size():
    run_and_check(W.WORKLOADS["v3"], W.WORKLOADS["v3"].tokens)


def test_ragged_serving_full_size():
    w = W.WORKLOADS["ragged"]              # 64 sequences x 2 query tokens = 128 tokens
    run_and_check(w, w.tokens, seed=5)


def test_zero_tokens_is_a_no_op():
    w = W.WORKLOADS["v2"]
    d = dims_of(w)
    o = torch.empty(0, w.n_heads, w.v_head, dtype=torch.bfloat16, device="cuda")
    w_o = torch.zeros(w.d_model, w.n_heads * w.v_head, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(0, w.d_model, dtype=torch.bfloat16, device="cuda")
    M.mla_out_proj(d, o, w_o, y)


def test_consumes_decode_output_layout():
    # mla_decode_attn writes out [B, nq, H, v_head]; the binding takes it as is
    w = W.WORKLOADS["v2"]
    x = W.make_out_proj_inputs(w, 3, w.tokens)
    o4 = dev_bf16(x["o"]).view(w.batch, w.nq, w.n_heads, w.v_head)
    y = torch.empty(w.tokens, w.d_model, dtype=torch.bfloat16, device="cuda")
    M.mla_out_proj(dims_of(w), o4, dev_bf16(x["w_o"]), y)
    torch.cuda.synchronize()
    ref = O.out_project(W.bf16_to_f32(x["o"]), W.bf16_to_f32(x["w_o"]))
    assert_close(f64_of(y), ref, "y")
    assert np.isfinite(f64_of(y)).all()
