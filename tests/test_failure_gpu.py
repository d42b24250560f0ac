"""Failure detection without a GPU fault: the split kernel's bounded waits.

With the spin budget cut to one cycle (MLA_SPIN_LIMIT, read at each call) every
wait between the kernel's roles runs out: the call must record MLA_ERR_TIMEOUT
in the caller's status word and end cleanly (drain its copies and MMAs, free
TMEM), and the same context must then produce correct results with the normal
budget.  Nothing here traps, faults or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import head_latent_attention_07_b200 as M
import workload as W
from mla_gpu_util import GpuStep, assert_close, f64_of, oracle_inputs
from oracle import mla as O

pytestmark = pytest.mark.gpu

SMALL = dict(n_heads=8, d_model=256, d_c=512, d_rope=64, qk_nope=128, v_head=128)


def test_bounded_waits_time_out_and_the_context_stays_usable(monkeypatch):
    w = W.Workload("timeout", batch=3, nq=1, context=None, ragged=(1, 1), **SMALL)
    x = W.make_decode_inputs(w, seed=90, lens=[300, 1000, 4097])
    g = GpuStep(x)
    g.append()
    g.absorb()
    torch.cuda.synchronize()
    monkeypatch.setenv("MLA_SPIN_LIMIT", "1")
    g.decode()
    assert g.device_status() == M.MLA_ERR_TIMEOUT
    monkeypatch.delenv("MLA_SPIN_LIMIT")
    M.mla_status_clear(g.status)
    g.decode()
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ref = O.decode_step(**oracle_inputs(x), form="absorbed")
    out = f64_of(g.out).reshape(w.tokens, w.n_heads, w.v_head)
    assert_close(out, ref["out"], "out after a timed-out call")
    assert_close(f64_of(g.lse).reshape(w.tokens, w.n_heads), ref["lse"], "lse after a timed-out call")
