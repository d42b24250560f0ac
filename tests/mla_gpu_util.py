"""Helpers of the GPU parity tests: move seeded inputs to the device, run the
three C-ABI calls through the binding, and compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import head_latent_attention_07_b200 as M
import workload as W

# Acceptance bounds for floating-point outputs (bf16 storage, fp32 accumulation)
MAX_ABS = 2e-2
REL_L2 = 1e-2


def dims_of(w: W.Workload, **kw) -> M.MlaDims:
    d = dict(n_heads=w.n_heads, d_c=w.d_c, d_rope=w.d_rope, qk_nope=w.qk_nope, v_head=w.v_head,
             d_model=w.d_model, page_size=w.page_size, softmax_scale=0.0, rope_theta=0.0)
    d.update(kw)
    return M.MlaDims(**d)


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16)).view(torch.bfloat16).cuda()


def dev_i32(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class GpuStep:
    """Device copies of one decode step's inputs and the outputs of the three calls."""

    def __init__(self, x: W.DecodeInputs, dims: M.MlaDims | None = None):
        w = x.workload
        self.x, self.w = x, w
        self.dims = dims if dims is not None else dims_of(w)
        self.h = dev_bf16(x.bits["h"])
        self.q = dev_bf16(x.bits["q"])
        self.w_dkv = dev_bf16(x.bits["w_dkv"])
        self.w_uk = dev_bf16(x.bits["w_uk"])
        self.w_uv = dev_bf16(x.bits["w_uv"])
        self.pool = dev_bf16(x.bits["pool"])
        self.page_table = dev_i32(x.page_table)
        self.seq_lens = dev_i32(x.lens)
        self.h_seq_idx = dev_i32(x.h_seq_idx)
        self.h_pos = dev_i32(x.h_pos)
        self.q_pos = dev_i32(x.pos)
        T = w.tokens
        self.q_lat = torch.empty((T, w.n_heads, w.row), dtype=torch.bfloat16, device="cuda")
        self.out = torch.full((w.batch, w.nq, w.n_heads, w.v_head), float("nan"), dtype=torch.bfloat16,
                              device="cuda")
        self.lse = torch.full((w.batch, w.nq, w.n_heads), float("nan"), dtype=torch.float32, device="cuda")
        self.ws = torch.empty(M.mla_decode_workspace_bytes(self.dims, w.batch, w.nq), dtype=torch.uint8,
                              device="cuda")
        self.status = torch.zeros(4, dtype=torch.int32, device="cuda")

    def append(self):
        M.mla_append_latent(self.dims, self.h, self.w_dkv, self.h_seq_idx, self.h_pos, self.page_table,
                            self.pool, dev_status=self.status)

    def absorb(self):
        M.mla_absorb_q(self.dims, self.q, self.q_pos, self.w_uk, self.q_lat)

    def decode(self, q_lat=None):
        w = self.w
        ql = (self.q_lat if q_lat is None else q_lat).view(w.batch, w.nq, w.n_heads, w.row)
        M.mla_decode_attn(self.dims, ql, self.pool, self.page_table, self.seq_lens, self.w_uv, self.ws,
                          self.out, self.lse, dev_status=self.status)

    def run(self):
        self.append()
        self.absorb()
        self.decode()
        torch.cuda.synchronize()
        return self

    def device_status(self) -> int:
        return M.mla_status_read(self.status)


def oracle_inputs(x: W.DecodeInputs) -> dict:
    """Keyword arguments of oracle.mla.decode_step on the bf16 inputs widened to float64."""
    return dict(h=x.f64("h"), h_seq_idx=x.h_seq_idx, h_pos=x.h_pos, q=x.f64("q"), q_pos=x.pos,
                pool=x.f64("pool"), page_table=x.page_table, lens=x.lens, nq=x.workload.nq,
                w_dkv=x.f64("w_dkv"), w_uk=x.f64("w_uk"), w_uv=x.f64("w_uv"), d_c=x.workload.d_c)


def assert_close(got, ref, name, max_abs=MAX_ABS, rel_l2=REL_L2):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    m = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), m), f"{name}: finite pattern differs"
    if not m.any():
        return
    d = np.abs(got[m] - ref[m])
    ma = d.max()
    rl = np.linalg.norm(got[m] - ref[m]) / max(np.linalg.norm(ref[m]), 1e-30)
    assert ma <= max_abs and rl <= rel_l2, f"{name}: max abs {ma:.3e} (<= {max_abs}), rel L2 {rl:.3e} (<= {rel_l2})"
    return ma, rl
