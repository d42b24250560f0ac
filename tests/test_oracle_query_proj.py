"""Pins the oracle's q-LoRA query path (query_project) and its bf16 rounding.

[eyestech-blog] sec. 3: a V3-shaped decoder with q_lora_rank = 1536, run in
bf16.  [songhuiming] "Note on Actual Implementation": the query side is
down-projected, then up-projected.  Checks: the rounding against torch's own
float32 -> bfloat16 conversion and hand-made ties; layout of c_Q and of the
per-head [q_nope || q_rope] split with selection weights; the two maps equal one
product with the folded matrix W_UQ W_DQ (associativity); the effect of the bf16
latent stays within the rounding bound.
"""
import numpy as np
import torch

from oracle import mla as O


def rnd(seed, *shape, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def test_round_bf16_hand_ties_and_exact_values():
    # bf16 spacing on [1, 2) is 2^-7: 1 + 2^-8 is a tie between 1 and 1 + 2^-7 (even: 1)
    assert O.round_bf16(1 + 2.0 ** -8) == 1.0
    # 1 + 3 * 2^-8 lies between 1 + 2^-7 (odd) and 1 + 2^-6 (even): ties go to 1 + 2^-6
    assert O.round_bf16(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6
    assert O.round_bf16(1 + 2.0 ** -8 + 2.0 ** -30) == 1 + 2.0 ** -7   # just above the tie
    assert O.round_bf16(-(1 + 2.0 ** -8 + 2.0 ** -30)) == -(1 + 2.0 ** -7)
    for v in (0.0, 1.0, -3.0, 0.5 + 2.0 ** -8, 2.0 ** 100, -(2.0 ** -100)):
        assert O.round_bf16(v) == v                      # already bf16 values
    assert np.isnan(O.round_bf16(np.nan)) and O.round_bf16(np.inf) == np.inf


def test_round_bf16_matches_torch_on_float32_inputs():
    # float32 inputs: one rounding from float32 (torch) equals one from float64 (oracle)
    x = (rnd(1, 20000) * np.exp(rnd(2, 20000) * 4)).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_bf16(x.astype(np.float64)), want)


def test_selection_weights_fix_latent_and_head_layout():
    # h holds small integers (exact in bf16); W_DQ copies channel k of h to latent k,
    # W_UQ row (head hh, j) picks latent (hh * 10 + j) % d_cq
    T, D, d_cq, H, d_h, d_r = 2, 12, 8, 3, 4, 2
    h = np.arange(T * D, dtype=np.float64).reshape(T, D) - 7.0
    w_dq = np.zeros((d_cq, D))
    for k in range(d_cq):
        w_dq[k, k + 2] = 1.0
    w_uq = np.zeros((H * (d_h + d_r), d_cq))
    for hh in range(H):
        for j in range(d_h + d_r):
            w_uq[hh * (d_h + d_r) + j, (hh * 10 + j) % d_cq] = 1.0
    c_q, q = O.query_project(h, w_dq, w_uq, H)
    np.testing.assert_array_equal(c_q, h[:, 2:2 + d_cq])
    assert q.shape == (T, H, d_h + d_r)
    for t in range(T):
        for hh in range(H):
            for j in range(d_h + d_r):
                assert q[t, hh, j] == h[t, 2 + (hh * 10 + j) % d_cq]


def test_two_maps_equal_the_folded_product():
    T, D, d_cq, H, d = 3, 40, 16, 4, 6
    h, w_dq, w_uq = rnd(3, T, D), rnd(4, d_cq, D), rnd(5, H * d, d_cq)
    _, q = O.query_project(h, w_dq, w_uq, H, latent_bf16=False)
    fold = w_uq @ w_dq                                    # [H * d, D]
    np.testing.assert_allclose(q.reshape(T, -1), h @ fold.T, rtol=1e-12, atol=1e-12)


def test_bf16_latent_error_within_rounding_bound():
    T, D, d_cq, H, d = 4, 64, 32, 2, 8
    h, w_dq, w_uq = rnd(6, T, D), rnd(7, d_cq, D, std=0.2), rnd(8, H * d, d_cq)
    c_exact, q_exact = O.query_project(h, w_dq, w_uq, H, latent_bf16=False)
    c_r, q_r = O.query_project(h, w_dq, w_uq, H)
    # each latent moves by at most half a bf16 spacing: the unit roundoff of an
    # 8-bit significand, 2^-8, times its magnitude
    assert (np.abs(c_r - c_exact) <= np.abs(c_exact) * 2.0 ** -8).all()
    bound = np.abs(c_exact) @ np.abs(w_uq).T * 2.0 ** -8
    assert (np.abs(q_r - q_exact).reshape(T, -1) <= bound + 1e-12).all()
    assert np.abs(q_r - q_exact).max() > 0                # the rounding is really applied
