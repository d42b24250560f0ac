"""Pins the oracle's layer output projection (out_project) to what the pages fix.

[distaisys] sec. 3: the heads' outputs are concatenated head after head and one
bias-free linear map (H * d_v -> d_model, weight stored [out, in]) gives the
layer output.  [from-scratch] "Absorption, and why RoPE breaks it": W_UV, applied
once after attending over the latents, folds into W_O by associativity.

The checks: identity and one-hot weights (layout of the concatenation and of the
weight), the fold of W_UV into W_O (a different order of the same products), and
plain loops on a tiny layer from the brute-force attention onwards.
"""
import numpy as np

from oracle import mla as O


def rnd(seed, *shape, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def test_identity_weight_gives_head_major_concatenation():
    T, H, d_v = 3, 4, 5
    o = rnd(1, T, H, d_v)
    y = O.out_project(o, np.eye(H * d_v))
    for t in range(T):
        for h in range(H):
            for j in range(d_v):
                assert y[t, h * d_v + j] == o[t, h, j]


def test_one_hot_rows_pick_head_and_channel():
    # non-square: 5 outputs from 3 heads x 4 channels; row d reads (h_d, j_d) twice
    T, H, d_v = 2, 3, 4
    picks = [(0, 0), (2, 3), (1, 2), (2, 0), (0, 3)]
    w_o = np.zeros((len(picks), H * d_v))
    for d, (h, j) in enumerate(picks):
        w_o[d, h * d_v + j] = 2.0
    o = rnd(2, T, H, d_v)
    y = O.out_project(o, w_o)
    assert y.shape == (T, len(picks))
    for t in range(T):
        for d, (h, j) in enumerate(picks):
            assert y[t, d] == 2.0 * o[t, h, j]


def test_value_side_fold_into_w_o():
    # y = W_O concat_h(W_UV,h o_lat,h) = W_fold concat_h(o_lat,h), with the block of
    # W_fold for head h equal to W_O[:, block h] W_UV,h
    H, d_c, d_r, d_v, D, n = 3, 16, 8, 6, 10, 9
    q_lat = rnd(3, H, d_c + d_r)
    C, KR = rnd(4, n, d_c), rnd(5, n, d_r)
    w_uv = rnd(6, H, d_v, d_c)
    w_o = rnd(7, D, H * d_v)
    scale = 0.3
    o, _ = O.attend_absorbed(q_lat, C, KR, w_uv, scale)
    o_lat, _ = O.attend_latent(q_lat, C, KR, scale)
    w_fold = np.zeros((D, H * d_c))
    for h in range(H):
        w_fold[:, h * d_c:(h + 1) * d_c] = w_o[:, h * d_v:(h + 1) * d_v] @ w_uv[h]
    y_fold = w_fold @ o_lat.reshape(-1)
    np.testing.assert_allclose(O.out_project(o[None], w_o)[0], y_fold, rtol=1e-12, atol=1e-12)


def test_tiny_layer_output_with_plain_loops():
    # brute-force attention (plain loops, no softmax trick) then the output map as
    # explicit sums, against the naive form followed by out_project
    H, d_h, d_c, d_r, d_v, D, n = 2, 3, 4, 2, 3, 5, 4
    q = rnd(8, H, d_h + d_r)
    C, KR = rnd(9, n, d_c), rnd(10, n, d_r)
    w_uk, w_uv = rnd(11, H, d_h, d_c), rnd(12, H, d_v, d_c)
    w_o = rnd(13, D, H * d_v)
    scale, pos = 0.5, n - 1
    ob, _ = O.attend_brute(q.tolist(), pos, C.tolist(), KR.tolist(), w_uk.tolist(), w_uv.tolist(), scale)
    y_loops = []
    for d in range(D):
        acc = 0.0
        for h in range(H):
            for j in range(d_v):
                acc += float(w_o[d][h * d_v + j]) * ob[h][j]
        y_loops.append(acc)
    o, _ = O.attend_naive(q, pos, C, KR, w_uk, w_uv, scale)
    np.testing.assert_allclose(O.out_project(o[None], w_o)[0], y_loops, rtol=1e-11, atol=1e-11)


def test_zero_tokens():
    y = O.out_project(np.zeros((0, 2, 3)), rnd(14, 4, 6))
    assert y.shape == (0, 4)
