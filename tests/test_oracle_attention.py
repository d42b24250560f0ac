"""Pins the float64 oracle (oracle/mla.py) to what the pages and the mathematics fix.

Every check here is independent of the oracle's own formulas: closed forms of
hand-built special cases, algebraic identities (absorbed == naive, the
associativity argument of the mla-from-scratch README), brute force with plain
loops, RoPE's defining properties, split-KV invariance and paging bijections.
"""
import math

import numpy as np
import pytest

import workload as W
from oracle import mla as O


def rnd(seed, *shape, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


# ----------------------------------------------------------------------------- RoPE

def test_rope_position_zero_is_identity():
    x = rnd(1, 5, 16)
    np.testing.assert_array_equal(O.rope(x, 0), x)


def test_rope_hand_values_interleaved_pairs():
    # pair (0,1) has frequency theta^0 = 1: at position 1 it rotates by 1 rad
    np.testing.assert_allclose(O.rope([1.0, 0.0, 0.0, 0.0], 1), [math.cos(1), math.sin(1), 0, 0], atol=1e-15)
    np.testing.assert_allclose(O.rope([0.0, 1.0, 0.0, 0.0], 1), [-math.sin(1), math.cos(1), 0, 0], atol=1e-15)
    # pair (2,3) of a width-4 RoPE has frequency 10000^(-2/4) = 1/100: position 100 -> 1 rad
    np.testing.assert_allclose(O.rope([0.0, 0.0, 1.0, 0.0], 100), [0, 0, math.cos(1), math.sin(1)], atol=1e-13)
    # width 64: pair i=16 has frequency 10000^(-32/64) = 1/100
    x = np.zeros(64)
    x[32] = 1.0
    y = O.rope(x, 50)
    assert abs(y[32] - math.cos(0.5)) < 1e-13 and abs(y[33] - math.sin(0.5)) < 1e-13
    assert np.count_nonzero(np.abs(y) > 1e-15) == 2


def test_rope_norm_and_composition():
    x = rnd(2, 7, 64)
    y = O.rope(x, 12345)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(O.rope(O.rope(x, 100), 23), O.rope(x, 123), atol=1e-11)


def test_rope_relative_position_property():
    # <RoPE(q, m), RoPE(k, n)> depends only on n - m (RoFormer; tested in mla-from-scratch)
    q, k = rnd(3, 64), rnd(4, 64)
    base = O.rope(q, 10) @ O.rope(k, 17)
    for shift in (0, 1, 1000, 65536):
        assert abs(O.rope(q, 10 + shift) @ O.rope(k, 17 + shift) - base) < 1e-9
    assert abs(O.rope(q, 10) @ O.rope(k, 18) - base) > 1e-6


# ----------------------------------------------------------------------------- append / absorb

def test_kv_rows_identity_weights():
    d_c, d_r = 8, 4
    D = d_c + d_r
    h = rnd(5, 3, D)
    rows = O.kv_rows(h, np.eye(D), np.array([0, 0, 0]), d_c)
    np.testing.assert_allclose(rows, h, atol=0)          # position 0: k^R = W_KR h
    rows = O.kv_rows(h, np.eye(D), np.array([1, 2, 3]), d_c)
    np.testing.assert_allclose(rows[:, :d_c], h[:, :d_c], atol=0)
    for t, p in enumerate([1, 2, 3]):
        a, b = h[t, d_c], h[t, d_c + 1]               # pair 0 rotates by p rad
        assert abs(rows[t, d_c] - (a * math.cos(p) - b * math.sin(p))) < 1e-14
        assert abs(rows[t, d_c + 1] - (a * math.sin(p) + b * math.cos(p))) < 1e-14


def test_kv_rows_latent_is_down_projection():
    # c = W_DKV h with W_DKV the first d_c rows: a unit hidden state picks a column
    d_c, d_r, D = 6, 2, 10
    w = rnd(6, d_c + d_r, D)
    h = np.zeros((1, D))
    h[0, 3] = 1.0
    rows = O.kv_rows(h, w, np.array([0]), d_c)
    np.testing.assert_allclose(rows[0], w[:, 3], atol=0)


def test_absorb_transposes_w_uk():
    # W_UK,h = [I | 0] (d_h x d_c): q~ = W_UK,h^T q_nope = [q_nope, 0]
    H, d_h, d_c, d_r = 2, 4, 10, 4
    w_uk = np.zeros((H, d_h, d_c))
    w_uk[:, :, :d_h] = np.eye(d_h)
    q = rnd(7, 3, H, d_h + d_r)
    ql = O.absorb_queries(q, np.array([0, 5, 9]), w_uk)
    np.testing.assert_allclose(ql[..., :d_h], q[..., :d_h], atol=0)
    np.testing.assert_allclose(ql[..., d_h:d_c], 0, atol=0)
    np.testing.assert_allclose(ql[0, :, d_c:], q[0, :, d_h:], atol=0)   # position 0
    # general weights: q~ . c == q_nope . (W_UK c) for any c (associativity)
    w_uk = rnd(8, H, d_h, d_c)
    ql = O.absorb_queries(q, np.array([0, 0, 0]), w_uk)
    c = rnd(9, d_c)
    for t in range(3):
        for h in range(H):
            assert abs(ql[t, h, :d_c] @ c - q[t, h, :d_h] @ (w_uk[h] @ c)) < 1e-12


# ----------------------------------------------------------------------------- attention closed forms

def test_single_token_gives_its_value():
    H, d_h, d_r, d_c, d_v = 3, 4, 4, 8, 5
    w_uk, w_uv = rnd(10, H, d_h, d_c), rnd(11, H, d_v, d_c)
    C, KR, q = rnd(12, 1, d_c), rnd(13, 1, d_r), rnd(14, H, d_h + d_r)
    scale = O.softmax_scale(d_h, d_r)
    o, lse = O.attend_naive(q, 0, C, KR, w_uk, w_uv, scale)
    for h in range(H):
        np.testing.assert_allclose(o[h], w_uv[h] @ C[0], atol=1e-14)
        s0 = scale * (q[h, :d_h] @ (w_uk[h] @ C[0]) + q[h, d_h:] @ KR[0])
        assert abs(lse[h] - s0) < 1e-13


def test_zero_query_gives_uniform_mean():
    H, d_h, d_r, d_c, d_v, n = 2, 4, 4, 8, 3, 37
    w_uk, w_uv = rnd(15, H, d_h, d_c), rnd(16, H, d_v, d_c)
    C, KR = rnd(17, n, d_c), rnd(18, n, d_r)
    o, lse = O.attend_naive(np.zeros((H, d_h + d_r)), n - 1, C, KR, w_uk, w_uv, 0.3)
    for h in range(H):
        np.testing.assert_allclose(o[h], w_uv[h] @ C.mean(axis=0), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(n), atol=1e-14)


def test_two_token_sigmoid_pins_scale():
    # d_h = 4, d_rope = 12 -> scale = 1/sqrt(16) = 1/4.  W_UK = W_UV = I, c_0 = e_0,
    # c_1 = 0, k^R = 0, q_nope = (4 ln 3) e_0: s_0 = ln 3, s_1 = 0 -> p = (3/4, 1/4).
    d_h, d_r, d_c = 4, 12, 4
    scale = O.softmax_scale(d_h, d_r)
    assert scale == 0.25
    w = np.eye(4)[None]
    C = np.array([[1.0, 0, 0, 0], [0, 0, 0, 0]])
    KR = np.zeros((2, d_r))
    q = np.zeros((1, d_h + d_r))
    q[0, 0] = 4 * math.log(3)
    q[0, d_h:] = rnd(19, d_r)                      # irrelevant: k^R = 0
    o, lse = O.attend_naive(q, 1, C, KR, w, w, scale)
    np.testing.assert_allclose(o[0], [0.75, 0, 0, 0], atol=1e-15)
    assert abs(lse[0] - math.log(4)) < 1e-15
    oa, la = O.attend_absorbed(O.absorb_queries(q[None], np.array([1]), w)[0], C, KR, w, scale)
    np.testing.assert_allclose(oa[0], [0.75, 0, 0, 0], atol=1e-15)


def test_rope_score_closed_form_pins_positions():
    # content path off (W_UK = 0); q_rope = (1, 0) at query position 1 rotates to
    # (cos 1, sin 1); stored keys k^R_0 = (1, 0), k^R_1 = (0, 1); W_UV = I and
    # c_0 = e_0, c_1 = e_1 read out the weights.  scale = 1/sqrt(2 + 2) = 1/2.
    d_h, d_r, d_c = 2, 2, 2
    scale = O.softmax_scale(d_h, d_r)
    w_uk = np.zeros((1, d_h, d_c))
    w_uv = np.eye(2)[None]
    C = np.eye(2)
    KR = np.eye(2)
    q = np.array([[0.3, -0.7, 1.0, 0.0]])
    s0, s1 = 0.5 * math.cos(1), 0.5 * math.sin(1)
    p0 = 1.0 / (1.0 + math.exp(s1 - s0))
    o, lse = O.attend_naive(q, 1, C, KR, w_uk, w_uv, scale)
    np.testing.assert_allclose(o[0], [p0, 1 - p0], atol=1e-15)
    assert abs(lse[0] - math.log(math.exp(s0) + math.exp(s1))) < 1e-15


def test_planted_key_dominates():
    H, d_h, d_r, d_c, d_v, n = 2, 8, 4, 16, 6, 50
    w_uk, w_uv = rnd(20, H, d_h, d_c, std=0.25), rnd(21, H, d_v, d_c)
    C, KR = rnd(22, n, d_c), rnd(23, n, d_r)
    q = rnd(24, H, d_h + d_r)
    scale = O.softmax_scale(d_h, d_r)
    q_lat = O.absorb_queries(q[None], np.array([n - 1]), w_uk)[0]
    # plant key 17 along q~ of head 0: its score is >100 above every other key,
    # so the output is its value up to e^-100
    direction = q_lat[0, :d_c] / np.linalg.norm(q_lat[0, :d_c])
    C2 = C.copy()
    C2[17] = 200.0 * direction
    s = scale * (C2 @ q_lat[0, :d_c] + KR @ q_lat[0, d_c:])
    assert s[17] - np.delete(s, 17).max() > 100
    o, _ = O.attend_naive(q[:1], n - 1, C2, KR, w_uk[:1], w_uv[:1], scale)
    np.testing.assert_allclose(o[0], w_uv[0] @ C2[17], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- naive == absorbed == brute

@pytest.mark.parametrize("d_c", [32, 64, 512])
@pytest.mark.parametrize("n", [1, 7, 128])
def test_absorbed_equals_naive_fp64(d_c, n):
    # the mla-from-scratch README asserts absorbed == naive over three latent
    # widths and three lengths including 1 (3.9e-16 in double precision)
    H, d_h, d_r, d_v = 4, 32, 16, 32
    w_uk = rnd(100 + d_c, H, d_h, d_c, std=d_c ** -0.5)
    w_uv = rnd(200 + d_c, H, d_v, d_c, std=d_c ** -0.5)
    C, KR = rnd(300 + n, n, d_c), rnd(400 + n, n, d_r)
    q = rnd(500, H, d_h + d_r)
    scale = O.softmax_scale(d_h, d_r)
    o_n, l_n = O.attend_naive(q, n - 1, C, KR, w_uk, w_uv, scale)
    q_lat = O.absorb_queries(q[None], np.array([n - 1]), w_uk)[0]
    o_a, l_a = O.attend_absorbed(q_lat, C, KR, w_uv, scale)
    assert np.abs(o_n - o_a).max() <= 1e-12
    assert np.abs(l_n - l_a).max() <= 1e-12


def test_brute_force_matches_naive_on_tiny_workload():
    w = W.WORKLOADS["tiny"]
    x = W.make_decode_inputs(w, seed=0, append_all=True)
    raw = x.raw
    rows = O.kv_rows(raw["h"], raw["w_dkv"], x.h_pos, w.d_c)
    C, KR = rows[:, :w.d_c], rows[:, w.d_c:]
    q = raw["q"][0]
    p = int(x.pos[0])
    scale = O.softmax_scale(w.qk_nope, w.d_rope)
    o_n, l_n = O.attend_naive(q, p, C, KR, raw["w_uk"], raw["w_uv"], scale)
    o_b, l_b = O.attend_brute(q.tolist(), p, C.tolist(), KR.tolist(), raw["w_uk"].tolist(),
                              raw["w_uv"].tolist(), scale)
    assert np.abs(np.array(o_b) - o_n).max() <= 1e-12
    assert np.abs(np.array(l_b) - l_n).max() <= 1e-12
    q_lat = O.absorb_queries(raw["q"], x.pos, raw["w_uk"])[0]
    o_a, l_a = O.attend_absorbed(q_lat, C, KR, raw["w_uv"], scale)
    assert np.abs(o_a - o_n).max() <= 1e-12
    # the same computed in float32 agrees to the fp32 magnitudes the README reports
    o32, _ = O.attend_absorbed(q_lat.astype(np.float32).astype(np.float64),
                               C.astype(np.float32).astype(np.float64), KR.astype(np.float32).astype(np.float64),
                               raw["w_uv"], scale)
    assert np.abs(o32 - o_n).max() < 1e-5


def test_brute_force_random_small_shapes():
    for seed, (H, d_h, d_r, d_c, d_v, n) in enumerate([(1, 2, 2, 3, 2, 1), (2, 3, 4, 5, 3, 9), (3, 4, 2, 6, 4, 17)]):
        w_uk, w_uv = rnd(600 + seed, H, d_h, d_c), rnd(700 + seed, H, d_v, d_c)
        C, KR, q = rnd(800 + seed, n, d_c), rnd(900 + seed, n, d_r), rnd(1000 + seed, H, d_h + d_r)
        scale = O.softmax_scale(d_h, d_r)
        o_n, l_n = O.attend_naive(q, n + 3, C, KR, w_uk, w_uv, scale)
        o_b, l_b = O.attend_brute(q.tolist(), n + 3, C.tolist(), KR.tolist(), w_uk.tolist(), w_uv.tolist(), scale)
        assert np.abs(np.array(o_b) - o_n).max() <= 1e-12
        assert np.abs(np.array(l_b) - l_n).max() <= 1e-12


# ----------------------------------------------------------------------------- split-KV and paging

def test_split_merge_invariance():
    H, d_c, d_r, n = 4, 64, 16, 300
    q_lat = rnd(30, H, d_c + d_r, std=0.3)
    C, KR = rnd(31, n, d_c), rnd(32, n, d_r)
    whole = O.attend_latent(q_lat, C, KR, 0.2)
    for bounds in ([0, n], [0, 100, 200, n], list(range(0, n, 5)) + [n], [0, 0, 150, 150, n]):
        o, l = O.merge_partials(O.split_partials(q_lat, C, KR, 0.2, bounds))
        assert np.abs(o - whole[0]).max() <= 1e-12
        assert np.abs(l - whole[1]).max() <= 1e-12


def test_paged_gather_matches_contiguous():
    lens = np.array([130, 64, 1, 257], dtype=np.int32)
    table, num_pages = W.make_page_table(lens, 64, seed=3, shuffle=True, spare_pages=2)
    assert sorted(table[table >= 0].tolist()) != list(range(len(table[table >= 0])))  # shuffled
    R = 12
    logical = [rnd(40 + b, int(n), R) for b, n in enumerate(lens)]
    pool = np.full((num_pages, 64, R), np.nan)
    for b, n in enumerate(lens):
        O.append_rows(pool, table, np.full(n, b), np.arange(n), logical[b])
    for b, n in enumerate(lens):
        np.testing.assert_array_equal(O.gather_cache(pool, table[b], int(n)), logical[b])
    # every written slot belongs to exactly one (sequence, index); spare pages untouched
    assert np.isnan(pool).all(axis=2).sum() == num_pages * 64 - int(lens.sum())


def test_causal_within_step():
    # two query tokens: the first must not see the second's row
    w = W.Workload("t2", batch=2, nq=2, n_heads=3, d_model=48, d_c=32, d_rope=8, qk_nope=16,
                   v_head=8, context=70)
    x = W.make_decode_inputs(w, seed=5)
    args = dict(h=x.f64("h"), h_seq_idx=x.h_seq_idx, h_pos=x.h_pos, q=x.f64("q"), q_pos=x.pos,
                pool=x.f64("pool"), page_table=x.page_table, lens=x.lens, nq=2,
                w_dkv=x.f64("w_dkv"), w_uk=x.f64("w_uk"), w_uv=x.f64("w_uv"), d_c=w.d_c)
    r1 = O.decode_step(**args)
    h2 = args["h"].copy()
    h2[1] *= -3.0                     # change the appended row of token 1 (index 69 of seq 0)
    r2 = O.decode_step(**{**args, "h": h2})
    np.testing.assert_array_equal(r1["out"][0], r2["out"][0])
    assert np.abs(r1["out"][1] - r2["out"][1]).max() > 1e-6
    np.testing.assert_array_equal(r1["out"][2:], r2["out"][2:])
    # and the full step agrees between the naive and absorbed forms
    r3 = O.decode_step(**args, form="absorbed")
    assert np.abs(r3["out"] - r1["out"]).max() <= 1e-12
    assert np.abs(r3["lse"] - r1["lse"]).max() <= 1e-12


def test_decode_step_matches_paged_latent_attention():
    w = W.Workload("t3", batch=3, nq=1, n_heads=4, d_model=40, d_c=16, d_rope=8, qk_nope=8,
                   v_head=6, context=None, ragged=(1, 200))
    x = W.make_decode_inputs(w, seed=9)
    f = x.f64
    r = O.decode_step(h=f("h"), h_seq_idx=x.h_seq_idx, h_pos=x.h_pos, q=f("q"), q_pos=x.pos,
                      pool=f("pool"), page_table=x.page_table, lens=x.lens, nq=1,
                      w_dkv=f("w_dkv"), w_uk=f("w_uk"), w_uv=f("w_uv"), d_c=w.d_c)
    pool = f("pool")
    O.append_rows(pool, x.page_table, x.h_seq_idx, x.h_pos, r["rows"])   # write, then read back
    q_lat = O.absorb_queries(f("q"), x.pos, f("w_uk"))
    o, l = O.attend_paged_latents(q_lat=q_lat, pool=pool, page_table=x.page_table, lens=x.lens,
                                  nq=1, w_uv=f("w_uv"), scale=O.softmax_scale(8, 8))
    assert np.abs(o - r["out"]).max() <= 1e-12
    assert np.abs(l - r["lse"]).max() <= 1e-12
