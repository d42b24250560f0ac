"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
identical seeded inputs.

Floating outputs (out, lse, q_lat, appended cache rows) must agree within max
abs <= 2e-2 and relative L2 <= 1e-2; paging is bit-exact (every slot the step
does not write keeps its bytes, canary pages included).  Sizes span several
pages and split pieces with ragged tails; the full-size workloads are checked on
sampled heads and queries, in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import workload as W
from oracle import mla as O
from mla_gpu_util import GpuStep, assert_close, bits_of, dims_of, f64_of, oracle_inputs, dev_bf16

pytestmark = pytest.mark.gpu


class Bf16Pool:
    """Read-only view of a bf16 pool that widens only the rows the oracle gathers."""

    def __init__(self, bits):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, idx):
        return W.bf16_to_f32(self.bits[idx])


def check_step(x, g, heads=None, queries=None, form="naive"):
    w = x.workload
    T, H = w.tokens, w.n_heads
    args = oracle_inputs(x)
    args["pool"] = Bf16Pool(x.bits["pool"])
    ref = O.decode_step(**args, form=form, heads=heads, queries=queries)
    out = f64_of(g.out).reshape(T, H, w.v_head)
    lse = f64_of(g.lse).reshape(T, H)
    hs = list(range(H)) if heads is None else list(heads)
    qs = list(range(T)) if queries is None else list(queries)
    sel = np.ix_(qs, hs)
    assert_close(out[sel], ref["out"][sel], "out")
    assert_close(lse[sel], ref["lse"][sel], "lse")
    # absorbed queries, all of them
    ql_ref = O.absorb_queries(x.f64("q"), x.pos, x.f64("w_uk"))
    assert_close(f64_of(g.q_lat), ql_ref, "q_lat")
    check_pool(x, g, ref["rows"])
    return ref


def check_pool(x, g, rows_ref):
    """Appended rows land in their slots (values within tolerance); every other
    slot is bit-identical to the input pool."""
    P = x.workload.page_size
    got = bits_of(g.pool)
    before = x.bits["pool"]
    pages = x.page_table[x.h_seq_idx, x.h_pos // P]
    slots = x.h_pos % P
    assert_close(W.bf16_to_f32(got[pages, slots]).astype(np.float64), rows_ref, "appended rows")
    mask = np.ones(before.shape[:2], dtype=bool)
    mask[pages, slots] = False
    assert np.array_equal(got[mask], before[mask]), "a slot outside this step's rows changed"


def test_tiny_workload_end_to_end():
    x = W.make_decode_inputs(W.WORKLOADS["tiny"], seed=0, append_all=True)
    g = GpuStep(x).run()
    assert g.device_status() == 0
    check_step(x, g)
    check_step(x, g, form="absorbed")


def test_v2_workload_end_to_end():
    x = W.make_decode_inputs(W.WORKLOADS["v2"], seed=0)
    g = GpuStep(x).run()
    assert g.device_status() == 0
    check_step(x, g)


SMALL = dict(n_heads=8, d_model=256, d_c=512, d_rope=64, qk_nope=128, v_head=128)


@pytest.mark.parametrize("nq,lens", [
    (1, [1]), (1, [63]), (1, [64]), (1, [65]), (1, [1, 64, 65, 128, 129, 300, 1000, 4097]),
    (2, [2, 3, 64, 65, 66, 127, 128, 129]), (2, [5000, 2, 7, 4096, 63]),
])
def test_ragged_lengths_and_pieces(nq, lens):
    w = W.Workload("ragged_small", batch=len(lens), nq=nq, context=None, ragged=(1, 1), **SMALL)
    x = W.make_decode_inputs(w, seed=11, spare_pages=3, lens=lens)
    g = GpuStep(x).run()
    assert g.device_status() == 0
    check_step(x, g)


@pytest.mark.parametrize("nq,lens", [
    (32, [32, 40, 300]),       # the first chunk is the whole sequence
    (64, [64, 65, 1000]),
    (128, [128, 129, 2000]),
])
def test_chunked_prefill(nq, lens):
    # a chunk of nq new tokens per sequence, appended then attending causally;
    # absorbed form for every (token, head), naive form on a few pairs
    w = W.Workload("prefill_small", batch=len(lens), nq=nq, context=None, ragged=(1, 1), **SMALL)
    x = W.make_decode_inputs(w, seed=50 + nq, lens=lens)
    g = GpuStep(x).run()
    assert g.device_status() == 0
    check_step(x, g, form="absorbed")
    args = oracle_inputs(x)
    args["pool"] = Bf16Pool(x.bits["pool"])
    out = f64_of(g.out).reshape(w.tokens, w.n_heads, w.v_head)
    for t, h in ((0, 0), (nq - 1, 7), (w.tokens - 1, 3)):
        ref = O.decode_step(**args, heads=[h], queries=[t])
        assert_close(out[t, h], ref["out"][t, h], f"out naive ({t},{h})")


def test_chunked_prefill_v3_heads_sampled():
    w = W.Workload("prefill_v3", batch=2, nq=64, n_heads=128, d_model=7168, d_c=512, d_rope=64,
                   qk_nope=128, v_head=128, context=4096)
    x = W.make_decode_inputs(w, seed=60)
    g = GpuStep(x).run()
    assert g.device_status() == 0
    check_step(x, g, heads=[0, 64, 127], queries=[0, 31, 63, 64, 100, 127], form="absorbed")


def test_output_invariant_under_physical_page_shuffle():
    # the same logical cache stored under another permutation of the physical
    # pages: every output bit and every appended row must be the same
    import dataclasses
    w = W.Workload("reshuffled", batch=3, nq=2, context=None, ragged=(1, 1), **SMALL)
    x1 = W.make_decode_inputs(w, seed=13, spare_pages=2, lens=[65, 300, 1000])
    perm = np.random.default_rng(99).permutation(x1.num_pages).astype(np.int32)
    pool2 = np.empty_like(x1.bits["pool"])
    pool2[perm] = x1.bits["pool"]
    table2 = np.where(x1.page_table >= 0, perm[np.maximum(x1.page_table, 0)], -1).astype(np.int32)
    x2 = dataclasses.replace(x1, page_table=table2, bits={**x1.bits, "pool": pool2})
    g1, g2 = GpuStep(x1).run(), GpuStep(x2).run()
    assert g1.device_status() == 0 and g2.device_status() == 0
    assert torch.equal(g1.out, g2.out)
    assert torch.equal(g1.lse, g2.lse)
    assert np.array_equal(bits_of(g2.pool)[perm], bits_of(g1.pool))


def test_decode_only_with_peaked_scores():
    # q_lat drawn directly; some keys planted along q~ so the running max jumps late
    w = W.Workload("peaked", batch=3, nq=1, context=3000, **SMALL)
    x = W.make_decode_inputs(w, seed=21)
    rng = np.random.default_rng(5)
    q_lat = rng.standard_normal((w.tokens, w.n_heads, w.row)).astype(np.float32)
    pool = W.bf16_to_f32(x.bits["pool"]).copy()
    for b in range(w.batch):
        for n in (17, 1500, 2999):                      # late keys with large scores
            pg, sl = x.page_table[b, n // 64], n % 64
            pool[pg, sl, :w.d_c] = q_lat[b * w.nq, 0, :w.d_c]
    x.bits["pool"] = W.bf16_bits(pool)
    ql_bits = W.bf16_bits(q_lat)
    g = GpuStep(x)
    ql_dev = dev_bf16(ql_bits)
    g.decode(ql_dev)
    torch.cuda.synchronize()
    assert g.device_status() == 0
    ref_o, ref_l = O.attend_paged_latents(q_lat=W.bf16_to_f32(ql_bits), pool=Bf16Pool(x.bits["pool"]),
                                          page_table=x.page_table, lens=x.lens, nq=1, w_uv=x.f64("w_uv"),
                                          scale=O.softmax_scale(w.qk_nope, w.d_rope))
    assert_close(f64_of(g.out).reshape(ref_o.shape), ref_o, "out")
    assert_close(f64_of(g.lse).reshape(ref_l.shape), ref_l, "lse")
    assert np.abs(ref_l).max() > 20        # the plants really dominate


def test_cancelling_column_halves():
    # Keys whose two latent halves give large partial scores of opposite sign for
    # one head: q~[0:256].c[0:256] ~ +600 and q~[256:512].c[256:512] ~ -600 + d (log2
    # units after the softmax scale), d 20 above every other key of that head.  Two
    # such keys per sequence with nearly equal d share the head's softmax, so the
    # output mixes their values with weights that depend on d to a small fraction
    # of a log2 unit: any path that forms the score from rounded halves (an fp16
    # half of 600 is only good to 0.25) misweights them.  The head's query is
    # scaled up (x8) so that the planted rows, and the outputs, stay of order one.
    w = W.Workload("cancel", batch=2, nq=1, context=3000, **SMALL)
    x = W.make_decode_inputs(w, seed=31)
    rng = np.random.default_rng(11)
    q_lat = rng.standard_normal((w.tokens, w.n_heads, w.row))
    planted = {0: (5, (700, 2060)), 1: (3, (1000, 2999))}
    for b, (h, _) in planted.items():
        q_lat[b, h] *= 8.0
    ql_bits = W.bf16_bits(q_lat.astype(np.float32))
    q_lat = W.bf16_to_f32(ql_bits).astype(np.float64)
    scale_log2 = O.softmax_scale(w.qk_nope, w.d_rope) / np.log(2.0)
    pool = W.bf16_to_f32(x.bits["pool"]).astype(np.float64)
    half = w.d_c // 2
    for b, (h, keys) in planted.items():
        seq_rows = pool[x.page_table[b, : (3000 + 63) // 64]].reshape(-1, w.row)[:3000]
        d = (seq_rows @ q_lat[b, h]).max() * scale_log2 + 20.0      # 20 above the head's other keys
        # a direction orthogonal to the query in each half: added with opposite signs
        # to the two keys, it leaves their scores alone and makes their values differ
        perp = rng.standard_normal(w.d_c)
        for lo_, hi_ in ((0, half), (half, w.d_c)):
            qh = q_lat[b, h, lo_:hi_]
            perp[lo_:hi_] -= (perp[lo_:hi_] @ qh) / (qh @ qh) * qh
        for sign, n, dd in zip((1.0, -1.0), keys, (d, d + 0.3)):
            qa, qb = q_lat[b, h, :half], q_lat[b, h, half:w.d_c]
            pg, sl = x.page_table[b, n // 64], n % 64
            row = pool[pg, sl].copy()
            row[:half] = qa * (600.0 / (scale_log2 * qa @ qa)) + sign * perp[:half]
            rest = row[w.d_c:] @ q_lat[b, h, w.d_c:]                 # RoPE part of this key's score
            target_b = (dd / scale_log2) - row[:half] @ qa - rest   # the second half brings the total to dd
            row[half:w.d_c] = qb * (target_b / (qb @ qb)) + sign * perp[half:w.d_c]
            pool[pg, sl] = row
    x.bits["pool"] = W.bf16_bits(pool.astype(np.float32))
    g = GpuStep(x)
    g.decode(dev_bf16(ql_bits))
    torch.cuda.synchronize()
    assert g.device_status() == 0
    pool_ref = Bf16Pool(x.bits["pool"])
    ref_o, ref_l = O.attend_paged_latents(q_lat=q_lat, pool=pool_ref, page_table=x.page_table, lens=x.lens, nq=1,
                                          w_uv=x.f64("w_uv"), scale=O.softmax_scale(w.qk_nope, w.d_rope))
    # the plants do what they are meant to: large opposite halves, totals within a
    # log2 unit of each other
    for b, (h, keys) in planted.items():
        tot = []
        for n in keys:
            r = pool_ref[x.page_table[b, n // 64], n % 64].astype(np.float64)
            hi = (r[:half] @ q_lat[b, h, :half]) * scale_log2
            lo = (r[half:w.d_c] @ q_lat[b, h, half:w.d_c]) * scale_log2
            assert hi > 500 and lo < -300
            tot.append((r @ q_lat[b, h]) * scale_log2)
        assert abs(tot[0] - tot[1]) < 1.0
    assert_close(f64_of(g.out).reshape(ref_o.shape), ref_o, "out")
    assert_close(f64_of(g.lse).reshape(ref_l.shape), ref_l, "lse")


def test_invalid_page_id_is_recorded_not_read():
    w = W.Workload("badpage", batch=2, nq=1, context=200, **SMALL)
    x = W.make_decode_inputs(w, seed=3)
    g = GpuStep(x)
    g.append()
    g.absorb()
    torch.cuda.synchronize()
    assert g.device_status() == 0
    pt = x.page_table.copy()
    pt[1, 1] = x.num_pages + 1000                     # sequence 1's second page: out of range
    g.page_table.copy_(torch.from_numpy(pt))
    g.decode()
    torch.cuda.synchronize()
    assert g.device_status() == -7                    # MLA_ERR_RANGE
    out = f64_of(g.out)
    assert np.isfinite(out).all()


def test_out_of_range_length_gives_zero_and_neg_inf():
    w = W.Workload("badlen", batch=3, nq=1, context=130, **SMALL)
    x = W.make_decode_inputs(w, seed=4)
    g = GpuStep(x)
    g.append()
    g.absorb()
    lens = x.lens.copy()
    lens[1] = x.page_table.shape[1] * 64 + 1            # longer than its page-table row
    g.seq_lens.copy_(torch.from_numpy(lens))
    g.decode()
    torch.cuda.synchronize()
    assert g.device_status() == -7
    out, lse = f64_of(g.out), f64_of(g.lse)
    assert (out[1] == 0).all() and np.isneginf(lse[1]).all()
    # the other sequences are unaffected
    args = oracle_inputs(x)
    args["pool"] = Bf16Pool(x.bits["pool"])
    ref = O.decode_step(**args, form="absorbed", queries=[0, 2])
    assert_close(out.reshape(3, -1, 128)[[0, 2]], ref["out"][[0, 2]], "out")


def test_status_clear_and_read():
    st = torch.zeros(4, dtype=torch.int32, device="cuda")
    st[0] = -7
    import head_latent_attention_07_b200 as M
    assert M.mla_status_read(st) == -7
    M.mla_status_clear(st)
    assert M.mla_status_read(st) == 0


# ------------------------------------------------------------------ full-size workloads, sampled

def _naive_heads(n_heads, seed=0, count=16):
    """16 seeded heads: 0 and the last always, the rest drawn so that every TMEM
    lane quarter (32 heads of the 128-row tile) holds at least three."""
    rng = np.random.default_rng(seed)
    picked = {0, n_heads - 1}
    for q0 in range(0, n_heads, 32):
        pool_ = [h for h in range(q0, min(q0 + 32, n_heads)) if h not in picked]
        picked.update(int(h) for h in rng.choice(pool_, size=min(3, len(pool_)), replace=False))
    rest = [h for h in range(n_heads) if h not in picked]
    picked.update(int(h) for h in rng.choice(rest, size=max(0, count - len(picked)), replace=False))
    return sorted(picked)


def _sampled(name, queries, naive_queries):
    """The full-size workload in the benchmark's launch configuration: every head
    of the sampled queries against the absorbed form, and 16 seeded heads of a
    few queries against the naive (decompressing) form."""
    x = W.make_decode_inputs(W.WORKLOADS[name], seed=0)
    g = GpuStep(x).run()
    assert g.device_status() == 0
    w = x.workload
    check_step(x, g, heads=None, queries=queries, form="absorbed")
    heads = _naive_heads(w.n_heads)
    assert len(heads) == 16 and {h // 32 for h in heads} == {0, 1, 2, 3}
    args = oracle_inputs(x)
    args["pool"] = Bf16Pool(x.bits["pool"])
    ref = O.decode_step(**args, heads=heads, queries=naive_queries)
    out = f64_of(g.out).reshape(w.tokens, w.n_heads, w.v_head)
    lse = f64_of(g.lse).reshape(w.tokens, w.n_heads)
    sel = np.ix_(naive_queries, heads)
    assert_close(out[sel], ref["out"][sel], "out (naive form, 16 heads)")
    assert_close(lse[sel], ref["lse"][sel], "lse (naive form, 16 heads)")


def test_v3_full_size_sampled():
    _sampled("v3", queries=None, naive_queries=[0, 15])


def test_long_context_full_size_sampled():
    _sampled("long", queries=None, naive_queries=[7])


def test_ragged_serving_full_size_sampled():
    _sampled("ragged", queries=[0, 1, 2, 3, 50, 51, 126, 127], naive_queries=[1, 126])
