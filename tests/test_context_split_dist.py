"""The context split's multi-rank plumbing, run as two gloo ranks on CPU.

Each rank computes the partial of its window of every sequence's pages (here with
the oracle's latent attention, on CPU), the package's gather_partials exchanges
the partials over the process group, and the log-sum-exp merge of the gathered
list must equal attention over the whole cache.  The windows (rank r of R takes
pages [P r / R, P (r+1) / R) of a sequence's P pages) must partition the pages.
"""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from oracle import mla as O  # noqa: E402

PAGE = 16
LENS = [100, 7, 300, 33]
H, D_C, D_R = 3, 32, 8


def window(n_pages, r, R):
    return n_pages * r // R, n_pages * (r + 1) // R


def test_windows_partition_the_pages():
    for P in range(0, 60):
        for R in range(1, 9):
            got = []
            for r in range(R):
                a, b = window(P, r, R)
                assert 0 <= a <= b <= P
                got.extend(range(a, b))
            assert got == list(range(P))


def _problem():
    rng = np.random.default_rng(7)
    n_pages = [(n + PAGE - 1) // PAGE for n in LENS]
    pool = rng.standard_normal((sum(n_pages), PAGE, D_C + D_R))
    table = np.full((len(LENS), max(n_pages)), -1, dtype=np.int64)
    ids = rng.permutation(sum(n_pages))
    k = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = ids[k:k + n]
        k += n
    q_lat = rng.standard_normal((len(LENS), H, D_C + D_R))
    return pool, table, q_lat


def _rank_partial(r, R):
    pool, table, q_lat = _problem()
    o = np.zeros((len(LENS), H, D_C))
    l = np.zeros((len(LENS), H))
    for b, n in enumerate(LENS):
        cache = O.gather_cache(pool, table[b], n)
        p0, p1 = window((n + PAGE - 1) // PAGE, r, R)
        win = cache[PAGE * p0:min(PAGE * p1, n)]
        o[b], l[b] = O.attend_latent(q_lat[b], win[:, :D_C], win[:, D_C:], 0.25)
    return torch.from_numpy(o), torch.from_numpy(l)


def _rank_main(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from head_latent_attention_07_b200.context_split import gather_partials
        o, l = _rank_partial(rank, world)
        o_lats, lses = gather_partials(o, l)
        queue.put((rank, [t.numpy() for t in o_lats], [t.numpy() for t in lses]))
    finally:
        dist.destroy_process_group()


def test_gather_then_merge_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, queue)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, o_lats, lses = queue.get(timeout=120)
        results[rank] = (o_lats, lses)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    pool, table, q_lat = _problem()
    for rank, (o_lats, lses) in results.items():
        # rank order: entry r is what rank r computed
        for r in range(world):
            o_r, l_r = _rank_partial(r, world)
            np.testing.assert_array_equal(o_lats[r], o_r.numpy())
            np.testing.assert_array_equal(lses[r], l_r.numpy())
        # the merge of the gathered partials is attention over the whole cache
        for b, n in enumerate(LENS):
            cache = O.gather_cache(pool, table[b], n)
            o_ref, l_ref = O.attend_latent(q_lat[b], cache[:, :D_C], cache[:, D_C:], 0.25)
            o_m, l_m = O.merge_partials([(o_lats[r][b], lses[r][b]) for r in range(world)])
            np.testing.assert_allclose(o_m, o_ref, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(l_m, l_ref, rtol=1e-12, atol=1e-12)
