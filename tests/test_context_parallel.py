"""Context-parallel decode, host side and oracle (no GPU).

* The oracle's partial records are pinned by the identity softmax attention
  over a sequence = the log-sum-exp merge of the records of any split of its
  rows (checked against the oracle's whole-sequence decode, which is pinned
  on its own), with empty ranges and merge order as special cases.
* rank_view covers every page of every sequence exactly once.
* Two gloo ranks exchange records with gather_records and merge to the
  whole-sequence answer.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

import harness as H
from bit_kv_cache_dqk_b200 import context_parallel as CP
from bit_kv_cache_dqk_b200 import inputs as I
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
W = I.CONFIGS["llama"].with_(name="cp-small", batch=3, hq=8, hkv=2, ctx=None, ctx_lo=1, ctx_hi=150,
                             page_order="random")


def _seq(w, b, L):
    cache = H.oracle_cache(w, b, L)
    q = I.queries(w, np.full(w.batch, max(L, 1), np.int32))[b]
    _, tq, _, _ = H.workload_transforms(w)
    return cache, q, tq


@pytest.mark.parametrize("cuts", [[0, 16, 48], [0, 1, 2, 3], [0, 70], [0, 5, 5, 90]])
def test_merge_of_split_equals_whole_sequence(cuts):
    L = 97
    cache, q, tq = _seq(W, 0, L)
    whole, _, _ = O.decode_seq(cache, q, tq, W.hq, W.pct, L=L)
    bounds = cuts + [L]
    recs = np.stack([O.decode_partial(cache, q, tq, W.hq, W.pct, t0=a, t1=b)
                     for a, b in zip(bounds[:-1], bounds[1:])])
    np.testing.assert_allclose(O.merge_partials(recs), whole, rtol=0, atol=1e-12)
    # any order of the records gives the same output
    np.testing.assert_allclose(O.merge_partials(recs[::-1]), whole, rtol=0, atol=1e-12)


def test_partial_record_of_whole_range():
    L = 40
    cache, q, tq = _seq(W, 1, L)
    whole, _, _ = O.decode_seq(cache, q, tq, W.hq, W.pct, L=L)
    rec = O.decode_partial(cache, q, tq, W.hq, W.pct)
    np.testing.assert_allclose(rec[:, 2:] / rec[:, 1:2], whole, rtol=0, atol=1e-12)
    # the max row contributes 2^0 = 1, every other row at most 1
    assert np.all(rec[:, 1] >= 1.0) and np.all(rec[:, 1] <= L)


def test_empty_ranges():
    cache, q, tq = _seq(W, 0, 20)
    empty = O.decode_partial(cache, q, tq, W.hq, W.pct, t0=7, t1=7)
    assert np.all(empty[:, 0] == -np.inf) and np.all(empty[:, 1:] == 0.0)
    full = O.decode_partial(cache, q, tq, W.hq, W.pct)
    np.testing.assert_array_equal(O.merge_partials(np.stack([empty, full, empty])),
                                  O.merge_partials(full[None]))
    assert np.all(O.merge_partials(np.stack([empty, empty])) == 0.0)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_rank_view_covers_each_page_once(world):
    lens = np.array([0, 1, 15, 16, 17, 100, 257, 4096], np.int32)
    w = W.with_(batch=len(lens))
    table, _ = I.page_table(w, np.maximum(lens, 1))
    seen = [[] for _ in lens]
    tok = np.zeros(len(lens), np.int64)
    for r in range(world):
        sub_lens, sub = CP.rank_view(lens, table, r, world)
        for b in range(len(lens)):
            n = (int(sub_lens[b]) + CP.PAGE - 1) // CP.PAGE
            seen[b] += sub[b, :n].tolist()
            # only the final page of a sequence may be partly filled
            p0, p1 = CP.page_range((int(lens[b]) + CP.PAGE - 1) // CP.PAGE, r, world)
            if p1 * CP.PAGE < lens[b]:
                assert sub_lens[b] == (p1 - p0) * CP.PAGE
        tok += sub_lens
    np.testing.assert_array_equal(tok, lens)
    for b, L in enumerate(lens):
        n = (int(L) + CP.PAGE - 1) // CP.PAGE
        assert seen[b] == table[b, :n].tolist()      # in logical order, no gaps, no repeats


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import harness as Hh
    from bit_kv_cache_dqk_b200 import context_parallel as CPr
    from bit_kv_cache_dqk_b200 import inputs as Ir
    from oracle import oracle as Or
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        lens = Ir.lengths(W)
        table, _ = Ir.page_table(W, np.maximum(lens, 1))
        sub_lens, _ = CPr.rank_view(lens, table, rank, world)
        qs = Ir.queries(W, np.maximum(lens, 1))
        _, tq, _, _ = Hh.workload_transforms(W)
        recs = []
        for b in range(W.batch):
            p0, _ = CPr.page_range((int(lens[b]) + CPr.PAGE - 1) // CPr.PAGE, rank, world)
            cache = Hh.oracle_cache(W, b, int(lens[b]))
            t0 = p0 * CPr.PAGE
            recs.append(Or.decode_partial(cache, qs[b], tq, W.hq, W.pct, t0=t0, t1=t0 + int(sub_lens[b])))
        part = torch.from_numpy(np.stack(recs))                   # fp64 records, [batch][hq][2+d]
        parts = CPr.gather_records(part).numpy()
        q.put((rank, Or.merge_partials(parts)))
    finally:
        dist.destroy_process_group()


def test_gloo_world2_exchange_and_merge():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(q.get(timeout=5) for _ in procs)
    lens = I.lengths(W)
    qs = I.queries(W, np.maximum(lens, 1))
    _, tq, _, _ = H.workload_transforms(W)
    for b in range(W.batch):
        cache = H.oracle_cache(W, b, int(lens[b]))
        whole, _, _ = O.decode_seq(cache, qs[b], tq, W.hq, W.pct, L=int(lens[b]))
        for r in (0, 1):
            np.testing.assert_allclose(res[r][b], whole, rtol=0, atol=1e-12)
