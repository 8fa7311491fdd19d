"""The benchmark's work accounting, on the host.

The roofline numerator is the algorithmic work: 4 d H_q flops per attended
(query, key) pair.  These tests count the pairs the oracle's own selections
attend, key by key, and check the benchmark's closed-form counts against them
(compression: visible blocks; selection: the keys of the selected blocks at or
before the query; window: min(w, i + 1); text: t + 1).  They also check the
executed-work count of the selection branch when tiles that one to three
queries of an item reach run tile-major (up to 18 such pairs of one tile per
128-row tile).
"""
import numpy as np
import pytest

import bench
import oracle
from parity_util import oracle_params
from sparse_attention_long_block_b200.inputs import (WORKLOADS, Workload, generate,
                                                     interleaved_mask)


def _pairs_by_enumeration(wl, x):
    o = oracle.forward(oracle_params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], want=("idx",))
    isv = x["is_vision"]
    vis = np.nonzero(isv)[0]
    txt = np.nonzero(isv == 0)[0]
    B = wl.block
    st = wl.stride or B
    cmp = slc = swa = imp = 0
    nb = len(vis) // B
    # compression blocks: start c s, tokens [c s, c s + B) all vision ranks
    starts = [c for c in range(0, len(vis)) if c % st == 0 and c + B <= len(vis)]
    for i, t in enumerate(vis):
        cmp += sum(1 for c0 in starts if c0 + B - 1 <= i)
        imp += min((i + 1) // B, nb)  # selection blocks with an importance
        swa += min(wl.window, i + 1)
        row = o["idx"][t, 0]  # group 0; every group selects as many keys
        for j in row[row >= 0]:
            slc += sum(1 for u in range(j * B, j * B + B) if u <= i)
    text = int((txt + 1).sum())
    return {"cmp": cmp, "slc": slc, "swa": swa, "text": text, "imp": imp}


@pytest.mark.parametrize("wl,mask", [
    (WORKLOADS["tiny_fp32_1k"], None),
    (Workload("acct64", 700, 60, h_q=8, h_kv=2, d=64, top_k=5, window=100, seed=3), "mix"),
    (Workload("acct36", 520, 40, h_q=8, h_kv=2, d=64, top_k=6, window=90, block=36,
              frame=36, seed=4), None),
    (Workload("acct_s16", 600, 30, h_q=8, h_kv=2, d=64, top_k=5, window=80, stride=16,
              seed=5), "mix"),
])
def test_algorithmic_pairs_match_enumeration(wl, mask):
    isv = interleaved_mask(wl.n_vision, wl.n_text, seed=2) if mask else None
    x = generate(wl, isv)
    got = bench.algorithmic_work(wl, x["is_vision"])
    want = _pairs_by_enumeration(wl, x)
    f = 4.0 * wl.d * wl.h_q
    for name in ("cmp", "slc", "swa", "text"):
        assert got[name] == f * want[name], name
    # top-k reads one fp32 importance per complete (group, query, selection
    # block) and writes top_k int32 per (group, query)
    nv = int(x["is_vision"].sum())
    assert got["topk_bytes"] == 4.0 * wl.h_kv * want["imp"] + 4.0 * wl.h_kv * nv * wl.top_k


def test_selection_executed_work_splits_one_to_three_query_tiles():
    # one group, 7 heads (18 queries per 128-row tile), block 64, two items
    wl = Workload("acct_split", 36 * 64, 0, h_q=7, h_kv=1, d=128, top_k=3, window=64)
    isv = np.ones(wl.n, np.uint8)
    nv = wl.n_vision
    idx = -np.ones((1, nv, 3), np.int32)
    idx[0, :, 0] = 0                      # block 0: every query, kept in the union
    idx[0, 0:18, 1] = np.arange(1, 19)    # item 0: 18 tiles reached by one query each
    idx[0, 18:36, 1] = np.arange(1, 19)   # item 1: the same 18 tiles, one query each
    idx[0, 0, 2] = 30                     # item 0: tile 30 reached by queries 0 and 1
    idx[0, 1, 2] = 30
    idx[0, 18:21, 2] = 31                 # item 1: tile 31 reached by three queries
    idx[0, 21:25, 2] = 32                 # item 1: tile 32 reached by four queries
    ex = bench.executed_work(wl, isv, idx)
    prod = 2.0 * 128 * 64 * wl.d
    # item 0 keeps block 0's tile, item 1 block 0's and tile 32; the 36
    # single-query pairs fall into 18 (group, tile) buckets of 2 pairs, the
    # two-query tile 30 and the three-query tile 31 add a bucket of 2 and one of
    # 3 pairs: one tile-major tile each; the other items (queries 36 ..) reach
    # block 0 only
    n_items = -(-nv // 18)
    union_tiles = 1 + 2 + (n_items - 2) * 1
    assert ex["slc"] == 2 * prod * (union_tiles + 20)
    # a query with more than 16 pairs: its 17th single-query tile stays, and so
    # does a two-query tile of a query without a free slot
    wl2 = Workload("acct_cap", 64 * 64, 0, h_q=7, h_kv=1, d=128, top_k=20, window=64)
    isv2 = np.ones(wl2.n, np.uint8)
    idx2 = -np.ones((1, wl2.n_vision, 20), np.int32)
    idx2[0, :, 0] = 0
    q = 2600                                # own block 40; item 144 (queries 2592 ..)
    idx2[0, q, 1:18] = np.arange(1, 18)     # 17 tiles reached by this query alone
    idx2[0, q, 18] = 30                     # and a tile shared with the next query
    idx2[0, q + 1, 1] = 30
    ex2 = bench.executed_work(wl2, isv2, idx2)
    prod2 = 2.0 * 128 * 64 * wl2.d
    n_items2 = -(-wl2.n_vision // 18)
    # item 144 keeps block 0's tile, the 17th single tile and tile 30; 16
    # pairs leave, one bucket each
    assert ex2["slc"] == 2 * prod2 * ((n_items2 - 1) + 3 + 16)
    # an item whose tiles all serve one query keeps them all (the plan cannot
    # be empty), so nothing leaves for the tile-major pass
    idx1 = -np.ones((1, nv, 3), np.int32)
    idx1[0, 0, 0] = 0
    ex1 = bench.executed_work(wl, isv, idx1)
    assert ex1["slc"] == 2 * prod * 1
