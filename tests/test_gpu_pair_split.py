"""The selection branch's split between union tiles and tile-major (query,
tile) pairs, driven by caller selections built to reach every case of the
split: queries with more single-query tiles than pair slots (the rest stay in
the union), tiles that two or three queries of an item share (they leave when
each of their queries has a slot left, else they stay), tiles that more
queries share (block 0 and the queries' own blocks: they stay), and a last
item of one query, whose every tile could leave (it keeps them all).  The selection output and the layer output of those queries are
compared with the fp64 oracle given the same selection ("VideoNSA: Native
Sparse Attention Scales Video Understanding", paper notes, section "Method":
each query attends to the tokens of its selected blocks; the split only
reorders that softmax).
"""
import numpy as np
import pytest

import oracle
from parity_util import TOL, oracle_params, run_gpu
from sparse_attention_long_block_b200.inputs import Workload, generate

pytestmark = pytest.mark.gpu

QT = 18  # queries per 128-row item for 7 query heads per KV head


def _selection(wl, band, seed):
    """[h_kv][n][top_k] caller selection: blocks 0 and the query's own for
    every vision query; in the band of items, per item disjoint private blocks
    (17 to 22 for every sixth query, more than the 16 pair slots, 0 to 6 for
    the others), blocks shared by neighbouring queries (two-query tiles) and
    by three queries; the first item of the band has private blocks only."""
    rng = np.random.default_rng(seed)
    nv, k = wl.n_vision, wl.top_k
    sel = -np.ones((wl.h_kv, wl.n, k), np.int32)
    for g in range(wl.h_kv):
        for i in range(nv):
            row = sorted({0, i // wl.block})
            sel[g, i, :len(row)] = row
        for it in range(band[0] // QT, band[1] // QT):
            q0 = it * QT
            own_lo = q0 // wl.block
            pool = rng.permutation(np.arange(1, own_lo))
            at = 0
            sets = [set() for _ in range(QT)]

            def take(c):
                nonlocal at
                got = pool[at:at + c].tolist()
                at += c
                return got
            for qi in range(QT):
                c = int(rng.integers(17, 23)) if qi % 6 == 0 else int(rng.integers(0, 7))
                sets[qi].update(take(c))
            if it != band[0] // QT:
                for qi in range(0, QT - 1, 2):
                    for b in take(int(rng.integers(0, 5))):
                        sets[qi].add(b)
                        sets[qi + 1].add(b)
                for qi in range(0, QT - 2, 3):
                    for b in take(2):
                        for d in range(3):
                            sets[qi + d].add(b)
            for qi in range(QT):
                i = q0 + qi
                own = i // wl.block
                extra = sorted(sets[qi])[: k - 2]
                row = sorted(set([0, own] + extra))
                sel[g, i, :] = -1
                sel[g, i, :len(row)] = row
    return sel


@pytest.mark.parametrize("seed", [5, 6])
def test_pair_split_cases_match_oracle(seed):
    # 16,381 vision tokens: the last item holds one query
    wl = Workload(name="pairsplit", n_vision=256 * 64 - 3, n_text=40, top_k=32, window=128,
                  seed=70 + seed)
    x = generate(wl)
    nv = wl.n_vision
    band = (12600, 12600 + 6 * QT)
    fidx = _selection(wl, band, seed)
    g = run_gpu(wl, x, want=("o_slc",), forced_idx=fidx)
    assert g["status"] == 0
    # the band's rows and a few rows outside it (vision ranks = positions:
    # the vision tokens come first)
    rows = np.concatenate([np.arange(band[0], band[1]), np.array([0, 63, 64, 5000, nv - 1])])
    rows = rows.astype(np.int32)
    oi = np.transpose(fidx[:, rows, :], (1, 0, 2)).copy()
    o = oracle.forward(oracle_params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], rows=rows, forced_idx=oi, want=("o_slc",))
    tol = TOL["bf16"]
    e_slc = float(np.abs(g["o_slc"][rows] - o["o_slc"]).max())
    e_out = float(np.abs(g["out"][rows] - o["out"]).max())
    assert e_slc <= tol and e_out <= tol, (e_slc, e_out)
