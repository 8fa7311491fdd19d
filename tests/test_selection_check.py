"""The selection check the GPU parity tests use must reject malformed
selections, not only sets outside the tie band: a row that drops its k-th
block, repeats a block, leaves a hole in its -1 padding, picks a block the
query cannot see or loses a forced block.  ("VideoNSA: Native Sparse Attention
Scales Video Understanding", paper notes, section "Method": each query keeps
its top-k blocks by importance; block 0 and its own block are always kept.)
These run on the CPU against selections the oracle itself produced."""
import numpy as np
import pytest

import oracle
from parity_util import check_selection, check_selection_row, oracle_params
from sparse_attention_long_block_b200.inputs import Workload, generate


@pytest.fixture(scope="module")
def sel():
    wl = Workload(name="selchk", n_vision=640, n_text=0, h_q=4, h_kv=2, d=16, top_k=4,
                  window=32, dtype="fp32", seed=11)
    x = generate(wl)
    ranks = np.array([0, 62, 63, 64, 130, 300, 639], np.int32)
    o = oracle.forward(oracle_params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], rows=ranks, want=("idx", "imp"))
    return wl, ranks, o["idx"].copy(), o["imp"].copy()


def _check(wl, ranks, gpu, o_idx, o_imp):
    return check_selection(gpu, o_idx, o_imp, wl.top_k, block=wl.block, ranks=ranks)


def test_oracle_rows_pass_against_themselves(sel):
    wl, ranks, idx, imp = sel
    assert _check(wl, ranks, idx.copy(), idx, imp) == []
    # the counts the rule expects: rank 0..62 see no complete block (only the
    # forced block 0), rank 63 sees block 0, rank 64 has blocks 0 and 1
    assert [int((idx[r, 0] >= 0).sum()) for r in range(4)] == [1, 1, 1, 2]


def test_row_missing_its_kth_block_fails(sel):
    wl, ranks, idx, imp = sel
    r = len(ranks) - 1  # rank 639: four blocks selected
    gpu = idx.copy()
    row = [j for j in gpu[r, 0] if j >= 0]
    assert len(row) == wl.top_k
    free = [j for j in row if j not in (0, ranks[r] // wl.block)]
    row.remove(free[-1])
    gpu[r, 0] = row + [-1]
    with pytest.raises(AssertionError, match="expected"):
        _check(wl, ranks, gpu, idx, imp)


def test_duplicated_block_fails(sel):
    wl, ranks, idx, imp = sel
    r = len(ranks) - 1
    gpu = idx.copy()
    gpu[r, 1, 2] = gpu[r, 1, 1]
    with pytest.raises(AssertionError, match="ascending"):
        _check(wl, ranks, gpu, idx, imp)


def test_hole_in_padding_fails():
    with pytest.raises(AssertionError, match="after the first -1"):
        check_selection_row([0, -1, 3, -1], i=300, top_k=4, block=64)
    with pytest.raises(AssertionError, match="after the first -1"):
        check_selection_row([0, 2, 4, -5], i=300, top_k=4, block=64, expect_count=3)


def test_block_not_visible_fails():
    # rank 130 sees blocks 0 and 1 (complete) and owns block 2; block 3 is ahead
    assert check_selection_row([0, 1, 2, -1], i=130, top_k=4, block=64) == [0, 1, 2]
    with pytest.raises(AssertionError, match="not visible"):
        check_selection_row([0, 1, 3, -1], i=130, top_k=4, block=64)


def test_missing_forced_block_fails():
    with pytest.raises(AssertionError, match="forced"):
        check_selection_row([1, 2, 3, 4], i=300, top_k=4, block=64)  # block 0 dropped
    with pytest.raises(AssertionError, match="forced"):
        check_selection_row([0, 1, 2, 3], i=300, top_k=4, block=64)  # own block 4 dropped


def test_swap_inside_and_outside_the_tie_band(sel):
    wl, ranks, idx, imp = sel
    r = len(ranks) - 1
    i = int(ranks[r])
    chosen = [int(j) for j in idx[r, 0] if j >= 0 and j not in (0, i // wl.block)]
    kth = min(chosen, key=lambda j: imp[r, 0, j])
    other = next(j for j in range(1, (i + 1) // wl.block) if j not in idx[r, 0])
    gpu = idx.copy()
    gpu[r, 0] = sorted([j for j in idx[r, 0] if j != kth] + [other])
    imp_tie = imp.copy()
    imp_tie[r, 0, other] = imp[r, 0, kth] * (1 - 5e-4)
    assert _check(wl, ranks, gpu, idx, imp_tie) == [r]
    imp_far = imp.copy()
    imp_far[r, 0, other] = imp[r, 0, kth] * 0.9
    with pytest.raises(AssertionError, match="tie band"):
        _check(wl, ranks, gpu, idx, imp_far)
