"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Sources: "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
notes), section "Method" (three gated branches over vision tokens, dense GQA
over text), and the readings R1-R10 at the top of oracle/vnsa_oracle.c.

Each check is chosen so that a plausible slip in the oracle fails it:
  * dense reductions vs torch's scaled_dot_product_attention (a library
    routine): a wrong scale, mask, GQA head map or softmax normalisation;
  * block size 1 with W = I vs dense attention: a wrong visibility rule (R2)
    or projection orientation;
  * closed forms of the pooling (mean, W = I, constant blocks);
  * V = 1 and w = 1: normalisation of each branch and the window extent;
  * an independent pure-Python brute force (dicts, subset enumeration for the
    top-k): index slips, tie rule, forced blocks, gate order;
  * permutation invariance of the vision rows under an interleaved mask.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from sparse_attention_long_block_b200.inputs import (Workload, bf16_round, generate,
                                                     interleaved_mask)

NEG, POS = -np.inf, np.inf


def sdpa_causal(q, k, v, scale):
    """Dense causal GQA via torch (fp64, CPU): q [n][hq][d], k, v [n][hkv][d]."""
    hq, hkv = q.shape[1], k.shape[1]
    r = hq // hkv
    qt = torch.from_numpy(np.asarray(q, np.float64)).permute(1, 0, 2)
    kt = torch.from_numpy(np.asarray(k, np.float64)).permute(1, 0, 2).repeat_interleave(r, 0)
    vt = torch.from_numpy(np.asarray(v, np.float64)).permute(1, 0, 2).repeat_interleave(r, 0)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o.permute(1, 0, 2).numpy()


def small_wl(**kw):
    base = dict(name="t", n_vision=200, n_text=24, h_q=4, h_kv=2, d=16, top_k=4,
                window=40, dtype="fp32", block=16)
    base.update(kw)
    return Workload(**base)


def params(wl, **kw):
    p = oracle.OracleParams(h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                            top_k=wl.top_k, window=wl.window,
                            round_cmp_bf16=(wl.dtype == "bf16"))
    for k_, v_ in kw.items():
        setattr(p, k_, v_)
    return p


def gates_onehot(x, n, hq, branch):
    g = np.full((n, hq, 3), NEG, np.float32)
    g[:, :, branch] = POS
    return g


# ----------------------------------------------------------------------------
def test_bf16_rounding_agrees_with_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-6, 6, 4000),
                        [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 3.0e-39]])
    t = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    o = np.array([oracle.round_bf16(float(np.float32(v))) for v in x])
    b = np.array([brute._bf16(float(np.float32(v))) for v in x])
    n = bf16_round(x.astype(np.float32)).astype(np.float64)
    assert np.array_equal(o, t)
    assert np.array_equal(b, t)
    assert np.array_equal(n, t)


@pytest.mark.parametrize("layout", ["suffix", "interleaved"])
def test_brute_force_matches_oracle(layout):
    wl = small_wl(n_vision=46, n_text=6, h_q=4, h_kv=2, d=6, top_k=4, window=5,
                  block=4, seed=11)
    mask = None if layout == "suffix" else interleaved_mask(46, 6, seed=5, text_runs=3)
    x = generate(wl, mask)
    p = params(wl)
    res = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], want=("o_cmp", "o_slc", "o_swa", "idx", "imp"))
    bf = brute.layer(x["q"], x["k"], x["v"], x["is_vision"], x["gate"], x["w_k"], x["w_v"],
                     h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block, top_k=wl.top_k,
                     window=wl.window)
    assert np.max(np.abs(res["out"] - np.array(bf["out"]))) < 1e-12
    n, r = wl.n, wl.h_q // wl.h_kv
    for t in range(n):
        if not x["is_vision"][t]:
            assert (res["idx"][t] == -1).all()
            continue
        for g in range(wl.h_kv):
            sel = [j for j in res["idx"][t, g] if j >= 0]
            assert sel == bf["idx"][(t, g)]
            for j, val in bf["imp"][(t, g)].items():
                assert abs(res["imp"][t, g, j] - val) < 1e-12
        for h in range(wl.h_q):
            for name in ("o_cmp", "o_slc", "o_swa"):
                assert np.max(np.abs(res[name][t, h] - np.array(bf[name][(t, h)]))) < 1e-12


def test_brute_force_matches_oracle_bf16_rounding_of_cmp():
    wl = small_wl(n_vision=40, n_text=4, h_q=2, h_kv=1, d=4, top_k=3, window=6,
                  block=8, seed=2, dtype="bf16")
    x = generate(wl)
    p = params(wl)
    kc, vc = oracle.pool_proj(p, x["k"], x["v"], x["is_vision"], x["w_k"], x["w_v"])
    res = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"], x["w_k"], x["w_v"])
    bf = brute.layer(x["q"], x["k"], x["v"], x["is_vision"], x["gate"], x["w_k"], x["w_v"],
                     h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block, top_k=wl.top_k,
                     window=wl.window, round_cmp_bf16=True)
    assert np.max(np.abs(res["out"] - np.array(bf["out"]))) < 1e-12
    # every rounded value is a bf16 value
    for a in (kc, vc):
        assert all(oracle.round_bf16(float(v)) == float(v) for v in a.ravel())


@pytest.mark.parametrize("branch", [1, 2])
def test_full_budget_reduces_to_dense_causal(branch):
    """top_k covering every block (incl. the query's own partial block) or a
    window >= N, with the gate on that branch only: vision rows equal dense causal
    attention over the vision tokens; text rows equal dense causal attention over
    the whole sequence."""
    wl = small_wl(n_vision=200, n_text=30, top_k=200 // 16 + 1, window=10_000, seed=4)
    mask = interleaved_mask(200, 30, seed=9, text_runs=3)
    x = generate(wl, mask)
    gate = gates_onehot(None, wl.n, wl.h_q, branch)
    p = params(wl)
    res = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], gate, x["w_k"], x["w_v"])
    scale = 1.0 / math.sqrt(wl.d)
    vis = np.nonzero(x["is_vision"])[0]
    txt = np.nonzero(x["is_vision"] == 0)[0]
    dense_v = sdpa_causal(x["q"][vis], x["k"][vis], x["v"][vis], scale)
    dense_all = sdpa_causal(x["q"], x["k"], x["v"], scale)
    assert np.max(np.abs(res["out"][vis] - dense_v)) < 1e-12
    assert np.max(np.abs(res["out"][txt] - dense_all[txt])) < 1e-12


def test_block_size_one_identity_projection_is_dense():
    """Block 1, W = I: every token is its own compressed key, so compression is
    dense causal attention (pins the visibility rule: a query sees its own token)."""
    wl = small_wl(n_vision=120, n_text=0, block=1, top_k=2, window=3, seed=6)
    x = generate(wl)
    eye = np.eye(wl.d, dtype=np.float32)
    gate = gates_onehot(None, wl.n, wl.h_q, 0)
    p = params(wl)
    res = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], gate, eye, eye,
                         want=("o_cmp",))
    dense = sdpa_causal(x["q"], x["k"], x["v"], 1.0 / math.sqrt(wl.d))
    assert np.max(np.abs(res["o_cmp"] - dense)) < 1e-12
    assert np.max(np.abs(res["out"] - dense)) < 1e-12


def test_pooling_closed_forms():
    wl = small_wl(n_vision=100, n_text=8, block=16, seed=7)
    mask = interleaved_mask(100, 8, seed=2)
    x = generate(wl, mask)
    p = params(wl)
    vis = np.nonzero(mask)[0]
    nb = 100 // 16
    eye = np.eye(wl.d, dtype=np.float32)
    kc, vc = oracle.pool_proj(p, x["k"], x["v"], mask, eye, eye)
    kv = x["k"][vis][: nb * 16].astype(np.float64).reshape(nb, 16, wl.h_kv, wl.d).mean(1)
    vv = x["v"][vis][: nb * 16].astype(np.float64).reshape(nb, 16, wl.h_kv, wl.d).mean(1)
    assert kc.shape == (nb, wl.h_kv, wl.d)
    assert np.max(np.abs(kc - kv)) < 1e-12 and np.max(np.abs(vc - vv)) < 1e-12
    # a constant block c maps to exactly c . W
    k2 = x["k"].copy()
    c = np.float32(0.375)
    k2[vis] = c
    kc2, _ = oracle.pool_proj(p, k2, x["v"], mask, x["w_k"], x["w_v"])
    expect = (np.full(wl.d, 0.375) @ x["w_k"].astype(np.float64))
    assert np.max(np.abs(kc2 - expect[None, None, :])) < 1e-12


def test_softmax_rows_sum_to_one_via_unit_values():
    wl = small_wl(n_vision=180, n_text=20, seed=8)
    x = generate(wl)
    ones = np.ones_like(x["v"])
    p = params(wl)
    res = oracle.forward(p, x["q"], x["k"], ones, x["is_vision"], x["gate"], x["w_k"],
                         np.eye(wl.d, dtype=np.float32),
                         want=("o_cmp", "o_slc", "o_swa"))
    vis = np.nonzero(x["is_vision"])[0]
    has_cmp = (np.arange(len(vis)) + 1) // wl.block > 0
    assert np.max(np.abs(res["o_slc"][vis] - 1)) < 1e-12
    assert np.max(np.abs(res["o_swa"][vis] - 1)) < 1e-12
    assert np.max(np.abs(res["o_cmp"][vis[has_cmp]] - 1)) < 1e-12
    assert np.all(res["o_cmp"][vis[~has_cmp]] == 0)
    sig = 1 / (1 + np.exp(-x["gate"].astype(np.float64)))
    expect = sig[vis, :, 0] * has_cmp[:, None] + sig[vis, :, 1] + sig[vis, :, 2]
    assert np.max(np.abs(res["out"][vis] - expect[:, :, None])) < 1e-12
    txt = np.nonzero(x["is_vision"] == 0)[0]
    assert np.max(np.abs(res["out"][txt] - 1)) < 1e-12


def test_window_of_one_returns_own_value():
    wl = small_wl(n_vision=90, n_text=0, window=1, seed=10)
    x = generate(wl)
    res = oracle.forward(params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], want=("o_swa",))
    r = wl.h_q // wl.h_kv
    expect = np.repeat(x["v"].astype(np.float64), r, axis=1)
    assert np.array_equal(res["o_swa"], expect)


def test_zero_gate_logits_average_the_branches():
    wl = small_wl(n_vision=150, n_text=10, seed=12)
    x = generate(wl)
    zero = np.zeros_like(x["gate"])
    res = oracle.forward(params(wl), x["q"], x["k"], x["v"], x["is_vision"], zero,
                         x["w_k"], x["w_v"], want=("o_cmp", "o_slc", "o_swa"))
    vis = np.nonzero(x["is_vision"])[0]
    expect = 0.5 * (res["o_cmp"] + res["o_slc"] + res["o_swa"])
    assert np.max(np.abs(res["out"][vis] - expect[vis])) < 1e-14
    # linearity in the gates: a branch turned off drops its term exactly
    g2 = zero.copy()
    g2[:, :, 0] = NEG
    res2 = oracle.forward(params(wl), x["q"], x["k"], x["v"], x["is_vision"], g2,
                          x["w_k"], x["w_v"])
    assert np.max(np.abs(res2["out"][vis] - 0.5 * (res["o_slc"] + res["o_swa"])[vis])) < 1e-14


def test_group_importance_sums_to_group_size():
    """Each head's compression probabilities sum to 1, so the group sum of the
    importance over visible blocks is H_q/H_kv; with one head per group it is the
    probability row itself."""
    for hq, hkv in ((4, 2), (3, 3)):
        wl = small_wl(n_vision=160, n_text=0, h_q=hq, h_kv=hkv, seed=13)
        x = generate(wl)
        res = oracle.forward(params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                             x["w_k"], x["w_v"], want=("imp", "lse_cmp"))
        nvis = (np.arange(wl.n) + 1) // wl.block
        tot = res["imp"].sum(-1)
        ok = nvis > 0
        assert np.max(np.abs(tot[ok] - hq // hkv)) < 1e-12
        assert np.all(tot[~ok] == 0)
        assert np.all(np.isneginf(res["lse_cmp"][~ok]))


def test_topk_ties_go_to_lower_blocks_and_forced_blocks_count():
    """All blocks equal (identical K in every block) -> every visible block has
    the same importance; the tie rule then takes the lowest non-forced blocks."""
    wl = small_wl(n_vision=16 * 12, n_text=0, top_k=4, block=16, seed=14)
    x = generate(wl)
    k = x["k"].copy()
    k[:] = k[:16].mean(0, keepdims=True)  # same key for every token
    res = oracle.forward(params(wl), x["q"], k, x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], want=("idx",))
    for i in range(wl.n):
        own = i // 16
        nvis = (i + 1) // 16
        forced = sorted({0, own})
        cands = [j for j in range(nvis) if j not in forced]
        expect = sorted(set(forced) | set(cands[: 4 - len(forced)]))
        expect = expect + [-1] * (4 - len(expect))
        for g in range(wl.h_kv):
            assert list(res["idx"][i, g]) == expect, (i, g)


def test_vision_rows_ignore_text_tokens_and_positions():
    """R1: vision rows depend only on the vision subsequence; moving text tokens
    around (interleaving) leaves them unchanged.  Text rows ignore gate logits."""
    wl = small_wl(n_vision=170, n_text=25, seed=15)
    mask = interleaved_mask(170, 25, seed=4, text_runs=5)
    x = generate(wl, mask)
    p = params(wl)
    res = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"])
    vis = np.nonzero(mask)[0]
    txt = np.nonzero(mask == 0)[0]
    only = oracle.forward(p, x["q"][vis], x["k"][vis], x["v"][vis],
                          np.ones(len(vis), np.uint8), x["gate"][vis], x["w_k"], x["w_v"])
    assert np.max(np.abs(res["out"][vis] - only["out"])) == 0.0
    g2 = x["gate"].copy()
    g2[txt] = 123.0
    res2 = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], g2, x["w_k"], x["w_v"])
    assert np.array_equal(res2["out"], res["out"])


def test_row_subset_equals_full_run():
    wl = small_wl(n_vision=130, n_text=12, seed=16)
    x = generate(wl)
    p = params(wl)
    full = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                          x["w_k"], x["w_v"], want=("idx", "imp"))
    rows = np.array([0, 5, 63, 64, 129, 130, 141])
    sub = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], rows=rows, want=("idx", "imp"))
    assert np.array_equal(sub["out"], full["out"][rows])
    assert np.array_equal(sub["idx"], full["idx"][rows])


def test_forced_idx_replaces_selection():
    wl = small_wl(n_vision=160, n_text=0, seed=17)
    x = generate(wl)
    p = params(wl)
    full = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                          x["w_k"], x["w_v"], want=("idx", "o_slc"))
    again = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                           x["w_k"], x["w_v"], forced_idx=full["idx"], want=("o_slc",))
    assert np.array_equal(again["out"], full["out"])
    # selecting only the own block gives attention over that block's prefix
    fidx = np.full_like(full["idx"], -1)
    fidx[:, :, 0] = (np.arange(wl.n) // wl.block)[:, None]
    own = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], forced_idx=fidx, want=("o_slc",))
    scale = 1.0 / math.sqrt(wl.d)
    r = wl.h_q // wl.h_kv
    for i in (0, 17, 47, 100, 159):
        lo = (i // wl.block) * wl.block
        kk = np.repeat(x["k"][lo:i + 1].astype(np.float64), r, axis=1)
        vv = np.repeat(x["v"][lo:i + 1].astype(np.float64), r, axis=1)
        s = np.einsum("hd,uhd->hu", x["q"][i].astype(np.float64), kk) * scale
        pr = np.exp(s - s.max(1, keepdims=True))
        pr /= pr.sum(1, keepdims=True)
        o = np.einsum("hu,uhd->hd", pr, vv)
        assert np.max(np.abs(own["o_slc"][i] - o)) < 1e-12


def test_invalid_arguments_rejected():
    wl = small_wl(n_vision=64, n_text=0, top_k=1)
    x = generate(wl)
    with pytest.raises(ValueError):
        oracle.forward(params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"])
