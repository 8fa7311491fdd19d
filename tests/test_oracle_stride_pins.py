"""Pins of the oracle's overlapping compression blocks (reading R13 at the top of
oracle/vnsa_oracle.c): a compression stride s below the block size B, the
native sparse attention design the VideoNSA pages build on ("VideoNSA: Native
Sparse Attention Scales Video Understanding", paper notes, section "Method";
the citation map's native-sparse-attention entry), with the compression
probability mass distributed over the selection blocks in proportion to the
tokens each compression block puts in them.

Each check catches a different slip:
  * the independent pure-Python brute force (explicit member lists, one token's
    share at a time): a wrong member range, visibility or remap weight;
  * s = B is bit-identical to the layer without a stride: the remap must be
    the identity there;
  * the remapped importance of a query sums to its group's head count when the
    vision tokens fill whole blocks (each head's probabilities sum to 1 and the
    remap moves mass without creating or losing any);
  * constant keys make every visible compression block equally likely, which
    gives each interior selection block r (B / s) / (visible blocks);
  * the visibility edge: no compression block before token B - 1, exactly one
    (whose output is then its own value) at B - 1, a second at B - 1 + s.
"""
import numpy as np
import pytest

import oracle
from oracle import brute
from sparse_attention_long_block_b200.inputs import Workload, generate, interleaved_mask


def wl_of(**kw):
    base = dict(name="s", n_vision=48, n_text=5, h_q=4, h_kv=2, d=6, top_k=4, window=7,
                dtype="fp32", block=4, seed=21)
    base.update(kw)
    return Workload(**base)


def params(wl, stride):
    return oracle.OracleParams(h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                               top_k=wl.top_k, window=wl.window, stride=stride,
                               round_cmp_bf16=(wl.dtype == "bf16"))


@pytest.mark.parametrize("block,stride,layout", [(4, 2, "suffix"), (4, 2, "interleaved"),
                                                 (6, 4, "suffix"), (5, 1, "interleaved"),
                                                 (4, 3, "suffix")])
def test_brute_force_matches_oracle_with_overlapping_blocks(block, stride, layout):
    wl = wl_of(block=block, top_k=3 if block > 4 else 4)
    mask = None if layout == "suffix" else interleaved_mask(wl.n_vision, wl.n_text, seed=3,
                                                            text_runs=2)
    x = generate(wl, mask)
    res = oracle.forward(params(wl, stride), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], want=("o_cmp", "o_slc", "o_swa", "idx", "imp"))
    bf = brute.layer(x["q"], x["k"], x["v"], x["is_vision"], x["gate"], x["w_k"], x["w_v"],
                     h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block, top_k=wl.top_k,
                     window=wl.window, stride=stride)
    assert np.max(np.abs(res["out"] - np.array(bf["out"]))) < 1e-12
    for t in range(wl.n):
        if not x["is_vision"][t]:
            continue
        for g in range(wl.h_kv):
            assert [j for j in res["idx"][t, g] if j >= 0] == bf["idx"][(t, g)]
            for j, val in bf["imp"][(t, g)].items():
                assert abs(res["imp"][t, g, j] - val) < 1e-12
        for h in range(wl.h_q):
            for name in ("o_cmp", "o_slc", "o_swa"):
                assert np.max(np.abs(res[name][t, h] - np.array(bf[name][(t, h)]))) < 1e-12


def test_stride_equal_to_block_is_the_plain_layer():
    wl = wl_of(n_vision=200, n_text=20, d=16, block=16, top_k=4, window=40, seed=5)
    x = generate(wl)
    want = ("o_cmp", "idx", "imp", "lse_cmp")
    a = oracle.forward(params(wl, None), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], want=want)
    b = oracle.forward(params(wl, 16), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], want=want)
    for name in ("out",) + want:
        assert np.array_equal(a[name], b[name]), name


@pytest.mark.parametrize("block,stride", [(8, 4), (8, 2), (6, 4), (8, 8)])
def test_remapped_importance_conserves_the_probability_mass(block, stride):
    wl = wl_of(n_vision=96, n_text=0, d=8, block=block, top_k=3, window=9, seed=8)
    x = generate(wl)
    res = oracle.forward(params(wl, stride), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], want=("imp",))
    r = wl.h_q // wl.h_kv
    for i in range(wl.n_vision):
        tot = res["imp"][i].sum(axis=1)  # per group
        expect = r if i >= block - 1 else 0.0
        assert np.allclose(tot, expect, atol=1e-12, rtol=0), (i, tot)


@pytest.mark.parametrize("block,stride", [(8, 4), (8, 2), (12, 4)])
def test_constant_keys_give_the_closed_form_importance(block, stride):
    wl = wl_of(n_vision=120, n_text=0, d=8, block=block, top_k=3, window=9, seed=9)
    x = generate(wl)
    x["k"][:] = x["k"][0:1]  # every token has the same key in each KV head
    res = oracle.forward(params(wl, stride), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], want=("imp",))
    r = wl.h_q // wl.h_kv
    i = wl.n_vision - 1
    ncv = (i - block + 1) // stride + 1            # visible compression blocks
    for j in range(1, (i + 1) // block - 1):       # interior selection blocks
        want = r * (block / stride) / ncv
        assert np.allclose(res["imp"][i, :, j], want, atol=1e-12, rtol=0), (j, res["imp"][i, :, j])


def test_visibility_edge_of_the_first_overlapping_blocks():
    block, stride = 8, 4
    wl = wl_of(n_vision=40, n_text=0, d=8, block=block, top_k=2, window=3, seed=10)
    x = generate(wl)
    p = params(wl, stride)
    kc, vc = oracle.pool_proj(p, x["k"], x["v"], x["is_vision"], x["w_k"], x["w_v"])
    assert kc.shape[0] == (40 - block) // stride + 1
    # block 1 averages tokens 4..11
    mean = x["v"][4:12].astype(np.float64).mean(axis=0)
    assert np.allclose(vc[1], mean @ x["w_v"].astype(np.float64), atol=1e-12, rtol=0)
    rows = np.array([block - 2, block - 1, block - 1 + stride - 1, block - 1 + stride], np.int32)
    res = oracle.forward(p, x["q"], x["k"], x["v"], x["is_vision"], x["gate"], x["w_k"],
                         x["w_v"], rows=rows, want=("o_cmp", "lse_cmp"))
    assert np.isneginf(res["lse_cmp"][0]).all() and (res["o_cmp"][0] == 0).all()
    r = wl.h_q // wl.h_kv
    for h in range(wl.h_q):
        for row in (1, 2):  # one visible compression block: its own value
            assert np.allclose(res["o_cmp"][row, h], vc[0, h // r], atol=1e-12, rtol=0)
        # two visible blocks: a convex combination that differs from block 0's value
        assert not np.allclose(res["o_cmp"][3, h], vc[0, h // r], atol=1e-9)
