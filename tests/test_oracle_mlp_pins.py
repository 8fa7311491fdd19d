"""Pins of the oracle's two perceptrons (the compression branch's "learnable
MLP" and the two-layer gate MLP of "VideoNSA: Native Sparse Attention Scales
Video Understanding" (paper notes), section "Method"; readings R11 and R12 at
the top of oracle/vnsa_oracle.c).

Each check comes from outside the oracle's code: a zero layer leaves the bias
(or SiLU of the bias, written here from the definition z / (1 + e^-z)); a
one-hot input through a single nonzero weight in each layer lands in exactly
one output column (a transposed weight or a swapped layer would move or drop
it); random weights agree with torch's Linear / SiLU in fp64 (a library
routine); the bf16 rounding of the gate's hidden layer agrees with torch's
bf16 conversion; and a layer whose compression keys are all equal has the
closed form of a uniform softmax (o_cmp = the common value, importance r/nvis).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sparse_attention_long_block_b200.inputs import Workload, generate


def silu(z):
    return z / (1.0 + math.exp(-z))


def params(wl):
    return oracle.OracleParams(h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                               top_k=wl.top_k, window=wl.window,
                               round_cmp_bf16=(wl.dtype == "bf16"))


def rand_cmp_mlp(rng, d, hidden, scale=1.0):
    m = {}
    for t in ("k", "v"):
        m["w1_" + t] = (rng.standard_normal((d, hidden)) * scale / np.sqrt(d)).astype(np.float32)
        m["b1_" + t] = (rng.standard_normal(hidden) * 0.1).astype(np.float32)
        m["w2_" + t] = (rng.standard_normal((hidden, d)) * scale / np.sqrt(hidden)).astype(np.float32)
        m["b2_" + t] = (rng.standard_normal(d) * 0.1).astype(np.float32)
    return m


def block_means(x, is_vision, block):
    xv = x[np.nonzero(is_vision)[0]].astype(np.float64)
    nb = len(xv) // block
    return xv[: nb * block].reshape(nb, block, *x.shape[1:]).mean(1)


def torch_mlp(x, w1, b1, w2, b2):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    h = torch.nn.functional.silu(t(x) @ t(w1) + t(b1))
    return (h @ t(w2) + t(b2)).numpy()


WL = Workload("mlp", 320, 16, h_q=4, h_kv=2, d=16, top_k=3, window=40, dtype="fp32", block=32)


def test_cmp_mlp_zero_second_layer_leaves_bias():
    x = generate(WL)
    m = rand_cmp_mlp(np.random.default_rng(1), WL.d, 24)
    m["w2_k"][:] = 0
    m["w2_v"][:] = 0
    kc, vc = oracle.pool_proj(params(WL), x["k"], x["v"], x["is_vision"], cmp_mlp=m)
    assert kc.shape == (10, WL.h_kv, WL.d)
    assert np.array_equal(kc, np.broadcast_to(m["b2_k"].astype(np.float64), kc.shape))
    assert np.array_equal(vc, np.broadcast_to(m["b2_v"].astype(np.float64), vc.shape))


def test_cmp_mlp_zero_first_layer_is_silu_of_bias():
    x = generate(WL)
    m = rand_cmp_mlp(np.random.default_rng(2), WL.d, 24)
    m["w1_k"][:] = 0
    m["w1_v"][:] = 0
    kc, vc = oracle.pool_proj(params(WL), x["k"], x["v"], x["is_vision"], cmp_mlp=m)
    for got, t in ((kc, "k"), (vc, "v")):
        h = np.array([silu(float(b)) for b in m["b1_" + t]])
        want = h @ m["w2_" + t].astype(np.float64) + m["b2_" + t]
        np.testing.assert_allclose(got, np.broadcast_to(want, got.shape), rtol=0, atol=1e-13)


def test_cmp_mlp_orientation_one_hot():
    # K equal to alpha * e_a on every token: the block mean is alpha * e_a.
    # W1 has one nonzero at [a][xh], W2 one at [xh][c], zero biases: only
    # column c of K_cmp is nonzero, = u * SiLU(alpha * w) (values exact in fp32).
    d, hid, a, xh, c, alpha, w, u = 16, 12, 3, 7, 11, 1.5, -0.75, 2.0
    x = generate(WL)
    k = np.zeros_like(x["k"])
    k[:, :, a] = alpha
    m = {nm: np.zeros(s, np.float32) for nm, s in
         (("w1_k", (d, hid)), ("b1_k", hid), ("w2_k", (hid, d)), ("b2_k", d),
          ("w1_v", (d, hid)), ("b1_v", hid), ("w2_v", (hid, d)), ("b2_v", d))}
    m["w1_k"][a, xh] = w
    m["w2_k"][xh, c] = u
    kc, _ = oracle.pool_proj(params(WL), k, x["v"], x["is_vision"], cmp_mlp=m)
    want = np.zeros(d)
    want[c] = u * silu(alpha * w)
    np.testing.assert_allclose(kc, np.broadcast_to(want, kc.shape), rtol=0, atol=1e-15)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_cmp_mlp_matches_torch(dtype):
    wl = WL.with_(dtype=dtype)
    x = generate(wl)
    m = rand_cmp_mlp(np.random.default_rng(3), wl.d, 40, scale=2.0)
    kc, vc = oracle.pool_proj(params(wl), x["k"], x["v"], x["is_vision"], cmp_mlp=m)
    for got, src, t in ((kc, x["k"], "k"), (vc, x["v"], "v")):
        want = torch_mlp(block_means(src, x["is_vision"], wl.block), m["w1_" + t], m["b1_" + t],
                         m["w2_" + t], m["b2_" + t])
        if dtype == "bf16":
            # R3/R11: the result is rounded once to bf16 (torch's bf16 cast is
            # round-to-nearest-even on the fp32 value; compare within one ulp)
            ulp = np.abs(want) * 2.0 ** -7 + 1e-30
            assert (np.abs(got - want) <= ulp).all()
        else:
            np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_layer_with_equal_compression_keys_is_uniform():
    # W2 = 0: every block key is b2_k and every block value b2_v, so the
    # compression softmax is uniform over the visible blocks: o_cmp = b2_v and
    # each visible block's group importance is r / nvis
    x = generate(WL)
    m = rand_cmp_mlp(np.random.default_rng(4), WL.d, 8)
    m["w2_k"][:] = 0
    m["w2_v"][:] = 0
    o = oracle.forward(params(WL), x["q"], x["k"], x["v"], x["is_vision"], x["gate"], None, None,
                       want=("o_cmp", "imp"), cmp_mlp=m)
    r = WL.h_q // WL.h_kv
    vis = np.nonzero(x["is_vision"])[0]
    for i, t in enumerate(vis):
        nvis = min((i + 1) // WL.block, o["nb"])
        if nvis == 0:
            assert np.all(o["o_cmp"][t] == 0)
            continue
        np.testing.assert_allclose(o["o_cmp"][t], np.broadcast_to(m["b2_v"], (WL.h_q, WL.d)),
                                   rtol=0, atol=1e-12)
        np.testing.assert_allclose(o["imp"][t][:, :nvis], r / nvis, rtol=1e-12)
        assert np.all(o["imp"][t][:, nvis:] == 0)


def rand_gate(rng, n, dm, hidden, n_out):
    x = rng.standard_normal((n, dm)).astype(np.float32)
    g1 = (rng.standard_normal((dm, hidden)) / np.sqrt(dm)).astype(np.float32)
    c1 = (rng.standard_normal(hidden) * 0.1).astype(np.float32)
    g2 = (rng.standard_normal((hidden, n_out)) / np.sqrt(hidden)).astype(np.float32)
    c2 = rng.standard_normal(n_out).astype(np.float32)
    return x, g1, c1, g2, c2


def test_gate_mlp_zero_layers():
    x, g1, c1, g2, c2 = rand_gate(np.random.default_rng(5), 9, 40, 16, 12)
    out = oracle.gate_mlp(x, g1, c1, np.zeros_like(g2), c2)
    assert np.array_equal(out, np.broadcast_to(c2.astype(np.float64), out.shape))
    out = oracle.gate_mlp(x, np.zeros_like(g1), c1, g2, c2)
    h = np.array([silu(float(b)) for b in c1])
    np.testing.assert_allclose(out, np.broadcast_to(h @ g2.astype(np.float64) + c2, out.shape),
                               rtol=0, atol=1e-13)


def test_gate_mlp_orientation_one_hot():
    n, dm, hid, n_out, a, xh, o_, alpha, w, u = 3, 40, 16, 12, 5, 9, 4, 0.75, 1.25, -1.125
    x = np.zeros((n, dm), np.float32)
    x[:, a] = alpha
    g1 = np.zeros((dm, hid), np.float32)
    g1[a, xh] = w
    g2 = np.zeros((hid, n_out), np.float32)
    g2[xh, o_] = u
    out = oracle.gate_mlp(x, g1, np.zeros(hid, np.float32), g2, np.zeros(n_out, np.float32))
    want = np.zeros(n_out)
    want[o_] = u * silu(alpha * w)
    np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=1e-15)


def test_gate_mlp_matches_torch():
    x, g1, c1, g2, c2 = rand_gate(np.random.default_rng(6), 33, 96, 48, 84)
    out = oracle.gate_mlp(x, g1, c1, g2, c2)
    np.testing.assert_allclose(out, torch_mlp(x, g1, c1, g2, c2), rtol=1e-12, atol=1e-12)


def test_gate_mlp_bf16_hidden_rounding_matches_torch():
    # g2 = identity: the logits are the (rounded) hidden activations themselves
    x, g1, c1, _, _ = rand_gate(np.random.default_rng(7), 17, 64, 32, 32)
    out = oracle.gate_mlp(x, g1, c1, np.eye(32, dtype=np.float32), np.zeros(32, np.float32),
                          round_hidden_bf16=True)
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    h = torch.nn.functional.silu(t(x) @ t(g1) + t(c1))
    # torch rounds fp64 -> bf16 to nearest even directly
    want = h.to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(out, want)


def test_gate_mlp_rejects_bad_shapes():
    x, g1, c1, g2, c2 = rand_gate(np.random.default_rng(8), 4, 8, 4, 6)
    with pytest.raises(ValueError):
        oracle.gate_mlp(x, g1.T, c1, g2, c2)
