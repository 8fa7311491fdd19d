"""GPU parity of the two perceptrons of the hybrid layer ("VideoNSA: Native
Sparse Attention Scales Video Understanding", paper notes, section "Method":
the compression branch's learnable MLP and the two-layer MLP behind the
per-head sigmoid gates) against the oracle.

Gate MLP: the tensor-core kernel (bf16, d_model a multiple of 64, hidden in
{64, 128, 192, 256}) on token counts that are not a multiple of its 128-token
tile, with the pages' model width (28 heads x 128 = 3,584) and smaller ones,
and the SIMT kernel (other widths, fp32).  Both sides round the hidden layer to
bf16 in bf16 runs; they can still round a hidden value h_a to neighbouring bf16
values where the fp32 and the fp64 pre-activation straddle a rounding midpoint,
which moves logit o by at most one bf16 ulp of h_a times |g2[a][o]| (ulp <=
2^-7 |h_a|).  So in bf16 each logit must agree within 1e-4 plus two such flips
of its largest term, and at most 5 % of the logits may differ by more than 1e-4
(flips are rare); in fp32 (no rounding) within 1e-4.

Compression MLP: K_cmp / V_cmp and the whole layer (every row) with the
perceptron, on the tensor-core path and the SIMT path, and a decode stream;
then the two perceptrons chained: the GPU's gate logits (checked against the
oracle's) fed to the layer with the compression perceptron, against the oracle
layer on the same logits.
"""
import numpy as np
import pytest

import oracle
from parity_util import compare_layer, compare_pool
from sparse_attention_long_block_b200.inputs import (Workload, cmp_mlp_weights, gate_mlp_inputs,
                                                     generate)

pytestmark = pytest.mark.gpu

GATE_TOL = {"fp32": 1e-4}


def gate_tolerance(g, dtype):
    """Per-logit bound [n][n_out]: 1e-4, plus in bf16 two one-ulp flips of the
    largest hidden term, 2 * max_a 2^-7 |h_a| |g2[a][o]| (h from the oracle
    itself: the logits of an identity second layer)."""
    if dtype != "bf16":
        return GATE_TOL["fp32"]
    hid = g["c1"].shape[0]
    h = oracle.gate_mlp(g["x"], g["g1"], g["c1"], np.eye(hid, dtype=np.float32),
                        np.zeros(hid, np.float32), round_hidden_bf16=True)
    g2 = np.abs(g["g2"].astype(np.float64))
    big = np.empty((h.shape[0], g2.shape[1]))
    for t0 in range(0, h.shape[0], 256):
        big[t0:t0 + 256] = (np.abs(h[t0:t0 + 256])[:, :, None] * g2[None]).max(axis=1)
    return 1e-4 + 2 * 2.0 ** -7 * big


def _gpu_gate(wl, g):
    import torch
    from sparse_attention_long_block_b200 import binding
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dev = "cuda"
    t = {k: torch.from_numpy(v).to(dev, td if k in ("x", "g1", "g2") else torch.float32)
         .contiguous() for k, v in g.items()}
    rng = np.random.default_rng(0)
    w = rng.standard_normal((wl.d, wl.d)).astype(np.float32)
    layer = binding.Layer(n_max=max(wl.n, 1), h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(w),
                          w_v=torch.from_numpy(w), dtype=wl.dtype)
    out = layer.gate_mlp(t["x"], t["g1"], t["c1"], t["g2"], t["c2"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    launches = layer.launches()
    layer.close()
    return out.cpu().numpy(), launches


@pytest.mark.parametrize("dtype,n,dm,hidden,h_q", [
    ("bf16", 1000, 3584, 256, 28),   # tensor cores, the pages' model width
    ("bf16", 129, 512, 64, 28),      # tensor cores, one full tile + 1 token
    ("bf16", 300, 192, 128, 28),     # tensor cores
    ("bf16", 257, 256, 192, 8),      # tensor cores, 24 logits
    ("bf16", 1, 3584, 256, 28),      # a single token
    ("bf16", 150, 200, 100, 28),     # SIMT: width and hidden off the tensor-core grid
    ("fp32", 90, 130, 48, 4),        # SIMT, fp32
])
def test_gate_mlp_matches_oracle(dtype, n, dm, hidden, h_q):
    wl = Workload("gate", n, 0, h_q=h_q, h_kv=h_q // 7 if h_q % 7 == 0 else 1, dtype=dtype)
    g = gate_mlp_inputs(wl, dm, hidden, n=n, seed=300 + n)
    got, launches = _gpu_gate(wl, g)
    ref = oracle.gate_mlp(g["x"], g["g1"], g["c1"], g["g2"], g["c2"],
                          round_hidden_bf16=(dtype == "bf16"))
    assert got.shape == (n, h_q, 3)
    err = np.abs(got.reshape(n, -1) - ref)
    assert launches == 1
    assert np.isfinite(got).all()
    assert (err <= gate_tolerance(g, dtype)).all(), (err.max(),
                                                     np.unravel_index(err.argmax(), err.shape))
    if dtype == "bf16":
        assert (err > 1e-4).mean() <= 0.05


@pytest.mark.parametrize("hidden", [128, 512])
def test_cmp_mlp_pool_matches_oracle(hidden):
    wl = Workload("cmlp", 3000, 0, top_k=8, window=128, seed=31)
    x = generate(wl)
    compare_pool(wl, x, cmp_mlp=cmp_mlp_weights(wl, hidden))


@pytest.mark.parametrize("dtype,h_q,h_kv,d", [("bf16", 28, 4, 128), ("fp32", 28, 4, 128),
                                              ("bf16", 4, 1, 64)])
def test_layer_with_cmp_mlp_full(dtype, h_q, h_kv, d):
    wl = Workload("cmlp_layer", 2900, 120, h_q=h_q, h_kv=h_kv, d=d, top_k=10, window=200,
                  dtype=dtype, seed=32)
    x = generate(wl)
    compare_layer(wl, x, cmp_mlp=cmp_mlp_weights(wl, 96 if d == 64 else 128))


def test_decode_with_cmp_mlp():
    from test_gpu_decode import _compare, _stream_mask
    tail = "1" * 70 + "0" * 4 + "1" * 20
    mask = _stream_mask(1400, 30, tail)
    n = len(mask)
    wl = Workload("decode_cmlp", int(mask.sum()), n - int(mask.sum()), top_k=8, window=150)
    x = generate(wl, is_vision=mask)
    _compare(wl, x, n0=n - len(tail), cmp_mlp=cmp_mlp_weights(wl, 128))


def test_gate_mlp_feeds_the_layer():
    # the GPU's gate logits ([n][h_q][3], the layout the layer reads) agree with
    # the oracle's, and the layer with the compression perceptron run on them
    # agrees with the oracle layer on the same logits (selection does not depend
    # on the gates)
    wl = Workload("chain", 2500, 200, top_k=8, window=160, seed=33)
    x = generate(wl)
    g = gate_mlp_inputs(wl, wl.h_q * wl.d, 256, seed=34)
    logits, _ = _gpu_gate(wl, g)
    ref = oracle.gate_mlp(g["x"], g["g1"], g["c1"], g["g2"], g["c2"], round_hidden_bf16=True)
    assert (np.abs(logits.reshape(wl.n, -1) - ref) <= gate_tolerance(g, "bf16")).all()
    x2 = dict(x, gate=np.ascontiguousarray(logits, np.float32))
    compare_layer(wl, x2, cmp_mlp=cmp_mlp_weights(wl, 128), want_branches=False)
