"""The seeded synthetic inputs follow the recipe the design notes state: per
frame and head a mean m_f ~ N(0, I) and tokens m_f + N(0, 0.5 I); with AR(1)
drift (the 128K workload) K/V frame means m_f = 0.9 m_{f-1} + sqrt(0.19) eps,
variance 1 and lag-1 correlation 0.9, while Q frame means stay independent;
text tokens N(0, I) + N(0, 0.5 I); gate logits N(0, 1); W ~ N(0, 1/d);
vision tokens first; bf16 workloads hold exact bf16 values; a seed fixes
every tensor."""
import numpy as np

from sparse_attention_long_block_b200.inputs import Workload, bf16_round, generate


def _frames(x, nv, frame):
    f = x[:nv].reshape(nv // frame, frame, *x.shape[1:])
    return f.mean(axis=1), f - f.mean(axis=1, keepdims=True)


def test_frame_mean_model_moments():
    wl = Workload("recipe", 512 * 64, 256, h_q=4, h_kv=2, d=64, dtype="fp32", seed=11)
    x = generate(wl)
    nv = wl.n_vision
    for name in ("q", "k", "v"):
        means, noise = _frames(x[name], nv, 64)
        # frame-mean variance 1 (+ 0.5/64 from the noise average), noise 0.5 (x 63/64)
        assert abs(means.var() - (1 + 0.5 / 64)) < 0.05, name
        assert abs(noise.var() - 0.5 * 63 / 64) < 0.01, name
        # frames are independent without AR(1)
        m = means.reshape(means.shape[0], -1)
        c = np.mean(np.sum(m[1:] * m[:-1], axis=1) / np.sum(m * m, axis=1).mean())
        assert abs(c) < 0.05, name
    txt = x["q"][nv:]
    assert abs(txt.var() - 1.5) < 0.05
    assert abs(x["gate"].var() - 1.0) < 0.05 and abs(x["gate"].mean()) < 0.02
    assert abs(x["w_k"].var() * wl.d - 1.0) < 0.1 and abs(x["w_v"].var() * wl.d - 1.0) < 0.1
    assert x["is_vision"][:nv].all() and not x["is_vision"][nv:].any()


def test_ar1_drift_of_key_and_value_frame_means():
    wl = Workload("recipe_ar1", 512 * 64, 0, h_q=4, h_kv=2, d=64, dtype="fp32", ar1=True, seed=12)
    x = generate(wl)
    for name, corr in (("k", 0.9), ("v", 0.9), ("q", 0.0)):
        means, _ = _frames(x[name], wl.n_vision, 64)
        m = means[32:]  # past the start-up of the recursion
        assert abs(m.var() - 1.0) < 0.15, name
        a = m[1:].reshape(len(m) - 1, -1)
        b = m[:-1].reshape(len(m) - 1, -1)
        c = float(np.sum(a * b) / np.sqrt(np.sum(a * a) * np.sum(b * b)))
        assert abs(c - corr) < 0.05, (name, c)


def test_bf16_workloads_hold_exact_bf16_values_and_seed_fixes_tensors():
    wl = Workload("recipe_bf16", 8 * 64, 32, h_q=8, h_kv=2, d=64, seed=13)
    x, y = generate(wl), generate(wl)
    for name in ("q", "k", "v", "w_k", "w_v"):
        assert np.array_equal(x[name], bf16_round(x[name].copy())), name
        assert np.array_equal(x[name], y[name]), name
    z = generate(wl.with_(seed=14))
    assert not np.array_equal(x["q"], z["q"])
