"""Seeded synthetic inputs for the hybrid layer prefill.

This module is shared by the tests, the benchmark and the oracle runs.  It holds
no arithmetic of the method itself: it only draws random tensors, rounds them to
the storage precision and lays them out.

The workloads mirror the shapes the VideoNSA pages describe (Qwen2.5-VL-7B
layer: 28 query heads, 4 KV heads, head dim 128; 64 tokens per frame; contexts
from 8K to the 36K training length and on to 128K), with video replaced by a
frame-mean model because no video data or trained weights are available:

* For each of Q, K and V separately, every frame f (64 vision tokens, or
  ``frame`` tokens: the pages call tokens per frame a task knob, and the
  block-size workloads match the compression block to it) and every head has a
  mean m_f ~ N(0, I_d); each vision token is m_f + N(0, 0.5 I_d).
  With ``ar1`` (the 128K workload) the K and V frame means drift:
  m_f = 0.9 m_{f-1} + sqrt(0.19) eps_f, which keeps their variance at 1.
* A text token is its own N(0, I_d) mean plus N(0, 0.5 I_d) noise.
* Gate logits are N(0, 1) per token, query head and branch (cmp, slc, swa).
* The compression projections W_K, W_V are N(0, 1/d) entries.
* Draw order: Q, K, V, gate logits, W_K, W_V from ``numpy.random.default_rng``.
* bf16 workloads round every tensor (Q, K, V, W_K, W_V) to bf16 with
  round-to-nearest-even; values are kept as float32 arrays holding exact bf16
  values, so the GPU and the oracle read identical numbers.
* Vision tokens come first and text tokens follow, unless a mask is given.
* ``dense`` workloads (Dense-NSA: the same tokens under full causal attention)
  draw the same tensors and mark every token as text, so every query attends
  to all earlier tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

FRAME = 64  # vision tokens per frame (= compression block) unless a workload sets its own


@dataclass(frozen=True)
class Workload:
    name: str
    n_vision: int
    n_text: int
    h_q: int = 28
    h_kv: int = 4
    d: int = 128
    top_k: int = 16
    window: int = 256
    dtype: str = "bf16"          # "bf16" or "fp32"
    ar1: bool = False            # AR(1) drift of K/V frame means
    seed: int = 0
    block: int = 64
    stride: int = 0              # compression stride (0: the block; below it blocks overlap)
    dense: bool = False          # Dense-NSA: every token attends densely (no vision set)
    frame: int = FRAME           # vision tokens per frame of the frame-mean model

    @property
    def n(self) -> int:
        return self.n_vision + self.n_text

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # Tiny fp32, NSA only: 16 frames, 4/1 heads, d 64, top-4, window 128.
    "tiny_fp32_1k": Workload("tiny_fp32_1k", 1024, 0, h_q=4, h_kv=1, d=64, top_k=4,
                             window=128, dtype="fp32"),
    # Qwen2.5-VL-7B layer shape: 128 frames + 256 text tokens.
    "qwen_8k": Workload("qwen_8k", 8192, 256, top_k=16, window=256),
    # Training-length context: 560 frames + 512 text tokens.
    "train_36k": Workload("train_36k", 35840, 512, top_k=16, window=256),
    # 128K context: 2,032 frames + 1,024 text tokens, drifting K/V frame means.
    "long_128k": Workload("long_128k", 130048, 1024, top_k=32, window=512, ar1=True),
    # Global/local budget sweep at 64K tokens.
    "sweep_64k_k8_w1024": Workload("sweep_64k_k8_w1024", 65024, 512, top_k=8, window=1024),
    "sweep_64k_k16_w512": Workload("sweep_64k_k16_w512", 65024, 512, top_k=16, window=512),
    "sweep_64k_k32_w128": Workload("sweep_64k_k32_w128", 65024, 512, top_k=32, window=128),
    # Dense-NSA: the 8K, 36K and 128K token streams under full causal attention.
    "dense_8k": Workload("dense_8k", 8192, 256, top_k=16, window=256, dense=True),
    "dense_36k": Workload("dense_36k", 35840, 512, top_k=16, window=256, dense=True),
    "dense_128k": Workload("dense_128k", 130048, 1024, top_k=32, window=512, ar1=True,
                           dense=True),
    # Tokens per frame as a knob (block = frame size) at the training length,
    # each with the 1,024-token selection budget of top-16 x 64: 16 tokens per
    # frame (top-64), 32 (top-32), 36 (6 x 6 patches, top-28) and 128 (top-8).
    "tpf16_36k": Workload("tpf16_36k", 35840, 512, top_k=64, window=256, block=16, frame=16),
    "tpf32_36k": Workload("tpf32_36k", 35840, 512, top_k=32, window=256, block=32, frame=32),
    "tpf36_36k": Workload("tpf36_36k", 35856, 512, top_k=28, window=256, block=36, frame=36),
    "tpf128_36k": Workload("tpf128_36k", 35840, 512, top_k=8, window=256, block=128,
                           frame=128),
}


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 value (ties to even), in float32."""
    a = np.array(a, dtype=np.float32, copy=True, order="C")
    u = a.view(np.uint32)
    t = u >> np.uint32(16)
    t &= np.uint32(1)
    t += np.uint32(0x7FFF)
    u += t
    u &= np.uint32(0xFFFF0000)
    return a


def _frame_tokens(rng, n_vision, h, d, ar1, frame):
    n_frames = (n_vision + frame - 1) // frame
    means = rng.standard_normal((n_frames, h, d), dtype=np.float32)
    if ar1 and n_frames > 1:
        c = np.float32(np.sqrt(0.19))
        for f in range(1, n_frames):
            means[f] = np.float32(0.9) * means[f - 1] + c * means[f]
    noise = rng.standard_normal((n_vision, h, d), dtype=np.float32)
    noise *= np.float32(np.sqrt(0.5))
    noise += np.repeat(means, frame, axis=0)[:n_vision]
    return noise


def _text_tokens(rng, n_text, h, d):
    m = rng.standard_normal((n_text, h, d), dtype=np.float32)
    e = rng.standard_normal((n_text, h, d), dtype=np.float32)
    return m + np.float32(np.sqrt(0.5)) * e


def generate(wl: Workload, is_vision: np.ndarray | None = None) -> dict:
    """Inputs of one layer prefill.

    Returns numpy arrays: q [n][h_q][d], k, v [n][h_kv][d] (float32 holding the
    storage-precision values), is_vision [n] uint8, gate [n][h_q][3] float32,
    w_k, w_v [d][d].  ``is_vision`` may place the vision tokens anywhere; it
    must hold wl.n_vision ones among wl.n entries.
    """
    n = wl.n
    if wl.dense and is_vision is not None:
        raise ValueError("a dense workload takes no mask")
    if is_vision is None:
        is_vision = np.zeros(n, np.uint8)
        is_vision[: wl.n_vision] = 1
    else:
        is_vision = np.ascontiguousarray(is_vision, dtype=np.uint8)
        if is_vision.shape != (n,) or int(is_vision.sum()) != wl.n_vision:
            raise ValueError("is_vision must have n entries with n_vision ones")
    vis_pos = np.nonzero(is_vision)[0]
    txt_pos = np.nonzero(is_vision == 0)[0]
    rng = np.random.default_rng(wl.seed)
    tensors = {}
    for name, h in (("q", wl.h_q), ("k", wl.h_kv), ("v", wl.h_kv)):
        x = np.empty((n, h, wl.d), np.float32)
        x[vis_pos] = _frame_tokens(rng, wl.n_vision, h, wl.d, wl.ar1 and name != "q", wl.frame)
        x[txt_pos] = _text_tokens(rng, wl.n_text, h, wl.d)
        tensors[name] = x
    gate = rng.standard_normal((n, wl.h_q, 3), dtype=np.float32)
    sd = np.float32(1.0 / np.sqrt(wl.d))
    w_k = rng.standard_normal((wl.d, wl.d), dtype=np.float32) * sd
    w_v = rng.standard_normal((wl.d, wl.d), dtype=np.float32) * sd
    if wl.dtype == "bf16":
        for name in ("q", "k", "v"):
            tensors[name] = bf16_round(tensors[name])
        w_k, w_v = bf16_round(w_k), bf16_round(w_v)
    elif wl.dtype != "fp32":
        raise ValueError(f"unknown dtype {wl.dtype}")
    if wl.dense:
        is_vision = np.zeros(n, np.uint8)
    return dict(q=tensors["q"], k=tensors["k"], v=tensors["v"], is_vision=is_vision,
                gate=gate, w_k=w_k, w_v=w_v)


def cmp_mlp_weights(wl: Workload, hidden: int, seed: int = 100) -> dict:
    """Random weights of the compression perceptron (hidden width `hidden`):
    w1_k, w1_v [d][H] ~ N(0, 1/d), w2_k, w2_v [H][d] ~ N(0, 1/H) (rounded to
    bf16 for bf16 workloads), biases b1 ~ N(0, 0.01), b2 ~ N(0, 0.01) in fp32."""
    rng = np.random.default_rng(seed)
    d = wl.d
    out = {}
    for t in ("k", "v"):
        w1 = rng.standard_normal((d, hidden), dtype=np.float32) * np.float32(1 / np.sqrt(d))
        b1 = rng.standard_normal(hidden, dtype=np.float32) * np.float32(0.1)
        w2 = rng.standard_normal((hidden, d), dtype=np.float32) * np.float32(1 / np.sqrt(hidden))
        b2 = rng.standard_normal(d, dtype=np.float32) * np.float32(0.1)
        if wl.dtype == "bf16":
            w1, w2 = bf16_round(w1), bf16_round(w2)
        out.update({"w1_" + t: w1, "b1_" + t: b1, "w2_" + t: w2, "b2_" + t: b2})
    return out


def gate_mlp_inputs(wl: Workload, d_model: int, hidden: int, n: int | None = None,
                    seed: int = 200) -> dict:
    """Layer input and gate-perceptron weights: x [n][d_model] ~ N(0, 1) (a
    normalised hidden state), g1 [d_model][H] ~ N(0, 1/d_model), c1 [H] ~
    N(0, 0.01), g2 [H][3 h_q] ~ N(0, 1/H), c2 [3 h_q] ~ N(0, 1); x, g1, g2
    rounded to bf16 for bf16 workloads."""
    rng = np.random.default_rng(seed)
    n = wl.n if n is None else n
    x = rng.standard_normal((n, d_model), dtype=np.float32)
    g1 = rng.standard_normal((d_model, hidden), dtype=np.float32) * np.float32(1 / np.sqrt(d_model))
    c1 = rng.standard_normal(hidden, dtype=np.float32) * np.float32(0.1)
    g2 = rng.standard_normal((hidden, 3 * wl.h_q), dtype=np.float32) * np.float32(1 / np.sqrt(hidden))
    c2 = rng.standard_normal(3 * wl.h_q, dtype=np.float32)
    if wl.dtype == "bf16":
        x, g1, g2 = bf16_round(x), bf16_round(g1), bf16_round(g2)
    return dict(x=x, g1=g1, c1=c1, g2=g2, c2=c2)


def interleaved_mask(n_vision: int, n_text: int, seed: int = 1,
                     text_runs: int = 4) -> np.ndarray:
    """A vision/text mask with the text split into runs placed between vision
    tokens (a prompt interleaved with video), for partition tests."""
    rng = np.random.default_rng(seed)
    n = n_vision + n_text
    mask = np.ones(n, np.uint8)
    if n_text == 0:
        return mask
    runs = max(1, min(text_runs, n_text))
    cuts = np.sort(rng.choice(np.arange(1, n_text), size=runs - 1, replace=False)) if runs > 1 else []
    lens = np.diff(np.concatenate([[0], cuts, [n_text]])).astype(int)
    starts = np.sort(rng.choice(np.arange(0, n_vision + 1), size=runs, replace=False))
    out, v_done = [], 0
    for s, ln in zip(starts, lens):
        out.append(np.ones(s - v_done, np.uint8))
        out.append(np.zeros(ln, np.uint8))
        v_done = s
    out.append(np.ones(n_vision - v_done, np.uint8))
    mask = np.concatenate(out)
    assert mask.shape == (n,) and int(mask.sum()) == n_vision
    return mask
