"""GPU parity of the decode step: after a prefill of the first n0 tokens, each
later token is decoded alone (vnsa_decode) and must equal the oracle's row of
the prefill over the whole stream (the definition of a decode step: causal
attention makes row t independent of tokens after t).

Streams mix vision and text tokens and cross block boundaries, so the steps
cover: a text token (dense over the stream), a vision token inside a block, the
vision token that completes a block (its K_cmp / V_cmp are pooled by the step)
and the first token of the next block.  Selections follow the same rule as the
prefill tests: identical block sets, except swaps within 1e-3 relative of the
oracle's k-th importance, where the oracle is rerun on the kernel's selection.
"""
import numpy as np
import pytest

import oracle
from parity_util import TOL, check_selection, oracle_params
from sparse_attention_long_block_b200.inputs import WORKLOADS, Workload, generate

pytestmark = pytest.mark.gpu


def _stream_mask(n_vision, n_text_head, tail):
    """Vision tokens, then n_text_head text tokens after vision rank
    n_vision - len(tail), then `tail` (a 0/1 string) for the decoded tokens."""
    n_tail_v = tail.count("1")
    head_v = n_vision - n_tail_v
    mask = [1] * head_v + [0] * n_text_head + [int(ch) for ch in tail]
    return np.array(mask, np.uint8)


def _run_decode(wl: Workload, x: dict, n0: int, cmp_mlp=None):
    import torch
    from sparse_attention_long_block_b200 import binding
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dev = "cuda"
    q = torch.from_numpy(x["q"]).to(dev, td).contiguous()
    k = torch.from_numpy(x["k"]).to(dev, td).contiguous()
    v = torch.from_numpy(x["v"]).to(dev, td).contiguous()
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    gate = torch.from_numpy(x["gate"]).to(dev)
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]), dtype=wl.dtype)
    if cmp_mlp is not None:
        layer.set_cmp_mlp({nm: torch.from_numpy(a) for nm, a in cmp_mlp.items()})
    layer.forward(q[:n0].contiguous(), k[:n0].contiguous(), v[:n0].contiguous(),
                  isv[:n0].contiguous(), gate[:n0].contiguous())
    outs, sels = [], []
    for t in range(n0, wl.n):
        sel = torch.full((wl.h_kv, wl.top_k), -7, dtype=torch.int32, device=dev)
        o = layer.decode(t + 1, q[t].contiguous(), k, v, isv, gate[t].contiguous(), sel_out=sel)
        outs.append(o)
        sels.append(sel)
    torch.cuda.synchronize()
    status = layer.device_status()
    nv, nt = layer.counts()
    out = torch.stack(outs).float().cpu().numpy()
    sel = torch.stack(sels).cpu().numpy()
    layer.close()
    return out, sel, status, (nv, nt)


def _compare(wl: Workload, x: dict, n0: int, cmp_mlp=None):
    out, sel, status, counts = _run_decode(wl, x, n0, cmp_mlp)
    assert status == 0
    isv = x["is_vision"]
    assert counts == (int(isv.sum()), wl.n - int(isv.sum()))
    rows = np.arange(n0, wl.n, dtype=np.int32)
    p = oracle_params(wl)
    o = oracle.forward(p, x["q"], x["k"], x["v"], isv, x["gate"], x["w_k"], x["w_v"],
                       rows=rows, want=("idx", "imp"), cmp_mlp=cmp_mlp)
    ref = o["out"].copy()
    is_v = isv[rows] != 0
    if is_v.any():
        vis = np.nonzero(isv)[0]
        rank_of = -np.ones(wl.n, np.int64)
        rank_of[vis] = np.arange(len(vis))
        ranks = rank_of[rows[is_v]]
        swapped = check_selection(sel[is_v], o["idx"][is_v], o["imp"][is_v], wl.top_k,
                                  block=wl.block, ranks=ranks)
        if swapped:
            sub = np.nonzero(is_v)[0][swapped]
            fidx = sel[sub]
            o2 = oracle.forward(p, x["q"], x["k"], x["v"], isv, x["gate"], x["w_k"], x["w_v"],
                                rows=rows[sub], forced_idx=fidx, cmp_mlp=cmp_mlp)
            ref[sub] = o2["out"]
    # a text step exports no selection
    assert (sel[~is_v] == -1).all()
    err = float(np.abs(out - ref).max())
    assert np.isfinite(out).all()
    assert err <= TOL[wl.dtype], err
    return err


def test_decode_bf16_mixed_stream():
    # 1,980 vision tokens and 40 text tokens are prefilled; the 96 decoded
    # tokens are text, vision ranks 1980..2027, text, then ranks 2028..2067
    # (rank 2047 completes block 31, the rest open block 32)
    tail = "0" * 3 + "1" * 48 + "0" * 5 + "1" * 40
    mask = _stream_mask(2068, 40, tail)
    n = len(mask)
    wl = Workload("decode_bf16", int(mask.sum()), n - int(mask.sum()), top_k=16, window=256)
    x = generate(wl, is_vision=mask)
    _compare(wl, x, n0=n - len(tail))


def test_decode_fp32_small_heads():
    tail = "1" * 20 + "0" * 4 + "1" * 50
    mask = _stream_mask(700, 12, tail)
    n = len(mask)
    wl = Workload("decode_fp32", int(mask.sum()), n - int(mask.sum()), h_q=4, h_kv=1, d=64,
                  top_k=4, window=128, dtype="fp32")
    x = generate(wl, is_vision=mask)
    _compare(wl, x, n0=n - len(tail))


def test_decode_from_short_prefill_crosses_first_blocks():
    # a prefill of 2 vision tokens, then 140 decoded vision tokens: blocks 0 and
    # 1 complete during decoding, and the first queries have no complete block
    mask = np.ones(142, np.uint8)
    wl = Workload("decode_short", 142, 0, top_k=3, window=32)
    x = generate(wl, is_vision=mask)
    _compare(wl, x, n0=2)


def test_decode_block_36_straddles_tiles():
    # block 36 (6 x 6 patches per frame): decoded vision ranks 1420..1499
    # complete blocks 39 and 40 and open block 41
    tail = "1" * 50 + "0" * 3 + "1" * 30
    mask = _stream_mask(1500, 20, tail)
    n = len(mask)
    wl = Workload("decode_b36", int(mask.sum()), n - int(mask.sum()), top_k=8, window=100,
                  block=36, frame=36)
    x = generate(wl, is_vision=mask)
    _compare(wl, x, n0=n - len(tail))


def test_decode_long_128k_tail():
    base = WORKLOADS["long_128k"]
    # the 128K stream; the last 80 tokens (text, then vision that completes the
    # last block, then text) are decoded after a prefill of the rest
    tail = "0" * 4 + "1" * 60 + "0" * 16
    nv = base.n_vision
    mask = np.concatenate([np.ones(nv - tail.count("1"), np.uint8),
                           np.zeros(base.n_text - tail.count("0"), np.uint8),
                           np.array([int(ch) for ch in tail], np.uint8)])
    wl = base.with_(name="decode_128k")
    x = generate(wl, is_vision=mask)
    _compare(wl, x, n0=wl.n - len(tail))


def test_decode_rejects_a_gap_in_the_stream():
    import torch
    from sparse_attention_long_block_b200 import binding
    wl = Workload("decode_gap", 256, 0, top_k=4, window=64)
    x = generate(wl)
    dev = "cuda"
    q, k, v = (torch.from_numpy(x[nm]).to(dev, torch.bfloat16).contiguous() for nm in ("q", "k", "v"))
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    gate = torch.from_numpy(x["gate"]).to(dev)
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]))
    # no prefill yet
    with pytest.raises(binding.VnsaError):
        layer.decode(10, q[9].contiguous(), k, v, isv, gate[9].contiguous())
    layer.forward(q[:100].contiguous(), k[:100].contiguous(), v[:100].contiguous(),
                  isv[:100].contiguous(), gate[:100].contiguous())
    with pytest.raises(binding.VnsaError):
        layer.decode(102, q[101].contiguous(), k, v, isv, gate[101].contiguous())
    layer.decode(101, q[100].contiguous(), k, v, isv, gate[100].contiguous())
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    layer.close()
