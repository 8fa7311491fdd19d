"""vnsa_forward inside a CUDA graph: the call allocates nothing and never
synchronises, so a caller can capture one layer prefill on its stream and
replay it; a replay recomputes the layer from whatever the captured input
buffers hold.  The replayed output equals the eager call bit for bit (the
kernels are deterministic), before and after new inputs are copied into the
captured buffers, and the oracle agrees with the replay on the new inputs.
"""
import numpy as np
import pytest

from parity_util import TOL, compare_layer
from sparse_attention_long_block_b200.inputs import Workload, generate

pytestmark = pytest.mark.gpu


def test_forward_replays_from_a_cuda_graph():
    import torch
    from sparse_attention_long_block_b200 import binding
    wl = Workload("graph", 3000, 200, top_k=8, window=160, seed=51)
    x = generate(wl)
    x2 = generate(wl.with_(seed=52))
    dev = "cuda"
    bf = torch.bfloat16
    q, k, v = (torch.from_numpy(x[nm]).to(dev, bf).contiguous() for nm in ("q", "k", "v"))
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    gate = torch.from_numpy(x["gate"]).to(dev)
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]))
    eager = layer.forward(q, k, v, isv, gate).clone()
    out = torch.empty_like(q)
    layer.forward(q, k, v, isv, gate, out=out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(q, k, v, isv, gate, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(out, eager)
    # new inputs in the captured buffers
    for nm, t in (("q", q), ("k", k), ("v", v)):
        t.copy_(torch.from_numpy(x2[nm]).to(dev, bf))
    gate.copy_(torch.from_numpy(x2["gate"]).to(dev))
    g.replay()
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    replayed = out.float().cpu().numpy()
    eager2 = layer.forward(q, k, v, isv, gate).float().cpu().numpy()
    assert np.array_equal(replayed, eager2)
    del g
    layer.close()
    # and the replayed result is the layer on the new inputs (oracle parity)
    stats = compare_layer(wl.with_(seed=52), x2, want_branches=False)
    assert stats["out_max_abs"] <= TOL["bf16"]
