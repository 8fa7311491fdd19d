"""Streamed layer calls from host memory (vnsa_forward_host_async): each call
copies its inputs to a device staging slot on a copy stream, runs the layer,
and copies its output back on a second copy stream, so the copies of
neighbouring calls overlap the attention in between.  The output of every
call equals vnsa_forward on the same inputs, bit for bit (the kernels are
deterministic), whatever the order in which the calls are waited for, with
token counts that change from call to call, and the oracle agrees with one of
them.
"""
import numpy as np
import pytest

from parity_util import TOL, compare_layer
from sparse_attention_long_block_b200.inputs import Workload, generate

pytestmark = pytest.mark.gpu


def test_streamed_host_calls_equal_device_calls():
    import torch
    from sparse_attention_long_block_b200 import binding
    base = Workload("hoststream", 2560, 128, top_k=8, window=160, seed=61)
    # five calls on one handle: two sizes, distinct inputs
    wls = [base.with_(seed=61 + c, n_vision=2560 if c % 2 == 0 else 1920,
                      n_text=128 if c % 2 == 0 else 64) for c in range(5)]
    xs = [generate(wl) for wl in wls]
    x0 = xs[0]
    layer = binding.Layer(n_max=base.n, h_q=base.h_q, h_kv=base.h_kv, d=base.d,
                          block=base.block, top_k=base.top_k, window=base.window,
                          w_k=torch.from_numpy(x0["w_k"]), w_v=torch.from_numpy(x0["w_v"]))
    bf = torch.bfloat16
    host = []
    for x in xs:
        t = {nm: torch.from_numpy(x[nm]).to(bf).pin_memory() for nm in ("q", "k", "v")}
        t["is_vision"] = torch.from_numpy(x["is_vision"]).pin_memory()
        t["gate"] = torch.from_numpy(x["gate"]).pin_memory()
        t["out"] = torch.full_like(t["q"], float("nan")).pin_memory()
        host.append(t)
    tickets = [layer.forward_host_async(t["q"], t["k"], t["v"], t["is_vision"], t["gate"],
                                        t["out"]) for t in host]
    assert tickets == list(range(5))
    # wait out of order: a later ticket first, then the rest
    layer.wait_host(tickets[3])
    for tk in (0, 1, 2, 4):
        layer.wait_host(tk)
    with pytest.raises(binding.VnsaError):
        layer.wait_host(5)  # not issued
    assert layer.device_status() == 0
    for x, t in zip(xs, host):
        dev = {nm: torch.from_numpy(x[nm]).to("cuda", bf) for nm in ("q", "k", "v")}
        ref = layer.forward(dev["q"], dev["k"], dev["v"],
                            torch.from_numpy(x["is_vision"]).cuda(),
                            torch.from_numpy(x["gate"]).cuda())
        torch.cuda.synchronize()
        assert torch.equal(t["out"], ref.cpu())
    # join: the caller's stream waits for every output copy
    tk = layer.forward_host_async(host[1]["q"], host[1]["k"], host[1]["v"],
                                  host[1]["is_vision"], host[1]["gate"], host[0]["out"])
    assert tk == 5
    layer.join_host()
    torch.cuda.current_stream().synchronize()
    assert torch.equal(host[0]["out"][:wls[1].n], host[1]["out"])
    layer.close()
    got = host[2]["out"].float().numpy()
    stats = compare_layer(wls[2], xs[2], want_branches=False)
    assert stats["out_max_abs"] <= TOL["bf16"]
    assert np.isfinite(got).all()
