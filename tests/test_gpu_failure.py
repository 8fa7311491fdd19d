"""Failure detection on the GPU, in forms that fault or hang nothing.

* A bounded wait that runs out: the handle's wait limit is set to 1 ns, so the
  first wait of the attention kernel that is not already satisfied gives up.
  The kernel's thread blocks stop, drain their own copies and tensor-core
  operations, free their tensor memory and exit; the status word must read
  VNSA_ERR_TIMEOUT.  With the default limit restored, the same handle (after
  its status is read) and a fresh handle must both compute the layer again.
* An index out of range: a caller selection (the debug override of the top-k)
  names a block after the query's own block.  The kernels check every entry
  before using it, skip it and report VNSA_ERR_BOUNDS.
"""
import numpy as np
import pytest

import oracle
from parity_util import TOL, compare_layer, oracle_params
from sparse_attention_long_block_b200 import binding
from sparse_attention_long_block_b200.inputs import Workload, generate

pytestmark = pytest.mark.gpu


def _tensors(wl, x):
    import torch
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    t = {n: torch.from_numpy(x[n]).to("cuda", td).contiguous() for n in ("q", "k", "v")}
    t["is_vision"] = torch.from_numpy(x["is_vision"]).to("cuda")
    t["gate"] = torch.from_numpy(x["gate"]).to("cuda")
    return t


def _layer(wl, x):
    import torch
    return binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                         top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                         w_v=torch.from_numpy(x["w_v"]), dtype=wl.dtype)


def _rows_match_oracle(wl, x, out, rows):
    ref = oracle.forward(oracle_params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                         x["w_k"], x["w_v"], rows=rows)["out"]
    err = float(np.abs(out.float().cpu().numpy()[rows] - ref).max())
    assert err <= TOL[wl.dtype], err


def test_wait_that_runs_out_reports_timeout_and_the_handle_recovers():
    import torch
    wl = Workload(name="timeout", n_vision=4096, n_text=128, top_k=8, window=128, seed=41)
    x = generate(wl)
    t = _tensors(wl, x)
    layer = _layer(wl, x)
    assert layer.path() == "tcgen05"
    layer.set_wait_limit(1)
    layer.forward(t["q"], t["k"], t["v"], t["is_vision"], t["gate"])
    torch.cuda.synchronize()
    assert layer.device_status() == binding.VNSA_ERR_TIMEOUT
    assert layer.device_status() == 0  # read and cleared
    # the default limit again: the same handle computes the layer
    layer.set_wait_limit(0)
    out = layer.forward(t["q"], t["k"], t["v"], t["is_vision"], t["gate"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    rows = np.array([0, 63, 64, 777, 2048, 4095, 4096, 4200, wl.n - 1], np.int32)
    _rows_match_oracle(wl, x, out, rows)
    layer.close()
    # and so does a fresh handle (full parity check on stratified rows)
    compare_layer(wl, x, rows=rows, want_branches=False)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_caller_selection_out_of_range_reports_bounds(dtype):
    import torch
    if dtype == "bf16":
        wl = Workload(name="bounds", n_vision=1024, n_text=32, top_k=4, window=64, seed=42)
    else:
        wl = Workload(name="bounds32", n_vision=512, n_text=16, h_q=4, h_kv=1, d=64, top_k=4,
                      window=64, dtype="fp32", seed=42)
    x = generate(wl)
    t = _tensors(wl, x)
    layer = _layer(wl, x)
    assert layer.path() == ("tcgen05" if dtype == "bf16" else "simt")
    nv = wl.n_vision
    sel = np.full((wl.h_kv, wl.n, wl.top_k), -1, np.int32)
    for i in range(nv):
        own = i // wl.block
        row = sorted({0, own})
        sel[:, i, :len(row)] = row
    i_bad = 100  # own block 1; block 5 lies ahead of the query
    sel[0, i_bad, :3] = [0, 1, 5]
    fidx = torch.from_numpy(sel).to("cuda")
    dbg, _ = binding.make_debug(wl.n, wl.h_q, wl.h_kv, wl.d, wl.top_k, wl.block,
                                forced_idx=fidx)
    layer.forward(t["q"], t["k"], t["v"], t["is_vision"], t["gate"], dbg=dbg)
    torch.cuda.synchronize()
    assert layer.device_status() == binding.VNSA_ERR_BOUNDS
    # a well-formed call afterwards is clean
    out = layer.forward(t["q"], t["k"], t["v"], t["is_vision"], t["gate"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    _rows_match_oracle(wl, x, out, np.array([0, 100, 511, wl.n - 1], np.int32))
    layer.close()
