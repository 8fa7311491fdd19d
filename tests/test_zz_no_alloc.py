"""vnsa_select_noalloc: block selection for callers that cannot allocate
device memory (code under stream capture, plugins confined to a host
framework's memory pool, latency-critical paths).  It keeps its intermediates
in a static library array; its outputs must agree with the regular entry
point's (vnsa_forward with the debug exports) on consecutive calls, including
after the array holds a previous, larger call's contents, and with the fp64
oracle.  The device status word of every call must read 0, and the rows past
the vision tokens of both outputs must be left as the caller filled them.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from parity_util import check_selection, oracle_params
from sparse_attention_long_block_b200 import binding
from sparse_attention_long_block_b200.inputs import WORKLOADS, Workload, generate

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def _regular(wl, x, dev):
    """o_cmp / idx / importance from vnsa_forward's debug exports."""
    import torch
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]), dtype=wl.dtype)
    dbg, t = binding.make_debug(wl.n, wl.h_q, wl.h_kv, wl.d, wl.top_k, dtype=td,
                                want=("o_cmp", "idx", "imp"))
    layer.forward(*(torch.from_numpy(x[n]).to(dev, td) for n in ("q", "k", "v")),
                  torch.from_numpy(x["is_vision"]).to(dev), torch.from_numpy(x["gate"]).to(dev),
                  dbg=dbg)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    layer.close()
    return t["o_cmp"].cpu().numpy(), t["idx"].cpu().numpy(), t["imp"].cpu().numpy()


O_SENTINEL = -1234.5
IDX_SENTINEL = -7


def _noalloc(wl, x, dev):
    import torch
    td = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(x[n]).to(dev, td) for n in ("q", "k", "v"))
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    w_k = torch.from_numpy(x["w_k"]).to(dev, td)
    w_v = torch.from_numpy(x["w_v"]).to(dev, td)
    o_cmp = torch.full((wl.n, wl.h_q, wl.d), O_SENTINEL, dtype=torch.float32, device=dev)
    idx = torch.full((wl.h_kv, wl.n, wl.top_k), IDX_SENTINEL, dtype=torch.int32, device=dev)
    cfg = binding.vnsa_config(wl.n, wl.h_q, wl.h_kv, wl.d, wl.block, wl.top_k, wl.window, 1, 1,
                              0.0, binding.VNSA_BF16 if wl.dtype == "bf16" else binding.VNSA_FP32)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    binding.vnsa_select_noalloc(cfg, wl.n, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                isv.data_ptr(), w_k.data_ptr(), w_v.data_ptr(),
                                o_cmp.data_ptr(), idx.data_ptr(), stream)
    assert binding.vnsa_select_noalloc_status(stream) == 0
    torch.cuda.synchronize()
    return o_cmp.cpu().numpy(), idx.cpu().numpy()


def _agree(wl, x, reg, mine):
    o_reg, idx_reg, imp_reg = reg
    o_me, idx_me = mine
    nv = wl.n_vision
    # rows past the vision tokens are the caller's
    assert (o_me[nv:] == O_SENTINEL).all()
    assert (idx_me[:, nv:] == IDX_SENTINEL).all()
    # the regular entry point
    assert np.abs(o_me[:nv] - o_reg[:nv]).max() <= TOL[wl.dtype]
    ranks = np.arange(nv)
    check_selection(np.transpose(idx_me[:, :nv], (1, 0, 2)),
                    np.transpose(idx_reg[:, :nv], (1, 0, 2)),
                    np.transpose(imp_reg[:, :nv], (1, 0, 2)), wl.top_k, block=wl.block,
                    ranks=ranks)
    # the fp64 oracle, on every vision row (sets within the tie band, o_cmp
    # within the workload's tolerance)
    rows = np.nonzero(x["is_vision"])[0].astype(np.int32)
    o = oracle.forward(oracle_params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], rows=rows, want=("o_cmp", "idx", "imp"))
    assert np.abs(o_me[:nv] - o["o_cmp"]).max() <= TOL[wl.dtype]
    check_selection(np.transpose(idx_me[:, :nv], (1, 0, 2)), o["idx"], o["imp"], wl.top_k,
                    block=wl.block, ranks=ranks)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_select_noalloc_matches_regular_entry_point_twice(dtype):
    import torch
    dev = "cuda"
    first = Workload(name="na1", n_vision=2560, n_text=96, top_k=8, window=128, dtype=dtype,
                     seed=31)
    second = Workload(name="na2", n_vision=1000, n_text=37, top_k=6, window=64, dtype=dtype,
                      seed=32)
    for wl in (first, second):  # the second call sees the first call's leftovers
        x = generate(wl)
        _agree(wl, x, _regular(wl, x, dev), _noalloc(wl, x, dev))
    torch.cuda.synchronize()


def test_select_noalloc_tiny_fp32_against_the_oracle():
    """The tiny fp32 workload (1,024 vision tokens, 4/1 heads, d 64, top-4)
    within 1e-4 of the fp64 oracle."""
    wl = WORKLOADS["tiny_fp32_1k"]
    x = generate(wl)
    _agree(wl, x, _regular(wl, x, "cuda"), _noalloc(wl, x, "cuda"))


def test_select_noalloc_rejects_what_vnsa_create_rejects():
    import torch
    buf = torch.zeros(16, device="cuda")
    p = buf.data_ptr()
    for bad, code in (((64, 28, 4, 96, 64, 8, 128), binding.VNSA_ERR_UNSUPPORTED),  # d 96
                      ((64, 28, 4, 128, 64, 80, 128), binding.VNSA_ERR_UNSUPPORTED),  # top-k 80
                      ((64, 28, 4, 128, 64, 8, 0), binding.VNSA_ERR_INVALID_ARG)):  # window 0
        cfg = binding.vnsa_config(*bad, 1, 1, 0.0, binding.VNSA_BF16)
        with pytest.raises(binding.VnsaError) as e:
            binding.vnsa_select_noalloc(cfg, 64, p, p, p, p, p, p, p, p, None)
        assert e.value.code == code
        n_max = cfg.n_max
        with pytest.raises(binding.VnsaError) as e2:
            binding.vnsa_workspace_bytes(cfg)
        assert e2.value.code == code and n_max == 64


def test_select_noalloc_rejects_sizes_beyond_its_scratch():
    import torch
    wl = Workload(name="big", n_vision=16384, n_text=0, top_k=8, window=128)
    cfg = binding.vnsa_config(wl.n, 28, 4, 128, 64, 8, 128, 1, 1, 0.0, binding.VNSA_BF16)
    buf = torch.zeros(16, device="cuda")
    p = buf.data_ptr()
    with pytest.raises(binding.VnsaError) as e:
        binding.vnsa_select_noalloc(cfg, wl.n, p, p, p, p, p, p, p, p, None)
    assert e.value.code == binding.VNSA_ERR_UNSUPPORTED
