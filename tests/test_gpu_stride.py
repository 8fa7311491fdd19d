"""GPU parity of overlapping compression blocks: a compression stride below the
block size (the native sparse attention design that "VideoNSA: Native Sparse
Attention Scales Video Understanding", paper notes, section "Method", builds
on), with the compression probability mass spread over the selection blocks
by the tokens each compression block puts in them (reading R13 of the
oracle).  Every case is compared with the fp64 oracle: the block keys/values,
then every row of the layer (selection sets within the tie band, branch
outputs, importance, output), on the tensor-core path (bf16, blocks aligned
and not aligned to the 64-key tiles) and the SIMT path (fp32), the
allocation-free selection chain, and a decode step, which takes the plain
stride only.
"""
import ctypes

import numpy as np
import pytest

import oracle
from parity_util import (TOL, check_selection, compare_layer, compare_pool, oracle_params,
                         run_gpu)
from sparse_attention_long_block_b200 import binding
from sparse_attention_long_block_b200.inputs import Workload, generate, interleaved_mask

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("block,stride,dtype", [(64, 32, "bf16"), (64, 16, "fp32"),
                                                (36, 12, "bf16")])
def test_overlapping_block_keys_and_values(block, stride, dtype):
    kw = dict(h_q=4, h_kv=1, d=64) if dtype == "fp32" else {}
    wl = Workload(name="spool", n_vision=1000, n_text=24, top_k=6, window=64, block=block,
                  stride=stride, dtype=dtype, seed=61, **kw)
    compare_pool(wl, generate(wl))


def test_stride_32_block_64_tensor_core_every_row():
    wl = Workload(name="s32", n_vision=2048, n_text=64, top_k=8, window=128, stride=32, seed=62)
    x = generate(wl)
    st = compare_layer(wl, x)
    assert st["rows"] == wl.n


def test_stride_32_block_64_interleaved_text():
    wl = Workload(name="s32i", n_vision=1536, n_text=96, top_k=8, window=100, stride=32, seed=63)
    x = generate(wl, interleaved_mask(wl.n_vision, wl.n_text, seed=4, text_runs=3))
    compare_layer(wl, x)


def test_stride_12_block_36_unaligned_tiles():
    wl = Workload(name="s12", n_vision=1800, n_text=40, top_k=10, window=90, block=36, stride=12,
                  seed=64)
    compare_layer(wl, generate(wl))


def test_stride_16_block_64_fp32_simt():
    wl = Workload(name="s16f", n_vision=1024, n_text=0, h_q=4, h_kv=1, d=64, top_k=4,
                  window=128, dtype="fp32", stride=16, seed=65)
    compare_layer(wl, generate(wl))


def test_stride_selection_without_allocation():
    import torch
    wl = Workload(name="s32n", n_vision=1200, n_text=30, top_k=6, window=64, stride=32, seed=66)
    x = generate(wl)
    td = torch.bfloat16
    dev = "cuda"
    q, k, v = (torch.from_numpy(x[nm]).to(dev, td) for nm in ("q", "k", "v"))
    isv = torch.from_numpy(x["is_vision"]).to(dev)
    w_k = torch.from_numpy(x["w_k"]).to(dev, td)
    w_v = torch.from_numpy(x["w_v"]).to(dev, td)
    o_cmp = torch.zeros((wl.n, wl.h_q, wl.d), dtype=torch.float32, device=dev)
    idx = torch.full((wl.h_kv, wl.n, wl.top_k), -7, dtype=torch.int32, device=dev)
    cfg = binding.vnsa_config(wl.n, wl.h_q, wl.h_kv, wl.d, wl.block, wl.top_k, wl.window, 1, 1,
                              0.0, binding.VNSA_BF16, wl.stride)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    binding.vnsa_select_noalloc(cfg, wl.n, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                isv.data_ptr(), w_k.data_ptr(), w_v.data_ptr(),
                                o_cmp.data_ptr(), idx.data_ptr(), stream)
    assert binding.vnsa_select_noalloc_status(stream) == 0
    nv = wl.n_vision
    rows = np.nonzero(x["is_vision"])[0].astype(np.int32)
    o = oracle.forward(oracle_params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], rows=rows, want=("o_cmp", "idx", "imp"))
    assert np.abs(o_cmp.cpu().numpy()[:nv] - o["o_cmp"]).max() <= TOL["bf16"]
    check_selection(np.transpose(idx.cpu().numpy()[:, :nv], (1, 0, 2)), o["idx"], o["imp"],
                    wl.top_k, block=wl.block, ranks=np.arange(nv))


def test_decode_takes_the_plain_stride_only():
    import torch
    wl = Workload(name="s32d", n_vision=300, n_text=4, top_k=4, window=64, stride=32, seed=67)
    x = generate(wl)
    layer = binding.Layer(n_max=wl.n, h_q=wl.h_q, h_kv=wl.h_kv, d=wl.d, block=wl.block,
                          top_k=wl.top_k, window=wl.window, w_k=torch.from_numpy(x["w_k"]),
                          w_v=torch.from_numpy(x["w_v"]), stride=wl.stride)
    t = {nm: torch.from_numpy(x[nm]).to("cuda", torch.bfloat16) for nm in ("q", "k", "v")}
    isv = torch.from_numpy(x["is_vision"]).to("cuda")
    gate = torch.from_numpy(x["gate"]).to("cuda")
    n0 = wl.n - 1
    layer.forward(t["q"][:n0].contiguous(), t["k"][:n0].contiguous(), t["v"][:n0].contiguous(),
                  isv[:n0].contiguous(), gate[:n0].contiguous())
    with pytest.raises(binding.VnsaError) as e:
        layer.decode(wl.n, t["q"][n0].contiguous(), t["k"], t["v"], isv, gate[n0].contiguous())
    assert e.value.code == binding.VNSA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    layer.close()
