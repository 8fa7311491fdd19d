"""GPU parity with compression/selection block sizes other than 64.

The VideoNSA pages match the block to the tokens per frame and call tokens per
frame a task-dependent knob (the pages' findings on tokens per frame against
number of frames), so the layer takes any block size B >= 1 (stride = B,
selection block = compression block).  The frame-mean inputs use B tokens per
frame.

The selection kernel works on 64-key tiles of vision ranks, so the cases cover
every way a block can sit on that grid: several blocks per tile (B = 1, 16,
32), blocks straddling tile edges (B = 36, 100), several tiles per block
(B = 128, 256), plus B = 64's neighbours through the SIMT kernels (fp32, and
bf16 with 2 query heads per KV head).  Sizes span several tiles and end on a
ragged block; the full comparison checks every row against the oracle, the
36K workloads check sampled rows at full size.
"""
import numpy as np
import pytest

from parity_util import compare_layer, compare_pool, stratified_rows
from sparse_attention_long_block_b200.inputs import WORKLOADS, Workload, generate, interleaved_mask

pytestmark = pytest.mark.gpu

# (block, top_k, vision tokens, text tokens)
CASES = [
    (1, 40, 700, 20),
    (16, 24, 2900, 70),
    (32, 12, 3000, 100),
    (36, 10, 2950, 64),
    (100, 5, 3010, 40),
    (128, 4, 3100, 90),
    (256, 3, 3300, 50),
]


def _wl(block, top_k, nv, nt, **kw):
    return Workload(f"b{block}", nv, nt, top_k=top_k, window=160, block=block, frame=block,
                    seed=40 + block, **kw)


@pytest.mark.parametrize("block,top_k,nv,nt", CASES)
def test_block_size_full(block, top_k, nv, nt):
    wl = _wl(block, top_k, nv, nt)
    compare_layer(wl, generate(wl))


@pytest.mark.parametrize("block", [36, 128])
def test_block_size_pool_projection(block):
    wl = _wl(block, 4, 2000, 0)
    compare_pool(wl, generate(wl))


def test_block_size_interleaved_text():
    # vision tokens not in one run: the selection tiles read the gathered
    # vision-order copies of K and V
    wl = _wl(36, 8, 2500, 300)
    x = generate(wl, is_vision=interleaved_mask(wl.n_vision, wl.n_text, seed=5))
    compare_layer(wl, x)


@pytest.mark.parametrize("dtype,h_q,h_kv,d", [("fp32", 28, 4, 128), ("bf16", 8, 4, 128),
                                              ("bf16", 4, 1, 64)])
def test_block_size_simt_kernels(dtype, h_q, h_kv, d):
    # settings outside the tensor-core path (fp32; fewer than 4 query heads per
    # KV head; d = 64) with a block of 32
    wl = _wl(32, 6, 1500, 60, dtype=dtype, h_q=h_q, h_kv=h_kv, d=d)
    compare_layer(wl, generate(wl))


@pytest.mark.parametrize("name", ["tpf16_36k", "tpf32_36k", "tpf36_36k", "tpf128_36k"])
def test_block_size_36k_sampled_rows(name):
    wl = WORKLOADS[name]
    x = generate(wl)
    rows = stratified_rows(x["is_vision"], block=wl.block, every=331, max_text=32)
    compare_layer(wl, x, rows=rows, want_branches=False)


def test_bf16_two_heads_per_group_block_64():
    # 2 query heads per KV head puts 64 queries in a 128-row tile, more than the
    # tensor-core selection masks hold: these layers run on the SIMT kernels
    wl = Workload("r2", 2100, 80, h_q=8, h_kv=4, top_k=6, window=200, seed=9)
    compare_layer(wl, generate(wl))
