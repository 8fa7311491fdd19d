"""GPU parity: the CUDA layer (through the C ABI) against the fp64 oracle.

Sizes: the tiny fp32 workload and the 8K layer in full; the 36K, 64K and 128K
workloads and the largest call the library takes (262,144 tokens) at their full
size on stratified rows (first rows, every 97th row, both sides of block
boundaries, text rows), in the launch configuration the benchmark times.  Edge cases: ragged vision counts, interleaved masks, no
complete block, text only, vision only, single token, full budgets, forced
blocks off, 4/1 heads with d 64 in bf16 and 28/4 heads in fp32.
"""
import numpy as np
import pytest

from parity_util import compare_layer, compare_pool, run_gpu, stratified_rows
from sparse_attention_long_block_b200.inputs import WORKLOADS, Workload, generate, interleaved_mask

pytestmark = pytest.mark.gpu


def _wl(base, **kw):
    return WORKLOADS[base].with_(**kw) if kw else WORKLOADS[base]


@pytest.mark.parametrize("name", ["tiny_fp32_1k", "qwen_8k"])
def test_pool_projection_matches_oracle(name):
    wl = WORKLOADS[name]
    compare_pool(wl, generate(wl))


def test_tiny_fp32_full():
    wl = WORKLOADS["tiny_fp32_1k"]
    stats = compare_layer(wl, generate(wl))
    assert stats["rows"] == wl.n


def test_qwen_8k_full():
    wl = WORKLOADS["qwen_8k"]
    compare_layer(wl, generate(wl))


@pytest.mark.parametrize("name", ["train_36k", "sweep_64k_k8_w1024", "sweep_64k_k16_w512",
                                  "sweep_64k_k32_w128"])
def test_large_workloads_sampled_rows(name):
    wl = WORKLOADS[name]
    x = generate(wl)
    rows = stratified_rows(x["is_vision"], every=397, max_text=48)
    compare_layer(wl, x, rows=rows, want_branches=False)


def test_long_128k_sampled_rows():
    wl = WORKLOADS["long_128k"]
    x = generate(wl)
    rows = stratified_rows(x["is_vision"], every=1021, first=96, max_text=32)
    compare_layer(wl, x, rows=rows, want_branches=False)


def test_max_tokens_sampled_rows():
    # the largest call the library takes (262,144 tokens: 261,120 vision + 1,024
    # text, 4,080 blocks), the long-context recipe; sampled rows on both sides
    # of block boundaries, the last rows and the text rows
    wl = Workload("max_256k", 261120, 1024, top_k=32, window=512, ar1=True, seed=9)
    assert wl.n == 262144
    x = generate(wl)
    rows = stratified_rows(x["is_vision"], every=4099, first=64, max_text=16)
    compare_layer(wl, x, rows=rows, want_branches=False)


def test_dense_nsa_8k_full():
    """Dense-NSA (every token attends densely; the text path over all tokens)."""
    wl = WORKLOADS["dense_8k"]
    x = generate(wl)
    assert int(x["is_vision"].sum()) == 0
    stats = compare_layer(wl, x, want_branches=False)
    assert stats["rows"] == wl.n


@pytest.mark.parametrize("name,max_text", [("dense_36k", 96), ("dense_128k", 48)])
def test_dense_nsa_sampled_rows(name, max_text):
    wl = WORKLOADS[name]
    x = generate(wl)
    rows = stratified_rows(x["is_vision"], max_text=max_text)
    compare_layer(wl, x, rows=rows, want_branches=False)


EDGE = [
    # ragged: vision count not a multiple of 64, odd text count
    dict(n_vision=1000, n_text=37),
    # fewer vision tokens than one block
    dict(n_vision=50, n_text=20),
    # text only / vision only / a single token
    dict(n_vision=0, n_text=300),
    dict(n_vision=700, n_text=0),
    dict(n_vision=1, n_text=0),
    dict(n_vision=0, n_text=1),
    # budgets covering everything: top-k >= blocks, window >= n
    dict(n_vision=640, n_text=64, top_k=11, window=5000),
    # window of one token
    dict(n_vision=512, n_text=8, window=1),
]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("case", range(len(EDGE)))
def test_edge_cases(case, dtype):
    wl = Workload(name="edge", h_q=28, h_kv=4, d=128, top_k=4, window=96, dtype=dtype,
                  seed=case + 3, **{k: v for k, v in EDGE[case].items()
                                    if k in ("n_vision", "n_text")})
    extra = {k: v for k, v in EDGE[case].items() if k not in ("n_vision", "n_text")}
    wl = wl.with_(**extra)
    compare_layer(wl, generate(wl))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_interleaved_vision_and_text(dtype):
    wl = Workload(name="inter", n_vision=1500, n_text=140, top_k=6, window=200, dtype=dtype,
                  seed=21)
    mask = interleaved_mask(1500, 140, seed=3, text_runs=6)
    compare_layer(wl, generate(wl, mask))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_small_heads_d64(dtype):
    wl = Workload(name="h4", n_vision=1344, n_text=100, h_q=4, h_kv=1, d=64, top_k=5,
                  window=160, dtype=dtype, seed=22)
    compare_layer(wl, generate(wl))


def test_forced_blocks_off_via_selection_override():
    """A caller-supplied selection replaces the top-k; compare with the oracle
    given the same selection (here: only the query's own block)."""
    import oracle
    from parity_util import oracle_params
    wl = Workload(name="forced", n_vision=768, n_text=32, top_k=3, window=64, seed=23)
    x = generate(wl)
    nv = wl.n_vision
    fidx = np.full((wl.h_kv, wl.n, wl.top_k), -1, np.int32)
    fidx[:, :nv, 0] = (np.arange(nv) // 64)[None, :]
    fidx[:, :nv, 1] = np.where(np.arange(nv) // 64 >= 2, 1, -1)[None, :]
    fidx = np.sort(np.where(fidx < 0, 1 << 30, fidx), axis=-1)
    fidx = np.where(fidx == 1 << 30, -1, fidx).astype(np.int32)
    g = run_gpu(wl, x, want=("o_slc",), forced_idx=fidx)
    assert g["status"] == 0
    rows = np.arange(wl.n)
    ranks = np.concatenate([np.arange(nv), -np.ones(wl.n - nv, int)])
    oi = np.transpose(fidx[:, np.maximum(ranks, 0), :], (1, 0, 2)).copy()
    oi[ranks < 0] = -1
    o = oracle.forward(oracle_params(wl), x["q"], x["k"], x["v"], x["is_vision"], x["gate"],
                       x["w_k"], x["w_v"], rows=rows, forced_idx=oi, want=("o_slc",))
    assert np.abs(g["out"] - o["out"]).max() <= 2e-2
    assert np.abs(g["o_slc"][:nv] - o["o_slc"][:nv]).max() <= 2e-2


def test_repeat_calls_are_deterministic_and_launch_count_stable():
    wl = Workload(name="rep", n_vision=2048, n_text=64, top_k=8, window=128, seed=24)
    x = generate(wl)
    a = run_gpu(wl, x)
    b = run_gpu(wl, x)
    assert np.array_equal(a["out"], b["out"])
    assert a["launches"] == b["launches"] and a["launches"] >= 5
