"""The C ABI on the host: the library loads, exports every symbol include/vnsa.h
declares, and rejects bad configurations before touching a device."""
import ctypes
import os
import re

import pytest

from sparse_attention_long_block_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "vnsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(vnsa_[a-z_]+)\s*\(", text)))


def cfg(**kw):
    base = dict(n_max=8448, h_q=28, h_kv=4, d=128, block=64, top_k=16, window=256,
                force_first=1, force_local=1, scale=0.0, dtype=binding.VNSA_BF16)
    base.update(kw)
    return binding.vnsa_config(**base)


def test_library_exports_every_declared_symbol():
    lib = binding.load()
    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(binding.EXPORTED) == names


def test_status_and_stage_strings():
    assert binding.status_string(0) == "ok"
    assert "invalid" in binding.status_string(1)
    assert binding.status_string(99) == "unknown status"
    assert [binding.stage_name(i) for i in range(binding.NUM_STAGES)] == [
        "partition", "pool", "cmp", "topk", "slc", "swa", "text"]
    assert binding.stage_name(7) is None


def test_workspace_bytes_valid_config():
    b = binding.vnsa_workspace_bytes(cfg())
    # imp alone is [h_kv][n_max][nb] fp32
    assert b > 4 * 8448 * (8448 // 64) * 4


@pytest.mark.parametrize("block", [1, 16, 32, 36, 100, 128, 256])
def test_any_block_size_is_accepted(block):
    # tokens per frame is a knob: every block size >= 1 is a valid layer, and
    # the importance workspace [h_kv][n_max][n_max / block] grows as it shrinks
    b = binding.vnsa_workspace_bytes(cfg(block=block))
    assert b >= 4 * 8448 * (8448 // block) * 4


@pytest.mark.parametrize("bad,code", [
    (dict(h_q=28, h_kv=3), binding.VNSA_ERR_INVALID_ARG),
    (dict(top_k=1), binding.VNSA_ERR_INVALID_ARG),
    (dict(window=0), binding.VNSA_ERR_INVALID_ARG),
    (dict(n_max=0), binding.VNSA_ERR_INVALID_ARG),
    (dict(force_first=2), binding.VNSA_ERR_INVALID_ARG),
    (dict(scale=-1.0), binding.VNSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.VNSA_ERR_INVALID_ARG),
    (dict(dtype=7), binding.VNSA_ERR_INVALID_ARG),
    (dict(d=96), binding.VNSA_ERR_UNSUPPORTED),
    (dict(block=0), binding.VNSA_ERR_INVALID_ARG),
    (dict(top_k=65), binding.VNSA_ERR_UNSUPPORTED),
    (dict(n_max=262145), binding.VNSA_ERR_UNSUPPORTED),
    (dict(h_q=34, h_kv=2), binding.VNSA_ERR_UNSUPPORTED),
])
def test_bad_configs_rejected_on_host(bad, code):
    with pytest.raises(binding.VnsaError) as e:
        binding.vnsa_workspace_bytes(cfg(**bad))
    assert e.value.code == code


def test_create_rejects_null_weights_and_handles_missing_device():
    lib = binding.load()
    h = ctypes.c_void_p(0)
    c = cfg()
    rc = lib.vnsa_create(ctypes.byref(c), None, None, ctypes.byref(h))
    assert rc == binding.VNSA_ERR_INVALID_ARG and not h.value
    import torch
    if not torch.cuda.is_available():
        fake = ctypes.c_void_p(4096)  # aligned, never dereferenced without a device
        rc = lib.vnsa_create(ctypes.byref(c), fake, fake, ctypes.byref(h))
        assert rc == binding.VNSA_ERR_NO_DEVICE and not h.value


def test_forward_rejects_null_handle_and_bad_n():
    lib = binding.load()
    rc = lib.vnsa_forward(None, 10, None, None, None, None, None, None, None, None)
    assert rc == binding.VNSA_ERR_INVALID_ARG
    rc = lib.vnsa_destroy(None)
    assert rc == binding.VNSA_ERR_INVALID_ARG


def test_perceptron_entry_points_reject_null_handle():
    lib = binding.load()
    p = ctypes.c_void_p(4096)
    rc = lib.vnsa_set_cmp_mlp(None, 16, p, p, p, p, p, p, p, p)
    assert rc == binding.VNSA_ERR_INVALID_ARG
    rc = lib.vnsa_gate_mlp(None, 8, 64, 16, p, p, p, p, p, p, None)
    assert rc == binding.VNSA_ERR_INVALID_ARG
    rc = lib.vnsa_decode(None, 2, p, p, p, p, p, p, None, None)
    assert rc == binding.VNSA_ERR_INVALID_ARG


def test_streamed_host_calls_reject_null_handle_and_unissued_tickets():
    lib = binding.load()
    p = ctypes.c_void_p(4096)
    t = ctypes.c_ulonglong(7)
    rc = lib.vnsa_forward_host_async(None, 10, p, p, p, p, p, p, None, ctypes.byref(t))
    assert rc == binding.VNSA_ERR_INVALID_ARG and t.value == 7
    assert lib.vnsa_host_wait(None, 0) == binding.VNSA_ERR_INVALID_ARG
    assert lib.vnsa_host_join(None, None) == binding.VNSA_ERR_INVALID_ARG


def test_new_knobs_reject_null_handle_and_noalloc_rejects_bad_config_on_host():
    lib = binding.load()
    assert lib.vnsa_set_wait_limit(None, 5) == binding.VNSA_ERR_INVALID_ARG
    out = ctypes.c_int(-1)
    assert lib.vnsa_get_path(None, ctypes.byref(out)) == binding.VNSA_ERR_INVALID_ARG
    assert lib.vnsa_select_noalloc_status(None, None) == binding.VNSA_ERR_INVALID_ARG
    # the allocation-free selection checks its config exactly as vnsa_create
    # does (n standing in for n_max), before touching a device
    p = ctypes.c_void_p(4096)
    for bad, code in ((dict(d=96), binding.VNSA_ERR_UNSUPPORTED),
                      (dict(top_k=65), binding.VNSA_ERR_UNSUPPORTED),
                      (dict(window=0), binding.VNSA_ERR_INVALID_ARG),
                      (dict(h_q=28, h_kv=3), binding.VNSA_ERR_INVALID_ARG)):
        c = cfg(**bad)
        rc = lib.vnsa_select_noalloc(ctypes.byref(c), 64, p, p, p, p, p, p, p, p, None)
        assert rc == code, bad
    c = cfg()
    rc = lib.vnsa_select_noalloc(ctypes.byref(c), 262145, p, p, p, p, p, p, p, p, None)
    assert rc == binding.VNSA_ERR_UNSUPPORTED


@pytest.mark.parametrize("stride,code", [(-1, binding.VNSA_ERR_INVALID_ARG),
                                         (65, binding.VNSA_ERR_INVALID_ARG)])
def test_compression_stride_beyond_the_block_is_rejected(stride, code):
    with pytest.raises(binding.VnsaError) as e:
        binding.vnsa_workspace_bytes(cfg(cmp_stride=stride))
    assert e.value.code == code


def test_overlapping_compression_blocks_grow_the_workspace():
    # stride 16 under block 64: four times the compression blocks, plus a
    # selection-importance buffer of its own
    plain = binding.vnsa_workspace_bytes(cfg())
    assert binding.vnsa_workspace_bytes(cfg(cmp_stride=64)) == plain
    assert binding.vnsa_workspace_bytes(cfg(cmp_stride=16)) > plain + 3 * 4 * 8448 * 132 * 4
