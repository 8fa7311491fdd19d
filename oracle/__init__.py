"""fp64 CPU oracle of the VideoNSA hybrid sparse-attention layer prefill.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
loads it, and it imports nothing from the library: the two share no code.  The
only thing they share is the seeded input generator, which holds none of the
method's arithmetic.

``vnsa_oracle.c`` holds the arithmetic (plain loops in fp64, OpenMP over query
rows); this module compiles it with gcc on first use and wraps it with ctypes.
``brute.py`` is a second, pure-Python implementation for tiny inputs.

Every function below follows "VideoNSA: Native Sparse Attention Scales Video
Understanding" (paper notes), section "Method", with the readings listed at the
top of ``vnsa_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vnsa_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libvnsa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile vnsa_oracle.c into a shared library (portable flags, no -march)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O3", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Cfg(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int), ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int),
                ("d", ctypes.c_int), ("block", ctypes.c_int), ("top_k", ctypes.c_int),
                ("window", ctypes.c_int), ("force_first", ctypes.c_int),
                ("force_local", ctypes.c_int), ("scale", ctypes.c_double),
                ("round_cmp_bf16", ctypes.c_int), ("stride", ctypes.c_int)]


class _CmpMLP(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int)] + [
        (nm, ctypes.c_void_p) for nm in ("w1_k", "b1_k", "w2_k", "b2_k",
                                         "w1_v", "b1_v", "w2_v", "b2_v")]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        p = ctypes.c_void_p
        lib.vnsa_oracle_forward.restype = ctypes.c_int
        lib.vnsa_oracle_forward.argtypes = [ctypes.POINTER(_Cfg)] + [p] * 7 + [
            ctypes.c_int] + [p] * 10
        lib.vnsa_oracle_pool_proj.restype = ctypes.c_int
        lib.vnsa_oracle_pool_proj.argtypes = [ctypes.POINTER(_Cfg)] + [p] * 7
        lib.vnsa_oracle_forward_mlp.restype = ctypes.c_int
        lib.vnsa_oracle_forward_mlp.argtypes = [ctypes.POINTER(_Cfg)] + [p] * 5 + [
            ctypes.POINTER(_CmpMLP), ctypes.c_int] + [p] * 10
        lib.vnsa_oracle_pool_mlp.restype = ctypes.c_int
        lib.vnsa_oracle_pool_mlp.argtypes = [ctypes.POINTER(_Cfg), p, p, p,
                                             ctypes.POINTER(_CmpMLP), p, p]
        lib.vnsa_oracle_gate_mlp.restype = ctypes.c_int
        lib.vnsa_oracle_gate_mlp.argtypes = [ctypes.c_int] * 4 + [p] * 5 + [ctypes.c_int, p]
        lib.vnsa_oracle_round_bf16.restype = ctypes.c_double
        lib.vnsa_oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.vnsa_oracle_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


@dataclass
class OracleParams:
    """Shape and method parameters (names follow the paper notes' notation)."""
    h_q: int
    h_kv: int
    d: int
    block: int = 64
    top_k: int = 32
    window: int = 256
    force_first: bool = True
    force_local: bool = True
    scale: float | None = None      # None -> 1/sqrt(d)
    round_cmp_bf16: bool = False
    stride: int | None = None       # compression stride (R13); None -> block


def _cfg(p: OracleParams, n: int) -> _Cfg:
    scale = p.scale if p.scale is not None else 1.0 / np.sqrt(p.d)
    return _Cfg(n, p.h_q, p.h_kv, p.d, p.block, p.top_k, p.window,
                int(p.force_first), int(p.force_local), float(scale),
                int(p.round_cmp_bf16), int(p.stride or 0))


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_load().vnsa_oracle_threads())


def round_bf16(x: float) -> float:
    """The oracle's own round-to-nearest-even onto bf16 (fp64 in, fp64 out)."""
    return float(_load().vnsa_oracle_round_bf16(float(x)))


CMP_MLP_KEYS = ("w1_k", "b1_k", "w2_k", "b2_k", "w1_v", "b1_v", "w2_v", "b2_v")


def _cmp_mlp(d: int, mlp: dict):
    """ctypes form of a compression perceptron {"w1_k": [d][H], "b1_k": [H],
    "w2_k": [H][d], "b2_k": [d], and the same for v} plus the arrays it points
    to (kept alive by the caller)."""
    arrs = {nm: _f32(mlp[nm]) for nm in CMP_MLP_KEYS}
    hidden = arrs["b1_k"].shape[0]
    for t in ("k", "v"):
        if (arrs["w1_" + t].shape != (d, hidden) or arrs["b1_" + t].shape != (hidden,)
                or arrs["w2_" + t].shape != (hidden, d) or arrs["b2_" + t].shape != (d,)):
            raise ValueError("compression MLP weights must be [d][H], [H], [H][d], [d]")
    s = _CmpMLP(hidden, *[arrs[nm].ctypes.data for nm in CMP_MLP_KEYS])
    return s, arrs


def pool_proj(p: OracleParams, k, v, is_vision, w_k=None, w_v=None, cmp_mlp=None):
    """K_cmp, V_cmp [nc][h_kv][d] in fp64 (compression keys/values of the nc
    compression blocks, overlapping when the stride is below the block): the
    linear map W_K, W_V, or the compression perceptron ``cmp_mlp`` (a dict of
    its weights, see ``_cmp_mlp``)."""
    k, v = _f32(k), _f32(v)
    isv = np.ascontiguousarray(is_vision, dtype=np.uint8)
    n = isv.shape[0]
    nv = int(isv.sum())
    stride = p.stride or p.block
    nb = (nv - p.block) // stride + 1 if nv >= p.block else 0
    kc = np.zeros((max(nb, 0), p.h_kv, p.d), np.float64)
    vc = np.zeros_like(kc)
    cfg = _cfg(p, n)
    if cmp_mlp is None:
        w_k, w_v = _f32(w_k), _f32(w_v)
        rc = _load().vnsa_oracle_pool_proj(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(isv),
                                           _ptr(w_k), _ptr(w_v), _ptr(kc), _ptr(vc))
    else:
        m, keep = _cmp_mlp(p.d, cmp_mlp)
        rc = _load().vnsa_oracle_pool_mlp(ctypes.byref(cfg), _ptr(k), _ptr(v), _ptr(isv),
                                          ctypes.byref(m), _ptr(kc), _ptr(vc))
        del keep
    if rc != 0:
        raise ValueError(f"oracle pool_proj rejected its arguments (code {rc})")
    return kc, vc


def gate_mlp(x, g1, c1, g2, c2, round_hidden_bf16=False):
    """Gate logits [n][n_out] of the layer input x [n][D] through the two-layer
    gate perceptron (g1 [D][H], c1 [H], g2 [H][n_out], c2 [n_out]); n_out =
    3 h_q with column 3h + c the logit of branch c of head h."""
    x, g1, c1, g2, c2 = _f32(x), _f32(g1), _f32(c1), _f32(g2), _f32(c2)
    n, dm = x.shape
    hidden = c1.shape[0]
    n_out = c2.shape[0]
    if g1.shape != (dm, hidden) or g2.shape != (hidden, n_out):
        raise ValueError("gate MLP weights must be [D][H] and [H][n_out]")
    out = np.zeros((n, n_out), np.float64)
    rc = _load().vnsa_oracle_gate_mlp(n, dm, hidden, n_out, _ptr(x), _ptr(g1), _ptr(c1),
                                      _ptr(g2), _ptr(c2), int(bool(round_hidden_bf16)),
                                      _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle gate_mlp rejected its arguments (code {rc})")
    return out


def forward(p: OracleParams, q, k, v, is_vision, gate, w_k, w_v, rows=None,
            forced_idx=None, want=(), cmp_mlp=None):
    """Layer prefill for the given global rows (all rows if None).  With
    ``cmp_mlp`` the compression branch maps block means through that
    perceptron instead of W_K, W_V.

    Returns a dict with "out" [R][h_q][d] and, for names in ``want``, any of
    "o_cmp", "o_slc", "o_swa" [R][h_q][d], "lse_cmp" [R][h_q], "idx" [R][h_kv][k],
    "imp" [R][h_kv][nb], plus "nb".  ``forced_idx`` [R][h_kv][k] replaces the
    top-k of vision rows.
    """
    q, k, v = _f32(q), _f32(k), _f32(v)
    gate = _f32(gate)
    if cmp_mlp is None:
        w_k, w_v = _f32(w_k), _f32(w_v)
    isv = np.ascontiguousarray(is_vision, dtype=np.uint8)
    n = isv.shape[0]
    if rows is None:
        rows_arr = None
        nr = n
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int32)
        nr = int(rows_arr.shape[0])
        if nr and (rows_arr.min() < 0 or rows_arr.max() >= n):
            raise ValueError("row index out of range")
    nb = int(isv.sum()) // p.block
    res = {"out": np.zeros((nr, p.h_q, p.d), np.float64), "nb": nb}
    for name in ("o_cmp", "o_slc", "o_swa"):
        if name in want:
            res[name] = np.zeros((nr, p.h_q, p.d), np.float64)
    if "lse_cmp" in want:
        res["lse_cmp"] = np.zeros((nr, p.h_q), np.float64)
    if "idx" in want:
        res["idx"] = np.zeros((nr, p.h_kv, p.top_k), np.int32)
    if "imp" in want:
        res["imp"] = np.zeros((nr, p.h_kv, max(nb, 0)), np.float64)
    fidx = None
    if forced_idx is not None:
        fidx = np.ascontiguousarray(forced_idx, dtype=np.int32)
        if fidx.shape != (nr, p.h_kv, p.top_k):
            raise ValueError("forced_idx must be [rows][h_kv][top_k]")
    cfg = _cfg(p, n)
    nb_out = ctypes.c_int(0)
    tail = (nr, _ptr(rows_arr), _ptr(fidx), _ptr(res["out"]),
            _ptr(res.get("o_cmp")), _ptr(res.get("o_slc")), _ptr(res.get("o_swa")),
            _ptr(res.get("lse_cmp")), _ptr(res.get("idx")), _ptr(res.get("imp")),
            ctypes.cast(ctypes.pointer(nb_out), ctypes.c_void_p))
    if cmp_mlp is None:
        rc = _load().vnsa_oracle_forward(
            ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(isv), _ptr(gate),
            _ptr(w_k), _ptr(w_v), *tail)
    else:
        m, keep = _cmp_mlp(p.d, cmp_mlp)
        rc = _load().vnsa_oracle_forward_mlp(
            ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(isv), _ptr(gate),
            ctypes.byref(m), *tail)
        del keep
    if rc != 0:
        raise ValueError(f"oracle forward rejected its arguments (code {rc})")
    return res
