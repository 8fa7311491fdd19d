"""ctypes binding of libvnsa.so (the C ABI of include/vnsa.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The functions keep the C names (vnsa_create, vnsa_forward, ...);
``Layer`` is a small convenience wrapper that takes torch tensors (used for
device memory and streams only) and passes their pointers through.

There is no fallback: if the library is missing or no CUDA device is visible,
the calls raise.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvnsa.so")

VNSA_OK, VNSA_ERR_INVALID_ARG, VNSA_ERR_UNSUPPORTED, VNSA_ERR_CUDA = 0, 1, 2, 3
VNSA_ERR_TIMEOUT, VNSA_ERR_BOUNDS, VNSA_ERR_NO_DEVICE = 4, 5, 6
VNSA_BF16, VNSA_FP32 = 0, 1
VNSA_PATH_SIMT, VNSA_PATH_TCGEN05 = 0, 1
NUM_STAGES = 7

EXPORTED = ("vnsa_status_string", "vnsa_stage_name", "vnsa_workspace_bytes", "vnsa_create",
            "vnsa_forward", "vnsa_forward_host", "vnsa_get_device_status", "vnsa_get_counts",
            "vnsa_set_timing", "vnsa_get_timing", "vnsa_get_launch_count", "vnsa_destroy",
            "vnsa_select_noalloc", "vnsa_decode", "vnsa_set_cmp_mlp", "vnsa_gate_mlp",
            "vnsa_forward_host_async", "vnsa_host_wait", "vnsa_host_join",
            "vnsa_select_noalloc_status", "vnsa_set_wait_limit", "vnsa_get_path")


class vnsa_config(ctypes.Structure):
    _fields_ = [("n_max", ctypes.c_int), ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int),
                ("d", ctypes.c_int), ("block", ctypes.c_int), ("top_k", ctypes.c_int),
                ("window", ctypes.c_int), ("force_first", ctypes.c_int),
                ("force_local", ctypes.c_int), ("scale", ctypes.c_float),
                ("dtype", ctypes.c_int), ("cmp_stride", ctypes.c_int)]


class vnsa_debug(ctypes.Structure):
    _fields_ = [("o_cmp", ctypes.c_void_p), ("o_slc", ctypes.c_void_p),
                ("o_swa", ctypes.c_void_p), ("lse_cmp", ctypes.c_void_p),
                ("idx", ctypes.c_void_p), ("imp", ctypes.c_void_p),
                ("imp_stride", ctypes.c_int), ("k_cmp", ctypes.c_void_p),
                ("v_cmp", ctypes.c_void_p), ("forced_idx", ctypes.c_void_p)]


class VnsaError(RuntimeError):
    def __init__(self, call, code):
        self.code = int(code)
        super().__init__(f"{call} failed: {status_string(code)} (code {code})")


_lib = None


def load(path: str = LIB_PATH):
    """Load the library (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libvnsa.so not built ({path}); run "
                           "python -m sparse_attention_long_block_b200.build")
    lib = ctypes.CDLL(path)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.vnsa_status_string.restype = ctypes.c_char_p
    lib.vnsa_status_string.argtypes = [I]
    lib.vnsa_stage_name.restype = ctypes.c_char_p
    lib.vnsa_stage_name.argtypes = [I]
    lib.vnsa_workspace_bytes.argtypes = [ctypes.POINTER(vnsa_config), ctypes.POINTER(S)]
    lib.vnsa_create.argtypes = [ctypes.POINTER(vnsa_config), P, P, ctypes.POINTER(P)]
    lib.vnsa_forward.argtypes = [P, I, P, P, P, P, P, P, ctypes.POINTER(vnsa_debug), P]
    lib.vnsa_forward_host.argtypes = [P, I, P, P, P, P, P, P, P]
    lib.vnsa_forward_host_async.argtypes = [P, I, P, P, P, P, P, P, P,
                                            ctypes.POINTER(ctypes.c_ulonglong)]
    lib.vnsa_host_wait.argtypes = [P, ctypes.c_ulonglong]
    lib.vnsa_host_join.argtypes = [P, P]
    lib.vnsa_decode.argtypes = [P, I, P, P, P, P, P, P, P, P]
    lib.vnsa_set_cmp_mlp.argtypes = [P, I] + [P] * 8
    lib.vnsa_gate_mlp.argtypes = [P, I, I, I] + [P] * 7
    lib.vnsa_get_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    lib.vnsa_get_counts.argtypes = [P, P, ctypes.POINTER(I), ctypes.POINTER(I)]
    lib.vnsa_set_timing.argtypes = [P, I]
    lib.vnsa_get_timing.argtypes = [P, ctypes.POINTER(ctypes.c_float)]
    lib.vnsa_get_launch_count.argtypes = [P, ctypes.POINTER(I)]
    lib.vnsa_destroy.argtypes = [P]
    lib.vnsa_select_noalloc.argtypes = [ctypes.POINTER(vnsa_config), I, P, P, P, P, P, P, P, P, P]
    lib.vnsa_select_noalloc_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.vnsa_set_wait_limit.argtypes = [P, ctypes.c_ulonglong]
    lib.vnsa_get_path.argtypes = [P, ctypes.POINTER(I)]
    for name in EXPORTED:
        if name not in ("vnsa_status_string", "vnsa_stage_name"):
            getattr(lib, name).restype = I
    _lib = lib
    return lib


def status_string(code) -> str:
    return load().vnsa_status_string(int(code)).decode()


def stage_name(i) -> str | None:
    r = load().vnsa_stage_name(int(i))
    return None if r is None else r.decode()


def _check(call, code):
    if code != VNSA_OK:
        raise VnsaError(call, code)


# --- same-name thin wrappers --------------------------------------------------
def vnsa_workspace_bytes(cfg: vnsa_config) -> int:
    out = ctypes.c_size_t(0)
    _check("vnsa_workspace_bytes", load().vnsa_workspace_bytes(ctypes.byref(cfg), ctypes.byref(out)))
    return int(out.value)


def vnsa_create(cfg: vnsa_config, w_k_ptr: int, w_v_ptr: int) -> int:
    h = ctypes.c_void_p(0)
    _check("vnsa_create", load().vnsa_create(ctypes.byref(cfg), w_k_ptr, w_v_ptr, ctypes.byref(h)))
    return h.value


def vnsa_forward(h, n, q, k, v, is_vision, gate, out, dbg=None, stream=0):
    d = ctypes.byref(dbg) if dbg is not None else None
    _check("vnsa_forward", load().vnsa_forward(h, n, q, k, v, is_vision, gate, out, d, stream))


def vnsa_forward_host(h, n, q, k, v, is_vision, gate, out, stream=0):
    _check("vnsa_forward_host", load().vnsa_forward_host(h, n, q, k, v, is_vision, gate, out, stream))


def vnsa_forward_host_async(h, n, q, k, v, is_vision, gate, out, stream=0) -> int:
    t = ctypes.c_ulonglong(0)
    _check("vnsa_forward_host_async", load().vnsa_forward_host_async(
        h, n, q, k, v, is_vision, gate, out, stream, ctypes.byref(t)))
    return int(t.value)


def vnsa_host_wait(h, ticket):
    _check("vnsa_host_wait", load().vnsa_host_wait(h, int(ticket)))


def vnsa_host_join(h, stream=0):
    _check("vnsa_host_join", load().vnsa_host_join(h, stream))


def vnsa_decode(h, n, q_new, k, v, is_vision, gate_new, out_new, sel_out=None, stream=0):
    _check("vnsa_decode", load().vnsa_decode(h, n, q_new, k, v, is_vision, gate_new, out_new,
                                             sel_out, stream))


def vnsa_set_cmp_mlp(h, hidden, w1_k, b1_k, w2_k, b2_k, w1_v, b1_v, w2_v, b2_v):
    _check("vnsa_set_cmp_mlp", load().vnsa_set_cmp_mlp(h, hidden, w1_k, b1_k, w2_k, b2_k,
                                                       w1_v, b1_v, w2_v, b2_v))


def vnsa_gate_mlp(h, n, d_model, hidden, x, g1, c1, g2, c2, gate_logits, stream=0):
    _check("vnsa_gate_mlp", load().vnsa_gate_mlp(h, n, d_model, hidden, x, g1, c1, g2, c2,
                                                 gate_logits, stream))


def vnsa_get_device_status(h, stream=0) -> int:
    c = ctypes.c_uint32(0)
    _check("vnsa_get_device_status", load().vnsa_get_device_status(h, stream, ctypes.byref(c)))
    return int(c.value)


def vnsa_get_counts(h, stream=0):
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    _check("vnsa_get_counts", load().vnsa_get_counts(h, stream, ctypes.byref(a), ctypes.byref(b)))
    return a.value, b.value


def vnsa_set_timing(h, enable: bool):
    _check("vnsa_set_timing", load().vnsa_set_timing(h, int(bool(enable))))


def vnsa_get_timing(h):
    arr = (ctypes.c_float * NUM_STAGES)()
    _check("vnsa_get_timing", load().vnsa_get_timing(h, arr))
    return {stage_name(i): float(arr[i]) for i in range(NUM_STAGES)}


def vnsa_get_launch_count(h) -> int:
    c = ctypes.c_int(0)
    _check("vnsa_get_launch_count", load().vnsa_get_launch_count(h, ctypes.byref(c)))
    return c.value


def vnsa_destroy(h):
    _check("vnsa_destroy", load().vnsa_destroy(h))


def vnsa_select_noalloc(cfg: vnsa_config, n, q, k, v, is_vision, w_k, w_v, o_cmp, idx,
                        stream=0):
    """Selection chain with no device allocation (static library scratch)."""
    _check("vnsa_select_noalloc", load().vnsa_select_noalloc(
        ctypes.byref(cfg), n, q, k, v, is_vision, w_k, w_v, o_cmp, idx, stream))


def vnsa_set_wait_limit(h, ns: int):
    _check("vnsa_set_wait_limit", load().vnsa_set_wait_limit(h, int(ns)))


def vnsa_get_path(h) -> int:
    out = ctypes.c_int(-1)
    _check("vnsa_get_path", load().vnsa_get_path(h, ctypes.byref(out)))
    return int(out.value)


def vnsa_select_noalloc_status(stream=0) -> int:
    """Synchronise `stream`, then read and clear the device status word of the
    last vnsa_select_noalloc call on the current device."""
    code = ctypes.c_uint32(0)
    _check("vnsa_select_noalloc_status",
           load().vnsa_select_noalloc_status(stream, ctypes.byref(code)))
    return int(code.value)


# --- torch-facing convenience -------------------------------------------------
class Layer:
    """One configured layer (a vnsa handle) fed with torch CUDA tensors."""

    def __init__(self, *, n_max, h_q, h_kv, d, top_k, window, w_k, w_v, block=64,
                 force_first=True, force_local=True, scale=0.0, dtype="bf16", stride=0):
        import torch
        if not torch.cuda.is_available():
            raise RuntimeError("vnsa needs a CUDA device; there is no CPU path")
        self.dtype = dtype
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.cfg = vnsa_config(int(n_max), int(h_q), int(h_kv), int(d), int(block), int(top_k),
                               int(window), int(bool(force_first)), int(bool(force_local)),
                               float(scale), VNSA_BF16 if dtype == "bf16" else VNSA_FP32,
                               int(stride))
        self.h_q, self.h_kv, self.d, self.top_k, self.block = h_q, h_kv, d, top_k, block
        w_k = self._dev(w_k)
        w_v = self._dev(w_v)
        self.handle = vnsa_create(self.cfg, w_k.data_ptr(), w_v.data_ptr())

    def _dev(self, t):
        import torch
        t = torch.as_tensor(t)
        return t.to(device="cuda", dtype=self.tdtype).contiguous()

    @staticmethod
    def _stream(stream):
        import torch
        s = stream if stream is not None else torch.cuda.current_stream()
        return ctypes.c_void_p(s.cuda_stream)

    def forward(self, q, k, v, is_vision, gate, out=None, dbg=None, stream=None):
        """Enqueue one layer prefill; returns `out` (allocated if None)."""
        import torch
        n = int(q.shape[0])
        for t in (q, k, v, is_vision, gate):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("inputs must be contiguous CUDA tensors")
        if q.dtype != self.tdtype or k.dtype != self.tdtype or v.dtype != self.tdtype:
            raise ValueError("q, k, v must match the layer dtype")
        if gate.dtype != torch.float32 or is_vision.dtype != torch.uint8:
            raise ValueError("gate must be float32 and is_vision uint8")
        if out is None:
            out = torch.empty_like(q)
        vnsa_forward(self.handle, n, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                     is_vision.data_ptr(), gate.data_ptr(), out.data_ptr(), dbg,
                     self._stream(stream))
        return out

    def decode(self, n, q_new, k, v, is_vision, gate_new, out=None, sel_out=None, stream=None):
        """One decode step: the output of token n-1 of the stream in k, v,
        is_vision (all n tokens), continuing the previous forward/decode call
        over tokens 0..n-2.  q_new [h_q][d], gate_new [h_q][3]."""
        import torch
        for t in (q_new, k, v, is_vision, gate_new):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("inputs must be contiguous CUDA tensors")
        if q_new.dtype != self.tdtype or k.dtype != self.tdtype or v.dtype != self.tdtype:
            raise ValueError("q, k, v must match the layer dtype")
        if out is None:
            out = torch.empty_like(q_new)
        vnsa_decode(self.handle, int(n), q_new.data_ptr(), k.data_ptr(), v.data_ptr(),
                    is_vision.data_ptr(), gate_new.data_ptr(), out.data_ptr(),
                    None if sel_out is None else sel_out.data_ptr(), self._stream(stream))
        return out

    CMP_MLP_KEYS = ("w1_k", "b1_k", "w2_k", "b2_k", "w1_v", "b1_v", "w2_v", "b2_v")

    def set_cmp_mlp(self, mlp=None):
        """Compression perceptron: a dict with w1_k [d][H], b1_k [H], w2_k
        [H][d], b2_k [d] and the same for v (weights in the layer dtype, biases
        fp32), or None for the linear W_K, W_V given at construction."""
        import torch
        if mlp is None:
            vnsa_set_cmp_mlp(self.handle, 0, *([None] * 8))
            return
        ts = []
        for nm in self.CMP_MLP_KEYS:
            dt = torch.float32 if nm.startswith("b") else self.tdtype
            ts.append(torch.as_tensor(mlp[nm]).to(device="cuda", dtype=dt).contiguous())
        hidden = int(ts[1].shape[0])
        vnsa_set_cmp_mlp(self.handle, hidden, *[t.data_ptr() for t in ts])

    def gate_mlp(self, x, g1, c1, g2, c2, out=None, stream=None):
        """Gate logits [n][h_q][3] fp32 of the layer input x [n][D] through the
        gate perceptron (g1 [D][H], g2 [H][3 h_q] in the layer dtype, c1, c2
        fp32); all contiguous CUDA tensors."""
        import torch
        for t in (x, g1, c1, g2, c2):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError("inputs must be contiguous CUDA tensors")
        if x.dtype != self.tdtype or g1.dtype != self.tdtype or g2.dtype != self.tdtype:
            raise ValueError("x, g1, g2 must match the layer dtype")
        if c1.dtype != torch.float32 or c2.dtype != torch.float32:
            raise ValueError("c1, c2 must be float32")
        n, dm = int(x.shape[0]), int(x.shape[1])
        hidden = int(c1.shape[0])
        if tuple(g1.shape) != (dm, hidden) or tuple(g2.shape) != (hidden, 3 * self.h_q):
            raise ValueError("g1 must be [D][H] and g2 [H][3 h_q]")
        if out is None:
            out = torch.empty((n, self.h_q, 3), dtype=torch.float32, device=x.device)
        vnsa_gate_mlp(self.handle, n, dm, hidden, x.data_ptr(), g1.data_ptr(), c1.data_ptr(),
                      g2.data_ptr(), c2.data_ptr(), out.data_ptr(), self._stream(stream))
        return out

    def forward_host(self, q, k, v, is_vision, gate, out, stream=None):
        """Host (CPU, ideally pinned) tensors in and out; synchronous."""
        n = int(q.shape[0])
        vnsa_forward_host(self.handle, n, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                          is_vision.data_ptr(), gate.data_ptr(), out.data_ptr(),
                          self._stream(stream))
        return out

    def forward_host_async(self, q, k, v, is_vision, gate, out, stream=None) -> int:
        """Enqueue one layer call on host (pinned) tensors; returns its ticket.
        The tensors must stay untouched until wait_host(ticket) returns."""
        n = int(q.shape[0])
        for t in (q, k, v, is_vision, gate, out):
            if t.is_cuda or not t.is_contiguous():
                raise ValueError("host tensors must be contiguous CPU tensors")
        return vnsa_forward_host_async(self.handle, n, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       is_vision.data_ptr(), gate.data_ptr(), out.data_ptr(),
                                       self._stream(stream))

    def wait_host(self, ticket):
        vnsa_host_wait(self.handle, ticket)

    def join_host(self, stream=None):
        vnsa_host_join(self.handle, self._stream(stream))

    def device_status(self, stream=None) -> int:
        return vnsa_get_device_status(self.handle, self._stream(stream))

    def counts(self, stream=None):
        return vnsa_get_counts(self.handle, self._stream(stream))

    def set_timing(self, enable=True):
        vnsa_set_timing(self.handle, enable)

    def timing(self):
        return vnsa_get_timing(self.handle)

    def launches(self) -> int:
        return vnsa_get_launch_count(self.handle)

    def set_wait_limit(self, ns: int):
        """Limit of the kernels' bounded waits in ns (0: the default)."""
        vnsa_set_wait_limit(self.handle, ns)

    def path(self) -> str:
        """"tcgen05" or "simt": the kernel family this layer runs on."""
        return "tcgen05" if vnsa_get_path(self.handle) == VNSA_PATH_TCGEN05 else "simt"

    def close(self):
        if getattr(self, "handle", None):
            vnsa_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def make_debug(n, h_q, h_kv, d, top_k, block=64, dtype=None, want=(), forced_idx=None,
               stride=0):
    """Allocate the requested debug exports as torch CUDA tensors.

    Returns (vnsa_debug struct, dict of tensors).  ``forced_idx``
    [h_kv][n][top_k] int32 CUDA tensor overrides the top-k.  ``stride``: the
    compression stride (0: the block), which sets the rows of k_cmp / v_cmp."""
    import torch
    dev = "cuda"
    t = {}
    dbg = vnsa_debug()
    for name in ("o_cmp", "o_slc", "o_swa"):
        if name in want:
            t[name] = torch.zeros((n, h_q, d), dtype=torch.float32, device=dev)
            setattr(dbg, name, t[name].data_ptr())
    if "lse_cmp" in want:
        t["lse_cmp"] = torch.full((n, h_q), float("nan"), dtype=torch.float32, device=dev)
        dbg.lse_cmp = t["lse_cmp"].data_ptr()
    if "idx" in want:
        t["idx"] = torch.full((h_kv, n, top_k), -7, dtype=torch.int32, device=dev)
        dbg.idx = t["idx"].data_ptr()
    if "imp" in want:
        stride = max(1, n // block)
        t["imp"] = torch.zeros((h_kv, n, stride), dtype=torch.float32, device=dev)
        dbg.imp = t["imp"].data_ptr()
        dbg.imp_stride = stride
    s = stride or block
    n_cmp = (n - block) // s + 1 if n >= block else 0
    for name in ("k_cmp", "v_cmp"):
        if name in want:
            t[name] = torch.zeros((max(1, n_cmp), h_kv, d), dtype=dtype, device=dev)
            setattr(dbg, name, t[name].data_ptr())
    if forced_idx is not None:
        t["forced_idx"] = forced_idx
        dbg.forced_idx = forced_idx.data_ptr()
    return dbg, t
