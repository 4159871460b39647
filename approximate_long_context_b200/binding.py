"""ctypes binding of libhyper_attn.so (include/hyper_attn.h). Argument marshalling only.

The in-tree library is loaded on first use; if it is missing this raises instead of falling back to
anything else (build it with ``python -m approximate_long_context_b200.build`` or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# HA_LIBRARY=debug selects the HA_DEBUG build (bounds-checked index reads), any other value a library path
LIB_PATH = os.path.join(_HERE, "libhyper_attn.so")
if os.environ.get("HA_LIBRARY"):
    LIB_PATH = (os.path.join(_HERE, "libhyper_attn_debug.so") if os.environ["HA_LIBRARY"] == "debug"
                else os.environ["HA_LIBRARY"])

HA_OK, HA_ERR_INVALID_ARG, HA_ERR_UNSUPPORTED, HA_ERR_CUDA, HA_ERR_OOM, HA_ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
DTYPES = {"bf16": 0, "fp32": 1}
KERNELS = {"auto": 0, "simt": 1, "tc": 2}
DBG = {"rank": 0, "near": 1, "perm": 2, "inv": 3, "lse": 4, "rn_s": 5, "rn_logw": 6}
SAMPLING = {"uniform": 0, "rownorm": 1}

# every symbol include/hyper_attn.h declares
EXPORTS = [
    "hyper_attn_create", "hyper_attn_set_options", "hyper_attn_default_options", "hyper_attn_forward",
    "hyper_attn_forward_host", "hyper_attn_draw", "hyper_attn_levels", "hyper_attn_debug_copy",
    "hyper_attn_status", "hyper_attn_last_launch_count", "hyper_attn_last_error", "hyper_attn_destroy",
    "hyper_attn_version", "hyper_attn_profile", "hyper_attn_profile_read",
    "hyper_attn_last_kernel", "hyper_attn_forward_noalloc", "hyper_attn_exact",
    "hyper_attn_diagnostics", "hyper_attn_backward", "hyper_attn_test_fail_alloc",
]
KERNEL_CLASSES = ["hash", "sort", "attn", "causal_base", "draws"]


class HAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"hyper_attn error {code}: {msg}")
        self.code = code


class Options(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("out_dtype", ctypes.c_int),
        ("batch", ctypes.c_int64),
        ("causal_base", ctypes.c_int64),
        ("stream", ctypes.c_void_p),
        ("kernel", ctypes.c_int),
        ("debug_captures", ctypes.c_int),
        ("bh_offset", ctypes.c_int64),
        ("test_stall_ms", ctypes.c_int),
        ("sampling", ctypes.c_int),
    ]


_lib = None


def lib():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: the CUDA library has not been built")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, u64, ci = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int
    L.hyper_attn_create.argtypes = [ctypes.POINTER(vp), ci]
    L.hyper_attn_set_options.argtypes = [vp, ctypes.POINTER(Options)]
    L.hyper_attn_default_options.argtypes = [ctypes.POINTER(Options)]
    L.hyper_attn_default_options.restype = None
    fwd = [vp, vp, vp, vp, vp, i64, ci, ci, ci, ci, ci, ci, u64]
    L.hyper_attn_forward.argtypes = fwd
    L.hyper_attn_forward_host.argtypes = fwd
    L.hyper_attn_exact.argtypes = [vp, vp, vp, vp, vp, i64, ci, ci, ci]
    L.hyper_attn_diagnostics.argtypes = [vp, vp, vp, i64, ci, ci, ci, ci, u64, i64, vp, vp]
    L.hyper_attn_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i64, ci, ci, ci, ci, ci, ci, u64]
    L.hyper_attn_test_fail_alloc.argtypes = [vp, ci]
    L.hyper_attn_draw.argtypes = [u64, ci, ci, i64, i64, ci, ci, i64, vp, vp]
    L.hyper_attn_levels.argtypes = [i64, ci, i64, ctypes.POINTER(ci), ctypes.POINTER(i64)]
    L.hyper_attn_debug_copy.argtypes = [vp, ci, ci, vp, ctypes.c_size_t]
    L.hyper_attn_status.argtypes = [vp]
    L.hyper_attn_last_launch_count.argtypes = [vp]
    L.hyper_attn_last_error.argtypes = [vp]
    L.hyper_attn_last_error.restype = ctypes.c_char_p
    L.hyper_attn_destroy.argtypes = [vp]
    L.hyper_attn_version.argtypes = []
    L.hyper_attn_profile.argtypes = [vp, ci]
    L.hyper_attn_last_kernel.argtypes = [vp]
    L.hyper_attn_forward_noalloc.argtypes = [vp, vp, vp, vp, i64, ci, ci, ci, ci, ci, u64, ci, vp]
    L.hyper_attn_profile_read.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ci), ci]
    _lib = L
    return L


def default_options() -> Options:
    o = Options()
    lib().hyper_attn_default_options(ctypes.byref(o))
    return o


def levels(n: int, causal: bool, base: int):
    L = ctypes.c_int()
    nodes = ctypes.c_int64()
    rc = lib().hyper_attn_levels(n, int(causal), base, ctypes.byref(L), ctypes.byref(nodes))
    if rc:
        raise HAError(rc, "invalid causal shape")
    return L.value, nodes.value


def draw(seed: int, d: int, r: int, bh: int, n: int, m: int, causal: bool = False, base: int = 4096):
    """The projection matrix (d, r) and samples (bh, nodes, m) the forward pass uses (host only)."""
    _, nodes = levels(n, causal, base) if causal else (0, 1)
    P = np.zeros((d, max(r, 1)), np.float32)
    S = np.zeros((bh, nodes, max(m, 1)), np.int32)
    rc = lib().hyper_attn_draw(seed, d, r, bh, n, m, int(causal), base, P.ctypes.data, S.ctypes.data)
    if rc:
        raise HAError(rc, "hyper_attn_draw failed")
    return P[:, :r].copy(), S[:, :, :m].copy()


def _ptr(x) -> int:
    if hasattr(x, "data_ptr"):
        if not x.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("arrays must be C-contiguous")
        return x.ctypes.data
    return int(x)


class HyperAttention:
    """One library handle bound to a CUDA device."""

    def __init__(self, device: int = 0):
        self._h = ctypes.c_void_p()
        rc = lib().hyper_attn_create(ctypes.byref(self._h), device)
        if rc:
            raise HAError(rc, f"hyper_attn_create(device={device}) failed")
        self.options = default_options()

    def _check(self, rc: int):
        if rc:
            raise HAError(rc, lib().hyper_attn_last_error(self._h).decode())

    def set_options(self, *, dtype="bf16", out_dtype=None, batch=1, causal_base=4096, stream=None,
                    kernel="auto", debug_captures=False, bh_offset=0, test_stall_ms=0, sampling="uniform"):
        o = Options()
        o.dtype = DTYPES[dtype]
        o.out_dtype = -1 if out_dtype is None else DTYPES[out_dtype]
        o.batch = batch
        o.causal_base = causal_base
        o.stream = stream
        o.kernel = KERNELS[kernel]
        o.debug_captures = int(bool(debug_captures))
        o.bh_offset = bh_offset
        o.test_stall_ms = test_stall_ms
        o.sampling = SAMPLING[sampling]
        self._check(lib().hyper_attn_set_options(self._h, ctypes.byref(o)))
        self.options = o

    def forward(self, Q, K, V, O, *, n, d, heads, block, m, r, causal, seed):
        """Device tensors (torch CUDA tensors or raw device addresses)."""
        self._check(lib().hyper_attn_forward(self._h, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), n, d, heads, block, m, r,
                                             int(causal), seed))

    def exact(self, Q, K, V, O, *, n, d, heads, causal):
        """Exact softmax attention (device tensors) on the tensor-core kernel; enqueued on the handle's stream."""
        self._check(lib().hyper_attn_exact(self._h, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), n, d, heads, int(causal)))

    def backward(self, Q, K, V, dO, dQ, dK, dV, *, n, d, heads, block, m, r, causal, seed):
        """Gradients of sum(dO * O) into fp32 device tensors dQ, dK, dV (the forward is recomputed); enqueued on
        the handle's stream."""
        self._check(lib().hyper_attn_backward(self._h, _ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(dQ), _ptr(dK),
                                              _ptr(dV), n, d, heads, block, m, r, int(causal), seed))

    def diagnostics(self, Q, K, *, n, d, heads, block, r, seed, first_col=0):
        """(alpha, kappa) arrays of length batch*heads for device tensors Q, K (synchronous)."""
        bh = self.options.batch * heads
        alpha = np.zeros(bh, np.float64)
        kappa = np.zeros(bh, np.float64)
        self._check(lib().hyper_attn_diagnostics(self._h, _ptr(Q), _ptr(K), n, d, heads, block, r, seed, first_col,
                                                 alpha.ctypes.data, kappa.ctypes.data))
        return alpha, kappa

    def forward_host(self, Q, K, V, O, *, n, d, heads, block, m, r, causal, seed):
        """Host buffers (numpy arrays or CPU torch tensors, preferably page-locked); blocks until O is ready."""
        self._check(lib().hyper_attn_forward_host(self._h, _ptr(Q), _ptr(K), _ptr(V), _ptr(O), n, d, heads, block, m,
                                                  r, int(causal), seed))

    def debug_copy(self, what: str, level: int, dtype, count: int) -> np.ndarray:
        out = np.zeros(count, dtype)
        self._check(lib().hyper_attn_debug_copy(self._h, DBG[what], level, out.ctypes.data, out.nbytes))
        return out

    def status(self) -> int:
        return lib().hyper_attn_status(self._h)

    def last_error(self) -> str:
        return lib().hyper_attn_last_error(self._h).decode()

    def test_fail_alloc(self, count: int):
        """Test hook: fail the handle's next `count` allocations as if memory had run out (HA_ERR_OOM)."""
        self._check(lib().hyper_attn_test_fail_alloc(self._h, count))

    def profile(self, enable: bool):
        self._check(lib().hyper_attn_profile(self._h, int(enable)))

    def profile_read(self):
        """{class: (total ms, launches)} since the previous read (synchronises the stream)."""
        n = len(KERNEL_CLASSES)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int * n)()
        self._check(lib().hyper_attn_profile_read(self._h, ms, cnt, n))
        return {k: (ms[i], cnt[i]) for i, k in enumerate(KERNEL_CLASSES)}

    def last_kernel(self) -> str:
        """'simt' or 'tc': the attention kernel family of the last forward call."""
        return {0: "none", 1: "simt", 2: "tc"}[lib().hyper_attn_last_kernel(self._h)]

    def last_launch_count(self) -> int:
        return lib().hyper_attn_last_launch_count(self._h)

    def close(self):
        if self._h:
            lib().hyper_attn_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
