"""Plain CPU oracle of the HyperAttention forward pass (test infrastructure).

Only the test suite, the package smoke check and the benchmark's CPU-baseline leg may import this
module. It wraps ``oracle.c`` (plain C, double precision, OpenMP) through ctypes and shares no code with
the CUDA library: it draws its own projections and samples from the seed and never reads anything the
CUDA library produced.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(dtype=np.uint16, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u64p = np.ctypeslib.ndpointer(dtype=np.uint64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile liboracle.so next to oracle.c (gcc, OpenMP, no contraction of multiply-adds)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    lib.ora_philox4x64_10.argtypes = [_u64p, _u64p, _u64p]
    lib.ora_philox4x64_10.restype = None
    lib.ora_draw_projection.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int, _f32p]
    lib.ora_draw_projection.restype = None
    lib.ora_draw_samples.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_int, _i32p]
    lib.ora_draw_samples.restype = ctypes.c_int
    lib.ora_gray_rank.argtypes = [ctypes.c_uint32]
    lib.ora_gray_rank.restype = ctypes.c_uint32
    lib.ora_hash_rows.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int, _f32p, ctypes.c_int, _u16p, _u8p]
    lib.ora_hash_rows.restype = ctypes.c_int
    lib.ora_sort_segment.argtypes = [_u16p, ctypes.c_int64, _i32p]
    lib.ora_sort_segment.restype = ctypes.c_int
    vp = ctypes.c_void_p
    lib.ora_forward.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int64,
                                vp, ctypes.c_int64, _f64p, vp, vp, vp, vp, vp]
    lib.ora_forward.restype = ctypes.c_int
    lib.ora_forward_sampling.argtypes = lib.ora_forward.argtypes + [ctypes.c_int]
    lib.ora_forward_sampling.restype = ctypes.c_int
    lib.ora_draw_rownorm.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64, _f32p, ctypes.c_int64,
                                     ctypes.c_int, ctypes.c_int, _i32p, _f64p]
    lib.ora_draw_rownorm.restype = ctypes.c_int
    lib.ora_level_perms.argtypes = [_u16p, ctypes.c_int64, ctypes.c_int, _i32p, _i32p]
    lib.ora_level_perms.restype = ctypes.c_int
    lib.ora_exact_attention.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        vp, ctypes.c_int64, _f64p]
    lib.ora_exact_attention.restype = ctypes.c_int
    lib.ora_diagnostics.argtypes = [_f32p, _f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                    ctypes.c_uint64, ctypes.c_int64, ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_double)]
    lib.ora_diagnostics.restype = ctypes.c_int
    lib.ora_weights.argtypes = [_f32p, _f32p, _f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int64,
                                ctypes.c_int, _f64p, _f64p]
    lib.ora_weights.restype = ctypes.c_int
    lib.ora_backward.argtypes = [_f32p, _f32p, _f32p, _f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                 ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                 ctypes.c_int64, ctypes.c_int, _f64p, _f64p, _f64p, _f64p, _f64p]
    lib.ora_backward.restype = ctypes.c_int
    lib.ora_backward_rows.argtypes = [_f32p, _f32p, _f32p, _f32p, ctypes.c_int64, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                                      ctypes.c_int64, ctypes.c_int, vp, ctypes.c_int64, _f64p]
    lib.ora_backward_rows.restype = ctypes.c_int
    lib.ora_num_threads.argtypes = []
    lib.ora_num_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} failed with status {rc}")


def num_threads() -> int:
    return _load().ora_num_threads()


def philox4x64_10(counter, key) -> np.ndarray:
    out = np.zeros(4, np.uint64)
    _load().ora_philox4x64_10(np.asarray(counter, np.uint64), np.asarray(key, np.uint64), out)
    return out


def draw_projection(seed: int, d: int, r: int) -> np.ndarray:
    """P as a (d, r) float32 array."""
    P = np.zeros((d, max(r, 1)), np.float32)
    _load().ora_draw_projection(seed, d, r, P)
    return P[:, :r].copy() if r > 0 else np.zeros((d, 0), np.float32)


def draw_samples(seed: int, bh: int, node: int, N: int, m: int) -> np.ndarray:
    S = np.zeros(max(m, 1), np.int32)
    _check(_load().ora_draw_samples(seed, bh, node, N, m, S), "draw_samples")
    return S[:m].copy()


def draw_rownorm(seed: int, bh: int, node: int, V: np.ndarray, m: int):
    """m row-norm draws over the rows of V (N, d) float32: indices (int32, -1 when every row is zero) and the
    log weights log(1 / (m p_j)), p_j = ||v_j||^2 / sum ||v||^2 (see oracle.c)."""
    V = np.ascontiguousarray(V, np.float32)
    N, d = V.shape
    S = np.zeros(max(m, 1), np.int32)
    lw = np.zeros(max(m, 1), np.float64)
    _check(_load().ora_draw_rownorm(seed, bh, node, V, N, d, m, S, lw), "draw_rownorm")
    return S[:m].copy(), lw[:m].copy()


SAMPLING = {"uniform": 0, "rownorm": 1}


def gray_rank(h: int) -> int:
    return int(_load().ora_gray_rank(h))


def hash_rows(X: np.ndarray, P: np.ndarray):
    """Ranks (uint16) and near-zero flags (uint8) of the rows of X (rows, d) float32."""
    X = np.ascontiguousarray(X, np.float32)
    rows, d = X.shape
    r = P.shape[1]
    Pc = np.ascontiguousarray(P if r > 0 else np.zeros((d, 1), np.float32), np.float32)
    rank = np.zeros(rows, np.uint16)
    near = np.zeros(rows, np.uint8)
    _check(_load().ora_hash_rows(X, rows, d, Pc, r, rank, near), "hash_rows")
    return rank, near


def sort_segment(rank: np.ndarray) -> np.ndarray:
    rank = np.ascontiguousarray(rank, np.uint16)
    perm = np.zeros(max(len(rank), 1), np.int32)
    _check(_load().ora_sort_segment(rank, len(rank), perm), "sort_segment")
    return perm[:len(rank)].copy()


def level_perms(rank: np.ndarray, n: int, level: int):
    """Sorted permutations of one level (0: non-causal; l >= 1: causal level l), see oracle.c."""
    rank = np.ascontiguousarray(rank, np.uint16)
    size = n if level == 0 else n // 2
    pq = np.zeros(size, np.int32)
    pk = np.zeros(size, np.int32)
    _check(_load().ora_level_perms(rank, n, level, pq, pk), "level_perms")
    return pq, pk


def forward(Q, K, V, *, block: int, m: int, r: int, causal: bool, seed: int, bh: int = 0,
            base: int = 0, rows=None, want_parts: bool = False, sampling: str = "uniform"):
    """One (batch*head) problem. Q, K, V: (n, d) float32 (bf16 inputs passed as their exact float32
    values). Returns a dict with O (nrows, d) float64, L (log of the estimated normaliser), and when
    requested L1/L2 (non-causal only), rank (2n,) and near (2n,). sampling "uniform" reuses the uniform
    samples for the product with V; "rownorm" draws that product's samples by the squared row norms of V."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    n, d = Q.shape
    sel = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nsel = n if sel is None else len(sel)
    O = np.zeros((max(nsel, 1), d), np.float64)
    L = np.zeros(max(nsel, 1), np.float64)
    L1 = np.zeros(max(nsel, 1), np.float64) if (want_parts and not causal) else None
    L2 = np.zeros(max(nsel, 1), np.float64) if (want_parts and not causal) else None
    rank = np.zeros(2 * n, np.uint16)
    near = np.zeros(2 * n, np.uint8)
    rc = _load().ora_forward_sampling(Q, K, V, n, d, block, m, r, int(causal), base, seed, bh,
                                      _ptr(sel), nsel, O, _ptr(L), _ptr(L1), _ptr(L2), _ptr(rank), _ptr(near),
                                      SAMPLING[sampling])
    _check(rc, "forward")
    out = {"O": O[:nsel], "L": L[:nsel], "rank": rank, "near": near}
    if L1 is not None:
        out["L1"] = L1[:nsel]
        out["L2"] = L2[:nsel]
    return out


def diagnostics(Q, K, *, block: int, r: int, seed: int, first_col: int = 0):
    """(alpha, kappa) of one non-causal problem: alpha = n * max_{j >= first_col} ||(D^-1 A) e_j||^2 and kappa =
    max/min over rows of the row sums of A outside the row's sortLSH block (see oracle.c for the readings)."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    n, d = Q.shape
    alpha, kappa = ctypes.c_double(), ctypes.c_double()
    _check(_load().ora_diagnostics(Q, K, n, d, block, r, seed, first_col, ctypes.byref(alpha), ctypes.byref(kappa)),
           "diagnostics")
    return alpha.value, kappa.value


def weights(Q, K, V, *, block: int, m: int, r: int, causal: bool, seed: int, bh: int = 0, base: int = 0,
            sampling: str = "uniform"):
    """Dense (n, n) numerator and normaliser weights (Wn, Wd) of one problem: O = (Wn o E) V / rowsum(Wd o E),
    E = exp(Q K^T) (see oracle.c). For small n."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    n, d = Q.shape
    Wn = np.zeros((n, n), np.float64)
    Wd = np.zeros((n, n), np.float64)
    _check(_load().ora_weights(Q, K, V, n, d, block, m, r, int(causal), base, seed, bh, SAMPLING[sampling], Wn, Wd),
           "weights")
    return Wn, Wd


def backward(Q, K, V, dO, *, block: int, m: int, r: int, causal: bool, seed: int, bh: int = 0, base: int = 0,
             sampling: str = "uniform"):
    """Gradients of sum(dO * O) of one problem with respect to Q, K, V (float64, (n, d) each), the sort and the
    draws held fixed; also O and the log normaliser L. Dense: for small n."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    dO = np.ascontiguousarray(dO, np.float32)
    n, d = Q.shape
    out = {k: np.zeros((n, d), np.float64) for k in ("dQ", "dK", "dV", "O")}
    out["L"] = np.zeros(n, np.float64)
    _check(_load().ora_backward(Q, K, V, dO, n, d, block, m, r, int(causal), base, seed, bh, SAMPLING[sampling],
                                out["dQ"], out["dK"], out["dV"], out["O"], out["L"]), "backward")
    return out


def backward_rows(Q, K, V, dO, rows, *, block: int, m: int, r: int, causal: bool, seed: int, bh: int = 0,
                  base: int = 0, sampling: str = "uniform") -> np.ndarray:
    """dQ (len(rows), d) float64 of the selected rows, for any n (no dense weights; see oracle.c)."""
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    dO = np.ascontiguousarray(dO, np.float32)
    n, d = Q.shape
    sel = np.ascontiguousarray(rows, np.int64)
    dQ = np.zeros((max(len(sel), 1), d), np.float64)
    _check(_load().ora_backward_rows(Q, K, V, dO, n, d, block, m, r, int(causal), base, seed, bh, SAMPLING[sampling],
                                     _ptr(sel), len(sel), dQ), "backward_rows")
    return dQ[:len(sel)]


def exact_attention(Q, K, V, *, causal: bool, rows=None) -> np.ndarray:
    Q = np.ascontiguousarray(Q, np.float32)
    K = np.ascontiguousarray(K, np.float32)
    V = np.ascontiguousarray(V, np.float32)
    n, d = Q.shape
    sel = None if rows is None else np.ascontiguousarray(rows, np.int64)
    nsel = n if sel is None else len(sel)
    O = np.zeros((max(nsel, 1), d), np.float64)
    _check(_load().ora_exact_attention(Q, K, V, n, d, int(causal), _ptr(sel), nsel, O), "exact_attention")
    return O[:nsel]
