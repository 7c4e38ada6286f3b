"""fp64 CPU oracle of the double-binary layer forward and backward (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package. The CUDA product path neither
imports it nor shares code with it.

The arithmetic lives in ``dbf_oracle.c`` (plain fp64 loops in the order the
LoRDBA page states the forward: gamma scaling, B2 sign accumulation, beta
scaling, B1 sign accumulation, alpha scaling, envelope sum). This module
builds that file with gcc, loads it with ctypes and adds the routing of
tokens to adapters for segmented serving (LoRDBA page, section 1: many
adapters served at once, as in S-LoRA / Punica).

Pins (tests/test_oracle_pins.py): dense reconstruction of Delta-W by library
matmuls, the all-plus / rank-one / Sylvester-Hadamard closed forms, the
matched sign-flip, envelope-linearity, power-of-two and rank-permutation
invariants, bit-identical agreement in exact dyadic arithmetic, decoder
agreement with numpy's fp16 / fp32 conversions, and the packed layout on
hand-worked words. The backward (tests/test_oracle_backward_pins.py), the
MBOK layer and SVID (tests/test_oracle_mbok_pins.py,
tests/test_oracle_svid_pins.py) and the DBF factorisation in
``dbf_factorize.py`` (tests/test_oracle_factorize_pins.py) carry their own
pins. Every function here is pinned; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dbf_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libdbf_oracle.so")
_lib = None

X_F32 = 0
X_BF16 = 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    i64, vp, i32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
    lib.dbf_oracle_forward.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, i32, vp, i64,
                                       vp, i32, i32, vp, i32]
    lib.dbf_oracle_forward.restype = i32
    lib.dbf_oracle_backward.argtypes = [i64, i64, i64, i64, vp, vp, vp, vp, vp, vp, i32, vp, i32, i64,
                                        vp, vp, vp, vp, vp, vp, i32]
    lib.dbf_oracle_backward.restype = i32
    lib.dbf_oracle_mbok_forward.argtypes = [i64, i64, i64, vp, vp, vp, vp, i32, i64, vp]
    lib.dbf_oracle_mbok_forward.restype = i32
    lib.dbf_oracle_pack.argtypes = [vp, i64, i64, vp]
    lib.dbf_oracle_unpack.argtypes = [vp, i64, i64, vp]
    lib.dbf_oracle_f16_to_f64.argtypes = [ctypes.c_uint16]
    lib.dbf_oracle_f16_to_f64.restype = ctypes.c_double
    lib.dbf_oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.dbf_oracle_bf16_to_f64.restype = ctypes.c_double
    lib.dbf_oracle_f32_to_f64.argtypes = [ctypes.c_uint32]
    lib.dbf_oracle_f32_to_f64.restype = ctypes.c_double
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _act(x: np.ndarray):
    """(contiguous array, kind) for fp32 values or bf16 bit patterns."""
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), X_F32
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), X_BF16
    raise TypeError(f"activations must be float32 values or uint16 bf16 bits, got {x.dtype}")


def forward(layer, x: np.ndarray, rows: Optional[Sequence[int]] = None,
            y_in: Optional[np.ndarray] = None, accumulate: bool = False,
            nthreads: Optional[int] = None) -> np.ndarray:
    """y = [acc] y_in + dW x for the token rows 'rows' of x (all rows if None).

    layer: object with M, N, R, ell, b1 (int8 N x R), b2 (int8 R x M) and the
    fp16 bit patterns alpha [ell, N], beta [ell, R], gamma [ell, M].
    x: T x M, float32 values or uint16 bf16 bits. y_in: T x N likewise.
    Returns float64 [len(rows), N].
    """
    lib = _load()
    M, N, R, ell = int(layer.M), int(layer.N), int(layer.R), int(layer.ell)
    b1 = np.ascontiguousarray(layer.b1, dtype=np.int8)
    b2 = np.ascontiguousarray(layer.b2, dtype=np.int8)
    al = np.ascontiguousarray(layer.alpha, dtype=np.uint16).reshape(ell, N)
    be = np.ascontiguousarray(layer.beta, dtype=np.uint16).reshape(ell, R)
    ga = np.ascontiguousarray(layer.gamma, dtype=np.uint16).reshape(ell, M)
    assert b1.shape == (N, R) and b2.shape == (R, M)
    xa, xk = _act(x)
    assert xa.ndim == 2 and xa.shape[1] == M
    T = xa.shape[0]
    rws = np.arange(T, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    if rws.size and (rws.min() < 0 or rws.max() >= T):
        raise IndexError("row index out of range")
    out = np.zeros((rws.size, N), dtype=np.float64)
    if accumulate:
        ya, yk = _act(y_in)
        assert ya.shape == (T, N)
        yp = _ptr(ya)
    else:
        ya, yk, yp = None, 0, None
    rc = lib.dbf_oracle_forward(M, N, R, ell, _ptr(b1), _ptr(b2), _ptr(al), _ptr(be), _ptr(ga),
                                _ptr(xa), xk, _ptr(rws), rws.size, yp, yk, int(bool(accumulate)),
                                _ptr(out), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return out


class Grads:
    """Backward outputs (float64): dx [T, M], dalpha [ell, N], dbeta [ell, R],
    dgamma [ell, M], db1 [N, R], db2 [R, M] (None when not requested)."""

    def __init__(self, dx, dalpha, dbeta, dgamma, db1, db2):
        self.dx, self.dalpha, self.dbeta, self.dgamma, self.db1, self.db2 = dx, dalpha, dbeta, dgamma, db1, db2


def backward(layer, x: np.ndarray, dy: np.ndarray, want_signs: bool = False,
             nthreads: Optional[int] = None) -> Grads:
    """Gradients of a loss through the forward, given dy = dL/dy (T x N).

    The chain rule through the forward's own steps (LoRDBA page, section 2:
    the training pipeline differentiates this forward; the straight-through
    estimator hands the sign-matrix gradients db1, db2 to the latents). x and
    dy: float32 values or uint16 bf16 bits. Scale gradients and db1, db2 sum
    over all tokens; dx is per token. db1, db2 only when want_signs.
    """
    lib = _load()
    M, N, R, ell = int(layer.M), int(layer.N), int(layer.R), int(layer.ell)
    b1 = np.ascontiguousarray(layer.b1, dtype=np.int8)
    b2 = np.ascontiguousarray(layer.b2, dtype=np.int8)
    al = np.ascontiguousarray(layer.alpha, dtype=np.uint16).reshape(ell, N)
    be = np.ascontiguousarray(layer.beta, dtype=np.uint16).reshape(ell, R)
    ga = np.ascontiguousarray(layer.gamma, dtype=np.uint16).reshape(ell, M)
    assert b1.shape == (N, R) and b2.shape == (R, M)
    xa, xk = _act(x)
    da, dk = _act(dy)
    T = xa.shape[0]
    assert xa.shape == (T, M) and da.shape == (T, N)
    dx = np.zeros((T, M))
    dal, dbe, dga = np.zeros((ell, N)), np.zeros((ell, R)), np.zeros((ell, M))
    db1 = np.zeros((N, R)) if want_signs else None
    db2 = np.zeros((R, M)) if want_signs else None
    rc = lib.dbf_oracle_backward(M, N, R, ell, _ptr(b1), _ptr(b2), _ptr(al), _ptr(be), _ptr(ga),
                                 _ptr(xa), xk, _ptr(da), dk, T, _ptr(dx), _ptr(dal), _ptr(dbe), _ptr(dga),
                                 _ptr(db1) if want_signs else None, _ptr(db2) if want_signs else None,
                                 int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return Grads(dx, dal, dbe, dga, db1, db2)


def mbok_forward(layer, x: np.ndarray) -> np.ndarray:
    """Multi-boolean-kernel layer forward (Multi-Boolean Architectures page,
    section 2): y = sum_k s_out_k . (W_k (s_in_k . x)), fp64.

    layer: object with M, N, K, w (int8 +-1 [K, N, M]), s_in (fp16 bits
    [K, M]), s_out (fp16 bits [K, N]). x: T x M float32 or bf16 bits."""
    lib = _load()
    M, N, K = int(layer.M), int(layer.N), int(layer.K)
    w = np.ascontiguousarray(layer.w, dtype=np.int8)
    si = np.ascontiguousarray(layer.s_in, dtype=np.uint16).reshape(K, M)
    so = np.ascontiguousarray(layer.s_out, dtype=np.uint16).reshape(K, N)
    assert w.shape == (K, N, M)
    xa, xk = _act(x)
    T = xa.shape[0]
    assert xa.shape == (T, M)
    out = np.zeros((T, N))
    if lib.dbf_oracle_mbok_forward(M, N, K, _ptr(w), _ptr(si), _ptr(so), _ptr(xa), xk, T, _ptr(out)) != 0:
        raise ValueError("oracle rejected its arguments")
    return out


def svid(X: np.ndarray):
    """Sign-value-independent decomposition (DBF page, section 2: the SVID
    projection from OneBit used inside ADMM; Multi-Boolean Architectures
    page, section 2: W ~ W_bool . (s_out s_in^T) with W_bool = sign(W)):
    X ~ sign(X) . (s_out s_in^T) with s_out s_in^T the best rank-1
    approximation of |X| in the Frobenius norm. sign(0) = +1. The rank-1
    factor sigma u v^T (u, v >= 0, unit norm) is split evenly:
    s_out = sqrt(sigma) u, s_in = sqrt(sigma) v. fp64.
    Returns (signs int8 [n, m], s_out [n], s_in [m])."""
    X = np.asarray(X, dtype=np.float64)
    S = np.where(X < 0, -1, 1).astype(np.int8)
    U, sig, Vt = np.linalg.svd(np.abs(X), full_matrices=False)
    u, v = U[:, 0], Vt[0]
    if u.sum() < 0:   # the Perron vectors of a nonnegative matrix are nonnegative
        u, v = -u, -v
    r = np.sqrt(sig[0])
    return S, r * u, r * v


def mbok_extract(W: np.ndarray, K: int):
    """Successive SVID extraction of K boolean kernels (Multi-Boolean
    Architectures page, section 2: the first kernel takes the main
    information, the next ones the residuals): R_0 = W, kernel k = SVID of
    R_{k-1}, R_k = R_{k-1} - kernel k. Scales are rounded to fp16 before
    the residual is formed (the layer stores them in fp16). fp64.
    Returns (w int8 [K, n, m], s_out fp16 bits [K, n], s_in fp16 bits [K, m],
    residual norms [K + 1])."""
    R = np.asarray(W, dtype=np.float64).copy()
    ws, so, si, norms = [], [], [], [float(np.linalg.norm(R))]
    for _ in range(K):
        S, a, b = svid(R)
        a16 = a.astype(np.float16)
        b16 = b.astype(np.float16)
        R -= S * np.outer(a16.astype(np.float64), b16.astype(np.float64))
        ws.append(S)
        so.append(a16.view(np.uint16))
        si.append(b16.view(np.uint16))
        norms.append(float(np.linalg.norm(R)))
    return np.stack(ws), np.stack(so), np.stack(si), np.array(norms)


def ste_backward(db: np.ndarray, h: np.ndarray, tau: float) -> np.ndarray:
    """Straight-through estimator for latents h with signs B = sign(h) (LoRDBA
    page, section 2, training pipeline; the surrogate is not given there):
    dH = dB * s'(h) with s(h) = tanh(h / tau) for tau > 0, else the identity
    clipped to |h| <= 1. fp64."""
    h = np.asarray(h, dtype=np.float64)
    db = np.asarray(db, dtype=np.float64)
    if tau > 0:
        th = np.tanh(h / tau)
        return db * (1.0 - th * th) / tau
    return db * (np.abs(h) <= 1.0)


def forward_segmented(layers, seg_offsets, seg_adapter, x: np.ndarray,
                      y_in: Optional[np.ndarray] = None, accumulate: bool = False,
                      nthreads: Optional[int] = None) -> np.ndarray:
    """Segmented multi-adapter forward over tokens pre-sorted into segments.

    Tokens seg_offsets[s] .. seg_offsets[s+1]-1 use layers[seg_adapter[s]].
    An adapter id of -1 means "no adapter": those rows get a zero branch,
    i.e. y_in when accumulating and 0 otherwise. Returns float64 [T, N].
    """
    xa, _ = _act(x)
    T = xa.shape[0]
    N = int(layers[0].N)
    out = np.zeros((T, N), dtype=np.float64)
    if accumulate:
        ya, yk = _act(y_in)
        base = (ya.astype(np.float64) if yk == X_F32 else bf16_to_f64(ya))
    offs = [int(v) for v in seg_offsets]
    for s, a in enumerate(int(v) for v in seg_adapter):
        lo, hi = offs[s], offs[s + 1]
        if hi <= lo:
            continue
        rows = np.arange(lo, hi, dtype=np.int64)
        if a < 0:
            out[lo:hi] = base[lo:hi] if accumulate else 0.0
            continue
        out[lo:hi] = forward(layers[a], xa, rows=rows, y_in=y_in, accumulate=accumulate,
                             nthreads=nthreads)
    return out


def pack(s: np.ndarray) -> np.ndarray:
    """Packed words (uint32, rows x ceil(k/32)) of a rows x k sign matrix."""
    lib = _load()
    s = np.ascontiguousarray(s, dtype=np.int8)
    rows, k = s.shape
    out = np.zeros((rows, (k + 31) // 32), dtype=np.uint32)
    lib.dbf_oracle_pack(_ptr(s), rows, k, _ptr(out))
    return out


def unpack(w: np.ndarray, rows: int, k: int) -> np.ndarray:
    lib = _load()
    w = np.ascontiguousarray(w, dtype=np.uint32)
    assert w.size == rows * ((k + 31) // 32)
    out = np.zeros((rows, k), dtype=np.int8)
    lib.dbf_oracle_unpack(_ptr(w), rows, k, _ptr(out))
    return out


def sign_of_latent(h: np.ndarray) -> np.ndarray:
    """B = sign(H) of the QAT forward (LoRDBA page, section 2 training
    pipeline, step 2) with sign(0) = +1 and -0.0 -> +1; NaN raises."""
    h = np.asarray(h, dtype=np.float64)
    if np.isnan(h).any():
        raise ValueError("NaN latent")
    return np.where(h < 0, -1, 1).astype(np.int8)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint16)
    return np.array([lib.dbf_oracle_f16_to_f64(int(v)) for v in b.ravel()]).reshape(b.shape)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64. Small arrays go through the C decoder;
    large ones through the fp32 bit view (a bf16 pattern shifted left by 16
    is the fp32 pattern of the same real number)."""
    b = np.asarray(bits, dtype=np.uint16)
    if b.size > 4096:
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    lib = _load()
    return np.array([lib.dbf_oracle_bf16_to_f64(int(v)) for v in b.ravel()]).reshape(b.shape)


def f32_to_f64(bits: np.ndarray) -> np.ndarray:
    lib = _load()
    b = np.asarray(bits, dtype=np.uint32)
    return np.array([lib.dbf_oracle_f32_to_f64(int(v)) for v in b.ravel()]).reshape(b.shape)


from .dbf_factorize import Factors, admm_u_step, admm_v_step, factorize, rho_of, svd_init, svid_project  # noqa: E402
