"""Python binding of libdbf.so, the sm_100a double-binary layer forward.

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels (see include/dbf.h for the operation, layouts and errors).
PyTorch supplies device memory and the current CUDA stream. There is no CPU
fallback: if the shared library is missing, importing this package raises.
Build it with ``python double_binary_rank_b200/build.py``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdbf.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: the CUDA library must be built "
                      "(python double_binary_rank_b200/build.py); there is no CPU fallback")

_lib = ctypes.CDLL(LIB_PATH)

# ---- enums (dbf.h)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ALIGNMENT, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(7)
F32, BF16, F16, I8 = range(4)
PATH_AUTO, PATH_GEMV, PATH_GEMM = range(3)
ACCUMULATE, WEIGHTS_STATIC = 1, 2
_PATHS = {"auto": PATH_AUTO, "gemv": PATH_GEMV, "gemm": PATH_GEMM}
_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16, torch.int8: I8}


class DbfLayerC(ctypes.Structure):
    """dbf_layer of dbf.h."""
    _fields_ = [("M", ctypes.c_int32), ("N", ctypes.c_int32), ("R", ctypes.c_int32),
                ("ell", ctypes.c_int32), ("b1_packed", ctypes.c_void_p),
                ("b2_packed", ctypes.c_void_p), ("alpha", ctypes.c_void_p),
                ("beta", ctypes.c_void_p), ("gamma", ctypes.c_void_p)]


class DbfMbokLayerC(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("w_packed", ctypes.c_void_p), ("s_in", ctypes.c_void_p), ("s_out", ctypes.c_void_p)]


_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
_LP = ctypes.POINTER(DbfLayerC)
_SIGS = {
    "dbf_packed_bytes": (_sz, [_i64, _i64]),
    "dbf_pack_signs": (ctypes.c_int, [_vp, ctypes.c_int, _i64, _i64, _vp, _sz, _vp, _vp]),
    "dbf_unpack_signs": (ctypes.c_int, [_vp, _i64, _i64, _vp, _vp]),
    "dbf_transpose_signs": (ctypes.c_int, [_vp, _i64, _i64, _vp, _sz, _vp]),
    "dbf_svid_scratch_bytes": (_sz, [_i64, _i64, _i32]),
    "dbf_svid": (ctypes.c_int, [_vp, _i64, _i64, _i32, ctypes.c_int, _vp, _i64, _vp, _vp, _vp, _sz, _vp]),
    "dbf_svid_iterations": (ctypes.c_int, [_vp, _i64, _i64, _i32, ctypes.POINTER(ctypes.c_int32)]),
    "dbf_factorize_workspace_bytes": (_sz, [_i64, _i64, _i64, _i32, _i32]),
    "dbf_factorize": (ctypes.c_int, [_vp, _i64, _i64, _i64, _vp, _vp, _i32, _i32, _i32, ctypes.c_float, _vp, _vp,
                                     _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "dbf_gemm_min_tokens": (_i64, [ctypes.c_void_p]),
    "dbf_workspace_bytes": (_sz, [_LP, _i64, ctypes.c_int]),
    "dbf_forward_launches": (_i32, [_LP, _i64, ctypes.c_int]),
    "dbf_forward": (ctypes.c_int, [_LP, _vp, ctypes.c_int, _vp, ctypes.c_int, _i64, ctypes.c_int,
                                   ctypes.c_int, _vp, _sz, _vp]),
    "dbf_backward_workspace_bytes": (_sz, [_LP, _i64, ctypes.c_int]),
    "dbf_backward": (ctypes.c_int, [_LP, _vp, _vp, _vp, ctypes.c_int, _vp, ctypes.c_int, _i64, _vp, _vp, _vp,
                                    _vp, _vp, _vp, ctypes.c_int, _vp, _sz, _vp]),
    "dbf_ste_backward": (ctypes.c_int, [_vp, _vp, ctypes.c_int, _i64, ctypes.c_float, _vp, ctypes.c_int, _vp]),
    "dbf_forward_segmented_planned_workspace_bytes": (_sz, [_LP, _i32, _vp, _vp, _i32, _i32, _i32, _i64]),
    "dbf_forward_segmented_planned": (ctypes.c_int, [_LP, _i32, _vp, _vp, _i32, _i32, _i32, _vp, ctypes.c_int, _vp,
                                                     ctypes.c_int, _i64, ctypes.c_int, _vp, _sz, _vp]),
    "dbf_mbok_workspace_bytes": (_sz, [ctypes.POINTER(DbfMbokLayerC), _i64]),
    "dbf_mbok_forward": (ctypes.c_int, [ctypes.POINTER(DbfMbokLayerC), _vp, ctypes.c_int, _vp, ctypes.c_int, _i64,
                                        ctypes.c_int, _vp, _sz, _vp]),
    "dbf_segmented_workspace_bytes": (_sz, [_i32, _i32, _i64]),
    "dbf_forward_segmented": (ctypes.c_int, [_vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                             _vp, ctypes.c_int, _vp, ctypes.c_int, _i64,
                                             ctypes.c_int, _vp, _sz, _vp, _vp]),
    "dbf_forward_decode_noalloc": (ctypes.c_int, [_LP, _vp, ctypes.c_int, _vp, ctypes.c_int, _i64,
                                                  ctypes.c_int, _vp]),
    "dbf_debug_set_decode_wait_ns": (None, [ctypes.c_uint64]),
    "dbf_debug_noalloc_header": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_int32)]),
    "dbf_debug_fused_schedule": (ctypes.c_int, [_LP, _i64, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32),
                                                ctypes.POINTER(ctypes.c_double)]),
    "dbf_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dbf_version": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


class DbfError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.dbf_status_string(status).decode()} (status {status})")


def _check(status: int, where: str) -> None:
    if status != OK:
        raise DbfError(status, where)


def _stream(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def version() -> str:
    return _lib.dbf_version().decode()


def status_string(status: int) -> str:
    return _lib.dbf_status_string(status).decode()


def packed_bytes(rows: int, k: int) -> int:
    return int(_lib.dbf_packed_bytes(rows, k))


def gemm_min_tokens(layer) -> int:
    """Smallest T at which the AUTO path takes the GEMM kernels on this layer
    (-1: never)."""
    d = layer.descriptor()
    return int(_lib.dbf_gemm_min_tokens(ctypes.byref(d)))


def pack_signs(src: torch.Tensor, out: Optional[torch.Tensor] = None,
               status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Pack a rows x k int8 (+-1) or float latent tensor (dbf_pack_signs).

    Returns int32 words [rows, ceil(k/32)] (the uint32 bit patterns)."""
    rows, k = src.shape
    src = src.contiguous()
    if out is None:
        out = torch.empty((rows, (k + 31) // 32), dtype=torch.int32, device=src.device)
    _check(_lib.dbf_pack_signs(_ptr(src), _DT[src.dtype], rows, k, _ptr(out),
                               out.numel() * 4, _ptr(status), _stream(stream)), "dbf_pack_signs")
    return out


def unpack_signs(words: torch.Tensor, rows: int, k: int, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((rows, k), dtype=torch.int8, device=words.device)
    _check(_lib.dbf_unpack_signs(_ptr(words), rows, k, _ptr(out), _stream(stream)),
           "dbf_unpack_signs")
    return out


def transpose_signs(words: torch.Tensor, rows: int, k: int, out: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Packed rows x k -> packed k x rows (dbf_transpose_signs); int32 words
    [k, ceil(rows/32)]."""
    if out is None:
        out = torch.empty((k, (rows + 31) // 32), dtype=torch.int32, device=words.device)
    _check(_lib.dbf_transpose_signs(_ptr(words), rows, k, _ptr(out), out.numel() * 4, _stream(stream)),
           "dbf_transpose_signs")
    return out


@dataclass
class Layer:
    """Device-resident layer: packed signs (int32 words) and fp16 scales.

    b1: [N, ceil(R/32)] packed words; b2: [R, ceil(M/32)] packed words;
    alpha [ell, N], beta [ell, R], gamma [ell, M] as torch.float16 tensors.
    """
    M: int
    N: int
    R: int
    ell: int
    b1: torch.Tensor
    b2: torch.Tensor
    alpha: torch.Tensor
    beta: torch.Tensor
    gamma: torch.Tensor

    def descriptor(self) -> DbfLayerC:
        return DbfLayerC(self.M, self.N, self.R, self.ell, _ptr(self.b1), _ptr(self.b2),
                         _ptr(self.alpha), _ptr(self.beta), _ptr(self.gamma))

    @staticmethod
    def from_signs(b1_signs: torch.Tensor, b2_signs: torch.Tensor, alpha: torch.Tensor,
                   beta: torch.Tensor, gamma: torch.Tensor, stream=None) -> "Layer":
        """Pack +-1 sign matrices (N x R and R x M, on the device) into a Layer."""
        N, R = b1_signs.shape
        R2, M = b2_signs.shape
        assert R == R2
        ell = alpha.shape[0]
        return Layer(M, N, R, ell, pack_signs(b1_signs, stream=stream),
                     pack_signs(b2_signs, stream=stream), alpha.contiguous(), beta.contiguous(),
                     gamma.contiguous())


def workspace_bytes(layer: Layer, T: int, path: str = "auto") -> int:
    d = layer.descriptor()
    return int(_lib.dbf_workspace_bytes(ctypes.byref(d), T, _PATHS[path]))


def forward_launches(layer: Layer, T: int, path: str = "auto") -> int:
    d = layer.descriptor()
    return int(_lib.dbf_forward_launches(ctypes.byref(d), T, _PATHS[path]))


WS_HEADER_BYTES, WS_STATUS_OFFSET = 256, 8


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    # zeroed: the first 256 bytes are a header that must start at zero
    return torch.zeros(max(int(nbytes), WS_HEADER_BYTES), dtype=torch.uint8, device=device)


def workspace_status(ws: torch.Tensor) -> int:
    """The workspace header's device status word (DBF_ERR_TIMEOUT after a
    bounded device wait expired in a call on this workspace, else OK); reads
    it with a device-to-host copy on the current stream."""
    return int(ws[WS_STATUS_OFFSET:WS_STATUS_OFFSET + 4].view(torch.int32).item())


def clear_workspace_status(ws: torch.Tensor) -> None:
    ws[WS_STATUS_OFFSET:WS_STATUS_OFFSET + 4].zero_()


def debug_set_decode_wait_ns(ns: int) -> None:
    """Time limit of the single-launch decode kernel's bounded waits for later
    calls (0 restores the default of 2 s); for tests of the timeout path."""
    _lib.dbf_debug_set_decode_wait_ns(int(ns))


def debug_noalloc_header() -> Tuple[int, int]:
    """(barrier word, status) of the fixed array dbf_forward_decode_noalloc
    uses on the current device; waits for all work on the device."""
    word = ctypes.c_uint64(0)
    status = ctypes.c_int32(0)
    _check(_lib.dbf_debug_noalloc_header(ctypes.byref(word), ctypes.byref(status)), "dbf_debug_noalloc_header")
    return int(word.value), int(status.value)


def _flags(accumulate: bool, static_weights: bool) -> int:
    return (ACCUMULATE if accumulate else 0) | (WEIGHTS_STATIC if static_weights else 0)


def forward(layer: Layer, x: torch.Tensor, y: Optional[torch.Tensor] = None,
            accumulate: bool = False, path: str = "auto", ws: Optional[torch.Tensor] = None,
            y_dtype: Optional[torch.dtype] = None, static_weights: bool = False,
            stream=None) -> torch.Tensor:
    """y = [acc] y + dW x (dbf_forward). x: [T, M] float32/bfloat16 on the device.

    static_weights: the packed signs were not written by the preceding work
    on the stream (lets the kernels prefetch them across the kernel boundary)."""
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, layer.N), dtype=y_dtype or x.dtype, device=x.device)
    d = layer.descriptor()
    need = int(_lib.dbf_workspace_bytes(ctypes.byref(d), T, _PATHS[path]))
    if ws is None:
        ws = alloc_workspace(need, x.device)
    _check(_lib.dbf_forward(ctypes.byref(d), _ptr(x), _DT[x.dtype], _ptr(y), _DT[y.dtype], T,
                            _flags(accumulate, static_weights), _PATHS[path], _ptr(ws), ws.numel(),
                            _stream(stream)), "dbf_forward")
    return y


@dataclass
class Grads:
    dx: Optional[torch.Tensor]       # [T, M] fp32
    dalpha: Optional[torch.Tensor]   # [ell, N] fp32
    dbeta: Optional[torch.Tensor]    # [ell, R] fp32
    dgamma: Optional[torch.Tensor]   # [ell, M] fp32
    db1: Optional[torch.Tensor] = None   # [N, R] fp32, sign-matrix gradient
    db2: Optional[torch.Tensor] = None   # [R, M] fp32


def transposed_signs(layer: Layer, stream=None):
    """(B1^T packed along N, B2^T packed along R) for dbf_backward."""
    return (transpose_signs(layer.b1, layer.N, layer.R, stream=stream),
            transpose_signs(layer.b2, layer.R, layer.M, stream=stream))


def backward_workspace_bytes(layer: Layer, T: int, sign_grads: bool = False) -> int:
    d = layer.descriptor()
    return int(_lib.dbf_backward_workspace_bytes(ctypes.byref(d), T, int(sign_grads)))


def backward(layer: Layer, x: torch.Tensor, dy: torch.Tensor, signs_t=None, grads: Optional[Grads] = None,
             want=("dx", "dalpha", "dbeta", "dgamma"), accumulate: bool = False,
             ws: Optional[torch.Tensor] = None, stream=None) -> Grads:
    """Gradients through the forward given dy = dL/dy (dbf_backward).

    signs_t: (B1^T, B2^T) packed, from transposed_signs(layer) (computed here
    if None). grads: output tensors to write (or add to, with accumulate)."""
    T = x.shape[0]
    dev = x.device
    if signs_t is None:
        signs_t = transposed_signs(layer, stream=stream)
    if grads is None:
        mk = lambda name, shape: torch.empty(shape, dtype=torch.float32, device=dev) if name in want else None
        grads = Grads(mk("dx", (T, layer.M)), mk("dalpha", (layer.ell, layer.N)), mk("dbeta", (layer.ell, layer.R)),
                      mk("dgamma", (layer.ell, layer.M)), mk("db1", (layer.N, layer.R)), mk("db2", (layer.R, layer.M)))
    d = layer.descriptor()
    if ws is None:
        ws = alloc_workspace(backward_workspace_bytes(layer, T, grads.db1 is not None or grads.db2 is not None), dev)
    _check(_lib.dbf_backward(ctypes.byref(d), _ptr(signs_t[0]), _ptr(signs_t[1]), _ptr(x), _DT[x.dtype], _ptr(dy),
                             _DT[dy.dtype], T, _ptr(grads.dx), _ptr(grads.dalpha), _ptr(grads.dbeta),
                             _ptr(grads.dgamma), _ptr(grads.db1), _ptr(grads.db2), ACCUMULATE if accumulate else 0,
                             _ptr(ws), ws.numel(), _stream(stream)), "dbf_backward")
    return grads


def ste_backward(db: torch.Tensor, h: torch.Tensor, tau: float = 0.0, dh: Optional[torch.Tensor] = None,
                 accumulate: bool = False, stream=None) -> torch.Tensor:
    """dH = dB * s'(H) (dbf_ste_backward): s = tanh(H / tau) for tau > 0, else
    the identity clipped to |H| <= 1."""
    db = db.contiguous()
    h = h.contiguous()
    if dh is None:
        dh = torch.empty(h.shape, dtype=torch.float32, device=h.device)
    _check(_lib.dbf_ste_backward(_ptr(db), _ptr(h), _DT[h.dtype], h.numel(), float(tau), _ptr(dh),
                                 ACCUMULATE if accumulate else 0, _stream(stream)), "dbf_ste_backward")
    return dh


def segmented_planned_workspace_bytes(layers, seg_offsets, seg_adapter, M: int, N: int, T: int) -> int:
    arr = (DbfLayerC * max(1, len(layers)))(*[l.descriptor() for l in layers])
    offs = np.ascontiguousarray(seg_offsets, dtype=np.int32)
    ids = np.ascontiguousarray(seg_adapter, dtype=np.int32)
    return int(_lib.dbf_forward_segmented_planned_workspace_bytes(arr, len(layers), offs.ctypes.data, ids.ctypes.data,
                                                                  int(ids.size), M, N, T))


def forward_segmented_planned(layers, seg_offsets, seg_adapter, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                              accumulate: bool = False, ws: Optional[torch.Tensor] = None,
                              y_dtype: Optional[torch.dtype] = None, static_weights: bool = False,
                              stream=None) -> torch.Tensor:
    """Segmented forward with the segment tables on the host
    (dbf_forward_segmented_planned): one dbf_forward per segment, each on the
    path its token count calls for.

    layers: list of Layer; seg_offsets: S+1 ints; seg_adapter: S ints (-1 = none)."""
    T = x.shape[0]
    N = layers[0].N if layers else (y.shape[1] if y is not None else 0)
    M = x.shape[1]
    if y is None:
        y = torch.empty((T, N), dtype=y_dtype or x.dtype, device=x.device)
    arr = (DbfLayerC * max(1, len(layers)))(*[l.descriptor() for l in layers])
    offs = np.ascontiguousarray(seg_offsets, dtype=np.int32)
    ids = np.ascontiguousarray(seg_adapter, dtype=np.int32)
    S = int(ids.size)
    if ws is None:
        need = int(_lib.dbf_forward_segmented_planned_workspace_bytes(arr, len(layers), offs.ctypes.data,
                                                                      ids.ctypes.data, S, M, N, T))
        ws = alloc_workspace(need, x.device)
    _check(_lib.dbf_forward_segmented_planned(arr, len(layers), offs.ctypes.data, ids.ctypes.data, S, M, N, _ptr(x),
                                              _DT[x.dtype], _ptr(y), _DT[y.dtype], T,
                                              _flags(accumulate, static_weights), _ptr(ws), ws.numel(),
                                              _stream(stream)), "dbf_forward_segmented_planned")
    return y


def svid(X: torch.Tensor, iters: int = 24, subtract: bool = False, signs: Optional[torch.Tensor] = None,
         s_out: Optional[torch.Tensor] = None, s_in: Optional[torch.Tensor] = None,
         scratch: Optional[torch.Tensor] = None, stream=None):
    """X ~ sign(X) . (s_out s_in^T) (dbf_svid). X: fp32 [n, m] on the device,
    replaced by the residual when subtract. Returns (packed signs, s_out, s_in)."""
    assert X.dtype == torch.float32 and X.is_contiguous()
    n, m = X.shape
    dev = X.device
    if signs is None:
        signs = torch.empty((n, (m + 31) // 32), dtype=torch.int32, device=dev)
    if s_out is None:
        s_out = torch.empty(n, dtype=torch.float16, device=dev)
    if s_in is None:
        s_in = torch.empty(m, dtype=torch.float16, device=dev)
    if scratch is None:
        scratch = alloc_workspace(int(_lib.dbf_svid_scratch_bytes(n, m, iters)), dev)
    _check(_lib.dbf_svid(_ptr(X), n, m, iters, int(subtract), _ptr(signs), signs.stride(0), _ptr(s_out), _ptr(s_in),
                         _ptr(scratch), scratch.numel(), _stream(stream)), "dbf_svid")
    return signs, s_out, s_in


def svid_iterations(scratch: torch.Tensor, n: int, m: int, iters: int) -> int:
    """Power iterations the last svid call with this scratch ran (synchronous)."""
    out = ctypes.c_int32(0)
    _check(_lib.dbf_svid_iterations(_ptr(scratch), n, m, iters, ctypes.byref(out)), "dbf_svid_iterations")
    return int(out.value)


def factorize_workspace_bytes(n: int, m: int, k: int, outer: int, svid_iters: int = 24) -> int:
    return int(_lib.dbf_factorize_workspace_bytes(n, m, k, outer, svid_iters))


def factorize(W: torch.Tensor, U0: torch.Tensor, V0: torch.Tensor, outer: int, admm_iters: int = 4,
              svid_iters: int = 24, rho_rel: float = 1.0, objective: bool = True, ws: Optional[torch.Tensor] = None,
              stream=None):
    """Double binary factorisation W ~ (a . A . mid^T)(B . b^T) (dbf_factorize).
    W: fp32 [n, m]; U0: fp32 [n, k]; V0: fp32 [k, m], on the device. Returns
    (Layer with M = m, N = n, R = k, ell = 1, objective fp32 [outer + 1] or None)."""
    for t in (W, U0, V0):
        assert t.dtype == torch.float32 and t.is_contiguous()
    n, m = W.shape
    k = U0.shape[1]
    assert U0.shape == (n, k) and V0.shape == (k, m)
    dev = W.device
    b1 = torch.empty((n, (k + 31) // 32), dtype=torch.int32, device=dev)
    b2 = torch.empty((k, (m + 31) // 32), dtype=torch.int32, device=dev)
    alpha = torch.empty((1, n), dtype=torch.float16, device=dev)
    beta = torch.empty((1, k), dtype=torch.float16, device=dev)
    gamma = torch.empty((1, m), dtype=torch.float16, device=dev)
    obj = torch.empty(outer + 1, dtype=torch.float32, device=dev) if objective else None
    if ws is None:
        ws = alloc_workspace(factorize_workspace_bytes(n, m, k, outer, svid_iters), dev)
    _check(_lib.dbf_factorize(_ptr(W), n, m, k, _ptr(U0), _ptr(V0), outer, admm_iters, svid_iters, rho_rel,
                              _ptr(b1), _ptr(b2), _ptr(alpha), _ptr(beta), _ptr(gamma),
                              _ptr(obj) if obj is not None else None, _ptr(ws), ws.numel(), _stream(stream)),
           "dbf_factorize")
    return Layer(m, n, k, 1, b1, b2, alpha, beta, gamma), obj


@dataclass
class MbokLayer:
    """Device-resident multi-boolean-kernel layer: w [N, ceil(K M / 32)] packed
    words (row n = the K kernels' rows side by side), fp16 s_in [K, M] and
    s_out [K, N]."""
    M: int
    N: int
    K: int
    w: torch.Tensor
    s_in: torch.Tensor
    s_out: torch.Tensor

    @staticmethod
    def from_signs(w_signs: torch.Tensor, s_in: torch.Tensor, s_out: torch.Tensor, stream=None) -> "MbokLayer":
        """w_signs: int8 +-1 [K, N, M] on the device; scales fp16."""
        K, N, M = w_signs.shape
        cat = w_signs.permute(1, 0, 2).reshape(N, K * M).contiguous()
        return MbokLayer(M, N, K, pack_signs(cat, stream=stream), s_in.contiguous(), s_out.contiguous())

    def descriptor(self) -> DbfMbokLayerC:
        return DbfMbokLayerC(self.M, self.N, self.K, _ptr(self.w), _ptr(self.s_in), _ptr(self.s_out))

    @staticmethod
    def extract(W: torch.Tensor, K: int, iters: int = 24, stream=None) -> "MbokLayer":
        """K boolean kernels extracted successively from a dense fp32 weight
        W [N, M] (SVID of W, then of each residual); W is not modified."""
        N, M = W.shape
        R = W.float().clone().contiguous()
        words = (K * M + 31) // 32
        assert M % 32 == 0, "kernels side by side in a packed row need M % 32 == 0"
        w = torch.empty((N, words), dtype=torch.int32, device=W.device)
        s_out = torch.empty((K, N), dtype=torch.float16, device=W.device)
        s_in = torch.empty((K, M), dtype=torch.float16, device=W.device)
        for k in range(K):
            svid(R, iters, subtract=True, signs=w[:, k * (M // 32):], s_out=s_out[k], s_in=s_in[k], stream=stream)
        return MbokLayer(M, N, K, w, s_in, s_out)


def mbok_workspace_bytes(layer: MbokLayer, T: int) -> int:
    d = layer.descriptor()
    return int(_lib.dbf_mbok_workspace_bytes(ctypes.byref(d), T))


def mbok_forward(layer: MbokLayer, x: torch.Tensor, y: Optional[torch.Tensor] = None, accumulate: bool = False,
                 ws: Optional[torch.Tensor] = None, y_dtype: Optional[torch.dtype] = None,
                 stream=None) -> torch.Tensor:
    """y = [acc] y + sum_k s_out_k . (W_k (s_in_k . x)) (dbf_mbok_forward)."""
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, layer.N), dtype=y_dtype or x.dtype, device=x.device)
    d = layer.descriptor()
    if ws is None:
        ws = alloc_workspace(mbok_workspace_bytes(layer, T), x.device)
    _check(_lib.dbf_mbok_forward(ctypes.byref(d), _ptr(x), _DT[x.dtype], _ptr(y), _DT[y.dtype], T,
                                 ACCUMULATE if accumulate else 0, _ptr(ws), ws.numel(), _stream(stream)),
           "dbf_mbok_forward")
    return y


def forward_decode_noalloc(layer: Layer, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                           accumulate: bool = False, y_dtype: Optional[torch.dtype] = None,
                           stream=None) -> torch.Tensor:
    """Decode forward with the library's fixed scratch array instead of a
    workspace (dbf_forward_decode_noalloc), for callers that cannot allocate
    device memory. At most 1 MiB of decode workspace per call; calls that
    overlap on the GPU share the array and must be ordered by the caller."""
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, layer.N), dtype=y_dtype or x.dtype, device=x.device)
    d = layer.descriptor()
    _check(_lib.dbf_forward_decode_noalloc(ctypes.byref(d), _ptr(x), _DT[x.dtype], _ptr(y), _DT[y.dtype], T,
                                           _flags(accumulate, False), _stream(stream)),
           "dbf_forward_decode_noalloc")
    return y


class AdapterTable:
    """Device array of dbf_layer descriptors for segmented serving."""

    def __init__(self, layers: Sequence[Layer], device):
        self.layers = list(layers)
        n = len(self.layers)
        arr = (DbfLayerC * max(n, 1))(*[l.descriptor() for l in self.layers])
        raw = bytes(ctypes.string_at(ctypes.addressof(arr), ctypes.sizeof(arr)))
        self.dev = torch.frombuffer(bytearray(raw), dtype=torch.uint8).to(device)
        self.num = n
        self.max_R = max(l.R for l in self.layers)
        self.max_ell = max(l.ell for l in self.layers)
        self.M = self.layers[0].M
        self.N = self.layers[0].N


def segmented_workspace_bytes(max_R: int, max_ell: int, T: int) -> int:
    return int(_lib.dbf_segmented_workspace_bytes(max_R, max_ell, T))


def forward_segmented(table: AdapterTable, seg_offsets: torch.Tensor, seg_adapter: torch.Tensor,
                      x: torch.Tensor, y: Optional[torch.Tensor] = None, accumulate: bool = False,
                      ws: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                      y_dtype: Optional[torch.dtype] = None, stream=None) -> torch.Tensor:
    """Segmented multi-adapter forward (dbf_forward_segmented)."""
    T = x.shape[0]
    S = seg_adapter.numel()
    if y is None:
        y = torch.empty((T, table.N), dtype=y_dtype or x.dtype, device=x.device)
    need = segmented_workspace_bytes(table.max_R, table.max_ell, T)
    if ws is None:
        ws = alloc_workspace(need, x.device)
    _check(_lib.dbf_forward_segmented(_ptr(table.dev), table.num, _ptr(seg_offsets),
                                      _ptr(seg_adapter), S, table.max_R, table.max_ell, table.M,
                                      table.N, _ptr(x), _DT[x.dtype], _ptr(y), _DT[y.dtype], T,
                                      _flags(accumulate, False), _ptr(ws), ws.numel(), _ptr(status),
                                      _stream(stream)), "dbf_forward_segmented")
    return y
