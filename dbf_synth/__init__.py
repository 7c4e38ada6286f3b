"""Seeded synthetic inputs for the double-binary layer forward.

This module is shared by the CUDA path's tests and benchmark and by the fp64
oracle's tests. It holds no arithmetic of the method itself: it only draws
numbers (signs, activations, scales, adapter ids) and rounds them to the
storage types the layer consumes.

Generator
---------
Counter-based splitmix64. A stream is named by a key derived from
(seed, tensor tag, adapter, envelope); element ``i`` of the stream is
``mix64(key + (i + 1) * 0x9E3779B97F4A7C15)`` with the splitmix64 finaliser
``mix64``. Everything below is a deterministic function of those words:

* uniform double: top 53 bits times 2**-53;
* normal: Box-Muller on a pair of words (cos and sin branches give two values);
* sign: one bit of a word, 64 signs per word, bit set -> -1;
* bf16: float64 -> float32 (RNE) -> bf16 (RNE on the float32 bits);
* fp16 scale: exp(sigma * normal) rounded RNE to fp16.

Workload shapes follow the double-binary layer configurations of the LoRDBA
page ("Arquitetura Central": B1 is N x R, B2 is R x M, scales per channel) and
the DBF page (section 2, the W ~ (a . A . m^T)(B . b^T) form), at Llama-7B
projection / MLP sizes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK64 = (1 << 64) - 1

# tensor tags used to derive independent streams
TAG_X = 1
TAG_B1 = 2
TAG_B2 = 3
TAG_ALPHA = 4
TAG_BETA = 5
TAG_GAMMA = 6
TAG_IDS = 7
TAG_YIN = 8
TAG_WEIGHT = 9
TAG_WROW = 10
TAG_WCOL = 11
TAG_U0 = 12
TAG_V0 = 13

BASE_SEED = 0xDBF00000


def _mix64_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tag: int, adapter: int = 0, envelope: int = 0) -> int:
    """Key of one named stream; distinct tuples give unrelated streams."""
    k = _mix64_int(seed)
    for part in (tag, adapter, envelope):
        k = _mix64_int(k ^ ((part + 0x632BE59BD9B4E019) & _MASK64))
    return k


def raw_u64(key: int, n: int, offset: int = 0) -> np.ndarray:
    """Words ``offset .. offset+n-1`` of the stream ``key`` (uint64)."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        z = np.uint64(key) + i * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform(key: int, n: int) -> np.ndarray:
    """n doubles in [0, 1)."""
    return (raw_u64(key, n) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(key: int, n: int) -> np.ndarray:
    """n standard normal doubles (Box-Muller, both branches)."""
    npair = (n + 1) // 2
    w = raw_u64(key, 2 * npair)
    u1 = ((w[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
    u2 = (w[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)          # [0, 1)
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * math.pi * u2
    out = np.empty(2 * npair, dtype=np.float64)
    out[0::2] = rad * np.cos(ang)
    out[1::2] = rad * np.sin(ang)
    return out[:n]


def signs(key: int, rows: int, cols: int) -> np.ndarray:
    """rows x cols int8 matrix of +-1 (iid, p = 1/2); stream bit set -> -1."""
    n = rows * cols
    words = raw_u64(key, (n + 63) // 64)
    bits = np.unpackbits(words.view(np.uint8), bitorder="little")[:n]
    s = (1 - 2 * bits.astype(np.int8)).astype(np.int8)
    return s.reshape(rows, cols)


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """float64/float32 -> bf16 bit patterns (uint16), RNE via float32."""
    f = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (f >> np.uint64(16)) & np.uint64(1)
    r = (f + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f16_bits(v: np.ndarray) -> np.ndarray:
    """float64 -> fp16 bit patterns (uint16), RNE."""
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def lognormal_f16_bits(key: int, n: int, sigma: float) -> np.ndarray:
    return to_f16_bits(np.exp(sigma * normal(key, n)))


# ----------------------------------------------------------------------------
# layer / workload containers


@dataclasses.dataclass
class Layer:
    """One double-binary layer or adapter, host side, unpacked.

    b1: int8 +-1, N x R.  b2: int8 +-1, R x M.
    alpha/beta/gamma: fp16 bit patterns (uint16), shapes [ell, N] / [ell, R] / [ell, M].
    """
    M: int
    N: int
    R: int
    ell: int
    b1: np.ndarray
    b2: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    gamma: np.ndarray


def make_layer(seed: int, M: int, N: int, R: int, ell: int, sigma: float,
               adapter: int = 0) -> Layer:
    b1 = signs(stream_key(seed, TAG_B1, adapter), N, R)
    b2 = signs(stream_key(seed, TAG_B2, adapter), R, M)
    alpha = np.stack([lognormal_f16_bits(stream_key(seed, TAG_ALPHA, adapter, i), N, sigma)
                      for i in range(ell)])
    beta = np.stack([lognormal_f16_bits(stream_key(seed, TAG_BETA, adapter, i), R, sigma)
                     for i in range(ell)])
    gamma = np.stack([lognormal_f16_bits(stream_key(seed, TAG_GAMMA, adapter, i), M, sigma)
                      for i in range(ell)])
    return Layer(M, N, R, ell, b1, b2, alpha, beta, gamma)


def make_x(seed: int, T: int, M: int, dtype: str, tag: int = TAG_X) -> np.ndarray:
    """Activations T x M ~ N(0,1): fp32 array (dtype 'f32') or bf16 bits ('bf16')."""
    v = normal(stream_key(seed, tag), T * M).reshape(T, M)
    if dtype == "f32":
        return v.astype(np.float32)
    if dtype == "bf16":
        return to_bf16_bits(v)
    raise ValueError(dtype)


@dataclasses.dataclass
class MbokLayer:
    """A multi-boolean-kernel layer, host side: K sign kernels w [K, N, M]
    (int8 +-1) with fp16 bit patterns s_in [K, M] and s_out [K, N]."""
    M: int
    N: int
    K: int
    w: np.ndarray
    s_in: np.ndarray
    s_out: np.ndarray


def make_weight(seed: int, n: int, m: int, sigma: float = 0.25) -> np.ndarray:
    """A dense fp32 weight n x m with the row and column scale structure of
    trained layers: W[i, j] = g[i, j] r[i] c[j], g ~ N(0, 1), r and c
    lognormal with parameter sigma."""
    g = normal(stream_key(seed, TAG_WEIGHT), n * m).reshape(n, m)
    r = np.exp(sigma * normal(stream_key(seed, TAG_WROW), n))
    c = np.exp(sigma * normal(stream_key(seed, TAG_WCOL), m))
    return (g * r[:, None] * c[None, :]).astype(np.float32)


def make_factor_start(seed: int, n: int, m: int, k: int, scale: float = 1.0):
    """A seeded random start (U0 n x k, V0 k x m, fp32) for the
    factorisation: N(0, s^2) entries with s = sqrt(scale) k^-1/4, so that
    U0 V0 has entries of about 'scale'."""
    s = np.sqrt(scale) * k ** -0.25
    U0 = (s * normal(stream_key(seed, TAG_U0), n * k)).astype(np.float32).reshape(n, k)
    V0 = (s * normal(stream_key(seed, TAG_V0), k * m)).astype(np.float32).reshape(k, m)
    return U0, V0


def make_mbok_layer(seed: int, M: int, N: int, K: int, sigma: float = 0.5) -> MbokLayer:
    """Seeded MBOK layer: iid +-1 kernels, lognormal(0, sigma) fp16 scales."""
    w = np.stack([signs(stream_key(seed, 0x31, k, 0), N, M) for k in range(K)])
    s_in = np.stack([lognormal_f16_bits(stream_key(seed, 0x32, k, 0), M, sigma) for k in range(K)])
    s_out = np.stack([lognormal_f16_bits(stream_key(seed, 0x33, k, 0), N, sigma) for k in range(K)])
    return MbokLayer(M, N, K, w, s_in, s_out)


@dataclasses.dataclass
class Segments:
    """Tokens sorted by adapter id into contiguous segments."""
    offsets: np.ndarray   # int32 [S+1], offsets[0] = 0, offsets[S] = T
    adapter: np.ndarray   # int32 [S]
    order: np.ndarray     # int64 [T], original token index of each sorted row


def make_segments(seed: int, T: int, num_adapters: int) -> Segments:
    ids = (raw_u64(stream_key(seed, TAG_IDS), T) % np.uint64(num_adapters)).astype(np.int64)
    order = np.argsort(ids, kind="stable")
    sorted_ids = ids[order]
    uniq, counts = np.unique(sorted_ids, return_counts=True)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return Segments(offsets=offsets, adapter=uniq.astype(np.int32), order=order)


# ----------------------------------------------------------------------------
# the five workload shapes (names describe the layer, sizes are fixed)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int            # seed = BASE_SEED + index
    M: int
    N: int
    R: int
    ell: int
    tokens: Tuple[int, ...]
    x_dtype: str          # 'f32' or 'bf16'
    sigma: float
    num_adapters: int = 1
    description: str = ""

    @property
    def seed(self) -> int:
        return BASE_SEED + self.index


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 256, 256, 16, 1, (4,), "f32", 0.25,
                     description="tiny double-binary layer M=N=256, R=16, ell=1, 4 tokens, fp32 x"),
    "adapter": Workload("adapter", 2, 4096, 4096, 64, 1, (1, 4, 16, 64), "bf16", 0.5,
                        description="LoRDBA adapter branch, Llama-7B projection M=N=4096, R=64, ell=1"),
    "dbf_mlp": Workload("dbf_mlp", 3, 4096, 11008, 5888, 1, (1, 2048), "bf16", 0.5,
                        description="DBF full-weight MLP layer 4096->11008, R=5888 (~1.97 bits/weight)"),
    "segmented": Workload("segmented", 4, 4096, 4096, 32, 2, (256,), "bf16", 0.5, num_adapters=32,
                          description="32 LoRDBA adapters M=N=4096, R=32, ell=2, 256 tokens routed by id"),
    "large_prefill": Workload("large_prefill", 5, 8192, 8192, 8192, 1, (8192,), "bf16", 0.5,
                              description="large DBF prefill layer M=N=R=8192, 8192 tokens"),
}


def workload_layers(w: Workload) -> List[Layer]:
    return [make_layer(w.seed, w.M, w.N, w.R, w.ell, w.sigma, adapter=a)
            for a in range(w.num_adapters)]


def sample_rows(seed: int, T: int, n: int) -> np.ndarray:
    """A fixed, sorted subset of n token rows of T, always holding 0 and T-1."""
    if n >= T:
        return np.arange(T, dtype=np.int64)
    key = stream_key(seed, 0x5A, 0, 0)
    r = raw_u64(key, 4 * n)
    picks = {0, T - 1}
    for v in r:
        if len(picks) >= n:
            break
        picks.add(int(v % np.uint64(T)))
    return np.array(sorted(picks), dtype=np.int64)


def sample_rows_per_tile(seed: int, T: int, n: int, tile: int) -> np.ndarray:
    """A fixed, sorted subset of n token rows of T, stratified over tiles of
    'tile' consecutive rows: every tile holds at least floor(n / tiles) rows
    (at least one when n >= tiles), and 0 and T-1 are always included."""
    tiles = (T + tile - 1) // tile
    if n >= T:
        return np.arange(T, dtype=np.int64)
    if n < max(2, tiles):
        raise ValueError("fewer rows than tiles")
    key = stream_key(seed, 0x5B, 0, 0)
    words = iter(raw_u64(key, 64 * n + 64).tolist())
    picks = {0, T - 1}
    per = n // tiles
    for t in range(tiles):
        lo, hi = t * tile, min(T, (t + 1) * tile)
        have = sum(1 for p in picks if lo <= p < hi)
        while have < per:
            r = lo + next(words) % (hi - lo)
            if r not in picks:
                picks.add(r)
                have += 1
    while len(picks) < n:
        r = next(words) % T
        picks.add(r)
    return np.array(sorted(picks), dtype=np.int64)
