"""dbf_forward_decode_noalloc: the decode forward for callers that cannot
allocate device memory (a runtime that owns every allocation, or a thread
that must not call cudaMalloc). It takes its scratch from a fixed device
array in the library instead of a caller workspace. Its output must match
dbf_forward's, and the oracle's, on calls in a row (the array is shared
between calls and keeps the previous call's contents). Collected last on
purpose: if it fails, a run that stops at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest
import torch

import dbf_synth as S
from gpu_util import TOL, dev_layer, dev_x, host_y, random_layer, rel_err

pytestmark = pytest.mark.gpu


def _call_noalloc(dbf, layer, x, y):
    d = layer.descriptor()
    return dbf._lib.dbf_forward_decode_noalloc(ctypes.byref(d), x.data_ptr(), dbf.BF16 if x.dtype == torch.bfloat16 else dbf.F32,
                                               y.data_ptr(), dbf.F32, x.shape[0], 0,
                                               torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_forward_twice():
    import double_binary_rank_b200 as dbf
    import oracle
    rng = np.random.default_rng(81)
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    # T = 1, 2, 16: the single-launch kernel (several calls sharing the
    # array's barrier word)
    for call, T in enumerate((1, 2, 16, 1, 2)):
        xh = S.make_x(w.seed + call, T, w.M, "bf16")
        x = dev_x(xh)
        ref = dbf.forward(dl, x, path="gemv", y_dtype=torch.float32)
        y = torch.full((T, w.N), float("nan"), device="cuda")
        st = _call_noalloc(dbf, dl, x, y)
        torch.cuda.synchronize()
        assert st == dbf.OK, dbf.status_string(st)
        got = host_y(y)
        assert rel_err(got, host_y(ref)) < TOL
        assert rel_err(got, oracle.forward(L, xh)) < TOL
    # between calls the array's header holds a barrier word with no arrivals
    # pending (the epoch moved on) and a clean status word
    word, status = dbf.debug_noalloc_header()
    assert word & 0xFFFFFFFF == 0 and word >> 32 > 0 and status == 0
    epoch = word >> 32
    # a layer wider than the single launch takes (M > 8192): the two-launch
    # path through the same array, then a single launch again
    Lw = random_layer(rng, 8224, 256, 96, 1)
    dw = dev_layer(Lw)
    xwh = S.to_bf16_bits(rng.standard_normal((2, 8224)))
    yw = torch.zeros((2, 256), device="cuda")
    assert dbf._lib.dbf_forward_launches(ctypes.byref(dw.descriptor()), 2, dbf.PATH_GEMV) == 2
    assert _call_noalloc(dbf, dw, dev_x(xwh), yw) == dbf.OK
    torch.cuda.synchronize()
    assert rel_err(host_y(yw), oracle.forward(Lw, xwh)) < TOL
    # a second layer shape right after, through the same array
    L2 = random_layer(rng, 300, 170, 96, 2)
    d2 = dev_layer(L2)
    x2h = S.to_bf16_bits(rng.standard_normal((3, 300)))
    x2 = dev_x(x2h)
    ref2 = dbf.forward(d2, x2, path="gemv", y_dtype=torch.float32)
    y2 = torch.zeros((3, 170), device="cuda")
    assert _call_noalloc(dbf, d2, x2, y2) == dbf.OK
    torch.cuda.synchronize()
    assert rel_err(host_y(y2), host_y(ref2)) < TOL
    assert rel_err(host_y(y2), oracle.forward(L2, x2h)) < TOL
    word, status = dbf.debug_noalloc_header()
    assert word & 0xFFFFFFFF == 0 and word >> 32 > epoch and status == 0


def test_noalloc_rejects_calls_beyond_its_scratch():
    import double_binary_rank_b200 as dbf
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    T = 256   # this layer's decode workspace at 256 tokens exceeds the 1 MiB array
    x = torch.zeros((T, w.M), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((T, w.N), device="cuda")
    assert _call_noalloc(dbf, dl, x, y) == dbf.ERR_WORKSPACE
