"""dbf_forward_segmented on the GPU against the oracle's segmented routing."""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import TOL, dev_layer, dev_x, host_y, random_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def i32(a):
    return torch.tensor(np.asarray(a, dtype=np.int32), device="cuda")


def test_segmented_workload_full(dbf):
    w = S.WORKLOADS["segmented"]
    layers = S.workload_layers(w)
    seg = S.make_segments(w.seed, 256, w.num_adapters)
    x = S.make_x(w.seed, 256, w.M, "bf16")[seg.order]
    ref = oracle.forward_segmented(layers, seg.offsets, seg.adapter, x)
    table = dbf.AdapterTable([dev_layer(L) for L in layers], "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = dbf.forward_segmented(table, i32(seg.offsets), i32(seg.adapter), dev_x(x),
                              y_dtype=torch.float32, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert rel_err(host_y(y), ref) < TOL


@pytest.mark.parametrize("acc", [False, True])
def test_segmented_edge_cases(dbf, acc):
    rng = np.random.default_rng(60)
    M, N = 200, 90
    layers = [random_layer(rng, M, N, R, ell) for R, ell in ((17, 1), (64, 2), (5, 3))]
    T = 13
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    offsets = [0, 4, 4, 9, 10, 13]     # an empty segment
    adapter = [1, 0, 2, -1, 0]          # a no-adapter segment
    ref = oracle.forward_segmented(layers, offsets, adapter, x, y_in=y_in, accumulate=acc)
    table = dbf.AdapterTable([dev_layer(L) for L in layers], "cuda")
    y = torch.from_numpy(y_in).cuda() if acc else None
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = dbf.forward_segmented(table, i32(offsets), i32(adapter), dev_x(x), y=y, accumulate=acc,
                                y_dtype=torch.float32, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert rel_err(host_y(out), ref) < TOL


def test_segmented_bad_adapter_sets_status(dbf):
    rng = np.random.default_rng(61)
    layers = [random_layer(rng, 64, 32, 16, 1) for _ in range(2)]
    table = dbf.AdapterTable([dev_layer(L) for L in layers], "cuda")
    x = dev_x(S.to_bf16_bits(rng.standard_normal((6, 64))))
    y = torch.full((6, 32), 3.0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dbf.forward_segmented(table, i32([0, 3, 6]), i32([0, 5]), x, y=y, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == dbf.ERR_INVALID_ARG
    # the bad segment is skipped: its rows keep their old values
    assert torch.all(y[3:] == 3.0)
    xh = x.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = oracle.forward(layers[0], xh, rows=[0, 1, 2])
    assert rel_err(host_y(y[:3]), ref) < TOL


def test_segmented_bad_offsets_sets_status(dbf):
    rng = np.random.default_rng(62)
    layers = [random_layer(rng, 64, 32, 16, 1)]
    table = dbf.AdapterTable([dev_layer(L) for L in layers], "cuda")
    x = dev_x(S.to_bf16_bits(rng.standard_normal((6, 64))))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dbf.forward_segmented(table, i32([0, 4, 9]), i32([0, 0]), x, y_dtype=torch.float32, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == dbf.ERR_INVALID_ARG
