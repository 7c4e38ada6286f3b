"""dbf_forward on the GPU against the fp64 oracle.

Tolerance: max|y - y_ref| / max|y_ref| <= 2e-3 for fp32 outputs; bf16
outputs within half a bf16 ulp of y_ref plus that bound. Exact dyadic
inputs must give bit-identical fp32 results, and the matched sign-flip and
power-of-two invariants must hold bit for bit on the GPU as well.
"""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import TOL, bf16_ok, dev_layer, dev_x, host_y, random_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def run(dbf, L, x, path="gemv", y_dtype=torch.float32, acc=False, y_in=None, dl=None):
    dl = dl or dev_layer(L)
    xd = dev_x(x)
    y = None
    if acc:
        y = torch.from_numpy(y_in).cuda().to(y_dtype)
    out = dbf.forward(dl, xd, y=y, accumulate=acc, path=path, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return host_y(out)


@pytest.mark.parametrize("y_dtype", [torch.float32, torch.bfloat16])
def test_tiny_workload(dbf, y_dtype):
    w = S.WORKLOADS["tiny"]
    L = S.workload_layers(w)[0]
    x = S.make_x(w.seed, 4, w.M, "f32")
    ref = oracle.forward(L, x)
    got = run(dbf, L, x, y_dtype=y_dtype)
    if y_dtype == torch.float32:
        assert rel_err(got, ref) < 1e-4          # 22-bit fixed point per column: far below 2e-3
    else:
        ok, worst = bf16_ok(got, ref)
        assert ok, worst


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_adapter_workload(dbf, T):
    w = S.WORKLOADS["adapter"]
    L = S.workload_layers(w)[0]
    x = S.make_x(w.seed, T, w.M, "bf16")
    ref = oracle.forward(L, x)
    got = run(dbf, L, x)
    err = rel_err(got, ref)
    assert err < TOL
    if T <= 4:
        assert err < 1e-4


def test_dbf_mlp_decode(dbf):
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    x = S.make_x(w.seed, 1, w.M, "bf16")
    ref = oracle.forward(L, x)
    got = run(dbf, L, x)
    assert rel_err(got, ref) < 1e-4
    got_b = run(dbf, L, x, y_dtype=torch.bfloat16)
    ok, worst = bf16_ok(got_b, ref)
    assert ok, worst


CASES = [  # M, N, R, ell, T  -- ragged sizes: not multiples of 16 / 32 / 512
    (1, 1, 1, 1, 1), (33, 17, 5, 1, 3), (100, 70, 48, 2, 2), (513, 129, 65, 3, 5),
    (1000, 300, 530, 1, 9), (64, 48, 1, 1, 4), (2048, 40, 700, 2, 1), (96, 1025, 128, 4, 1),
    (300, 200, 100, 8, 2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "M{}N{}R{}l{}T{}".format(*c))
@pytest.mark.parametrize("acc", [False, True])
def test_random_shapes(dbf, case, acc):
    M, N, R, ell, T = case
    rng = np.random.default_rng(M * 31 + N * 7 + R + ell + T)
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    y_in = rng.standard_normal((T, N)).astype(np.float32)
    ref = oracle.forward(L, x, y_in=y_in, accumulate=acc)
    got = run(dbf, L, x, acc=acc, y_in=y_in)
    assert rel_err(got, ref) < TOL
    assert rel_err(got, ref) < 1e-4


@pytest.mark.parametrize("T", [1, 2, 7])
def test_exact_dyadic_bit_identical(dbf, T):
    # integer x, power-of-two scales: every partial sum, both fp16 parts and the
    # fp32 accumulations are exact, so the GPU result equals the oracle's
    rng = np.random.default_rng(40 + T)
    M, N, R = 48, 72, 40
    L = random_layer(rng, M, N, R, 1, dyadic=True)
    x = rng.integers(-2, 3, size=(T, M)).astype(np.float32)
    ref = oracle.forward(L, x)
    got = run(dbf, L, x)
    assert np.array_equal(got, ref)


def test_matched_sign_flip_bit_identical(dbf):
    rng = np.random.default_rng(50)
    L = random_layer(rng, 700, 300, 90, 2)
    x = S.to_bf16_bits(rng.standard_normal((2, 700)))
    y0 = run(dbf, L, x)
    flip = rng.random(90) < 0.5
    L.b1[:, flip] *= -1
    L.b2[flip, :] *= -1
    y1 = run(dbf, L, x)
    assert np.array_equal(y0, y1)


def test_power_of_two_alpha_bit_exact(dbf):
    rng = np.random.default_rng(51)
    L = random_layer(rng, 700, 300, 90, 1)
    x = S.to_bf16_bits(rng.standard_normal((3, 700)))
    y0 = run(dbf, L, x)
    L.alpha[:] = S.to_f16_bits(2.0 * L.alpha.view(np.float16).astype(np.float64))
    y1 = run(dbf, L, x)
    assert np.array_equal(y1, 2.0 * y0)


def test_envelope_linearity(dbf):
    rng = np.random.default_rng(52)
    L = random_layer(rng, 256, 128, 64, 2)
    x = S.to_bf16_bits(rng.standard_normal((2, 256)))
    y2 = run(dbf, L, x)
    parts = [run(dbf, S.Layer(L.M, L.N, L.R, 1, L.b1, L.b2, L.alpha[i:i + 1], L.beta[i:i + 1],
                              L.gamma[i:i + 1]), x) for i in range(2)]
    assert rel_err(y2, parts[0] + parts[1]) < 1e-4


@pytest.mark.parametrize("static", [False, True])
def test_back_to_back_calls_static_weights(dbf, static):
    # many calls queued on one stream, each a programmatic dependent of the
    # previous one; with static weights the sign prefetch crosses the kernel
    # boundary. Every call must still see the previous call's output (the
    # chain feeds y back as the next x) and match the oracle.
    rng = np.random.default_rng(56)
    M = N = 640
    L = random_layer(rng, M, N, 96, 1, sigma=0.1)
    dl = dev_layer(L)
    x0 = S.to_bf16_bits(rng.standard_normal((2, M)))
    xs = dev_x(x0).float()
    torch.cuda.synchronize()
    outs = []
    cur = xs
    for _ in range(4):
        cur = dbf.forward(dl, cur, y_dtype=torch.float32, static_weights=static)
        outs.append(cur)
    torch.cuda.synchronize()
    ref = x0
    for k in range(4):
        r = oracle.forward(L, ref if k == 0 else ref.astype(np.float32))
        got = host_y(outs[k])
        assert rel_err(got, r) < 1e-4
        ref = got.astype(np.float32)


def test_zero_tokens_noop(dbf):
    rng = np.random.default_rng(53)
    L = random_layer(rng, 64, 32, 16, 1)
    dl = dev_layer(L)
    x = torch.empty((0, 64), device="cuda")
    y = dbf.forward(dl, x)
    assert y.shape == (0, 32)


def test_host_errors_with_device_buffers(dbf):
    rng = np.random.default_rng(54)
    L = random_layer(rng, 64, 32, 16, 1)
    dl = dev_layer(L)
    x = torch.zeros((4, 65), device="cuda")[:, 1:]          # misaligned rows
    with pytest.raises(dbf.DbfError) as e:
        dbf.forward(dl, x)
    assert e.value.status == dbf.ERR_ALIGNMENT
    x = torch.zeros((4, 64), device="cuda")
    with pytest.raises(dbf.DbfError) as e:
        dbf.forward(dl, x, ws=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == dbf.ERR_WORKSPACE
    with pytest.raises(dbf.DbfError) as e:
        dbf.forward(dl, x, path="gemm")
    assert e.value.status == dbf.ERR_UNSUPPORTED


def test_output_guard_bytes_untouched(dbf):
    # y is a slice of a larger buffer; nothing outside the slice may change
    rng = np.random.default_rng(55)
    L = random_layer(rng, 130, 50, 33, 1)
    dl = dev_layer(L)
    x = dev_x(S.to_bf16_bits(rng.standard_normal((3, 130))))
    buf = torch.full((3 * 50 + 64,), 7.25, device="cuda")
    y = buf[32:32 + 150].view(3, 50)
    dbf.forward(dl, x, y=y)
    torch.cuda.synchronize()
    b = buf.cpu().numpy()
    assert np.all(b[:32] == 7.25) and np.all(b[182:] == 7.25)
