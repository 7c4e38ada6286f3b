"""The single-launch decode path (one layer or segmented adapters, M <=
8192) against the fp64 oracle.

That path exchanges the rank-R intermediate through a grid-wide barrier
whose word lives in the workspace header (arrival count in the low 32 bits,
epoch in the high 32 bits), so besides plain parity these tests check that
many calls sharing one workspace (with different grid sizes) stay correct,
that every call leaves the arrival count at zero and advances the epoch by
one, that a barrier wait that runs out of time is reported in the header's
status word and leaves the workspace usable, the chunking of many tokens
(ragged last chunks, several items per CTA), segments of adapters with
different ranks and envelope counts, and the limits where the library
switches to the two-launch path (M above 8192, more than 512 segments).
"""
import numpy as np
import pytest
import torch

import dbf_synth as S
import oracle
from gpu_util import dev_layer, dev_x, host_y, random_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbf():
    import double_binary_rank_b200 as m
    return m


def header_words(ws):
    """(arrival count, epoch) of the header's barrier word."""
    lo, hi = ws[:8].view(torch.int32).cpu().tolist()
    return lo & 0xFFFFFFFF, hi & 0xFFFFFFFF


@pytest.mark.parametrize("T,ell", [(8, 1), (4, 2), (1, 8), (2, 3), (9, 1), (3, 3)])
def test_token_envelope_mix(dbf, T, ell):
    # chunks of whole tokens with up to eight (token, envelope) columns
    rng = np.random.default_rng(700 + 10 * T + ell)
    L = random_layer(rng, 512, 384, 160, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, 512)))
    ref = oracle.forward(L, x)
    got = host_y(dbf.forward(dev_layer(L), dev_x(x), y_dtype=torch.float32))
    assert rel_err(got, ref) < 1e-4


@pytest.mark.parametrize("M", [8192, 8224])
def test_input_width_limit(dbf, M):
    # the single launch takes up to 8192 inputs; wider inputs take two launches
    rng = np.random.default_rng(710 + M)
    L = random_layer(rng, M, 256, 96, 1)
    x = S.to_bf16_bits(rng.standard_normal((1, M)))
    ref = oracle.forward(L, x)
    got = host_y(dbf.forward(dev_layer(L), dev_x(x), y_dtype=torch.float32))
    assert rel_err(got, ref) < 1e-4


def test_fp32_input_unaligned_gamma(dbf):
    # fp32 activations, and gamma at an odd 2-byte offset (scalar loads)
    rng = np.random.default_rng(720)
    L = random_layer(rng, 264, 200, 70, 2)
    dl = dev_layer(L)
    g = torch.empty(dl.gamma.numel() + 1, dtype=torch.float16, device="cuda")
    g[1:] = dl.gamma.reshape(-1)
    dl2 = dbf.Layer(dl.M, dl.N, dl.R, dl.ell, dl.b1, dl.b2, dl.alpha, dl.beta, g[1:].view(dl.gamma.shape))
    x = rng.standard_normal((3, 264)).astype(np.float32)
    ref = oracle.forward(L, x)
    got = host_y(dbf.forward(dl2, torch.from_numpy(x).cuda(), y_dtype=torch.float32))
    assert rel_err(got, ref) < 1e-4


def test_shared_workspace_many_layers(dbf):
    # layers of different sizes (so different grid sizes) take turns on one
    # workspace; each call queued behind the previous one on one stream
    rng = np.random.default_rng(730)
    shapes = [(256, 256, 16), (1024, 2048, 512), (4096, 700, 48), (96, 5000, 300)]
    layers = [random_layer(rng, M, N, R, 1) for M, N, R in shapes]
    dls = [dev_layer(L) for L in layers]
    xs = [S.to_bf16_bits(rng.standard_normal((1, M))) for M, _, _ in shapes]
    refs = [oracle.forward(L, x) for L, x in zip(layers, xs)]
    need = max(dbf.workspace_bytes(d, 1) for d in dls)
    ws = dbf.alloc_workspace(need, "cuda")
    xd = [dev_x(x) for x in xs]
    outs = []
    for k in range(40):
        i = k % len(layers)
        outs.append((i, dbf.forward(dls[i], xd[i], ws=ws, y_dtype=torch.float32, static_weights=bool(k & 1))))
    torch.cuda.synchronize()
    for i, y in outs:
        assert rel_err(host_y(y), refs[i]) < 1e-4
    assert header_words(ws) == (0, 40)
    assert dbf.workspace_status(ws) == dbf.OK


def test_epoch_wraps(dbf):
    # only a change of the epoch matters, not its value: it wraps past 2^32
    rng = np.random.default_rng(740)
    L = random_layer(rng, 640, 320, 96, 1)
    dl = dev_layer(L)
    x = S.to_bf16_bits(rng.standard_normal((2, 640)))
    ref = oracle.forward(L, x)
    ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, 2), "cuda")
    ws[4:8].view(torch.int32).fill_(-2)   # epoch 0xFFFFFFFE
    for _ in range(3):
        got = host_y(dbf.forward(dl, dev_x(x), ws=ws, y_dtype=torch.float32))
        assert rel_err(got, ref) < 1e-4
    assert header_words(ws) == (0, 1)


def test_barrier_timeout_reported_and_workspace_recovers(dbf):
    # A grid-barrier time limit of 1 ns: every CTA but the last to arrive gives
    # up at once, stores DBF_ERR_TIMEOUT in the workspace status word and skips
    # its stage-2 rows (the waits end; nothing faults or hangs). The barrier
    # word is left consistent, and the next call, with the default limit, is
    # correct.
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    xh = S.make_x(w.seed, 1, w.M, "bf16")
    x = dev_x(xh)
    ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, 1), "cuda")
    try:
        dbf.debug_set_decode_wait_ns(1)
        dbf.forward(dl, x, ws=ws, y_dtype=torch.float32)
        torch.cuda.synchronize()
    finally:
        dbf.debug_set_decode_wait_ns(0)
    assert dbf.workspace_status(ws) == dbf.ERR_TIMEOUT
    assert header_words(ws) == (0, 1)
    dbf.clear_workspace_status(ws)
    y = dbf.forward(dl, x, ws=ws, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert dbf.workspace_status(ws) == dbf.OK
    assert header_words(ws) == (0, 2)
    assert rel_err(host_y(y), oracle.forward(L, xh)) < 1e-4


def test_dbf_mlp_decode_repeat_bit_identical(dbf):
    # integer accumulation: the result does not depend on timing or on which
    # call came before
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    dl = dev_layer(L)
    x = dev_x(S.make_x(w.seed, 1, w.M, "bf16"))
    ws = dbf.alloc_workspace(dbf.workspace_bytes(dl, 1), "cuda")
    ys = [dbf.forward(dl, x, ws=ws, y_dtype=torch.float32, static_weights=True) for _ in range(6)]
    torch.cuda.synchronize()
    first = host_y(ys[0])
    for y in ys[1:]:
        assert np.array_equal(host_y(y), first)
    ref = oracle.forward(L, S.make_x(w.seed, 1, w.M, "bf16"))
    assert rel_err(first, ref) < 1e-4


@pytest.mark.parametrize("M,N,R,ell,T", [(320, 200, 70, 3, 37), (256, 160, 128, 2, 300), (1000, 33, 7, 1, 129),
                                          (4096, 4096, 64, 1, 64)])
def test_many_tokens(dbf, M, N, R, ell, T):
    # many chunks (ragged last chunk), several items per CTA with slice reloads
    rng = np.random.default_rng(750 + T)
    L = random_layer(rng, M, N, R, ell)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    rows = None if M * N * R * T < 4e9 else list(range(0, T, 7)) + [T - 1]
    ref = oracle.forward(L, x, rows=rows)
    got = host_y(dbf.forward(dev_layer(L), dev_x(x), path="gemv", y_dtype=torch.float32))
    assert rel_err(got if rows is None else got[rows], ref) < 1e-4


def test_dbf_mlp_many_tokens_sampled(dbf):
    # the DBF MLP layer through the decode kernel at 24 tokens (several chunks
    # over the long rank), checked on sampled rows
    w = S.WORKLOADS["dbf_mlp"]
    L = S.workload_layers(w)[0]
    x = S.make_x(w.seed + 7, 24, w.M, "bf16")
    rows = [0, 5, 11, 17, 23]
    ref = oracle.forward(L, x, rows=rows)
    got = host_y(dbf.forward(dev_layer(L), dev_x(x), path="gemv", y_dtype=torch.float32))
    assert rel_err(got[rows], ref) < 1e-4


def i32(a):
    return torch.tensor(np.asarray(a, dtype=np.int32), device="cuda")


@pytest.mark.parametrize("S_,shapes", [(40, [(33, 1), (96, 2), (7, 3), (128, 1)]),
                                       (40, [(33, 1), (300, 2), (7, 3)]),
                                       (600, [(33, 1), (96, 2), (7, 3), (128, 1)])])
def test_segmented_mixed_adapters(dbf, S_, shapes):
    # adapters of different ranks (below the largest: small ranks in the
    # per-word or the group layout of stage 2) and envelope counts, segments of
    # 0..9 tokens, some without an adapter; 600 segments take the two-launch
    # path
    rng = np.random.default_rng(760 + S_ + len(shapes))
    M, N = 288, 136
    layers = [random_layer(rng, M, N, R, ell) for R, ell in shapes]
    counts = rng.integers(0, 10, size=S_)
    if S_ > 100:
        counts = np.minimum(counts, 1)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    T = int(offsets[-1])
    adapter = rng.integers(-1, len(layers), size=S_)
    x = S.to_bf16_bits(rng.standard_normal((T, M)))
    ref = oracle.forward_segmented(layers, offsets, adapter, x)
    table = dbf.AdapterTable([dev_layer(L) for L in layers], "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = dbf.forward_segmented(table, i32(offsets), i32(adapter), dev_x(x), y_dtype=torch.float32, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert rel_err(host_y(y), ref) < 1e-4
