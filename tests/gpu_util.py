"""Helpers shared by the GPU parity tests: move seeded host inputs to the
device, run the library, compare with the fp64 oracle."""
import numpy as np
import torch

import dbf_synth as S

TOL = 2e-3   # max|y - y_ref| / max|y_ref| for fp32 outputs


def dev_layer(L, device="cuda"):
    """Pack a host Layer's signs with the library and move its scales."""
    import double_binary_rank_b200 as dbf
    b1 = torch.from_numpy(L.b1).to(device)
    b2 = torch.from_numpy(L.b2).to(device)
    f16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.float16)).to(device)
    return dbf.Layer.from_signs(b1, b2, f16(L.alpha), f16(L.beta), f16(L.gamma))


def dev_x(x, device="cuda"):
    """fp32 array -> float32 tensor; uint16 bf16 bits -> bfloat16 tensor."""
    if x.dtype == np.float32:
        return torch.from_numpy(x).to(device)
    return torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)


def host_y(y):
    return y.float().cpu().numpy().astype(np.float64)


def rel_err(got, ref):
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-300))


def bf16_ok(got, ref, tol=TOL):
    """bf16 outputs: per element within half a bf16 ulp of y_ref plus tol*max|y_ref|."""
    ref32 = np.abs(ref).astype(np.float32)
    e = np.floor(np.log2(np.maximum(ref32, 1e-30)))
    half_ulp = 0.5 * np.exp2(e - 7)
    bound = half_ulp + tol * np.max(np.abs(ref))
    return bool(np.all(np.abs(got - ref) <= bound)), float(np.max(np.abs(got - ref) - bound))


def random_layer(rng, M, N, R, ell, sigma=0.5, dyadic=False):
    b1 = rng.choice(np.array([-1, 1], dtype=np.int8), size=(N, R))
    b2 = rng.choice(np.array([-1, 1], dtype=np.int8), size=(R, M))
    if dyadic:
        mk = lambda n: S.to_f16_bits(rng.choice([0.5, 1.0, 2.0, -0.5, -1.0, -2.0], n))
    else:
        mk = lambda n: S.to_f16_bits(np.exp(sigma * rng.standard_normal(n)))
    return S.Layer(M, N, R, ell, b1, b2, np.stack([mk(N) for _ in range(ell)]),
                   np.stack([mk(R) for _ in range(ell)]), np.stack([mk(M) for _ in range(ell)]))
