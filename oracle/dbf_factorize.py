"""fp64 oracle of the DBF factorisation (test infrastructure).

DBF page, section 2 ("Metodologia" and "Algoritmo de Computação"): a dense
weight W (n x m) is approximated by (a . A . m^T)(B . b^T): sign matrices
A (n x k) and B (k x m) with fp16 scale vectors a (n), m (k), b (m). The page
says how the factors are found only in outline: a heuristic alternating
minimisation that uses ADMM, with the SVID decomposition (from OneBit) as
the projection that keeps the factors binary, optionally weighted by input
and output importance. The steps below are the plainest reading of that
outline; the page gives no update formulas, penalty, iteration counts or
starting point.

- The constraint set P(r, c): r x c matrices diag(p) S diag(q) with S a sign
  matrix and p, q >= 0, i.e. a sign matrix times a rank-1 nonnegative
  pattern. U = a . A . m1^T is in P(n, k), V = m2 . B . b^T is in P(k, m),
  and U V is the page's product with m = m1 . m2.
- SVID is the Euclidean projection onto P: sign(X) . (best rank-1
  approximation of |X|) (``oracle.svid``).
- Alternating minimisation of ||W - U V||_F^2: the U-subproblem with V
  fixed, then the V-subproblem with U fixed, ``outer`` times.
- Each subproblem is ADMM in scaled form on
  1/2 ||W - U V||^2 + indicator_P(Z) subject to U = Z, starting from the
  current factor as Z and a zero dual Lam:
    U   <- (W V^T + rho (Z - Lam)) (V V^T + rho I)^-1   (the exact minimiser)
    Z   <- SVID(U + Lam)
    Lam <- Lam + U - Z
  ``admm_iters`` times; the factor becomes Z. The V-subproblem is the same
  with the operands transposed: V <- (U^T U + rho I)^-1 (U^T W + rho (Z - Lam)).
- rho = rho_rel * trace(Gram) / k, with Gram = V V^T or U^T U, so the
  penalty scales with the data.
- Unweighted: the importance weights need activations and gradients of a
  trained model.
- The starting point (U0, V0) is an input; the projection of it starts the
  iteration.

Pins (tests/test_oracle_factorize_pins.py): the least-squares steps satisfy
their first-order conditions; an exact product of two members of P is a
fixed point; at k = 1 the set P holds every vector, the projection is the
identity and the iteration converges to the best rank-1 approximation
(Eckart-Young, checked against numpy's SVD); the returned factors, packed as
a layer, reproduce U V through the layer forward.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List

import numpy as np


def svid_project(X: np.ndarray):
    """The SVID projection onto P: returns (Z, S, p, q) with Z = S . p q^T."""
    from . import svid
    S, p, q = svid(X)
    return S * np.outer(p, q), S, p, q


def rho_of(gram: np.ndarray, rho_rel: float) -> float:
    """The penalty: rho_rel times the mean diagonal of the Gram matrix."""
    return rho_rel * float(np.trace(gram)) / gram.shape[0]


def admm_u_step(WVt: np.ndarray, VVt: np.ndarray, rho: float, Z: np.ndarray, Lam: np.ndarray) -> np.ndarray:
    """argmin_U 1/2 ||W - U V||^2 + rho/2 ||U - Z + Lam||^2 from W V^T and V V^T."""
    k = VVt.shape[0]
    return np.linalg.solve(VVt + rho * np.eye(k), (WVt + rho * (Z - Lam)).T).T


def admm_v_step(UtW: np.ndarray, UtU: np.ndarray, rho: float, Z: np.ndarray, Lam: np.ndarray) -> np.ndarray:
    """argmin_V 1/2 ||W - U V||^2 + rho/2 ||V - Z + Lam||^2 from U^T W and U^T U."""
    k = UtU.shape[0]
    return np.linalg.solve(UtU + rho * np.eye(k), UtW + rho * (Z - Lam))


@dataclass
class Factors:
    """Result of ``factorize``.

    A: int8 +-1 [n, k]; B: int8 +-1 [k, m]; a [n], mid [k], b [m] fp64
    (mid = m1 . m2); alpha/beta/gamma: the same rounded to fp16 bit patterns;
    U, V: the final fp64 factors (U V is the approximation);
    objective: ||W - U V||_F for the projected start and after each outer
    iteration."""
    A: np.ndarray
    B: np.ndarray
    a: np.ndarray
    mid: np.ndarray
    b: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray
    gamma: np.ndarray
    U: np.ndarray
    V: np.ndarray
    objective: List[float]

    def layer(self):
        """The factors as a one-envelope layer: B1 = A, B2 = B, alpha = a,
        beta = mid, gamma = b (fp16)."""
        import dbf_synth as S
        n, k = self.A.shape
        m = self.B.shape[1]
        return S.Layer(M=m, N=n, R=k, ell=1, b1=self.A.astype(np.int8), b2=self.B.astype(np.int8),
                       alpha=self.alpha[None, :], beta=self.beta[None, :], gamma=self.gamma[None, :])


def _f16_bits(v: np.ndarray) -> np.ndarray:
    return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def factorize(W: np.ndarray, U0: np.ndarray, V0: np.ndarray, outer: int, admm_iters: int,
              rho_rel: float = 1.0) -> Factors:
    """DBF factorisation of W (n x m) at inner dimension k = U0.shape[1] by
    alternating ADMM with the SVID projection (steps in the module
    docstring). fp64."""
    W = np.asarray(W, dtype=np.float64)
    U, Su, a, m1 = svid_project(np.asarray(U0, dtype=np.float64))
    V, Sv, m2, b = svid_project(np.asarray(V0, dtype=np.float64))
    obj = [float(np.linalg.norm(W - U @ V))]
    for _ in range(outer):
        # U-subproblem, V fixed
        G, C = V @ V.T, W @ V.T
        rho = rho_of(G, rho_rel)
        Z, Lam = U, np.zeros_like(U)
        for _ in range(admm_iters):
            Uf = admm_u_step(C, G, rho, Z, Lam)
            Z, Su, a, m1 = svid_project(Uf + Lam)
            Lam = Lam + Uf - Z
        U = Z
        # V-subproblem, U fixed
        G, C = U.T @ U, U.T @ W
        rho = rho_of(G, rho_rel)
        Z, Lam = V, np.zeros_like(V)
        for _ in range(admm_iters):
            Vf = admm_v_step(C, G, rho, Z, Lam)
            Z, Sv, m2, b = svid_project(Vf + Lam)
            Lam = Lam + Vf - Z
        V = Z
        obj.append(float(np.linalg.norm(W - U @ V)))
    mid = m1 * m2
    return Factors(A=Su, B=Sv, a=a, mid=mid, b=b, alpha=_f16_bits(a), beta=_f16_bits(mid), gamma=_f16_bits(b),
                   U=U, V=V, objective=obj)


def svd_init(W: np.ndarray, k: int):
    """A starting point: the rank-k truncated SVD split evenly,
    U0 = U_k sqrt(S_k), V0 = sqrt(S_k) V_k^T (k <= min(n, m))."""
    Uw, s, Vt = np.linalg.svd(np.asarray(W, dtype=np.float64), full_matrices=False)
    r = np.sqrt(s[:k])
    return Uw[:, :k] * r, r[:, None] * Vt[:k]
