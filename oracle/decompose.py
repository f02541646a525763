"""Binary low-rank decomposition W ~= U diag(alpha) V^T + R: plain FP64 restatement.

TEST INFRASTRUCTURE ONLY (part of the CPU oracle).  Only the tests, the smoke
check and the benchmark's CPU-baseline leg may import it.

Source passage: BiLoCo README (github jindavid/BiLoCo), section "Decomposition":
each rank-one term starts from random signs and alternates u = sign(R v),
v = sign(R^T u) for T steps, takes the Frobenius-optimal coefficient and deflates
the residual; after all r terms the coefficients are refit jointly by least
squares for the fixed signs.

Readings where the passage is silent (listed in the design notes):
  * The random start is the vector v (the first alternation computes u from it);
    its signs are an input here (`v0`, r x K), drawn by the caller from a seeded
    generator, so that the oracle and the GPU see the same draws.
  * sign(0) = +1, the convention of the sign packing.
  * One step = u = sign(R v) followed by v = sign(R^T u); T steps, T >= 1.
  * The coefficient of a term is the Frobenius-optimal one for the current
    residual and the final (u, v): alpha = u^T R v / (N K), because
    ||u v^T||_F^2 = N K for sign vectors.
  * Deflation: R <- R - alpha u v^T, in FP64.
  * The refit minimises ||W - sum_i alpha_i u_i v_i^T||_F over alpha with the
    signs fixed.  Its normal equations are G alpha = b with
    G_ij = (u_i . u_j)(v_i . v_j) and b_i = u_i^T W v_i; they are solved here by a
    least-squares solve of that small system, which gives the minimum-norm
    coefficients when terms repeat (G singular; the fitted matrix is unique).
  * The returned residual is R = W - U diag(alpha) V^T with the refit alpha, the
    matrix that is then quantised to NVFP4.
Everything is FP64; W enters as FP32 values.
"""

from __future__ import annotations

import numpy as np


def sign_pm1(a: np.ndarray) -> np.ndarray:
    """+1 where a >= 0, -1 where a < 0 (sign(0) = +1), as float64."""
    return np.where(np.asarray(a) < 0, -1.0, 1.0)


def peel_term(R: np.ndarray, v0: np.ndarray, T: int):
    """One rank-one term from residual R [N, K] and start signs v0 [K].

    Returns (u [N], v [K], alpha) after T alternations u = sign(R v), v = sign(R^T u)
    and the Frobenius-optimal coefficient alpha = u^T R v / (N K)."""
    if T < 1:
        raise ValueError("T >= 1 alternations")
    N, K = R.shape
    v = sign_pm1(v0)
    u = None
    for _ in range(T):
        u = sign_pm1(R @ v)
        v = sign_pm1(R.T @ u)
    alpha = float(u @ R @ v) / float(N * K)
    return u, v, alpha


def gram(U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """G_ij = <u_i v_i^T, u_j v_j^T>_F = (u_i . u_j)(v_i . v_j)."""
    return (U.T @ U) * (V.T @ V)


def refit_alpha(W: np.ndarray, U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """Least-squares coefficients for fixed signs: G alpha = b (minimum norm if G
    is singular)."""
    W = np.asarray(W, dtype=np.float64)
    b = np.einsum("ni,nk,ki->i", U, W, V)          # u_i^T W v_i
    return np.linalg.lstsq(gram(U, V), b, rcond=None)[0]


def decompose(W: np.ndarray, r: int, T: int, v0: np.ndarray, refit: bool = True):
    """Greedy sign peeling of W [N, K] into r binary rank-one terms, then the joint
    refit.  v0: [r, K] start signs (one row per term).

    Returns dict(U [N, r] int8, V [K, r] int8, alpha [r] float64 (refit),
    alpha_greedy [r], R [N, K] float64 = W - U diag(alpha) V^T, greedy_norms [r + 1]
    = ||residual||_F before the first term and after each deflation)."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    R = W.copy()
    U = np.zeros((N, r))
    V = np.zeros((K, r))
    a_greedy = np.zeros(r)
    norms = [float(np.linalg.norm(R))]
    for i in range(r):
        u, v, a = peel_term(R, v0[i], T)
        R -= a * np.outer(u, v)
        U[:, i], V[:, i], a_greedy[i] = u, v, a
        norms.append(float(np.linalg.norm(R)))
    alpha = refit_alpha(W, U, V) if (refit and r > 0) else a_greedy.copy()
    R_final = W - (U * alpha[None, :]) @ V.T
    return dict(U=U.astype(np.int8), V=V.astype(np.int8), alpha=alpha, alpha_greedy=a_greedy,
                R=R_final, greedy_norms=np.array(norms))
