"""Oracle of the online basis construction of "DepthWeave-KV: Token-Adaptive Cross-Layer
Residual Factorization for Long-Context KV Cache Compression", §3 Method, the paragraph on the
shared bases: per depth window, per kv head and separately for keys and values, a randomized
low-rank sketch of the cached vectors after prefill gives the basis, and an exponential moving
average updates it as generation proceeds.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the bench's CPU baseline
are the only callers; the product library never imports this module.

The pages name the steps but not their numbers; this module fixes the plainest reading (every
step in fp64 with numpy):

1. the window's channel second moment C = sum over its layers and tokens of x x^T (d x d);
2. the sketch Y = C Omega, Omega a d x r Gaussian test matrix (an input: the random numbers
   the method draws are passed in), orthonormalised by modified Gram-Schmidt (columns in
   order), then ``power_steps`` subspace iterations Q <- MGS(C Q);
3. a Rayleigh-Ritz step: the eigenvectors U of T = Q^T C Q, eigenvalues in descending order,
   B = Q U, so that the first r_t columns of B are the best rank-r_t subspace the sketch
   found (a token of rank r_t uses the first r_t columns); each column's sign is fixed so
   that its entry of largest magnitude (the lowest channel among equal ones) is positive;
4. the update: C <- beta C + (1 - beta) C_new over the vectors appended since the last
   update, then one subspace iteration warm-started from the current basis, Q = MGS(C B),
   and the Rayleigh-Ritz step of 3.
"""
from __future__ import annotations

import numpy as np


def gram(x) -> np.ndarray:
    """C = sum_t x_t x_t^T of the rows of x [n][d] (fp64)."""
    x = np.asarray(x, np.float64)
    return x.T @ x


def mgs(y) -> np.ndarray:
    """Modified Gram-Schmidt over the columns of y [d][k], in order: Q with Q^T Q = I and
    span(Q[:, :j]) = span(y[:, :j]) for every j.  Raises if a column keeps less than 1e-12 of
    its norm (numerically dependent on the previous ones)."""
    q = np.array(y, np.float64, copy=True)
    d, k = q.shape
    for j in range(k):
        n0 = np.sqrt(q[:, j] @ q[:, j])
        for i in range(j):
            q[:, j] -= (q[:, i] @ q[:, j]) * q[:, i]
        n = np.sqrt(q[:, j] @ q[:, j])
        if not n > 1e-12 * n0:
            raise ValueError(f"column {j} is dependent on the previous ones")
        q[:, j] /= n
    return q


def sign_normalize(b) -> np.ndarray:
    """Each column's entry of largest magnitude made positive (the lowest row among equals)."""
    b = np.array(b, np.float64, copy=True)
    for j in range(b.shape[1]):
        k = int(np.argmax(np.abs(b[:, j])))
        if b[k, j] < 0.0:
            b[:, j] = -b[:, j]
    return b


def rayleigh_ritz(c, q):
    """B = Q U with U the eigenvectors of Q^T C Q in descending eigenvalue order (signs by
    sign_normalize), and the eigenvalues."""
    c = np.asarray(c, np.float64)
    q = np.asarray(q, np.float64)
    t = q.T @ c @ q
    t = 0.5 * (t + t.T)
    w, u = np.linalg.eigh(t)
    order = np.argsort(-w, kind="stable")
    return sign_normalize(q @ u[:, order]), w[order]


def sketch_basis(c, omega, power_steps: int = 2):
    """Basis of a window from its second moment C and the test matrix omega [d][r]."""
    c = np.asarray(c, np.float64)
    q = mgs(c @ np.asarray(omega, np.float64))
    for _ in range(power_steps):
        q = mgs(c @ q)
    return rayleigh_ritz(c, q)


def ema(c_old, c_new, beta: float) -> np.ndarray:
    """C <- beta C_old + (1 - beta) C_new."""
    return float(beta) * np.asarray(c_old, np.float64) + (1.0 - float(beta)) * np.asarray(c_new, np.float64)


def refresh_basis(c, b_old):
    """One subspace iteration from the current basis, then Rayleigh-Ritz."""
    return rayleigh_ritz(c, mgs(np.asarray(c, np.float64) @ np.asarray(b_old, np.float64)))
