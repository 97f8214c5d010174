"""Pins of the oracle's online basis construction ("DepthWeave-KV ...", §3 Method, the shared
bases paragraph: a randomized low-rank sketch after prefill, then a moving-average update) and
of the re-projection of a stored token onto an updated basis.  Checks rest on closed forms
(planted spectra whose eigenvectors are known, exact test matrices, the moving average's
algebra) and invariants, not on the formulas themselves."""
import numpy as np
import pytest
import torch

import oracle
from oracle import basis as ob
from helpers import bf16_np, signed_permutation


def _planted(n, d, sig, seed):
    """Rows x_t = sum_k z_tk sig_k v_k with V orthonormal and Z orthonormal columns: the
    second moment is exactly V diag(sig^2) V^T."""
    rng = np.random.default_rng(seed)
    v, _ = np.linalg.qr(rng.standard_normal((d, d)))
    z, _ = np.linalg.qr(rng.standard_normal((n, d)))
    return z @ np.diag(sig) @ v.T, v


def _proj(b, r):
    return b[:, :r] @ b[:, :r].T


def test_gram_invariants():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((300, 16))
    c = ob.gram(x)
    assert np.allclose(c, c.T)
    assert np.all(np.linalg.eigvalsh(c) >= -1e-9)                        # positive semidefinite
    assert np.isclose(np.trace(c), (x * x).sum())                        # trace = total energy
    assert np.allclose(ob.gram(x[rng.permutation(300)]), c)              # order of the tokens
    assert np.allclose(ob.gram(x[:100]) + ob.gram(x[100:]), c)           # additive over blocks


def test_mgs_is_orthonormal_and_nested():
    rng = np.random.default_rng(2)
    y = rng.standard_normal((32, 12))
    q = ob.mgs(y)
    assert np.allclose(q.T @ q, np.eye(12), atol=1e-12)
    # span(Q[:, :j]) = span(Y[:, :j]): Q^T Y upper triangular with a positive diagonal
    r = q.T @ y
    assert np.allclose(np.tril(r, -1), 0.0, atol=1e-10)
    assert np.all(np.diag(r) > 0)
    with pytest.raises(ValueError):
        ob.mgs(np.stack([y[:, 0], 2.0 * y[:, 0]], 1))


def test_exact_test_matrix_gives_the_exact_top_subspace():
    """If omega spans the top-r eigenvectors, no power step is needed: B = V[:, :r] up to
    sign, in eigenvalue order."""
    d, r = 24, 6
    sig = 2.0 ** -np.arange(d)
    x, v = _planted(200, d, sig, 3)
    c = ob.gram(x)
    rng = np.random.default_rng(4)
    omega = v[:, :r] @ rng.standard_normal((r, r))                       # an invertible mixing
    b, w = ob.sketch_basis(c, omega, power_steps=0)
    assert np.allclose(np.abs(np.sum(b * v[:, :r], 0)), 1.0, atol=1e-9)
    assert np.allclose(w, sig[:r] ** 2, rtol=1e-9)


@pytest.mark.parametrize("power_steps,tol", [(2, 1e-3), (6, 1e-9)])
def test_power_steps_converge_on_a_planted_spectrum(power_steps, tol):
    d, r = 64, 16
    sig = 0.6 ** np.arange(d)                                            # gap ratio 0.36 per step squared
    x, v = _planted(500, d, sig, 5)
    c = ob.gram(x)
    omega = np.random.default_rng(6).standard_normal((d, r))
    b, w = ob.sketch_basis(c, omega, power_steps=power_steps)
    for k in (4, 8):                                                     # nested tier subspaces
        assert np.linalg.norm(_proj(b, k) - _proj(v, k)) < tol, k


def test_rayleigh_ritz_orders_and_diagonalises():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((400, 20)) * (1.5 ** -np.arange(20))
    c = ob.gram(x)
    b, w = ob.sketch_basis(c, rng.standard_normal((20, 8)), power_steps=3)
    assert np.allclose(b.T @ b, np.eye(8), atol=1e-12)
    t = b.T @ c @ b
    assert np.allclose(t, np.diag(np.diag(t)), atol=1e-9 * np.abs(t).max())
    assert np.all(np.diff(np.diag(t)) <= 0)                              # descending
    assert np.allclose(np.diag(t), w)
    for j in range(8):                                                   # the sign rule
        k = int(np.argmax(np.abs(b[:, j])))
        assert b[k, j] > 0


def test_moving_average_algebra():
    rng = np.random.default_rng(8)
    a, b1, b2 = (ob.gram(rng.standard_normal((50, 6))) for _ in range(3))
    assert np.allclose(ob.ema(a, b1, 1.0), a)
    assert np.allclose(ob.ema(a, b1, 0.0), b1)
    two = ob.ema(ob.ema(a, b1, 0.9), b2, 0.9)
    assert np.allclose(two, 0.81 * a + 0.09 * b1 + 0.1 * b2)


def test_refresh_keeps_a_basis_that_already_spans_the_eigenvectors():
    d, r = 16, 5
    sig = 1.7 ** -np.arange(d)
    x, v = _planted(100, d, sig, 9)
    c = ob.gram(x)
    b_old = ob.sign_normalize(v[:, :r])
    b, w = ob.refresh_basis(c, b_old)
    assert np.allclose(np.abs(np.sum(b * v[:, :r], 0)), 1.0, atol=1e-10)
    assert np.allclose(b, b_old, atol=1e-10)


@pytest.mark.parametrize("bits", [8, 4])
def test_reprojection_onto_a_new_permutation_basis(bits):
    """A token stored on one signed-permutation basis, re-encoded on another at the same rank:
    its reconstruction x^ is exact, and the new coefficients are sign'_j x^_{perm'(j)} (one
    nonzero term each), with the residual off the new directions."""
    d, r_max, r = 128, 64, 32
    b_old, perm, sign = signed_permutation(d, r_max, 11)
    b_new, perm2, sign2 = signed_permutation(d, r_max, 12)
    g = torch.Generator().manual_seed(13)
    c = torch.zeros(r_max)
    c[:r] = torch.randn(r, generator=g)
    c = c.to(torch.bfloat16)
    idx = torch.randperm(d, generator=g)[:16].sort().values.to(torch.uint8)
    qmax = 127 if bits == 8 else 7
    codes = torch.randint(-qmax, qmax + 1, (16,), generator=g).to(torch.int8)
    scale = torch.tensor([0.02], dtype=torch.float16)
    out = oracle.reencode_vector(b_old, r, c, idx, codes, scale, r, bits, basis_new=b_new)
    xh = bf16_np(torch.from_numpy(out["xh"].view(np.int16)).view(torch.bfloat16)).astype(np.float64)
    want = np.array([float(sign2[j]) * xh[int(perm2[j])] for j in range(r)])
    got = bf16_np(torch.from_numpy(out["coeff"][:r].view(np.int16)).view(torch.bfloat16))
    assert np.array_equal(got, want)
    covered = {int(perm2[j]) for j in range(r)}
    nz = [int(i) for i, q in zip(out["idx"], out["codes"]) if q != 0]
    assert not (set(nz) & covered)
    # the same basis on both sides is the plain re-tier
    same = oracle.reencode_vector(b_old, r, c, idx, codes, scale, r, bits, basis_new=b_old)
    plain = oracle.reencode_vector(b_old, r, c, idx, codes, scale, r, bits)
    for key in ("coeff", "idx", "codes"):
        assert np.array_equal(same[key], plain[key])
