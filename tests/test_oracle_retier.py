"""Pins of the oracle's re-tiering step (a stored token re-encoded at another rank from its
bf16-rounded reconstruction): closed forms with signed-permutation bases, where every
projection and reconstruction has one nonzero term and is exact, and a bound against the fp64
reconstruction for a dense orthonormal basis."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import bf16_np, signed_permutation


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _token(d, r_max, r_old, s, bits, seed):
    """A stored token: bf16 coefficients (zero past r_old), s distinct ascending channels,
    codes in range and an fp16 scale."""
    g = torch.Generator().manual_seed(seed)
    qmax = synth.qmax_of(bits)
    c = torch.zeros(r_max)
    c[:r_old] = torch.randn(r_old, generator=g)
    idx = torch.randperm(d, generator=g)[:s].sort().values.to(torch.uint8)
    codes = torch.randint(-qmax, qmax + 1, (s,), generator=g).to(torch.int8)
    scale = torch.tensor([0.013], dtype=torch.float16)
    return c.to(torch.bfloat16), idx, codes, scale


def _xh_perm(B_bits, perm, sign, r_old, c, idx, codes, scale):
    """The bf16 reconstruction with a signed-permutation basis, from its definition:
    x_{perm(j)} = sign_j c_j for j < r_old (exact), plus scale * code on the residual channels,
    rounded to bf16 once (numpy fp32 add of exact terms)."""
    d = B_bits.shape[0]
    a = np.zeros(d, np.float32)
    cf = bf16_np(c).astype(np.float32)
    for j in range(r_old):
        a[int(perm[j])] = np.float32(sign[j]) * cf[j]
    sf = np.float32(bf16_np(scale)[0])
    for i, q in zip(idx.numpy(), codes.numpy()):
        a[int(i)] = np.float32(a[int(i)] + np.float32(sf * np.float32(q)))
    return _bf16_bits(a)


@pytest.mark.parametrize("bits", [8, 4])
def test_same_rank_without_residual_is_the_identity(bits):
    d, r_max, r, s = 128, 64, 32, 16
    Bm, perm, sign = signed_permutation(d, r_max, 5)
    c, idx, codes, _ = _token(d, r_max, r, s, bits, 1)
    zero = torch.tensor([0.0], dtype=torch.float16)
    out = oracle.reencode_vector(Bm, r, c, idx, codes, zero, r, bits)
    assert np.array_equal(out["coeff"], c.view(torch.int16).numpy().view(np.uint16))
    assert out["scale"] == 0 and not out["codes"].any()
    assert list(out["idx"]) == list(range(s))            # all-zero residual: ties to the lowest channels


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("r_old,r_new", [(16, 64), (8, 32), (32, 64)])
def test_promotion_with_a_permutation_basis_matches_the_closed_form(bits, r_old, r_new):
    """Promotion: the new coefficients past r_old pick up the reconstruction on the new
    basis directions (sign_j x_{perm(j)}); the coefficients below r_old are kept."""
    d, r_max, s = 128, 64, 16
    Bm, perm, sign = signed_permutation(d, r_max, 9 + r_old)
    c, idx, codes, scale = _token(d, r_max, r_old, s, bits, 3 + r_new)
    # put a few residual channels on the new basis directions so the promotion moves them
    new_dirs = [int(perm[j]) for j in range(r_old, r_new)]
    idx = torch.tensor(sorted(set(new_dirs[:6]) | set(idx.tolist()[: s - 6]))[:s], dtype=torch.uint8)
    if idx.numel() < s:
        extra = [i for i in range(d) if i not in set(idx.tolist())][: s - idx.numel()]
        idx = torch.tensor(sorted(idx.tolist() + extra), dtype=torch.uint8)
    out = oracle.reencode_vector(Bm, r_old, c, idx, codes, scale, r_new, bits)
    xh = _xh_perm(Bm, perm, sign, r_old, c, idx, codes, scale)
    assert np.array_equal(out["xh"], xh)
    xf = bf16_np(torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16)).astype(np.float32)
    # exact: one nonzero term each; a chain that starts from +0 turns -0 into +0
    want = np.array([np.float32(sign[j]) * xf[int(perm[j])] + np.float32(0.0) for j in range(r_new)], np.float32)
    assert np.array_equal(out["coeff"][:r_new], _bf16_bits(want))
    assert not out["coeff"][r_new:].any()
    # the new residual lives off the first r_new basis directions, on the old residual's channels
    covered = {int(perm[j]) for j in range(r_new)}
    nz = [int(i) for i, q in zip(out["idx"], out["codes"]) if q != 0]
    assert not (set(nz) & covered)
    assert set(nz) <= set(idx.tolist())


@pytest.mark.parametrize("bits", [8, 4])
def test_demotion_with_a_permutation_basis_moves_dropped_coefficients_to_the_residual(bits):
    d, r_max, s, r_old, r_new = 128, 64, 16, 64, 16
    Bm, perm, sign = signed_permutation(d, r_max, 21)
    c, idx, codes, scale = _token(d, r_max, r_old, s, bits, 22)
    out = oracle.reencode_vector(Bm, r_old, c, idx, codes, scale, r_new, bits)
    xh = _xh_perm(Bm, perm, sign, r_old, c, idx, codes, scale)
    xf = bf16_np(torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16)).astype(np.float64)
    want = np.array([sign[j] * xf[int(perm[j])] for j in range(r_new)], np.float64)
    assert np.array_equal(bf16_np(torch.from_numpy(out["coeff"][:r_new].view(np.int16)).view(torch.bfloat16)), want)
    # residual = xh off the kept directions: its s largest magnitudes, ties to the lower channel
    r = xf.copy()
    for j in range(r_new):
        r[int(perm[j])] = 0.0
    order = sorted(range(d), key=lambda i: (-abs(r[i]), i))[:s]
    assert list(out["idx"]) == sorted(order)


def test_dense_basis_reconstruction_is_within_bf16_rounding_of_fp64():
    wl = synth.workload("llama8b_64k")
    bases = synth.make_bases(wl.scaled(num_layers=2))
    Bm = bases[0][0, 3]
    for seed in range(20):
        r_old = (16, 32, 64)[seed % 3]
        c, idx, codes, scale = _token(128, 64, r_old, 16, 4, 100 + seed)
        out = oracle.reencode_vector(Bm, r_old, c, idx, codes, scale, 64, 4)
        ref = oracle.reconstruct(Bm, r_old, c, idx, codes, scale)
        xh = bf16_np(torch.from_numpy(out["xh"].view(np.int16)).view(torch.bfloat16))
        # bf16 rounding (half an ulp, 2^-9 relative) plus the fp32 chain's error
        assert np.all(np.abs(xh - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6 * np.linalg.norm(ref)), seed


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("s_old,s_new", [(8, 2), (2, 8), (4, 0), (0, 4)])
def test_residual_count_change_at_one_rank(bits, s_old, s_new):
    """A tier move of the residual-count routing reading (same rank, another residual count)
    with a signed-permutation basis: the coefficients are kept exactly when the old residual
    stays off the basis directions, and the new residual is the s_new largest |xh| off the
    kept directions, ties to the lower channel, codes by the scale of the largest."""
    d, r_max, r = 128, 64, 32
    Bm, perm, sign = signed_permutation(d, r_max, 40 + s_old)
    g = torch.Generator().manual_seed(41 + s_new)
    c = torch.zeros(r_max)
    c[:r] = torch.randn(r, generator=g)
    c = c.to(torch.bfloat16)
    covered = {int(perm[j]) for j in range(r)}
    free = [i for i in range(d) if i not in covered]
    pick = torch.randperm(len(free), generator=g)[:s_old].tolist()
    idx = torch.tensor(sorted(free[i] for i in pick), dtype=torch.uint8)
    qmax = synth.qmax_of(bits)
    codes = torch.randint(-qmax, qmax + 1, (s_old,), generator=g).to(torch.int8)
    scale = torch.tensor([0.021], dtype=torch.float16)
    out = oracle.reencode_vector(Bm, r, c, idx, codes, scale, r, bits, s_new=s_new)
    assert out["idx"].shape == (s_new,) and out["codes"].shape == (s_new,)
    assert np.array_equal(out["coeff"], c.view(torch.int16).numpy().view(np.uint16))
    xf = bf16_np(torch.from_numpy(out["xh"].view(np.int16)).view(torch.bfloat16)).astype(np.float64)
    res = xf.copy()
    for j in range(r):
        res[int(perm[j])] = 0.0
    # the old residual is the only mass off the kept directions
    assert np.count_nonzero(res) <= s_old
    order = sorted(range(d), key=lambda i: (-abs(res[i]), i))[:s_new]
    assert list(out["idx"]) == sorted(order)
    if s_new:
        amax = max(abs(res[i]) for i in order)
        sf = float(np.float16(np.float32(amax) / np.float32(qmax)))
        assert abs(float(bf16_np(torch.tensor([out["scale"]], dtype=torch.int16).view(torch.float16))[0]) - sf) == 0.0
        for i, q in zip(out["idx"], out["codes"]):
            want = 0 if sf == 0 else int(np.clip(np.rint(np.float32(res[int(i)]) / np.float32(sf)), -qmax, qmax))
            assert int(q) == want, (i, q, want)
    else:
        assert out["scale"] == 0
