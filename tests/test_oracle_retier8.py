"""Pins of the oracle's re-encode of a token stored with 8-bit blockwise coefficients ("DepthWeave-KV
...", §3 Method: a re-tier moves the token to another rank, a basis update moves it onto the
updated basis; the coefficients are kept as 8-bit codes, a block of 16 with one fp16 scale).
Closed forms with signed-permutation bases, where every projection and reconstruction has one
nonzero term, and power-of-two block scales whose blocks reach |code| 127, where the blockwise
quantiser is exact; a bound against the fp64 reconstruction written with numpy for a dense
basis; and the bf16 re-encode's reconstruction on coefficients both forms hold exactly."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import bf16_np, signed_permutation


def _bf16_bits(x) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _fp16_bits(x) -> np.ndarray:
    return np.asarray(x, np.float16).view(np.uint16)


def _bits_to_f64(bits, dtype) -> np.ndarray:
    return bf16_np(torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(dtype))


def _token8(d, r_max, r_old, s, bits, seed, exps=None):
    """A stored token: 8-bit codes in [-127, 127] with every block of r_old reaching |code| 127,
    power-of-two block scales 2^e (e in [-6, 1], or ``exps``), garbage past r_old; s distinct
    ascending residual channels, codes in range and an fp16 scale."""
    g = torch.Generator().manual_seed(seed)
    cc = torch.randint(-127, 128, (r_max,), generator=g).to(torch.int8).numpy()
    nb = r_max // 16
    e = torch.randint(-6, 2, (nb,), generator=g).numpy() if exps is None else np.asarray(exps)
    for b in range(r_old // 16):
        k = 16 * b + int(torch.randint(0, 16, (1,), generator=g))
        cc[k] = 127 if int(torch.randint(0, 2, (1,), generator=g)) else -127
    cs = _fp16_bits(np.ldexp(1.0, e.astype(np.int64)))
    qmax = synth.qmax_of(bits)
    idx = torch.randperm(d, generator=g)[:s].sort().values.to(torch.uint8).numpy()
    codes = torch.randint(-qmax, qmax + 1, (s,), generator=g).to(torch.int8).numpy()
    scale = _fp16_bits([0.013])
    return cc, cs, idx, codes, scale


def _cbar(cc, cs, r):
    """fp64 values of the first r coefficients: code x block scale."""
    sc = _bits_to_f64(cs, torch.float16)
    return np.array([float(cc[j]) * sc[j // 16] for j in range(r)], np.float64)


def _xh_perm(d, perm, sign, r_old, cc, cs, idx, codes, scale):
    """The bf16 reconstruction with a signed-permutation basis from its definition: channel
    perm(j) holds sign_j cbar_j (exact), the residual channels add scale x code (one fp32
    rounding), and the vector rounds to bf16 once."""
    a = np.zeros(d, np.float32)
    cb = _cbar(cc, cs, r_old)
    for j in range(r_old):
        a[int(perm[j])] = np.float32(sign[j] * cb[j])
    sf = np.float32(_bits_to_f64(scale, torch.float16)[0])
    for i, q in zip(idx, codes):
        a[int(i)] = np.float32(a[int(i)] + np.float32(sf * np.float32(q)))
    return _bf16_bits(a)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("r", [16, 32, 64])
def test_same_rank_without_residual_is_the_identity(bits, r):
    d, r_max, s = 128, 64, 16
    Bm, perm, sign = signed_permutation(d, r_max, 50 + r)
    cc, cs, idx, codes, _ = _token8(d, r_max, r, s, bits, 51 + r)
    out = oracle.reencode_vector8(Bm, r, cc, cs, idx, codes, _fp16_bits([0.0]), r, bits)
    assert np.array_equal(out["ccodes"][:r], cc[:r]) and not out["ccodes"][r:].any()
    assert np.array_equal(out["cscales"][:r // 16], cs[:r // 16]) and not out["cscales"][r // 16:].any()
    assert out["scale"] == 0 and not out["codes"].any()
    assert list(out["idx"]) == list(range(s))            # all-zero residual: ties to the lowest channels


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("r_old,r_new", [(16, 64), (32, 64), (16, 32)])
def test_promotion_with_a_permutation_basis_matches_the_closed_form(bits, r_old, r_new):
    """The new projections are sign_j xh_{perm(j)} (one term each); their blockwise form is the
    pinned quantiser's; the residual is xh less the dequantised coefficients on their channels
    (one fp32 subtraction) and keeps its s largest magnitudes, ties to the lower channel."""
    d, r_max, s = 128, 64, 16
    Bm, perm, sign = signed_permutation(d, r_max, 60 + r_old)
    cc, cs, idx, codes, scale = _token8(d, r_max, r_old, s, bits, 61 + r_new)
    new_dirs = sorted(int(perm[j]) for j in range(r_old, r_new))[:6]          # residual on new directions
    idx = np.array(sorted(set(new_dirs) | set(idx.tolist()[: s - len(new_dirs)])), np.uint8)
    if idx.size < s:
        extra = [i for i in range(d) if i not in set(idx.tolist())][: s - idx.size]
        idx = np.array(sorted(idx.tolist() + extra), np.uint8)
    out = oracle.reencode_vector8(Bm, r_old, cc, cs, idx, codes, scale, r_new, bits)
    xh = _xh_perm(d, perm, sign, r_old, cc, cs, idx, codes, scale)
    assert np.array_equal(out["xh"], xh)
    xf = _bits_to_f64(xh, torch.bfloat16).astype(np.float32)
    proj = np.zeros(r_max, np.float32)
    proj[:r_new] = [np.float32(sign[j]) * xf[int(perm[j])] + np.float32(0.0) for j in range(r_new)]
    q = oracle.quantize_coeffs8(proj, r_new)
    assert np.array_equal(out["ccodes"], q["codes"]) and np.array_equal(out["cscales"], q["scales"])
    # the kept coefficients of the old blocks are unchanged (their blocks reach 127 at 2^e)
    # where no residual channel falls on their directions
    for b in range(r_old // 16):
        if not set(idx.tolist()) & {int(perm[j]) for j in range(16 * b, 16 * b + 16)}:
            assert np.array_equal(out["ccodes"][16 * b:16 * b + 16], cc[16 * b:16 * b + 16]) and out["cscales"][b] == cs[b]
    res = xf.copy()
    for j in range(r_new):
        res[int(perm[j])] = np.float32(xf[int(perm[j])] - np.float32(sign[j]) * q["cbar"][j])
    order = sorted(range(d), key=lambda i: (-abs(float(res[i])), i))[:s]
    assert list(out["idx"]) == sorted(order)


@pytest.mark.parametrize("bits", [8, 4])
def test_demotion_with_a_permutation_basis_moves_dropped_coefficients_to_the_residual(bits):
    d, r_max, s, r_old, r_new = 128, 64, 16, 64, 16
    Bm, perm, sign = signed_permutation(d, r_max, 71)
    cc, cs, idx, codes, scale = _token8(d, r_max, r_old, s, bits, 72)
    out = oracle.reencode_vector8(Bm, r_old, cc, cs, idx, codes, scale, r_new, bits)
    xh = _xh_perm(d, perm, sign, r_old, cc, cs, idx, codes, scale)
    assert np.array_equal(out["xh"], xh)
    xf = _bits_to_f64(xh, torch.bfloat16)
    # the first block is unchanged unless a residual channel landed on its directions
    if not set(idx.tolist()) & {int(perm[j]) for j in range(16)}:
        assert np.array_equal(out["ccodes"][:16], cc[:16]) and out["cscales"][0] == cs[0]
    got = _cbar(out["ccodes"], out["cscales"], r_new)
    r = xf.copy()
    for j in range(r_new):
        r[int(perm[j])] = float(np.float32(xf[int(perm[j])] - sign[j] * got[j]))
    order = sorted(range(d), key=lambda i: (-abs(r[i]), i))[:s]
    assert list(out["idx"]) == sorted(order)
    assert not out["ccodes"][r_new:].any() and not out["cscales"][r_new // 16:].any()


def test_dense_basis_reconstruction_is_within_bf16_rounding_of_fp64():
    """xh against x = B cbar + scatter(scale x code), written in fp64 with numpy."""
    wl = synth.workload("llama8b_64k")
    bases = synth.make_bases(wl.scaled(num_layers=2))
    Bm = bases[0][0, 1]
    B = bf16_np(Bm)
    for seed in range(20):
        r_old = (16, 32, 64)[seed % 3]
        cc, cs, idx, codes, scale = _token8(128, 64, r_old, 16, 4, 200 + seed)
        out = oracle.reencode_vector8(Bm, r_old, cc, cs, idx, codes, scale, 64, 4)
        ref = B[:, :r_old] @ _cbar(cc, cs, r_old)
        ref[idx.astype(np.int64)] += _bits_to_f64(scale, torch.float16)[0] * codes.astype(np.float64)
        xh = _bits_to_f64(out["xh"], torch.bfloat16)
        assert np.all(np.abs(xh - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6 * np.linalg.norm(ref)), seed


@pytest.mark.parametrize("r_old", [16, 32, 64])
def test_reconstruction_matches_the_bf16_form_on_shared_values(r_old):
    """Power-of-two block scales make every cbar_j = code x 2^e a bf16 value: the bf16 re-encode
    of those coefficients reconstructs the same xh."""
    wl = synth.workload("llama8b_64k")
    Bm = synth.make_bases(wl.scaled(num_layers=2))[1][0, 0]
    cc, cs, idx, codes, scale = _token8(128, 64, r_old, 16, 4, 300 + r_old)
    cb = np.zeros(64)
    cb[:r_old] = _cbar(cc, cs, r_old)
    c16 = torch.from_numpy(cb).to(torch.bfloat16)
    assert np.array_equal(bf16_np(c16), cb)
    sc = torch.from_numpy(np.asarray(scale).view(np.float16).copy())
    a = oracle.reencode_vector8(Bm, r_old, cc, cs, idx, codes, scale, 32, 4)
    b = oracle.reencode_vector(Bm, r_old, c16, torch.from_numpy(idx), torch.from_numpy(codes), sc, 32, 4)
    assert np.array_equal(a["xh"], b["xh"])
    # and the same residual-count change, at the same rank, on both
    a2 = oracle.reencode_vector8(Bm, r_old, cc, cs, idx, codes, scale, r_old, 4, s_new=8)
    b2 = oracle.reencode_vector(Bm, r_old, c16, torch.from_numpy(idx), torch.from_numpy(codes), sc, r_old, 4, s_new=8)
    assert np.array_equal(a2["xh"], b2["xh"]) and a2["idx"].shape == (8,)


def test_basis_update_moves_onto_the_new_permutation():
    """basis_new another signed permutation: the new projections are sign'_j xh_{perm'(j)};
    basis_new equal to the basis is the plain re-encode."""
    d, r_max, r, s, bits = 128, 64, 32, 16, 4
    B0, p0, s0 = signed_permutation(d, r_max, 81)
    B1, p1, s1 = signed_permutation(d, r_max, 82)
    cc, cs, idx, codes, scale = _token8(d, r_max, r, s, bits, 83)
    out = oracle.reencode_vector8(B0, r, cc, cs, idx, codes, scale, r, bits, basis_new=B1)
    xh = _xh_perm(d, p0, s0, r, cc, cs, idx, codes, scale)
    assert np.array_equal(out["xh"], xh)
    xf = _bits_to_f64(xh, torch.bfloat16).astype(np.float32)
    proj = np.zeros(r_max, np.float32)
    proj[:r] = [np.float32(s1[j]) * xf[int(p1[j])] + np.float32(0.0) for j in range(r)]
    q = oracle.quantize_coeffs8(proj, r)
    assert np.array_equal(out["ccodes"], q["codes"]) and np.array_equal(out["cscales"], q["scales"])
    same = oracle.reencode_vector8(B0, r, cc, cs, idx, codes, scale, r, bits, basis_new=B0)
    plain = oracle.reencode_vector8(B0, r, cc, cs, idx, codes, scale, r, bits)
    for k in ("ccodes", "cscales", "idx", "codes", "xh"):
        assert np.array_equal(same[k], plain[k]), k
    assert same["scale"] == plain["scale"]


def test_bad_arguments_are_refused():
    Bm, _, _ = signed_permutation(128, 64, 1)
    cc, cs, idx, codes, scale = _token8(128, 64, 32, 16, 4, 2)
    with pytest.raises(ValueError):
        oracle.reencode_vector8(Bm, 24, cc, cs, idx, codes, scale, 32, 4)       # r_old not a multiple of 16
    with pytest.raises(ValueError):
        oracle.reencode_vector8(Bm, 32, cc, cs, idx, codes, scale, 40, 4)       # r_new not a multiple of 16
