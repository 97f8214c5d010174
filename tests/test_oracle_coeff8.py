"""Pins of the oracle's 8-bit blockwise coefficient form ("DepthWeave-KV: Token-Adaptive
Cross-Layer Residual Factorization for Long-Context KV Cache Compression", §3 Method: the
coefficient vector is the projection onto the current basis, kept as 8-bit codes with one
scale per block of coefficients).  The block of 16 and the symmetric max-scaled codes are
the reading taken here (the pages give no block size); the checks rest on values that sit
exactly on the code grid, the rounding rule, the quantiser's error bound, block locality and
exact signed-permutation bases, and the decode path is checked against dense attention over
the dequantised cache."""
import numpy as np
import pytest
import torch

import oracle
from helpers import bf16_np, np_attention, signed_permutation, tau_of

D = 128


def _fp16_bits(v: float) -> int:
    return int(np.array([v], np.float16).view(np.uint16)[0])


def test_grid_values_are_kept_exactly():
    """Coefficients k 2^-8 with |k| <= 127 and one |k| = 127 in every block: the scale is
    exactly 2^-8, the codes are k and the dequantised values are the inputs."""
    rng = np.random.default_rng(1)
    r_max, r_t = 64, 48
    k = rng.integers(-127, 128, r_max)
    for b in range(r_max // 16):
        k[16 * b + int(rng.integers(16))] = 127 if b % 2 else -127
    c = (k * 2.0 ** -8).astype(np.float32)
    out = oracle.quantize_coeffs8(c, r_t)
    assert out["codes"][:r_t].tolist() == k[:r_t].tolist()
    assert not out["codes"][r_t:].any() and not out["cbar"][r_t:].any()
    assert out["scales"].tolist() == [_fp16_bits(2.0 ** -8)] * 3 + [0]
    assert np.array_equal(out["cbar"][:r_t], c[:r_t])


def test_rounding_is_to_nearest_even():
    """Scale 2^-4 (set by a 127 x 2^-4 entry); codes of x.5 grid points round to even."""
    c = np.zeros(16, np.float32)
    c[0] = 127 * 2.0 ** -4
    c[1:7] = np.array([2.5, 3.5, -2.5, -3.5, 0.49, -126.5]) * 2.0 ** -4
    out = oracle.quantize_coeffs8(c, 16)
    assert out["codes"][:7].tolist() == [127, 2, 4, -2, -4, 0, -126]
    assert out["scales"][0] == _fp16_bits(2.0 ** -4)


def test_zero_and_empty_blocks():
    c = np.zeros(32, np.float32)
    c[16:] = np.linspace(-1, 1, 16)
    out = oracle.quantize_coeffs8(c, 32)
    assert out["scales"][0] == 0 and not out["codes"][:16].any() and not out["cbar"][:16].any()
    out0 = oracle.quantize_coeffs8(c, 0)
    assert not out0["codes"].any() and not out0["scales"].any()
    with pytest.raises(ValueError):
        oracle.quantize_coeffs8(c, 8)                 # ranks come in whole blocks


def test_error_bound_and_block_locality():
    """|c - cbar| <= scale / 2 (plus the clamp of the block's largest entry, within 2^-11 of
    its scale-relative value), every code within [-127, 127], and each block's codes depend
    on its own coefficients only."""
    rng = np.random.default_rng(2)
    for trial in range(50):
        c = (rng.standard_normal(128) * 10.0 ** rng.uniform(-4, 3, 128)).astype(np.float32)
        out = oracle.quantize_coeffs8(c, 128)
        sc = oracle.fp16_to_f64(out["scales"])
        err = np.abs(c.astype(np.float64) - out["cbar"].astype(np.float64))
        bound = np.repeat(sc, 16) * (0.5 + 127 * 2.0 ** -10)
        assert np.all(err <= bound), trial
        assert np.all(np.abs(out["codes"].astype(int)) <= 127)
        # one block changed: the others keep their codes and scales
        c2 = c.copy()
        c2[32:48] = rng.standard_normal(16).astype(np.float32)
        out2 = oracle.quantize_coeffs8(c2, 128)
        keep = np.r_[0:32, 48:128]
        assert np.array_equal(out2["codes"][keep], out["codes"][keep])
        assert np.array_equal(np.delete(out2["scales"], 2), np.delete(out["scales"], 2))


def test_dequant_is_code_times_block_scale():
    codes = np.arange(-16, 16, dtype=np.int8)
    scales = np.array([_fp16_bits(0.5), _fp16_bits(-0.0)], np.uint16)
    got = oracle.dequant_coeffs8(codes, scales)
    assert np.array_equal(got, np.r_[np.arange(-16, 0) * 0.5, np.zeros(16)])


@pytest.mark.parametrize("bits", [8, 4])
def test_encode_on_a_signed_permutation_basis(bits):
    """Projections onto e_perm(j) * sign_j are exact (c_j = sign_j x_perm(j)); the residual is
    taken against the dequantised coefficients, so off the basis support it is x itself and
    on it the quantiser's error."""
    r_max, r_t, s = 64, 32, 16
    B, perm, sign = signed_permutation(D, r_max, 3)
    x = (torch.randn(D, generator=torch.Generator().manual_seed(4)) * 2).to(torch.bfloat16)
    xf = bf16_np(x).astype(np.float64)
    out = oracle.encode_vector8(B, x, r_t, s, bits)
    c = np.array([float(sign[j]) * xf[int(perm[j])] for j in range(r_t)])
    assert np.array_equal(out["c32"][:r_t].astype(np.float64), c)
    q = oracle.quantize_coeffs8(out["c32"], r_t)
    assert np.array_equal(out["ccodes"], q["codes"]) and np.array_equal(out["cscales"], q["scales"])
    # the residual the encoder selected from: x minus the dequantised basis part
    r = xf.copy()
    for j in range(r_t):
        r[int(perm[j])] -= float(sign[j]) * float(q["cbar"][j])
    sel = oracle.quantize_residual(r.astype(np.float32), s, bits)
    assert np.array_equal(out["idx"], sel["idx"]) and np.array_equal(out["codes"], sel["codes"])
    assert out["scale"] == sel["scale"]
    covered = {int(perm[j]) for j in range(r_t)}
    top = set(np.argsort(-np.abs(xf), kind="stable")[:4].tolist()) - covered
    assert top <= set(out["idx"].tolist())           # the largest uncovered channels are kept


def test_given_projections_replace_step_one():
    r_max = 32
    B, _, _ = signed_permutation(D, r_max, 5)
    x = torch.randn(D, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    c_in = np.random.default_rng(7).standard_normal(r_max).astype(np.float32)
    out = oracle.encode_vector8(B, x, 32, 8, 8, c_in=c_in)
    q = oracle.quantize_coeffs8(c_in, 32)
    assert np.array_equal(out["ccodes"], q["codes"])
    many = oracle.encode_many8(B, torch.stack([x, x]), [32, 16], 8, 8, c32=np.stack([c_in, c_in]))
    assert np.array_equal(many["ccodes"][0], q["codes"])
    assert np.array_equal(many["ccodes"][1], oracle.quantize_coeffs8(c_in, 16)["codes"])


def _problem8(seed, T=90, r_max=64, s=8, bits=8, tiers=(16, 32, 64)):
    g = torch.Generator().manual_seed(seed)
    bk = (torch.randn(D, r_max, generator=g) / 8).to(torch.bfloat16)
    bv = (torch.randn(D, r_max, generator=g) / 8).to(torch.bfloat16)
    x = torch.randn(2, T, D, generator=g).to(torch.bfloat16)
    ranks = np.array(tiers)[torch.randint(0, len(tiers), (T,), generator=g).numpy()].astype(np.int32)
    enc = [oracle.encode_many8(b, x[z], ranks, s, bits) for z, b in enumerate((bk, bv))]
    q = torch.randn(4, D, generator=g).to(torch.bfloat16)
    return bk, bv, ranks, enc, q


def test_decode_with_8bit_coefficients_is_dense_attention():
    """The decode path fed the dequantised coefficients equals softmax attention over the
    vectors B cbar + scale codes on their channels, built here densely."""
    bk, bv, ranks, enc, q = _problem8(8)
    ek, ev = enc
    ckf, cvf = oracle.dequant_coeffs8(ek["ccodes"], ek["cscales"]), oracle.dequant_coeffs8(ev["ccodes"], ev["cscales"])
    zero = np.zeros(ckf.shape, np.uint16)
    prob = oracle.HeadProblem(bk, bv, ranks, zero, ek["idx"], ek["codes"], ek["scale"],
                              zero, ev["idx"], ev["codes"], ev["scale"], q, coeff_k_f=ckf, coeff_v_f=cvf)
    tau = tau_of(D)
    got = oracle.decode_head(prob, tau=tau)

    def dense(b, cf, e):
        X = cf @ bf16_np(b).astype(np.float64).T
        sc = oracle.fp16_to_f64(e["scale"])
        for t in range(X.shape[0]):
            X[t, e["idx"][t]] += sc[t] * e["codes"][t].astype(np.float64)
        return X

    want, _ = np_attention(bf16_np(q).astype(np.float64), dense(bk, ckf, ek), dense(bv, cvf, ev), tau)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)
    # the bf16 coefficient arrays are not read when the fp64 values are given
    garbage = np.full(ckf.shape, 0x7FC0, np.uint16)
    prob2 = oracle.HeadProblem(bk, bv, ranks, garbage, ek["idx"], ek["codes"], ek["scale"],
                               garbage, ev["idx"], ev["codes"], ev["scale"], q, coeff_k_f=ckf, coeff_v_f=cvf)
    assert np.array_equal(oracle.decode_head(prob2, tau=tau), got)
    assert np.array_equal(oracle.decode_many([prob, prob2], tau=tau)[1], got)
    err, o_full, _ = oracle.probe_head(prob, tau=tau)
    assert np.array_equal(o_full, got) and err >= 0.0


def test_fp64_path_with_bf16_values_is_the_bf16_path():
    bk, bv, ranks, enc, q = _problem8(9, T=40)
    ek, ev = enc
    g = torch.Generator().manual_seed(10)
    ck = torch.randn(40, 64, generator=g).to(torch.bfloat16)
    cv = torch.randn(40, 64, generator=g).to(torch.bfloat16)
    base = oracle.HeadProblem(bk, bv, ranks, ck, ek["idx"], ek["codes"], ek["scale"],
                              cv, ev["idx"], ev["codes"], ev["scale"], q)
    viaf = oracle.HeadProblem(bk, bv, ranks, ck, ek["idx"], ek["codes"], ek["scale"],
                              cv, ev["idx"], ev["codes"], ev["scale"], q,
                              coeff_k_f=bf16_np(ck).astype(np.float64), coeff_v_f=bf16_np(cv).astype(np.float64))
    assert np.array_equal(oracle.decode_head(base), oracle.decode_head(viaf))
    # decode_many mixes problems with and without fp64 values
    outs = oracle.decode_many([base, viaf])
    assert np.array_equal(outs[0], outs[1])


def test_residual_is_taken_against_the_dequantised_coefficients():
    """x on the basis support only, off the code grid: the residual is exactly the quantiser's
    error, so it is nonzero, sits on covered channels and shrinks the reconstruction error."""
    r_max, r_t, s = 32, 32, 8
    B, perm, sign = signed_permutation(D, r_max, 11)
    g = torch.Generator().manual_seed(12)
    x = torch.zeros(D)
    x[perm] = torch.randn(r_max, generator=g) * sign.float()
    x = x.to(torch.bfloat16)
    xf = bf16_np(x).astype(np.float64)
    out = oracle.encode_vector8(B, x, r_t, s, 8)
    assert out["scale"] != 0
    assert set(out["idx"].tolist()) <= {int(p) for p in perm}
    cb = oracle.dequant_coeffs8(out["ccodes"], out["cscales"])
    base = bf16_np(B).astype(np.float64) @ cb
    full = base.copy()
    full[out["idx"]] += oracle.fp16_to_f64(np.array([out["scale"]]))[0] * out["codes"].astype(np.float64)
    assert np.linalg.norm(full - xf) < 0.9 * np.linalg.norm(base - xf)
    # the kept channels are those of the largest quantiser errors
    assert sorted(out["idx"].tolist()) == sorted(np.argsort(-np.abs(xf - base), kind="stable")[:s].tolist())
