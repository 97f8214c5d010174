"""Pins of the oracle's residual gate ("DepthWeave-KV ...", §3 Method, Eq. (1): the residual
enters the reconstruction as g R with g in [0, 1]); the build folds g into the dequantisation,
storing fp16_rn(g * scale) in place of the token's residual scale.  Checks: g = 1 is the
identity on every finite fp16 scale, g = 1/2 and 1/4 move the exponent exactly, g = 0 gives
+0, and decode over gated scales is dense attention with the residual scaled by g."""
import numpy as np
import torch

import oracle
from helpers import bf16_np, np_attention, signed_permutation, tau_of

D = 128


def _finite_fp16_bits():
    b = np.arange(0x7c00, dtype=np.uint16)                 # +0 .. largest finite, positive
    return b


def test_gate_one_is_the_identity():
    b = _finite_fp16_bits()
    assert np.array_equal(oracle.gate_scales(b, np.ones(b.size, np.float32)), b)


def test_power_of_two_gates_shift_the_exponent():
    b = _finite_fp16_bits()
    normal = b[(b >> 10) >= 3]                             # halving twice stays normal
    assert np.array_equal(oracle.gate_scales(normal, np.full(normal.size, 0.5, np.float32)), normal - 0x0400)
    assert np.array_equal(oracle.gate_scales(normal, np.full(normal.size, 0.25, np.float32)), normal - 0x0800)
    assert not oracle.gate_scales(b, np.zeros(b.size, np.float32)).any()


def test_gate_rounds_once_from_the_fp32_product():
    rng = np.random.default_rng(3)
    s = (rng.random(5000) * 0.1).astype(np.float16)
    g = rng.random(5000).astype(np.float32)
    want = (g * s.astype(np.float32)).astype(np.float16)    # fp32 product, then RNE to fp16
    assert np.array_equal(oracle.gate_scales(s.view(np.uint16), g), want.view(np.uint16))


def test_decode_with_a_half_gate_is_attention_over_half_residuals():
    r_max, T, s = 32, 70, 8
    g = torch.Generator().manual_seed(5)
    B, _, _ = signed_permutation(D, r_max, 6)
    bk = bv = B
    ranks = np.full(T, 16, np.int32)
    coeff = (torch.randn(2, T, r_max, generator=g) * 0.5).to(torch.bfloat16)
    coeff[:, :, 16:] = 0
    idx = torch.stack([torch.randperm(D, generator=g)[:s].sort().values for _ in range(2 * T)]).view(2, T, s).to(torch.uint8)
    codes = torch.randint(-127, 128, (2, T, s), generator=g).to(torch.int8)
    scales = (torch.rand(2, T, generator=g) * 0.01 + 0.001).to(torch.float16)
    q = torch.randn(4, D, generator=g).to(torch.bfloat16)
    gated = [oracle.gate_scales(scales[z], np.full(T, 0.5, np.float32)) for z in range(2)]
    prob = oracle.HeadProblem(bk, bv, ranks, coeff[0], idx[0], codes[0], gated[0], coeff[1], idx[1], codes[1],
                              gated[1], q)
    got = oracle.decode_head(prob, tau=tau_of(D))

    def dense(z):
        X = bf16_np(coeff[z]).astype(np.float64) @ bf16_np(B).astype(np.float64).T
        sc = scales[z].numpy().astype(np.float64) * 0.5
        for t in range(T):
            X[t, idx[z, t].numpy()] += sc[t] * codes[z, t].numpy().astype(np.float64)
        return X

    want, _ = np_attention(bf16_np(q).astype(np.float64), dense(0), dense(1), tau_of(D))
    assert np.allclose(got, want, rtol=1e-12, atol=1e-14)
