"""Pins of the oracle's per-token residual counts ("DepthWeave-KV ...", §3 Eq. (2): the
router's level rho in {0, 2, 4, 8} is the number of residual channels a token keeps, at a fixed
basis rank): decode and probe against a numpy restatement that scatter-adds only each token's
kept entries, entries past a token's count ignored whatever they hold, and the encoder's
selection of rho channels against a brute-force sort."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import bf16_np, np_attention, np_reconstruct, rel_l2, tau_of

D = 128


def _routed_problem(T, s_max, levels, seed, garbage=False):
    g = torch.Generator().manual_seed(seed)
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl.scaled(r_max=32), seed=seed)
    bk, bv = bases[0][0, 0], bases[1][0, 0]
    ranks = torch.full((T,), 32, dtype=torch.int32)
    nres = torch.tensor(levels, dtype=torch.int32)[torch.randint(0, len(levels), (T,), generator=g)]
    def part():
        c = (torch.randn(T, 32, generator=g) * 0.5).to(torch.bfloat16)
        idx = torch.stack([torch.randperm(D, generator=g)[:s_max].sort().values for _ in range(T)]).to(torch.uint8)
        codes = torch.randint(-127, 128, (T, s_max), generator=g).to(torch.int8)
        if not garbage:
            keep = torch.arange(s_max)[None, :] < nres[:, None]
            codes = torch.where(keep, codes, torch.zeros_like(codes))
        scales = (torch.rand(T, generator=g) * 0.01).to(torch.float16)
        return c, idx, codes, scales
    ck, ik, qk, sk = part()
    cv, iv, qv, sv = part()
    q = (torch.randn(4, D, generator=g) * 0.6).to(torch.bfloat16)
    prob = oracle.HeadProblem(bk, bv, ranks, ck, ik, qk, sk, cv, iv, qv, sv, q, nres=nres)
    return prob, (bk, bv, ranks, ck, ik, qk, sk, cv, iv, qv, sv, q, nres)


def _np_routed(bk, ranks, c, idx, codes, scales, nres):
    """Reconstruction keeping only each token's first nres entries (numpy matmul + scatter)."""
    keep = (torch.arange(idx.shape[1])[None, :] < nres[:, None])
    return np_reconstruct(bk, ranks, c, idx, torch.where(keep, codes, torch.zeros_like(codes)), scales)


@pytest.mark.parametrize("garbage", [False, True])
def test_decode_with_residual_counts_matches_numpy(garbage):
    T, s_max = 300, 8
    prob, (bk, bv, ranks, ck, ik, qk, sk, cv, iv, qv, sv, q, nres) = _routed_problem(T, s_max, (0, 2, 4, 8), 5, garbage)
    K = _np_routed(bk, ranks, ck, ik, qk, sk, nres)
    V = _np_routed(bv, ranks, cv, iv, qv, sv, nres)
    want, _ = np_attention(bf16_np(q), K, V, tau_of(D) * 8.0)
    got = oracle.decode_head(prob, tau=tau_of(D) * 8.0)
    assert rel_l2(got, want) < 1e-12


def test_counts_of_zero_everywhere_give_a_zero_probe():
    T = 200
    prob, _ = _routed_problem(T, 8, (0,), 6, garbage=True)
    err, _, _ = oracle.probe_head(prob)
    assert err == 0.0


def test_decode_many_carries_the_counts():
    probs = [_routed_problem(150 + 17 * k, 8, (0, 2, 4, 8), 40 + k, garbage=True)[0] for k in range(4)]
    outs = oracle.decode_many(probs, nthreads=2)
    for p, o in zip(probs, outs):
        assert np.array_equal(o, oracle.decode_head(p))


@pytest.mark.parametrize("bits", [8, 4])
def test_encode_keeps_the_rho_largest_residual_channels(bits):
    """Per-vector counts: the kept channels are the rho largest |r| (ties to the lower channel),
    in ascending order, exactly as an encode with s = rho; entries past rho stay zero."""
    wl = synth.workload("llama8b_64k")
    bases = synth.make_bases(wl.scaled(num_layers=2))
    Bm = bases[0][0, 0]
    n, s_max = 64, 8
    x = synth.make_dense_vectors(wl.scaled(noise_var=0.05), 0, 0, n, bases)[0][:, 0]
    ranks = torch.full((n,), 32, dtype=torch.int32)
    nres = torch.tensor([0, 2, 4, 8] * (n // 4), dtype=torch.int32)
    got = oracle.encode_many(Bm, x, ranks, s_max, bits, nres=nres)
    for t in range(n):
        k = int(nres[t])
        one = oracle.encode_vector(Bm, x[t], 32, k, bits)
        assert list(got["idx"][t, :k]) == list(one["idx"]) and list(got["codes"][t, :k]) == list(one["codes"])
        assert not got["idx"][t, k:].any() and not got["codes"][t, k:].any()
        r = oracle.encode_vector(Bm, x[t], 32, 0, bits)["resid"].astype(np.float64)
        order = sorted(range(D), key=lambda i: (-abs(r[i]), i))[:k]
        assert list(got["idx"][t, :k]) == sorted(order)
