"""Pins of the CPU oracle's decode and probe ("DepthWeave-KV: Token-Adaptive Cross-Layer
Residual Factorization for Long-Context KV Cache Compression", §3 Method, Eq. (1) and
Eq. (3)) against closed forms, exact special cases and numpy library routines."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import (bf16_np, head_problem, np_attention, np_reconstruct, rel_l2,
                     signed_permutation, tau_of)

D = 128


def _random_kv(T, seed):
    g = torch.Generator().manual_seed(seed)
    K = torch.randn(T, D, generator=g).to(torch.bfloat16)
    V = torch.randn(T, D, generator=g).to(torch.bfloat16)
    q = (torch.randn(4, D, generator=g) * 0.5).to(torch.bfloat16)
    return K, V, q


def _zero_resid(T, s=8):
    return (torch.zeros(T, s, dtype=torch.uint8), torch.zeros(T, s, dtype=torch.int8),
            torch.zeros(T, dtype=torch.float16))


def _problem(bk, bv, ranks, ck, cv, rk, rv, q):
    return oracle.HeadProblem(bk, bv, ranks, ck, rk[0], rk[1], rk[2], cv, rv[0], rv[1], rv[2], q)


def test_full_rank_orthonormal_zero_residual_is_dense_attention():
    """Invariant (a): r_t = d, orthonormal B, zero residual -> dense attention on K, V.
    A signed permutation basis is exactly orthonormal in bf16, so c = B^T K is exact."""
    T = 200
    K, V, q = _random_kv(T, 1)
    B, perm, sign = signed_permutation(D, D, 7)
    Bf = B.float()
    ck = (K.float() @ Bf).to(torch.bfloat16)      # exact: each entry is +-one element of K
    cv = (V.float() @ Bf).to(torch.bfloat16)
    assert torch.equal(ck.float() @ Bf.T, K.float())
    prob = _problem(B, B, np.full(T, D, np.int32), ck, cv, _zero_resid(T), _zero_resid(T), q)
    out = oracle.decode_head(prob)
    ref, _ = np_attention(bf16_np(q), bf16_np(K), bf16_np(V), tau_of(D))
    assert np.max(np.abs(out - ref)) < 1e-12


def test_full_rank_qr_basis_matches_numpy_reconstruction():
    """Full rank with a general (bf16-rounded QR) basis: same as numpy matmul reconstruction."""
    wl = synth.workload("tiny_1k").scaled(r_max=128, tiers=(128,), tier_probs=(1.0,))
    bases = synth.make_bases(wl)
    T = 96
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    comp["scales"].zero_()
    q = synth.make_queries(wl, 0)[0]
    prob = head_problem(wl, bases, tiers, comp, q, 0, 0)
    out = oracle.decode_head(prob)
    K = np_reconstruct(bases[0][0, 0], prob.rank, comp["coeff"][:, 0, 0], comp["idx"][:, 0, 0],
                       comp["codes"][:, 0, 0], comp["scales"][:, 0, 0])
    V = np_reconstruct(bases[1][0, 0], prob.rank, comp["coeff"][:, 0, 1], comp["idx"][:, 0, 1],
                       comp["codes"][:, 0, 1], comp["scales"][:, 0, 1])
    ref, _ = np_attention(bf16_np(q[:4]), K, V, tau_of(D))
    assert rel_l2(out, ref) < 1e-13


@pytest.mark.parametrize("r", [8, 32, 96])
def test_uniform_rank_is_attention_over_projected_keys(r):
    """Invariant (b): uniform rank r, zero residual -> attention over B_r B_r^T K, B_r B_r^T V.
    With a signed permutation basis the projection keeps r channels and zeroes the rest."""
    T = 150
    K, V, q = _random_kv(T, 2 + r)
    B, perm, sign = signed_permutation(D, D, 11 + r)
    Bf = B.float()
    ck = (K.float() @ Bf).to(torch.bfloat16)
    cv = (V.float() @ Bf).to(torch.bfloat16)
    prob = _problem(B, B, np.full(T, r, np.int32), ck, cv, _zero_resid(T), _zero_resid(T), q)
    out = oracle.decode_head(prob)
    keep = np.zeros(D)
    keep[perm[:r].numpy()] = 1.0
    ref, _ = np_attention(bf16_np(q), bf16_np(K) * keep, bf16_np(V) * keep, tau_of(D))
    assert np.max(np.abs(out - ref)) < 1e-12


def test_brute_force_loop_tiny():
    """Invariant (c): one head, 8 tokens, mixed ranks and residuals, pure-Python loops."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 8
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 1, tiers)
    q = synth.make_queries(wl, 1)[0] * 4
    prob = head_problem(wl, bases, tiers, comp, q, 1, 0)
    out, p = oracle.decode_head(prob, want_p=True)

    Bk = bf16_np(bases[0][0, 0]).tolist()
    Bv = bf16_np(bases[1][0, 0]).tolist()
    qq = bf16_np(q[:4]).tolist()
    ranks = prob.rank.tolist()

    def vec(basis, z, t):
        c = bf16_np(comp["coeff"][t, 0, z]).tolist()
        x = [0.0] * D
        for i in range(D):
            for j in range(ranks[t]):
                x[i] += basis[i][j] * c[j]
        sc = float(comp["scales"][t, 0, z].double())
        for k in range(comp["idx"].shape[-1]):
            x[int(comp["idx"][t, 0, z, k])] += sc * int(comp["codes"][t, 0, z, k])
        return x

    Ks = [vec(Bk, 0, t) for t in range(T)]
    Vs = [vec(Bv, 1, t) for t in range(T)]
    tau = 1.0 / math.sqrt(D)
    for h in range(4):
        sc = [tau * sum(qq[h][i] * Ks[t][i] for i in range(D)) for t in range(T)]
        m = max(sc)
        e = [math.exp(x - m) for x in sc]
        z = sum(e)
        w = [x / z for x in e]
        for i in range(D):
            o = sum(w[t] * Vs[t][i] for t in range(T))
            assert abs(o - out[h, i]) < 1e-12
        for t in range(T):
            assert abs(w[t] - p[h, t]) < 1e-14


@pytest.mark.parametrize("temp", [1.0, 8.0, 32.0])
def test_softmax_weights_sum_to_one_and_match_numpy(temp):
    """Invariant (d) plus a numpy restatement over the tiny workload, at several query
    temperatures (x32 makes the softmax peaky)."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 1024
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    q = synth.make_queries(wl, 0, temperature=temp)[0]
    prob = head_problem(wl, bases, tiers, comp, q, 0, 0)
    out, p = oracle.decode_head(prob, want_p=True)
    assert np.all(p >= 0)
    assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-12
    K = np_reconstruct(bases[0][0, 0], prob.rank, comp["coeff"][:, 0, 0], comp["idx"][:, 0, 0],
                       comp["codes"][:, 0, 0], comp["scales"][:, 0, 0])
    V = np_reconstruct(bases[1][0, 0], prob.rank, comp["coeff"][:, 0, 1], comp["idx"][:, 0, 1],
                       comp["codes"][:, 0, 1], comp["scales"][:, 0, 1])
    ref, pref = np_attention(bf16_np(q[:4]), K, V, tau_of(D))
    assert rel_l2(out, ref) < 1e-12
    assert np.max(np.abs(p - pref)) < 1e-13


def test_token_permutation_invariance():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 300
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    q = synth.make_queries(wl, 0, temperature=8.0)[0]
    out = oracle.decode_head(head_problem(wl, bases, tiers, comp, q, 0, 0))
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(5))
    comp2 = {k: v[perm] for k, v in comp.items()}
    out2 = oracle.decode_head(head_problem(wl, bases, tiers[perm], comp2, q, 0, 0))
    assert np.max(np.abs(out - out2)) < 1e-13


def test_single_token_output_is_its_value_vector():
    """T = 1: the softmax weight is 1, so o = V^_0 for every query head."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    tiers = synth.make_tiers(wl, 3, 0, 1)
    comp = synth.make_compressed(wl, 3, 0, tiers)
    q = synth.make_queries(wl, 0, temperature=32.0)[0]
    prob = head_problem(wl, bases, tiers, comp, q, 0, 0)
    out = oracle.decode_head(prob)
    V = np_reconstruct(bases[1][0, 0], prob.rank, comp["coeff"][:, 0, 1], comp["idx"][:, 0, 1],
                       comp["codes"][:, 0, 1], comp["scales"][:, 0, 1])
    for h in range(4):
        assert np.max(np.abs(out[h] - V[0])) < 1e-15


def test_zero_query_gives_mean_value():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 77
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    q = torch.zeros(4, D, dtype=torch.bfloat16)
    prob = head_problem(wl, bases, tiers, comp, q, 0, 0)
    out = oracle.decode_head(prob)
    V = np_reconstruct(bases[1][0, 0], prob.rank, comp["coeff"][:, 0, 1], comp["idx"][:, 0, 1],
                       comp["codes"][:, 0, 1], comp["scales"][:, 0, 1])
    assert np.max(np.abs(out - V.mean(axis=0)[None, :])) < 1e-14


def test_coefficients_beyond_rank_are_ignored():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 64
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    q = synth.make_queries(wl, 0, temperature=8.0)[0]
    out = oracle.decode_head(head_problem(wl, bases, tiers, comp, q, 0, 0))
    ranks = synth.ranks_of(wl, tiers)
    junk = torch.randn(comp["coeff"].shape, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    j = torch.arange(wl.r_max).view(1, 1, 1, -1)
    comp2 = dict(comp)
    comp2["coeff"] = torch.where(j < ranks.view(T, 1, 1, 1), comp["coeff"], junk)
    assert not torch.equal(comp2["coeff"], comp["coeff"])
    out2 = oracle.decode_head(head_problem(wl, bases, tiers, comp2, q, 0, 0))
    assert np.array_equal(out, out2)


def test_residual_only_cache():
    """Zero coefficients: K^ and V^ are the scattered residuals alone."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 40
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    comp["coeff"].zero_()
    q = synth.make_queries(wl, 0, temperature=32.0)[0]
    prob = head_problem(wl, bases, tiers, comp, q, 0, 0)
    out = oracle.decode_head(prob)
    K = np.zeros((T, D))
    V = np.zeros((T, D))
    sk = bf16_np(comp["scales"][:, 0, 0])
    sv = bf16_np(comp["scales"][:, 0, 1])
    for t in range(T):
        for k in range(wl.resid_channels):
            K[t, int(comp["idx"][t, 0, 0, k])] += sk[t] * int(comp["codes"][t, 0, 0, k])
            V[t, int(comp["idx"][t, 0, 1, k])] += sv[t] * int(comp["codes"][t, 0, 1, k])
    ref, _ = np_attention(bf16_np(q[:4]), K, V, tau_of(D))
    assert np.max(np.abs(out - ref)) < 1e-14


def test_identical_query_heads_give_identical_outputs():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 50
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    q = synth.make_queries(wl, 0)[0]
    q[1:4] = q[0]
    out = oracle.decode_head(head_problem(wl, bases, tiers, comp, q, 0, 0))
    for h in range(1, 4):
        assert np.array_equal(out[h], out[0])


def test_empty_cache_gives_zero_output():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    tiers = torch.zeros(0, 1, dtype=torch.uint8)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    q = synth.make_queries(wl, 0)[0]
    out = oracle.decode_head(head_problem(wl, bases, tiers, comp, q, 0, 0))
    assert np.array_equal(out, np.zeros((4, D)))


def test_custom_softmax_scale():
    """tau enters only as a multiplier of the scores."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 64
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    q = synth.make_queries(wl, 0)[0]
    prob = head_problem(wl, bases, tiers, comp, q, 0, 0)
    out = oracle.decode_head(prob, tau=0.5)
    K = np_reconstruct(bases[0][0, 0], prob.rank, comp["coeff"][:, 0, 0], comp["idx"][:, 0, 0],
                       comp["codes"][:, 0, 0], comp["scales"][:, 0, 0])
    V = np_reconstruct(bases[1][0, 0], prob.rank, comp["coeff"][:, 0, 1], comp["idx"][:, 0, 1],
                       comp["codes"][:, 0, 1], comp["scales"][:, 0, 1])
    ref, _ = np_attention(bf16_np(q[:4]), K, V, 0.5)
    assert rel_l2(out, ref) < 1e-12


# ------------------------------------------------------------------------------ probe (Eq. 3)
def test_probe_zero_residual_is_zero():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 128
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 0, tiers)
    comp["scales"].zero_()
    q = synth.make_queries(wl, 0)[0]
    err, of, on = oracle.probe_head(head_problem(wl, bases, tiers, comp, q, 0, 0))
    assert err == 0.0
    assert np.array_equal(of, on)


def test_probe_single_token_closed_form():
    """T = 1: both softmaxes put weight 1 on the token, so o_full - o_nores is the value
    residual R^V for every query head: e = sqrt(gq)|R^V| / (sqrt(gq)|V^| + eps)."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    tiers = synth.make_tiers(wl, 1, 0, 1)
    comp = synth.make_compressed(wl, 1, 0, tiers)
    q = synth.make_queries(wl, 0)[0]
    prob = head_problem(wl, bases, tiers, comp, q, 0, 0)
    err, of, on = oracle.probe_head(prob, eps=1e-6)
    R = np.zeros(D)
    sv = float(comp["scales"][0, 0, 1].double())
    for k in range(wl.resid_channels):
        R[int(comp["idx"][0, 0, 1, k])] += sv * int(comp["codes"][0, 0, 1, k])
    V = np_reconstruct(bases[1][0, 0], prob.rank, comp["coeff"][:, 0, 1], comp["idx"][:, 0, 1],
                       comp["codes"][:, 0, 1], comp["scales"][:, 0, 1])[0]
    expect = 2.0 * np.linalg.norm(R) / (2.0 * np.linalg.norm(V) + 1e-6)
    assert abs(err - expect) < 1e-13


def test_probe_matches_numpy_two_caches():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T = 512
    tiers = synth.make_tiers(wl, 0, 0, T)
    comp = synth.make_compressed(wl, 0, 1, tiers)
    q = synth.make_queries(wl, 1, temperature=8.0)[0]
    prob = head_problem(wl, bases, tiers, comp, q, 1, 0)
    err, of, on = oracle.probe_head(prob)
    args = (comp["coeff"][:, 0, 0], comp["idx"][:, 0, 0], comp["codes"][:, 0, 0], comp["scales"][:, 0, 0])
    argv = (comp["coeff"][:, 0, 1], comp["idx"][:, 0, 1], comp["codes"][:, 0, 1], comp["scales"][:, 0, 1])
    a, _ = np_attention(bf16_np(q[:4]), np_reconstruct(bases[0][0, 0], prob.rank, *args),
                        np_reconstruct(bases[1][0, 0], prob.rank, *argv), tau_of(D))
    b, _ = np_attention(bf16_np(q[:4]), np_reconstruct(bases[0][0, 0], prob.rank, *args, with_residual=False),
                        np_reconstruct(bases[1][0, 0], prob.rank, *argv, with_residual=False), tau_of(D))
    expect = np.linalg.norm(a - b) / (np.linalg.norm(a) + 1e-6)
    assert abs(err - expect) < 1e-12
    assert rel_l2(of, a) < 1e-12 and rel_l2(on, b) < 1e-12
    assert 0.0 < err < 1.0


def test_decode_many_equals_single_calls():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    probs = []
    for layer in range(2):
        T = 100 + 37 * layer
        tiers = synth.make_tiers(wl, 0, 0, T)
        comp = synth.make_compressed(wl, 0, layer, tiers)
        q = synth.make_queries(wl, layer)[0]
        probs.append(head_problem(wl, bases, tiers, comp, q, layer, 0))
    many = oracle.decode_many(probs, nthreads=2)
    for pr, o in zip(probs, many):
        assert np.array_equal(o, oracle.decode_head(pr))
