"""Pins of the oracle's encoder ("DepthWeave-KV: Token-Adaptive Cross-Layer Residual
Factorization for Long-Context KV Cache Compression", §3 Method: coefficients are the
projection of the original vector onto the current basis; the residual is quantised and
kept on the routed channels) against hand-worked cases, exact constructions and
properties that fix the selection and the quantiser."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import bf16_np, bits16, signed_permutation

D = 128
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "encode_hand_cases.json")


def _x_from_sparse(entries):
    x = torch.zeros(D, dtype=torch.float32)
    for ch, v in entries.items():
        x[int(ch)] = v
    xb = x.to(torch.bfloat16)
    assert torch.equal(xb.float(), x) or all(v == 0 for v in entries.values())
    return xb


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_cases(case):
    basis = torch.zeros(D, 8, dtype=torch.bfloat16)
    x = _x_from_sparse(case["x"])
    out = oracle.encode_vector(basis, x, 0, case["s"], case["bits"])
    assert out["idx"].tolist() == case["idx"]
    assert out["codes"].tolist() == case["codes"]
    assert int(out["scale"]) == case["scale_bits"]
    assert not out["coeff"].any()


def test_hand_case_scales_agree_with_numpy_fp16():
    for case in json.load(open(GOLDEN))["cases"]:
        qmax = 127 if case["bits"] == 8 else 7
        vals = [abs(v) for v in case["x"].values()]
        amax = np.float32(sorted(vals, reverse=True)[0] if vals else 0.0)
        ref = (np.float32(amax) / np.float32(qmax)).astype(np.float16).view(np.uint16)
        assert int(ref) == case["scale_bits"], case["name"]


def _planted(seed, r_max, r_t, s, bits, n_planted):
    """x = B[:, :r_t] cb + sum of planted code*2^-k on channels outside the basis support,
    with B a signed permutation: every step of the encoder is exact, so the expected
    output is known in closed form."""
    g = torch.Generator().manual_seed(seed)
    B, perm, sign = signed_permutation(D, r_max, seed)
    qmax = 127 if bits == 8 else 7
    cb = torch.zeros(r_max)
    cb[:r_t] = (torch.randn(r_t, generator=g) * 4).to(torch.bfloat16).float()
    x = torch.zeros(D)
    for j in range(r_t):
        x[perm[j]] += sign[j] * cb[j]
    free = [c for c in range(D) if c not in set(perm[:r_t].tolist())]
    chans = sorted(torch.tensor(free)[torch.randperm(len(free), generator=g)[:n_planted]].tolist())
    k = 7
    codes = torch.randint(1, qmax + 1, (n_planted,), generator=g) * (torch.randint(0, 2, (n_planted,), generator=g) * 2 - 1)
    codes[int(torch.randint(0, n_planted, (1,), generator=g))] = qmax * (1 if bool(torch.rand(1, generator=g) < 0.5) else -1)
    # distinct magnitudes so the top-s choice is unique
    mags = torch.randperm(qmax, generator=g)[:n_planted] + 1
    mags[0] = qmax
    codes = mags * torch.sign(codes)
    for c, v in zip(chans, codes.tolist()):
        x[c] = v * 2.0 ** -k
    xb = x.to(torch.bfloat16)
    assert torch.equal(xb.float(), x)
    return B, xb, cb, chans, codes, k


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("r_t,s", [(8, 4), (32, 6), (0, 5), (64, 7)])
def test_exact_recovery_of_planted_residual(bits, r_t, s):
    r_max = 64
    n_planted = s if bits == 8 else min(s, 7)
    s = n_planted
    B, x, cb, chans, codes, k = _planted(100 * r_t + s + bits, r_max, r_t, s, bits, n_planted)
    out = oracle.encode_vector(B, x, r_t, s, bits)
    got_c = torch.from_numpy(out["coeff"].view(np.int16).copy()).view(torch.bfloat16).float()
    assert torch.equal(got_c[:r_t], cb[:r_t])
    assert not got_c[r_t:].any()
    qmax = 127 if bits == 8 else 7
    order = sorted(range(len(chans)), key=lambda i: chans[i])
    assert out["idx"].tolist() == [chans[i] for i in order]
    assert out["codes"].tolist() == [int(codes[i]) for i in order]
    # scale = fp16_rn(qmax * 2^-k / qmax) = 2^-k exactly
    assert oracle.fp16_to_f64(np.array([out["scale"]], np.uint16))[0] == 2.0 ** -k


def test_planted_with_zero_ties_fills_lowest_free_channels():
    """s larger than the planted set: the remaining picks are zero-residual channels, and
    ties at zero go to the lowest channel numbers."""
    r_max, r_t, bits = 32, 16, 8
    B, x, cb, chans, codes, k = _planted(7, r_max, r_t, 3, bits, 3)
    s = 6
    out = oracle.encode_vector(B, x, r_t, s, bits)
    zero_ch = [c for c in range(D) if c not in chans][:s - 3]
    assert out["idx"].tolist() == sorted(chans + zero_ch)
    codes_by_ch = dict(zip(out["idx"].tolist(), out["codes"].tolist()))
    for c in zero_ch:
        assert codes_by_ch[c] == 0


def test_zero_vector():
    wl = synth.workload("llama8b_encode_16k")
    bk, _ = synth.make_bases(wl.scaled(num_layers=2))
    x = torch.zeros(D, dtype=torch.bfloat16)
    out = oracle.encode_vector(bk[0, 0], x, 32, 16, 4)
    assert not out["coeff"].any() and out["scale"] == 0 and not out["codes"].any()
    assert out["idx"].tolist() == list(range(16))


@pytest.fixture(scope="module")
def encoded_batch():
    wl = synth.workload("llama8b_encode_16k").scaled(num_layers=2, batch=1)
    bases = synth.make_bases(wl)
    n = 256
    k, v = synth.make_dense_vectors(wl, 0, 0, n, bases)
    tiers = synth.make_tiers(wl, 0, 0, n)
    ranks = synth.ranks_of(wl, tiers)[:, 0]
    B = bases[0][0, 0]
    outs = [oracle.encode_vector(B, k[t, 0], int(ranks[t]), wl.resid_channels, wl.resid_bits) for t in range(n)]
    return wl, B, k[:, 0], ranks, outs


def test_projection_within_fp32_bound_of_fp64(encoded_batch):
    wl, B, X, ranks, outs = encoded_batch
    Bd = bf16_np(B)
    for t, o in enumerate(outs):
        x = bf16_np(X[t])
        r = int(ranks[t])
        c64 = Bd[:, :r].T @ x
        assert np.max(np.abs(o["c32"][:r] - c64)) <= 1e-5 * np.linalg.norm(x)


def test_stored_coefficients_are_bf16_rounding_of_projection(encoded_batch):
    wl, B, X, ranks, outs = encoded_batch
    for t, o in enumerate(outs):
        r = int(ranks[t])
        ref = torch.from_numpy(o["c32"][:r].copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(o["coeff"][:r], ref)
        assert not o["coeff"][r:].any()


def test_residual_is_taken_against_stored_coefficients(encoded_batch):
    wl, B, X, ranks, outs = encoded_batch
    Bd = bf16_np(B)
    for t, o in enumerate(outs):
        x = bf16_np(X[t])
        r = int(ranks[t])
        cb = torch.from_numpy(o["coeff"].view(np.int16).copy()).view(torch.bfloat16).double().numpy()
        r64 = x - Bd[:, :r] @ cb[:r]
        bound = 2.0 ** -22 * (np.abs(x) + np.abs(Bd[:, :r]) @ np.abs(cb[:r]))
        assert np.all(np.abs(o["resid"] - r64) <= bound)


def test_selection_is_top_s_with_low_channel_ties(encoded_batch):
    wl, B, X, ranks, outs = encoded_batch
    s = wl.resid_channels
    for o in outs:
        mag = np.abs(o["resid"].astype(np.float32))
        sel = o["idx"].astype(int)
        assert list(sel) == sorted(set(sel)) and len(sel) == s
        rest = np.setdiff1d(np.arange(D), sel)
        assert mag[sel].min() >= mag[rest].max()
        edge = mag[sel].min()
        tied_out = rest[mag[rest] == edge]
        tied_in = sel[mag[sel] == edge]
        if tied_out.size:
            assert tied_in.max() < tied_out.min()


def test_quantiser_round_trip_bound(encoded_batch):
    wl, B, X, ranks, outs = encoded_batch
    qmax = 7
    for o in outs:
        sel = o["idx"].astype(int)
        r = o["resid"][sel].astype(np.float64)
        sc = oracle.fp16_to_f64(np.array([o["scale"]], np.uint16))[0]
        amax = np.float32(np.abs(o["resid"][sel]).max())
        ref = (amax / np.float32(qmax)).astype(np.float16).view(np.uint16)
        assert int(ref) == int(o["scale"])
        codes = o["codes"].astype(np.float64)
        assert np.all(np.abs(codes) <= qmax)
        free = np.abs(codes) < qmax
        assert np.all(np.abs(r[free] - codes[free] * sc) <= 0.5 * sc * (1 + 1e-6))
        # clamped codes sit on the side of the residual
        assert np.all(np.sign(codes[~free]) == np.sign(r[~free]))


def test_encode_many_matches_single_calls(encoded_batch):
    wl, B, X, ranks, outs = encoded_batch
    many = oracle.encode_many(B, X, ranks, wl.resid_channels, wl.resid_bits, nthreads=3)
    for t, o in enumerate(outs):
        assert np.array_equal(many["coeff"][t], o["coeff"])
        assert np.array_equal(many["idx"][t], o["idx"])
        assert np.array_equal(many["codes"][t], o["codes"])
        assert many["scale"][t] == o["scale"]
