"""Shared test helpers: slicing synthetic inputs into oracle problems, and independent
numpy restatements used as pins (library matmul / softmax on dense tensors)."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import synth


def bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 values of a bf16 / fp16 tensor."""
    return t.detach().cpu().to(torch.float64).numpy()


def head_problem(wl, bases, tier_idx, comp, q, layer, head) -> oracle.HeadProblem:
    """Oracle problem for one (layer, kv-head) from token-ordered synthetic arrays.

    ``tier_idx`` uint8 [T][Hkv]; ``comp`` the dict of ``synth.make_compressed``; ``q`` bf16
    [Hq][d] (all query heads of the sequence)."""
    g = layer // wl.layers_per_group
    gq = wl.gqa
    ranks = synth.ranks_of(wl, tier_idx.cpu())[:, head]
    c = {k: v.cpu() for k, v in comp.items()}
    return oracle.HeadProblem(
        bases[0][g, head], bases[1][g, head], ranks,
        c["coeff"][:, head, 0], c["idx"][:, head, 0], c["codes"][:, head, 0], c["scales"][:, head, 0],
        c["coeff"][:, head, 1], c["idx"][:, head, 1], c["codes"][:, head, 1], c["scales"][:, head, 1],
        q.cpu()[head * gq:(head + 1) * gq])


def np_reconstruct(basis, ranks, coeff, idx, codes, scales, with_residual=True) -> np.ndarray:
    """Dense [T][d] fp64 reconstruction with numpy primitives (matmul + scatter-add).

    basis [d][r_max], coeff [T][r_max] (bf16 tensors), idx/codes [T][s], scales [T] fp16."""
    B = bf16_np(basis)
    c = bf16_np(coeff).copy()
    T, r_max = c.shape
    rk = np.asarray(ranks).reshape(T)
    mask = np.arange(r_max)[None, :] < rk[:, None]
    c = np.where(mask, c, 0.0)
    X = c @ B.T
    if with_residual and idx.shape[-1] > 0:
        ix = idx.cpu().numpy().astype(np.int64)
        val = codes.cpu().numpy().astype(np.float64) * bf16_np(scales)[:, None]
        rows = np.repeat(np.arange(T), ix.shape[1])
        np.add.at(X, (rows, ix.reshape(-1)), val.reshape(-1))
    return X


def np_attention(q, K, V, tau) -> tuple:
    """Dense softmax attention in fp64: q [gq][d], K/V [T][d] -> (o [gq][d], p [gq][T])."""
    s = tau * (q @ K.T)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ V, p


def signed_permutation(d: int, r: int, seed: int) -> torch.Tensor:
    """bf16 [d][r] with orthonormal columns in exact arithmetic: e_{perm(j)} * (+-1)."""
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(d, generator=g)[:r]
    sign = torch.randint(0, 2, (r,), generator=g) * 2 - 1
    B = torch.zeros(d, r, dtype=torch.float32)
    B[perm, torch.arange(r)] = sign.float()
    return B.to(torch.bfloat16), perm, sign


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def tau_of(d: int) -> float:
    return 1.0 / math.sqrt(d)
