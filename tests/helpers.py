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


# One (layer, kv-head) decode problem of the oracle, sliced from token-ordered arrays.
head_problem = oracle.head_problem


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


# ----------------------------------------------------------------------------- GPU cache
def cfg_for(wl, max_batch=None, max_context=None, softmax_scale=0.0):
    import decode_attention_depthweave_b200 as dw
    return dw.config_from(
        num_layers=wl.num_layers, layers_per_group=wl.layers_per_group, num_q_heads=wl.num_q_heads,
        num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, r_max=wl.r_max, tiers=wl.tiers,
        resid_channels=wl.resid_channels, resid_bits=wl.resid_bits,
        max_batch=max_batch or wl.batch, max_context=max_context or wl.context, softmax_scale=softmax_scale,
        tier_resid=wl.tier_resid or None, coeff_bits=wl.coeff_bits)


def to_dev(d: dict, device="cuda") -> dict:
    return {k: v.to(device).contiguous() for k, v in d.items()}


def import_workload(cache, wl, lengths, gen_device="cpu", garbage=False, seed=None, layers=None):
    """Import synthetic compressed tokens of every (sequence, layer) into ``cache``.
    Returns {(seq, layer): (tier_idx, comp)} on the generation device."""
    data = {}
    layers = range(wl.num_layers) if layers is None else layers
    for seq, T in enumerate(lengths):
        tiers_by_group = {}
        for layer in layers:
            g = layer // wl.layers_per_group
            if g not in tiers_by_group:
                tiers_by_group[g] = synth.make_tiers(wl, seq, g, T, device=gen_device, seed=seed)
            tiers = tiers_by_group[g]
            comp = synth.make_compressed(wl, seq, layer, tiers, device=gen_device, seed=seed, garbage_tail=garbage)
            c = to_dev(comp)
            coeff = (c["ccodes"], c["cscales"]) if "ccodes" in c else c["coeff"]
            cache.append_compressed(layer, [seq], [T], tiers.to("cuda").contiguous(), coeff, c["idx"],
                                    c["codes"], c["scales"])
            data[(seq, layer)] = (tiers, comp)
    return data


def check_close(got, ref, max_abs=2e-3, rel=1e-3, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    ma = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rl = rel_l2(got, ref) if np.linalg.norm(ref) > 0 else float(np.linalg.norm(got))
    assert ma <= max_abs and rl <= rel, f"{what}: max_abs {ma:.3e} rel_l2 {rl:.3e}"
    return ma, rl


def oracle_encode_rows(wl, bases, layer, k, v, tier_idx, nthreads=None, c32=None, gate=None) -> dict:
    """The oracle's encoding of dense rows k, v (bf16 [n][Hkv][d]) at their tiers, in the
    token-ordered compressed format of ``synth.make_compressed`` (CPU tensors).  With ``c32``
    (fp32 [n][Hkv][2][r_max], an encoder's exported projection) the oracle runs encode steps
    2-6 on those coefficients instead of its own step 1."""
    g = layer // wl.layers_per_group
    k, v, tier_idx = k.cpu(), v.cpu(), tier_idx.cpu()
    n, H, s = k.shape[0], wl.num_kv_heads, wl.resid_channels
    ranks = synth.ranks_of(wl, tier_idx)
    nres = synth.resid_counts_of(wl, tier_idx) if wl.tier_resid else None
    c8 = wl.coeff_bits == 8
    coeff = np.zeros((n, H, 2, wl.r_max), np.uint16)
    ccodes = np.zeros((n, H, 2, wl.r_max), np.int8)
    cscales = np.zeros((n, H, 2, wl.r_max // 16), np.uint16)
    idx = np.zeros((n, H, 2, s), np.uint8)
    codes = np.zeros((n, H, 2, s), np.int8)
    scales = np.zeros((n, H, 2), np.uint16)
    if c32 is not None:
        c32 = np.nan_to_num(np.asarray(c32.cpu() if hasattr(c32, "cpu") else c32, np.float32))
    for h in range(H):
        for z, x in enumerate((k, v)):
            nr = None if nres is None else nres[:, h]
            if c8:
                r = oracle.encode_many8(bases[z][g, h], x[:, h], ranks[:, h], s, wl.resid_bits,
                                        c32=None if c32 is None else c32[:, h, z], nthreads=nthreads, nres=nr)
                ccodes[:, h, z], cscales[:, h, z] = r["ccodes"], r["cscales"]
            elif c32 is not None:
                r = oracle.encode_many_from_coeffs(bases[z][g, h], x[:, h], c32[:, h, z], ranks[:, h], s, wl.resid_bits,
                                                   nthreads=nthreads, nres=nr)
            else:
                r = oracle.encode_many(bases[z][g, h], x[:, h], ranks[:, h], s, wl.resid_bits, nthreads=nthreads,
                                       nres=nr)
            if not c8:
                coeff[:, h, z] = r["coeff"]
            idx[:, h, z], codes[:, h, z], scales[:, h, z] = r["idx"], r["codes"], r["scale"]
            if gate is not None:                    # the residual gate folded into the scale
                scales[:, h, z] = oracle.gate_scales(scales[:, h, z], np.asarray(gate.cpu())[:, h, z])
    out = {"idx": torch.from_numpy(idx), "codes": torch.from_numpy(codes),
           "scales": torch.from_numpy(scales.view(np.int16)).view(torch.float16)}
    if c8:
        out["ccodes"] = torch.from_numpy(ccodes)
        out["cscales"] = torch.from_numpy(cscales.view(np.int16)).view(torch.float16)
    else:
        out["coeff"] = torch.from_numpy(coeff.view(np.int16)).view(torch.bfloat16)
    return out


def cat_comp(a: dict, b: dict) -> dict:
    return {key: torch.cat([a[key].cpu(), b[key].cpu()]) for key in a}
