"""Seeded synthetic inputs for the compressed-cache decode path.

This module only *draws* inputs: bases, per-token rank tiers, stored coefficients,
residual channel indices / integer codes / fp16 scales, queries and the dense
key/value vectors that the encoder compresses.  It holds none of the method's
arithmetic (no reconstruction, no attention, no projection of data onto a basis,
no quantiser).  Tests, ``bench.py`` and the CPU oracle's checks all take their
inputs from here, so the GPU path and the oracle see the same bytes.

Workload shapes follow the 64K-context decode setting of
"DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization for Long-Context
KV Cache Compression" (§4 Experiments, setup paragraph), at Llama-3-8B head
geometry.  Distribution notation ``N(0, x)`` below means *variance* x.

Every draw comes from a ``torch.Generator`` seeded from (base seed, purpose,
indices) so one layer / sequence / group can be regenerated alone.  Draws made
on a CUDA device differ from draws made on the CPU for the same seed; a caller
that needs both sides to see the same values generates once and copies.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field, replace

import torch

__all__ = [
    "Workload", "WORKLOADS", "workload", "seed_for", "make_bases", "make_context_lengths",
    "make_tiers", "make_compressed", "make_queries", "make_dense_vectors",
    "ranks_of", "qmax_of", "make_residual_cases",
]


@dataclass(frozen=True)
class Workload:
    """Shapes and input distributions of one synthetic workload."""
    name: str
    num_layers: int
    layers_per_group: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    r_max: int
    tiers: tuple
    tier_probs: tuple
    resid_channels: int
    resid_bits: int
    batch: int
    context: int                      # fixed context, or the upper bound when ragged
    context_min: int = 0              # >0: per-sequence context ~ U[context_min, context]
    span_tier: int = -1               # >=0: tier index forced on seeded spans
    num_spans: int = 0
    span_len: int = 0
    new_tokens: int = 0               # encode workload: tokens compressed per sequence
    base_seed: int = 1000
    coeff_var_rank: int = 0           # encode workload: c_j ~ N(0, 1/j) for j <= this
    outlier_frac: float = 0.0
    outlier_var: float = 0.0
    noise_var: float = 0.0
    resid_var: float = 0.05           # scale drawn from max |N(0, resid_var)| / qmax
    tier_resid: tuple = ()            # per-tier residual counts (every tier at one rank), or ()
    coeff_bits: int = 16              # 16: bf16 coefficients; 8: int8 codes + fp16 scale per block of 16
    extra: dict = field(default_factory=dict)

    @property
    def num_groups(self) -> int:
        return self.num_layers // self.layers_per_group

    @property
    def gqa(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The workloads.  Names say what they are; sizes are the full ones.
WORKLOADS = {
    "tiny_1k": Workload(
        name="tiny_1k", num_layers=2, layers_per_group=2, num_q_heads=4, num_kv_heads=1,
        head_dim=128, r_max=32, tiers=(8, 16, 32), tier_probs=(0.7, 0.2, 0.1),
        resid_channels=8, resid_bits=8, batch=1, context=1024, base_seed=1001),
    "llama8b_64k": Workload(
        name="llama8b_64k", num_layers=32, layers_per_group=2, num_q_heads=32, num_kv_heads=8,
        head_dim=128, r_max=64, tiers=(16, 32, 64), tier_probs=(0.6, 0.3, 0.1),
        resid_channels=16, resid_bits=4, batch=1, context=65536, base_seed=1002,
        coeff_var_rank=64, noise_var=0.01),
    "llama8b_64k_c8": Workload(
        name="llama8b_64k_c8", num_layers=32, layers_per_group=2, num_q_heads=32, num_kv_heads=8,
        head_dim=128, r_max=64, tiers=(16, 32, 64), tier_probs=(0.6, 0.3, 0.1),
        resid_channels=16, resid_bits=4, batch=1, context=65536, base_seed=1007,
        coeff_var_rank=64, noise_var=0.01, coeff_bits=8),
    "llama8b_ragged_b8": Workload(
        name="llama8b_ragged_b8", num_layers=32, layers_per_group=2, num_q_heads=32,
        num_kv_heads=8, head_dim=128, r_max=64, tiers=(16, 32, 64),
        tier_probs=(0.5, 0.35, 0.15), resid_channels=16, resid_bits=8, batch=8,
        context=32768, context_min=16384, base_seed=1003, coeff_var_rank=64, noise_var=0.01),
    "llama8b_131k_deep": Workload(
        name="llama8b_131k_deep", num_layers=32, layers_per_group=4, num_q_heads=32,
        num_kv_heads=8, head_dim=128, r_max=128, tiers=(8, 16, 32, 64, 128),
        tier_probs=(0.4, 0.3, 0.15, 0.1, 0.05), resid_channels=8, resid_bits=4, batch=1,
        context=131072, span_tier=4, num_spans=3, span_len=256, base_seed=1004,
        coeff_var_rank=128, noise_var=0.01),
    "llama8b_routed_64k": Workload(
        name="llama8b_routed_64k", num_layers=32, layers_per_group=2, num_q_heads=32, num_kv_heads=8,
        head_dim=128, r_max=32, tiers=(32, 32, 32, 32), tier_probs=(0.4, 0.3, 0.2, 0.1),
        resid_channels=8, resid_bits=4, batch=1, context=65536, base_seed=1006,
        coeff_var_rank=32, noise_var=0.01, tier_resid=(0, 2, 4, 8)),
    "llama8b_encode_16k": Workload(
        name="llama8b_encode_16k", num_layers=32, layers_per_group=2, num_q_heads=32,
        num_kv_heads=8, head_dim=128, r_max=64, tiers=(16, 32, 64), tier_probs=(0.6, 0.3, 0.1),
        resid_channels=16, resid_bits=4, batch=4, context=16384, new_tokens=16384,
        base_seed=1005, coeff_var_rank=64, outlier_frac=0.02, outlier_var=0.3, noise_var=0.01),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def qmax_of(bits: int) -> int:
    """Largest code magnitude of the symmetric residual codec (int8: 127, int4: 7)."""
    return 127 if bits == 8 else 7


def seed_for(base: int, tag: str, *idx: int) -> int:
    """Deterministic 63-bit seed from a base seed, a purpose tag and indices."""
    h = zlib.crc32(tag.encode()) & 0xFFFFFFFF
    v = (base * 0x9E3779B1 + h) & 0x7FFFFFFFFFFFFFFF
    for i in idx:
        v = (v * 1_000_003 + (int(i) & 0xFFFFFFFF) + 0x5BD1E995) & 0x7FFFFFFFFFFFFFFF
    return v


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_bases(wl: Workload, seed: int | None = None):
    """Per (group, kv-head) bases for K and for V, bf16 ``[G][Hkv][d][r_max]``.

    Columns are orthonormal in fp64 (QR of a seeded N(0, 1) d x r_max matrix),
    then rounded to bf16.  Drawn on the CPU so every device sees the same bases.
    """
    seed = wl.base_seed if seed is None else seed
    out = []
    for z, tag in enumerate(("basis_k", "basis_v")):
        mats = torch.empty(wl.num_groups, wl.num_kv_heads, wl.head_dim, wl.r_max, dtype=torch.float64)
        for g in range(wl.num_groups):
            for h in range(wl.num_kv_heads):
                a = torch.randn(wl.head_dim, wl.r_max, dtype=torch.float64,
                                generator=_gen("cpu", seed_for(seed, tag, g, h)))
                qm, _ = torch.linalg.qr(a)
                mats[g, h] = qm
        out.append(mats.to(torch.bfloat16))
    return out[0], out[1]


def make_context_lengths(wl: Workload, seed: int | None = None) -> list:
    """Per-sequence context lengths: fixed, or ~ U[context_min, context] (integers)."""
    seed = wl.base_seed if seed is None else seed
    if wl.context_min <= 0:
        return [wl.context] * wl.batch
    g = _gen("cpu", seed_for(seed, "ctx"))
    return torch.randint(wl.context_min, wl.context + 1, (wl.batch,), generator=g).tolist()


def make_tiers(wl: Workload, seq: int, group: int, n: int, device="cpu",
               seed: int | None = None, start: int = 0) -> torch.Tensor:
    """Tier indices (into ``wl.tiers``) for positions [start, start+n), uint8 ``[n][Hkv]``.

    i.i.d. categorical with ``wl.tier_probs`` per (sequence, group, kv-head, token).
    With ``span_tier >= 0`` the tokens of ``num_spans`` seeded, non-overlapping spans of
    ``span_len`` positions (the same positions for every group and head of a sequence) take
    tier ``span_tier``, and the others draw from the remaining tiers with renormalised
    probabilities.
    """
    seed = wl.base_seed if seed is None else seed
    g = _gen(device, seed_for(seed, "tiers", seq, group, start))
    probs = torch.tensor(wl.tier_probs, dtype=torch.float64)
    if wl.span_tier >= 0:
        probs[wl.span_tier] = 0.0
    probs = probs / probs.sum()
    cum = torch.cumsum(probs, 0).to(device=device, dtype=torch.float64)
    u = torch.rand(n, wl.num_kv_heads, generator=g, device=device, dtype=torch.float64)
    t = torch.searchsorted(cum, u.reshape(-1), right=True).clamp_(max=len(wl.tiers) - 1)
    t = t.reshape(n, wl.num_kv_heads).to(torch.uint8)
    if wl.span_tier >= 0 and wl.num_spans > 0:
        total = max(wl.context, start + n)
        for a, b in _spans(wl, seq, seed, total):
            lo, hi = max(a, start), min(b, start + n)
            if lo < hi:
                t[lo - start:hi - start, :] = wl.span_tier
    return t


def _spans(wl: Workload, seq: int, seed: int, total: int):
    """Seeded, non-overlapping [a, b) spans of ``span_len`` positions in [0, total)."""
    g = _gen("cpu", seed_for(seed, "spans", seq))
    slots = total // wl.span_len
    pick = torch.randperm(slots, generator=g)[: wl.num_spans].sort().values.tolist()
    return [(p * wl.span_len, (p + 1) * wl.span_len) for p in pick]


def ranks_of(wl: Workload, tier_idx: torch.Tensor) -> torch.Tensor:
    """Rank r_t of each token (a table lookup, ``int32``)."""
    return torch.tensor(wl.tiers, dtype=torch.int32, device=tier_idx.device)[tier_idx.long()]


def resid_counts_of(wl: Workload, tier_idx: torch.Tensor) -> torch.Tensor:
    """Residual channels each token keeps (a table lookup, ``int32``): ``wl.tier_resid`` of its
    tier, or ``wl.resid_channels`` for every token without per-tier counts."""
    if not wl.tier_resid:
        return torch.full(tier_idx.shape, wl.resid_channels, dtype=torch.int32, device=tier_idx.device)
    return torch.tensor(wl.tier_resid, dtype=torch.int32, device=tier_idx.device)[tier_idx.long()]


def make_compressed(wl: Workload, seq: int, layer: int, tier_idx: torch.Tensor,
                    device="cpu", seed: int | None = None, garbage_tail: bool = False,
                    start: int = 0) -> dict:
    """Stored compressed form of ``n = len(tier_idx)`` tokens of one (sequence, layer).

    Token-ordered arrays, K at ``[..., 0, ...]`` and V at ``[..., 1, ...]``:

    * ``coeff``  bf16 ``[n][Hkv][2][r_max]``: c_j ~ N(0, 1/j) for rank index j = 1..r_t;
      entries at j > r_t are zero, or N(0, 1) garbage with ``garbage_tail`` (they must be ignored).
    * ``idx``    uint8 ``[n][Hkv][2][s]``: s distinct channels, uniform without replacement,
      ascending.
    * ``codes``  int8 ``[n][Hkv][2][s]``: a discretised Gaussian, round(N(0, (qmax/2.5)^2))
      clipped to [-qmax, qmax].
    * ``scales`` fp16 ``[n][Hkv][2]``: max_i |N(0, resid_var)| over s draws, divided by qmax.

    With per-tier residual counts (``wl.tier_resid``) a token of tier k keeps the first
    ``tier_resid[k]`` entries of idx / codes; the entries past them are zero (the scale too
    when the count is 0), or left as drawn with ``garbage_tail`` (they must be ignored).

    With 8-bit coefficients (``wl.coeff_bits == 8``) ``coeff`` is replaced by

    * ``ccodes``  int8 ``[n][Hkv][2][r_max]``: round(N(0, (127/2.5)^2)) clipped to [-127, 127];
    * ``cscales`` fp16 ``[n][Hkv][2][r_max / 16]``: for block b, max |N(0, 1/j)| over its 16
      rank indices j, divided by 127,

    zero past r_t (blocks past r_t / 16), or N(0, 1)-scaled garbage with ``garbage_tail``.
    """
    seed = wl.base_seed if seed is None else seed
    n = tier_idx.shape[0]
    H, d, R, s = wl.num_kv_heads, wl.head_dim, wl.r_max, wl.resid_channels
    qmax = qmax_of(wl.resid_bits)
    g = _gen(device, seed_for(seed, "cache", seq, layer, start))
    tier_idx = tier_idx.to(device)
    ranks = ranks_of(wl, tier_idx)                                 # [n][H]
    j = torch.arange(1, R + 1, device=device, dtype=torch.float32)
    coeff = torch.randn(n, H, 2, R, generator=g, device=device) * j.rsqrt()
    keep = (j.view(1, 1, 1, R) <= ranks.view(n, H, 1, 1).float())
    if garbage_tail:
        junk = torch.randn(n, H, 2, R, generator=g, device=device)
        coeff = torch.where(keep, coeff, junk)
    else:
        coeff = coeff * keep
    coeff = coeff.to(torch.bfloat16)
    c8 = None
    if wl.coeff_bits == 8:
        nb = R // 16
        codes8 = (torch.randn(n, H, 2, R, generator=g, device=device) * (127 / 2.5)).round().clamp_(-127, 127)
        amax = (torch.randn(n, H, 2, nb, 16, generator=g, device=device) * j.view(nb, 16).rsqrt()).abs().amax(-1)
        sc8 = amax / 127
        if garbage_tail:
            junk_c = torch.randint(-128, 128, (n, H, 2, R), generator=g, device=device).float()
            junk_s = torch.rand(n, H, 2, nb, generator=g, device=device) * 4
            codes8 = torch.where(keep, codes8, junk_c)
            sc8 = torch.where(keep[..., ::16], sc8, junk_s)
        else:
            codes8 = codes8 * keep
            sc8 = sc8 * keep[..., ::16]
        c8 = (codes8.to(torch.int8), sc8.to(torch.float16))
    if s > 0:
        keys = torch.rand(n, H, 2, d, generator=g, device=device)
        idx = keys.topk(s, dim=-1).indices.sort(dim=-1).values.to(torch.uint8)
        codes = torch.randn(n, H, 2, s, generator=g, device=device) * (qmax / 2.5)
        codes = codes.round().clamp_(-qmax, qmax).to(torch.int8)
        amax = (torch.randn(n, H, 2, s, generator=g, device=device) * math.sqrt(wl.resid_var)).abs().amax(-1)
        scales = (amax / qmax).to(torch.float16)
    else:
        idx = torch.zeros(n, H, 2, 0, dtype=torch.uint8, device=device)
        codes = torch.zeros(n, H, 2, 0, dtype=torch.int8, device=device)
        scales = torch.zeros(n, H, 2, dtype=torch.float16, device=device)
    if wl.tier_resid and not garbage_tail:
        nres = resid_counts_of(wl, tier_idx)                           # [n][H]
        on = torch.arange(s, device=device).view(1, 1, 1, s) < nres.view(n, H, 1, 1)
        idx = idx * on
        codes = codes * on
        scales = scales * (nres.view(n, H, 1) > 0)
    if c8 is not None:
        return {"ccodes": c8[0], "cscales": c8[1], "idx": idx, "codes": codes, "scales": scales}
    return {"coeff": coeff, "idx": idx, "codes": codes, "scales": scales}


def make_queries(wl: Workload, layer: int, batch: int | None = None, device="cpu",
                 seed: int | None = None, temperature: float = 1.0, step: int = 0) -> torch.Tensor:
    """Decode queries, bf16 ``[B][Hq][d]`` ~ N(0, 1/sqrt(d)) (variance), times ``temperature``."""
    seed = wl.base_seed if seed is None else seed
    batch = wl.batch if batch is None else batch
    g = _gen(device, seed_for(seed, "query", layer, step))
    std = (1.0 / math.sqrt(wl.head_dim)) ** 0.5
    q = torch.randn(batch, wl.num_q_heads, wl.head_dim, generator=g, device=device) * (std * temperature)
    return q.to(torch.bfloat16)


def make_dense_vectors(wl: Workload, seq: int, layer: int, n: int, bases, device="cpu",
                       seed: int | None = None, start: int = 0):
    """Dense keys and values to compress, bf16 ``[n][Hkv][d]`` each.

    x = B_{m,h}[:, :r] c + outliers + noise, with c_j ~ N(0, 1/j) (j = 1..r,
    r = ``coeff_var_rank``), sparse N(0, outlier_var) outliers on a seeded fixed set of
    ceil(outlier_frac * d) channels per (layer, kv-head, K/V) present on every token, and
    N(0, noise_var) noise on every channel; rounded to bf16.
    """
    seed = wl.base_seed if seed is None else seed
    H, d = wl.num_kv_heads, wl.head_dim
    r = wl.coeff_var_rank or wl.r_max
    grp = layer // wl.layers_per_group
    out = []
    for z in range(2):
        g = _gen(device, seed_for(seed, "dense", seq, layer, z, start))
        basis = bases[z][grp].to(device=device, dtype=torch.float32)[:, :, :r]     # [H][d][r]
        j = torch.arange(1, r + 1, device=device, dtype=torch.float32)
        c = torch.randn(n, H, r, generator=g, device=device) * j.rsqrt()
        x = torch.einsum("hdr,nhr->nhd", basis, c)
        if wl.noise_var > 0:
            x = x + torch.randn(n, H, d, generator=g, device=device) * math.sqrt(wl.noise_var)
        if wl.outlier_frac > 0:
            k = math.ceil(wl.outlier_frac * d)
            gc = _gen("cpu", seed_for(seed, "outlier_ch", layer, z))
            for h in range(H):
                ch = torch.randperm(d, generator=gc)[:k].to(device)
                x[:, h, ch] += torch.randn(n, k, generator=g, device=device) * math.sqrt(wl.outlier_var)
        out.append(x.to(torch.bfloat16).contiguous())
    return out[0], out[1]


def make_test_matrix(wl: Workload, seed: int | None = None, device="cpu") -> torch.Tensor:
    """The basis sketch's Gaussian test matrix, fp32 ``[d][r_max]`` ~ N(0, 1)."""
    seed = wl.base_seed if seed is None else seed
    g = _gen("cpu", seed_for(seed, "omega"))
    return torch.randn(wl.head_dim, wl.r_max, generator=g, dtype=torch.float32).to(device)


RESIDUAL_CASE_KINDS = ("gaussian", "boundary_ulp", "boundary_tie", "top_tie", "few_nonzero", "zeros",
                       "subnormal", "huge", "half_steps")


def make_residual_cases(n: int, d: int = 128, s: int = 16, seed: int = 77):
    """Residual vectors fp32 ``[n][d]`` (numpy) for the selection / quantiser steps alone, made
    to stress their boundaries; kind ``v % 9`` per vector (``RESIDUAL_CASE_KINDS``):
    gaussian N(0, 1); the (s+1)-th largest magnitude moved to one ulp above or below the s-th;
    a group of equal magnitudes (random signs) straddling rank s; equal magnitudes at the top;
    fewer than s nonzero entries (the rest +0 / -0); all +0 / -0; subnormal magnitudes;
    magnitudes so large that the fp16 scale overflows; values on exact half steps of a
    power-of-two scale (an int4 scale of exactly 2^e: round-half-even cases).  Inputs only:
    no selection happens here."""
    import numpy as np
    rng = np.random.default_rng(seed_for(seed, "resid_cases", n, d, s) & 0xFFFFFFFF)
    out = rng.standard_normal((n, d)).astype(np.float32)
    for v in range(n):
        kind = v % len(RESIDUAL_CASE_KINDS)
        r = out[v]
        if kind == 1 and s < d:
            order = np.argsort(-np.abs(r), kind="stable")
            a, b = order[s - 1], order[s]
            up = rng.integers(0, 2) == 1
            mag = np.nextafter(np.abs(r[a]), np.float32(np.inf) if up else np.float32(0))
            r[b] = np.float32(mag) * np.float32(1 if rng.integers(0, 2) else -1)
        elif kind == 2 and s < d:
            order = np.argsort(-np.abs(r), kind="stable")
            lo, hi = max(0, s - 3), min(d, s + 3)
            mag = np.abs(r[order[lo]])
            for c in order[lo:hi]:
                r[c] = mag * np.float32(1 if rng.integers(0, 2) else -1)
        elif kind == 3:
            ch = rng.choice(d, size=min(d, 5), replace=False)
            r[ch] = np.float32(4.0) * np.where(rng.integers(0, 2, size=ch.size) == 1, 1, -1).astype(np.float32)
        elif kind == 4:
            k = int(rng.integers(0, max(1, s)))
            keep = rng.choice(d, size=k, replace=False)
            z = np.where(rng.integers(0, 2, size=d) == 1, np.float32(0.0), np.float32(-0.0))
            z[keep] = r[keep]
            out[v] = z
        elif kind == 5:
            out[v] = np.where(rng.integers(0, 2, size=d) == 1, np.float32(0.0), np.float32(-0.0))
        elif kind == 6:
            out[v] = (r * np.float32(1e-39)).astype(np.float32)
        elif kind == 7:
            out[v] = (r * np.float32(1e6)).astype(np.float32)
        elif kind == 8:                 # int4: scale exactly 2^e, so r / scale lands on halves
            e = int(rng.integers(-6, 3))
            steps = rng.integers(-14, 15, size=d).astype(np.float32)
            steps[int(rng.integers(0, d))] = np.float32(14 if rng.integers(0, 2) else -14)
            out[v] = (steps * np.float32(0.5) * np.float32(2.0 ** e)).astype(np.float32)
    return out
