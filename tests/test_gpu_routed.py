"""Residual-count routing (the reading of "DepthWeave-KV ...", §3 Eq. (2) in which the router's
level rho is the number of residual channels a token keeps, rho in {0, 2, 4, 8}, at one basis
rank), through the C ABI against the oracle: import / export keep the first rho entries of a
token and read zeros past them; decode and the probe over ragged residual lengths; encode bit
for bit on both projection paths; fused append + decode; and the full 64K context at every
head.  Re-tiering between residual counts is in test_gpu_retier.py."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cat_comp, cfg_for, check_close, head_problem, import_workload, oracle_encode_rows
from test_gpu_encode import _assert_same, _encode_case

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")

ROUTED = "llama8b_routed_64k"


def _small(**kw):
    wl = synth.workload(ROUTED).scaled(num_layers=4, num_q_heads=8, num_kv_heads=2, batch=2)
    return wl.scaled(**kw) if kw else wl


def _clean(wl, tiers, comp):
    """What the cache stores of imported arrays: +0 past the rank, zeros past the count."""
    n = tiers.shape[0]
    c = {k: v.clone().cpu() for k, v in comp.items()}
    keep = torch.arange(wl.r_max).view(1, 1, 1, -1) < synth.ranks_of(wl, tiers.cpu()).view(n, -1, 1, 1)
    c["coeff"] = torch.where(keep, c["coeff"], torch.zeros_like(c["coeff"]))
    nres = synth.resid_counts_of(wl, tiers.cpu())
    on = torch.arange(wl.resid_channels).view(1, 1, 1, -1) < nres.view(n, -1, 1, 1)
    c["idx"], c["codes"] = c["idx"] * on, c["codes"] * on
    c["scales"] = c["scales"] * (nres.view(n, -1, 1) > 0)
    return c


@pytest.mark.parametrize("bits", [4, 8])
def test_import_export_keeps_the_first_rho_entries(bits):
    wl = _small(resid_bits=bits)
    lengths = [700, 129]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=800), bases[0], bases[1])
    data = import_workload(cache, wl, lengths, garbage=True)
    for (b, layer), (tiers, comp) in data.items():
        got = cache.export(layer, b, 0, lengths[b])
        want = _clean(wl, tiers, comp)
        assert torch.equal(got["tier_idx"].cpu(), tiers.cpu())
        for key in ("coeff", "idx", "codes", "scales"):
            assert torch.equal(got[key].cpu().contiguous().view(torch.uint8), want[key].contiguous().view(torch.uint8)), \
                (b, layer, key)


@pytest.mark.parametrize("bits,temp", [(4, 1.0), (4, 8.0), (8, 8.0), (8, 32.0)])
def test_decode_and_probe_over_ragged_residual_lengths(bits, temp):
    """Garbage past each token's count must be ignored; every layer, head and sequence."""
    wl = _small(resid_bits=bits)
    lengths = [3000, 777]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=3100), bases[0], bases[1])
    data = import_workload(cache, wl, lengths, garbage=True)
    for layer in range(wl.num_layers):
        q = synth.make_queries(wl, layer, batch=2, temperature=temp)
        out = cache.decode(layer, [0, 1], q.cuda())
        err, out_full = cache.probe(layer, [0, 1], q.cuda(), want_out=True)
        cache.sync()
        out, err, out_full = out.cpu().numpy(), err.cpu().numpy(), out_full.cpu().numpy()
        for b in range(2):
            tiers, comp = data[(b, layer)]
            for h in range(wl.num_kv_heads):
                prob = head_problem(wl, bases, tiers, comp, q[b], layer, h)
                check_close(out[b, h * 4:(h + 1) * 4], oracle.decode_head(prob), what=f"layer {layer} seq {b} head {h}")
                e_ref, of, _ = oracle.probe_head(prob)
                assert abs(err[b, h] - e_ref) <= 2e-3, (layer, b, h, err[b, h], e_ref)
                check_close(out_full[b, h * 4:(h + 1) * 4], of, what="probe out_full")


def test_single_count_tiers_and_all_zero_counts():
    """A page of rho = 0 tokens has no residual at all: with every token at rho = 0 the probe
    error is 0 and decode is the coefficient-space attention."""
    wl = _small(tier_probs=(1.0, 0.0, 0.0, 0.0), num_layers=2)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=600), bases[0], bases[1])
    data = import_workload(cache, wl, [500, 64], garbage=True)
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0)
    err = cache.probe(1, [0, 1], q.cuda())
    out = cache.decode(1, [0, 1], q.cuda())
    cache.sync()
    assert float(err.abs().max()) == 0.0
    for b in range(2):
        tiers, comp = data[(b, 1)]
        for h in range(wl.num_kv_heads):
            ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], 1, h), with_residual=False)
            check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"rho=0 seq {b} head {h}")


@pytest.mark.parametrize("bits", [4, 8])
def test_encode_bit_exact_on_both_paths(bits):
    """Chunks of 1 and 4 tokens take the fp32-chain path, the others the tensor-core path;
    each token keeps the rho largest residual channels of its tier."""
    wl = _small(resid_bits=bits, num_layers=2)
    lengths = [260, 131]
    chunks = (1, 4, 37, 64, None)
    cache, bases, dense, c32 = _encode_case(wl, lengths, chunks=chunks)
    for b, T in enumerate(lengths):
        for layer in range(wl.num_layers):
            got = cache.export(layer, b, 0, T)
            tiers = dense[(b, "t", layer // wl.layers_per_group)]
            k, v = dense[(b, layer)]
            ref = oracle_encode_rows(wl, bases, layer, k, v, tiers, c32=c32[(b, layer)])
            _assert_same(got, ref, tiers, f"seq {b} layer {layer}")


def test_fused_append_decode_steps():
    wl = _small()
    lengths = [1500, 300]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1600), bases[0], bases[1])
    data = import_workload(cache, wl, lengths)
    state = dict(data)
    for step in range(4):
        for layer in range(wl.num_layers):
            g = layer // wl.layers_per_group
            ks, vs, ts = [], [], []
            for b, T in enumerate(lengths):
                k, v = synth.make_dense_vectors(wl, b, layer, 1, bases, start=T + step)
                ks.append(k)
                vs.append(v)
                ts.append(synth.make_tiers(wl, b, g, 1, start=T + step))
            k, v, t = torch.cat(ks), torch.cat(vs), torch.cat(ts)
            q = synth.make_queries(wl, layer, batch=2, temperature=8.0, step=step)
            first = layer % wl.layers_per_group == 0
            out = cache.append_decode(layer, [0, 1], k.cuda(), v.cuda(), t.cuda() if first else None, q.cuda())
            cache.sync()
            for b in range(2):
                tiers, comp = state[(b, layer)]
                enc = oracle_encode_rows(wl, bases, layer, k[b:b + 1], v[b:b + 1], t[b:b + 1])
                state[(b, layer)] = (torch.cat([tiers.cpu(), t[b:b + 1]]), cat_comp(comp, enc))
                for h in range(wl.num_kv_heads):
                    ref = oracle.decode_head(head_problem(wl, bases, *state[(b, layer)], q[b], layer, h))
                    check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref,
                                what=f"step {step} layer {layer} seq {b} head {h}")
    for b, T in enumerate(lengths):
        got = cache.export(1, b, T, 4)
        tiers, comp = state[(b, 1)]
        want = {k_: v_[T:T + 4] for k_, v_ in comp.items()}
        _assert_same(got, want, tiers[T:T + 4], f"appended seq {b}")


@pytest.mark.slow
def test_routed_64k_full_context_every_head():
    """Full 64K context, 8 kv heads, batch 1, one group of two layers: 65535 imported tokens
    plus one fused append + decode step; every head against the oracle."""
    wl = synth.workload(ROUTED).scaled(num_layers=2)
    T = wl.context
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=T + 64), bases[0], bases[1])
    data = import_workload(cache, wl, [T - 1], gen_device="cuda", garbage=True)
    tn = synth.make_tiers(wl, 0, 0, 1, device="cuda", start=T - 1)
    kv = {l: synth.make_dense_vectors(wl, 0, l, 1, bases, device="cuda", start=T - 1) for l in range(2)}
    q = synth.make_queries(wl, 1, batch=1, device="cuda", temperature=8.0)
    cache.append(0, [0], [1], kv[0][0], kv[0][1], tn)
    out = cache.append_decode(1, [0], kv[1][0], kv[1][1], None, q)
    cache.sync()
    out = out.cpu().numpy()
    tiers, comp = data[(0, 1)]
    new = oracle_encode_rows(wl, bases, 1, kv[1][0], kv[1][1], tn)
    tt = torch.cat([tiers.cpu(), tn.cpu()])
    full = cat_comp({k: v.cpu() for k, v in comp.items()}, new)
    refs = oracle.decode_many([head_problem(wl, bases, tt, full, q[0].cpu(), 1, h) for h in range(wl.num_kv_heads)],
                              nthreads=os.cpu_count())
    for h, ref in enumerate(refs):
        check_close(out[0, h * 4:(h + 1) * 4], ref, what=f"routed 64K head {h}")
