"""The residual gate of "DepthWeave-KV ...", §3 Method, Eq. (1) (X^ = A B + g R) folded into the
dequantisation (dwkv_append_gated: the stored residual scale is fp16_rn(g * scale)), through
the C ABI against the oracle: the stored bytes on both projection paths, g = 1 equal to the
plain append, g = 0 leaving no residual (probe error 0), and decode over a gated cache."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cfg_for, check_close, head_problem, oracle_encode_rows

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _wl(**kw):
    return synth.workload("llama8b_encode_16k").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=2, **kw)


def _append(wl, lengths, chunks, gates):
    """Append seeded dense rows of both layers in the given chunk sizes, gated; returns the
    cache, bases, rows, tiers and the exported projections."""
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_batch=len(lengths), max_context=max(lengths) + 8), bases[0], bases[1])
    rows, c32 = {}, {}
    for b, T in enumerate(lengths):
        rows[b] = [synth.make_dense_vectors(wl, b, layer, T, bases) for layer in range(2)]
        rows[(b, "t")] = synth.make_tiers(wl, b, 0, T)
    for layer in range(2):
        for b, T in enumerate(lengths):
            a, ci = 0, 0
            c32[(b, layer)] = torch.full((T, wl.num_kv_heads, 2, wl.r_max), float("nan"))
            while a < T:                            # the chunk sizes, repeated
                n = min(chunks[ci % len(chunks)], T - a)
                ci += 1
                k, v = rows[b][layer]
                dbg = torch.full((n, wl.num_kv_heads, 2, wl.r_max), float("nan"), device="cuda")
                gt = None if gates is None else gates[(b, layer)][a:a + n].cuda().contiguous()
                cache.append(layer, [b], [n], k[a:a + n].cuda(), v[a:a + n].cuda(),
                             rows[(b, "t")][a:a + n].cuda() if layer == 0 else None, coeff_dbg=dbg, gate=gt)
                c32[(b, layer)][a:a + n] = dbg.cpu()
                a += n
    cache.sync()
    return cache, bases, rows, c32


@pytest.mark.parametrize("chunks,coeff_bits", [((1, 3, 4), 16), ((37, 64, 1000), 16), ((1, 3, 4), 8), ((37, 64, 1000), 8)])
def test_gated_append_bytes_and_decode(chunks, coeff_bits):
    wl = _wl(coeff_bits=coeff_bits)
    lengths = [150, 77]
    g = torch.Generator().manual_seed(9)
    gates = {(b, layer): torch.rand(T, wl.num_kv_heads, 2, generator=g) for b, T in enumerate(lengths) for layer in range(2)}
    cache, bases, rows, c32 = _append(wl, lengths, chunks, gates)
    for b, T in enumerate(lengths):
        tiers = rows[(b, "t")]
        for layer in range(2):
            k, v = rows[b][layer]
            got = cache.export(layer, b, 0, T)
            ref = oracle_encode_rows(wl, bases, layer, k, v, tiers, c32=c32[(b, layer)], gate=gates[(b, layer)])
            for key in ref:
                assert torch.equal(got[key].cpu().contiguous().view(torch.uint8), ref[key].contiguous().view(torch.uint8)), \
                    (b, layer, key)
    for layer in range(2):
        q = synth.make_queries(wl, layer, batch=2, temperature=8.0)
        out = cache.decode(layer, [0, 1], q.cuda())
        cache.sync()
        for b in range(2):
            k, v = rows[b][layer]
            comp = oracle_encode_rows(wl, bases, layer, k, v, rows[(b, "t")], c32=c32[(b, layer)], gate=gates[(b, layer)])
            for h in range(wl.num_kv_heads):
                ref = oracle.decode_head(head_problem(wl, bases, rows[(b, "t")], comp, q[b], layer, h))
                check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"gated layer {layer} seq {b} head {h}")


def test_unit_gates_equal_the_plain_append_and_zero_gates_drop_the_residual():
    wl = _wl()
    lengths = [90, 40]
    ones = {(b, layer): torch.ones(T, wl.num_kv_heads, 2) for b, T in enumerate(lengths) for layer in range(2)}
    zeros = {(b, layer): torch.zeros(T, wl.num_kv_heads, 2) for b, T in enumerate(lengths) for layer in range(2)}
    c1, _, _, _ = _append(wl, lengths, (64, 1000), ones)
    c0, _, _, _ = _append(wl, lengths, (64, 1000), None)
    cz, _, _, _ = _append(wl, lengths, (64, 1000), zeros)
    for b, T in enumerate(lengths):
        for layer in range(2):
            x, y, z = c1.export(layer, b, 0, T), c0.export(layer, b, 0, T), cz.export(layer, b, 0, T)
            for key in x:
                assert torch.equal(x[key].cpu().view(torch.uint8), y[key].cpu().view(torch.uint8)), (b, layer, key)
            assert not z["scales"].cpu().view(torch.int16).any()
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0)
    err = cz.probe(1, [0, 1], q.cuda())
    cz.sync()
    assert float(err.abs().max()) == 0.0


def test_gate_pointer_is_checked_on_the_host():
    wl = _wl()
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=64), bases[0], bases[1])
    k, v = synth.make_dense_vectors(wl, 0, 0, 4, bases)
    t = synth.make_tiers(wl, 0, 0, 4)
    with pytest.raises(dw.DwkvError, match="gate"):
        dw.dwkv_append_gated(cache.h, 0, [0], [4], k.cuda(), v.cuda(), t.cuda(), None)
    g = torch.ones(4 * 2 * 2 + 1, device="cuda")
    with pytest.raises(dw.DwkvError, match="aligned"):
        dw.dwkv_append_gated(cache.h, 0, [0], [4], k.cuda(), v.cuda(), t.cuda(), g[1:].view(torch.uint8)[1:].view(-1))
