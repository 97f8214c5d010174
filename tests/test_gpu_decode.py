"""GPU parity of decode attention and the probe (through the C ABI) against the fp64 CPU
oracle.  Bars: decode max-abs <= 2e-3 and relative L2 <= 1e-3 (fp32 outputs vs fp64);
probe |delta e| <= 2e-3.  Sizes span several pages per split, ragged last pages and
every tier; the full-size case checks every head at 64K (the fused launches at full size are in
test_gpu_fullsize.py)."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cat_comp, check_close, cfg_for, head_problem, import_workload, oracle_encode_rows

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _decode_and_check(wl, cache, data, lengths, layer, temp=1.0, seed=None, step=0, what=""):
    B = len(lengths)
    bases = synth.make_bases(wl, seed)
    q = synth.make_queries(wl, layer, batch=B, temperature=temp, seed=seed, step=step)
    out = cache.decode(layer, list(range(B)), q.cuda())
    cache.sync()
    out = out.cpu().numpy()
    for b in range(B):
        tiers, comp = data[(b, layer)]
        for h in range(wl.num_kv_heads):
            ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], layer, h))
            check_close(out[b, h * 4:(h + 1) * 4], ref, what=f"{what} seq {b} layer {layer} head {h}")
    return out


@pytest.mark.parametrize("seed", [None, 11, 12])
@pytest.mark.parametrize("temp", [1.0, 8.0, 32.0])
def test_tiny_workload(seed, temp):
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl, seed)
    cache = dw.Cache(cfg_for(wl, max_context=1100), bases[0], bases[1])
    data = import_workload(cache, wl, [wl.context], seed=seed)
    for layer in range(wl.num_layers):
        _decode_and_check(wl, cache, data, [wl.context], layer, temp=temp, seed=seed, what="tiny")


def test_ragged_batch_int8():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=4, num_q_heads=8, num_kv_heads=2, batch=4)
    lengths = [1000, 137, 2500, 64]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=2600), bases[0], bases[1])
    data = import_workload(cache, wl, lengths)
    for layer in range(wl.num_layers):
        _decode_and_check(wl, cache, data, lengths, layer, temp=8.0, what="ragged")


def test_deep_groups_full_rank_spans_int4():
    wl = synth.workload("llama8b_131k_deep").scaled(num_layers=8, num_q_heads=8, num_kv_heads=2, context=3000)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=3000), bases[0], bases[1])
    data = import_workload(cache, wl, [3000])
    tiers = data[(0, 0)][0]
    assert int((tiers == 4).sum()) == 3 * 256 * 2   # the three spans, every kv head
    for layer in (0, 3, 5):
        _decode_and_check(wl, cache, data, [3000], layer, temp=8.0, what="deep")


def test_garbage_beyond_rank_is_ignored():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    data = import_workload(cache, wl, [700], garbage=True)
    _decode_and_check(wl, cache, data, [700], 1, temp=8.0, what="garbage tail")


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 129])
def test_short_contexts(T):
    wl = synth.workload("tiny_1k").scaled(num_q_heads=8, num_kv_heads=2)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    data = import_workload(cache, wl, [T])
    _decode_and_check(wl, cache, data, [T], 0, temp=32.0, what=f"T={T}")


def test_empty_sequence_gives_zeros_and_others_unaffected():
    wl = synth.workload("tiny_1k").scaled(batch=3)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    lengths = [300, 0, 90]
    data = import_workload(cache, wl, lengths)
    q = synth.make_queries(wl, 0, batch=3)
    out = cache.decode(0, [0, 1, 2], q.cuda())
    cache.sync()
    out = out.cpu().numpy()
    assert np.array_equal(out[1], np.zeros_like(out[1]))
    for b in (0, 2):
        tiers, comp = data[(b, 0)]
        check_close(out[b], oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], 0, 0)))


def test_sequence_subset_and_order():
    """Decode a permuted subset of the sequences: outputs follow the list order."""
    wl = synth.workload("tiny_1k").scaled(batch=4)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    lengths = [200, 333, 64, 1000]
    data = import_workload(cache, wl, lengths)
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0)
    out = cache.decode(1, [3, 1], q.cuda())
    cache.sync()
    for i, b in enumerate((3, 1)):
        tiers, comp = data[(b, 1)]
        check_close(out[i].cpu().numpy(), oracle.decode_head(head_problem(wl, bases, tiers, comp, q[i], 1, 0)))


@pytest.mark.parametrize("ctas,waves,stages", [(1, 1, 0), (1, 2, 0), (1, 3, 4), (1, 1, 8), (1, 1, 2), (1, 2, 3)])
def test_launch_tunings_agree(ctas, waves, stages):
    wl = synth.workload("llama8b_64k").scaled(num_layers=2, context=5000)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    data = import_workload(cache, wl, [5000])
    cache.set_decode_tuning(ctas, waves, stages)
    _decode_and_check(wl, cache, data, [5000], 1, temp=8.0, what=f"tuning {ctas},{waves},{stages}")


# ------------------------------------------------------------------------------ probe
@pytest.mark.parametrize("name,lengths", [("tiny_1k", [1024]), ("llama8b_ragged_b8", [700, 1500])])
def test_probe_matches_oracle(name, lengths):
    wl = synth.workload(name)
    if name != "tiny_1k":
        wl = wl.scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=len(lengths))
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=max(lengths)), bases[0], bases[1])
    data = import_workload(cache, wl, lengths)
    layer = wl.num_layers - 1
    q = synth.make_queries(wl, layer, batch=len(lengths), temperature=8.0)
    err, out = cache.probe(layer, list(range(len(lengths))), q.cuda(), want_out=True)
    dec = cache.decode(layer, list(range(len(lengths))), q.cuda())
    cache.sync()
    err, out, dec = err.cpu().numpy(), out.cpu().numpy(), dec.cpu().numpy()
    for b in range(len(lengths)):
        tiers, comp = data[(b, layer)]
        for h in range(wl.num_kv_heads):
            e_ref, of, _ = oracle.probe_head(head_problem(wl, bases, tiers, comp, q[b], layer, h))
            assert abs(err[b, h] - e_ref) <= 2e-3, (b, h, err[b, h], e_ref)
            check_close(out[b, h * 4:(h + 1) * 4], of, what="probe out_full")
    assert np.allclose(out, dec, rtol=1e-5, atol=1e-6)


def test_probe_zero_residual_is_zero():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    tiers = synth.make_tiers(wl, 0, 0, 500)
    for layer in range(2):
        comp = synth.make_compressed(wl, 0, layer, tiers)
        comp["scales"].zero_()
        c = {k: v.cuda() for k, v in comp.items()}
        cache.append_compressed(layer, [0], [500], tiers.cuda(), c["coeff"], c["idx"], c["codes"], c["scales"])
    q = synth.make_queries(wl, 0)
    err = cache.probe(0, [0], q.cuda())
    cache.sync()
    assert float(err.abs().max()) == 0.0


# ------------------------------------------------------------------------------ full size
@pytest.mark.slow
def test_llama8b_64k_full_context_every_head():
    """Full 64K context, 8 kv heads, batch 1 (one group of two layers; the launch shape does
    not depend on the layer count).  65535 imported tokens plus one encoded by dwkv_append,
    then decode with the separate calls; every head against the oracle (which encodes the
    appended token itself)."""
    wl = synth.workload("llama8b_64k").scaled(num_layers=2)
    T = wl.context
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=T + 64), bases[0], bases[1])
    data = import_workload(cache, wl, [T - 1], gen_device="cuda")
    kn, vn = synth.make_dense_vectors(wl, 0, 0, 1, bases, device="cuda", start=T - 1)
    tn = synth.make_tiers(wl, 0, 0, 1, device="cuda", start=T - 1)
    kv = {0: (kn, vn)}
    kv[1] = synth.make_dense_vectors(wl, 0, 1, 1, bases, device="cuda", start=T - 1)
    for layer in range(2):
        cache.append(layer, [0], [1], kv[layer][0], kv[layer][1], tn)
    q = synth.make_queries(wl, 1, batch=1, device="cuda", temperature=8.0)
    out = cache.decode(1, [0], q)
    cache.sync()
    out = out.cpu().numpy()
    tiers, comp = data[(0, 1)]
    new = oracle_encode_rows(wl, bases, 1, kv[1][0], kv[1][1], tn)
    tt = torch.cat([tiers.cpu(), tn.cpu()])
    full = cat_comp(comp, new)
    refs = oracle.decode_many([head_problem(wl, bases, tt, full, q[0].cpu(), 1, h) for h in range(wl.num_kv_heads)],
                              nthreads=os.cpu_count())
    for h, ref in enumerate(refs):
        check_close(out[0, h * 4:(h + 1) * 4], ref, what=f"64K head {h}")


# ------------------------------------------------------------------------------ residual widths
@pytest.mark.parametrize("s,bits", [(0, 8), (0, 4), (32, 8), (32, 4)])
def test_residual_channel_counts_decode_and_probe(s, bits):
    """No residual at all (pure low-rank: the degenerate case of Eq. 1) and the widest
    residual the kernels take; the probe is exactly 0 without a residual."""
    wl = synth.workload("tiny_1k").scaled(resid_channels=s, resid_bits=bits, num_q_heads=8, num_kv_heads=2)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    data = import_workload(cache, wl, [700])
    for layer in range(wl.num_layers):
        _decode_and_check(wl, cache, data, [700], layer, temp=8.0, what=f"s={s} bits={bits}")
    q = synth.make_queries(wl, 1, temperature=8.0)
    err = cache.probe(1, [0], q.cuda())
    cache.sync()
    err = err.cpu().numpy()
    tiers, comp = data[(0, 1)]
    for h in range(wl.num_kv_heads):
        e_ref, _, _ = oracle.probe_head(head_problem(wl, bases, tiers, comp, q[0], 1, h))
        assert abs(err[0, h] - e_ref) <= 2e-3, (h, err[0, h], e_ref)
    if s == 0:
        assert float(np.abs(err).max()) == 0.0
