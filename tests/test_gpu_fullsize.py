"""GPU parity at the decode workloads' full sizes, in the launch configuration the bench times:
one fused append + decode launch per layer of a group over all sequences, every kv-head of
every layer of the group checked against the fp64 oracle (which encodes each step's new token
itself).  Bars: max-abs <= 2e-3 and relative L2 <= 1e-3.

 * 64K: Llama-3-8B shapes, one sequence of 65536 tokens, int4 residual, r_max 64; and the
   same with 8-bit blockwise coefficients.
 * ragged batch: 8 sequences of 16K-32K tokens (seeded), int8 residual: the split-K
   apportionment across sequences of different lengths.
 * 131K deep: one sequence of 131072 tokens, 4-layer groups, r_max 128 with the full-rank
   tier on three 256-token spans, int4 residual with s = 8."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cat_comp, cfg_for, check_close, head_problem, import_workload, oracle_encode_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _fused_group_step(wl, lengths, temp=8.0):
    """Import T_b - 1 tokens per sequence, then one fused step over the layers of group 0;
    returns the number of (sequence, layer, kv-head) problems checked."""
    assert wl.num_layers == wl.layers_per_group
    bases = synth.make_bases(wl)
    B = len(lengths)
    seqs = list(range(B))
    cache = dw.Cache(cfg_for(wl, max_batch=B, max_context=max(lengths) + 64), bases[0], bases[1])
    data = import_workload(cache, wl, [T - 1 for T in lengths], gen_device="cuda")
    tn = [synth.make_tiers(wl, b, 0, 1, device="cuda", start=lengths[b] - 1) for b in seqs]
    t_dev = torch.cat(tn).contiguous()
    checked = 0
    for layer in range(wl.num_layers):
        kv = [synth.make_dense_vectors(wl, b, layer, 1, bases, device="cuda", start=lengths[b] - 1) for b in seqs]
        k = torch.cat([x[0] for x in kv]).contiguous()
        v = torch.cat([x[1] for x in kv]).contiguous()
        q = synth.make_queries(wl, layer, batch=B, device="cuda", temperature=temp)
        out = cache.append_decode(layer, seqs, k, v, t_dev if layer == 0 else None, q)
        cache.sync()
        out = out.cpu().numpy()
        probs, where = [], []
        for b in seqs:
            tiers, comp = data[(b, layer)]
            new = oracle_encode_rows(wl, bases, layer, kv[b][0], kv[b][1], tn[b])
            tt = torch.cat([tiers.cpu(), tn[b].cpu()])
            full = cat_comp(comp, new)
            for h in range(wl.num_kv_heads):
                probs.append(head_problem(wl, bases, tt, full, q[b].cpu(), layer, h))
                where.append((b, h))
        refs = oracle.decode_many(probs, nthreads=os.cpu_count())
        for (b, h), ref in zip(where, refs):
            check_close(out[b, h * 4:(h + 1) * 4], ref, what=f"{wl.name} layer {layer} seq {b} head {h}")
            checked += 1
        del probs, refs
    cache.close()
    return checked


def test_llama8b_64k_fused_step_every_head_both_layers():
    wl = synth.workload("llama8b_64k").scaled(num_layers=2)
    assert _fused_group_step(wl, [wl.context]) == 2 * 8


def test_llama8b_64k_8bit_coefficients_fused_step_every_head_both_layers():
    wl = synth.workload("llama8b_64k_c8").scaled(num_layers=2)
    assert _fused_group_step(wl, [wl.context]) == 2 * 8


def test_ragged_batch8_16k_32k_int8_every_sequence_and_head():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2)
    lengths = synth.make_context_lengths(wl)
    assert len(lengths) == 8 and min(lengths) >= 16384 and max(lengths) <= 32768
    assert _fused_group_step(wl, lengths) == 2 * 8 * 8


def test_131k_deep_groups_full_rank_spans_every_head_all_layers():
    wl = synth.workload("llama8b_131k_deep").scaled(num_layers=4)
    T = wl.context
    tiers = synth.make_tiers(wl, 0, 0, T)
    assert int((tiers == 4).sum()) == 3 * 256 * wl.num_kv_heads          # the three full-rank spans
    assert _fused_group_step(wl, [T]) == 4 * 8
