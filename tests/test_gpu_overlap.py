"""Decode launches that overlap their predecessor (programmatic dependent launch): a launch
may start, read the tier counts and page tables and stream pages while the previous decode of
the stream still runs, and waits for it only before reading its inputs or writing (and before
reading the cache when the previous launch was a fused step of the same group).  Results must
not depend on it: overlapped and serialised launches store identical bytes and agree to fp32
rounding, and both match the oracle, including back-to-back launches that place tokens in the
same group (a one-layer model), probes between decode steps, and graph replays."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cat_comp, cfg_for, check_close, head_problem, import_workload, oracle_encode_rows

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _run_steps(wl, T0s, steps, overlap, probe_every=0):
    """Fused append + decode of every layer for `steps` steps over all sequences, captured as
    one CUDA graph and replayed once; returns (cache, outputs [steps][L][B][Hq][d], probe
    errors or None, per-(seq, layer) oracle state)."""
    bases = synth.make_bases(wl)
    B = len(T0s)
    seqs = list(range(B))
    cache = dw.Cache(cfg_for(wl, max_batch=B, max_context=max(T0s) + steps + 8), bases[0], bases[1])
    cache.set_decode_overlap(overlap)
    data = import_workload(cache, wl, T0s)
    L, G = wl.num_layers, wl.num_groups
    K = torch.stack([torch.stack([synth.make_dense_vectors(wl, b, l, steps, bases, start=T0s[b])[0]
                                  for b in seqs], 1) for l in range(L)], 1).cuda().contiguous()   # [steps][L][B][H][d]
    V = torch.stack([torch.stack([synth.make_dense_vectors(wl, b, l, steps, bases, start=T0s[b])[1]
                                  for b in seqs], 1) for l in range(L)], 1).cuda().contiguous()
    Tn = torch.stack([torch.stack([synth.make_tiers(wl, b, g, steps, start=T0s[b]) for b in seqs], 1)
                      for g in range(G)], 1).cuda().contiguous()                                 # [steps][G][B][H]
    Q = torch.stack([synth.make_queries(wl, l, batch=steps * B, temperature=8.0).view(steps, B, -1, wl.head_dim)
                     for l in range(L)], 1).cuda().contiguous()                                   # [steps][L][B][Hq][d]
    out = torch.zeros(steps, L, B, wl.num_q_heads, wl.head_dim, dtype=torch.float32, device="cuda")
    err = torch.zeros(steps, L, B, wl.num_kv_heads, dtype=torch.float32, device="cuda") if probe_every else None
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for st in range(steps):
            for l in range(L):
                g = l // wl.layers_per_group
                dw.dwkv_append_decode_attention(cache.h, l, seqs, K[st, l], V[st, l],
                                                Tn[st, g] if l % wl.layers_per_group == 0 else None, Q[st, l],
                                                out[st, l], cache.workspace, s)
                if probe_every and st % probe_every == 0:
                    dw.dwkv_probe(cache.h, l, seqs, Q[st, l], err[st, l], None, cache.workspace, s)
    graph.replay()
    torch.cuda.synchronize()
    cache.sync()
    state = {}
    for b in seqs:
        for l in range(L):
            g = l // wl.layers_per_group
            enc = oracle_encode_rows(wl, bases, l, K[:, l, b].cpu(), V[:, l, b].cpu(), Tn[:, g, b].cpu())
            tiers, comp = data[(b, l)]
            state[(b, l)] = (tiers, comp, enc, Tn[:, g, b].cpu())
    return cache, out.cpu(), None if err is None else err.cpu(), state, bases, Q.cpu()


def _oracle_at(wl, bases, state, Q, b, l, st, h, probe=False):
    tiers, comp, enc, tn = state[(b, l)]
    part = {k: v[:st + 1] for k, v in enc.items()}
    tt = torch.cat([tiers.cpu(), tn[:st + 1]])
    prob = head_problem(wl, bases, tt, cat_comp(comp, part), Q[st, l, b], l, h)
    return oracle.probe_head(prob)[0] if probe else oracle.decode_head(prob)


def test_overlapped_and_serialised_launches_agree():
    """Stored bytes bit for bit; outputs to fp32 rounding (warps take half pages from a shared
    queue, so the order of a CTA's fp32 sums differs from run to run either way)."""
    wl = synth.workload("llama8b_64k").scaled(num_layers=4, context=3000, batch=2)
    T0s, steps = [2900, 1700], 5
    c_on, o_on, _, st_on, bases, Q = _run_steps(wl, T0s, steps, True)
    c_off, o_off, _, _, _, _ = _run_steps(wl, T0s, steps, False)
    d = (o_on - o_off).abs().max().item()
    assert d <= 1e-6 * max(o_off.abs().max().item(), 1.0), d
    for b, T0 in enumerate(T0s):
        for l in range(wl.num_layers):
            x, y = c_on.export(l, b, 0, T0 + steps), c_off.export(l, b, 0, T0 + steps)
            for key in x:
                assert torch.equal(x[key].view(torch.uint8), y[key].view(torch.uint8)), (b, l, key)
    # the last step of every layer, every head, against the oracle
    probs, where = [], []
    for b in range(2):
        for l in range(wl.num_layers):
            for h in range(wl.num_kv_heads):
                tiers, comp, enc, tn = st_on[(b, l)]
                tt = torch.cat([tiers.cpu(), tn])
                probs.append(head_problem(wl, bases, tt, cat_comp(comp, enc), Q[steps - 1, l, b], l, h))
                where.append((b, l, h))
    refs = oracle.decode_many(probs, nthreads=os.cpu_count())
    for (b, l, h), ref in zip(where, refs):
        check_close(o_on[steps - 1, l, b, h * 4:(h + 1) * 4].numpy(), ref, what=f"seq {b} layer {l} head {h}")


def test_one_layer_model_back_to_back_placing_launches():
    """Every launch places a token in the group the previous launch placed one in: a launch
    that starts early sees the previous launch's count addition in flight and must wait."""
    wl = synth.workload("tiny_1k").scaled(num_layers=1, layers_per_group=1, num_q_heads=8, num_kv_heads=2)
    T0s, steps = [190, 64], 12                   # tier pages fill and open during the steps
    _, out, _, state, bases, Q = _run_steps(wl, T0s, steps, True)
    for st in range(steps):
        for b in range(2):
            for h in range(wl.num_kv_heads):
                ref = _oracle_at(wl, bases, state, Q, b, 0, st, h)
                check_close(out[st, 0, b, h * 4:(h + 1) * 4].numpy(), ref, what=f"step {st} seq {b} head {h}")


def test_probes_between_overlapped_decode_steps():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=2)
    T0s, steps = [900, 333], 4
    _, out, err, state, bases, Q = _run_steps(wl, T0s, steps, True, probe_every=2)
    for st in (0, 2):
        for b in range(2):
            for l in range(2):
                for h in range(wl.num_kv_heads):
                    e_ref = _oracle_at(wl, bases, state, Q, b, l, st, h, probe=True)
                    assert abs(float(err[st, l, b, h]) - e_ref) <= 2e-3, (st, b, l, h, float(err[st, l, b, h]), e_ref)
    for b in range(2):
        for h in range(wl.num_kv_heads):
            ref = _oracle_at(wl, bases, state, Q, b, 1, steps - 1, h)
            check_close(out[steps - 1, 1, b, h * 4:(h + 1) * 4].numpy(), ref, what=f"last step seq {b} head {h}")
