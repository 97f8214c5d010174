"""dwkv_append_decode_attention: one decode step (append one token, attend) in a single launch.
Its stored bytes must equal the separate dwkv_append's (and the oracle's encode) bit for bit,
and its outputs the oracle's decode over the cache with the new token, across tier page
boundaries, for the group's first layer (which places the token) and the others, for a batch
of sequences, and under CUDA-graph replay."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cat_comp, cfg_for, check_close, head_problem, import_workload, oracle_encode_rows

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _steps(wl, T0s, steps, fused, check=True, temp=8.0):
    bases = synth.make_bases(wl)
    B = len(T0s)
    cache = dw.Cache(cfg_for(wl, max_batch=B, max_context=max(T0s) + steps + 8), bases[0], bases[1])
    data = import_workload(cache, wl, T0s)
    new = {(b, l): synth.make_dense_vectors(wl, b, l, steps, bases, start=T0s[b])
           for b in range(B) for l in range(wl.num_layers)}
    newt = {(b, g): synth.make_tiers(wl, b, g, steps, start=T0s[b]) for b in range(B) for g in range(wl.num_groups)}
    state = {(b, l): data[(b, l)] for b in range(B) for l in range(wl.num_layers)}
    for step in range(steps):
        for layer in range(wl.num_layers):
            g = layer // wl.layers_per_group
            first = layer % wl.layers_per_group == 0
            k = torch.cat([new[(b, layer)][0][step:step + 1] for b in range(B)]).cuda()
            v = torch.cat([new[(b, layer)][1][step:step + 1] for b in range(B)]).cuda()
            t = torch.cat([newt[(b, g)][step:step + 1] for b in range(B)]).cuda() if first else None
            q = synth.make_queries(wl, layer, batch=B, temperature=temp, step=step)
            if fused:
                out = cache.append_decode(layer, list(range(B)), k, v, t, q.cuda())
            else:
                cache.append(layer, list(range(B)), [1] * B, k, v, t)
                out = cache.decode(layer, list(range(B)), q.cuda())
            cache.sync()
            for b in range(B):
                tiers, comp = state[(b, layer)]
                tt = newt[(b, g)][step:step + 1]
                enc = oracle_encode_rows(wl, bases, layer, new[(b, layer)][0][step:step + 1],
                                         new[(b, layer)][1][step:step + 1], tt)
                state[(b, layer)] = (torch.cat([tiers, tt]), cat_comp(comp, enc))
                if check:
                    tiers, comp = state[(b, layer)]
                    o = out[b].cpu().numpy()
                    for h in range(wl.num_kv_heads):
                        ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], layer, h))
                        check_close(o[h * 4:(h + 1) * 4], ref, what=f"step {step} layer {layer} seq {b} head {h}")
    return cache, state


def _assert_same_bytes(c1, c2, wl, lengths):
    for b, T in enumerate(lengths):
        for layer in range(wl.num_layers):
            x, y = c1.export(layer, b, 0, T), c2.export(layer, b, 0, T)
            for key in x:
                assert torch.equal(x[key].view(torch.uint8), y[key].view(torch.uint8)), (b, layer, key)


def test_fused_steps_match_the_oracle_and_the_separate_calls_across_page_boundaries():
    wl = synth.workload("tiny_1k")
    T0, steps = 160, 24                      # tier 0 crosses a page boundary within the steps
    fused, _ = _steps(wl, [T0], steps, fused=True)
    plain, _ = _steps(wl, [T0], steps, fused=False, check=False)
    _assert_same_bytes(fused, plain, wl, [T0 + steps])


def test_fused_batch_of_ragged_sequences_int8():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=3)
    T0s, steps = [700, 64, 1300], 6
    fused, _ = _steps(wl, T0s, steps, fused=True)
    plain, _ = _steps(wl, T0s, steps, fused=False, check=False)
    _assert_same_bytes(fused, plain, wl, [t + steps for t in T0s])


def test_fused_deep_group_int4_full_rank():
    wl = synth.workload("llama8b_131k_deep").scaled(num_layers=4, num_q_heads=4, num_kv_heads=1, context=2000)
    _steps(wl, [2000], 3, fused=True)


def test_fused_step_under_graph_replay():
    """The captured step reads the cache state from device memory on every replay."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T0, steps = 130, 3
    cache = dw.Cache(cfg_for(wl, max_context=T0 + 8), bases[0], bases[1])
    data = import_workload(cache, wl, [T0])
    kin = torch.empty(1, 1, 128, dtype=torch.bfloat16, device="cuda")
    vin = torch.empty_like(kin)
    tin = torch.empty(1, 1, dtype=torch.uint8, device="cuda")
    qin = torch.empty(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, 4, 128, dtype=torch.float32, device="cuda")
    newk = [synth.make_dense_vectors(wl, 0, l, steps, bases, start=T0) for l in range(2)]
    newt = synth.make_tiers(wl, 0, 0, steps, start=T0)
    qs = synth.make_queries(wl, 1, temperature=8.0)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    kin.copy_(newk[0][0][0:1]); vin.copy_(newk[0][1][0:1]); tin.copy_(newt[0:1]); qin.copy_(qs)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=s):
        cache.append_decode(0, [0], kin, vin, tin, qin, out=out, stream=s)
        cache.append_decode(1, [0], kin, vin, None, qin, out=out, stream=s)
    torch.cuda.synchronize()
    tiers, comp = data[(0, 1)]
    for step in range(steps):
        kin.copy_(newk[1][0][step:step + 1]); vin.copy_(newk[1][1][step:step + 1])
        tin.copy_(newt[step:step + 1])
        graph.replay()
        torch.cuda.synchronize()
        new = oracle_encode_rows(wl, bases, 1, newk[1][0][step:step + 1], newk[1][1][step:step + 1],
                                 newt[step:step + 1])
        tiers = torch.cat([tiers, newt[step:step + 1]])
        comp = cat_comp(comp, new)
        ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, qs[0], 1, 0))
        check_close(out[0].cpu().numpy(), ref, what=f"replay {step}")
    cache.sync()


def test_fused_falls_back_to_two_launches_when_the_ring_is_capped():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=200), bases[0], bases[1])
    import_workload(cache, wl, [100])
    cache.set_decode_tuning(1, 1, 2)          # a ring of two page chunks: too small to stage the bases
    k, v = synth.make_dense_vectors(wl, 0, 0, 1, bases, start=100)
    t = synth.make_tiers(wl, 0, 0, 1, start=100)
    q = synth.make_queries(wl, 0, temperature=8.0)
    out = cache.append_decode(0, [0], k.cuda(), v.cuda(), t.cuda(), q.cuda())
    cache.sync()
    assert np.isfinite(out.cpu().numpy()).all()
    assert cache.seq_length(0, 0) == 101


@pytest.mark.parametrize("s,bits", [(0, 4), (32, 8)])
def test_fused_steps_residual_counts(s, bits):
    wl = synth.workload("tiny_1k").scaled(resid_channels=s, resid_bits=bits)
    T0, steps = 120, 10
    fused, _ = _steps(wl, [T0], steps, fused=True)
    plain, _ = _steps(wl, [T0], steps, fused=False, check=False)
    _assert_same_bytes(fused, plain, wl, [T0 + steps])
