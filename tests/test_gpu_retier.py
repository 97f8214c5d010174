"""dwkv_retier (through the C ABI): stored tokens moved to other rank tiers are re-encoded from
their reconstruction at the new rank, bit for bit as the oracle's re-encode; every other token
keeps its bytes; decode over the re-tiered cache matches the oracle; fused decode steps go on
after it; pages emptied by the moves are reused, so repeated moves do not grow the pool.
Also the whole probe -> threshold -> promotion loop of the tier controller."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cat_comp, cfg_for, check_close, head_problem, import_workload, oracle_encode_rows

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _expected_after(wl, bases, data, moves):
    """Expected token-ordered arrays of every (seq, layer) after the moves {(seq): (positions,
    new_tier [n][H])}, from the oracle's re-encode of the imported values."""
    exp = {}
    tiers_new = {}
    nres_of = wl.tier_resid or (wl.resid_channels,) * len(wl.tiers)
    for (b, layer), (tiers, comp) in data.items():
        g = layer // wl.layers_per_group
        c = {k: v.clone().cpu() for k, v in comp.items()}
        t = tiers.clone().cpu()
        # the cache stores (and exports) +0 past each token's rank, whatever the input held there,
        # and zeros past its residual count
        keep = torch.arange(wl.r_max).view(1, 1, 1, -1) < synth.ranks_of(wl, t).view(t.shape[0], -1, 1, 1)
        c["coeff"] = torch.where(keep, c["coeff"], torch.zeros_like(c["coeff"]))
        nres = synth.resid_counts_of(wl, t)
        on = torch.arange(wl.resid_channels).view(1, 1, 1, -1) < nres.view(t.shape[0], -1, 1, 1)
        c["idx"], c["codes"] = c["idx"] * on, c["codes"] * on
        c["scales"] = c["scales"] * (nres.view(t.shape[0], -1, 1) > 0)
        if b in moves:
            pos, nt = moves[b]
            for n, p in enumerate(pos.tolist()):
                for h in range(wl.num_kv_heads):
                    k_old, k_new = int(tiers[p, h]), int(nt[n, h])
                    t[p, h] = k_new
                    if k_old == k_new:
                        continue
                    s_old, s_new = int(nres_of[k_old]), int(nres_of[k_new])
                    for z in range(2):
                        c["coeff"][p, h, z] = 0
                        r = oracle.reencode_vector(bases[z][g, h], wl.tiers[k_old], comp["coeff"][p, h, z],
                                                   comp["idx"][p, h, z, :s_old], comp["codes"][p, h, z, :s_old],
                                                   comp["scales"][p, h, z], wl.tiers[k_new], wl.resid_bits, s_new=s_new)
                        c["coeff"][p, h, z] = torch.from_numpy(r["coeff"].view(np.int16)).view(torch.bfloat16)
                        c["idx"][p, h, z] = 0
                        c["codes"][p, h, z] = 0
                        c["idx"][p, h, z, :s_new] = torch.from_numpy(r["idx"])
                        c["codes"][p, h, z, :s_new] = torch.from_numpy(r["codes"])
                        c["scales"][p, h, z] = torch.from_numpy(np.array([r["scale"]], np.uint16).view(np.int16)).view(torch.float16)[0]
        exp[(b, layer)] = (t, c)
        tiers_new[b] = t
    return exp


def _export_equal(cache, wl, exp, lengths):
    for (b, layer), (t, c) in exp.items():
        x = cache.export(layer, b, 0, lengths[b])
        assert torch.equal(x["tier_idx"].cpu(), t), (b, layer)
        for key in ("coeff", "idx", "codes", "scales"):
            assert torch.equal(x[key].cpu().view(torch.uint8), c[key].contiguous().view(torch.uint8)), (b, layer, key)


def _moves(wl, lengths, n, seed):
    g = torch.Generator().manual_seed(seed)
    out = {}
    for b, T in enumerate(lengths):
        pos = torch.randperm(T, generator=g)[:n].to(torch.int32)
        nt = torch.randint(0, len(wl.tiers), (n, wl.num_kv_heads), generator=g).to(torch.uint8)
        out[b] = (pos, nt)
    return out


def _retier(cache, wl, group, moves):
    seqs = sorted(moves)
    pos = torch.cat([moves[b][0] for b in seqs]).cuda()
    nt = torch.cat([moves[b][1] for b in seqs]).cuda().contiguous()
    cache.retier(group, seqs, [len(moves[b][0]) for b in seqs], pos, nt)


@pytest.mark.parametrize("name", ["llama8b_64k", "llama8b_ragged_b8", "llama8b_131k_deep", "llama8b_routed_64k"])
def test_moved_tokens_are_reencoded_bit_exact_and_decode_matches(name):
    wl = synth.workload(name).scaled(num_q_heads=8, num_kv_heads=2, batch=2)
    wl = wl.scaled(num_layers=wl.layers_per_group)
    lengths = [700, 333]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=800), bases[0], bases[1])
    data = import_workload(cache, wl, lengths)
    moves = _moves(wl, lengths, 90, seed=7)
    _retier(cache, wl, 0, moves)
    cache.sync()
    exp = _expected_after(wl, bases, data, moves)
    _export_equal(cache, wl, exp, lengths)
    for layer in range(wl.num_layers):
        q = synth.make_queries(wl, layer, batch=2, temperature=8.0)
        out = cache.decode(layer, [0, 1], q.cuda())
        cache.sync()
        for b in range(2):
            t, c = exp[(b, layer)]
            for h in range(wl.num_kv_heads):
                ref = oracle.decode_head(head_problem(wl, bases, t, c, q[b], layer, h))
                check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"{name} layer {layer} seq {b} head {h}")


def test_repeated_moves_reuse_pages_and_fused_steps_continue():
    wl = synth.workload("tiny_1k").scaled(num_q_heads=8, num_kv_heads=2)
    T0 = 600
    bases = synth.make_bases(wl)
    cfg = cfg_for(wl, max_context=T0 + 16)
    cache = dw.Cache(cfg, bases[0], bases[1], arena_bytes=dw.dwkv_arena_bytes_all_tiers(cfg))
    data = import_workload(cache, wl, [T0])
    state = {(0, l): data[(0, l)] for l in range(2)}
    reserved = []
    for cycle in range(4):
        # promote every tier-0 token of head 0 / the first 200 positions of head 1 to the top tier,
        # then (next cycle) take them back down: tiers empty and refill their pages
        tiers = state[(0, 0)][0]
        top = len(wl.tiers) - 1
        pos = torch.arange(0, T0, dtype=torch.int32)
        nt = tiers.clone()
        if cycle % 2 == 0:
            nt[:, 0] = torch.where(tiers[:, 0] == 0, torch.full_like(tiers[:, 0], top), tiers[:, 0])
            nt[:200, 1] = top
        else:
            nt[:, 0] = torch.where(tiers[:, 0] == top, torch.zeros_like(tiers[:, 0]), tiers[:, 0])
            nt[:200, 1] = 0
        moves = {0: (pos, nt)}
        _retier(cache, wl, 0, moves)
        cache.sync()
        exp = _expected_after(wl, bases, state, moves)
        _export_equal(cache, wl, exp, [T0])
        state = exp
        reserved.append(cache.pool_usage()["data_bytes_reserved"])
    # after one promote / demote cycle every page a move needs comes back through the free rings
    assert reserved[1] == reserved[2] == reserved[3], reserved
    # fused append + decode steps after the moves: the new token is the last slot of its tier again
    steps = 5
    for step in range(steps):
        for layer in range(2):
            k, v = synth.make_dense_vectors(wl, 0, layer, 1, bases, start=T0 + step)
            t = synth.make_tiers(wl, 0, 0, 1, start=T0 + step)
            q = synth.make_queries(wl, layer, temperature=8.0, step=step)
            out = cache.append_decode(layer, [0], k.cuda(), v.cuda(), t.cuda() if layer == 0 else None, q.cuda())
            cache.sync()
            tiers, comp = state[(0, layer)]
            enc = oracle_encode_rows(wl, bases, layer, k, v, t)
            state[(0, layer)] = (torch.cat([tiers, t]), cat_comp(comp, enc))
            for h in range(wl.num_kv_heads):
                ref = oracle.decode_head(head_problem(wl, bases, *state[(0, layer)], q[0], layer, h))
                check_close(out[0, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"step {step} layer {layer} head {h}")


def test_retier_refuses_a_group_with_unequal_layers_and_checks_on_device():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=300), bases[0], bases[1])
    import_workload(cache, wl, [200], layers=[0])            # layer 1 of the group still empty
    pos = torch.tensor([3], dtype=torch.int32, device="cuda")
    nt = torch.tensor([[2]], dtype=torch.uint8, device="cuda")
    with pytest.raises(dw.DwkvError, match="same positions"):
        cache.retier(0, [0], [1], pos, nt)
    import_workload(cache, wl, [200], layers=[1])
    bad = torch.tensor([[7]], dtype=torch.uint8, device="cuda")               # tier index out of range
    cache.retier(0, [0], [1], pos, bad)
    with pytest.raises(dw.DwkvError, match="tier index"):
        cache.sync()
    cache.retier(0, [0], [1], torch.tensor([250], dtype=torch.int32, device="cuda"), nt)   # never placed
    with pytest.raises(dw.DwkvError, match="never placed"):
        cache.sync()


def test_probe_threshold_promotion_loop():
    """The controller loop of the pages: probe every p steps; when a group's error is above the
    tolerance its threshold drops and the tokens whose salience now clears it are promoted to
    the top tier; the probe error of that group does not grow, and decode still matches."""
    wl = synth.workload("llama8b_64k").scaled(num_layers=4, num_q_heads=8, num_kv_heads=2, context=900)
    T = 900
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=T + 8), bases[0], bases[1])
    data = import_workload(cache, wl, [T])
    pol = dw.dwkv_tier_policy()
    pol.tol, pol.tau_init, pol.tau_min, pol.tau_max = 1e-4, 0.95, 0.05, 0.99
    pol.tau_step_down, pol.tau_step_up, pol.quiet_intervals, pol.probe_every = 0.3, 0.05, 2, 1
    ctrl = dw.dwkv_tier_controller_create(pol, wl.num_groups)
    g = torch.Generator().manual_seed(3)
    salience = torch.rand(wl.num_groups, T, wl.num_kv_heads, generator=g).numpy()
    state = dict(data)
    top = len(wl.tiers) - 1
    try:
        for group in range(wl.num_groups):
            layers = range(group * wl.layers_per_group, (group + 1) * wl.layers_per_group)
            q = {l: synth.make_queries(wl, l, temperature=8.0) for l in layers}
            errs = [cache.probe(l, [0], q[l].cuda()) for l in layers]
            cache.sync()
            e0 = max(float(e.max()) for e in errs)
            assert dw.dwkv_tier_controller_observe(ctrl, group, e0)          # tol 1e-4: always above
            tiers = state[(0, layers[0])][0]
            new = np.stack([dw.dwkv_tier_controller_route(ctrl, group, salience[group, :, h], tiers[:, h].numpy(), top)
                            for h in range(wl.num_kv_heads)], 1)
            tau = dw.dwkv_tier_controller_threshold(ctrl, group)
            assert tau == pytest.approx(0.65)
            assert ((new == top) == ((salience[group] > tau) | (tiers.numpy() == top))).all()
            moves = {0: (torch.arange(T, dtype=torch.int32), torch.from_numpy(new))}
            _retier(cache, wl, group, moves)
            cache.sync()
            sub = {(0, l): state[(0, l)] for l in layers}
            exp = _expected_after(wl, bases, sub, moves)
            state.update(exp)
            errs1 = [cache.probe(l, [0], q[l].cuda()) for l in layers]
            cache.sync()
            for l, e in zip(layers, errs1):
                for h in range(wl.num_kv_heads):
                    e_ref, _, _ = oracle.probe_head(head_problem(wl, bases, *state[(0, l)], q[l][0], l, h))
                    assert abs(float(e[0, h]) - e_ref) <= 2e-3
            out = cache.decode(layers[-1], [0], q[layers[-1]].cuda())
            cache.sync()
            refs = oracle.decode_many([head_problem(wl, bases, *state[(0, layers[-1])], q[layers[-1]][0], layers[-1], h)
                                       for h in range(wl.num_kv_heads)], nthreads=os.cpu_count())
            for h, ref in enumerate(refs):
                check_close(out[0, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"group {group} head {h}")
    finally:
        dw.dwkv_tier_controller_destroy(ctrl)
