"""8-bit blockwise coefficients ("DepthWeave-KV ...", §3 Method, the shared-bases paragraph:
the projection onto the basis kept as 8-bit codes, a block of 16 at a time with one fp16
scale) through the C ABI against the oracle: import / export of the coefficient records
(bytes past each token's rank ignored and read back as zero), decode and the probe over the
dequantised coefficients, encode bit for bit on both projection paths, fused append + decode,
the residual-count routing layout, r_max 128, re-tiering and the basis update's re-projection."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cat_comp, cfg_for, check_close, head_problem, import_workload, oracle_encode_rows
from test_gpu_encode import _check_projection, _encode_case

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _small(name="llama8b_64k", **kw):
    wl = synth.workload(name).scaled(num_layers=4, num_q_heads=8, num_kv_heads=2, batch=2, coeff_bits=8)
    return wl.scaled(**kw) if kw else wl


def _clean(wl, tiers, comp):
    """What the cache stores of imported arrays: zeros past the rank (codes and block scales)
    and, with routed counts, past the count."""
    n = tiers.shape[0]
    c = {k: v.clone().cpu() for k, v in comp.items()}
    ranks = synth.ranks_of(wl, tiers.cpu()).view(n, -1, 1, 1)
    keep = torch.arange(wl.r_max).view(1, 1, 1, -1) < ranks
    c["ccodes"] = c["ccodes"] * keep
    c["cscales"] = torch.where(keep[..., ::16], c["cscales"], torch.zeros_like(c["cscales"]))
    if wl.tier_resid:
        nres = synth.resid_counts_of(wl, tiers.cpu())
        on = torch.arange(wl.resid_channels).view(1, 1, 1, -1) < nres.view(n, -1, 1, 1)
        c["idx"], c["codes"] = c["idx"] * on, c["codes"] * on
        c["scales"] = c["scales"] * (nres.view(n, -1, 1) > 0)
    return c


def _assert_same8(got, ref, tiers, what=""):
    assert torch.equal(got["tier_idx"].cpu(), tiers.cpu()), what
    for key in ("ccodes", "cscales", "idx", "codes", "scales"):
        if key in ("idx", "codes") and not ref[key].shape[-1]:
            continue
        a = got[key].cpu().contiguous().view(torch.uint8)
        b = ref[key].cpu().contiguous().view(torch.uint8)
        assert torch.equal(a, b), f"{what} {key}"


@pytest.mark.parametrize("name,bits", [("llama8b_64k", 4), ("llama8b_ragged_b8", 8), ("llama8b_routed_64k", 4)])
def test_import_export_round_trip(name, bits):
    wl = _small(name, resid_bits=bits)
    lengths = [700, 129]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=800), bases[0], bases[1])
    data = import_workload(cache, wl, lengths, garbage=True)
    for (b, layer), (tiers, comp) in data.items():
        got = cache.export(layer, b, 0, lengths[b])
        _assert_same8(got, _clean(wl, tiers, comp), tiers, f"seq {b} layer {layer}")


@pytest.mark.parametrize("name,bits,temp", [("llama8b_64k", 4, 1.0), ("llama8b_64k", 4, 8.0),
                                            ("llama8b_ragged_b8", 8, 32.0), ("llama8b_routed_64k", 4, 8.0)])
def test_decode_and_probe(name, bits, temp):
    """Every layer, head and sequence; garbage past each token's rank must be ignored; a ragged
    last page (777 tokens) and several half pages."""
    wl = _small(name, resid_bits=bits)
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


def test_decode_r_max_128_and_extreme_queries():
    """r_max 128 (eight blocks a token at the full-rank tier), and queries scaled by 2^12 and
    2^-12: q~ is scaled into the f16 range by a power of two and back."""
    wl = synth.workload("llama8b_131k_deep").scaled(num_layers=4, num_q_heads=8, num_kv_heads=2, batch=2,
                                                   coeff_bits=8, tiers=(16, 32, 64, 128),
                                                   tier_probs=(0.4, 0.3, 0.2, 0.1), num_spans=0, span_tier=-1)
    lengths = [1500, 200]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1600), bases[0], bases[1])
    data = import_workload(cache, wl, lengths, garbage=True)
    for temp in (1.0, 4096.0, 1.0 / 4096.0):
        q = synth.make_queries(wl, 1, batch=2, temperature=temp)
        out = cache.decode(1, [0, 1], q.cuda())
        cache.sync()
        for b in range(2):
            tiers, comp = data[(b, 1)]
            for h in range(wl.num_kv_heads):
                ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], 1, h))
                check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"temp {temp} seq {b} head {h}")


@pytest.mark.parametrize("name,bits", [("llama8b_encode_16k", 4), ("llama8b_ragged_b8", 8), ("llama8b_routed_64k", 4)])
def test_encode_bit_exact_on_both_paths(name, bits):
    """Chunks of 1 and 4 tokens take the fp32-chain path (the oracle's own projection), the
    others the tensor-core path (the exported projection, checked against fp64, then the
    oracle's 8-bit step 2 and steps 3-6 on it)."""
    wl = _small(name, resid_bits=bits, num_layers=2)
    lengths = [260, 131]
    chunks = (1, 4, 37, 64, None)
    cache, bases, dense, c32 = _encode_case(wl, lengths, chunks=chunks)
    for b, T in enumerate(lengths):
        for layer in range(wl.num_layers):
            got = cache.export(layer, b, 0, T)
            tiers = dense[(b, "t", layer // wl.layers_per_group)]
            k, v = dense[(b, layer)]
            _check_projection(wl, bases, layer, k, v, tiers, c32[(b, layer)], f"seq {b} layer {layer}")
            ref = oracle_encode_rows(wl, bases, layer, k, v, tiers, c32=c32[(b, layer)])
            _assert_same8(got, ref, tiers, f"seq {b} layer {layer}")
    # the single-token appends project with the oracle's fp32 chain: the oracle's own bytes
    k, v = dense[(0, 0)]
    tiers = dense[(0, "t", 0)]
    own = oracle_encode_rows(wl, bases, 0, k[:1], v[:1], tiers[:1])
    _assert_same8(cache.export(0, 0, 0, 1), own, tiers[:1], "first token, own projection")


def test_encoded_cache_decodes_like_the_oracle():
    wl = _small("llama8b_encode_16k", num_layers=2)
    lengths = [900, 333]
    cache, bases, dense, c32 = _encode_case(wl, lengths)
    for layer in range(wl.num_layers):
        q = synth.make_queries(wl, layer, batch=2, temperature=8.0)
        out = cache.decode(layer, [0, 1], q.cuda())
        cache.sync()
        for b in range(2):
            tiers = dense[(b, "t", 0)]
            k, v = dense[(b, layer)]
            comp = oracle_encode_rows(wl, bases, layer, k, v, tiers, c32=c32[(b, layer)])
            for h in range(wl.num_kv_heads):
                ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], layer, h))
                check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"layer {layer} seq {b} head {h}")


def test_fused_append_decode_steps():
    wl = _small()
    lengths = [1500, 300]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1600), bases[0], bases[1])
    data = import_workload(cache, wl, lengths)
    state = dict(data)
    for step in range(3):
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
        got = cache.export(1, b, T, 3)
        tiers, comp = state[(b, 1)]
        want = {k_: v_[T:T + 3] for k_, v_ in comp.items()}
        _assert_same8(got, want, tiers[T:T + 3], f"appended seq {b}")


def _expected_after_moves(wl, bases, data, moves):
    """Token-ordered arrays of every (seq, layer) after the moves {seq: (positions, new_tier
    [n][H])}: the stored (clean) bytes, with each moved (token, head) re-encoded by the oracle
    from its stored 8-bit form at the new tier."""
    exp = {}
    nres_of = wl.tier_resid or (wl.resid_channels,) * len(wl.tiers)
    for (b, layer), (tiers, comp) in data.items():
        g = layer // wl.layers_per_group
        c = _clean(wl, tiers, comp)
        t = tiers.clone().cpu()
        if b in moves:
            pos, nt = moves[b]
            for n, p in enumerate(pos.tolist()):
                for h in range(wl.num_kv_heads):
                    k_old, k_new = int(t[p, h]), int(nt[n, h])
                    if k_old == k_new:
                        continue
                    t[p, h] = k_new
                    s_old, s_new = int(nres_of[k_old]), int(nres_of[k_new])
                    for z in range(2):
                        r = oracle.reencode_vector8(bases[z][g, h], wl.tiers[k_old], c["ccodes"][p, h, z],
                                                    c["cscales"][p, h, z], c["idx"][p, h, z, :s_old],
                                                    c["codes"][p, h, z, :s_old], c["scales"][p, h, z],
                                                    wl.tiers[k_new], wl.resid_bits, s_new=s_new)
                        c["ccodes"][p, h, z] = torch.from_numpy(r["ccodes"])
                        c["cscales"][p, h, z] = torch.from_numpy(r["cscales"].view(np.float16).copy())
                        c["idx"][p, h, z] = 0
                        c["codes"][p, h, z] = 0
                        c["idx"][p, h, z, :s_new] = torch.from_numpy(r["idx"])
                        c["codes"][p, h, z, :s_new] = torch.from_numpy(r["codes"])
                        c["scales"][p, h, z] = torch.from_numpy(np.array([r["scale"]], np.uint16).view(np.float16))[0]
        exp[(b, layer)] = (t, c)
    return exp


def _moves(wl, lengths, n, seed):
    g = torch.Generator().manual_seed(seed)
    out = {}
    for b, T in enumerate(lengths):
        pos = torch.randperm(T, generator=g)[:n].to(torch.int32)
        out[b] = (pos, torch.randint(0, len(wl.tiers), (n, wl.num_kv_heads), generator=g).to(torch.uint8))
    return out


def _retier(cache, group, moves):
    seqs = sorted(moves)
    pos = torch.cat([moves[b][0] for b in seqs]).cuda()
    nt = torch.cat([moves[b][1] for b in seqs]).cuda().contiguous()
    cache.retier(group, seqs, [len(moves[b][0]) for b in seqs], pos, nt)


def _deep128():
    return synth.workload("llama8b_131k_deep").scaled(num_q_heads=8, num_kv_heads=2, batch=2, coeff_bits=8,
                                                      tiers=(16, 32, 64, 128), tier_probs=(0.4, 0.3, 0.2, 0.1),
                                                      num_spans=0, span_tier=-1)


@pytest.mark.parametrize("name,bits", [("llama8b_64k", 4), ("llama8b_ragged_b8", 8), ("llama8b_routed_64k", 4),
                                       ("r_max_128", 4)])
def test_retier_reencodes_moved_tokens_bit_exact_and_decode_matches(name, bits):
    """Moved tokens are re-encoded from code x scale at their new tier (the last slot of the
    old tier fills the hole, with its codes, block scales and residual), bit for bit as the
    oracle; every other token keeps its bytes; decode over the result matches the oracle."""
    wl = _deep128() if name == "r_max_128" else _small(name)
    wl = wl.scaled(num_layers=wl.layers_per_group, resid_bits=bits)
    lengths = [700, 333]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=800), bases[0], bases[1])
    data = import_workload(cache, wl, lengths, garbage=True)
    moves = _moves(wl, lengths, 90, seed=17)
    _retier(cache, 0, moves)
    cache.sync()
    exp = _expected_after_moves(wl, bases, data, moves)
    for (b, layer), (t, c) in exp.items():
        _assert_same8(cache.export(layer, b, 0, lengths[b]), c, t, f"{name} seq {b} layer {layer}")
    for layer in range(wl.num_layers):
        q = synth.make_queries(wl, layer, batch=2, temperature=8.0)
        out = cache.decode(layer, [0, 1], q.cuda())
        cache.sync()
        for b in range(2):
            t, c = exp[(b, layer)]
            for h in range(wl.num_kv_heads):
                ref = oracle.decode_head(head_problem(wl, bases, t, c, q[b], layer, h))
                check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"{name} layer {layer} seq {b} head {h}")


def test_retier_back_and_forth_then_fused_steps():
    """Two rounds of moves (the second undoing part of the first) and fused append + decode
    steps after them: the appended token lands at the end of its tier again."""
    wl = _small(num_layers=2)
    T0 = 500
    bases = synth.make_bases(wl)
    cfg = cfg_for(wl, max_context=T0 + 8)
    cache = dw.Cache(cfg, bases[0], bases[1], arena_bytes=dw.dwkv_arena_bytes_all_tiers(cfg))
    data = import_workload(cache, wl, [T0, 200])
    state = dict(data)
    for rnd in range(2):
        moves = {0: (torch.arange(0, T0, 3, dtype=torch.int32),
                     torch.full((len(range(0, T0, 3)), wl.num_kv_heads), (len(wl.tiers) - 1) * (1 - rnd),
                                dtype=torch.uint8))}
        _retier(cache, 0, moves)
        cache.sync()
        state = _expected_after_moves(wl, bases, state, moves)
        for layer in range(2):
            t, c = state[(0, layer)]
            _assert_same8(cache.export(layer, 0, 0, T0), c, t, f"round {rnd} layer {layer}")
    for step in range(3):
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


def test_basis_update_reprojects_8bit_tokens():
    """The moving-average update re-projects every stored token of the window: reconstruction
    from code x scale on the previous basis, the 8-bit encode on the new one, bit for bit as the
    oracle; decode over the result on the new bases."""
    wl = synth.workload("llama8b_encode_16k").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=2,
                                                     coeff_bits=8)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=800), bases[0], bases[1])
    lengths = [400, 222]
    tiers = [synth.make_tiers(wl, b, 0, n) for b, n in enumerate(lengths)]
    for layer in range(2):
        ks, vs = zip(*[synth.make_dense_vectors(wl, b, layer, n, bases) for b, n in enumerate(lengths)])
        cache.append(layer, [0, 1], lengths, torch.cat(ks).cuda(), torch.cat(vs).cuda(),
                     torch.cat(tiers).cuda() if layer == 0 else None)
    cache.sync()
    before = {(b, layer): {k_: v_.cpu() for k_, v_ in cache.export(layer, b, 0, n).items()}
              for b, n in enumerate(lengths) for layer in range(2)}
    wl2 = wl.scaled(base_seed=wl.base_seed + 91)
    b2 = synth.make_bases(wl2)
    rows = [synth.make_dense_vectors(wl2, 0, layer, 300, b2, start=2000) for layer in range(2)]
    k_rows = torch.stack([r[0] for r in rows]).contiguous()
    v_rows = torch.stack([r[1] for r in rows]).contiguous()
    cache.basis_update(0, k_rows.cuda(), v_rows.cuda(), 0.0, [0, 1])
    bk1, bv1 = cache.bases(0)
    cache.sync()
    bk1, bv1 = bk1.cpu(), bv1.cpu()
    old = (bases[0][0], bases[1][0])
    for (b, layer), oc in before.items():
        got = cache.export(layer, b, 0, lengths[b])
        assert torch.equal(got["tier_idx"].cpu(), oc["tier_idx"])
        for t in range(0, lengths[b], 5):
            for h in range(wl.num_kv_heads):
                r = wl.tiers[int(oc["tier_idx"][t, h])]
                for z in range(2):
                    ref = oracle.reencode_vector8(old[z][h], r, oc["ccodes"][t, h, z], oc["cscales"][t, h, z],
                                                  oc["idx"][t, h, z], oc["codes"][t, h, z], oc["scales"][t, h, z], r,
                                                  wl.resid_bits, basis_new=(bk1, bv1)[z][h])
                    what = (b, layer, t, h, z)
                    assert np.array_equal(got["ccodes"][t, h, z].cpu().numpy(), ref["ccodes"]), what
                    assert np.array_equal(got["cscales"][t, h, z].cpu().view(torch.int16).numpy().view(np.uint16),
                                          ref["cscales"]), what
                    assert np.array_equal(got["idx"][t, h, z].cpu().numpy(), ref["idx"]), what
                    assert np.array_equal(got["codes"][t, h, z].cpu().numpy(), ref["codes"]), what
                    assert (int(got["scales"][t, h, z].cpu().view(torch.int16).item()) & 0xffff) == int(ref["scale"])
    nb = (bk1.unsqueeze(0), bv1.unsqueeze(0))
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0)
    out = cache.decode(1, [0, 1], q.cuda())
    cache.sync()
    for b in range(2):
        comp = {k_: v_.cpu() for k_, v_ in cache.export(1, b, 0, lengths[b]).items() if k_ != "tier_idx"}
        for h in range(wl.num_kv_heads):
            ref = oracle.decode_head(head_problem(wl, nb, tiers[b], comp, q[b], 1, h))
            check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"after update seq {b} head {h}")
