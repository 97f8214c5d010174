"""GPU encode/append (through the C ABI) against the oracle's encoder, bit for bit:
stored bf16 coefficients, channel indices, integer codes and fp16 scales, plus the
tier each token was placed in.  Appends of up to 4 tokens per sequence project with the
fp32 fma chain the oracle runs, so their bytes and exported projections equal the oracle's
own; larger appends project on the tensor cores, so their projection is checked against the
fp64 projection (within 1e-5 |x|) and their bytes against the oracle's steps 2-6 on the
exported projection.  Then decode over an encoded cache against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import (cat_comp, cfg_for, check_close, head_problem, oracle_encode_rows, signed_permutation)

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _assert_same(got: dict, ref: dict, tiers, what=""):
    assert torch.equal(got["tier_idx"].cpu(), tiers.cpu()), what
    assert torch.equal(got["coeff"].cpu().view(torch.int16), ref["coeff"].view(torch.int16)), what + " coeff"
    if ref["idx"].shape[-1]:
        assert torch.equal(got["idx"].cpu(), ref["idx"]), what + " idx"
        assert torch.equal(got["codes"].cpu(), ref["codes"]), what + " codes"
    assert torch.equal(got["scales"].cpu().view(torch.int16), ref["scales"].view(torch.int16)), what + " scales"


def _check_projection(wl, bases, layer, k, v, tiers, c32, what=""):
    """The exported fp32 projection against the fp64 one (numpy matmul of the exact bf16
    values), within 1e-5 |x| for every kept coefficient."""
    g = layer // wl.layers_per_group
    ranks = synth.ranks_of(wl, tiers.cpu()).numpy()
    c32 = np.asarray(c32.cpu(), np.float64)
    for z, x in enumerate((k, v)):
        xf = x.cpu().to(torch.float64).numpy()                     # [n][H][d]
        for h in range(wl.num_kv_heads):
            Bm = bases[z][g, h].to(torch.float64).numpy()            # [d][r_max]
            exact = xf[:, h] @ Bm                                    # [n][r_max]
            keep = np.arange(wl.r_max)[None, :] < ranks[:, h][:, None]
            err = np.abs(np.where(keep, c32[:, h, z] - exact, 0.0)).max(axis=1)
            assert np.all(err <= 1e-5 * np.linalg.norm(xf[:, h], axis=1) + 1e-30), what


def _encode_case(wl, lengths, chunks=(None,), gen_device="cpu"):
    """Appends the dense rows in chunks; returns the cache, the bases, the inputs and, per
    (sequence, layer), the projection each row's append exported (fp32 [T][H][2][r_max])."""
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_batch=len(lengths), max_context=max(lengths) + 8), bases[0], bases[1])
    dense = {}
    c32 = {(b, layer): torch.full((T, wl.num_kv_heads, 2, wl.r_max), float("nan"))
           for b, T in enumerate(lengths) for layer in range(wl.num_layers)}
    for b, T in enumerate(lengths):
        for layer in range(wl.num_layers):
            dense[(b, layer)] = synth.make_dense_vectors(wl, b, layer, T, bases, device=gen_device)
        for g in range(wl.num_groups):
            dense[(b, "t", g)] = synth.make_tiers(wl, b, g, T, device=gen_device)
    for layer in range(wl.num_layers):
        g = layer // wl.layers_per_group
        # append in chunks (all sequences per call), splitting each sequence the same way
        bounds = {b: [0] for b in range(len(lengths))}
        for c in chunks:
            for b, T in enumerate(lengths):
                bounds[b].append(T if c is None else min(T, bounds[b][-1] + c))
        for step in range(len(chunks)):
            seqs, ns, ks, vs, ts = [], [], [], [], []
            for b in range(len(lengths)):
                a, e = bounds[b][step], bounds[b][step + 1]
                if e > a:
                    seqs.append(b)
                    ns.append(e - a)
                    ks.append(dense[(b, layer)][0][a:e])
                    vs.append(dense[(b, layer)][1][a:e])
                    ts.append(dense[(b, "t", g)][a:e])
            if seqs:
                lay0 = layer % wl.layers_per_group == 0
                dbg = torch.full((sum(ns), wl.num_kv_heads, 2, wl.r_max), float("nan"), device="cuda")
                cache.append(layer, seqs, ns, torch.cat(ks).cuda(), torch.cat(vs).cuda(),
                             torch.cat(ts).cuda() if lay0 else None, coeff_dbg=dbg)
                dbg = dbg.cpu()
                o = 0
                for b, n_ in zip(seqs, ns):
                    a = bounds[b][step]
                    c32[(b, layer)][a:a + n_] = dbg[o:o + n_]
                    o += n_
    cache.sync()
    return cache, bases, dense, c32


@pytest.mark.parametrize("name", ["llama8b_encode_16k", "llama8b_ragged_b8", "llama8b_131k_deep", "tiny_1k"])
def test_encode_bit_exact(name):
    wl = synth.workload(name)
    lpg = wl.layers_per_group
    wl = wl.scaled(num_layers=lpg, num_q_heads=8 if wl.num_kv_heads > 1 else 4,
                   num_kv_heads=2 if wl.num_kv_heads > 1 else 1, batch=2)
    lengths = [300, 77]
    cache, bases, dense, c32 = _encode_case(wl, lengths)
    for b, T in enumerate(lengths):
        for layer in range(wl.num_layers):
            got = cache.export(layer, b, 0, T)
            tiers = dense[(b, "t", layer // lpg)]
            k, v = dense[(b, layer)]
            _check_projection(wl, bases, layer, k, v, tiers, c32[(b, layer)], f"{name} seq {b} layer {layer}")
            ref = oracle_encode_rows(wl, bases, layer, k, v, tiers, c32=c32[(b, layer)])
            _assert_same(got, ref, tiers, f"{name} seq {b} layer {layer}")


def test_chunked_appends_bit_exact_on_both_paths():
    """Chunks of 1 and 4 tokens take the fp32-chain path (bytes and projection equal the
    oracle's own), the others the tensor-core path (bytes equal the oracle's steps 2-6 on the
    exported projection)."""
    wl = synth.workload("llama8b_encode_16k").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=2)
    lengths = [200, 131]
    chunks = (1, 1, 37, 4, 64, 5, None)
    cache, bases, dense, c32 = _encode_case(wl, lengths, chunks=chunks)
    for b, T in enumerate(lengths):
        small = np.zeros(T, bool)
        a = 0
        for c in chunks:
            e = T if c is None else min(T, a + c)
            if c is not None and c <= 4:
                small[a:e] = True
            a = e
        for layer in range(2):
            got = cache.export(layer, b, 0, T)
            tiers = dense[(b, "t", 0)]
            k, v = dense[(b, layer)]
            _check_projection(wl, bases, layer, k, v, tiers, c32[(b, layer)], f"seq {b} layer {layer}")
            _assert_same(got, oracle_encode_rows(wl, bases, layer, k, v, tiers, c32=c32[(b, layer)]), tiers,
                         f"seq {b} layer {layer}")
            own = oracle_encode_rows(wl, bases, layer, k[small], v[small], tiers[small])
            _assert_same({key: val.cpu()[torch.from_numpy(small)] for key, val in got.items()}, own, tiers[small],
                         f"chain rows seq {b} layer {layer}")


def test_decode_sized_appends_bit_exact():
    """Appends of 1-4 tokens per sequence take the one-launch place + encode path; the stored
    bytes must equal the oracle's for every row, with sequences joining and leaving calls."""
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=3)
    lengths = [23, 9, 30]
    cache, bases, dense, c32 = _encode_case(wl, lengths, chunks=(1, 4, 2, 3, 1, 4, 4, 4, 4, 4))
    g = 0
    for b, T in enumerate(lengths):
        for layer in range(wl.num_layers):
            got = cache.export(layer, b, 0, T)
            tiers = dense[(b, "t", layer // wl.layers_per_group)]
            ref = oracle_encode_rows(wl, bases, layer, dense[(b, layer)][0], dense[(b, layer)][1], tiers)
            _assert_same(got, ref, tiers, f"small appends seq {b} layer {layer}")
            # the exported projection is the oracle's fp32 chain, bit for bit
            ranks = synth.ranks_of(wl, tiers.cpu())
            for h in range(wl.num_kv_heads):
                for z in range(2):
                    x = dense[(b, layer)][z][:, h]
                    for t in range(T):
                        r = int(ranks[t, h])
                        own = oracle.encode_vector(bases[z][g, h], x[t], r, wl.resid_channels, wl.resid_bits)["c32"]
                        assert np.array_equal(c32[(b, layer)][t, h, z, :r].numpy(), own[:r]), (b, layer, t, h, z)


def test_exact_planted_vectors_and_zero_vectors():
    """Signed-permutation bases and planted residuals (every encoder step exact), and zero
    vectors (ties at zero go to the lowest channels)."""
    wl = synth.workload("tiny_1k").scaled(r_max=32, tiers=(8, 16, 32), resid_channels=8, resid_bits=4)
    B0, perm, sign = signed_permutation(128, 32, 3)
    B1, _, _ = signed_permutation(128, 32, 4)
    bk = B0.view(1, 1, 128, 32).contiguous()
    bv = B1.view(1, 1, 128, 32).contiguous()
    cache = dw.Cache(cfg_for(wl, max_context=64), bk, bv)
    n = 40
    g = torch.Generator().manual_seed(9)
    tiers = torch.randint(0, 3, (n, 1), generator=g).to(torch.uint8)
    x = torch.zeros(n, 1, 128)
    for t in range(n - 4):
        r = wl.tiers[int(tiers[t, 0])]
        cvals = (torch.randint(-8, 9, (r,), generator=g) * 0.25)
        for j in range(r):
            x[t, 0, perm[j]] += sign[j] * cvals[j]
        free = [c for c in range(128) if c not in set(perm[:r].tolist())]
        ch = torch.tensor(free)[torch.randperm(len(free), generator=g)[:5]]
        x[t, 0, ch] = torch.randint(-7, 8, (5,), generator=g).float() * 2.0 ** -6
    k = x.to(torch.bfloat16)
    v = (x * 0.5).to(torch.bfloat16)
    cache.append(0, [0], [n], k.cuda(), v.cuda(), tiers.cuda())          # tensor-core projection:
    cache.append(1, [0], [n], v.cuda(), k.cuda(), None)                  # one nonzero term, exact
    cache.sync()
    for layer, (kk, vv) in enumerate(((k, v), (v, k))):
        got = cache.export(layer, 0, 0, n)
        ref = oracle_encode_rows(wl, (bk, bv), layer, kk, vv, tiers)
        _assert_same(got, ref, tiers, f"planted layer {layer}")
    got = cache.export(0, 0, n - 4, 4)
    assert not got["coeff"].view(torch.int16).any() and not got["codes"].any()
    assert got["idx"][0, 0, 0].tolist() == list(range(8))


@pytest.mark.slow
def test_encode_full_size_sampled():
    """Encode workload at its full per-layer size (4 sequences x 16384 tokens x 8 kv heads,
    keys and values) for one group of two layers; bit-exact check on sampled tokens."""
    wl = synth.workload("llama8b_encode_16k").scaled(num_layers=2)
    bases = synth.make_bases(wl)
    n = wl.new_tokens
    cache = dw.Cache(cfg_for(wl, max_context=n), bases[0], bases[1])
    dense, tiers = {}, {}
    for layer in range(2):
        ks, vs, ts = [], [], []
        for b in range(wl.batch):
            k, v = synth.make_dense_vectors(wl, b, layer, n, bases, device="cuda")
            ks.append(k)
            vs.append(v)
            if layer == 0:
                tiers[b] = synth.make_tiers(wl, b, 0, n, device="cuda")
            ts.append(tiers[b])
            dense[(b, layer)] = (k, v)
        dbg = torch.full((wl.batch * n, wl.num_kv_heads, 2, wl.r_max), float("nan"), device="cuda")
        cache.append(layer, list(range(wl.batch)), [n] * wl.batch, torch.cat(ks), torch.cat(vs),
                     torch.cat(ts) if layer == 0 else None, coeff_dbg=dbg)
        dense[("dbg", layer)] = dbg.cpu()
    cache.sync()
    sel = torch.randperm(n, generator=torch.Generator().manual_seed(1))[:512].sort().values
    for b in (0, 3):
        for layer in range(2):
            got = cache.export(layer, b, 0, n)
            got = {key: val.cpu()[sel] for key, val in got.items()}
            k, v = dense[(b, layer)]
            c = dense[("dbg", layer)][b * n:(b + 1) * n][sel]
            _check_projection(wl, bases, layer, k.cpu()[sel], v.cpu()[sel], tiers[b].cpu()[sel], c, f"full seq {b}")
            ref = oracle_encode_rows(wl, bases, layer, k.cpu()[sel], v.cpu()[sel], tiers[b].cpu()[sel], c32=c)
            _assert_same(got, ref, tiers[b].cpu()[sel], f"full seq {b} layer {layer}")


def test_decode_over_encoded_cache():
    wl = synth.workload("llama8b_encode_16k").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=2)
    lengths = [900, 257]
    cache, bases, dense, c32 = _encode_case(wl, lengths, chunks=(500, None))
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0)
    out = cache.decode(1, [0, 1], q.cuda())
    err = cache.probe(1, [0, 1], q.cuda())
    cache.sync()
    out, err = out.cpu().numpy(), err.cpu().numpy()
    for b in range(2):
        tiers = dense[(b, "t", 0)]
        comp = oracle_encode_rows(wl, bases, 1, dense[(b, 1)][0], dense[(b, 1)][1], tiers, c32=c32[(b, 1)])
        for h in range(2):
            prob = head_problem(wl, bases, tiers, comp, q[b], 1, h)
            check_close(out[b, h * 4:(h + 1) * 4], oracle.decode_head(prob), what=f"seq {b} head {h}")
            e_ref, _, _ = oracle.probe_head(prob)
            assert abs(err[b, h] - e_ref) <= 2e-3


def test_cuda_graph_replay_of_append_and_decode():
    """One decode step (append one token to each layer, then attend) captured in a CUDA
    graph and replayed: every replay reads the cache state from device memory, so the
    context grows by one token per replay.  Checked against the oracle after each replay."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T0 = 130
    cache = dw.Cache(cfg_for(wl, max_context=T0 + 8), bases[0], bases[1])
    from helpers import import_workload
    data = import_workload(cache, wl, [T0])
    cache.sync()
    steps = 3
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
        cache.append(0, [0], [1], kin, vin, tin, stream=s)
        cache.append(1, [0], [1], kin, vin, None, stream=s)
        cache.decode(1, [0], qin, out=out, stream=s)
    torch.cuda.synchronize()
    tiers, comp = data[(0, 1)]
    for step in range(steps):
        kin.copy_(newk[0][0][step:step + 1]); vin.copy_(newk[0][1][step:step + 1])
        tin.copy_(newt[step:step + 1])
        graph.replay()
        torch.cuda.synchronize()
        new = oracle_encode_rows(wl, bases, 1, newk[0][0][step:step + 1], newk[0][1][step:step + 1],
                                 newt[step:step + 1])
        tiers = torch.cat([tiers, newt[step:step + 1]])
        comp = cat_comp(comp, new)
        ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, qs[0], 1, 0))
        check_close(out[0].cpu().numpy(), ref, what=f"replay {step}")
    cache.sync()


def test_decode_right_after_one_token_appends_across_page_boundaries():
    """The decode launched right after a one-token append may start while the append runs
    (it waits for the placement's counts and reads each tier's last page after the append
    completes).  Step through page boundaries of every tier, eagerly, checking each step."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    T0, steps = 160, 24
    cache = dw.Cache(cfg_for(wl, max_context=T0 + steps + 8), bases[0], bases[1])
    from helpers import import_workload
    data = import_workload(cache, wl, [T0])
    newk = [synth.make_dense_vectors(wl, 0, l, steps, bases, start=T0) for l in range(2)]
    newt = synth.make_tiers(wl, 0, 0, steps, start=T0)
    qs = synth.make_queries(wl, 1, temperature=8.0)
    tiers, comp = data[(0, 1)]
    pages0 = [(int((tiers == k).sum()) + 63) // 64 for k in range(len(wl.tiers))]
    for step in range(steps):
        for layer in range(2):
            cache.append(layer, [0], [1], newk[layer][0][step:step + 1].cuda(), newk[layer][1][step:step + 1].cuda(),
                         newt[step:step + 1].cuda() if layer == 0 else None)
        out = cache.decode(1, [0], qs.cuda())
        cache.sync()
        new = oracle_encode_rows(wl, bases, 1, newk[1][0][step:step + 1], newk[1][1][step:step + 1],
                                 newt[step:step + 1])
        tiers = torch.cat([tiers, newt[step:step + 1]])
        comp = cat_comp(comp, new)
        ref = oracle.decode_head(head_problem(wl, bases, tiers, comp, qs[0], 1, 0))
        check_close(out[0].cpu().numpy(), ref, what=f"step {step}")
    pages1 = [(int((tiers == k).sum()) + 63) // 64 for k in range(len(wl.tiers))]
    assert pages1 != pages0, "the steps should have opened a new page in some tier"


@pytest.mark.parametrize("s,bits", [(0, 8), (32, 4), (32, 8)])
def test_encode_bit_exact_residual_counts(s, bits):
    """Bulk encode with no residual and with the widest one, bit for bit against the oracle."""
    wl = synth.workload("tiny_1k").scaled(resid_channels=s, resid_bits=bits, num_q_heads=8, num_kv_heads=2,
                                          batch=2)
    lengths = [300, 77]
    cache, bases, dense, c32 = _encode_case(wl, lengths)
    for b, T in enumerate(lengths):
        for layer in range(wl.num_layers):
            got = cache.export(layer, b, 0, T)
            tiers = dense[(b, "t", layer // wl.layers_per_group)]
            ref = oracle_encode_rows(wl, bases, layer, dense[(b, layer)][0], dense[(b, layer)][1], tiers,
                                     c32=c32[(b, layer)])
            _assert_same(got, ref, tiers, f"s={s} bits={bits} seq {b} layer {layer}")
