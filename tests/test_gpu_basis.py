"""Online bases through the C ABI against the oracle ("DepthWeave-KV ...", §3 Method, the
shared-bases paragraph): the window's second moment (tensor-core Gram, fp32) against the fp64
Gram of the same rows; the sketched basis against the oracle's sketch of the same moment and
test matrix (column by column up to bf16 rounding where the eigenvalues are separated); encode
and decode on the sketched basis; the moving-average update (moment, refreshed basis) and the
re-projection of every stored token onto it, bit for bit against the oracle's re-encode with
the previous and the new basis; decode after it."""
import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import basis as ob
from helpers import cat_comp, cfg_for, check_close, head_problem, oracle_encode_rows, to_dev

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _wl(**kw):
    wl = synth.workload("llama8b_encode_16k").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=2)
    return wl.scaled(**kw) if kw else wl


def _rows(wl, bases, lengths, start=0):
    """Dense rows of the window's two layers: per layer (K, V) bf16 [sum n][H][d], sequences in
    order, and the stacked [LPG][sum n][H][d] arrays the sketch takes."""
    per_layer = []
    for layer in range(wl.num_layers):
        ks, vs = [], []
        for b, n in enumerate(lengths):
            k, v = synth.make_dense_vectors(wl, b, layer, n, bases, start=start)
            ks.append(k)
            vs.append(v)
        per_layer.append((torch.cat(ks), torch.cat(vs)))
    k_rows = torch.stack([p[0] for p in per_layer]).contiguous()
    v_rows = torch.stack([p[1] for p in per_layer]).contiguous()
    return per_layer, k_rows, v_rows


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


def _check_basis(b_gpu, b_or, w_or, what):
    """Columns whose eigenvalue is separated from its neighbours by > 1e-4 relative agree to
    bf16 rounding (up to sign); every column is unit norm to bf16 rounding."""
    r = b_gpu.shape[1]
    bo = b_or.astype(np.float64)
    for j in range(r):
        lo = abs(w_or[j] - w_or[j - 1]) if j > 0 else np.inf
        hi = abs(w_or[j] - w_or[j + 1]) if j + 1 < r else np.inf
        assert abs(np.linalg.norm(b_gpu[:, j]) - 1.0) < 2e-3, (what, j)
        if min(lo, hi) <= 1e-4 * abs(w_or[j]):
            continue
        d = min(np.abs(b_gpu[:, j] - bo[:, j]).max(), np.abs(b_gpu[:, j] + bo[:, j]).max())
        assert d <= 2.0 ** -8 * np.abs(bo[:, j]).max() + 1e-6, (what, j, d)


def _sketch(cache, wl, k_rows, v_rows, omega):
    eig = cache.basis_sketch(0, k_rows.cuda(), v_rows.cuda(), omega.cuda(), power_steps=2)
    bk, bv = cache.bases(0)
    mom = cache.moment(0)
    cache.sync()
    return eig.cpu(), (bk.cpu(), bv.cpu()), mom.cpu()


def test_sketch_moment_and_basis_match_the_oracle():
    wl = _wl()
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1100), bases[0], bases[1])
    lengths = [700, 500]
    _, k_rows, v_rows = _rows(wl, bases, lengths)
    omega = synth.make_test_matrix(wl)
    eig, (bk, bv), mom = _sketch(cache, wl, k_rows, v_rows, omega)
    for h in range(wl.num_kv_heads):
        for z, rows in enumerate((k_rows, v_rows)):
            x = _f64(rows[:, :, h].reshape(-1, wl.head_dim))
            c_or = ob.gram(x)
            c_gpu = mom[h, z].numpy().astype(np.float64)
            assert np.linalg.norm(c_gpu - c_or) <= 1e-5 * np.linalg.norm(c_or), (h, z)
            # the basis from the GPU's own moment (isolates the sketch from the Gram's rounding)
            b_or, w_or = ob.sketch_basis(c_gpu, omega.numpy().astype(np.float64), power_steps=2)
            b_gpu = _f64((bk, bv)[z][h])
            _check_basis(b_gpu, b_or, w_or, f"head {h} z {z}")
            assert np.allclose(eig[h, z].numpy(), w_or, rtol=1e-5, atol=1e-6 * w_or[0]), (h, z)


def test_encode_and_decode_on_a_sketched_basis():
    wl = _wl()
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1100), bases[0], bases[1])
    lengths = [600, 257]
    per_layer, k_rows, v_rows = _rows(wl, bases, lengths)
    _, (bk, bv), _ = _sketch(cache, wl, k_rows, v_rows, synth.make_test_matrix(wl))
    nb = (bk.unsqueeze(0), bv.unsqueeze(0))                      # [G=1][H][d][r]
    tiers = [synth.make_tiers(wl, b, 0, n) for b, n in enumerate(lengths)]
    for layer in range(2):
        k, v = per_layer[layer]
        dbg = torch.full((k.shape[0], wl.num_kv_heads, 2, wl.r_max), float("nan"), device="cuda")
        cache.append(layer, [0, 1], lengths, k.cuda(), v.cuda(), torch.cat(tiers).cuda() if layer == 0 else None,
                     coeff_dbg=dbg)
        cache.sync()
        o = 0
        for b, n in enumerate(lengths):
            got = cache.export(layer, b, 0, n)
            ref = oracle_encode_rows(wl, nb, layer, k[o:o + n], v[o:o + n], tiers[b], c32=dbg[o:o + n].cpu())
            for key in ("coeff", "idx", "codes", "scales"):
                assert torch.equal(got[key].cpu().contiguous().view(torch.uint8), ref[key].contiguous().view(torch.uint8)), \
                    (layer, b, key)
            o += n
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0)
    out = cache.decode(1, [0, 1], q.cuda())
    cache.sync()
    for b in range(2):
        comp = cache.export(1, b, 0, lengths[b])
        comp = {k_: v_.cpu() for k_, v_ in comp.items() if k_ != "tier_idx"}
        for h in range(wl.num_kv_heads):
            ref = oracle.decode_head(head_problem(wl, nb, tiers[b], comp, q[b], 1, h))
            check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"seq {b} head {h}")


@pytest.mark.parametrize("beta", [0.9, 0.0])
def test_update_refreshes_the_basis_and_reprojects_the_cache(beta):
    wl = _wl()
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1100), bases[0], bases[1])
    lengths = [400, 222]
    per_layer, k_rows, v_rows = _rows(wl, bases, lengths)
    _, (bk0, bv0), mom0 = _sketch(cache, wl, k_rows, v_rows, synth.make_test_matrix(wl))
    tiers = [synth.make_tiers(wl, b, 0, n) for b, n in enumerate(lengths)]
    for layer in range(2):
        k, v = per_layer[layer]
        cache.append(layer, [0, 1], lengths, k.cuda(), v.cuda(), torch.cat(tiers).cuda() if layer == 0 else None)
    cache.sync()
    before = {(b, layer): cache.export(layer, b, 0, n) for b, n in enumerate(lengths) for layer in range(2)}
    # new rows (later positions, another distribution: a different seed), then the update
    wl2 = wl.scaled(base_seed=wl.base_seed + 77)
    _, k_new, v_new = _rows(wl2, synth.make_bases(wl2), [300], start=2000)
    eig = cache.basis_update(0, k_new.cuda(), v_new.cuda(), beta, [0, 1])
    bk1, bv1 = cache.bases(0)
    mom1 = cache.moment(0)
    cache.sync()
    bk1, bv1, mom1, eig = bk1.cpu(), bv1.cpu(), mom1.cpu(), eig.cpu()
    for h in range(wl.num_kv_heads):
        for z, rows in enumerate((k_new, v_new)):
            c_rows = ob.gram(_f64(rows[:, :, h].reshape(-1, wl.head_dim)))
            want = ob.ema(mom0[h, z].numpy().astype(np.float64), c_rows, beta)
            got = mom1[h, z].numpy().astype(np.float64)
            assert np.linalg.norm(got - want) <= 1e-5 * np.linalg.norm(want), (h, z)
            b_or, w_or = ob.refresh_basis(got, _f64((bk0, bv0)[z][h]))
            _check_basis(_f64((bk1, bv1)[z][h]), b_or, w_or, f"update head {h} z {z}")
            assert np.allclose(eig[h, z].numpy(), w_or, rtol=1e-5, atol=1e-6 * w_or[0]), (h, z)
    # every stored token re-projected: the oracle's re-encode on the previous and the new basis
    s = wl.resid_channels
    for (b, layer), old in before.items():
        got = cache.export(layer, b, 0, lengths[b])
        assert torch.equal(got["tier_idx"].cpu(), old["tier_idx"].cpu())
        oc = {k_: v_.cpu() for k_, v_ in old.items()}
        for t in range(0, lengths[b], 7):                       # every 7th token, every head, K and V
            for h in range(wl.num_kv_heads):
                r = wl.tiers[int(oc["tier_idx"][t, h])]
                for z in range(2):
                    ref = oracle.reencode_vector((bk0, bv0)[z][h], r, oc["coeff"][t, h, z], oc["idx"][t, h, z],
                                                 oc["codes"][t, h, z], oc["scales"][t, h, z], r, wl.resid_bits,
                                                 s_new=s, basis_new=(bk1, bv1)[z][h])
                    gc = got["coeff"][t, h, z].cpu().view(torch.int16).numpy().view(np.uint16)
                    assert np.array_equal(gc, ref["coeff"]), (b, layer, t, h, z)
                    assert np.array_equal(got["idx"][t, h, z].cpu().numpy(), ref["idx"]), (b, layer, t, h, z)
                    assert np.array_equal(got["codes"][t, h, z].cpu().numpy(), ref["codes"]), (b, layer, t, h, z)
                    assert (int(got["scales"][t, h, z].cpu().view(torch.int16).item()) & 0xffff) == int(ref["scale"])
    # decode over the re-projected cache, on the new bases
    nb = (bk1.unsqueeze(0), bv1.unsqueeze(0))
    q = synth.make_queries(wl, 0, batch=2, temperature=8.0)
    out = cache.decode(0, [0, 1], q.cuda())
    cache.sync()
    for b in range(2):
        comp = {k_: v_.cpu() for k_, v_ in cache.export(0, b, 0, lengths[b]).items() if k_ != "tier_idx"}
        for h in range(wl.num_kv_heads):
            ref = oracle.decode_head(head_problem(wl, nb, tiers[b], comp, q[b], 0, h))
            check_close(out[b, h * 4:(h + 1) * 4].cpu().numpy(), ref, what=f"after update seq {b} head {h}")


def test_basis_calls_refuse_bad_arguments():
    wl = _wl()
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=600), bases[0], bases[1])
    _, k_rows, v_rows = _rows(wl, bases, [100])
    omega = synth.make_test_matrix(wl).cuda()
    with pytest.raises(dw.DwkvError):
        dw.dwkv_basis_sketch(cache.h, 1, 100, k_rows.cuda(), v_rows.cuda(), omega)     # one group only
    with pytest.raises(dw.DwkvError):
        dw.dwkv_basis_sketch(cache.h, 0, 100, k_rows.cuda(), v_rows.cuda(), None)
    with pytest.raises(dw.DwkvError):
        dw.dwkv_basis_update(cache.h, 0, 0, None, None, 1.5, [0])
    # a sequence whose layers hold different positions
    k, v = synth.make_dense_vectors(wl, 0, 0, 50, bases)
    cache.append(0, [0], [50], k.cuda(), v.cuda(), synth.make_tiers(wl, 0, 0, 50).cuda())
    cache.sync()
    with pytest.raises(dw.DwkvError, match="same positions"):
        dw.dwkv_basis_update(cache.h, 0, 0, None, None, 0.5, [0])
    # online bases need r_max <= 64
    big = synth.workload("llama8b_131k_deep").scaled(num_layers=4, num_q_heads=8, num_kv_heads=2, context=256)
    bb = synth.make_bases(big)
    c2 = dw.Cache(cfg_for(big), bb[0], bb[1])
    kr = torch.zeros(4, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dw.DwkvError):
        dw.dwkv_basis_sketch(c2.h, 0, 16, kr, kr, torch.zeros(128, 128, device="cuda"))


def test_every_window_in_one_call():
    """DWKV_ALL_GROUPS: one launch sketches (and updates) every window from all layers' rows;
    each window's moment and basis match the oracle as for a single window, and the update
    re-projects the tokens of every window."""
    wl = _wl(num_layers=4)                                       # two windows of two layers
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=700), bases[0], bases[1])
    lengths = [300, 199]
    per_layer, k_rows, v_rows = _rows(wl, bases, lengths)       # [4][n][H][d]
    omega = synth.make_test_matrix(wl)
    eig = cache.basis_sketch(dw.DWKV_ALL_GROUPS, k_rows.cuda(), v_rows.cuda(), omega.cuda(), power_steps=2)
    cache.sync()
    assert eig.shape[0] == 2
    bw = {}
    for g in range(2):
        bk, bv = cache.bases(g)
        mom = cache.moment(g)
        cache.sync()
        bw[g] = (bk.cpu(), bv.cpu())
        for h in range(wl.num_kv_heads):
            for z, rows in enumerate((k_rows, v_rows)):
                x = _f64(rows[2 * g:2 * g + 2, :, h].reshape(-1, wl.head_dim))
                c_gpu = mom[h, z].cpu().numpy().astype(np.float64)
                c_or = ob.gram(x)
                assert np.linalg.norm(c_gpu - c_or) <= 1e-5 * np.linalg.norm(c_or), (g, h, z)
                b_or, w_or = ob.sketch_basis(c_gpu, omega.numpy().astype(np.float64), power_steps=2)
                _check_basis(_f64(bw[g][z][h]), b_or, w_or, f"window {g} head {h} z {z}")
    tiers = {g: [synth.make_tiers(wl, b, g, n) for b, n in enumerate(lengths)] for g in range(2)}
    for layer in range(4):
        k, v = per_layer[layer]
        g = layer // 2
        cache.append(layer, [0, 1], lengths, k.cuda(), v.cuda(), torch.cat(tiers[g]).cuda() if layer % 2 == 0 else None)
    cache.sync()
    before = {(b, layer): cache.export(layer, b, 0, lengths[b]) for b in range(2) for layer in (1, 2)}
    cache.basis_update(dw.DWKV_ALL_GROUPS, k_rows[:, :64].contiguous().cuda(), v_rows[:, :64].contiguous().cuda(),
                       0.5, [0, 1])
    cache.sync()
    new = {g: tuple(t.cpu() for t in cache.bases(g)) for g in range(2)}
    cache.sync()
    for (b, layer), old in before.items():
        g = layer // 2
        got = cache.export(layer, b, 0, lengths[b])
        oc = {k_: v_.cpu() for k_, v_ in old.items()}
        for t in range(0, lengths[b], 23):
            for h in range(wl.num_kv_heads):
                r = wl.tiers[int(oc["tier_idx"][t, h])]
                for z in range(2):
                    ref = oracle.reencode_vector(bw[g][z][h], r, oc["coeff"][t, h, z], oc["idx"][t, h, z],
                                                 oc["codes"][t, h, z], oc["scales"][t, h, z], r, wl.resid_bits,
                                                 basis_new=new[g][z][h])
                    gc = got["coeff"][t, h, z].cpu().view(torch.int16).numpy().view(np.uint16)
                    assert np.array_equal(gc, ref["coeff"]), (b, layer, t, h, z)
                    assert np.array_equal(got["idx"][t, h, z].cpu().numpy(), ref["idx"]), (b, layer, t, h, z)


def test_update_before_any_sketch_averages_from_zero():
    """A window's moment starts at zero: an update without a sketch gives (1 - beta) C_rows."""
    wl = _wl()
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=300), bases[0], bases[1])
    _, k_rows, v_rows = _rows(wl, bases, [200])
    cache.basis_update(0, k_rows.cuda(), v_rows.cuda(), 0.75, [])
    mom = cache.moment(0)
    cache.sync()
    for h in range(wl.num_kv_heads):
        for z, rows in enumerate((k_rows, v_rows)):
            want = 0.25 * ob.gram(_f64(rows[:, :, h].reshape(-1, wl.head_dim)))
            got = mom[h, z].cpu().numpy().astype(np.float64)
            assert np.linalg.norm(got - want) <= 1e-5 * np.linalg.norm(want), (h, z)


@pytest.mark.parametrize("coeff_bits", [16, 8])
def test_update_reprojects_tokens_with_repeated_residual_channels(coeff_bits):
    """Stored tokens whose residual entries repeat a channel (the format allows it; decode sums
    them): the re-projection adds such a token's entries one at a time in entry order, as the
    oracle's reconstruction does, and the other tokens of its warp's group by the scatter.
    Every token, head and side is checked bit for bit."""
    wl = _wl(coeff_bits=coeff_bits)
    bases = synth.make_bases(wl)
    lengths = [300, 150]
    cache = dw.Cache(cfg_for(wl, max_context=400), bases[0], bases[1])
    for seq, T in enumerate(lengths):
        tiers = synth.make_tiers(wl, seq, 0, T)
        for layer in range(2):
            comp = synth.make_compressed(wl, seq, layer, tiers)
            idx = comp["idx"].clone()
            idx[::3, :, :, 1] = idx[::3, :, :, 0]          # every third token: entry 1 repeats entry 0's
            idx[::3, :, :, -1] = idx[::3, :, :, 2]         # channel, the last entry repeats entry 2's
            comp["idx"] = idx
            c = to_dev(comp)
            coeff = (c["ccodes"], c["cscales"]) if "ccodes" in c else c["coeff"]
            cache.append_compressed(layer, [seq], [T], tiers.cuda().contiguous(), coeff, c["idx"], c["codes"],
                                    c["scales"])
    cache.sync()
    before = {(b, layer): {k_: v_.cpu() for k_, v_ in cache.export(layer, b, 0, n).items()}
              for b, n in enumerate(lengths) for layer in range(2)}
    assert (before[(0, 0)]["idx"][0, 0, 0, 1] == before[(0, 0)]["idx"][0, 0, 0, 0]).item()
    wl2 = wl.scaled(base_seed=wl.base_seed + 55)
    _, k_new, v_new = _rows(wl2, synth.make_bases(wl2), [200], start=1000)
    cache.basis_update(0, k_new.cuda(), v_new.cuda(), 0.0, [0, 1])
    bk1, bv1 = cache.bases(0)
    cache.sync()
    new = (bk1.cpu(), bv1.cpu())
    old = (bases[0][0], bases[1][0])
    for (b, layer), oc in before.items():
        got = {k_: v_.cpu() for k_, v_ in cache.export(layer, b, 0, lengths[b]).items()}
        for t in range(lengths[b]):
            for h in range(wl.num_kv_heads):
                r = wl.tiers[int(oc["tier_idx"][t, h])]
                for z in range(2):
                    what = (b, layer, t, h, z)
                    args = (oc["idx"][t, h, z], oc["codes"][t, h, z], oc["scales"][t, h, z], r, wl.resid_bits)
                    if coeff_bits == 8:
                        ref = oracle.reencode_vector8(old[z][h], r, oc["ccodes"][t, h, z], oc["cscales"][t, h, z], *args,
                                                      basis_new=new[z][h])
                        assert np.array_equal(got["ccodes"][t, h, z].numpy(), ref["ccodes"]), what
                        assert np.array_equal(got["cscales"][t, h, z].view(torch.int16).numpy().view(np.uint16),
                                              ref["cscales"]), what
                    else:
                        ref = oracle.reencode_vector(old[z][h], r, oc["coeff"][t, h, z], *args, basis_new=new[z][h])
                        assert np.array_equal(got["coeff"][t, h, z].view(torch.int16).numpy().view(np.uint16),
                                              ref["coeff"]), what
                    assert np.array_equal(got["idx"][t, h, z].numpy(), ref["idx"]), what
                    assert np.array_equal(got["codes"][t, h, z].numpy(), ref["codes"]), what
                    assert (int(got["scales"][t, h, z].view(torch.int16).item()) & 0xffff) == int(ref["scale"]), what


@pytest.mark.parametrize("n_rows", [1, 7, 65, 1000])
def test_moment_of_few_and_ragged_rows(n_rows):
    """An update whose rows a layer leave a partial chunk of 64 (rows past the end staged as
    zeros) or less than one chunk in all: C = 0.5 C_0 + 0.5 C_rows against the fp64 Gram of the
    same rows, C_0 a sketched full-rank moment (a missing or doubled row would move C by far
    more than the bound); an update with no rows only scales the moment."""
    wl = _wl()
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=64), bases[0], bases[1])
    _, k0, v0 = _rows(wl, bases, [200])
    _, _, mom0 = _sketch(cache, wl, k0, v0, synth.make_test_matrix(wl))
    wl2 = wl.scaled(base_seed=wl.base_seed + 3)
    _, k_rows, v_rows = _rows(wl2, synth.make_bases(wl2), [n_rows], start=500)
    cache.basis_update(0, k_rows.cuda(), v_rows.cuda(), 0.5, [])
    mom = cache.moment(0)
    cache.sync()
    mom = mom.cpu()
    for h in range(wl.num_kv_heads):
        for z, rows in enumerate((k_rows, v_rows)):
            g = 0.5 * ob.gram(_f64(rows[:, :, h].reshape(-1, wl.head_dim)))
            want = 0.5 * mom0[h, z].numpy().astype(np.float64) + g
            got = mom[h, z].numpy().astype(np.float64)
            assert np.linalg.norm(got - want) <= 1e-5 * np.linalg.norm(want), (n_rows, h, z)
            assert np.linalg.norm(g) > 1e-3 * np.linalg.norm(want)          # the rows' share is visible
    cache.basis_update(0, None, None, 0.5, [])
    mom2 = cache.moment(0)
    cache.sync()
    assert torch.equal(mom2.cpu(), 0.5 * mom)
