"""Cache bookkeeping on the GPU: import/export round trip (bit-exact), sequence reset and
page reuse, device-side checks that report instead of faulting, and host-side argument
checks that refuse a call before anything is launched."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cfg_for, check_close, head_problem, import_workload, to_dev

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def _expected_export(wl, tiers, comp):
    ranks = synth.ranks_of(wl, tiers.cpu())
    j = torch.arange(wl.r_max).view(1, 1, 1, -1)
    coeff = torch.where(j < ranks.view(*ranks.shape, 1, 1), comp["coeff"].cpu(), torch.zeros((), dtype=torch.bfloat16))
    return coeff


@pytest.mark.parametrize("name", ["tiny_1k", "llama8b_64k", "llama8b_ragged_b8", "llama8b_131k_deep"])
def test_import_export_round_trip(name):
    wl = synth.workload(name)
    wl = wl.scaled(num_layers=wl.layers_per_group, num_q_heads=4 * min(wl.num_kv_heads, 2),
                   num_kv_heads=min(wl.num_kv_heads, 2), batch=2)
    lengths = [333, 1000]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1024), bases[0], bases[1])
    data = import_workload(cache, wl, lengths, garbage=True)
    for (b, layer), (tiers, comp) in data.items():
        got = cache.export(layer, b, 0, lengths[b])
        assert torch.equal(got["tier_idx"].cpu(), tiers)
        assert torch.equal(got["coeff"].cpu().view(torch.int16), _expected_export(wl, tiers, comp).view(torch.int16))
        assert torch.equal(got["idx"].cpu(), comp["idx"])
        assert torch.equal(got["codes"].cpu(), comp["codes"])
        assert torch.equal(got["scales"].cpu().view(torch.int16), comp["scales"].view(torch.int16))
        part = cache.export(layer, b, 17, 40)
        assert torch.equal(part["codes"].cpu(), comp["codes"][17:57])


def test_incremental_import_matches_bulk():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, num_q_heads=8, num_kv_heads=2, batch=1)
    bases = synth.make_bases(wl)
    T = 500
    tiers = synth.make_tiers(wl, 0, 0, T)
    comps = [synth.make_compressed(wl, 0, l, tiers) for l in range(2)]
    cache = dw.Cache(cfg_for(wl, max_context=T), bases[0], bases[1])
    # layer 0 in uneven chunks, layer 1 in one call (its tiers come from layer 0's placement)
    a = 0
    for n in (1, 63, 64, 65, 7, 300):
        c = to_dev({k: v[a:a + n] for k, v in comps[0].items()})
        cache.append_compressed(0, [0], [n], tiers[a:a + n].cuda().contiguous(), c["coeff"], c["idx"], c["codes"], c["scales"])
        a += n
    c = to_dev(comps[1])
    cache.append_compressed(1, [0], [T], None, c["coeff"], c["idx"], c["codes"], c["scales"])
    cache.sync()
    for l in range(2):
        got = cache.export(l, 0, 0, T)
        assert torch.equal(got["tier_idx"].cpu(), tiers)
        assert torch.equal(got["codes"].cpu(), comps[l]["codes"])
    q = synth.make_queries(wl, 1, batch=1, temperature=8.0)
    out = cache.decode(1, [0], q.cuda()).cpu().numpy()
    for h in range(2):
        check_close(out[0, 4 * h:4 * h + 4], oracle.decode_head(head_problem(wl, bases, tiers, comps[1], q[0], 1, h)))


def test_reset_reuses_pages_and_stays_correct():
    wl = synth.workload("tiny_1k").scaled(batch=2)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=1024), bases[0], bases[1])
    import_workload(cache, wl, [1000, 500])
    used = cache.pool_usage()["data_bytes_reserved"]
    for rnd in range(3):
        cache.reset(0)
        assert cache.seq_length(0, 0) == 0
        data = import_workload(cache, wl, [600], seed=50 + rnd)
        assert cache.pool_usage()["data_bytes_reserved"] == used   # pages came from the free rings
        q = synth.make_queries(wl, 0, batch=1, seed=50 + rnd, temperature=8.0)
        out = cache.decode(0, [0], q.cuda()).cpu().numpy()
        tiers, comp = data[(0, 0)]
        check_close(out[0], oracle.decode_head(head_problem(wl, bases, tiers, comp, q[0], 0, 0)))
    cache.sync()


def test_device_checks_report_instead_of_faulting():
    wl = synth.workload("tiny_1k").scaled(resid_bits=4)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=256), bases[0], bases[1])
    tiers = synth.make_tiers(wl, 0, 0, 10)
    comp = to_dev(synth.make_compressed(wl, 0, 0, tiers))
    bad = tiers.clone()
    bad[3, 0] = 7                                   # tier index out of range
    cache.append_compressed(0, [0], [10], bad.cuda(), comp["coeff"], comp["idx"], comp["codes"], comp["scales"])
    with pytest.raises(dw.DwkvError, match="tier index"):
        cache.sync()
    cache.sync()                                    # the word was cleared
    cache.reset(0)
    codes = comp["codes"].clone()
    codes[0, 0, 0, 0] = 9                           # not an int4 value
    cache.append_compressed(0, [0], [10], tiers.cuda(), comp["coeff"], comp["idx"], codes, comp["scales"])
    with pytest.raises(dw.DwkvError, match="int4"):
        cache.sync()
    cache.reset(0)
    idx = comp["idx"].clone()
    idx[1, 0, 1, 2] = 200                           # channel beyond head_dim
    cache.append_compressed(0, [0], [10], tiers.cuda(), comp["coeff"], idx, comp["codes"], comp["scales"])
    with pytest.raises(dw.DwkvError, match="channel"):
        cache.sync()


def test_pool_exhaustion_is_reported():
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    cfg = cfg_for(wl, max_context=4096)
    small = dw.dwkv_metadata_bytes(cfg) + 3 * dw.dwkv_page_bytes(cfg, 2)
    cache = dw.Cache(cfg, bases[0], bases[1], arena_bytes=(small + 255) // 256 * 256)
    tiers = synth.make_tiers(wl, 0, 0, 2000)
    comp = to_dev(synth.make_compressed(wl, 0, 0, tiers))
    cache.append_compressed(0, [0], [2000], tiers.cuda(), comp["coeff"], comp["idx"], comp["codes"], comp["scales"])
    with pytest.raises(dw.DwkvError, match="pool exhausted"):
        cache.sync()


def test_host_side_checks():
    wl = synth.workload("tiny_1k").scaled(batch=2)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=100), bases[0], bases[1])
    tiers = synth.make_tiers(wl, 0, 0, 50)
    comp = to_dev(synth.make_compressed(wl, 0, 0, tiers))
    cache.append_compressed(0, [0], [50], tiers.cuda(), comp["coeff"], comp["idx"], comp["codes"], comp["scales"])
    q = synth.make_queries(wl, 1, batch=1).cuda()
    with pytest.raises(dw.DwkvError, match="append every layer"):
        cache.decode(1, [0], q)                     # layer 1 not appended yet
    with pytest.raises(dw.DwkvError, match="DWKV_ERR_CAPACITY"):
        cache.append_compressed(0, [0], [60], tiers.cuda(), comp["coeff"], comp["idx"], comp["codes"], comp["scales"])
    with pytest.raises(dw.DwkvError, match="listed twice"):
        cache.decode(0, [0, 0], torch.cat([q, q]))
    with pytest.raises(dw.DwkvError, match="out of"):
        cache.decode(0, [5], q)
    with pytest.raises(dw.DwkvError, match="tier_idx is NULL"):
        cache.append_compressed(0, [1], [5], None, comp["coeff"], comp["idx"], comp["codes"], comp["scales"])
    small_ws = torch.empty(16, dtype=torch.float32, device="cuda")
    out = torch.empty(1, 4, 128, device="cuda")
    with pytest.raises(dw.DwkvError, match="workspace"):
        dw.dwkv_decode_attention(cache.h, 0, [0], q, out, small_ws)
    with pytest.raises(dw.DwkvError, match="positions"):
        cache.export(0, 0, 40, 20)
    cache.decode(0, [], q[:0])                      # empty call is a no-op
    cache.sync()


def test_bounded_wait_runs_out_reports_and_leaves_the_context_usable():
    """A wait that nothing ends: the kernels' bounded-wait routine gives up after its limit
    (20 ms here), the error word says so through dwkv_sync_status, and decoding afterwards is
    unaffected (the word is cleared by the report)."""
    wl = synth.workload("tiny_1k")
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl), bases[0], bases[1])
    data = import_workload(cache, wl, [500])
    cache.sync()
    dw.dwkv_check_bounded_wait(cache.h, 20000)
    with pytest.raises(dw.DwkvError, match="bounded wait timed out"):
        cache.sync()
    cache.sync()                                    # cleared
    q = synth.make_queries(wl, 0, temperature=8.0)
    out = cache.decode(0, [0], q.cuda())
    cache.sync()
    tiers, comp = data[(0, 0)]
    check_close(out[0].cpu().numpy(), oracle.decode_head(head_problem(wl, bases, tiers, comp, q[0], 0, 0)))
    with pytest.raises(dw.DwkvError, match="limit_us"):
        dw.dwkv_check_bounded_wait(cache.h, 0)
