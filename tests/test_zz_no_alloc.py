"""dwkv_decode_attention_noalloc: decode for callers that cannot allocate device memory
when they decode (engine plugin hooks, serving loops whose pool owns all of HBM) and have
no workspace to lend.  It uses scratch built into the library image; its output must match
the oracle and dwkv_decode_attention (which uses a caller workspace) on two calls in a row.

The file is named so that pytest collects it last: a run that stops at the first failure has
then run every other test before this one.  No test depends on that order; the entry point
resolves its scratch address on its first call in any process, fresh or not."""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import cfg_for, check_close, head_problem, import_workload

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def test_noalloc_decode_matches_oracle_and_workspace_decode_twice():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, batch=2)
    lengths = [3000, 1234]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=3072), bases[0], bases[1])
    data = import_workload(cache, wl, lengths)
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0)
    ref = cache.decode(1, [0, 1], q.cuda())
    outs = []
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        dw.dwkv_decode_attention_noalloc(cache.h, 1, [0, 1], q.cuda(), out)
        cache.sync()
        outs.append(out.cpu().numpy())
    ref = ref.cpu().numpy()
    for out in outs:
        assert np.isfinite(out).all()
        check_close(out, ref, what="no-allocation decode vs workspace decode")
        for b in range(2):
            tiers, comp = data[(b, 1)]
            for h in range(wl.num_kv_heads):
                exp = oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], 1, h))
                check_close(out[b, h * 4:(h + 1) * 4], exp, what=f"no-allocation decode seq {b} head {h}")


def test_noalloc_capacity_edge_seven_sequences_accepted_eight_refused():
    """8 kv heads, head_dim 128: a sequence's records take 8 x 64 x 520 floats, so the 8 MiB
    scratch holds 7 sequences per call and refuses 8."""
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, batch=8)
    assert wl.num_kv_heads == 8
    bases = synth.make_bases(wl)
    lengths = [100 + 37 * b for b in range(8)]
    cache = dw.Cache(cfg_for(wl, max_context=512), bases[0], bases[1])
    data = import_workload(cache, wl, lengths)
    q = synth.make_queries(wl, 0, batch=8, temperature=8.0)
    out = torch.full((8, wl.num_q_heads, wl.head_dim), float("nan"), device="cuda")
    dw.dwkv_decode_attention_noalloc(cache.h, 0, list(range(7)), q[:7].cuda().contiguous(), out[:7])
    cache.sync()
    got = out.cpu().numpy()
    for b in range(7):
        tiers, comp = data[(b, 0)]
        for h in (0, wl.num_kv_heads - 1):
            exp = oracle.decode_head(head_problem(wl, bases, tiers, comp, q[b], 0, h))
            check_close(got[b, h * 4:(h + 1) * 4], exp, what=f"7-sequence call seq {b} head {h}")
    with pytest.raises(dw.DwkvError, match="built-in scratch"):
        dw.dwkv_decode_attention_noalloc(cache.h, 0, list(range(8)), q.cuda(), out)
    cache.sync()
