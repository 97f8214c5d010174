"""dwkv_decode_attention_noalloc: decode for callers that cannot allocate device memory
when they decode (engine plugin hooks, serving loops whose pool owns all of HBM) and have
no workspace to lend.  It uses scratch built into the library image; its output must match
dwkv_decode_attention (which uses a caller workspace) on two calls in a row.

This file is named so that pytest collects it last."""
import numpy as np
import pytest
import torch

import synth
from helpers import cfg_for, check_close, import_workload

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


def test_noalloc_decode_matches_workspace_decode_twice():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, batch=2)
    lengths = [3000, 1234]
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=3072), bases[0], bases[1])
    import_workload(cache, wl, lengths)
    q = synth.make_queries(wl, 1, batch=2, temperature=8.0).cuda()
    ref = cache.decode(1, [0, 1], q)
    outs = []
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        dw.dwkv_decode_attention_noalloc(cache.h, 1, [0, 1], q, out)
        cache.sync()
        outs.append(out.cpu().numpy())
    ref = ref.cpu().numpy()
    for out in outs:
        assert np.isfinite(out).all()
        check_close(out, ref, what="no-allocation decode vs workspace decode")


def test_noalloc_rejects_calls_beyond_its_scratch():
    wl = synth.workload("llama8b_ragged_b8").scaled(num_layers=2, batch=8)
    bases = synth.make_bases(wl)
    cache = dw.Cache(cfg_for(wl, max_context=128), bases[0], bases[1])
    import_workload(cache, wl, [100] * 8)
    q = synth.make_queries(wl, 0, batch=8).cuda()
    out = torch.empty(8, wl.num_q_heads, wl.head_dim, device="cuda")
    with pytest.raises(dw.DwkvError, match="built-in scratch"):
        dw.dwkv_decode_attention_noalloc(cache.h, 0, list(range(8)), q, out)
    cache.sync()
