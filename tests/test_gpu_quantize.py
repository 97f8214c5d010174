"""Encode steps 4-6 on the GPU (the device code every encoder runs, through
dwkv_quantize_residuals) against the oracle on the same residuals, bit for bit: selected
channels, codes and fp16 scales.  The residuals stress the selection boundary: one-ulp and
exact ties at rank s (where the device's fast selection hands over to the exact one),
zeros, subnormals, fp16 scale overflow and half-step codes."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

dw = pytest.importorskip("decode_attention_depthweave_b200")


@pytest.mark.parametrize("s,bits", [(16, 4), (8, 8), (32, 8), (128, 4), (0, 8), (24, 4)])
def test_quantize_matches_oracle(s, bits):
    cases = synth.make_residual_cases(9 * 300, 128, max(s, 1))
    idx, codes, scales = dw.dwkv_quantize_residuals(torch.from_numpy(cases).cuda(), s, bits)
    torch.cuda.synchronize()
    idx, codes, scales = idx.cpu().numpy(), codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16)
    for v, r in enumerate(cases):
        ref = oracle.quantize_residual(r, s, bits)
        kind = synth.RESIDUAL_CASE_KINDS[v % len(synth.RESIDUAL_CASE_KINDS)]
        assert np.array_equal(idx[v], ref["idx"]), (v, kind, idx[v], ref["idx"])
        assert np.array_equal(codes[v], ref["codes"]), (v, kind, codes[v], ref["codes"])
        assert scales[v] == ref["scale"], (v, kind, scales[v], ref["scale"])


def test_quantize_rejects_bad_arguments():
    r = torch.zeros(4, 128, device="cuda")
    with pytest.raises(dw.DwkvError, match="multiple of 8"):
        dw.dwkv_quantize_residuals(r, 12, 8)
    with pytest.raises(dw.DwkvError, match="bits"):
        dw.dwkv_quantize_residuals(r, 16, 6)
