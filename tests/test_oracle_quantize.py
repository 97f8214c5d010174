"""The oracle's encode steps 4-6 on given residuals (top-s selection with ties to the lower
channel, fp16 scale, symmetric codes; "DepthWeave-KV", §3 Method, the routed residual
channels) against a brute-force restatement of the same definition in numpy: a full sort
by (-|r|, channel), IEEE fp32 division, round-to-nearest-even to fp16 and rint.  The inputs
stress the selection boundary (one-ulp and exact ties at rank s, zeros, subnormals, scale
overflow, half-step codes)."""
import numpy as np
import pytest

import oracle
import synth


def brute_force(r, s, bits):
    qmax = np.float32(127 if bits == 8 else 7)
    mag = np.abs(r.astype(np.float32))
    order = sorted(range(r.shape[0]), key=lambda i: (-float(mag[i]), i))
    sel = sorted(order[:s])
    amax = np.float32(max((mag[i] for i in sel), default=np.float32(0)))
    with np.errstate(over="ignore"):
        scale = np.float16(np.float32(amax) / qmax)
    sf = np.float32(scale)
    codes = []
    for i in sel:
        c = np.float32(0)
        if sf != 0:
            with np.errstate(divide="ignore", invalid="ignore"):
                c = np.float32(np.rint(np.float32(r[i]) / sf))
            c = min(max(c, -qmax), qmax)
        codes.append(int(c))
    return np.array(sel, np.uint8), np.array(codes, np.int8), np.array([scale], np.float16).view(np.uint16)[0]


@pytest.mark.parametrize("s,bits", [(8, 8), (16, 4), (32, 8), (0, 4), (128, 4)])
def test_quantize_residual_matches_brute_force(s, bits):
    cases = synth.make_residual_cases(180, 128, max(s, 1))
    for v, r in enumerate(cases):
        got = oracle.quantize_residual(r, s, bits)
        idx, codes, scale = brute_force(r, s, bits)
        kind = synth.RESIDUAL_CASE_KINDS[v % len(synth.RESIDUAL_CASE_KINDS)]
        assert np.array_equal(got["idx"], idx), (v, kind)
        assert np.array_equal(got["codes"], codes), (v, kind)
        assert got["scale"] == scale, (v, kind)


def test_half_steps_round_to_even():
    """An int4 scale of exactly 1 (amax 7): r = 2.5 -> 2, 3.5 -> 4, -0.5 -> -0 (code 0)."""
    r = np.zeros(128, np.float32)
    r[[3, 9, 40, 77]] = [7.0, 2.5, 3.5, -0.5]
    got = oracle.quantize_residual(r, 8, 4)
    assert got["scale"] == np.array([1.0], np.float16).view(np.uint16)[0]
    sel = dict(zip(got["idx"].tolist(), got["codes"].tolist()))
    assert sel[3] == 7 and sel[9] == 2 and sel[40] == 4 and sel[77] == 0
    # the four zeros that fill the selection are the lowest zero channels
    assert [c for c in got["idx"].tolist() if c not in (3, 9, 40, 77)] == [0, 1, 2, 4]
