"""The probe-driven router threshold (host code of libdwkv, no GPU): the schedule of
"DepthWeave-KV ...", §3 -- tau_m is lowered when a probe's error exceeds the tolerance and
raised after several quiet probe intervals, within [tau_min, tau_max] -- pinned on trajectories
worked out by hand from that rule, and the two-level routing of Eq. (2)."""
import math

import numpy as np
import pytest

import decode_attention_depthweave_b200 as dw


def _policy(**kw):
    p = dict(tol=0.05, tau_init=0.6, tau_min=0.2, tau_max=0.9, tau_step_down=0.1, tau_step_up=0.05,
             quiet_intervals=3, probe_every=4)
    p.update(kw)
    pol = dw.dwkv_tier_policy()
    for k, v in p.items():
        setattr(pol, k, v)
    return pol


def test_threshold_follows_the_probe_errors():
    c = dw.dwkv_tier_controller_create(_policy(), 2)
    try:
        # (error, lowered?, tau after) worked by hand: tol 0.05, down 0.1, up 0.05 after 3 quiet
        steps = [
            (0.10, True, 0.5),    # over tol: lower
            (0.02, False, 0.5),   # quiet 1
            (0.05, False, 0.5),   # quiet 2 (equal to tol is quiet)
            (0.01, False, 0.55),  # quiet 3: raise, count restarts
            (0.00, False, 0.55),  # quiet 1
            (0.30, True, 0.45),   # over: lower, count restarts
            (0.01, False, 0.45),  # quiet 1
            (0.01, False, 0.45),  # quiet 2
            (0.20, True, 0.35),   # over before the third quiet probe: no raise
            (0.20, True, 0.25),
            (0.20, True, 0.2),    # clamped at tau_min
            (0.20, True, 0.2),
        ]
        for i, (err, low, tau) in enumerate(steps):
            assert dw.dwkv_tier_controller_observe(c, 0, err) is low, i
            assert dw.dwkv_tier_controller_threshold(c, 0) == pytest.approx(tau, abs=1e-6), i
        # the other group never moved
        assert dw.dwkv_tier_controller_threshold(c, 1) == pytest.approx(0.6)
    finally:
        dw.dwkv_tier_controller_destroy(c)


def test_threshold_rises_to_tau_max_and_stays():
    c = dw.dwkv_tier_controller_create(_policy(tau_init=0.8, quiet_intervals=1, tau_step_up=0.07), 1)
    try:
        seen = [dw.dwkv_tier_controller_observe(c, 0, 0.0) or dw.dwkv_tier_controller_threshold(c, 0)
                for _ in range(4)]
        assert seen == pytest.approx([0.87, 0.9, 0.9, 0.9], abs=1e-6)
    finally:
        dw.dwkv_tier_controller_destroy(c)


def test_probe_cadence():
    c = dw.dwkv_tier_controller_create(_policy(probe_every=4), 1)
    try:
        assert [dw.dwkv_tier_controller_due(c, s) for s in range(10)] == [s % 4 == 0 for s in range(10)]
        assert dw.dwkv_tier_controller_due(c, -1) is False
    finally:
        dw.dwkv_tier_controller_destroy(c)


def test_route_is_the_two_level_rule_with_the_current_threshold():
    c = dw.dwkv_tier_controller_create(_policy(tau_init=0.5), 1)
    try:
        sal = np.array([0.1, 0.5, 0.500001, 0.9, 0.7, 0.99], np.float32)
        base = np.array([0, 0, 1, 2, 0, 2], np.uint8)
        # strictly above tau and below the high tier: raised to it; otherwise kept
        assert list(dw.dwkv_tier_controller_route(c, 0, sal, base, 2)) == [0, 0, 2, 2, 2, 2]
        dw.dwkv_tier_controller_observe(c, 0, 1.0)                      # tau 0.5 -> 0.4
        assert list(dw.dwkv_tier_controller_route(c, 0, np.float32([0.45, 0.35]), np.uint8([0, 1]), 1)) == [1, 1]
    finally:
        dw.dwkv_tier_controller_destroy(c)


@pytest.mark.parametrize("bad", [dict(tau_min=0.7), dict(tau_init=1.0), dict(quiet_intervals=0), dict(probe_every=0),
                                 dict(tol=-1.0), dict(tau_step_down=-0.1), dict(tau_max=math.inf)])
def test_invalid_policies_are_refused(bad):
    with pytest.raises(dw.DwkvError):
        dw.dwkv_tier_controller_create(_policy(**bad), 1)


def test_nan_error_and_bad_group_are_refused():
    c = dw.dwkv_tier_controller_create(_policy(), 1)
    try:
        with pytest.raises(dw.DwkvError):
            dw.dwkv_tier_controller_observe(c, 0, float("nan"))
        with pytest.raises(dw.DwkvError):
            dw.dwkv_tier_controller_observe(c, 1, 0.0)
        assert dw.dwkv_tier_controller_threshold(c, 0) == pytest.approx(0.6)
    finally:
        dw.dwkv_tier_controller_destroy(c)
