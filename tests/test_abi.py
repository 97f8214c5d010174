"""The C-ABI library loads, exports every symbol its header declares, and validates
arguments on the host before touching a GPU (these tests run without one)."""
import ctypes as C
import os
import re

import pytest
import torch

import decode_attention_depthweave_b200 as dw
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "dwkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dwkv_[a-z_]+)\s*\(", text)))


def test_header_declarations_are_exported():
    L = C.CDLL(dw.LIB_PATH)
    names = _declared()
    assert "dwkv_decode_attention" in names and "dwkv_probe" in names and "dwkv_create" in names
    for n in names:
        assert hasattr(L, n), n
    assert sorted(dw.EXPORTED_SYMBOLS) == names


def _cfg(wl, **over):
    kw = dict(num_layers=wl.num_layers, layers_per_group=wl.layers_per_group, num_q_heads=wl.num_q_heads,
              num_kv_heads=wl.num_kv_heads, head_dim=wl.head_dim, r_max=wl.r_max, tiers=wl.tiers,
              resid_channels=wl.resid_channels, resid_bits=wl.resid_bits, max_batch=wl.batch,
              max_context=wl.context + 64, tier_resid=wl.tier_resid or None, coeff_bits=wl.coeff_bits)
    kw.update(over)
    return dw.config_from(**kw)


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_configs_are_supported(name):
    assert dw.dwkv_config_check(_cfg(synth.workload(name))) == 0, dw.dwkv_last_error()


@pytest.mark.parametrize("over,status", [
    (dict(num_layers=3), 1), (dict(head_dim=64), 5), (dict(num_q_heads=16), 5), (dict(r_max=12), 1),
    (dict(r_max=48, tiers=(16, 32)), 5), (dict(tiers=(16, 16)), 1), (dict(tiers=(8, 24)), 5), (dict(tiers=(16, 128)), 1),
    (dict(resid_channels=12), 1), (dict(resid_channels=24), 5), (dict(resid_bits=2), 1), (dict(max_batch=0), 1),
    (dict(max_context=1 << 24), 1),
])
def test_invalid_configs_are_rejected(over, status):
    cfg = _cfg(synth.workload("llama8b_64k"), **over)
    assert dw.dwkv_config_check(cfg) == status
    assert dw.dwkv_last_error()


def test_token_and_page_bytes():
    cfg = _cfg(synth.workload("llama8b_64k"))
    # one token, one layer, one kv-head, K + V: 2 * (2 r + s + s*bits/8 + 2)
    assert [dw.dwkv_token_bytes(cfg, k) for k in range(3)] == [2 * (2 * r + 16 + 8 + 2) for r in (16, 32, 64)]
    assert dw.dwkv_token_bytes(cfg, 3) == 0
    for k, r in enumerate((16, 32, 64)):
        # two layers x (K + V) blocks, then the 64 slots' positions (int32)
        assert dw.dwkv_page_bytes(cfg, k) == 2 * 2 * (128 * r + 64 * 16 + 8 * 16 * 4 + 128) + 64 * 4
        assert dw.dwkv_page_bytes(cfg, k) % 128 == 0
    # room for every tier at its largest (re-tiering): metadata + pages of every tier
    G = cfg.num_layers // cfg.layers_per_group
    pages = (cfg.max_context + 63) // 64 + 1
    want = dw.dwkv_metadata_bytes(cfg) + cfg.max_batch * G * cfg.num_kv_heads * pages * sum(
        dw.dwkv_page_bytes(cfg, k) for k in range(cfg.num_tiers))
    assert dw.dwkv_arena_bytes_all_tiers(cfg) == want
    meta = dw.dwkv_metadata_bytes(cfg)
    assert 0 < meta < dw.dwkv_arena_bytes(cfg)
    assert dw.dwkv_workspace_bytes(cfg, 8) == 8 * dw.dwkv_workspace_bytes(cfg, 1)


@pytest.mark.parametrize("over", [
    dict(tier_resid=(0, 2, 4, 8), tiers=(32, 32, 32, 16)),      # routed tiers share one rank
    dict(tier_resid=(0, 2, 3, 8)),                              # counts in {0, 2, 4, 8}
    dict(tier_resid=(0, 4, 2, 8)),                              # strictly ascending
    dict(tier_resid=(0, 2, 4, 8), resid_channels=16),           # array stride 8
])
def test_invalid_routed_configs_are_rejected(over):
    cfg = _cfg(synth.workload("llama8b_routed_64k"), **over)
    assert dw.dwkv_config_check(cfg) == 1
    assert dw.dwkv_last_error()


def test_routed_token_and_page_bytes():
    """Per-tier residual counts: 2 * (2 r + rho + rho * bits / 8 + 2) bytes a token; a page's
    code part is padded to 128 bytes."""
    cfg = _cfg(synth.workload("llama8b_routed_64k"))
    assert [dw.dwkv_token_bytes(cfg, k) for k in range(4)] == [2 * (64 + n + n // 2 + 2) for n in (0, 2, 4, 8)]
    for k, n in enumerate((0, 2, 4, 8)):
        code = (8 * n * 4 + 127) // 128 * 128
        assert dw.dwkv_page_bytes(cfg, k) == 2 * 2 * (128 * 32 + 64 * n + code + 128) + 64 * 4


@pytest.mark.parametrize("over", [
    dict(coeff_bits=8, tiers=(8, 16, 32), r_max=32),            # whole blocks of 16
    dict(coeff_bits=8, tiers=(8,), r_max=8),                    # r_max a multiple of 16
    dict(coeff_bits=4),
    dict(coeff_bits=32),
])
def test_invalid_coefficient_widths_are_rejected(over):
    cfg = _cfg(synth.workload("llama8b_64k"), **over)
    assert dw.dwkv_config_check(cfg) == 1
    assert dw.dwkv_last_error()


def test_8bit_coefficient_token_and_page_bytes():
    """8-bit coefficients: r codes + r/16 fp16 scales a vector (r + r/8 bytes); a page block
    holds 72 r bytes of them (1 KB of codes and 128 bytes of scales per block of 16)."""
    cfg = _cfg(synth.workload("llama8b_64k_c8"))
    assert cfg.coeff_bits == 8 and dw.dwkv_config_check(cfg) == 0
    assert [dw.dwkv_token_bytes(cfg, k) for k in range(3)] == [2 * (r + r // 8 + 16 + 8 + 2) for r in (16, 32, 64)]
    for k, r in enumerate((16, 32, 64)):
        assert dw.dwkv_page_bytes(cfg, k) == 2 * 2 * (72 * r + 64 * 16 + 8 * 16 * 4 + 128) + 64 * 4
        assert dw.dwkv_page_bytes(cfg, k) % 128 == 0
    bf = _cfg(synth.workload("llama8b_64k"))
    assert all(dw.dwkv_page_bytes(cfg, k) < dw.dwkv_page_bytes(bf, k) for k in range(3))


def test_create_rejects_bad_arguments_without_a_gpu():
    cfg = _cfg(synth.workload("tiny_1k"))
    h = C.c_void_p()
    L = dw.lib()
    assert L.dwkv_create(C.byref(cfg), None, 0, None, None, None, C.byref(h)) == 1
    assert "non-NULL" in dw.dwkv_last_error()
    bad = _cfg(synth.workload("tiny_1k"), resid_bits=3)
    assert L.dwkv_create(C.byref(bad), C.c_void_p(256), 1 << 20, C.c_void_p(256), C.c_void_p(256), None,
                         C.byref(h)) == 1
    assert L.dwkv_create(C.byref(cfg), C.c_void_p(257), 1 << 20, C.c_void_p(256), C.c_void_p(256), None,
                         C.byref(h)) == 1
    assert "aligned" in dw.dwkv_last_error()
    assert h.value is None


def test_null_handle_calls_fail_cleanly():
    L = dw.lib()
    assert L.dwkv_destroy(None) == 1
    assert L.dwkv_sync_status(None, None) == 1
    assert L.dwkv_decode_attention(None, 0, 0, None, None, None, None, 0, None) == 1
    assert L.dwkv_append(None, 0, 0, None, None, None, None, None, None, None) == 1


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "decode_attention_depthweave_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f


def test_test_support_entries_validate_on_the_host():
    """The test-support calls refuse bad arguments before any launch (so without a GPU)."""
    L = dw.lib()
    assert L.dwkv_check_bounded_wait(None, 1000, None) == 1
    r = C.c_void_p(256)
    # s must be a multiple of 8 in 0..128, bits 8 or 4, pointers non-NULL, work large enough
    assert L.dwkv_quantize_residuals(4, 12, 8, r, r, r, r, r, 1 << 20, None) == 1
    assert "multiple of 8" in dw.dwkv_last_error()
    assert L.dwkv_quantize_residuals(4, 16, 6, r, r, r, r, r, 1 << 20, None) == 1
    assert L.dwkv_quantize_residuals(4, 16, 8, None, r, r, r, r, 1 << 20, None) == 1
    need = dw.dwkv_quantize_work_bytes(4, 16, 8)
    assert need > 0 and need % 16 == 0
    assert L.dwkv_quantize_residuals(4, 16, 8, r, r, r, r, r, need - 16, None) == 1
    assert "needs" in dw.dwkv_last_error()
    assert L.dwkv_quantize_residuals(0, 16, 8, None, None, None, None, None, 0, None) == 0   # nothing to do
    # one page-layout block a vector: s idx bytes, then the codes at 64 s, the scale at 64 s + 8 s b
    for s, b in ((16, 4), (32, 8), (0, 8)):
        per = (64 * s + 8 * s * b + 2 + 15) // 16 * 16
        assert dw.dwkv_quantize_work_bytes(3, s, b) == 3 * per
    assert dw.dwkv_quantize_work_bytes(3, 16, 5) == 0
