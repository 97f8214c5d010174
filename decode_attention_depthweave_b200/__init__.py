"""Python binding of libdwkv: decode attention read directly from a DepthWeave-KV
compressed KV cache on a B200 ("DepthWeave-KV: Token-Adaptive Cross-Layer Residual
Factorization for Long-Context KV Cache Compression", §3 Method).

Argument marshalling only.  Every step of the hot path runs in the CUDA kernels of
``_lib/libdwkv.so``; the functions below have the names of the C ABI in
``include/dwkv.h`` and take torch tensors (device pointers are passed through) or host
integer lists.  PyTorch provides device memory and streams, nothing else.  There is no
CPU fallback: importing this package fails if the library has not been built.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

__all__ = [
    "DwkvError", "dwkv_config", "lib", "config_from", "dwkv_version", "dwkv_last_error",
    "dwkv_config_check", "dwkv_token_bytes", "dwkv_page_bytes", "dwkv_metadata_bytes",
    "dwkv_arena_bytes", "dwkv_workspace_bytes", "dwkv_create", "dwkv_destroy",
    "dwkv_reset_sequence", "dwkv_seq_length", "dwkv_append", "dwkv_append_gated", "dwkv_append_compressed",
    "dwkv_decode_attention", "dwkv_probe", "dwkv_export", "dwkv_pool_usage",
    "dwkv_sync_status", "dwkv_set_decode_tuning", "dwkv_decode_attention_noalloc", "dwkv_append_decode_attention",
    "dwkv_quantize_work_bytes", "dwkv_quantize_residuals", "dwkv_check_bounded_wait", "dwkv_set_decode_overlap",
    "dwkv_retier", "dwkv_tier_policy", "dwkv_tier_controller_create", "dwkv_tier_controller_destroy",
    "dwkv_tier_controller_due", "dwkv_tier_controller_threshold", "dwkv_tier_controller_observe",
    "dwkv_tier_controller_route", "dwkv_arena_bytes_all_tiers", "dwkv_basis_sketch", "dwkv_basis_update",
    "dwkv_get_bases", "dwkv_get_moment", "DWKV_ALL_GROUPS", "Cache", "EXPORTED_SYMBOLS",
    "pack_coeff8", "unpack_coeff8",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libdwkv.so")

DWKV_OK = 0
DWKV_ALL_GROUPS = -1
STATUS_NAMES = {0: "DWKV_OK", 1: "DWKV_ERR_INVALID_ARG", 2: "DWKV_ERR_CAPACITY", 3: "DWKV_ERR_CUDA",
                4: "DWKV_ERR_DEVICE_CHECK", 5: "DWKV_ERR_UNSUPPORTED"}

EXPORTED_SYMBOLS = (
    "dwkv_version", "dwkv_last_error", "dwkv_config_check", "dwkv_token_bytes", "dwkv_page_bytes",
    "dwkv_metadata_bytes", "dwkv_arena_bytes", "dwkv_workspace_bytes", "dwkv_create", "dwkv_destroy",
    "dwkv_reset_sequence", "dwkv_seq_length", "dwkv_append", "dwkv_append_gated", "dwkv_append_compressed",
    "dwkv_decode_attention", "dwkv_probe", "dwkv_export", "dwkv_pool_usage", "dwkv_sync_status",
    "dwkv_set_decode_tuning", "dwkv_decode_attention_noalloc", "dwkv_append_decode_attention",
    "dwkv_quantize_work_bytes", "dwkv_quantize_residuals", "dwkv_check_bounded_wait", "dwkv_set_decode_overlap",
    "dwkv_retier", "dwkv_tier_controller_create", "dwkv_tier_controller_destroy", "dwkv_tier_controller_due",
    "dwkv_tier_controller_threshold", "dwkv_tier_controller_observe", "dwkv_tier_controller_route",
    "dwkv_arena_bytes_all_tiers", "dwkv_basis_sketch", "dwkv_basis_update", "dwkv_get_bases", "dwkv_get_moment",
)


class DwkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


class dwkv_config(C.Structure):
    _fields_ = [
        ("num_layers", C.c_int32), ("layers_per_group", C.c_int32), ("num_q_heads", C.c_int32),
        ("num_kv_heads", C.c_int32), ("head_dim", C.c_int32), ("r_max", C.c_int32),
        ("num_tiers", C.c_int32), ("tiers", C.c_int32 * 8), ("resid_channels", C.c_int32),
        ("resid_bits", C.c_int32), ("max_batch", C.c_int32), ("max_context", C.c_int32),
        ("softmax_scale", C.c_float), ("resid_routed", C.c_int32), ("tier_resid", C.c_int32 * 8),
        ("coeff_bits", C.c_int32),
    ]


class dwkv_tier_policy(C.Structure):
    _fields_ = [("tol", C.c_float), ("tau_init", C.c_float), ("tau_min", C.c_float), ("tau_max", C.c_float),
                ("tau_step_down", C.c_float), ("tau_step_up", C.c_float), ("quiet_intervals", C.c_int32),
                ("probe_every", C.c_int32)]


class dwkv_pool_stats(C.Structure):
    _fields_ = [("data_bytes_total", C.c_uint64), ("data_bytes_reserved", C.c_uint64),
                ("free_pages", C.c_uint32 * 8)]


_LIB = None


def lib():
    """The loaded libdwkv (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libdwkv is not built ({LIB_PATH} missing); run "
                              "`python -m decode_attention_depthweave_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
        cfgp = C.POINTER(dwkv_config)
        sig = {
            "dwkv_version": ([], C.c_char_p),
            "dwkv_last_error": ([], C.c_char_p),
            "dwkv_config_check": ([cfgp], C.c_int),
            "dwkv_token_bytes": ([cfgp, i32], sz),
            "dwkv_page_bytes": ([cfgp, i32], sz),
            "dwkv_metadata_bytes": ([cfgp], sz),
            "dwkv_arena_bytes": ([cfgp], sz),
            "dwkv_arena_bytes_all_tiers": ([cfgp], sz),
            "dwkv_workspace_bytes": ([cfgp, i32], sz),
            "dwkv_create": ([cfgp, vp, sz, vp, vp, vp, C.POINTER(vp)], C.c_int),
            "dwkv_destroy": ([vp], C.c_int),
            "dwkv_reset_sequence": ([vp, i32, vp], C.c_int),
            "dwkv_seq_length": ([vp, i32, i32, C.POINTER(i32)], C.c_int),
            "dwkv_append": ([vp, i32, i32, vp, vp, vp, vp, vp, vp, vp], C.c_int),
            "dwkv_append_gated": ([vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp], C.c_int),
            "dwkv_append_compressed": ([vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp], C.c_int),
            "dwkv_decode_attention": ([vp, i32, i32, vp, vp, vp, vp, sz, vp], C.c_int),
            "dwkv_append_decode_attention": ([vp, i32, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp], C.c_int),
            "dwkv_probe": ([vp, i32, i32, vp, vp, vp, vp, vp, sz, vp], C.c_int),
            "dwkv_export": ([vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp], C.c_int),
            "dwkv_pool_usage": ([vp, vp, C.POINTER(dwkv_pool_stats)], C.c_int),
            "dwkv_sync_status": ([vp, vp], C.c_int),
            "dwkv_set_decode_tuning": ([vp, i32, i32, i32], C.c_int),
            "dwkv_decode_attention_noalloc": ([vp, i32, i32, vp, vp, vp, vp], C.c_int),
            "dwkv_quantize_work_bytes": ([i32, i32, i32], sz),
            "dwkv_quantize_residuals": ([i32, i32, i32, vp, vp, vp, vp, vp, sz, vp], C.c_int),
            "dwkv_check_bounded_wait": ([vp, C.c_uint32, vp], C.c_int),
            "dwkv_set_decode_overlap": ([vp, i32], C.c_int),
            "dwkv_retier": ([vp, i32, i32, vp, vp, vp, vp, vp], C.c_int),
            "dwkv_basis_sketch": ([vp, i32, i32, vp, vp, vp, i32, vp, vp], C.c_int),
            "dwkv_basis_update": ([vp, i32, i32, vp, vp, C.c_float, i32, vp, vp, vp], C.c_int),
            "dwkv_get_bases": ([vp, i32, vp, vp, vp], C.c_int),
            "dwkv_get_moment": ([vp, i32, vp, vp], C.c_int),
            "dwkv_tier_controller_create": ([C.POINTER(dwkv_tier_policy), i32, C.POINTER(vp)], C.c_int),
            "dwkv_tier_controller_destroy": ([vp], C.c_int),
            "dwkv_tier_controller_due": ([vp, C.c_int64], i32),
            "dwkv_tier_controller_threshold": ([vp, i32, C.POINTER(C.c_float)], C.c_int),
            "dwkv_tier_controller_observe": ([vp, i32, C.c_float, C.POINTER(i32)], C.c_int),
            "dwkv_tier_controller_route": ([vp, i32, i32, vp, vp, i32, vp], C.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _LIB = L
    return _LIB


def _check(status: int):
    if status != DWKV_OK:
        raise DwkvError(status, dwkv_last_error())


def _ptr(t):
    """Device / host pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("tensors passed to libdwkv must be contiguous")
        return C.c_void_p(t.data_ptr())
    return t


def _i32(xs):
    arr = (C.c_int32 * max(len(xs), 1))(*[int(x) for x in xs])
    return arr


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def config_from(num_layers, layers_per_group, num_q_heads, num_kv_heads, head_dim, r_max, tiers,
                resid_channels, resid_bits, max_batch, max_context, softmax_scale=0.0,
                tier_resid=None, coeff_bits=16) -> dwkv_config:
    """tier_resid: per-tier residual channel counts (residual-count routing; every tier then has
    the same rank and resid_channels is 8), or None for one count, resid_channels, everywhere.
    coeff_bits: 16 (bf16 coefficients) or 8 (int8 codes with an fp16 scale per block of 16)."""
    c = dwkv_config()
    c.coeff_bits = int(coeff_bits)
    if tier_resid is not None:
        c.resid_routed = 1
        for k, n in enumerate(tier_resid):
            c.tier_resid[k] = int(n)
    c.num_layers, c.layers_per_group = num_layers, layers_per_group
    c.num_q_heads, c.num_kv_heads, c.head_dim, c.r_max = num_q_heads, num_kv_heads, head_dim, r_max
    c.num_tiers = len(tiers)
    for k, r in enumerate(tiers):
        c.tiers[k] = int(r)
    c.resid_channels, c.resid_bits = resid_channels, resid_bits
    c.max_batch, c.max_context, c.softmax_scale = max_batch, max_context, float(softmax_scale)
    return c


# ------------------------------------------------------------------------------ C ABI
def dwkv_version() -> str:
    return lib().dwkv_version().decode()


def dwkv_last_error() -> str:
    return lib().dwkv_last_error().decode()


def dwkv_config_check(cfg: dwkv_config) -> int:
    return lib().dwkv_config_check(C.byref(cfg))


def dwkv_token_bytes(cfg, tier) -> int:
    return lib().dwkv_token_bytes(C.byref(cfg), tier)


def dwkv_page_bytes(cfg, tier) -> int:
    return lib().dwkv_page_bytes(C.byref(cfg), tier)


def dwkv_metadata_bytes(cfg) -> int:
    return lib().dwkv_metadata_bytes(C.byref(cfg))


def dwkv_arena_bytes(cfg) -> int:
    return lib().dwkv_arena_bytes(C.byref(cfg))


def dwkv_arena_bytes_all_tiers(cfg) -> int:
    return lib().dwkv_arena_bytes_all_tiers(C.byref(cfg))


def dwkv_workspace_bytes(cfg, n_seqs) -> int:
    return lib().dwkv_workspace_bytes(C.byref(cfg), n_seqs)


def dwkv_create(cfg, arena: torch.Tensor, basis_k: torch.Tensor, basis_v: torch.Tensor, stream=None,
                arena_bytes=None) -> C.c_void_p:
    h = C.c_void_p()
    nbytes = arena.numel() * arena.element_size() if arena_bytes is None else arena_bytes
    _check(lib().dwkv_create(C.byref(cfg), _ptr(arena), nbytes, _ptr(basis_k), _ptr(basis_v),
                             _stream(stream), C.byref(h)))
    return h


def dwkv_destroy(h):
    _check(lib().dwkv_destroy(h))


def dwkv_reset_sequence(h, seq, stream=None):
    _check(lib().dwkv_reset_sequence(h, seq, _stream(stream)))


def dwkv_seq_length(h, seq, layer) -> int:
    v = C.c_int32()
    _check(lib().dwkv_seq_length(h, seq, layer, C.byref(v)))
    return v.value


def dwkv_append(h, layer, seq_ids, n_new, k_new, v_new, tier_idx, coeff_dbg=None, stream=None):
    _check(lib().dwkv_append(h, layer, len(seq_ids), _i32(seq_ids), _i32(n_new), _ptr(k_new), _ptr(v_new),
                             _ptr(tier_idx), _ptr(coeff_dbg), _stream(stream)))


def dwkv_append_gated(h, layer, seq_ids, n_new, k_new, v_new, tier_idx, gate, coeff_dbg=None, stream=None):
    _check(lib().dwkv_append_gated(h, layer, len(seq_ids), _i32(seq_ids), _i32(n_new), _ptr(k_new), _ptr(v_new),
                                   _ptr(tier_idx), _ptr(gate), _ptr(coeff_dbg), _stream(stream)))


def dwkv_append_compressed(h, layer, seq_ids, n_new, tier_idx, coeff, idx, codes, scales, stream=None):
    _check(lib().dwkv_append_compressed(h, layer, len(seq_ids), _i32(seq_ids), _i32(n_new), _ptr(tier_idx),
                                        _ptr(coeff), _ptr(idx), _ptr(codes), _ptr(scales), _stream(stream)))


def dwkv_decode_attention(h, layer, seq_ids, q, out, workspace, stream=None):
    _check(lib().dwkv_decode_attention(h, layer, len(seq_ids), _i32(seq_ids), _ptr(q), _ptr(out),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)))


def dwkv_append_decode_attention(h, layer, seq_ids, k_new, v_new, tier_idx, q, out, workspace, stream=None):
    _check(lib().dwkv_append_decode_attention(h, layer, len(seq_ids), _i32(seq_ids), _ptr(k_new), _ptr(v_new),
                                              _ptr(tier_idx), _ptr(q), _ptr(out), _ptr(workspace),
                                              workspace.numel() * workspace.element_size(), _stream(stream)))


def dwkv_decode_attention_noalloc(h, layer, seq_ids, q, out, stream=None):
    _check(lib().dwkv_decode_attention_noalloc(h, layer, len(seq_ids), _i32(seq_ids), _ptr(q), _ptr(out),
                                               _stream(stream)))


def dwkv_probe(h, layer, seq_ids, q, err, out_full, workspace, stream=None):
    _check(lib().dwkv_probe(h, layer, len(seq_ids), _i32(seq_ids), _ptr(q), _ptr(err), _ptr(out_full),
                            _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def dwkv_check_bounded_wait(h, limit_us, stream=None):
    _check(lib().dwkv_check_bounded_wait(h, int(limit_us), _stream(stream)))


def dwkv_quantize_work_bytes(n, s, bits) -> int:
    return int(lib().dwkv_quantize_work_bytes(n, s, bits))


def dwkv_quantize_residuals(r, s, bits, stream=None):
    """Encode steps 4-6 on residuals r (device fp32 [n][128]): (idx uint8 [n][s], codes int8
    [n][s], scales fp16 bits as int16 [n]), all on r's device."""
    n = r.shape[0]
    dev = r.device
    idx = torch.empty(n, s, dtype=torch.uint8, device=dev)
    codes = torch.empty(n, s, dtype=torch.int8, device=dev)
    scales = torch.empty(n, dtype=torch.int16, device=dev)
    work = torch.empty(max(dwkv_quantize_work_bytes(n, s, bits), 16), dtype=torch.uint8, device=dev)
    _check(lib().dwkv_quantize_residuals(n, s, bits, _ptr(r), _ptr(idx), _ptr(codes), _ptr(scales), _ptr(work),
                                         work.numel(), _stream(stream)))
    return idx, codes, scales


def dwkv_export(h, layer, seq, t0, n, tier_idx=None, coeff=None, idx=None, codes=None, scales=None, stream=None):
    _check(lib().dwkv_export(h, layer, seq, t0, n, _ptr(tier_idx), _ptr(coeff), _ptr(idx), _ptr(codes),
                             _ptr(scales), _stream(stream)))


def dwkv_pool_usage(h, stream=None) -> dict:
    s = dwkv_pool_stats()
    _check(lib().dwkv_pool_usage(h, _stream(stream), C.byref(s)))
    return {"data_bytes_total": s.data_bytes_total, "data_bytes_reserved": s.data_bytes_reserved,
            "free_pages": list(s.free_pages)}


def dwkv_sync_status(h, stream=None):
    _check(lib().dwkv_sync_status(h, _stream(stream)))


def dwkv_set_decode_tuning(h, ctas_per_sm=1, waves=1, stages=0):
    _check(lib().dwkv_set_decode_tuning(h, ctas_per_sm, waves, stages))


def dwkv_set_decode_overlap(h, enable):
    _check(lib().dwkv_set_decode_overlap(h, int(enable)))


def dwkv_retier(h, group, seq_ids, n_tok, positions, new_tier, stream=None):
    _check(lib().dwkv_retier(h, group, len(seq_ids), _i32(seq_ids), _i32(n_tok), _ptr(positions), _ptr(new_tier),
                             _stream(stream)))


def dwkv_basis_sketch(h, group, n_rows, k_rows, v_rows, omega, power_steps=2, eigenvalues=None, stream=None):
    _check(lib().dwkv_basis_sketch(h, group, n_rows, _ptr(k_rows), _ptr(v_rows), _ptr(omega), int(power_steps),
                                   _ptr(eigenvalues), _stream(stream)))


def dwkv_basis_update(h, group, n_rows, k_rows, v_rows, beta, seq_ids, eigenvalues=None, stream=None):
    _check(lib().dwkv_basis_update(h, group, n_rows, _ptr(k_rows), _ptr(v_rows), float(beta), len(seq_ids),
                                   _i32(seq_ids), _ptr(eigenvalues), _stream(stream)))


def dwkv_get_bases(h, group, basis_k, basis_v, stream=None):
    _check(lib().dwkv_get_bases(h, group, _ptr(basis_k), _ptr(basis_v), _stream(stream)))


def dwkv_get_moment(h, group, moment, stream=None):
    _check(lib().dwkv_get_moment(h, group, _ptr(moment), _stream(stream)))


def dwkv_tier_controller_create(policy: dwkv_tier_policy, num_groups: int) -> C.c_void_p:
    c = C.c_void_p()
    _check(lib().dwkv_tier_controller_create(C.byref(policy), num_groups, C.byref(c)))
    return c


def dwkv_tier_controller_destroy(c):
    _check(lib().dwkv_tier_controller_destroy(c))


def dwkv_tier_controller_due(c, step) -> bool:
    return bool(lib().dwkv_tier_controller_due(c, int(step)))


def dwkv_tier_controller_threshold(c, group) -> float:
    v = C.c_float()
    _check(lib().dwkv_tier_controller_threshold(c, group, C.byref(v)))
    return v.value


def dwkv_tier_controller_observe(c, group, err) -> bool:
    low = C.c_int32()
    _check(lib().dwkv_tier_controller_observe(c, group, float(err), C.byref(low)))
    return bool(low.value)


def dwkv_tier_controller_route(c, group, salience, base_tier, high_tier):
    """Host arrays: salience float32 [n], base_tier uint8 [n] -> tier uint8 [n] (numpy)."""
    import numpy as np
    sal = np.ascontiguousarray(salience, np.float32)
    base = np.ascontiguousarray(base_tier, np.uint8)
    out = np.empty_like(base)
    _check(lib().dwkv_tier_controller_route(c, group, sal.size, sal.ctypes.data_as(C.c_void_p),
                                            base.ctypes.data_as(C.c_void_p), int(high_tier),
                                            out.ctypes.data_as(C.c_void_p)))
    return out


# ------------------------------------------------------------------------------ plumbing
def pack_coeff8(codes: torch.Tensor, scales: torch.Tensor) -> torch.Tensor:
    """Coefficient records of the 8-bit form, uint8 [..][r_max + r_max / 8]: the int8 codes
    [..][r_max], then the fp16 block scales [..][r_max / 16] (byte marshalling only)."""
    return torch.cat([codes.contiguous().view(torch.uint8), scales.contiguous().view(torch.uint8)], dim=-1).contiguous()


def unpack_coeff8(records: torch.Tensor, r_max: int):
    """(codes int8 [..][r_max], scales fp16 [..][r_max / 16]) of packed coefficient records."""
    return (records[..., :r_max].contiguous().view(torch.int8),
            records[..., r_max:].contiguous().view(torch.float16))


class Cache:
    """Owns the torch allocations around one handle (arena and workspace) and exposes the
    C ABI calls with tensors.  Allocation is torch's; computation is libdwkv's."""

    def __init__(self, cfg: dwkv_config, basis_k: torch.Tensor, basis_v: torch.Tensor, device="cuda",
                 arena_bytes=None, ws_seqs=None, stream=None):
        if not torch.cuda.is_available():
            raise RuntimeError("libdwkv needs a CUDA device")
        _check(dwkv_config_check(cfg))
        self.cfg = cfg
        self.device = torch.device(device)
        nbytes = dwkv_arena_bytes(cfg) if arena_bytes is None else int(arena_bytes)
        self.arena = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        ws = dwkv_workspace_bytes(cfg, ws_seqs or cfg.max_batch)
        self.workspace = torch.empty((ws + 15) // 16 * 4, dtype=torch.float32, device=self.device)
        self.h = dwkv_create(cfg, self.arena, basis_k.to(self.device).contiguous(),
                             basis_v.to(self.device).contiguous(), stream)

    def close(self):
        if getattr(self, "h", None):
            dwkv_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def append(self, layer, seq_ids, n_new, k_new, v_new, tier_idx, stream=None, coeff_dbg=None, gate=None):
        """gate: optional fp32 [sum(n_new)][Hkv][2] residual gates (dwkv_append_gated)."""
        if gate is not None:
            dwkv_append_gated(self.h, layer, seq_ids, n_new, k_new, v_new, tier_idx, gate, coeff_dbg, stream)
        else:
            dwkv_append(self.h, layer, seq_ids, n_new, k_new, v_new, tier_idx, coeff_dbg, stream)

    def append_compressed(self, layer, seq_ids, n_new, tier_idx, coeff, idx, codes, scales, stream=None):
        """coeff: bf16 [n][Hkv][2][r_max], or with 8-bit coefficients the pair (codes int8
        [n][Hkv][2][r_max], block scales fp16 [n][Hkv][2][r_max / 16]) or its packed records."""
        if isinstance(coeff, (tuple, list)):
            coeff = pack_coeff8(*coeff)
        dwkv_append_compressed(self.h, layer, seq_ids, n_new, tier_idx, coeff, idx, codes, scales, stream)

    def decode(self, layer, seq_ids, q, out=None, stream=None):
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        dwkv_decode_attention(self.h, layer, seq_ids, q, out, self.workspace, stream)
        return out

    def append_decode(self, layer, seq_ids, k_new, v_new, tier_idx, q, out=None, stream=None):
        """One new token per sequence appended and attended in one launch."""
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        dwkv_append_decode_attention(self.h, layer, seq_ids, k_new, v_new, tier_idx, q, out, self.workspace, stream)
        return out

    def probe(self, layer, seq_ids, q, want_out=False, stream=None):
        err = torch.empty(len(seq_ids), self.cfg.num_kv_heads, dtype=torch.float32, device=q.device)
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device) if want_out else None
        dwkv_probe(self.h, layer, seq_ids, q, err, out, self.workspace, stream)
        return (err, out) if want_out else err

    def export(self, layer, seq, t0, n, stream=None):
        c = self.cfg
        H, R, s = c.num_kv_heads, c.r_max, c.resid_channels
        dev = self.device
        c8 = c.coeff_bits == 8
        out = {
            "tier_idx": torch.empty(n, H, dtype=torch.uint8, device=dev),
            "coeff": (torch.empty(n, H, 2, R + R // 8, dtype=torch.uint8, device=dev) if c8
                      else torch.empty(n, H, 2, R, dtype=torch.bfloat16, device=dev)),
            "idx": torch.empty(n, H, 2, s, dtype=torch.uint8, device=dev),
            "codes": torch.empty(n, H, 2, s, dtype=torch.int8, device=dev),
            "scales": torch.empty(n, H, 2, dtype=torch.float16, device=dev),
        }
        if n:
            dwkv_export(self.h, layer, seq, t0, n, out["tier_idx"], out["coeff"], out["idx"] if s else None,
                        out["codes"] if s else None, out["scales"], stream)
        if c8:
            out["ccodes"], out["cscales"] = unpack_coeff8(out.pop("coeff"), R)
        return out

    def reset(self, seq, stream=None):
        dwkv_reset_sequence(self.h, seq, stream)

    def seq_length(self, seq, layer) -> int:
        return dwkv_seq_length(self.h, seq, layer)

    def sync(self, stream=None):
        dwkv_sync_status(self.h, stream)

    def pool_usage(self, stream=None):
        return dwkv_pool_usage(self.h, stream)

    def set_decode_tuning(self, ctas_per_sm=1, waves=1, stages=0):
        dwkv_set_decode_tuning(self.h, ctas_per_sm, waves, stages)

    def set_decode_overlap(self, enable: bool):
        dwkv_set_decode_overlap(self.h, 1 if enable else 0)

    def retier(self, group, seq_ids, n_tok, positions, new_tier, stream=None):
        dwkv_retier(self.h, group, seq_ids, n_tok, positions, new_tier, stream)

    def _windows(self, group):
        return self.cfg.num_layers // self.cfg.layers_per_group if group == DWKV_ALL_GROUPS else 1

    def basis_sketch(self, group, k_rows, v_rows, omega, power_steps=2, stream=None):
        """k_rows / v_rows: bf16 [layers][n][Hkv][d] (the window's layers, or every layer with
        group = DWKV_ALL_GROUPS); omega fp32 [d][r_max].  Returns the Rayleigh-Ritz eigenvalues
        fp32 [windows][Hkv][2][r_max] ([Hkv][2][r_max] for one window)."""
        w = self._windows(group)
        eig = torch.empty(w, self.cfg.num_kv_heads, 2, self.cfg.r_max, dtype=torch.float32, device=self.device)
        dwkv_basis_sketch(self.h, group, k_rows.shape[1], k_rows, v_rows, omega, power_steps, eig, stream)
        return eig[0] if group != DWKV_ALL_GROUPS else eig

    def basis_update(self, group, k_rows, v_rows, beta, seq_ids, stream=None):
        w = self._windows(group)
        eig = torch.empty(w, self.cfg.num_kv_heads, 2, self.cfg.r_max, dtype=torch.float32, device=self.device)
        n = 0 if k_rows is None else k_rows.shape[1]
        dwkv_basis_update(self.h, group, n, k_rows, v_rows, beta, seq_ids, eig, stream)
        return eig[0] if group != DWKV_ALL_GROUPS else eig

    def bases(self, group, stream=None):
        c = self.cfg
        bk = torch.empty(c.num_kv_heads, c.head_dim, c.r_max, dtype=torch.bfloat16, device=self.device)
        bv = torch.empty_like(bk)
        dwkv_get_bases(self.h, group, bk, bv, stream)
        return bk, bv

    def moment(self, group, stream=None):
        c = self.cfg
        m = torch.empty(c.num_kv_heads, 2, c.head_dim, c.head_dim, dtype=torch.float32, device=self.device)
        dwkv_get_moment(self.h, group, m, stream)
        return m
