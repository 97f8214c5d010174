"""CPU oracle for decode attention over the DepthWeave-KV compressed cache.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the bench's CPU
baseline are the only callers.  The product library never imports this package and this
package never imports the product library.

This module is argument marshalling only (numpy <-> the C functions of
``dwkv_oracle.c``); every step of the arithmetic lives in that C file, in fp64 for
decode / probe and in an explicitly ordered fp32 for encode.  Cited source:
"DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization for Long-Context KV
Cache Compression", §3 Method, Eq. (1) (reconstruction) and Eq. (3) (probe error).
"""
from __future__ import annotations

import ctypes as C
import math
import os

import numpy as np

from . import build as _build

_LIB = None


def lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i = C.c_int
        d = C.c_double
        L.oracle_decode_head.argtypes = [i, i, i, i, i, p, p, p, p, p, p, p, p, p, p, p, p, d, i, p, p, p, p, p]
        L.oracle_decode_head.restype = i
        L.oracle_probe_head.argtypes = [i, i, i, i, i, p, p, p, p, p, p, p, p, p, p, p, p, d, d, p, p, p, p, p, p]
        L.oracle_probe_head.restype = i
        L.oracle_decode_many.argtypes = [i, i, i, i, i, p] + [p] * 12 + [d, p, i, p, p, p]
        L.oracle_decode_many.restype = i
        L.oracle_encode_vector.argtypes = [i, i, p, p, i, i, i, p, p, p, p, p, p]
        L.oracle_encode_vector.restype = i
        L.oracle_quantize_residual.argtypes = [i, i, i, p, p, p, p]
        L.oracle_quantize_residual.restype = i
        L.oracle_encode_many.argtypes = [i, i, i, p, p, p, i, i, p, p, p, p, p, i, p]
        L.oracle_encode_many.restype = i
        L.oracle_encode_many_from_coeffs.argtypes = [i, i, i, p, p, p, p, i, i, p, p, p, p, i, p]
        L.oracle_encode_many_from_coeffs.restype = i
        L.oracle_reencode_vector.argtypes = [i, i, p, i, p, i, p, p, C.c_uint16, i, i, i, p, p, p, p, p, p]
        L.oracle_reencode_vector.restype = i
        L.oracle_reconstruct.argtypes = [i, i, p, i, p, i, p, p, C.c_uint16, i, p]
        L.oracle_reconstruct.restype = None
        L.oracle_gate_scales.argtypes = [C.c_int64, p, p, p]
        L.oracle_gate_scales.restype = None
        L.oracle_quantize_coeffs8.argtypes = [i, i, p, p, p, p]
        L.oracle_quantize_coeffs8.restype = i
        L.oracle_encode_vector8.argtypes = [i, i, p, p, p, i, i, i, p, p, p, p, p, p]
        L.oracle_encode_vector8.restype = i
        L.oracle_encode_many8.argtypes = [i, i, i, p, p, p, p, i, i, p, p, p, p, p, p, i, p]
        L.oracle_encode_many8.restype = i
        L.oracle_reencode_vector8.argtypes = [i, i, p, i, p, p, i, p, p, C.c_uint16, i, i, i, p, p, p, p, p, p, p]
        L.oracle_reencode_vector8.restype = i
        for name in ("oracle_f32_to_bf16_rn_many", "oracle_f32_to_fp16_rn_many",
                     "oracle_fp16_to_f64_many", "oracle_bf16_to_f64_many"):
            getattr(L, name).argtypes = [C.c_int64, p, p]
            getattr(L, name).restype = None
        _LIB = L
    return _LIB


# ----------------------------------------------------------------------------- marshalling
def _bits16(a) -> np.ndarray:
    """Raw 16-bit patterns (bf16 / fp16) of a torch tensor or numpy array, C-contiguous."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype in (torch.bfloat16, torch.float16):
                a = a.view(torch.int16)
            return np.ascontiguousarray(a.numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    return np.ascontiguousarray(a.astype(np.uint16, copy=False))


def _arr(a, dtype) -> np.ndarray:
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a).astype(dtype, copy=False))


def _p(a: np.ndarray):
    return a.ctypes.data_as(C.c_void_p)


def default_tau(d: int) -> float:
    return 1.0 / math.sqrt(d)


# ----------------------------------------------------------------------------- conversions
def f32_to_bf16_rn(x) -> np.ndarray:
    x = _arr(x, np.float32).reshape(-1)
    out = np.empty(x.size, np.uint16)
    lib().oracle_f32_to_bf16_rn_many(x.size, _p(x), _p(out))
    return out


def f32_to_fp16_rn(x) -> np.ndarray:
    x = _arr(x, np.float32).reshape(-1)
    out = np.empty(x.size, np.uint16)
    lib().oracle_f32_to_fp16_rn_many(x.size, _p(x), _p(out))
    return out


def fp16_to_f64(bits) -> np.ndarray:
    b = _bits16(bits).reshape(-1)
    out = np.empty(b.size, np.float64)
    lib().oracle_fp16_to_f64_many(b.size, _p(b), _p(out))
    return out


def bf16_to_f64(bits) -> np.ndarray:
    b = _bits16(bits).reshape(-1)
    out = np.empty(b.size, np.float64)
    lib().oracle_bf16_to_f64_many(b.size, _p(b), _p(out))
    return out


# ----------------------------------------------------------------------------- reconstruct
def reconstruct(basis, r_t, coeff, idx, codes, scale, with_residual=True) -> np.ndarray:
    """One reconstructed vector (fp64 [d]); basis bf16 [d][r_max], coeff bf16 [r_max]."""
    b = _bits16(basis)
    d, r_max = b.shape
    c = _bits16(coeff)
    ix = _arr(idx, np.uint8)
    cd = _arr(codes, np.int8)
    sc = int(_bits16(scale).reshape(-1)[0])
    out = np.empty(d, np.float64)
    lib().oracle_reconstruct(d, r_max, _p(b), int(r_t), _p(c), ix.size, _p(ix), _p(cd), sc,
                             1 if with_residual else 0, _p(out))
    return out


# ----------------------------------------------------------------------------- decode
class HeadProblem:
    """Token-ordered inputs of one (sequence, layer, kv-head) decode problem."""

    def __init__(self, basis_k, basis_v, ranks, coeff_k, idx_k, codes_k, scale_k,
                 coeff_v, idx_v, codes_v, scale_v, q, nres=None, coeff_k_f=None, coeff_v_f=None):
        self.bk = _bits16(basis_k)
        self.bv = _bits16(basis_v)
        self.d, self.r_max = self.bk.shape
        self.rank = _arr(ranks, np.int32).reshape(-1)
        self.T = self.rank.size
        self.ck = _bits16(coeff_k).reshape(self.T, self.r_max)
        self.cv = _bits16(coeff_v).reshape(self.T, self.r_max)
        ik = _arr(idx_k, np.uint8)
        self.s = ik.shape[-1] if ik.ndim >= 1 else 0
        self.ik = ik.reshape(self.T, self.s)
        self.iv = _arr(idx_v, np.uint8).reshape(self.T, self.s)
        self.qk = _arr(codes_k, np.int8).reshape(self.T, self.s)
        self.qv = _arr(codes_v, np.int8).reshape(self.T, self.s)
        self.sk = _bits16(scale_k).reshape(self.T)
        self.sv = _bits16(scale_v).reshape(self.T)
        self.q = _bits16(q).reshape(-1, self.d)
        self.gq = self.q.shape[0]
        # per-token residual counts (each <= s), or None: every token keeps s entries
        self.nres = None if nres is None else _arr(nres, np.int32).reshape(self.T)
        # the coefficients as fp64 values [T][r_max] (the 8-bit blockwise form, dequantised),
        # used instead of coeff_k / coeff_v when given
        self.ckf = None if coeff_k_f is None else _arr(coeff_k_f, np.float64).reshape(self.T, self.r_max)
        self.cvf = None if coeff_v_f is None else _arr(coeff_v_f, np.float64).reshape(self.T, self.r_max)

    def _ptrs(self):
        return [_p(self.bk), _p(self.bv), _p(self.rank), _p(self.ck), _p(self.ik), _p(self.qk),
                _p(self.sk), _p(self.cv), _p(self.iv), _p(self.qv), _p(self.sv), _p(self.q)]

    def _fptrs(self):
        return [_p(self.ckf) if self.ckf is not None else None, _p(self.cvf) if self.cvf is not None else None]


def head_problem(wl, bases, tier_idx, comp, q, layer, head) -> HeadProblem:
    """The decode problem of one (layer, kv-head) of one sequence, sliced from token-ordered
    arrays: ``wl`` a workload (tiers, optional per-tier residual counts ``tier_resid``,
    layers_per_group, gqa), ``bases`` the (K, V) bases
    bf16 [G][Hkv][d][r_max], ``tier_idx`` uint8 [T][Hkv] (index into ``wl.tiers``), ``comp``
    the stored arrays (coeff [T][Hkv][2][r_max], idx / codes [T][Hkv][2][s], scales
    [T][Hkv][2]; K at [..][0], V at [..][1]; with 8-bit coefficients ``ccodes`` int8
    [T][Hkv][2][r_max] and ``cscales`` fp16 bits [T][Hkv][2][r_max / 16] instead of coeff) and
    ``q`` bf16 [Hq][d], every query head of the sequence."""
    g = layer // wl.layers_per_group
    gq = wl.gqa
    ti = _arr(tier_idx, np.int64)[:, head]
    ranks = np.asarray(wl.tiers, np.int32)[ti]
    tr = getattr(wl, "tier_resid", ())
    nres = np.asarray(tr, np.int32)[ti] if tr else None
    sl = lambda key, z: comp[key][:, head, z]   # noqa: E731
    if "ccodes" in comp:
        cf = [dequant_coeffs8(sl("ccodes", z), sl("cscales", z)) for z in (0, 1)]
        zero = np.zeros(cf[0].shape, np.uint16)
        return HeadProblem(bases[0][g, head], bases[1][g, head], ranks,
                           zero, sl("idx", 0), sl("codes", 0), comp["scales"][:, head, 0],
                           zero, sl("idx", 1), sl("codes", 1), comp["scales"][:, head, 1],
                           _bits16(q)[head * gq:(head + 1) * gq], nres=nres, coeff_k_f=cf[0], coeff_v_f=cf[1])
    return HeadProblem(bases[0][g, head], bases[1][g, head], ranks,
                       sl("coeff", 0), sl("idx", 0), sl("codes", 0), comp["scales"][:, head, 0],
                       sl("coeff", 1), sl("idx", 1), sl("codes", 1), comp["scales"][:, head, 1],
                       _bits16(q)[head * gq:(head + 1) * gq], nres=nres)


def decode_head(prob: HeadProblem, tau=None, with_residual=True, want_p=False):
    """fp64 attention output [gq][d] (and softmax weights [gq][T] when ``want_p``)."""
    tau = default_tau(prob.d) if tau is None else tau
    out = np.empty((prob.gq, prob.d), np.float64)
    pw = np.empty((prob.gq, max(prob.T, 1)), np.float64) if want_p else None
    rc = lib().oracle_decode_head(prob.d, prob.r_max, prob.T, prob.gq, prob.s, *prob._ptrs(),
                                  float(tau), 1 if with_residual else 0, _p(out),
                                  _p(pw) if want_p else None, _p(prob.nres) if prob.nres is not None else None,
                                  *prob._fptrs())
    if rc != 0:
        raise MemoryError("oracle_decode_head failed")
    if want_p:
        return out, pw[:, :prob.T]
    return out


def probe_head(prob: HeadProblem, tau=None, eps=1e-6):
    """Relative L2 error (Eq. 3 reading) and both outputs (fp64)."""
    tau = default_tau(prob.d) if tau is None else tau
    err = np.zeros(1, np.float64)
    of = np.empty((prob.gq, prob.d), np.float64)
    on = np.empty((prob.gq, prob.d), np.float64)
    rc = lib().oracle_probe_head(prob.d, prob.r_max, prob.T, prob.gq, prob.s, *prob._ptrs(),
                                 float(tau), float(eps), _p(err), _p(of), _p(on),
                                 _p(prob.nres) if prob.nres is not None else None, *prob._fptrs())
    if rc != 0:
        raise MemoryError("oracle_probe_head failed")
    return float(err[0]), of, on


def decode_many(problems, tau=None, nthreads=None):
    """Run many independent problems on ``nthreads`` host threads; list of [gq][d] outputs."""
    if not problems:
        return []
    n = len(problems)
    p0 = problems[0]
    tau = default_tau(p0.d) if tau is None else tau
    nthreads = nthreads or os.cpu_count() or 1
    T = np.array([pr.T for pr in problems], np.int32)
    cols = list(zip(*[pr._ptrs() for pr in problems]))
    arrs = [(C.c_void_p * n)(*col) for col in cols]
    outs = [np.empty((pr.gq, pr.d), np.float64) for pr in problems]
    oarr = (C.c_void_p * n)(*[_p(o) for o in outs])
    narr = None
    if any(pr.nres is not None for pr in problems):
        full = [pr.nres if pr.nres is not None else np.full(pr.T, pr.s, np.int32) for pr in problems]
        narr = (C.c_void_p * n)(*[_p(a) for a in full])
    farr, keep = [None, None], []
    for z, key in enumerate(("ckf", "cvf")):
        if any(getattr(pr, key) is not None for pr in problems):
            full = [getattr(pr, key) if getattr(pr, key) is not None
                    else bf16_to_f64(getattr(pr, key[:2])).reshape(pr.T, pr.r_max) for pr in problems]
            keep.append(full)                       # alive until the call returns
            farr[z] = (C.c_void_p * n)(*[_p(a) for a in full])
    rc = lib().oracle_decode_many(n, p0.d, p0.r_max, p0.gq, p0.s, _p(T), *arrs, float(tau), oarr,
                                  int(nthreads), narr, *farr)
    if rc != 0:
        raise MemoryError("oracle_decode_many failed")
    return outs


# ----------------------------------------------------------------------------- encode
def encode_vector(basis, x, r_t, s, bits):
    """Encode one bf16 vector; dict of coeff (bf16 bits), c32, idx, codes, scale (fp16 bits), resid."""
    b = _bits16(basis)
    d, r_max = b.shape
    xv = _bits16(x).reshape(d)
    coeff = np.zeros(r_max, np.uint16)
    c32 = np.zeros(r_max, np.float32)
    idx = np.zeros(s, np.uint8)
    codes = np.zeros(s, np.int8)
    scale = np.zeros(1, np.uint16)
    resid = np.zeros(d, np.float32)
    rc = lib().oracle_encode_vector(d, r_max, _p(b), _p(xv), int(r_t), int(s), int(bits), _p(coeff),
                                    _p(c32), _p(idx), _p(codes), _p(scale), _p(resid))
    if rc != 0:
        raise ValueError("oracle_encode_vector: bad arguments")
    return {"coeff": coeff, "c32": c32, "idx": idx, "codes": codes, "scale": scale[0], "resid": resid}


def quantize_residual(r, s, bits):
    """Encode steps 4-6 on a given fp32 residual [d]: dict of idx (ascending), codes, scale (fp16 bits)."""
    rv = _arr(r, np.float32).reshape(-1)
    idx = np.zeros(s, np.uint8)
    codes = np.zeros(s, np.int8)
    scale = np.zeros(1, np.uint16)
    rc = lib().oracle_quantize_residual(rv.shape[0], int(s), int(bits), _p(rv), _p(idx), _p(codes), _p(scale))
    if rc != 0:
        raise ValueError("oracle_quantize_residual: bad arguments")
    return {"idx": idx, "codes": codes, "scale": scale[0]}


def encode_many(basis, x, ranks, s, bits, nthreads=None, want_c32=False, nres=None):
    """Encode n vectors [n][d] sharing one basis; arrays token-ordered.  ``nres`` (optional,
    int [n], each <= s): per-vector residual counts; entries past them stay zero."""
    b = _bits16(basis)
    d, r_max = b.shape
    xv = _bits16(x).reshape(-1, d)
    n = xv.shape[0]
    rk = _arr(ranks, np.int32).reshape(n)
    coeff = np.zeros((n, r_max), np.uint16)
    c32 = np.zeros((n, r_max), np.float32) if want_c32 else None
    idx = np.zeros((n, s), np.uint8)
    codes = np.zeros((n, s), np.int8)
    scale = np.zeros(n, np.uint16)
    nr = None if nres is None else _arr(nres, np.int32).reshape(n)
    rc = lib().oracle_encode_many(n, d, r_max, _p(b), _p(xv), _p(rk), int(s), int(bits), _p(coeff),
                                  _p(c32) if want_c32 else None, _p(idx), _p(codes), _p(scale),
                                  int(nthreads or os.cpu_count() or 1), _p(nr) if nr is not None else None)
    if rc != 0:
        raise ValueError("oracle_encode_many: bad arguments")
    out = {"coeff": coeff, "idx": idx, "codes": codes, "scale": scale}
    if want_c32:
        out["c32"] = c32
    return out


def reencode_vector(basis, r_old, coeff, idx, codes, scale, r_new, bits, s_new=None, basis_new=None):
    """Re-tier one stored vector: re-encode its bf16-rounded reconstruction at rank r_new with
    s_new residual channels (default: as many as stored) on basis_new (default: the same basis)
    (``oracle_reencode_vector``).  Returns the encode dict plus ``xh`` (bf16 bits [d])."""
    b = _bits16(basis)
    d, r_max = b.shape
    c = _bits16(coeff).reshape(r_max)
    ix = _arr(idx, np.uint8).reshape(-1)
    cd = _arr(codes, np.int8).reshape(-1)
    s = ix.size
    sc = int(_bits16(scale).reshape(-1)[0])
    sn = s if s_new is None else int(s_new)
    out_c = np.zeros(r_max, np.uint16)
    out_i = np.zeros(sn, np.uint8)
    out_q = np.zeros(sn, np.int8)
    out_s = np.zeros(1, np.uint16)
    xh = np.zeros(d, np.uint16)
    bn = None if basis_new is None else _bits16(basis_new)
    if bn is not None and bn.shape != b.shape:
        raise ValueError("basis_new must have the basis' shape")
    rc = lib().oracle_reencode_vector(d, r_max, _p(b), int(r_old), _p(c), s, _p(ix), _p(cd), sc, int(r_new), sn,
                                      int(bits), _p(out_c), _p(out_i), _p(out_q), _p(out_s), _p(xh),
                                      _p(bn) if bn is not None else None)
    if rc != 0:
        raise ValueError("oracle_reencode_vector: bad arguments")
    return {"coeff": out_c, "idx": out_i, "codes": out_q, "scale": out_s[0], "xh": xh}


def encode_many_from_coeffs(basis, x, c32, ranks, s, bits, nthreads=None, nres=None):
    """Encode steps 2-6 of n vectors [n][d] sharing one basis, from given fp32 projections
    c32 [n][r_max] (only [:r_t] read): the stored bytes of an encoder that computed c32."""
    b = _bits16(basis)
    d, r_max = b.shape
    xv = _bits16(x).reshape(-1, d)
    n = xv.shape[0]
    cv = _arr(c32, np.float32).reshape(n, r_max)
    rk = _arr(ranks, np.int32).reshape(n)
    coeff = np.zeros((n, r_max), np.uint16)
    idx = np.zeros((n, s), np.uint8)
    codes = np.zeros((n, s), np.int8)
    scale = np.zeros(n, np.uint16)
    nr = None if nres is None else _arr(nres, np.int32).reshape(n)
    rc = lib().oracle_encode_many_from_coeffs(n, d, r_max, _p(b), _p(xv), _p(cv), _p(rk), int(s), int(bits), _p(coeff),
                                              _p(idx), _p(codes), _p(scale), int(nthreads or os.cpu_count() or 1),
                                              _p(nr) if nr is not None else None)
    if rc != 0:
        raise ValueError("oracle_encode_many_from_coeffs: bad arguments")
    return {"coeff": coeff, "idx": idx, "codes": codes, "scale": scale}


# ----------------------------------------------------------------------------- 8-bit coefficients
def quantize_coeffs8(c, r_t):
    """The 8-bit blockwise form of fp32 coefficients c [r_max] (only [:r_t] read, r_t a multiple
    of 16): dict of codes int8 [r_max], scales (fp16 bits [r_max / 16]) and the dequantised
    values cbar fp32 [r_max] (``oracle_quantize_coeffs8``)."""
    cv = _arr(c, np.float32).reshape(-1)
    r_max = cv.size
    q = np.zeros(r_max, np.int8)
    sc = np.zeros(max(r_max // 16, 1), np.uint16)
    cbar = np.zeros(r_max, np.float32)
    if lib().oracle_quantize_coeffs8(int(r_t), r_max, _p(cv), _p(q), _p(sc), _p(cbar)) != 0:
        raise ValueError("oracle_quantize_coeffs8: bad arguments")
    return {"codes": q, "scales": sc, "cbar": cbar}


def dequant_coeffs8(codes, scales) -> np.ndarray:
    """fp64 values of 8-bit blockwise coefficients: code_j x scale of block j // 16 (exact)."""
    q = _arr(codes, np.int8)
    sc = fp16_to_f64(_bits16(scales).reshape(-1)).reshape(_bits16(scales).shape)
    return q.astype(np.float64) * np.repeat(sc, 16, axis=-1)[..., :q.shape[-1]]


def encode_vector8(basis, x, r_t, s, bits, c_in=None):
    """Encode one bf16 vector with 8-bit blockwise coefficients: dict of ccodes (int8 [r_max]),
    cscales (fp16 bits [r_max / 16]), c32, idx, codes, scale (fp16 bits)."""
    b = _bits16(basis)
    d, r_max = b.shape
    xv = _bits16(x).reshape(d)
    ci = None if c_in is None else _arr(c_in, np.float32).reshape(r_max)
    cc = np.zeros(r_max, np.int8)
    cs = np.zeros(r_max // 16, np.uint16)
    c32 = np.zeros(r_max, np.float32)
    idx = np.zeros(s, np.uint8)
    codes = np.zeros(s, np.int8)
    scale = np.zeros(1, np.uint16)
    rc = lib().oracle_encode_vector8(d, r_max, _p(b), _p(xv), _p(ci) if ci is not None else None, int(r_t), int(s),
                                     int(bits), _p(cc), _p(cs), _p(c32), _p(idx), _p(codes), _p(scale))
    if rc != 0:
        raise ValueError("oracle_encode_vector8: bad arguments")
    return {"ccodes": cc, "cscales": cs, "c32": c32, "idx": idx, "codes": codes, "scale": scale[0]}


def encode_many8(basis, x, ranks, s, bits, c32=None, nthreads=None, nres=None, want_c32=False):
    """encode_vector8 over n vectors [n][d] sharing one basis, token-ordered; ``c32`` (optional
    [n][r_max]) the fp32 projections to use instead of step 1; ``nres`` as encode_many."""
    b = _bits16(basis)
    d, r_max = b.shape
    xv = _bits16(x).reshape(-1, d)
    n = xv.shape[0]
    rk = _arr(ranks, np.int32).reshape(n)
    ci = None if c32 is None else _arr(c32, np.float32).reshape(n, r_max)
    cc = np.zeros((n, r_max), np.int8)
    cs = np.zeros((n, r_max // 16), np.uint16)
    co = np.zeros((n, r_max), np.float32) if want_c32 else None
    idx = np.zeros((n, s), np.uint8)
    codes = np.zeros((n, s), np.int8)
    scale = np.zeros(n, np.uint16)
    nr = None if nres is None else _arr(nres, np.int32).reshape(n)
    rc = lib().oracle_encode_many8(n, d, r_max, _p(b), _p(xv), _p(ci) if ci is not None else None, _p(rk), int(s),
                                   int(bits), _p(cc), _p(cs), _p(co) if want_c32 else None, _p(idx), _p(codes),
                                   _p(scale), int(nthreads or os.cpu_count() or 1), _p(nr) if nr is not None else None)
    if rc != 0:
        raise ValueError("oracle_encode_many8: bad arguments")
    out = {"ccodes": cc, "cscales": cs, "idx": idx, "codes": codes, "scale": scale}
    if want_c32:
        out["c32"] = co
    return out


def reencode_vector8(basis, r_old, ccodes, cscales, idx, codes, scale, r_new, bits, s_new=None, basis_new=None):
    """reencode_vector for the 8-bit blockwise coefficient form: the stored codes int8 [r_max]
    and block scales (fp16 bits [r_max / 16]) in, the new ones out
    (``oracle_reencode_vector8``).  Returns the encode8 dict plus ``xh`` (bf16 bits [d])."""
    b = _bits16(basis)
    d, r_max = b.shape
    cc = _arr(ccodes, np.int8).reshape(r_max)
    cs = _bits16(cscales).reshape(r_max // 16)
    ix = _arr(idx, np.uint8).reshape(-1)
    cd = _arr(codes, np.int8).reshape(-1)
    s = ix.size
    sc = int(_bits16(scale).reshape(-1)[0])
    sn = s if s_new is None else int(s_new)
    out_cc = np.zeros(r_max, np.int8)
    out_cs = np.zeros(r_max // 16, np.uint16)
    out_i = np.zeros(sn, np.uint8)
    out_q = np.zeros(sn, np.int8)
    out_s = np.zeros(1, np.uint16)
    xh = np.zeros(d, np.uint16)
    bn = None if basis_new is None else _bits16(basis_new)
    if bn is not None and bn.shape != b.shape:
        raise ValueError("basis_new must have the basis' shape")
    rc = lib().oracle_reencode_vector8(d, r_max, _p(b), int(r_old), _p(cc), _p(cs), s, _p(ix), _p(cd), sc,
                                       int(r_new), sn, int(bits), _p(out_cc), _p(out_cs), _p(out_i), _p(out_q),
                                       _p(out_s), _p(xh), _p(bn) if bn is not None else None)
    if rc != 0:
        raise ValueError("oracle_reencode_vector8: bad arguments")
    return {"ccodes": out_cc, "cscales": out_cs, "idx": out_i, "codes": out_q, "scale": out_s[0], "xh": xh}

# ----------------------------------------------------------------------------- residual gate
def gate_scales(scales, gates) -> np.ndarray:
    """Stored residual scales with the gate folded in: fp16_rn(g * scale) elementwise (fp16
    bits in, fp16 bits out; ``oracle_gate_scale``)."""
    sc = _bits16(scales)
    g = _arr(gates, np.float32).reshape(sc.shape)
    out = np.empty(sc.shape, np.uint16)
    lib().oracle_gate_scales(sc.size, _p(sc), _p(g), _p(out))
    return out
