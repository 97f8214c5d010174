// Reads and moves of one stored token in a (layer, K / V) block of a page (the block layout of
// dwkv_common.cuh), for the kernels that re-encode stored tokens: re-tiering ("DepthWeave-KV
// ...", §3 Method, the Eq. (2)-(3) paragraphs) and the basis update's re-projection (§3, the
// shared-bases paragraph).  Both coefficient forms: bf16, and 8-bit codes in blocks of 16
// with one fp16 scale a block.
#pragma once

#include "dwkv_common.cuh"

namespace dwkv {

// Coefficient j (< R) of the token in `row` of a block of rank R, as the value decode uses:
// the bf16 value, or code x block scale (exact in fp32: 8 x 11 significant bits).
__device__ __forceinline__ float stored_coeff(const uint8_t* blk, int c8, int z, int R, int row, int j) {
    if (c8) {
        const int8_t code = (int8_t)blk[z ? vc8_code_off(j, row) : kc8_code_off(j, row)];
        const float sc = __half2float(*reinterpret_cast<const __half*>(
            blk + (z ? vc8_scale_off(R, j >> 4, row) : kc8_scale_off(R, j >> 4, row))));
        return __fmul_rn((float)code, sc);
    }
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(blk + (size_t)(j >> 3) * 1024 + row * 16 + (j & 7) * 2));
}

// Residual entry e (< s) of the token in `row`: its channel and scale x code (exact in fp32:
// 11 x 7 significant bits).
template <int BITS>
__device__ __forceinline__ void stored_resid(const uint8_t* blk, int c8, int R, int s, int row, int e, int& ch,
                                             float& v) {
    const float sf = __half2float(*reinterpret_cast<const __half*>(blk + off_scales_of(R, s, BITS, c8) + row * 2));
    ch = blk[off_idx_of(R, c8) + row * s + e];
    int code;
    if (BITS == 8) {
        code = (int8_t)blk[off_codes_of(R, s, c8) + row * s + e];
    } else {
        const uint32_t byte = blk[off_codes_of(R, s, c8) + row * (s / 2) + (e >> 1)];
        code = (int)(((e & 1) ? byte >> 4 : byte) & 0xfu);
        code = (code ^ 8) - 8;
    }
    v = __fmul_rn(sf, (float)code);
}

// Copy every stored byte of the token in row `from` of block src to row `to` of block dst (same
// tier, so the same layout), by one warp.  dst and src may be the same block; the rows differ.
template <int BITS>
__device__ __forceinline__ void move_row(uint8_t* dst, const uint8_t* src, int c8, int z, int R, int s, int to,
                                         int from) {
    const int lane = threadIdx.x & 31;
    if (!c8) {
        for (int c = lane; c < R / 8; c += 32)           // 8-coefficient columns, 16 bytes a token
            *reinterpret_cast<uint4*>(dst + (size_t)c * 1024 + to * 16) =
                *reinterpret_cast<const uint4*>(src + (size_t)c * 1024 + from * 16);
    } else if (!z) {
        for (int b = lane; b < R / 16; b += 32) {        // a block's 16 codes are 16 bytes a token
            *reinterpret_cast<uint4*>(dst + (size_t)b * 1024 + to * 16) =
                *reinterpret_cast<const uint4*>(src + (size_t)b * 1024 + from * 16);
            *reinterpret_cast<uint16_t*>(dst + kc8_scale_off(R, b, to)) =
                *reinterpret_cast<const uint16_t*>(src + kc8_scale_off(R, b, from));
        }
    } else {
        for (int j = lane; j < R; j += 32) dst[vc8_code_off(j, to)] = src[vc8_code_off(j, from)];
        for (int b = lane; b < R / 16; b += 32)
            *reinterpret_cast<uint16_t*>(dst + vc8_scale_off(R, b, to)) =
                *reinterpret_cast<const uint16_t*>(src + vc8_scale_off(R, b, from));
    }
    const uint32_t coff = off_idx_of(R, c8), qo = off_codes_of(R, s, c8);
    const uint32_t nidx = (uint32_t)s, ncode = (uint32_t)s * BITS / 8;
    for (uint32_t b = lane; b < nidx; b += 32) dst[coff + to * nidx + b] = src[coff + from * nidx + b];
    for (uint32_t b = lane; b < ncode; b += 32) dst[qo + to * ncode + b] = src[qo + from * ncode + b];
    if (lane == 0) {
        const uint32_t so = off_scales_of(R, s, BITS, c8);
        *reinterpret_cast<uint16_t*>(dst + so + to * 2) = *reinterpret_cast<const uint16_t*>(src + so + from * 2);
    }
}

}  // namespace dwkv
