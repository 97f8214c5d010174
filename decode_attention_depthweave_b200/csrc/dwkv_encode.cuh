// dwkv_encode.cuh -- the per-vector encode steps shared by the append kernels and the fused
// append-and-decode path.  "DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization
// for Long-Context KV Cache Compression", §3 Method (coefficients are the projection of the
// original vector onto the current basis; the residual is quantised and kept only on the
// routed channels), in this library's fixed fp32 operation order, which makes the stored
// bytes reproducible bit for bit:
//   1. c_j  = fma chain over i = 0..d-1 of B[i][j] * x_i from +0            (j < r_t)
//   2. cb_j = bf16_rn(c_j)                                                 (stored)
//   3. r_i  = x_i - a_i, a_i = fma chain over j = 0..r_t-1 of B[i][j] * cb_j from +0
//   4. the s largest |r_i|, ties to the lower channel, stored in ascending channel order
//   5. scale = fp16_rn(max |r_sel| / qmax) with IEEE division, qmax = 127 (int8) / 7 (int4)
//   6. code  = clamp(rint(r / float(scale)), -qmax, qmax), all zero when scale == 0
#pragma once
#include "dwkv_common.cuh"

namespace dwkv {

// Destination block of (sequence, group, kv-head, position) at a layer, or nullptr.
struct Dest {
    uint8_t* blk;   // K block; V block = blk + blk_bytes
    int k, row, R;
};
__device__ __forceinline__ bool find_dest(const Geom& G, const State& S, int seq, int g, int lig, int h,
                                          int pos, Dest& d) {
    const uint32_t sm = S.slot_map[slot_index(G, seq, g, h, pos)];
    if (sm == 0u) return false;
    const int k = (int)(sm >> 24) - 1;
    const uint32_t slot = sm & 0xffffffu;
    const uint32_t unit = S.pages[page_index(G, seq, g, h, k) + slot / kPage];
    d.k = k;
    d.row = (int)(slot % kPage);
    d.R = G.tiers[k];
    d.blk = S.data + (size_t)unit * kUnit + (size_t)lig * G.chunk_bytes[k];
    return true;
}

// Slot of one new position of (seq, group g, kv-head h) in tier k, the counts left as they are
// (the caller adds the position to them later): the tier's next slot, and a fresh page when the
// slot opens one (the tier's free ring first, then the pool's bump pointer).  Single thread.
__device__ __forceinline__ bool place_one(const Geom& G, const State& S, int seq, int g, int h, int pos,
                                          uint32_t k, Dest& d, int lig) {
    const uint32_t old = __ldcg(S.counts + cnt_index(G, seq, g, h) + k);
    const uint32_t pi = old / kPage;
    if (pi >= (uint32_t)G.max_pages) {
        set_dev_error(S, 1u /*DWKV_DEV_POOL_EXHAUSTED*/, (uint32_t)seq, (uint32_t)h);
        return false;
    }
    uint32_t unit;
    if (old % kPage == 0) {
        const uint32_t t = atomicAdd(&S.free_head[k], 1u);
        const uint32_t tail = *((volatile uint32_t*)&S.free_tail[k]);
        if ((int)(tail - t) > 0) {
            unit = S.free_list[(size_t)k * G.free_cap + (t & (G.free_cap - 1))];
        } else {
            const unsigned long long base = atomicAdd(S.bump, (unsigned long long)G.page_units[k]);
            if (base + G.page_units[k] > S.data_units) {
                set_dev_error(S, 1u /*DWKV_DEV_POOL_EXHAUSTED*/, (uint32_t)seq, (uint32_t)h);
                return false;
            }
            unit = (uint32_t)base;
        }
        S.pages[page_index(G, seq, g, h, k) + pi] = unit;
    } else {
        unit = __ldcg(S.pages + page_index(G, seq, g, h, k) + pi);
    }
    S.slot_map[slot_index(G, seq, g, h, pos)] = ((k + 1u) << 24) | old;
    d.k = (int)k;
    d.row = (int)(old % kPage);
    d.R = G.tiers[k];
    d.blk = S.data + (size_t)unit * kUnit + (size_t)lig * G.chunk_bytes[k];
    return true;
}

// Shared-memory scratch of one encode warp: x [d], stored coefficients [kMaxRank], code staging.
struct EncScratch {
    float* xs;
    float* cs;
    int8_t* cstage;
};
__device__ __forceinline__ EncScratch enc_scratch(const Geom& G, uint8_t* smem, int warp) {
    float* xs = reinterpret_cast<float*>(smem + (size_t)2 * kD * (G.r_max + 2) * 2) + (size_t)warp * (kD + kMaxRank + 32);
    return {xs, xs + kD, reinterpret_cast<int8_t*>(xs + kD + kMaxRank)};
}

// Inputs of one encode unit (token row, keys z = 0 or values z = 1): x (channel lane + 32 m)
// and the destination block, both requested together.
struct UnitIn {
    Dest dst;
    float xr[4];
    bool ok;
};

// The six encode steps of one unit on one warp.
template <int BITS>
__device__ __forceinline__ void encode_body(const Geom& G, const State& S, const __nv_bfloat16* bs,
                                            const EncScratch& W, int unit, const UnitIn& in) {
    const int lane = threadIdx.x & 31;
    const int P = G.r_max + 2, s = G.s;
    float* xs = W.xs;
    float* cs = W.cs;
    int8_t* cstage = W.cstage;
    const float qmax = BITS == 8 ? 127.f : 7.f;
    do {
        const int z = unit & 1;
        if (!in.ok) break;
        const Dest& dst = in.dst;
        float xr[4] = {in.xr[0], in.xr[1], in.xr[2], in.xr[3]};
        const int R = dst.R;
        const __nv_bfloat16* bz = bs + (size_t)z * kD * P;
        uint8_t* blk = dst.blk + (z ? G.blk_bytes[dst.k] : 0u);
#pragma unroll
        for (int m = 0; m < 4; ++m) xs[lane + 32 * m] = xr[m];
        __syncwarp();
        // ---- 1-2: projection (fma chain over i from +0), bf16 rounding, coefficient store.
        //      Lane takes j = lane + 32 jj; the chains of one lane run interleaved.
        {
            float acc[kMaxRank / 32];
#pragma unroll
            for (int jj = 0; jj < kMaxRank / 32; ++jj) acc[jj] = 0.f;
#pragma unroll 8
            for (int i = 0; i < kD; ++i) {
                const float xi = xs[i];
                const __nv_bfloat16* brow = bz + (size_t)i * P + lane;
#pragma unroll
                for (int jj = 0; jj < kMaxRank / 32; ++jj)
                    if (lane + 32 * jj < R) acc[jj] = __fmaf_rn(__bfloat162float(brow[32 * jj]), xi, acc[jj]);
            }
#pragma unroll
            for (int jj = 0; jj < kMaxRank / 32; ++jj) {
                const int j = lane + 32 * jj;
                if (j < R) {
                    const __nv_bfloat16 cb = __float2bfloat16_rn(acc[jj]);
                    cs[j] = __bfloat162float(cb);
                    *reinterpret_cast<__nv_bfloat16*>(blk + (size_t)(j >> 3) * 1024 + dst.row * 16 + (j & 7) * 2) = cb;
                }
            }
        }
        __syncwarp();
        // ---- 3: residual against the stored coefficients (fma chain over j from +0)
        float r[4];
        {
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j0 = 0; j0 < R; j0 += 8) {           // R is a multiple of 8
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const float cj = cs[j0 + jj];
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        a[m] = __fmaf_rn(__bfloat162float(bz[(size_t)(lane + 32 * m) * P + j0 + jj]), cj, a[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) r[m] = __fsub_rn(xr[m], a[m]);
        }
        // ---- 4: top-s by magnitude, ties to the lower channel (channel = lane + 32 m)
        uint32_t key[4], sel = 0u;
#pragma unroll
        for (int m = 0; m < 4; ++m) key[m] = __float_as_uint(fabsf(r[m])) + 1u;
        for (int it = 0; it < s; ++it) {
            uint32_t best = 0u, bm = 0u;
#pragma unroll
            for (int m = 0; m < 4; ++m)
                if (!((sel >> m) & 1u) && key[m] > best) { best = key[m]; bm = (uint32_t)m; }
            const uint32_t wmax = __reduce_max_sync(0xffffffffu, best);
            const uint32_t cand = (best == wmax && best != 0u) ? (bm * 32u + (uint32_t)lane) : 0xffffffffu;
            const uint32_t wch = __reduce_min_sync(0xffffffffu, cand);
            if ((int)(wch & 31u) == lane) sel |= 1u << (wch >> 5);
        }
        // ---- 5-6: scale and codes; ranks give ascending channel order
        {
            uint32_t mx = 0u;
#pragma unroll
            for (int m = 0; m < 4; ++m)
                if ((sel >> m) & 1u) mx = max(mx, key[m] - 1u);
            const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, mx));
            const __half sh = __float2half_rn(__fdiv_rn(amax, qmax));
            const float sf = __half2float(sh);
            uint32_t before = 0u;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const bool on = (sel >> m) & 1u;
                const uint32_t bal = __ballot_sync(0xffffffffu, on);
                if (on) {
                    const int rank = (int)(before + __popc(bal & ((1u << lane) - 1u)));
                    float c = 0.f;
                    if (sf != 0.f) c = fminf(fmaxf(rintf(__fdiv_rn(r[m], sf)), -qmax), qmax);
                    blk[off_idx_of(R) + dst.row * s + rank] = (uint8_t)(lane + 32 * m);
                    if (BITS == 8) blk[off_codes_of(R, s) + dst.row * s + rank] = (uint8_t)(int8_t)c;
                    else cstage[rank] = (int8_t)c;
                }
                before += __popc(bal);
            }
            if (lane == 0) *reinterpret_cast<__half*>(blk + off_scales_of(R, s, BITS) + dst.row * 2) = sh;
        }
        if (BITS == 4) {
            __syncwarp();
            for (int b = lane; b < s / 2; b += 32) {
                const uint8_t lo = (uint8_t)cstage[2 * b] & 0xfu;
                const uint8_t hi = (uint8_t)cstage[2 * b + 1] & 0xfu;
                blk[off_codes_of(R, s) + dst.row * (s / 2) + b] = (uint8_t)(lo | (hi << 4));
            }
        }
    } while (false);
    __syncwarp();
}


}  // namespace dwkv
