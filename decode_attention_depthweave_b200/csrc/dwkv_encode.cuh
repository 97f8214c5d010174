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
//      With a residual gate g (Eq. (1)'s g R, folded into the dequantisation): the stored
//      scale is fp16_rn(g * float(scale)) (an fp32 product); the codes are those of step 6.
// With 8-bit coefficients (the blockwise form kept by the pages), step 2 becomes, per block of
// 16 coefficients: sc = fp16_rn(max |c| / 127) (IEEE division), q_j = clamp(rint(c_j /
// float(sc)), -127, 127) (0 when sc == 0), cb_j = q_j float(sc) (exact); steps 3-6 as above.
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
// (the caller adds the position to them later): the tier's next slot, and, when the slot opens
// a page, a page the tier already holds or else a fresh one (the tier's free ring first, then
// the pool's bump pointer).  Records the slot in the slot map and the position in the page.
// Single thread.
__device__ __forceinline__ bool place_one(const Geom& G, const State& S, int seq, int g, int h, int pos,
                                          uint32_t k, Dest& d, int lig) {
    const uint32_t old = __ldcg(S.counts + cnt_index(G, seq, g, h) + k);
    const uint32_t pi = old / kPage;
    if (pi >= (uint32_t)G.max_pages) {
        set_dev_error(S, 1u /*DWKV_DEV_POOL_EXHAUSTED*/, (uint32_t)seq, (uint32_t)h);
        return false;
    }
    uint32_t unit;
    if (old % kPage == 0 && pi < __ldcg(S.owned + cnt_index(G, seq, g, h) + k)) {
        unit = __ldcg(S.pages + page_index(G, seq, g, h, k) + pi);
    } else if (old % kPage == 0) {
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
        S.owned[cnt_index(G, seq, g, h) + k] = pi + 1;
    } else {
        unit = __ldcg(S.pages + page_index(G, seq, g, h, k) + pi);
    }
    S.slot_map[slot_index(G, seq, g, h, pos)] = ((k + 1u) << 24) | old;
    reinterpret_cast<int32_t*>(S.data + (size_t)unit * kUnit + pos_block_of(G, (int)k))[old % kPage] = pos;
    d.k = (int)k;
    d.row = (int)(old % kPage);
    d.R = G.tiers[k];
    d.blk = S.data + (size_t)unit * kUnit + (size_t)lig * G.chunk_bytes[k];
    return true;
}

// Shared memory of the bulk encode kernel (one tile of kEncTile rows, one of K or V):
// the basis bf16 [kD][PB] (PB = RP + 2, RP = r_max rounded up to 16; the odd word pitch
// makes column reads conflict-free) for the residual step, the basis transposed bf16
// [RP][kEncXB] and the tile's x bf16 [kEncTile][kEncXB] by slot (the tensor-core operands of
// the projection; a 272-byte row pitch keeps ldmatrix conflict-free), the stored
// coefficients fp32 [RP][kEncXP] by slot, per-slot destinations and input rows, tier counts,
// and each warp's code staging.
constexpr int kEncTile = 64;
constexpr int kEncXP = kEncTile + 4;
constexpr int kEncXB = kD + 8;
constexpr int kEncStage = kD * 4 + kD;   // per warp: residuals and channels in rank order
struct EncTileLayout {
    uint32_t bs, bt, xb, cs, sblk, sR, sprow, srow, rslot, misc, cst, total;
    int RP, PB;
};
__host__ __device__ inline EncTileLayout enc_tile_layout(int r_max) {
    EncTileLayout L;
    L.RP = (r_max + 15) / 16 * 16;
    L.PB = L.RP + 2;
    uint32_t o = 0;
    L.bs = o;    o += (uint32_t)kD * L.PB * 2;  o = (o + 15u) & ~15u;
    L.bt = o;    o += (uint32_t)L.RP * kEncXB * 2;
    L.xb = o;    o += (uint32_t)kEncTile * kEncXB * 2;
    L.cs = o;    o += (uint32_t)L.RP * kEncXP * 4;
    L.sblk = o;  o += kEncTile * 8;
    L.sR = o;    o += kEncTile * 4;
    L.sprow = o; o += kEncTile * 4;
    L.srow = o;  o += kEncTile * 4;
    L.rslot = o; o += kEncTile * 4;
    L.misc = o;  o += 128;
    L.cst = o;   o += 8 * kEncStage;
    L.total = o;
    return L;
}

// Shared memory of an 8-warp encoder block: both bases with padded rows, then the warps'
// scratch (enc_scratch).
__host__ __device__ inline size_t encode_smem_bytes(int r_max) {
    return (size_t)2 * kD * (r_max + 2) * 2 + (size_t)8 * (kD + kMaxRank + 32) * 4;
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
    float* dbg = nullptr;   // the unit's fp32 projection c[j], j < r_t (coefficient export), or none
    float gate = 1.f;       // residual gate folded into the stored scale
};

// Step 4 by its definition: s rounds of "largest remaining |r|, ties to the lower channel"
// (channel = lane + 32 m).  Returns the selected channels as a bit mask over m.
static __device__ __noinline__ uint32_t select_exact(float r0, float r1, float r2, float r3, int s) {
    const int lane = threadIdx.x & 31;
    const float r[4] = {r0, r1, r2, r3};
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
    return sel;
}

// Steps 4-6 of one vector on one warp, from its residual r (channel lane + 32 m): top-s
// selection, scale, codes, and the stores of indices, codes and scale into the vector's block
// (blk: this vector's K or V block, row: its row in the page, s: the residual channels its
// tier keeps).  rstage / chstage: s floats and s bytes of the warp's shared memory.
//
// Selection: each channel gets a 32-bit key, its |r| with the 7 lowest mantissa bits replaced
// by 127 - channel.  The keys are distinct, and ordering them orders |r| at 2^-16 relative
// resolution with ties to the lower channel.  The s largest keys come out of a warp merge of
// each lane's 4 keys (sorted in registers) with one max-reduction per round.  If the s-th and
// (s+1)-th largest keys differ above the 7 replaced bits, every selected |r| exceeds every
// other one, so the set equals the exact top-s; otherwise (a near-tie at the boundary, e.g.
// exact zeros) the selection is redone by its definition (select_exact).
template <int BITS>
__device__ __forceinline__ void quantize_store(const float (&r)[4], uint8_t* blk, int R, int row, int s,
                                               float* rstage, uint8_t* chstage, int c8, float gate = 1.f) {
    const int lane = threadIdx.x & 31;
    const float qmax = BITS == 8 ? 127.f : 7.f;
    uint32_t sel = 0u, mxb = 0u;
    if (s > 0) {
        uint32_t kk[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t b = __float_as_uint(fabsf(r[m]));
            mxb = max(mxb, b);
            kk[m] = (b & ~0x7fu) | (uint32_t)(127 - lane - 32 * m);
        }
        // the lane's keys, descending (distinct, so min / max order them fully)
        uint32_t h0 = max(kk[0], kk[1]), h1 = min(kk[0], kk[1]);
        uint32_t h2 = max(kk[2], kk[3]), h3 = min(kk[2], kk[3]);
        {
            const uint32_t a0 = max(h0, h2), a2 = min(h0, h2), a1 = max(h1, h3), a3 = min(h1, h3);
            h0 = a0;
            h1 = max(a1, a2);
            h2 = min(a1, a2);
            h3 = a3;
        }
        uint32_t K = 0u;
        for (int it = 0; it < s; ++it) {
            K = __reduce_max_sync(0xffffffffu, h0);
            if (h0 == K) {
                h0 = h1;
                h1 = h2;
                h2 = h3;
                h3 = 0u;
            }
        }
        const uint32_t K1 = s < kD ? __reduce_max_sync(0xffffffffu, h0) : 0u;
        if (s < kD && ((K ^ K1) >> 7) == 0u) {
            sel = select_exact(r[0], r[1], r[2], r[3], s);
        } else {
#pragma unroll
            for (int m = 0; m < 4; ++m) sel |= (kk[m] >= K ? 1u : 0u) << m;
        }
    }
    // ---- 5-6: scale from the largest selected |r| (the largest of all), codes by rank
    //      (ascending channel order); lane b takes rank b
    const float amax = s > 0 ? __uint_as_float(__reduce_max_sync(0xffffffffu, mxb)) : 0.f;
    const __half sh = __float2half_rn(__fdiv_rn(amax, qmax));
    const float sf = __half2float(sh);
    uint32_t before = 0u;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const bool on = (sel >> m) & 1u;
        const uint32_t bal = __ballot_sync(0xffffffffu, on);
        if (on) {
            const int rank = (int)(before + __popc(bal & ((1u << lane) - 1u)));
            rstage[rank] = r[m];
            chstage[rank] = (uint8_t)(lane + 32 * m);
        }
        before += __popc(bal);
    }
    if (lane == 0)
        *reinterpret_cast<__half*>(blk + off_scales_of(R, s, BITS, c8) + row * 2) =
            gate == 1.f ? sh : __float2half_rn(__fmul_rn(gate, sf));
    __syncwarp();
    for (int b0 = 0; b0 < s; b0 += 32) {
        const int b = b0 + lane;
        int code = 0;
        if (b < s) {
            float c = 0.f;
            if (sf != 0.f) c = fminf(fmaxf(rintf(__fdiv_rn(rstage[b], sf)), -qmax), qmax);
            code = (int)c;
            blk[off_idx_of(R, c8) + row * s + b] = chstage[b];
            if (BITS == 8) blk[off_codes_of(R, s, c8) + row * s + b] = (uint8_t)(int8_t)code;
        }
        if (BITS == 4) {
            const int hi = __shfl_down_sync(0xffffffffu, code, 1);
            if (b < s && !(b & 1))
                blk[off_codes_of(R, s, c8) + row * (s / 2) + (b >> 1)] = (uint8_t)((code & 0xf) | ((hi & 0xf) << 4));
        }
    }
    __syncwarp();
}

// Step 2 of the 8-bit coefficient form for one value per lane, the lanes of each half warp one
// block of 16 (every lane of the warp calls it): the block's scale (fp16 bits) and this lane's
// code and dequantised value.
__device__ __forceinline__ void quantize_coeff8(float v, uint16_t& sh_out, int& q_out, float& cb_out) {
    float m = fabsf(v);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const __half sh = __float2half_rn(__fdiv_rn(m, 127.f));
    const float sf = __half2float(sh);
    float q = 0.f;
    if (sf != 0.f) q = fminf(fmaxf(rintf(__fdiv_rn(v, sf)), -127.f), 127.f);
    sh_out = __half_as_ushort(sh);
    q_out = (int)q;
    cb_out = q * sf;
}

// The six encode steps of one unit on one warp.
template <int BITS>
__device__ __forceinline__ void encode_body(const Geom& G, const State& S, const __nv_bfloat16* bs,
                                            const EncScratch& W, int unit, const UnitIn& in) {
    const int lane = threadIdx.x & 31;
    const int P = G.r_max + 2;
    float* xs = W.xs;
    float* cs = W.cs;
    int8_t* cstage = W.cstage;
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
        //      Lane takes the pairs j = 2 lane, 2 lane + 1 and 64 + 2 lane, 65 + 2 lane (one
        //      32-bit basis load a pair, x four channels a load); each j's chain runs over i in
        //      order, so the lane assignment does not change a result.
        {
            float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
            const bool on1 = 64 + 2 * lane < R;           // R is a multiple of 8: pairs are whole
            const bool on0 = 2 * lane < R;
#pragma unroll 2
            for (int i = 0; i < kD; i += 4) {
                const float4 x4 = *reinterpret_cast<const float4*>(xs + i);
                const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
                for (int ii = 0; ii < 4; ++ii) {
                    const __nv_bfloat16* brow = bz + (size_t)(i + ii) * P + 2 * lane;
                    if (on0) {
                        const uint32_t w = *reinterpret_cast<const uint32_t*>(brow);
                        acc[0][0] = __fmaf_rn(bf16lo(w), xv[ii], acc[0][0]);
                        acc[0][1] = __fmaf_rn(bf16hi(w), xv[ii], acc[0][1]);
                    }
                    if (on1) {
                        const uint32_t w = *reinterpret_cast<const uint32_t*>(brow + 64);
                        acc[1][0] = __fmaf_rn(bf16lo(w), xv[ii], acc[1][0]);
                        acc[1][1] = __fmaf_rn(bf16hi(w), xv[ii], acc[1][1]);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int j = 64 * q + 2 * lane;
                if (j >= R) continue;
                if (in.dbg) *reinterpret_cast<float2*>(in.dbg + j) = make_float2(acc[q][0], acc[q][1]);
                if (G.c8) {                               // raw projections; the blocks below
                    *reinterpret_cast<float2*>(cs + j) = make_float2(acc[q][0], acc[q][1]);
                } else {
                    __nv_bfloat162 cb;
                    cb.x = __float2bfloat16_rn(acc[q][0]);
                    cb.y = __float2bfloat16_rn(acc[q][1]);
                    *reinterpret_cast<float2*>(cs + j) = make_float2(__bfloat162float(cb.x), __bfloat162float(cb.y));
                    *reinterpret_cast<__nv_bfloat162*>(blk + (size_t)(j >> 3) * 1024 + dst.row * 16 + (j & 7) * 2) = cb;
                }
            }
            if (G.c8) {
                // the 8-bit blockwise form: lane j = lane + 32 jj, a half warp a block of 16
                __syncwarp();
#pragma unroll
                for (int jj = 0; jj < kMaxRank / 32; ++jj) {
                    if (32 * jj >= R) break;                   // uniform: R is a multiple of 16
                    const int j = lane + 32 * jj;
                    uint16_t sh;
                    int qc;
                    float cb;
                    quantize_coeff8(j < R ? cs[j] : 0.f, sh, qc, cb);
                    if (j < R) {
                        cs[j] = cb;
                        blk[z ? vc8_code_off(j, dst.row) : kc8_code_off(j, dst.row)] = (uint8_t)(int8_t)qc;
                        if ((j & 15) == 0)
                            *reinterpret_cast<uint16_t*>(blk + (z ? vc8_scale_off(R, j >> 4, dst.row)
                                                                  : kc8_scale_off(R, j >> 4, dst.row))) = sh;
                    }
                }
            }
        }
        __syncwarp();
        // ---- 3: residual against the stored coefficients (fma chain over j from +0), the
        //      basis read a pair of j at a time
        float r[4];
        {
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j0 = 0; j0 < R; j0 += 8) {           // R is a multiple of 8
                const float4 c0 = *reinterpret_cast<const float4*>(cs + j0);
                const float4 c1 = *reinterpret_cast<const float4*>(cs + j0 + 4);
                const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int jj = 0; jj < 8; jj += 2) {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const uint32_t w = *reinterpret_cast<const uint32_t*>(bz + (size_t)(lane + 32 * m) * P + j0 + jj);
                        a[m] = __fmaf_rn(bf16lo(w), cv[jj], a[m]);
                        a[m] = __fmaf_rn(bf16hi(w), cv[jj + 1], a[m]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) r[m] = __fsub_rn(xr[m], a[m]);
        }
        quantize_store<BITS>(r, blk, R, dst.row, G.ts[dst.k], xs, reinterpret_cast<uint8_t*>(cstage), G.c8, in.gate);
    } while (false);
    __syncwarp();
}


}  // namespace dwkv
