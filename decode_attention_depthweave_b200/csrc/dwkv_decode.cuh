// dwkv_decode.cuh -- fused split-K decode attention (and the probe) over the compressed
// cache.  "DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization for
// Long-Context KV Cache Compression", §3 Method: the fused kernel loads the shared basis,
// dequantises only the routed residual channels and feeds the attention score directly,
// never writing reconstructed keys / values (Eq. (1) evaluated inside attention); the
// probe is Eq. (3) with the with-residual output as the reference.
//
// For the 4 query heads q_h of kv-head h (tau * log2 e folded in, so exp2 can be used):
//   qt = B_K^T q                                   (once per CTA, B_K bulk-copied to smem)
//   s_t = qt[:r_t] . c^K_t + scale^K_t sum_i q[idx^K_ti] code^K_ti
//   online softmax over t;  acc_c += C^V^T p (coefficient space);
//   acc_r += R^V^T (p * scale^V) (residual space, R^V the dense residual codes)
//   o = (B_V acc_c + acc_r) / l                   (B_V applied once per CTA)
//
// Tensor cores take the dense, tier-homogeneous coefficient blocks: the page's 64 x r_t
// coefficient tile against q~ (scores) and against p (values), with q~ and p split into bf16
// hi + lo halves (two MMA columns each), so products keep ~16 significant bits and accumulate
// in fp32.  The value residual is expanded into a dense int8 tile [128 channels x 32 tokens]
// and multiplied by the weights p * scale^V held as 16-bit fixed point (two byte limbs per
// head, relative to the half page's largest weight) with integer MMAs.  The key residual is
// a gather-dot on the CUDA cores (lane = token) from a bf16 table of q.
//
// Work split: a CTA takes a cost-balanced run of one (sequence, kv-head)'s pages (pages are
// tier-homogeneous; a page costs its bytes plus a per-token weight), visited from the highest
// tier down.  The producer warp (lane 0) places the page chunks back to back in a byte ring
// of shared memory with cp.async.bulk (no multicast); its 32 lanes resolve page ids a batch
// ahead.  The 12 consumer warps take the half pages (32 tokens) round robin, each with its
// own softmax state.  The CTA merges its warps' states into one partial record {M, L, o},
// and the last CTA of the (sequence, kv-head) (atomic ticket, no waiting) merges the records
// and writes the output.
#pragma once
#include "dwkv_encode.cuh"

namespace dwkv {

namespace decode_detail {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;   // keep a stale max while the new one is < 2^8 larger

// x ~= hi + lo with both halves bf16, rounding to nearest (prologue only)
__device__ __forceinline__ void split_bf16_rn(float x, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    hi = (uint32_t)__bfloat16_as_ushort(h);
    lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x - __bfloat162float(h)));
}
// Two values as bf16 hi halves (truncated) in one word, and their remainders' hi halves in
// another: x - trunc16(x) is exact in fp32 and its own truncation leaves < 2^-14 |x|.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
    const float ra = a - __uint_as_float(ua & 0xffff0000u);
    const float rb = b - __uint_as_float(ub & 0xffff0000u);
    hi = __byte_perm(ua, ub, 0x7632);
    lo = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Four residual codes as signed bytes in one word (byte j = code j): int8 codes as stored;
// int4 codes as 16 x code (the nibble moved to the byte's high half, which keeps its sign), the
// factor 1/16 going into the dequantisation.  `cw` holds the 4 codes in its low 32 / 16 bits.
template <int BITS>
__device__ __forceinline__ uint32_t code_bytes(uint32_t cw) {
    if (BITS == 8) return cw;
    const uint32_t y = __byte_perm(cw, 0u, 0x1100);              // bytes b0 b0 b1 b1
    // bytes 0, 2 from y << 4 (low nibbles moved up), bytes 1, 3 from y; clear the low nibbles
    const uint32_t z = ((y << 4) & 0x00FF00FFu) | (y & 0xFF00FF00u);
    return z & 0xF0F0F0F0u;
}
constexpr float kCodeUnit4 = 1.0f / 16.0f;              // value of one int4 tile unit

// A row of NB bytes (NB a multiple of 4, the address aligned to the widest access used) as
// 32-bit words, in as few shared-memory accesses as the size allows.
template <int NB>
__device__ __forceinline__ void ld_row(const uint8_t* p, uint32_t (&w)[NB / 4 > 0 ? NB / 4 : 1]) {
    if constexpr (NB % 16 == 0) {
#pragma unroll
        for (int i = 0; i < NB / 16; ++i) {
            const uint4 v = reinterpret_cast<const uint4*>(p)[i];
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else if constexpr (NB % 8 == 0) {
#pragma unroll
        for (int i = 0; i < NB / 8; ++i) {
            const uint2 v = reinterpret_cast<const uint2*>(p)[i];
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < NB / 4; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
    }
}

// A row of n in {1, 2, 4, 8} bytes (aligned to its size) into one or two words.
__device__ __forceinline__ void load_small_row(const uint8_t* p, int n, uint32_t& w0, uint32_t& w1) {
    if (n == 8) {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        w0 = v.x;
        w1 = v.y;
    } else if (n == 4) {
        w0 = *reinterpret_cast<const uint32_t*>(p);
    } else if (n == 2) {
        w0 = *reinterpret_cast<const uint16_t*>(p);
    } else if (n == 1) {
        w0 = *p;
    }
}
// Code e of a row of at most 8 codes held in (w0, w1): int8 bytes, or int4 nibbles with the
// even slot low.
template <int BITS>
__device__ __forceinline__ float small_code(uint32_t w0, uint32_t w1, int e) {
    if (BITS == 8) return (float)(int8_t)__byte_perm(e < 4 ? w0 : w1, 0u, 0x4440 + (e & 3));
    return (float)((int32_t)(w0 << (28 - 4 * e)) >> 28);
}

// Score buffer of a half page: the hi and lo column halves as two [32 tokens][4 heads] fp32
// blocks, the second 16 floats further on so that the stores of both halves from one MMA
// fragment fall in distinct banks.
constexpr int kSLo = 32 * 4 + 16;

template <int RMAX, bool PROBE>
struct WarpAcc {
    float c[RMAX / 16][4];                 // coefficient-space values, D layout (row j, col n)
    float r[8][2];                         // residual-space values: channels 16i+g, 16i+g+8 of head c
    float c2[PROBE ? RMAX / 16 : 1][4];    // probe: no-residual coefficient-space values
    float m[kGQ], l[kGQ], m2[kGQ], l2[kGQ];
};

// Rescale the D-layout accumulators: lane column pair (2c, 2c+1) holds heads (2c)&3, (2c+1)&3.
template <int N>
__device__ __forceinline__ void rescale_d(float (&d)[N][4], float a0, float a1) {
#pragma unroll
    for (int i = 0; i < N; ++i) { d[i][0] *= a0; d[i][1] *= a1; d[i][2] *= a0; d[i][3] *= a1; }
}

// Dense value-residual tile of one warp: 128 channel rows x 32 tokens of int8 codes (zero
// where a token has no entry), stored as two sub-tiles [128][16] (tokens 0-15, 16-31) with
// 16-byte rows: the 8 rows of an ldmatrix are then 128 contiguous bytes.
__device__ __forceinline__ uint32_t rd_off(uint32_t row, uint32_t tok) {
    return (tok >> 4) * 2048u + row * 16u + (tok & 15u);
}
// 16-bit fixed-point weights of a half page: one row of 32 tokens per head, 96-byte pitch.  A
// token's weight is one 16-bit store; the integer MMA's B operand (column n = 2 h + limb, limb
// 0 the high byte, 1 the low byte; k = token) is rebuilt from 8-byte loads by byte permutes.
// With the 96-byte pitch the four heads' rows fall on distinct banks for both fragment loads.
constexpr uint32_t kWhPitch = 96;
__device__ __forceinline__ void store_w16(uint8_t* tile, int h, int lane, uint32_t v) {
    *reinterpret_cast<uint16_t*>(tile + h * kWhPitch + 2 * lane) = (uint16_t)v;
}
__device__ __forceinline__ void load_wfrag(const uint8_t* tile, int g, int c, uint32_t (&b)[2]) {
    const uint8_t* row = tile + (g >> 1) * kWhPitch + 8 * c;
    const uint2 x0 = *reinterpret_cast<const uint2*>(row);          // tokens 4c .. 4c + 3
    const uint2 x1 = *reinterpret_cast<const uint2*>(row + 32);     // tokens 16 + 4c ..
    const uint32_t sel = (g & 1) ? 0x6420u : 0x7531u;               // low bytes : high bytes
    b[0] = __byte_perm(x0.x, x0.y, sel);
    b[1] = __byte_perm(x1.x, x1.y, sel);
}

// Rescale the 8-bit-coefficient accumulators: [i][0] row g, [i][1] row g + 8, both of head c.
template <int N>
__device__ __forceinline__ void rescale_c8(float (&d)[N][4], float a) {
#pragma unroll
    for (int i = 0; i < N; ++i) { d[i][0] *= a; d[i][1] *= a; }
}

// One warp's half of a tier-R page: tokens [32*half, 32*half + 32) of the page's 64 slots,
// `nv` of them live.  `K` points at the page chunk's key block.
// S >= 0: every token has S residual channels.  S < 0 (routed residual counts): the page's
// tokens have s_rt in {0, 2, 4, 8}.
// C8: coefficients in the 8-bit blockwise form (kc8_* / vc8_* layouts): qb holds q~ 2^E as
// f16 hi / lo fragments (kexp = 2^-E), and the A.c / A.c2 accumulators hold rows g, g + 8 of
// head c at [i][0], [i][1]; cw is the warp's two coefficient limb tiles.
template <int R, int S, int BITS, bool PROBE, int RMAX, bool C8>
__device__ __forceinline__ void half_page(const uint8_t* __restrict__ K, int half, int nv,
                                          const uint32_t (&qb)[RMAX / 16][2], const uint2* __restrict__ qh,
                                          float qscale, uint8_t* small, uint8_t* rd, uint32_t zero_addr,
                                          WarpAcc<RMAX, PROBE>& A, int lane, int s_rt, uint8_t* cw, float kexp) {
    constexpr bool ROUTED = S < 0;
    constexpr int KS = R >= 16 ? R / 16 : 1;         // 16-wide coefficient steps
    static_assert(!C8 || R % 16 == 0, "8-bit coefficients come in blocks of 16");
    const int s_ = ROUTED ? s_rt : S;                // residual channels of this page's tokens
    const uint32_t kOffIdx = (C8 ? 72u : 128u) * R, kOffCodes = kOffIdx + 64u * s_;
    const uint32_t kOffSc = kOffCodes + ((8u * s_ * BITS + 127u) & ~127u);
    const uint32_t kBlk = kOffSc + 128u;
    const uint8_t* V = K + kBlk;
    const int tb = 32 * half;
    const uint32_t kaddr = smem_addr(K), vaddr = smem_addr(V);
    float* Ssm = reinterpret_cast<float*>(small);
    uint8_t* Psm = small + 32 * 16;
    uint8_t* Wsm = small + 64 * 16;
    uint8_t* P2sm = small + 96 * 16;
    const int g = lane >> 2, c = lane & 3, mi = lane >> 3, rr = lane & 7;

    // ---------------- 1. coefficient scores: [32 tokens x R] . [R x 8] on the tensor cores
    {
        float d[2][4];
        if constexpr (C8) {
            // per block of 16: the codes as exact f16 against q~ 2^E (f16 hi / lo), then the
            // block's per-token scale on the two rows of the fragment (2^-E once at the end)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                d[mt][0] = d[mt][1] = d[mt][2] = d[mt][3] = 0.f;
                const int t0 = tb + 16 * mt + g;
#pragma unroll
                for (int b = 0; b < KS; ++b) {
                    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(K + b * 1024 + t0 * 16 + 4 * c);
                    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(K + b * 1024 + (t0 + 8) * 16 + 4 * c);
                    const uint32_t a[4] = {s8x2_to_f16x2(w0, 0), s8x2_to_f16x2(w1, 0), s8x2_to_f16x2(w0, 1),
                                           s8x2_to_f16x2(w1, 1)};
                    float e[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_f16(e, a, qb[b]);
                    const uint32_t sw = *reinterpret_cast<const uint32_t*>(K + kc8_scale_off(R, b, t0));
                    const float s0 = __half2float(__ushort_as_half((unsigned short)(sw & 0xffffu)));
                    const float s1 = __half2float(__ushort_as_half((unsigned short)(sw >> 16)));
                    d[mt][0] = fmaf(s0, e[0], d[mt][0]);
                    d[mt][1] = fmaf(s0, e[1], d[mt][1]);
                    d[mt][2] = fmaf(s1, e[2], d[mt][2]);
                    d[mt][3] = fmaf(s1, e[3], d[mt][3]);
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) d[mt][e] *= kexp;           // 2^-E: exact
            }
        } else {
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            d[mt][0] = d[mt][1] = d[mt][2] = d[mt][3] = 0.f;
            const uint32_t tok = tb + 16 * mt + (mi & 1) * 8 + rr;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const uint32_t kc = 2 * ks + (mi >> 1);
                const uint32_t addr = (kc * 8 < (uint32_t)R) ? kaddr + kc * 1024 + tok * 16 : zero_addr;
                uint32_t a[4];
                ldsm_x4(addr, a);
                mma_bf16(d[mt], a, qb[ks]);
            }
        }
        }
        // S: MMA columns 0-3 (the hi parts of heads 0-3) at [token][head], columns 4-7 (the lo
        // parts) kSLo floats on (summed per token below); S spans the P buffer and the start of
        // the W buffer too, both written only after every lane has read S
        float* sp = Ssm + (c >> 1) * kSLo + 2 * (c & 1);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            *reinterpret_cast<float2*>(sp + (16 * mt + g) * 4) = make_float2(d[mt][0], d[mt][1]);
            *reinterpret_cast<float2*>(sp + (16 * mt + g + 8) * 4) = make_float2(d[mt][2], d[mt][3]);
        }
    }
    __syncwarp();

    // ---------------- 2. key residual gather-dot and the full scores (lane = token)
    const int t = tb + lane;
    const bool live = lane < nv;
    float sc[kGQ], sc2[kGQ];
    {
#pragma unroll
        for (int h = 0; h < kGQ; ++h) { sc[h] = -INFINITY; sc2[h] = -INFINITY; }
        float4 sv;
        {
            const float4 s0 = *reinterpret_cast<const float4*>(Ssm + lane * 4);
            const float4 s1 = *reinterpret_cast<const float4*>(Ssm + kSLo + lane * 4);
            sv = make_float4(s0.x + s1.x, s0.y + s1.y, s0.z + s1.z, s0.w + s1.w);
        }
        __syncwarp();                                   // S is dead from here (P overwrites it)
        if (live) {
            float ra[kGQ] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (ROUTED) {
                // a page of the routed layout: s_ in {0, 2, 4, 8} channels a token, each row in one load
                if (s_ > 0) {
                    uint32_t i0 = 0, i1 = 0, c0 = 0, c1 = 0;
                    load_small_row(K + kOffIdx + t * s_, s_, i0, i1);
                    load_small_row(K + kOffCodes + t * (s_ * BITS / 8), s_ * BITS / 8, c0, c1);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (e < s_) {
                            const uint32_t i = __byte_perm(e < 4 ? i0 : i1, 0u, 0x4440 + (e & 3));
                            const float cf = small_code<BITS>(c0, c1, e);
                            const uint2 q = qh[i];
                            ra[0] = fmaf(bf16lo(q.x), cf, ra[0]);
                            ra[1] = fmaf(bf16hi(q.x), cf, ra[1]);
                            ra[2] = fmaf(bf16lo(q.y), cf, ra[2]);
                            ra[3] = fmaf(bf16hi(q.y), cf, ra[3]);
                        }
                    }
                }
            }
            // the token's channel indices and codes, each row in one or two vector loads
            constexpr int SF = ROUTED ? 0 : S;
            constexpr int kCB = SF * BITS / 8;
            uint32_t ixw[SF / 4 > 0 ? SF / 4 : 1], cw[kCB / 4 > 0 ? kCB / 4 : 1];
            if (SF) {
                ld_row<SF>(K + kOffIdx + t * SF, ixw);
                ld_row<kCB>(K + kOffCodes + t * kCB, cw);
            }
#pragma unroll
            for (int ch = 0; ch < SF; ch += 8) {
                const uint2 ix = make_uint2(ixw[ch / 4], ixw[ch / 4 + 1]);
                // codes as biased bytes (code + 2^(b-1)), each turned into a float by placing it in
                // the mantissa of 2^23 and subtracting 2^23 + 2^(b-1)
                uint32_t cb0, cb1;
                if (BITS == 8) {
                    cb0 = cw[ch / 4] ^ 0x80808080u;
                    cb1 = cw[ch / 4 + 1] ^ 0x80808080u;
                } else {
                    const uint32_t w = cw[ch / 8] ^ 0x88888888u;
                    cb0 = w & 0x0F0F0F0Fu;                      // codes 0, 2, 4, 6
                    cb1 = (w >> 4) & 0x0F0F0F0Fu;               // codes 1, 3, 5, 7
                }
                constexpr float kBias = BITS == 8 ? 8388736.0f : 8388616.0f;    // 2^23 + 2^(b-1)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t i = __byte_perm(e < 4 ? ix.x : ix.y, 0u, 0x4440 + (e & 3));
                    const uint32_t src = BITS == 8 ? (e < 4 ? cb0 : cb1) : ((e & 1) ? cb1 : cb0);
                    const uint32_t sel = BITS == 8 ? (e & 3) : (e >> 1);
                    const float cf = __uint_as_float(__byte_perm(src, 0x4B000000u, 0x7440 + sel)) - kBias;
                    const uint2 q = qh[i];                // the 4 heads' q_i as bf16 (exact)
                    ra[0] = fmaf(bf16lo(q.x), cf, ra[0]);
                    ra[1] = fmaf(bf16hi(q.x), cf, ra[1]);
                    ra[2] = fmaf(bf16lo(q.y), cf, ra[2]);
                    ra[3] = fmaf(bf16hi(q.y), cf, ra[3]);
                }
            }
            const float scale =
                s_ ? __half2float(*reinterpret_cast<const __half*>(K + kOffSc + t * 2)) * qscale : 0.f;
            sc[0] = fmaf(scale, ra[0], sv.x);
            sc[1] = fmaf(scale, ra[1], sv.y);
            sc[2] = fmaf(scale, ra[2], sv.z);
            sc[3] = fmaf(scale, ra[3], sv.w);
            sc2[0] = sv.x; sc2[1] = sv.y; sc2[2] = sv.z; sc2[3] = sv.w;
        }
    }

    // ---------------- 3. online softmax (lazy rescale), p as bf16 hi/lo rows, p * scale^V as
    //                     fixed-point byte limbs
    float wdq = 0.f;                                   // this lane's head c: value of one limb unit
    float p1[kGQ], p2v[PROBE ? kGQ : 1];               // this lane's token weights (with / without residual)
    {
        // The running max only moves when some score exceeds it by the slack (one vote);
        // otherwise p = exp2(s - m) <= 2^slack stays safe in fp32.
        float alpha[kGQ];
        bool over = false;
#pragma unroll
        for (int h = 0; h < kGQ; ++h) over |= sc[h] > A.m[h] + kRescaleSlack;
        if (__any_sync(0xffffffffu, over)) {
#pragma unroll
            for (int h = 0; h < kGQ; ++h) {
                const float ml = warp_max(sc[h]);
                alpha[h] = 1.f;
                if (ml > A.m[h] + kRescaleSlack) {
                    alpha[h] = exp2f(A.m[h] - ml);
                    A.m[h] = ml;
                }
                A.l[h] *= alpha[h];
            }
            const float ac = alpha[c];
            if constexpr (C8) rescale_c8(A.c, ac);
            else rescale_d(A.c, alpha[(2 * c) & 3], alpha[(2 * c + 1) & 3]);
#pragma unroll
            for (int i = 0; i < 8; ++i) { A.r[i][0] *= ac; A.r[i][1] *= ac; }
        }
        float p[kGQ];
#pragma unroll
        for (int h = 0; h < kGQ; ++h) {
            p[h] = exp2f(sc[h] - A.m[h]);      // dead lanes: exp2(-inf) = 0
            A.l[h] += p[h];
            p1[h] = p[h];
        }
        if constexpr (!C8) {
            uint4 pr;
            split2(p[0], p[1], pr.x, pr.z);
            split2(p[2], p[3], pr.y, pr.w);
            *reinterpret_cast<uint4*>(Psm + lane * 16) = pr;
        }
        if (s_) {
            // w = p * scale^V as 16-bit fixed point per head, in units of 2^(E-15) with E the
            // exponent of the half page's largest w: two byte limbs (hi, lo) per head
            const float scv = live ? __half2float(*reinterpret_cast<const __half*>(V + kOffSc + t * 2)) : 0.f;
#pragma unroll
            for (int h = 0; h < kGQ; ++h) {
                const float wv = p[h] * scv;                              // >= 0
                const uint32_t eb = __reduce_max_sync(0xffffffffu, __float_as_uint(wv) >> 23);
                uint32_t v = 0;
                if (eb >= 16u) v = min(__float2uint_rn(wv * __uint_as_float((269u - eb) << 23)), 65535u);
                store_w16(Wsm, h, lane, v);
                if (c == h) wdq = eb >= 16u ? __uint_as_float((eb - 15u) << 23) : 0.f;   // 2^(E-15)
            }
            if (BITS == 4) wdq *= kCodeUnit4;
        }
        if (PROBE) {
            bool over2 = false;
#pragma unroll
            for (int h = 0; h < kGQ; ++h) over2 |= sc2[h] > A.m2[h] + kRescaleSlack;
            if (__any_sync(0xffffffffu, over2)) {
#pragma unroll
                for (int h = 0; h < kGQ; ++h) {
                    const float ml = warp_max(sc2[h]);
                    alpha[h] = 1.f;
                    if (ml > A.m2[h] + kRescaleSlack) {
                        alpha[h] = exp2f(A.m2[h] - ml);
                        A.m2[h] = ml;
                    }
                    A.l2[h] *= alpha[h];
                }
                if constexpr (C8) rescale_c8(A.c2, alpha[c]);
                else rescale_d(A.c2, alpha[(2 * c) & 3], alpha[(2 * c + 1) & 3]);
            }
#pragma unroll
            for (int h = 0; h < kGQ; ++h) {
                p[h] = exp2f(sc2[h] - A.m2[h]);
                A.l2[h] += p[h];
                p2v[h] = p[h];
            }
            if constexpr (!C8) {
                uint4 p2;
                split2(p[0], p[1], p2.x, p2.z);
                split2(p[2], p[3], p2.y, p2.w);
                *reinterpret_cast<uint4*>(P2sm + lane * 16) = p2;
            }
        }
    }
    __syncwarp();

    // ---------------- 4. coefficient-space values: acc_c[j][n] += sum_t C^V[t][j] P[t][n]
    if constexpr (C8) {
        // 8-bit form, per block b of 16: acc_c[16 b + e][h] += sum_t code[t][e] w_b[t][h] with
        // w_b = p scale_b as 16-bit fixed point (two byte limbs, unit 2^(E-15) from the half
        // page's largest w_b of head h), one integer MMA over the half page's 32 tokens
        constexpr int NB = R / 16;
        constexpr uint32_t kTile = PROBE ? 768u : 384u;
        float svb[NB];
        {
            const uint8_t* sp = V + vc8_scale_off(R, 0, live ? t : 0);
            uint16_t hs[NB];
            if constexpr (NB == 1) hs[0] = *reinterpret_cast<const uint16_t*>(sp);
            else if constexpr (NB == 2) { const uint32_t w = *reinterpret_cast<const uint32_t*>(sp); hs[0] = (uint16_t)w; hs[1] = (uint16_t)(w >> 16); }
            else if constexpr (NB == 4) {
                const uint2 w = *reinterpret_cast<const uint2*>(sp);
                hs[0] = (uint16_t)w.x; hs[1] = (uint16_t)(w.x >> 16); hs[2] = (uint16_t)w.y; hs[3] = (uint16_t)(w.y >> 16);
            } else {
                const uint4 w = *reinterpret_cast<const uint4*>(sp);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) { hs[2 * q] = (uint16_t)ww[q]; hs[2 * q + 1] = (uint16_t)(ww[q] >> 16); }
            }
#pragma unroll
            for (int b = 0; b < NB; ++b) svb[b] = live ? __half2float(__ushort_as_half(hs[b])) : 0.f;
        }
        const int arow = rr + 8 * (mi & 1), tcq = (tb >> 4) + (mi >> 1);
        const uint32_t aoff = (uint32_t)arow * 64u + 16u * (uint32_t)((tcq ^ (arow >> 1)) & 3);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            uint8_t* tile = cw + (b & 1) * kTile;
            float wq = 0.f, wq2 = 0.f;
#pragma unroll
            for (int h = 0; h < kGQ; ++h) {
                const float wv = p1[h] * svb[b];                          // >= 0
                const uint32_t eb = __reduce_max_sync(0xffffffffu, __float_as_uint(wv) >> 23);
                uint32_t v = 0;
                if (eb >= 16u) v = min(__float2uint_rn(wv * __uint_as_float((269u - eb) << 23)), 65535u);
                store_w16(tile, h, lane, v);
                if (c == h) wq = eb >= 16u ? __uint_as_float((eb - 15u) << 23) : 0.f;
                if constexpr (PROBE) {
                    const float w2 = p2v[h] * svb[b];
                    const uint32_t e2 = __reduce_max_sync(0xffffffffu, __float_as_uint(w2) >> 23);
                    uint32_t v2 = 0;
                    if (e2 >= 16u) v2 = min(__float2uint_rn(w2 * __uint_as_float((269u - e2) << 23)), 65535u);
                    store_w16(tile + 4 * kWhPitch, h, lane, v2);
                    if (c == h) wq2 = e2 >= 16u ? __uint_as_float((e2 - 15u) << 23) : 0.f;
                }
            }
            __syncwarp();
            uint32_t a[4];
            ldsm_x4(vaddr + (uint32_t)b * 1024u + aoff, a);
            {
                uint32_t bb[2];
                load_wfrag(tile, g, c, bb);
                int dd[4] = {0, 0, 0, 0};
                mma_s8u8(dd, a, bb);
                A.c[b][0] = fmaf(wq, (float)(dd[0] * 256 + dd[1]), A.c[b][0]);
                A.c[b][1] = fmaf(wq, (float)(dd[2] * 256 + dd[3]), A.c[b][1]);
            }
            if constexpr (PROBE) {
                uint32_t bb[2];
                load_wfrag(tile + 4 * kWhPitch, g, c, bb);
                int dd[4] = {0, 0, 0, 0};
                mma_s8u8(dd, a, bb);
                A.c2[b][0] = fmaf(wq2, (float)(dd[0] * 256 + dd[1]), A.c2[b][0]);
                A.c2[b][1] = fmaf(wq2, (float)(dd[2] * 256 + dd[3]), A.c2[b][1]);
            }
        }
    } else {
        const uint32_t paddr = smem_addr(Psm), p2addr = smem_addr(P2sm);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t b[2], b2[2];
            ldsm_x2_t(paddr + (16 * ks + (lane & 15)) * 16, b);
            if (PROBE) ldsm_x2_t(p2addr + (16 * ks + (lane & 15)) * 16, b2);
            const uint32_t tloc = 16 * ks + (mi >> 1) * 8 + rr;
#pragma unroll
            for (int mt = 0; mt < KS; ++mt) {
                const uint32_t kc = 2 * mt + (mi & 1);
                const bool ok = (kc * 8 < (uint32_t)R) && ((int)tloc < nv);
                uint32_t a[4];
                ldsm_x4_t(ok ? vaddr + kc * 1024 + (tb + tloc) * 16 : zero_addr, a);
                mma_bf16(A.c[mt], a, b);
                if (PROBE) mma_bf16(A.c2[mt], a, b2);
            }
        }
    }

    // ---------------- 5. residual-space values: acc_r[ch][h] += sum_t R^V[t][ch] w[t][h] as one
    //                     integer MMA per 16 channels over the half page's 32 tokens
    if (s_) {
        if (lane < nv && ROUTED) {                      // scatter this token's codes (lane = token)
            const int tok = tb + lane;
            uint32_t i0 = 0, i1 = 0, c0 = 0, c1 = 0;
            load_small_row(V + kOffIdx + tok * s_, s_, i0, i1);
            load_small_row(V + kOffCodes + tok * (s_ * BITS / 8), s_ * BITS / 8, c0, c1);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                if (e < s_) {
                    const uint32_t ch = __byte_perm(e < 4 ? i0 : i1, 0u, 0x4440 + (e & 3));
                    // int8 codes as stored, int4 codes as 16 x code (see code_bytes)
                    const uint32_t v = BITS == 8 ? __byte_perm(e < 4 ? c0 : c1, 0u, 0x4440 + (e & 3))
                                                 : ((c0 >> (4 * e)) & 0xfu) << 4;
                    rd[rd_off(ch, (uint32_t)lane)] = (uint8_t)v;
                }
            }
        }
        if (lane < nv && !ROUTED) {                     // scatter this token's codes (lane = token)
            const int tok = tb + lane;
            constexpr int SF = ROUTED ? 0 : S;
            constexpr int kCB = SF * BITS / 8;
            uint32_t ixw[SF / 4 > 0 ? SF / 4 : 1], cw[kCB / 4 > 0 ? kCB / 4 : 1];
            ld_row<SF>(V + kOffIdx + tok * SF, ixw);
            ld_row<kCB>(V + kOffCodes + tok * kCB, cw);
#pragma unroll
            for (int e = 0; e < SF; e += 4) {
                const uint32_t ix = ixw[e / 4];
                const uint32_t cbw = code_bytes<BITS>(BITS == 8 ? cw[e / 4] : (cw[e / 8] >> (16 * ((e / 4) & 1))) & 0xffffu);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t ch = __byte_perm(ix, 0u, 0x4440 + q);
                    rd[rd_off(ch, (uint32_t)lane)] = (uint8_t)(cbw >> (8 * q));
                }
            }
        }
        __syncwarp();
        uint32_t b[2];
        load_wfrag(Wsm, g, c, b);
        const uint32_t rdaddr = smem_addr(rd);
        const uint32_t arow = (uint32_t)(rr + 8 * (mi & 1));
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t a[4];
            ldsm_x4(rdaddr + (uint32_t)(mi >> 1) * 2048u + (16u * mt + arow) * 16u, a);
            int d[4] = {0, 0, 0, 0};
            mma_s8u8(d, a, b);
            // |d| <= 32 * 128 * 255, so hi * 256 + lo is exact in int32
            A.r[mt][0] = fmaf(wdq, (float)(d[0] * 256 + d[1]), A.r[mt][0]);
            A.r[mt][1] = fmaf(wdq, (float)(d[2] * 256 + d[3]), A.r[mt][1]);
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i)                     // clear the 4 KB tile for the next half page
            reinterpret_cast<uint4*>(rd)[lane + 32 * i] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
    }
}

template <int S, int BITS, bool PROBE, int RMAX, bool C8>
__device__ __forceinline__ void run_page(int R, const uint8_t* K, int half, int nv, const uint32_t (&qb)[RMAX / 16][2],
                                         const uint2* qs, float qscale, uint8_t* small, uint8_t* rd, uint32_t zero_addr,
                                         WarpAcc<RMAX, PROBE>& A, int lane, int s_rt, uint8_t* cw, float kexp) {
#define DWKV_HP(RR) half_page<RR, S, BITS, PROBE, RMAX, C8>(K, half, nv, qb, qs, qscale, small, rd, zero_addr, A, lane, s_rt, cw, kexp)
    switch (R) {
        case 8: if constexpr (!C8) DWKV_HP(8); break;     // 8-bit coefficient tiers are multiples of 16
        case 16: DWKV_HP(16); break;
        case 32: DWKV_HP(32); break;
        case 64: DWKV_HP(64); break;
        case 128:
            if constexpr (RMAX >= 128) DWKV_HP(128);
            break;
        default: break;
    }
#undef DWKV_HP
}

// Store the 8-bit-coefficient accumulators ([i][0] row 16 i + g, [i][1] row 16 i + g + 8, head
// c) as acc[j][h] (float4 per row j).
template <int N>
__device__ __forceinline__ void store_c8(const float (&d)[N][4], float* dst, int rows, int lane) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int i = 0; i < N; ++i) {
        const int j0 = 16 * i + g, j1 = j0 + 8;
        if (j0 < rows) dst[j0 * 4 + c] = d[i][0];
        if (j1 < rows) dst[j1 * 4 + c] = d[i][1];
    }
}

// Sum hi + lo columns of a D-layout accumulator and store acc[j][h] (float4 per row j).
template <int N>
__device__ __forceinline__ void store_d(float (&d)[N][4], float* dst, int rows, int lane) {
    const int g = lane >> 2, c = lane & 3;
#pragma unroll
    for (int i = 0; i < N; ++i) {
#pragma unroll
        for (int e = 0; e < 4; ++e) d[i][e] += __shfl_xor_sync(0xffffffffu, d[i][e], 2);
        if (c < 2) {
            const int j0 = 16 * i + g, j1 = j0 + 8;
            if (j0 < rows) *reinterpret_cast<float2*>(dst + j0 * 4 + 2 * c) = make_float2(d[i][0], d[i][1]);
            if (j1 < rows) *reinterpret_cast<float2*>(dst + j1 * 4 + 2 * c) = make_float2(d[i][2], d[i][3]);
        }
    }
}

// The fused append's new token, as the CTA that placed and encoded it sees it.
struct TokDest {
    Dest d;
    int ok;
};

// First CTA of a (sequence, kv-head) in a fused append: place the sequence's new position (when
// this layer is its group's first to append it; the counts are left for the last CTA), then
// encode the token's keys (warp 0) and values (warp 1) with both bases staged in the still
// empty page ring.  All threads; ends with the CTA synchronised.
template <int BITS>
__device__ __forceinline__ void owner_append(const Geom& G, const State& St, const DecodeCall& C, int ci, int seq,
                                             int h, uint8_t* ring, TokDest* td) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        Dest d{};
        bool ok;
        if (C.place[ci]) {
            const uint32_t k = C.tier_idx[(size_t)ci * G.Hkv + h];
            ok = k < (uint32_t)G.ntiers;
            if (!ok) set_dev_error(St, 2u /*DWKV_DEV_BAD_TIER*/, (uint32_t)seq, (uint32_t)C.pos[ci]);
            else ok = place_one(G, St, seq, C.g, h, C.pos[ci], k, d, C.lig);
        } else {
            ok = find_dest(G, St, seq, C.g, C.lig, h, C.pos[ci], d);
            if (!ok) set_dev_error(St, 5u /*DWKV_DEV_NO_SLOT*/, (uint32_t)seq, (uint32_t)C.pos[ci]);
        }
        td->d = d;
        td->ok = ok ? 1 : 0;
    }
    // both bases, padded rows, at the start of the ring
    {
        const int RM = G.r_max, P = G.r_max + 2;
        const size_t boff = ((size_t)C.g * G.Hkv + h) * kD * RM;
        const int nvec = kD * RM / 8;
        const uint4* srck = reinterpret_cast<const uint4*>(St.basis_k + boff);
        const uint4* srcv = reinterpret_cast<const uint4*>(St.basis_v + boff);
        __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(ring);
        for (int e = tid; e < 2 * nvec; e += blockDim.x) {
            const uint4 v = __ldg(e < nvec ? srck + e : srcv + (e - nvec));
            const int z = e >= nvec, ev = z ? e - nvec : e;
            const int i = (ev * 8) / RM, j = (ev * 8) % RM;
            uint32_t* dst = reinterpret_cast<uint32_t*>(bs + (size_t)z * kD * P + (size_t)i * P + j);
            dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
        }
    }
    __syncthreads();
    if (warp < 2 && td->ok) {
        UnitIn in;
        in.dst = td->d;
        in.ok = true;
        const __nv_bfloat16* src = (warp ? C.v_new : C.k_new) + ((size_t)ci * G.Hkv + h) * kD;
#pragma unroll
        for (int m = 0; m < 4; ++m) in.xr[m] = __bfloat162float(src[lane + 32 * m]);
        encode_body<BITS>(G, St, reinterpret_cast<const __nv_bfloat16*>(ring), enc_scratch(G, ring, warp), warp, in);
    }
    __syncthreads();
}

// One consumer warp of that CTA (the first to finish its pages), after its pages: attend to the
// new token from its stored bytes (the score over its coefficients and residual, the
// online-softmax update, and its value in both spaces), so no other CTA waits for it.
template <int S, int BITS, int RMAX, bool C8>
__device__ __forceinline__ void add_new_token(const Geom& G, const TokDest& td, const float4* qt, const float4* qs,
                                              WarpAcc<RMAX, false>& A, int lane) {
    const Dest& d = td.d;
    const int R = d.R, row = d.row;
    const int s_ = S < 0 ? G.ts[d.k] : S;            // the token's residual channels
    const uint32_t offIdx = off_idx_of(R, C8), offCodes = off_codes_of(R, s_, C8), offSc = off_scales_of(R, s_, BITS, C8);
    const uint8_t* Kb = d.blk;
    const uint8_t* Vb = d.blk + G.blk_bytes[d.k];
    auto coeff = [&](const uint8_t* blk, int j) -> float {
        if constexpr (C8) {
            const bool key = blk == Kb;
            const int8_t q = (int8_t)blk[key ? kc8_code_off(j, row) : vc8_code_off(j, row)];
            const uint32_t so = key ? kc8_scale_off(R, j >> 4, row) : vc8_scale_off(R, j >> 4, row);
            return (float)q * __half2float(*reinterpret_cast<const __half*>(blk + so));     // exact
        }
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(blk + (size_t)(j >> 3) * 1024 + row * 16 + (j & 7) * 2));
    };
    auto code = [&](const uint8_t* blk, int e) -> float {
        if (BITS == 8) return (float)(int8_t)blk[offCodes + row * s_ + e];
        const uint32_t b = blk[offCodes + row * (s_ / 2) + e / 2];
        return (float)((int32_t)(b << (28 - 4 * (e & 1))) >> 28);
    };
    // score (log2 units: q~ and q carry tau log2 e)
    float sc[kGQ] = {0.f, 0.f, 0.f, 0.f}, rs[kGQ] = {0.f, 0.f, 0.f, 0.f};
    for (int j = lane; j < R; j += 32) {
        const float c = coeff(Kb, j);
        const float4 t = qt[j];
        sc[0] = fmaf(t.x, c, sc[0]); sc[1] = fmaf(t.y, c, sc[1]);
        sc[2] = fmaf(t.z, c, sc[2]); sc[3] = fmaf(t.w, c, sc[3]);
    }
    if (s_ && lane < s_) {
        const float cf = code(Kb, lane);
        const float4 q = qs[Kb[offIdx + row * s_ + lane]];
        rs[0] = q.x * cf; rs[1] = q.y * cf; rs[2] = q.z * cf; rs[3] = q.w * cf;
    }
    const float scK = s_ ? __half2float(*reinterpret_cast<const __half*>(Kb + offSc + row * 2)) : 0.f;
    float s_t[kGQ];
#pragma unroll
    for (int hh = 0; hh < kGQ; ++hh) s_t[hh] = fmaf(scK, warp_sum(rs[hh]), warp_sum(sc[hh]));
    // online softmax: move the max when the token exceeds it by the slack, as the pages do
    float alpha[kGQ];
    bool over = false;
#pragma unroll
    for (int hh = 0; hh < kGQ; ++hh) {
        alpha[hh] = 1.f;
        if (s_t[hh] > A.m[hh] + kRescaleSlack) {
            alpha[hh] = exp2f(A.m[hh] - s_t[hh]);
            A.m[hh] = s_t[hh];
            over = true;
        }
        A.l[hh] *= alpha[hh];
    }
    const int g = lane >> 2, c = lane & 3;
    if (over) {
        if constexpr (C8) rescale_c8(A.c, alpha[c]);
        else rescale_d(A.c, alpha[(2 * c) & 3], alpha[(2 * c + 1) & 3]);
#pragma unroll
        for (int i = 0; i < 8; ++i) { A.r[i][0] *= alpha[c]; A.r[i][1] *= alpha[c]; }
    }
    float p[kGQ];
#pragma unroll
    for (int hh = 0; hh < kGQ; ++hh) {
        p[hh] = exp2f(s_t[hh] - A.m[hh]);
        if (lane == 0) A.l[hh] += p[hh];               // A.l is summed over the lanes later
    }
    // values, coefficient space: rows j = 16 i + g (+8), hi columns (lanes c < 2: heads 2c, 2c+1);
    // 8-bit form: rows j of head c
    if constexpr (C8) {
#pragma unroll
        for (int i = 0; i < RMAX / 16; ++i) {
            const int j0 = 16 * i + g, j1 = j0 + 8;
            if (j0 < R) A.c[i][0] = fmaf(p[c], coeff(Vb, j0), A.c[i][0]);
            if (j1 < R) A.c[i][1] = fmaf(p[c], coeff(Vb, j1), A.c[i][1]);
        }
    } else if (c < 2) {
#pragma unroll
        for (int i = 0; i < RMAX / 16; ++i) {
            const int j0 = 16 * i + g, j1 = j0 + 8;
            if (j0 < R) {
                const float v = coeff(Vb, j0);
                A.c[i][0] = fmaf(p[2 * c], v, A.c[i][0]);
                A.c[i][1] = fmaf(p[2 * c + 1], v, A.c[i][1]);
            }
            if (j1 < R) {
                const float v = coeff(Vb, j1);
                A.c[i][2] = fmaf(p[2 * c], v, A.c[i][2]);
                A.c[i][3] = fmaf(p[2 * c + 1], v, A.c[i][3]);
            }
        }
    }
    // values, residual space: channel ch sits in row (ch & 15) of tile ch >> 4, at lanes g = ch & 7
    if (s_) {
        const float scV = __half2float(*reinterpret_cast<const __half*>(Vb + offSc + row * 2));
        const float pc = p[c] * scV;
        for (int e = 0; e < s_; ++e) {
            const int ch = Vb[offIdx + row * s_ + e];
            if ((ch & 7) != g) continue;
            const float v = pc * code(Vb, e);
            const int mt = ch >> 4, r2 = (ch >> 3) & 1;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i == mt) { if (r2) A.r[i][1] += v; else A.r[i][0] += v; }
        }
    }
}

}  // namespace decode_detail

// BITS: code width; PROBE: second softmax state without the residual; RMAX: accumulator
// rows (>= r_max); S: residual channels per token (0, 8, 16 or 32), or -1 for per-tier counts;
// C8: coefficients in the 8-bit blockwise form.
template <int BITS, bool PROBE, int RMAX, int S, bool C8>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_kernel(const Geom G, const State St, const DecodeCall C) {
    using namespace decode_detail;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    const DecodeSmem L = decode_smem_layout(G, (uint32_t)C.ring_bytes, PROBE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);   // full[kSlots] empty[kSlots] basis table
    const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + kSlots),
                   basis_bar = smem_addr(bars + 2 * kSlots), table_bar = smem_addr(bars + 2 * kSlots + 1);
    float4* qt = reinterpret_cast<float4*>(smem + L.qt);
    float4* qs = reinterpret_cast<float4*>(smem + L.q);
    uint32_t* m_cnt = reinterpret_cast<uint32_t*>(smem + L.misc);      // [8]
    uint32_t* m_P = m_cnt + 8;                                          // [9] page prefix
    uint32_t* m_R = m_P + 9;                                            // [8]
    uint32_t* m_chunk = m_R + 8;                                        // [8]
    uint32_t* m_misc = m_chunk + 8;                                     // p_begin p_end last work
    float* m_state = reinterpret_cast<float*>(smem + L.misc + kMiscState);     // [warps][16]
    float* mf = reinterpret_cast<float*>(smem + L.misc + kMiscFactors);        // [2][warps][4] factors
    uint32_t* m_slot = reinterpret_cast<uint32_t*>(smem + L.misc + kMiscSlots); // ring offset per slot

    // ---- which sequence / split
    int ci = 0;
    {
        int lo = 0, hi = C.n - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (C.split_begin[mid] <= (int)blockIdx.x) lo = mid; else hi = mid - 1;
        }
        ci = lo;
    }
    const int split = blockIdx.x - C.split_begin[ci];
    const int nsplit = C.split_begin[ci + 1] - C.split_begin[ci];
    const int seq = C.seq[ci];
    const size_t basis_off = ((size_t)C.g * G.Hkv + h) * kD * G.r_max;
    TokDest* tokd = reinterpret_cast<TokDest*>(smem + L.tok);
    const bool owner = !PROBE && C.fused && split == 0;
    if (owner) {
        // the new token's keys, values and tier may come from the previous kernel
        grid_dep_wait();
        owner_append<BITS>(G, St, C, ci, seq, h, smem + L.ring, tokd);
    }

    uint32_t cv[kMaxTiers];                 // tier counts (producer lane 0)
    static_assert(kSlots == 32, "the producer's lane i sets up ring slot i");
    if (warp == kConsumerWarps) {
        mbar_init(full0 + 8 * lane, 1);
        mbar_init(empty0 + 8 * lane, 2);      // released by the warps of its two halves
        if (lane == 0) {
            mbar_init(basis_bar, 1);
            mbar_init(table_bar, 1);
        }
        fence_mbar_init();
        __syncwarp();
    }
    if (warp == kConsumerWarps && lane == 0) {
        // B_K into the residual tiles (free until the main loop) and the counts, both in
        // flight across the barrier below
        const uint32_t bytes = (uint32_t)kD * G.r_max * 2;
        mbar_arrive_expect_tx(basis_bar, bytes);
        bulk_g2s(smem_addr(smem + L.rd), St.basis_kt + basis_off, bytes, basis_bar);
        // Until this CTA waits on the previous kernel (programmatic dependent launch), that
        // kernel may still be running; the host says whether the cache state read from here on
        // (counts, slot map, page tables, page bytes) is already final.
        if (!C.early) grid_dep_wait();
        const uint32_t* cnt = St.counts + cnt_index(G, seq, C.g, h);
#pragma unroll
        for (int k = 0; k < kMaxTiers; ++k) cv[k] = k < G.ntiers ? __ldcg(cnt + k) : 0u;
        // fused append: the pages are attended without the new token.  Where it was placed by
        // an earlier layer of the group the counts include it (it is the last slot of its tier);
        // where this launch places it they do not yet (the last CTA adds it).
        if (C.fused && !C.place[ci]) {
            const uint32_t sm = __ldcg(St.slot_map + slot_index(G, seq, C.g, h, C.pos[ci]));
            const uint32_t kt = (sm >> 24) - 1u;
#pragma unroll
            for (int k = 0; k < kMaxTiers; ++k)
                if (sm != 0u && (uint32_t)k == kt && cv[k] > 0u) cv[k] -= 1u;
        }
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ================= producer warp: B_K, the CTA's page range, then page chunks
        if (lane == 0) {
            // Integer costs; each boundary is computed by the same operations in the two CTAs
            // that share it, and the divisions are fp32 estimates corrected to the exact result.
            uint32_t P = 0, rP[kMaxTiers + 1];
            unsigned long long W = 0;
            uint32_t rw[kMaxTiers];
            const uint32_t tokw = (uint32_t)C.tok_weight * kPage;
#pragma unroll
            for (int k = 0; k < kMaxTiers; ++k) {
                const uint32_t np = k < G.ntiers ? (cv[k] + kPage - 1) / kPage : 0u;
                rP[k] = P;
                rw[k] = k < G.ntiers ? G.chunk_bytes[k] + tokw : 1u;
                if (k < G.ntiers) {
                    m_cnt[k] = cv[k];
                    m_P[k] = P;
                    m_R[k] = (uint32_t)G.tiers[k];
                    m_chunk[k] = G.chunk_bytes[k];
                }
                P += np;
                W += (unsigned long long)np * rw[k];
            }
            rP[kMaxTiers] = P;
            m_P[G.ntiers] = P;
            // cost-balanced page range: pages whose first cost unit lies in [lo, hi).  With a
            // fused append, split 0 also places and encodes the token, a fixed cost E
            // (owner_cost, in cost units): it takes an even share of W + E less E (at least 0)
            // and the other splits share the rest evenly, boundary s >= 1 at
            // own + (W - own) (s - 1) / (nsplit - 1), in integers.
            const unsigned long long E = (unsigned long long)C.owner_cost;
            const unsigned long long even = (W + E) / (unsigned long long)nsplit;
            const unsigned long long own = nsplit == 1 ? W : (even > E ? min(even - E, W) : 0ull);
            auto bound = [&](int sidx) -> unsigned long long {
                return sidx == 0 ? 0ull
                                 : own + (W - own) * (unsigned long long)(sidx - 1) / (unsigned long long)(nsplit - 1);
            };
            // ceil(x / w): an fp32 estimate (within a few units for these sizes), then exact
            auto cdiv = [](unsigned long long x, uint32_t w) -> uint32_t {
                uint32_t q = (uint32_t)ceilf(__fdividef((float)x, (float)w));
                while ((unsigned long long)q * w < x) ++q;
                while (q > 0u && (unsigned long long)(q - 1u) * w >= x) --q;
                return q;
            };
            const unsigned long long lo = bound(split);
            const unsigned long long hi = split + 1 == nsplit ? W : min(bound(split + 1), W);
            uint32_t pb = P, pe = P;
            unsigned long long Wk = W;
#pragma unroll
            for (int k = kMaxTiers - 1; k >= 0; --k) {
                const uint32_t np = rP[k + 1] - rP[k];
                const uint32_t w = rw[k];
                Wk -= (unsigned long long)np * w;        // first cost unit of tier k
                if (!np) continue;
                if (lo <= Wk + (unsigned long long)(np - 1) * w) pb = rP[k] + (lo > Wk ? cdiv(lo - Wk, w) : 0u);
                if (hi <= Wk + (unsigned long long)(np - 1) * w) pe = rP[k] + (hi > Wk ? cdiv(hi - Wk, w) : 0u);
            }
            m_misc[0] = pb;
            m_misc[1] = pe > pb ? pe : pb;
            mbar_arrive(table_bar);
        }
        __syncwarp();
        const uint32_t p_begin = m_misc[0], p_end = m_misc[1];
        const uint32_t npages = p_end - p_begin;
        const size_t pbase = page_index(G, seq, C.g, h, 0);
        // The warp resolves 32 pages at a time (global page ids, byte counts) into a small
        // table; lane 0 then places each chunk in the ring and issues its copy.  Chunks are
        // reclaimed oldest first, so the ring holds pages [tail, u) at any time.
        uint32_t* t_src = reinterpret_cast<uint32_t*>(smem + L.misc + kMiscPages);   // [32] pool units
        uint32_t* t_len = t_src + 32;                                                // [32] bytes
        const uint32_t RB = (uint32_t)C.ring_bytes;
        const uint32_t ring = smem_addr(smem + L.ring);
        uint32_t head = 0, tail = 0;
        bool ok = true;
        const uint64_t pol = l2_evict_first_policy();        // pages are read once a launch
        // lane j resolves page b0 + j of each batch; the next batch's ids are requested before
        // lane 0 issues the current batch, so their latency hides behind the issuing
        auto page_id = [&](uint32_t u, uint32_t& len) -> uint32_t {
            const uint32_t p = p_end - 1 - u;               // highest tier first: cheap pages end the run
            int k = 0;
#pragma unroll
            for (int kk = 1; kk < kMaxTiers; ++kk)
                if (kk < G.ntiers && p >= m_P[kk]) k = kk;
            len = m_chunk[k];
            return __ldcg(St.pages + pbase + (size_t)k * G.max_pages + (p - m_P[k]));
        };
        uint32_t nxt_src = 0, nxt_len = 0;
        if (lane < npages) nxt_src = page_id(lane, nxt_len);
        for (uint32_t b0 = 0; b0 < npages && ok; b0 += 32) {
            t_src[lane] = nxt_src;
            t_len[lane] = nxt_len;
            __syncwarp();
            if (b0 + 32 + lane < npages) nxt_src = page_id(b0 + 32 + lane, nxt_len);
            if (lane == 0) {
                const uint32_t nb = min(32u, npages - b0);
                for (uint32_t j = 0; j < nb && ok; ++j) {
                    const uint32_t v = b0 + j, len = t_len[j];
                    uint32_t off = 0;
                    for (;;) {
                        const uint32_t inflight = v - tail;
                        if (inflight == 0) { off = 0; break; }
                        if (inflight < (uint32_t)kSlots) {
                            const uint32_t toff = m_slot[tail % kSlots];
                            if (head > toff) {                     // occupied [toff, head)
                                if (head + len <= RB) { off = head; break; }
                                if (len <= toff) { off = 0; break; }
                            } else if (head + len <= toff) {       // occupied [toff, end) + [0, head)
                                off = head;
                                break;
                            }
                        }
                        if (!mbar_wait(empty0 + 8 * (tail % kSlots), (tail / kSlots) & 1u)) {
                            set_dev_error(St, 6u /*DWKV_DEV_TIMEOUT*/, (uint32_t)seq, v);
                            ok = false;
                            break;
                        }
                        ++tail;
                    }
                    if (!ok) break;
                    const uint32_t sl = v % kSlots;
                    m_slot[sl] = off;
                    head = off + len;
                    mbar_arrive_expect_tx(full0 + 8 * sl, len);
                    bulk_g2s_hint(ring + off, St.data + (size_t)t_src[j] * kUnit + (size_t)C.lig * len, len,
                                  full0 + 8 * sl, pol);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            __syncwarp();
        }
    } else {
        // ================= consumer warps
        uint8_t* rd = smem + L.rd + warp * kRdBytes;
        uint8_t* small = smem + L.small + warp * L.small_stride;
        uint8_t* cw = small + L.CW;
        const uint32_t zero_addr = smem_addr(smem + L.zero);
        const float qscale = G.tau * kLog2e;
        uint2* qh = reinterpret_cast<uint2*>(smem + L.qh);
        {   // B_V, copied into the ring for the CTA merge at the end: warm it into L2 now
            const int lines = kD * G.r_max * 2 / 128;
            for (int x = tid; x < lines; x += kConsumerWarps * 32)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(St.basis_v + basis_off) + 128 * x));
        }
        // q may come from the previous kernel, and so may everything this CTA writes from here
        // on (records, tickets, outputs); the next decode may start once every CTA is past here
        grid_dep_wait();
        grid_dep_launch();
        if (tid < kD) {
            const __nv_bfloat16* q = C.q + ((size_t)ci * G.Hq + (size_t)h * kGQ) * kD + tid;
            const __nv_bfloat16 q0 = q[0], q1 = q[kD], q2 = q[2 * kD], q3 = q[3 * kD];
            qs[tid] = make_float4(__bfloat162float(q0) * qscale, __bfloat162float(q1) * qscale,
                                  __bfloat162float(q2) * qscale, __bfloat162float(q3) * qscale);
            qh[tid] = make_uint2((uint32_t)__bfloat16_as_ushort(q0) | ((uint32_t)__bfloat16_as_ushort(q1) << 16),
                                 (uint32_t)__bfloat16_as_ushort(q2) | ((uint32_t)__bfloat16_as_ushort(q3) << 16));
        }
        if (tid < 8) reinterpret_cast<uint4*>(smem + L.zero)[tid] = make_uint4(0u, 0u, 0u, 0u);
        named_barrier(1, kConsumerWarps * 32);
        bool ok = mbar_wait(basis_bar, 0);
        if (!ok && lane == 0) set_dev_error(St, 6u, (uint32_t)seq, 0xffffffffu);
        // q~[j] = qscale sum_i B_K[i][j] q[i] on the tensor cores: warp m < rq / 16 takes rows
        // j in [16 m, 16 m + 16) as one MMA row tile, A = B_K^T (ldmatrix.trans of the 8 x 8
        // tiles of B_K in the residual tiles), B = q as bf16 (exact) in columns 0-3, fp32
        // accumulation.
        const int rq = G.r_max < 16 ? 16 : G.r_max;
        if (warp < rq / 16) {
            const int g = lane >> 2, c = lane & 3, mi = lane >> 3, rr = lane & 7;
            const uint32_t bk = smem_addr(smem + L.rd);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < kD / 16; ++ks) {
                // matrix mi: rows j 16 warp + 8 (mi & 1) .., columns i 16 ks + 8 (mi >> 1) ..
                const int i = 16 * ks + 8 * (mi >> 1) + rr, j0 = 16 * warp + 8 * (mi & 1);
                uint32_t a[4];
                ldsm_x4_t(bk + tiled_basis_off(i, j0, G.r_max) * 2u, a);
                uint32_t b[2] = {0u, 0u};
                if (g < kGQ) {
#pragma unroll
                    for (int r2 = 0; r2 < 2; ++r2) {
                        const int i0 = 16 * ks + 8 * r2 + 2 * c;
                        const uint2 w0 = qh[i0], w1 = qh[i0 + 1];
                        const uint32_t x0 = g < 2 ? w0.x : w0.y, x1 = g < 2 ? w1.x : w1.y;
                        const uint32_t sh = 16u * (uint32_t)(g & 1);
                        b[r2] = ((x0 >> sh) & 0xffffu) | (((x1 >> sh) & 0xffffu) << 16);
                    }
                }
                mma_bf16(d, a, b);
            }
            if (c < 2) {                                  // columns 2c, 2c+1 = heads
#pragma unroll
                for (int rr2 = 0; rr2 < 2; ++rr2) {
                    const int j = 16 * warp + g + 8 * rr2;
                    const bool on = ok && j < G.r_max;
                    reinterpret_cast<float2*>(qt + j)[c] =
                        make_float2(on ? d[2 * rr2] * qscale : 0.f, on ? d[2 * rr2 + 1] * qscale : 0.f);
                }
            }
        }
        named_barrier(1, kConsumerWarps * 32);
        // q~ as the score MMA's B operand, the same fragments in every warp: built once into
        // qbs [ks][r2][lane] (column n < 4 = bf16 hi of head n, n >= 4 = lo of head n-4).
        // 8-bit coefficients: f16 hi / lo of q~ 2^E instead, E putting max |q~| in [2^14, 2^15)
        // (the f16 range; each warp finds the max itself), and kexp = 2^-E.
        float qsc = 1.f, kexp = 1.f;
        if constexpr (C8) {
            uint32_t mb = 0u;
            for (int k = lane; k < rq; k += 32) {
                const float4 t4 = qt[k];
                mb = max(mb, max(max(__float_as_uint(fabsf(t4.x)), __float_as_uint(fabsf(t4.y))),
                                 max(__float_as_uint(fabsf(t4.z)), __float_as_uint(fabsf(t4.w)))));
            }
            const uint32_t eb = __reduce_max_sync(0xffffffffu, mb) >> 23;      // biased exponent of the max
            if (eb >= 15u && eb < 255u) {
                qsc = __uint_as_float((268u - eb) << 23);                       // 2^(141 - eb)
                kexp = __uint_as_float((eb - 14u) << 23);                       // 2^(eb - 141)
            }
        }
        uint32_t* qbs = reinterpret_cast<uint32_t*>(smem + L.qb);
        for (int x = tid; x < 32 * 2 * (RMAX / 16); x += kConsumerWarps * 32) {
            const int ln = x & 31, ks = (x >> 5) >> 1, r2 = (x >> 5) & 1;
            const int g = ln >> 2, c = ln & 3, n = g & 3;
            const bool lo_half = g >= 4;
            uint32_t pk = 0;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int k = 16 * ks + 8 * r2 + 2 * c + e;
                float v = 0.f;
                if (k < rq) {
                    const float4 t4 = qt[k];
                    v = n == 0 ? t4.x : n == 1 ? t4.y : n == 2 ? t4.z : t4.w;
                }
                uint32_t hi, lo;
                if constexpr (C8) {
                    const float vs = v * qsc;                                   // exact (power of two)
                    const __half hh = __float2half_rn(vs);
                    hi = __half_as_ushort(hh);
                    lo = __half_as_ushort(__float2half_rn(vs - __half2float(hh)));
                } else {
                    split_bf16_rn(v, hi, lo);
                }
                pk |= (lo_half ? lo : hi) << (16 * e);
            }
            qbs[x] = pk;
        }
        named_barrier(1, kConsumerWarps * 32);
        uint32_t qb[RMAX / 16][2];
#pragma unroll
        for (int ks = 0; ks < RMAX / 16; ++ks) {
            qb[ks][0] = qbs[(2 * ks) * 32 + lane];
            qb[ks][1] = qbs[(2 * ks + 1) * 32 + lane];
        }
        {   // the residual tiles held B_K until now; clear this warp's tile
            uint4* z = reinterpret_cast<uint4*>(rd);
            for (int i = lane; i < kRdBytes / 16; i += 32) z[i] = make_uint4(0u, 0u, 0u, 0u);
            __syncwarp();
        }

        WarpAcc<RMAX, PROBE> A;
#pragma unroll
        for (int i = 0; i < RMAX / 16; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) A.c[i][e] = 0.f;
#pragma unroll
        for (int i = 0; i < (PROBE ? RMAX / 16 : 1); ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) A.c2[i][e] = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) { A.r[i][0] = 0.f; A.r[i][1] = 0.f; }
#pragma unroll
        for (int hh = 0; hh < kGQ; ++hh) { A.m[hh] = -INFINITY; A.l[hh] = 0.f; A.m2[hh] = -INFINITY; A.l2[hh] = 0.f; }

        if (ok && !mbar_wait(table_bar, 0)) {
            if (lane == 0) set_dev_error(St, 6u, (uint32_t)seq, 0xfffffffeu);
            ok = false;
        }
        // Work items are half pages, dealt round robin: warp w takes items w, w + 12, ...;
        // item i is half i & 1 of the CTA's page i >> 1.  Both halves of a page release its
        // stage, so the stage frees once the second of its two warps is done.  (A warp only
        // waits for a page the producer will issue: the oldest unreleased page belongs to an
        // item earlier in some warp's sequence than anything that warp waits for.)  Claims from
        // a shared counter balanced the warps' finish no better and cost ~430 cycles an item.
        const uint32_t p_begin = m_misc[0], p_end = m_misc[1];
        const uint32_t nitems = 2 * (p_end - p_begin);
        uint32_t w = (uint32_t)warp;
        while (ok && w < nitems) {
            const uint32_t wn = w + kConsumerWarps;
            const uint32_t u = w >> 1, p = p_end - 1 - u, sl = u % kSlots;
            const int half = (int)(w & 1);
            int k = 0;
            while (k + 1 < G.ntiers && p >= m_P[k + 1]) ++k;
            const int R = (int)m_R[k];
            const uint32_t pit = p - m_P[k], npk = m_P[k + 1] - m_P[k];
            const int nvalid = pit + 1 < npk ? kPage : (int)(m_cnt[k] - pit * kPage);
            if (!mbar_wait(full0 + 8 * sl, (u / kSlots) & 1)) {
                if (lane == 0) set_dev_error(St, 6u, (uint32_t)seq, u);
                ok = false;
                break;
            }
            const int nv = min(max(nvalid - 32 * half, 0), 32);
            if (nv > 0)
                run_page<S, BITS, PROBE, RMAX, C8>(R, smem + L.ring + m_slot[sl], half, nv, qb, qh,
                                               qscale, small, rd, zero_addr, A, lane, G.ts[k], cw, kexp);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * sl);
            w = wn;
        }
        if constexpr (!PROBE) {
            // the warp whose last item comes first in the final round (item nitems - 12) is the
            // first to finish: it attends to the new token
            if (owner && warp == (int)(nitems % kConsumerWarps) && tokd->ok)
                add_new_token<S, BITS, RMAX, C8>(G, *tokd, reinterpret_cast<const float4*>(smem + L.qt), qs, A, lane);
        }
        // ---- per-warp results: acc_c [r_max][4] and acc_r [d][4] into the residual tile,
        //      the probe's acc_c2 into the small buffers; m / l into m_state
        float* oc = reinterpret_cast<float*>(rd);
        float* orr = oc + G.r_max * 4;
        if constexpr (C8) store_c8(A.c, oc, G.r_max, lane);
        else store_d(A.c, oc, G.r_max, lane);
        {
            const int g = lane >> 2, c = lane & 3;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                orr[(16 * i + g) * 4 + c] = A.r[i][0];
                orr[(16 * i + g + 8) * 4 + c] = A.r[i][1];
            }
        }
        if constexpr (PROBE && C8) store_c8(A.c2, reinterpret_cast<float*>(small), G.r_max, lane);
        else if constexpr (PROBE) store_d(A.c2, reinterpret_cast<float*>(small), G.r_max, lane);
        float* ms = m_state + warp * 16;
        float l[kGQ], l2[kGQ];
#pragma unroll
        for (int hh = 0; hh < kGQ; ++hh) { l[hh] = A.l[hh]; l2[hh] = PROBE ? A.l2[hh] : 0.f; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)             // the heads' sums side by side
#pragma unroll
            for (int hh = 0; hh < kGQ; ++hh) {
                l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], o);
                if (PROBE) l2[hh] += __shfl_xor_sync(0xffffffffu, l2[hh], o);
            }
        if (lane == 0) {
#pragma unroll
            for (int hh = 0; hh < kGQ; ++hh) {
                ms[hh] = A.m[hh]; ms[4 + hh] = l[hh];
                ms[8 + hh] = A.m2[hh]; ms[12 + hh] = l2[hh];
            }
        }
    }
    __syncthreads();

    // ================= CTA merge: the warp states -> one partial record
    //   {M[4], L[4], (M2[4], L2[4]), o[4][d] = B_V acc_c + acc_r, (o2[4][d] = B_V acc_c2)}
    // B_V is applied here, once per CTA (tensor cores), so the final merge is a weighted sum.
    // Every page has been attended, so the ring is idle: B_V [d][r_max] goes into it (one bulk
    // copy, in flight while the states merge) after the merged sums' region.
    const uint32_t bv_bytes = (uint32_t)kD * G.r_max * 2;
    const __nv_bfloat16* bvs = reinterpret_cast<const __nv_bfloat16*>(smem + L.ring + kMergeBvOff);
    if (tid == 0) {
        mbar_arrive_expect_tx(basis_bar, bv_bytes);
        bulk_g2s(smem_addr(smem + L.ring + kMergeBvOff), St.basis_v + basis_off, bv_bytes, basis_bar);
    }
    const int nrec = C.total_splits;
    float* rec = C.ws + ((size_t)h * nrec + blockIdx.x) * C.rec_floats;
    const int hdr = PROBE ? 16 : 8;
    if (warp < (PROBE ? 2 : 1)) {
        // lane = (warp w2 = lane / 4 + 8 i, head hh): the CTA max and rescaled sum by shuffles
        const int which = warp, hh = lane & 3;
        constexpr int kRounds = (kConsumerWarps + 7) / 8;
        float m[kRounds];
        float M = -INFINITY;
#pragma unroll
        for (int i = 0; i < kRounds; ++i) {
            const int w2 = (lane >> 2) + 8 * i;
            m[i] = w2 < kConsumerWarps ? m_state[w2 * 16 + which * 8 + hh] : -INFINITY;
            M = fmaxf(M, m[i]);
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float Lsum = 0.f;
#pragma unroll
        for (int i = 0; i < kRounds; ++i) {
            const int w2 = (lane >> 2) + 8 * i;
            if (w2 < kConsumerWarps) {
                const float f = m[i] == -INFINITY ? 0.f : exp2f(m[i] - M);
                mf[which * kConsumerWarps * 4 + w2 * 4 + hh] = f;
                Lsum = fmaf(f, m_state[w2 * 16 + which * 8 + 4 + hh], Lsum);
            }
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
        if (lane < kGQ) {
            rec[which * 8 + hh] = M;
            rec[which * 8 + 4 + hh] = Lsum;
        }
    }
    __syncthreads();
    // merged sums into the idle ring, rows of the 4 heads: cm [r_max][4], racc [d][4],
    // (cm2 [r_max][4]); each warp's sums sit in its residual tile ([j][4] then [i][4]) and,
    // for acc_c2, its small buffer.  A thread per row.
    float* cm = reinterpret_cast<float*>(smem + L.ring);
    const int nrows = G.r_max + kD + (PROBE ? G.r_max : 0);
    for (int e = tid; e < nrows; e += blockDim.x) {
        int which = 0;
        const uint8_t* base = smem + L.rd + (size_t)e * 16;
        uint32_t stride = kRdBytes;
        if (e >= G.r_max + kD) {
            which = 1;
            base = smem + L.small + (size_t)(e - G.r_max - kD) * 16;
            stride = L.small_stride;
        }
        const float4* fw = reinterpret_cast<const float4*>(mf + which * kConsumerWarps * 4);
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w2 = 0; w2 < kConsumerWarps; ++w2) {
            const float4 f = fw[w2];
            const float4 x = *reinterpret_cast<const float4*>(base + w2 * stride);
            v.x = fmaf(f.x, x.x, v.x);
            v.y = fmaf(f.y, x.y, v.y);
            v.z = fmaf(f.z, x.z, v.z);
            v.w = fmaf(f.w, x.w, v.w);
        }
        reinterpret_cast<float4*>(cm)[e] = v;
    }
    __syncthreads();
    const bool bv_ok = mbar_wait(basis_bar, 1);
    if (!bv_ok && tid == 0) set_dev_error(St, 6u, (uint32_t)seq, 0xfffffffdu);
    if (warp < kD / 16) {
        // o[i][h] for the warp's 16 channels: B_V rows (A, ldmatrix) against the merged acc_c as
        // bf16 hi (columns 0-3) + lo (columns 4-7) halves (B), fp32 accumulation
        const int g = lane >> 2, c = lane & 3, n = g & 3;
        const bool lo_half = g >= 4;
        const float* racc = cm + 4 * G.r_max;
        const float* cm2 = cm + 4 * (G.r_max + kD);
        float d[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f};
        // this warp's 16 B_V rows as mma A fragments: rows 16 warp + g (+8), columns
        // 16 ks + 2c (+1, +8, +9)
        const __nv_bfloat16* b0 = bvs + (size_t)(16 * warp + g) * G.r_max + 2 * c;
#pragma unroll
        for (int ks = 0; ks < RMAX / 16; ++ks) {
            if (16 * ks >= G.r_max) break;
            const int k0 = 16 * ks, k1 = 16 * ks + 8;
            uint32_t a[4];
            a[0] = *reinterpret_cast<const uint32_t*>(b0 + k0);
            a[1] = *reinterpret_cast<const uint32_t*>(b0 + 8 * G.r_max + k0);
            a[2] = *reinterpret_cast<const uint32_t*>(b0 + k1);
            a[3] = *reinterpret_cast<const uint32_t*>(b0 + 8 * G.r_max + k1);
            uint32_t b[2], b2[2];
#pragma unroll
            for (int r2 = 0; r2 < 2; ++r2) {
                uint32_t pk = 0, pk2 = 0;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int k = 16 * ks + 8 * r2 + 2 * c + e;
                    uint32_t hi, lo;
                    split_bf16_rn(k < G.r_max ? cm[k * 4 + n] : 0.f, hi, lo);
                    pk |= (lo_half ? lo : hi) << (16 * e);
                    if (PROBE) {
                        split_bf16_rn(k < G.r_max ? cm2[k * 4 + n] : 0.f, hi, lo);
                        pk2 |= (lo_half ? lo : hi) << (16 * e);
                    }
                }
                b[r2] = pk;
                b2[r2] = pk2;
            }
            mma_bf16(d, a, b);
            if (PROBE) mma_bf16(d2, a, b2);
        }
        // lanes c and c^2 hold the hi and lo columns of heads 2(c&1), 2(c&1)+1
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            d[e] += __shfl_xor_sync(0xffffffffu, d[e], 2);
            if (PROBE) d2[e] += __shfl_xor_sync(0xffffffffu, d2[e], 2);
        }
        if (c < 2) {
#pragma unroll
            for (int rr2 = 0; rr2 < 2; ++rr2) {
                const int i = 16 * warp + g + 8 * rr2;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int hh = 2 * c + q;
                    rec[hdr + hh * kD + i] = d[2 * rr2 + q] + racc[i * 4 + hh];
                    if (PROBE) rec[hdr + kGQ * kD + hh * kD + i] = d2[2 * rr2 + q];
                }
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        // one acq_rel ticket: it releases the CTA's record (ordered before this thread by the
        // barrier) at GPU scope, and the last CTA acquires every other CTA's record with it
        uint32_t t;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                     : "=r"(t) : "l"(St.tickets + (size_t)seq * G.Hkv + h) : "memory");
        m_misc[2] = (t == (uint32_t)(nsplit - 1)) ? 1u : 0u;
    }
    __syncthreads();
    if (!m_misc[2]) return;

    // ================= last CTA of (sequence, kv-head): log-sum-exp merge of the records.
    // Every thread requests its outputs' values from the first kChunk records at once while
    // warps 0 (and 1, probe) turn the record headers into weights with shuffles.
    const int r0 = C.split_begin[ci];
    const int RF = C.rec_floats;
    const float* recs = C.ws + ((size_t)h * nrec + r0) * RF;
    float* wgt = reinterpret_cast<float*>(smem + L.small);                        // [2][kMaxSplits][4]
    float* Ls = wgt + 2 * kMaxSplits * kGQ;                                        // [2][4]
    float* red = Ls + 8;                                                           // [2][warps]
    constexpr int kPer = (kGQ * kD + kDecodeThreads - 1) / kDecodeThreads;   // outputs per thread
    constexpr int kChunk = PROBE ? 8 : 32;         // records whose values are held at once
    float v1[kPer][kChunk], v2[kPer][PROBE ? kChunk : 1];
    auto load_chunk = [&](int j0) {
        const int nj = min(kChunk, nsplit - j0);
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int q = tid + k * kDecodeThreads;
#pragma unroll
            for (int j = 0; j < kChunk; ++j) {
                const bool in = q < kGQ * kD && j < nj;
                v1[k][j] = in ? __ldcg(recs + (size_t)(j0 + j) * RF + hdr + q) : 0.f;
                if (PROBE) v2[k][j] = in ? __ldcg(recs + (size_t)(j0 + j) * RF + hdr + kGQ * kD + q) : 0.f;
            }
        }
    };
    // the headers first: the weights wait on them, the values only at the sums
    const bool hdr_warp = warp < (PROBE ? 2 : 1);
    float mj[2][kGQ], lj[2][kGQ];
    if (hdr_warp) {
        const int which = warp;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            const int j = lane + 32 * jj;                 // kMaxSplits = 64
            float4 m4 = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY), l4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (j < nsplit) {
                m4 = __ldcg(reinterpret_cast<const float4*>(recs + (size_t)j * RF + which * 8));
                l4 = __ldcg(reinterpret_cast<const float4*>(recs + (size_t)j * RF + which * 8 + 4));
            }
            mj[jj][0] = m4.x; mj[jj][1] = m4.y; mj[jj][2] = m4.z; mj[jj][3] = m4.w;
            lj[jj][0] = l4.x; lj[jj][1] = l4.y; lj[jj][2] = l4.z; lj[jj][3] = l4.w;
        }
    }
    load_chunk(0);
    if (hdr_warp) {
        const int which = warp;
        // the four heads' reductions side by side (independent shuffle chains)
        float M[kGQ], Lsum[kGQ];
#pragma unroll
        for (int hh = 0; hh < kGQ; ++hh) M[hh] = fmaxf(mj[0][hh], mj[1][hh]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int hh = 0; hh < kGQ; ++hh) M[hh] = fmaxf(M[hh], __shfl_xor_sync(0xffffffffu, M[hh], o));
#pragma unroll
        for (int hh = 0; hh < kGQ; ++hh) {
            Lsum[hh] = 0.f;
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const float f = mj[jj][hh] == -INFINITY ? 0.f : exp2f(mj[jj][hh] - M[hh]);
                if (lane + 32 * jj < nsplit) wgt[(which * kMaxSplits + lane + 32 * jj) * kGQ + hh] = f;
                Lsum[hh] = fmaf(f, lj[jj][hh], Lsum[hh]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int hh = 0; hh < kGQ; ++hh) Lsum[hh] += __shfl_xor_sync(0xffffffffu, Lsum[hh], o);
        if (lane < kGQ) Ls[which * 4 + lane] = lane == 0 ? Lsum[0] : lane == 1 ? Lsum[1] : lane == 2 ? Lsum[2] : Lsum[3];
    }
    __syncthreads();
    float acc1[kPer], acc2[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) { acc1[k] = 0.f; acc2[k] = 0.f; }
    for (int j0 = 0; j0 < nsplit; j0 += kChunk) {
        if (j0 > 0) load_chunk(j0);
        const int nj = min(kChunk, nsplit - j0);
#pragma unroll
        for (int k = 0; k < kPer; ++k) {
            const int q = tid + k * kDecodeThreads;
            const int hh = (q < kGQ * kD ? q : 0) / kD;
            const float* w1 = wgt + j0 * kGQ + hh;
            const float* w2 = wgt + (kMaxSplits + j0) * kGQ + hh;
#pragma unroll
            for (int j = 0; j < kChunk; ++j) {
                if (j < nj) {
                    acc1[k] = fmaf(w1[j * kGQ], v1[k][j], acc1[k]);
                    if (PROBE) acc2[k] = fmaf(w2[j * kGQ], v2[k][j], acc2[k]);
                }
            }
        }
    }
    float dn = 0.f, nn = 0.f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int q = tid + k * kDecodeThreads;
        if (q < kGQ * kD) {
            const int hh = q / kD, i = q % kD;
            const float L1 = Ls[hh];
            const float o = L1 > 0.f ? acc1[k] / L1 : 0.f;
            const size_t oi = ((size_t)ci * G.Hq + (size_t)h * kGQ + hh) * kD + i;
            if (!PROBE) {
                C.out[oi] = o;
            } else {
                const float L2 = Ls[4 + hh];
                const float o2 = L2 > 0.f ? acc2[k] / L2 : 0.f;
                if (C.out_full) C.out_full[oi] = o;
                dn += (o - o2) * (o - o2);
                nn += o * o;
            }
        }
    }
    if (PROBE) {
        dn = warp_sum(dn);
        nn = warp_sum(nn);
        if (lane == 0) { red[warp] = dn; red[kDecodeThreads / 32 + warp] = nn; }
        __syncthreads();
        if (tid == 0) {
            float a = 0.f, b = 0.f;
            for (int t = 0; t < kDecodeThreads / 32; ++t) { a += red[t]; b += red[kDecodeThreads / 32 + t]; }
            C.err[(size_t)ci * G.Hkv + h] = sqrtf(a) / (sqrtf(b) + 1e-6f);
        }
    }
    if (tid == 0) {
        St.tickets[(size_t)seq * G.Hkv + h] = 0u;
        if (C.fused && C.place[ci]) {
            // every CTA has read the counts: add the position placed by the first CTA
            const uint32_t k = C.tier_idx[(size_t)ci * G.Hkv + h];
            if (k < (uint32_t)G.ntiers) St.counts[cnt_index(G, seq, C.g, h) + k] += 1u;
        }
    }
}

}  // namespace dwkv

// Explicit instantiations for one (BITS, PROBE, C8) triple: RMAX in {64, 128}, S in {0, 8, 16,
// 32} and -1 (routed residual counts).
#define DWKV_DECODE_INSTANTIATE(B, P, C)                                                          \
    namespace dwkv {                                                                               \
    template __global__ void decode_kernel<B, P, 64, 0, C>(const Geom, const State, const DecodeCall);   \
    template __global__ void decode_kernel<B, P, 64, 8, C>(const Geom, const State, const DecodeCall);   \
    template __global__ void decode_kernel<B, P, 64, 16, C>(const Geom, const State, const DecodeCall);  \
    template __global__ void decode_kernel<B, P, 64, 32, C>(const Geom, const State, const DecodeCall);  \
    template __global__ void decode_kernel<B, P, 128, 0, C>(const Geom, const State, const DecodeCall);  \
    template __global__ void decode_kernel<B, P, 128, 8, C>(const Geom, const State, const DecodeCall);  \
    template __global__ void decode_kernel<B, P, 128, 16, C>(const Geom, const State, const DecodeCall); \
    template __global__ void decode_kernel<B, P, 128, 32, C>(const Geom, const State, const DecodeCall); \
    template __global__ void decode_kernel<B, P, 64, -1, C>(const Geom, const State, const DecodeCall);  \
    template __global__ void decode_kernel<B, P, 128, -1, C>(const Geom, const State, const DecodeCall); \
    }
