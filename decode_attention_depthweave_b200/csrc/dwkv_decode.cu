// dwkv_decode.cu -- fused split-K decode attention (and the probe) over the compressed
// cache.  "DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization for
// Long-Context KV Cache Compression", §3 Method: the fused kernel loads the shared basis,
// dequantises only the routed residual channels and feeds the attention score directly,
// never writing reconstructed keys / values (Eq. (1) evaluated inside attention); the
// probe is Eq. (3) with the with-residual output as the reference.
//
// For one query head q of kv-head h (tau folded with log2 e so exp2 can be used):
//   qt = B_K^T q                                 (once per CTA, from B_K in shared memory)
//   s_t = qt[:r_t] . c^K_t + scale^K_t * sum_i q[idx^K_ti] code^K_ti
//   online softmax over t;  acc_c += p_t c^V_t (coefficient space);
//   acc_r[idx^V_ti] += p_t scale^V_t code^V_ti (residual space)
//   o = (B_V acc_c + acc_r) / l                 (B_V applied once, in the combine)
//
// Work split: a CTA takes a byte-balanced run of one (sequence, kv-head)'s pages (pages are
// tier-homogeneous; tiers are visited in order).  Warp 4 lane 0 streams page chunks into
// a ring of shared-memory stages with cp.async.bulk (no multicast); warps 0-3 consume
// pages round-robin, each keeping its own softmax state; the CTA merges its 4 states into
// one partial record, and the last CTA of the (sequence, kv-head) (atomic ticket, no
// waiting) merges all partial records and writes the output.
#include "dwkv_common.cuh"

namespace dwkv {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack = 8.0f;   // keep a stale max while the new one is < 2^8 larger

struct WarpState {
    float m[kGQ], l[kGQ];          // running max (log2 domain) and per-lane partial sums
    float acc[kGQ][4];             // per-lane coefficient-space partials (tier mapping)
    float m2[kGQ], l2[kGQ];        // probe: no-residual state
    float acc2[kGQ][4];
};

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

// signed int8 / int4 code -> float (exact) by biasing into a float's mantissa
__device__ __forceinline__ float code8(uint32_t word, int e) {
    const uint32_t b = (word >> (8 * e)) & 0xffu;
    return __uint_as_float(0x4B400000u | (b ^ 0x80u)) - 12583040.0f;   // 2^23 + 2^22 + 128
}
__device__ __forceinline__ float code4(uint32_t word, int e) {
    const uint32_t b = (word >> (4 * e)) & 0xfu;
    return __uint_as_float(0x4B400000u | (b ^ 0x8u)) - 12582920.0f;    // 2^23 + 2^22 + 8
}

// Sum the per-lane partials of a tier mapping into the warp's shared accumulator.
template <int R, bool PROBE>
__device__ __forceinline__ void flush(WarpState& w, float4* accc, float4* accc2, int lane) {
    constexpr int NG = R / 4;
#pragma unroll
    for (int o = NG; o < 32; o <<= 1)
#pragma unroll
        for (int h = 0; h < kGQ; ++h)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                w.acc[h][c] += __shfl_xor_sync(0xffffffffu, w.acc[h][c], o);
                if (PROBE) w.acc2[h][c] += __shfl_xor_sync(0xffffffffu, w.acc2[h][c], o);
            }
    if (lane < NG) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float4 v = accc[4 * lane + c];
            v.x += w.acc[0][c]; v.y += w.acc[1][c]; v.z += w.acc[2][c]; v.w += w.acc[3][c];
            accc[4 * lane + c] = v;
            if (PROBE) {
                float4 u = accc2[4 * lane + c];
                u.x += w.acc2[0][c]; u.y += w.acc2[1][c]; u.z += w.acc2[2][c]; u.w += w.acc2[3][c];
                accc2[4 * lane + c] = u;
            }
        }
    }
#pragma unroll
    for (int h = 0; h < kGQ; ++h)
#pragma unroll
        for (int c = 0; c < 4; ++c) { w.acc[h][c] = 0.f; w.acc2[h][c] = 0.f; }
    __syncwarp();
}

__device__ __forceinline__ void flush_any(int R, WarpState& w, float4* accc, float4* accc2, int lane, bool probe) {
    if (probe) {
        switch (R) {
            case 8: flush<8, true>(w, accc, accc2, lane); break;
            case 16: flush<16, true>(w, accc, accc2, lane); break;
            case 32: flush<32, true>(w, accc, accc2, lane); break;
            case 64: flush<64, true>(w, accc, accc2, lane); break;
            case 128: flush<128, true>(w, accc, accc2, lane); break;
            default: break;
        }
    } else {
        switch (R) {
            case 8: flush<8, false>(w, accc, accc2, lane); break;
            case 16: flush<16, false>(w, accc, accc2, lane); break;
            case 32: flush<32, false>(w, accc, accc2, lane); break;
            case 64: flush<64, false>(w, accc, accc2, lane); break;
            case 128: flush<128, false>(w, accc, accc2, lane); break;
            default: break;
        }
    }
}

// Rescale one softmax state (registers + the warp's shared accumulators) by alpha per head.
__device__ __forceinline__ void rescale_state(float (&l)[kGQ], float (&acc)[kGQ][4], float4* accc,
                                              float* accr, const float (&alpha)[kGQ], int r_max, int lane) {
#pragma unroll
    for (int h = 0; h < kGQ; ++h) {
        l[h] *= alpha[h];
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[h][c] *= alpha[h];
    }
    for (int j = lane; j < r_max; j += 32) {
        float4 v = accc[j];
        v.x *= alpha[0]; v.y *= alpha[1]; v.z *= alpha[2]; v.w *= alpha[3];
        accc[j] = v;
    }
    if (accr) {
#pragma unroll
        for (int h = 0; h < kGQ; ++h)
#pragma unroll
            for (int m = 0; m < 4; ++m) accr[h * kD + lane + 32 * m] *= alpha[h];
    }
}

// One tier-homogeneous page of 64 token slots (nvalid of them live) for one warp.
template <int R, int BITS, bool PROBE>
__device__ __forceinline__ void page_step(const uint8_t* __restrict__ K, int nvalid, int s,
                                          const float4* __restrict__ qt, const float4* __restrict__ qs,
                                          float4* p_s, float4* p2_s, float4* accc, float4* accc2, float* accr,
                                          WarpState& w, int r_max, int lane) {
    constexpr uint32_t kCo = 128u * R;
    const uint32_t off_idx = kCo, off_codes = kCo + 64u * s, off_sc = kCo + 64u * s + 8u * s * BITS;
    const uint8_t* __restrict__ V = K + off_sc + 128u;
    float sc[2][kGQ], sc2[2][kGQ];
    // ---------------- scores (keys): coefficient dot + residual gather-dot
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
        const int t = lane + 32 * tt;
#pragma unroll
        for (int h = 0; h < kGQ; ++h) { sc[tt][h] = -INFINITY; sc2[tt][h] = -INFINITY; }
        if (t < nvalid) {
            float a[kGQ] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kc = 0; kc < R / 8; ++kc) {
                const uint4 cw = *reinterpret_cast<const uint4*>(K + kc * 1024 + t * 16);
                const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float c0 = bf16lo(wv[e]), c1 = bf16hi(wv[e]);
                    const float4 q0 = qt[kc * 8 + 2 * e], q1 = qt[kc * 8 + 2 * e + 1];
                    a[0] = fmaf(q0.x, c0, a[0]); a[1] = fmaf(q0.y, c0, a[1]);
                    a[2] = fmaf(q0.z, c0, a[2]); a[3] = fmaf(q0.w, c0, a[3]);
                    a[0] = fmaf(q1.x, c1, a[0]); a[1] = fmaf(q1.y, c1, a[1]);
                    a[2] = fmaf(q1.z, c1, a[2]); a[3] = fmaf(q1.w, c1, a[3]);
                }
            }
            float ra[kGQ] = {0.f, 0.f, 0.f, 0.f};
            for (int ch = 0; ch < s; ch += 8) {
                const uint2 ix = *reinterpret_cast<const uint2*>(K + off_idx + t * s + ch);
                uint32_t cw0, cw1 = 0;
                if (BITS == 8) {
                    const uint2 c = *reinterpret_cast<const uint2*>(K + off_codes + t * s + ch);
                    cw0 = c.x; cw1 = c.y;
                } else {
                    cw0 = *reinterpret_cast<const uint32_t*>(K + off_codes + t * (s / 2) + ch / 2);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t i = ((e < 4 ? ix.x : ix.y) >> (8 * (e & 3))) & 0xffu;
                    const float c = BITS == 8 ? code8(e < 4 ? cw0 : cw1, e & 3) : code4(cw0, e);
                    const float4 q = qs[i];
                    ra[0] = fmaf(q.x, c, ra[0]); ra[1] = fmaf(q.y, c, ra[1]);
                    ra[2] = fmaf(q.z, c, ra[2]); ra[3] = fmaf(q.w, c, ra[3]);
                }
            }
            const float scale = __half2float(*reinterpret_cast<const __half*>(K + off_sc + t * 2));
#pragma unroll
            for (int h = 0; h < kGQ; ++h) {
                sc[tt][h] = fmaf(scale, ra[h], a[h]);
                sc2[tt][h] = a[h];
            }
        }
    }
    // ---------------- online softmax (per warp; lazily rescaled)
    float p[2][kGQ], p2[2][kGQ];
    {
        float mloc[kGQ], alpha[kGQ];
        bool any = false;
#pragma unroll
        for (int h = 0; h < kGQ; ++h) {
            mloc[h] = warp_max(fmaxf(sc[0][h], sc[1][h]));
            alpha[h] = 1.f;
            if (mloc[h] > w.m[h] + kRescaleSlack) {
                alpha[h] = exp2f(w.m[h] - mloc[h]);
                w.m[h] = mloc[h];
                any = true;
            }
        }
        if (any) rescale_state(w.l, w.acc, accc, accr, alpha, r_max, lane);
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
            for (int h = 0; h < kGQ; ++h) {
                p[tt][h] = exp2f(sc[tt][h] - w.m[h]);     // -inf -> 0 for dead slots
                w.l[h] += p[tt][h];
            }
        if (PROBE) {
            bool any2 = false;
#pragma unroll
            for (int h = 0; h < kGQ; ++h) {
                mloc[h] = warp_max(fmaxf(sc2[0][h], sc2[1][h]));
                alpha[h] = 1.f;
                if (mloc[h] > w.m2[h] + kRescaleSlack) {
                    alpha[h] = exp2f(w.m2[h] - mloc[h]);
                    w.m2[h] = mloc[h];
                    any2 = true;
                }
            }
            if (any2) rescale_state(w.l2, w.acc2, accc2, nullptr, alpha, r_max, lane);
#pragma unroll
            for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                for (int h = 0; h < kGQ; ++h) {
                    p2[tt][h] = exp2f(sc2[tt][h] - w.m2[h]);
                    w.l2[h] += p2[tt][h];
                }
        }
    }
    // ---------------- residual-space values: scatter p * scale * code
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
        const int t = lane + 32 * tt;
        if (t < nvalid) {
            p_s[t] = make_float4(p[tt][0], p[tt][1], p[tt][2], p[tt][3]);
            if (PROBE) p2_s[t] = make_float4(p2[tt][0], p2[tt][1], p2[tt][2], p2[tt][3]);
            const float scale = __half2float(*reinterpret_cast<const __half*>(V + off_sc + t * 2));
            float wt[kGQ];
#pragma unroll
            for (int h = 0; h < kGQ; ++h) wt[h] = p[tt][h] * scale;
            for (int ch = 0; ch < s; ch += 8) {
                const uint2 ix = *reinterpret_cast<const uint2*>(V + off_idx + t * s + ch);
                uint32_t cw0, cw1 = 0;
                if (BITS == 8) {
                    const uint2 c = *reinterpret_cast<const uint2*>(V + off_codes + t * s + ch);
                    cw0 = c.x; cw1 = c.y;
                } else {
                    cw0 = *reinterpret_cast<const uint32_t*>(V + off_codes + t * (s / 2) + ch / 2);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const uint32_t i = ((e < 4 ? ix.x : ix.y) >> (8 * (e & 3))) & 0xffu;
                    const float c = BITS == 8 ? code8(e < 4 ? cw0 : cw1, e & 3) : code4(cw0, e);
#pragma unroll
                    for (int h = 0; h < kGQ; ++h) atomicAdd(&accr[h * kD + i], wt[h] * c);
                }
            }
        }
    }
    __syncwarp();
    // ---------------- coefficient-space values: lane = (4-column group, token subset)
    {
        constexpr int NG = R / 4, NSUB = 32 / NG;
        const int g4 = lane % NG, sub = lane / NG;
        const uint8_t* vb = V + (g4 >> 1) * 1024 + (g4 & 1) * 8;
#pragma unroll 4
        for (int t = sub; t < nvalid; t += NSUB) {
            const uint2 cw = *reinterpret_cast<const uint2*>(vb + t * 16);
            const float v[4] = {bf16lo(cw.x), bf16hi(cw.x), bf16lo(cw.y), bf16hi(cw.y)};
            const float4 pp = p_s[t];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                w.acc[0][c] = fmaf(pp.x, v[c], w.acc[0][c]);
                w.acc[1][c] = fmaf(pp.y, v[c], w.acc[1][c]);
                w.acc[2][c] = fmaf(pp.z, v[c], w.acc[2][c]);
                w.acc[3][c] = fmaf(pp.w, v[c], w.acc[3][c]);
            }
            if (PROBE) {
                const float4 qq = p2_s[t];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    w.acc2[0][c] = fmaf(qq.x, v[c], w.acc2[0][c]);
                    w.acc2[1][c] = fmaf(qq.y, v[c], w.acc2[1][c]);
                    w.acc2[2][c] = fmaf(qq.z, v[c], w.acc2[2][c]);
                    w.acc2[3][c] = fmaf(qq.w, v[c], w.acc2[3][c]);
                }
            }
        }
    }
    __syncwarp();
}

}  // namespace

template <int BITS, bool PROBE>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_kernel(const Geom G, const State S, const DecodeCall C) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.y;
    const int NS = C.stages;
    const DecodeSmem L = decode_smem_layout(G, NS, PROBE);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars);   // full[NS] empty[NS] basis
    const uint32_t full0 = smem_addr(bars), empty0 = smem_addr(bars + NS), basis_bar = smem_addr(bars + 2 * NS);
    float4* qt = reinterpret_cast<float4*>(smem + L.qt);
    float4* qs = reinterpret_cast<float4*>(smem + L.q);
    // per-CTA tier table
    uint32_t* m_cnt = reinterpret_cast<uint32_t*>(smem + L.misc);      // [8]
    uint32_t* m_P = m_cnt + 8;                                          // [9] page prefix
    uint32_t* m_R = m_P + 9;                                            // [8]
    uint32_t* m_chunk = m_R + 8;                                        // [8]
    uint32_t* m_misc = m_chunk + 8;                                     // p_begin p_end last flag
    float* m_state = reinterpret_cast<float*>(m_misc + 8);              // [4 warps][16]

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

    if (tid == 0) {
        const uint32_t* cnt = S.counts + cnt_index(G, seq, C.g, h);
        unsigned long long Bs[kMaxTiers + 1];
        uint32_t P = 0;
        unsigned long long B = 0;
        for (int k = 0; k < G.ntiers; ++k) {
            const uint32_t c = cnt[k], np = (c + kPage - 1) / kPage;
            m_cnt[k] = c;
            m_P[k] = P;
            m_R[k] = (uint32_t)G.tiers[k];
            m_chunk[k] = G.chunk_bytes[k];
            Bs[k] = B;
            P += np;
            B += (unsigned long long)np * G.chunk_bytes[k];
        }
        m_P[G.ntiers] = P;
        Bs[G.ntiers] = B;
        // byte-balanced page range: pages whose first byte lies in [lo, hi)
        const unsigned long long lo = B * (unsigned long long)split / nsplit;
        const unsigned long long hi = B * (unsigned long long)(split + 1) / nsplit;
        uint32_t pb = P, pe = P;
        for (int k = G.ntiers - 1; k >= 0; --k) {
            const uint32_t np = m_P[k + 1] - m_P[k];
            if (!np) continue;
            const unsigned long long ch = G.chunk_bytes[k];
            if (lo <= Bs[k] + (np - 1) * ch) {
                const unsigned long long d = lo > Bs[k] ? (lo - Bs[k] + ch - 1) / ch : 0;
                pb = m_P[k] + (uint32_t)d;
            }
            if (hi <= Bs[k] + (np - 1) * ch) {
                const unsigned long long d = hi > Bs[k] ? (hi - Bs[k] + ch - 1) / ch : 0;
                pe = m_P[k] + (uint32_t)d;
            }
        }
        m_misc[0] = pb;
        m_misc[1] = pe > pb ? pe : pb;
        for (int s = 0; s < NS; ++s) {
            mbar_init(full0 + 8 * s, 1);
            mbar_init(empty0 + 8 * s, 1);
        }
        mbar_init(basis_bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const uint32_t p_begin = m_misc[0], p_end = m_misc[1];
    const size_t basis_off = ((size_t)C.g * G.Hkv + h) * kD * G.r_max;

    if (warp == kConsumerWarps) {
        // ================= producer warp: basis, then the page chunks
        if (lane == 0) {
            const uint32_t bytes = (uint32_t)kD * G.r_max * 2;
            mbar_arrive_expect_tx(basis_bar, bytes);
            bulk_g2s(smem_addr(smem + L.basis), S.basis_k + basis_off, bytes, basis_bar);
        }
        const uint32_t npages = p_end - p_begin;
        const size_t pbase = page_index(G, seq, C.g, h, 0);
        const size_t tier_stride = (size_t)G.max_pages;
        // page units are fetched 32 at a time by the whole warp, one batch ahead
        auto fetch = [&](uint32_t u) -> uint32_t {
            if (u >= npages) return 0u;
            const uint32_t p = p_begin + u;
            int k = 0;
            while (k + 1 < G.ntiers && p >= m_P[k + 1]) ++k;
            return S.pages[pbase + (size_t)k * tier_stride + (p - m_P[k])];
        };
        uint32_t next = fetch(lane);
        bool ok = true;
        for (uint32_t b0 = 0; b0 < npages && ok; b0 += 32) {
            const uint32_t cur = next;
            next = fetch(b0 + 32 + lane);
            const uint32_t nb = min(32u, npages - b0);
            for (uint32_t j = 0; j < nb; ++j) {
                const uint32_t unit = __shfl_sync(0xffffffffu, cur, j);
                if (lane == 0) {
                    const uint32_t u = b0 + j, st = u % NS, p = p_begin + u;
                    int k = 0;
                    while (k + 1 < G.ntiers && p >= m_P[k + 1]) ++k;
                    if (u >= (uint32_t)NS && !mbar_wait(empty0 + 8 * st, ((u / NS) - 1) & 1)) {
                        set_dev_error(S, 6u /*DWKV_DEV_TIMEOUT*/, (uint32_t)seq, u);
                        ok = false;
                    }
                    if (ok) {
                        const uint32_t bytes = m_chunk[k];
                        mbar_arrive_expect_tx(full0 + 8 * st, bytes);
                        bulk_g2s(smem_addr(smem + L.stages + (size_t)st * G.stage_bytes),
                                 S.data + (size_t)unit * kUnit + (size_t)C.lig * bytes, bytes, full0 + 8 * st);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
    } else {
        // ================= consumer warps
        uint8_t* wbase = smem + L.warp + warp * L.warp_stride;
        float4* p_s = reinterpret_cast<float4*>(wbase + L.p);
        float4* p2_s = reinterpret_cast<float4*>(wbase + L.p2);
        float4* accc = reinterpret_cast<float4*>(wbase + L.accc);
        float4* accc2 = reinterpret_cast<float4*>(wbase + L.accc2);
        float* accr = reinterpret_cast<float*>(wbase + L.accr);
        const float qscale = G.tau * kLog2e;
        if (tid < kD) {
            const __nv_bfloat16* q = C.q + ((size_t)ci * G.Hq + (size_t)h * kGQ) * kD + tid;
            qs[tid] = make_float4(__bfloat162float(q[0]) * qscale, __bfloat162float(q[kD]) * qscale,
                                  __bfloat162float(q[2 * kD]) * qscale, __bfloat162float(q[3 * kD]) * qscale);
        }
        for (int j = lane; j < G.r_max; j += 32) {
            accc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (PROBE) accc2[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int e = lane; e < kGQ * kD; e += 32) accr[e] = 0.f;
        named_barrier(1, kConsumerWarps * 32);
        bool ok = mbar_wait(basis_bar, 0);
        if (!ok && lane == 0) set_dev_error(S, 6u, (uint32_t)seq, 0xffffffffu);
        if (ok && tid < G.r_max) {
            const __nv_bfloat16* bk = reinterpret_cast<const __nv_bfloat16*>(smem + L.basis) + tid;
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
            for (int i = 0; i < kD; ++i) {
                const float b = __bfloat162float(bk[i * G.r_max]);
                const float4 q = qs[i];
                a.x = fmaf(b, q.x, a.x); a.y = fmaf(b, q.y, a.y);
                a.z = fmaf(b, q.z, a.z); a.w = fmaf(b, q.w, a.w);
            }
            qt[tid] = a;
        }
        named_barrier(1, kConsumerWarps * 32);

        WarpState w;
#pragma unroll
        for (int hh = 0; hh < kGQ; ++hh) {
            w.m[hh] = -INFINITY; w.l[hh] = 0.f; w.m2[hh] = -INFINITY; w.l2[hh] = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) { w.acc[hh][c] = 0.f; w.acc2[hh][c] = 0.f; }
        }
        int curR = 0;
        const int s = G.s;
        for (uint32_t u = warp; ok && p_begin + u < p_end; u += kConsumerWarps) {
            const uint32_t p = p_begin + u, st = u % NS;
            int k = 0;
            while (k + 1 < G.ntiers && p >= m_P[k + 1]) ++k;
            const int R = (int)m_R[k];
            const uint32_t pit = p - m_P[k], npk = m_P[k + 1] - m_P[k];
            const int nvalid = pit + 1 < npk ? kPage : (int)(m_cnt[k] - pit * kPage);
            if (R != curR) {
                flush_any(curR, w, accc, accc2, lane, PROBE);
                curR = R;
            }
            if (!mbar_wait(full0 + 8 * st, (u / NS) & 1)) {
                if (lane == 0) set_dev_error(S, 6u, (uint32_t)seq, u);
                ok = false;
                break;
            }
            const uint8_t* stg = smem + L.stages + (size_t)st * G.stage_bytes;
            switch (R) {
                case 8: page_step<8, BITS, PROBE>(stg, nvalid, s, qt, qs, p_s, p2_s, accc, accc2, accr, w, G.r_max, lane); break;
                case 16: page_step<16, BITS, PROBE>(stg, nvalid, s, qt, qs, p_s, p2_s, accc, accc2, accr, w, G.r_max, lane); break;
                case 32: page_step<32, BITS, PROBE>(stg, nvalid, s, qt, qs, p_s, p2_s, accc, accc2, accr, w, G.r_max, lane); break;
                case 64: page_step<64, BITS, PROBE>(stg, nvalid, s, qt, qs, p_s, p2_s, accc, accc2, accr, w, G.r_max, lane); break;
                case 128: page_step<128, BITS, PROBE>(stg, nvalid, s, qt, qs, p_s, p2_s, accc, accc2, accr, w, G.r_max, lane); break;
                default: break;
            }
            if (lane == 0) mbar_arrive(empty0 + 8 * st);
        }
        flush_any(curR, w, accc, accc2, lane, PROBE);
        float* ms = m_state + warp * 16;
#pragma unroll
        for (int hh = 0; hh < kGQ; ++hh) {
            const float l = warp_sum(w.l[hh]);
            const float l2 = PROBE ? warp_sum(w.l2[hh]) : 0.f;
            if (lane == 0) {
                ms[hh] = w.m[hh]; ms[4 + hh] = l;
                ms[8 + hh] = w.m2[hh]; ms[12 + hh] = l2;
            }
        }
    }
    __syncthreads();

    // ================= CTA merge of the 4 warp states -> partial record
    const int nrec = C.total_splits;
    float* rec = C.ws + ((size_t)h * nrec + blockIdx.x) * C.rec_floats;
    float* mf = reinterpret_cast<float*>(smem + L.stages);   // [2][4 warps][4 heads] factors; stages are idle now
    if (tid < 2 * kGQ) {
        const int which = tid / kGQ, hh = tid % kGQ;
        if (which == 0 || PROBE) {
            float M = -INFINITY;
            for (int w2 = 0; w2 < kConsumerWarps; ++w2) M = fmaxf(M, m_state[w2 * 16 + which * 8 + hh]);
            float Lsum = 0.f;
            for (int w2 = 0; w2 < kConsumerWarps; ++w2) {
                const float mw = m_state[w2 * 16 + which * 8 + hh];
                const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
                mf[which * 16 + w2 * 4 + hh] = f;
                Lsum += f * m_state[w2 * 16 + which * 8 + 4 + hh];
            }
            rec[which * 8 + hh] = M;
            rec[which * 8 + 4 + hh] = Lsum;
        }
    }
    __syncthreads();
    {
        const int hdr = PROBE ? 16 : 8;
        float* rc = rec + hdr;
        float* rc2 = rc + kGQ * G.r_max;
        float* rr = rc + (PROBE ? 2 : 1) * kGQ * G.r_max;
        for (int e = tid; e < kGQ * G.r_max; e += blockDim.x) {
            const int hh = e / G.r_max, j = e % G.r_max;
            float v = 0.f, v2 = 0.f;
            for (int w2 = 0; w2 < kConsumerWarps; ++w2) {
                const uint8_t* wb = smem + L.warp + w2 * L.warp_stride;
                v += mf[w2 * 4 + hh] * reinterpret_cast<const float*>(wb + L.accc)[j * 4 + hh];
                if (PROBE) v2 += mf[16 + w2 * 4 + hh] * reinterpret_cast<const float*>(wb + L.accc2)[j * 4 + hh];
            }
            rc[e] = v;
            if (PROBE) rc2[e] = v2;
        }
        for (int e = tid; e < kGQ * kD; e += blockDim.x) {
            const int hh = e / kD;
            float v = 0.f;
            for (int w2 = 0; w2 < kConsumerWarps; ++w2)
                v += mf[w2 * 4 + hh] * reinterpret_cast<const float*>(smem + L.warp + w2 * L.warp_stride + L.accr)[e];
            rr[e] = v;
        }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t t = atomicAdd(&S.tickets[(size_t)seq * G.Hkv + h], 1u);
        m_misc[2] = (t == (uint32_t)(nsplit - 1)) ? 1u : 0u;
    }
    __syncthreads();
    if (!m_misc[2]) return;
    __threadfence();

    // ================= last CTA of (sequence, kv-head): merge all splits, apply B_V
    const int r0 = C.split_begin[ci];
    const int hdr = PROBE ? 16 : 8;
    float* wgt = reinterpret_cast<float*>(smem + L.stages);           // [2][kMaxSplits][4]
    float* cc = wgt + 2 * kMaxSplits * kGQ;                            // [4][r_max]
    float* cc2 = cc + kGQ * G.r_max;                                   // [4][r_max]
    float* cr = cc2 + kGQ * G.r_max;                                   // [4][d]
    float* Ls = cr + kGQ * kD;                                         // [2][4]
    float* red = Ls + 8;                                               // [2][160] reductions
    if (tid < 2 * kGQ) {
        const int which = tid / kGQ, hh = tid % kGQ;
        if (which == 0 || PROBE) {
            float M = -INFINITY;
            for (int j = 0; j < nsplit; ++j)
                M = fmaxf(M, __ldcg(C.ws + ((size_t)h * nrec + r0 + j) * C.rec_floats + which * 8 + hh));
            float Lsum = 0.f;
            for (int j = 0; j < nsplit; ++j) {
                const float* rj = C.ws + ((size_t)h * nrec + r0 + j) * C.rec_floats;
                const float mj = __ldcg(rj + which * 8 + hh);
                const float f = mj == -INFINITY ? 0.f : exp2f(mj - M);
                wgt[(which * kMaxSplits + j) * kGQ + hh] = f;
                Lsum += f * __ldcg(rj + which * 8 + 4 + hh);
            }
            Ls[which * 4 + hh] = Lsum;
        }
    }
    __syncthreads();
    for (int e = tid; e < kGQ * G.r_max; e += blockDim.x) {
        const int hh = e / G.r_max;
        float v = 0.f, v2 = 0.f;
        for (int j = 0; j < nsplit; ++j) {
            const float* rj = C.ws + ((size_t)h * nrec + r0 + j) * C.rec_floats + hdr;
            v += wgt[j * kGQ + hh] * __ldcg(rj + e);
            if (PROBE) v2 += wgt[(kMaxSplits + j) * kGQ + hh] * __ldcg(rj + kGQ * G.r_max + e);
        }
        cc[e] = v;
        if (PROBE) cc2[e] = v2;
    }
    for (int e = tid; e < kGQ * kD; e += blockDim.x) {
        const int hh = e / kD;
        float v = 0.f;
        for (int j = 0; j < nsplit; ++j) {
            const float* rj = C.ws + ((size_t)h * nrec + r0 + j) * C.rec_floats + hdr + (PROBE ? 2 : 1) * kGQ * G.r_max;
            v += wgt[j * kGQ + hh] * __ldcg(rj + e);
        }
        cr[e] = v;
    }
    __syncthreads();
    const __nv_bfloat16* bv = S.basis_v + basis_off;
    float dn = 0.f, nn = 0.f;
    for (int e = tid; e < kGQ * kD; e += blockDim.x) {
        const int hh = e / kD, i = e % kD;
        const __nv_bfloat16* row = bv + (size_t)i * G.r_max;
        float a = 0.f, a2 = 0.f;
        for (int j = 0; j < G.r_max; ++j) {
            const float b = __bfloat162float(row[j]);
            a = fmaf(b, cc[hh * G.r_max + j], a);
            if (PROBE) a2 = fmaf(b, cc2[hh * G.r_max + j], a2);
        }
        const float L1 = Ls[hh];
        const float o = L1 > 0.f ? (a + cr[e]) / L1 : 0.f;
        const size_t oi = ((size_t)ci * G.Hq + (size_t)h * kGQ + hh) * kD + i;
        if (!PROBE) {
            C.out[oi] = o;
        } else {
            const float L2 = Ls[4 + hh];
            const float o2 = L2 > 0.f ? a2 / L2 : 0.f;
            if (C.out_full) C.out_full[oi] = o;
            dn += (o - o2) * (o - o2);
            nn += o * o;
        }
    }
    if (PROBE) {
        red[tid] = dn;
        red[kDecodeThreads + tid] = nn;
        __syncthreads();
        if (tid == 0) {
            float a = 0.f, b = 0.f;
            for (int t = 0; t < (int)blockDim.x; ++t) { a += red[t]; b += red[kDecodeThreads + t]; }
            C.err[(size_t)ci * G.Hkv + h] = sqrtf(a) / (sqrtf(b) + 1e-6f);
        }
    }
    if (tid == 0) S.tickets[(size_t)seq * G.Hkv + h] = 0u;
}

// explicit instantiations
template __global__ void decode_kernel<8, false>(const Geom, const State, const DecodeCall);
template __global__ void decode_kernel<4, false>(const Geom, const State, const DecodeCall);
template __global__ void decode_kernel<8, true>(const Geom, const State, const DecodeCall);
template __global__ void decode_kernel<4, true>(const Geom, const State, const DecodeCall);

}  // namespace dwkv
