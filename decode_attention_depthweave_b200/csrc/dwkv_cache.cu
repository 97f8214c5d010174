// dwkv_cache.cu -- page placement, encode/append, import, export and reset kernels.  The
// per-vector encode steps and their fixed operation order are in dwkv_encode.cuh.
#include "dwkv_encode.cuh"
#include "dwkv_stored.cuh"

namespace dwkv {

// ------------------------------------------------------------------------------------
// Slot placement for the group's first layer that appends a position.  One block per
// (sequence in call, kv-head).  Slots inside a tier are numbered in position order; new
// pages come from the tier's free ring first, then from the pool's bump pointer.
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void place_block(const Geom& G, const State& S, const AppendCall& C,
                                            const uint8_t* __restrict__ tier_idx, int i, int h) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int na = C.na[i];
    if (na <= 0) return;                     // uniform across the block
    const int seq = C.seq[i], a0 = C.a0[i];
    const int rowbase = C.tok0[i] + (a0 - C.pos0[i]);
    __shared__ uint32_t s_cnt[kMaxTiers], s_old[kMaxTiers], s_run[kMaxTiers], s_fail;
    __shared__ uint32_t s_warp[8][kMaxTiers];
    const size_t ci = cnt_index(G, seq, C.g, h);
    if (tid < kMaxTiers) {
        s_cnt[tid] = 0;
        s_old[tid] = tid < G.ntiers ? S.counts[ci + tid] : 0u;
    }
    if (tid == 0) s_fail = 0;
    __syncthreads();
    for (int p = tid; p < na; p += blockDim.x) {
        uint32_t k = tier_idx[(size_t)(rowbase + p) * G.Hkv + h];
        if (k < (uint32_t)G.ntiers) atomicAdd(&s_cnt[k], 1u);
        else set_dev_error(S, 2u /*DWKV_DEV_BAD_TIER*/, (uint32_t)seq, (uint32_t)(a0 + p));
    }
    __syncthreads();
    if (tid < G.ntiers) {
        const int k = tid;
        const uint32_t old = s_old[k], nw = old + s_cnt[k];
        const uint32_t pn = (nw + kPage - 1) / kPage;
        // pages the tier already holds (emptied by re-tiering, or partly filled) are reused
        const uint32_t po = S.owned[ci + k];
        const size_t pi = page_index(G, seq, C.g, h, k);
        if (pn > (uint32_t)G.max_pages) {
            set_dev_error(S, 1u /*DWKV_DEV_POOL_EXHAUSTED*/, (uint32_t)seq, (uint32_t)h);
            s_fail = 1;
        } else if (pn > po) {
            const uint32_t need = pn - po;
            const uint32_t t = atomicAdd(&S.free_head[k], need);
            const uint32_t tail = *((volatile uint32_t*)&S.free_tail[k]);
            const int avail = (int)(tail - t);
            const uint32_t take = avail <= 0 ? 0u : ((uint32_t)avail < need ? (uint32_t)avail : need);
            for (uint32_t q = 0; q < take; ++q)
                S.pages[pi + po + q] = S.free_list[(size_t)k * G.free_cap + ((t + q) & (G.free_cap - 1))];
            const uint32_t rest = need - take;
            if (rest) {
                const unsigned long long units = (unsigned long long)rest * G.page_units[k];
                const unsigned long long base = atomicAdd(S.bump, units);
                if (base + units > S.data_units) {
                    set_dev_error(S, 1u /*DWKV_DEV_POOL_EXHAUSTED*/, (uint32_t)seq, (uint32_t)h);
                    s_fail = 1;
                } else {
                    for (uint32_t q = 0; q < rest; ++q)
                        S.pages[pi + po + take + q] = (uint32_t)(base + (unsigned long long)q * G.page_units[k]);
                }
            }
            if (!s_fail) S.owned[ci + k] = pn;
        }
    }
    __syncthreads();
    const size_t si = slot_index(G, seq, C.g, h, a0);
    if (s_fail) {
        for (int p = tid; p < na; p += blockDim.x) S.slot_map[si + p] = 0u;
        return;
    }
    if (tid < kMaxTiers) s_run[tid] = s_old[tid];
    __syncthreads();
    for (int base = 0; base < na; base += blockDim.x) {
        const int p = base + tid;
        uint32_t k = 0xffu;
        if (p < na) {
            k = tier_idx[(size_t)(rowbase + p) * G.Hkv + h];
            if (k >= (uint32_t)G.ntiers) k = 0xffu;
        }
        uint32_t rank = 0;
        for (int kk = 0; kk < G.ntiers; ++kk) {
            const uint32_t m = __ballot_sync(0xffffffffu, k == (uint32_t)kk);
            if (k == (uint32_t)kk) rank = __popc(m & ((1u << lane) - 1u));
            if (lane == 0) s_warp[warp][kk] = __popc(m);
        }
        __syncthreads();
        if (p < na) {
            if (k != 0xffu) {
                uint32_t off = s_run[k];
                for (int w = 0; w < warp; ++w) off += s_warp[w][k];
                const uint32_t slot = off + rank;
                S.slot_map[si + p] = ((k + 1u) << 24) | slot;
                const uint32_t unit = S.pages[page_index(G, seq, C.g, h, k) + slot / kPage];
                reinterpret_cast<int32_t*>(S.data + (size_t)unit * kUnit + pos_block_of(G, k))[slot % kPage] = a0 + p;
            } else {
                S.slot_map[si + p] = 0u;
            }
        }
        __syncthreads();
        if (tid < G.ntiers) {
            uint32_t tot = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += s_warp[w][tid];
            s_run[tid] += tot;
        }
        __syncthreads();
    }
    if (tid < G.ntiers) S.counts[ci + tid] = s_old[tid] + s_cnt[tid];
}

__global__ void __launch_bounds__(256) place_kernel(const Geom G, const State S, const AppendCall C,
                                                    const uint8_t* __restrict__ tier_idx) {
    place_block(G, S, C, tier_idx, blockIdx.x, blockIdx.y);
}

// Row of the call's input arrays -> (index in call, sequence, position).
__device__ __forceinline__ int call_index_of(const AppendCall& C, int row) {
    int lo = 0, hi = C.n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (C.tok0[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
}


// ------------------------------------------------------------------------------------
// Both bases of the block's (group, kv-head) into shared memory, [2][d][P] bf16 with
// P = r_max + 2, in two steps so that other global round trips overlap its latency: the
// block's share of both bases into registers (at most 16 x 16 bytes a thread for 256
// threads), then into shared memory.
constexpr int kBasisRegs = 2 * kD * kMaxRank / 8 / 256;
__device__ __forceinline__ void bases_issue(const Geom& G, const State& S, int g, int h, uint4 (&v)[kBasisRegs]) {
    const int tid = threadIdx.x, RM = G.r_max;
    const size_t boff = ((size_t)g * G.Hkv + h) * kD * RM;
    const int nvec = kD * RM / 8;
    const uint4* srck = reinterpret_cast<const uint4*>(S.basis_k + boff);
    const uint4* srcv = reinterpret_cast<const uint4*>(S.basis_v + boff);
#pragma unroll
    for (int b = 0; b < kBasisRegs; ++b) {
        const int e = tid + b * 256;
        v[b] = e < 2 * nvec ? __ldg(e < nvec ? srck + e : srcv + (e - nvec)) : make_uint4(0u, 0u, 0u, 0u);
    }
}
__device__ __forceinline__ void bases_store(const Geom& G, const uint4 (&v)[kBasisRegs], __nv_bfloat16* bs) {
    const int tid = threadIdx.x, RM = G.r_max, P = G.r_max + 2;
    const int nvec = kD * RM / 8;
#pragma unroll
    for (int b = 0; b < kBasisRegs; ++b) {
        const int e = tid + b * 256;
        if (e >= 2 * nvec) break;
        const int z = e >= nvec, ev = z ? e - nvec : e;
        const int i = (ev * 8) / RM, j = (ev * 8) % RM;
        uint32_t* dst = reinterpret_cast<uint32_t*>(bs + (size_t)z * kD * P + (size_t)i * P + j);
        dst[0] = v[b].x; dst[1] = v[b].y; dst[2] = v[b].z; dst[3] = v[b].w;
    }
}

__device__ __forceinline__ UnitIn encode_fetch(const Geom& G, const State& S, const AppendCall& C,
                                               const __nv_bfloat16* __restrict__ k_new,
                                               const __nv_bfloat16* __restrict__ v_new, int h, int unit,
                                               float* coeff_dbg) {
    const int lane = threadIdx.x & 31;
    const int row = unit >> 1, z = unit & 1;
    const int ci = call_index_of(C, row);
    const int seq = C.seq[ci];
    const int pos = C.pos0[ci] + (row - C.tok0[ci]);
    UnitIn in;
    const __nv_bfloat16* src = (z ? v_new : k_new) + ((size_t)row * G.Hkv + h) * kD;
#pragma unroll
    for (int m = 0; m < 4; ++m) in.xr[m] = __bfloat162float(src[lane + 32 * m]);
    in.ok = find_dest(G, S, seq, C.g, C.lig, h, pos, in.dst);
    in.dbg = coeff_dbg ? coeff_dbg + (((size_t)row * G.Hkv + h) * 2 + z) * G.r_max : nullptr;
    in.gate = C.gate ? C.gate[((size_t)row * G.Hkv + h) * 2 + z] : 1.f;
    // a0..a0+na were placed by the placement; a zero entry means placement failed (already
    // reported) or the group never placed this position
    if (!in.ok && lane == 0 && z == 0 && !(pos >= C.a0[ci] && pos < C.a0[ci] + C.na[ci]))
        set_dev_error(S, 5u /*DWKV_DEV_NO_SLOT*/, (uint32_t)seq, (uint32_t)pos);
    return in;
}

// ------------------------------------------------------------------------------------
// Bulk encode kernel.  A block per (kv-head, keys or values) strides over tiles of kEncTile
// input rows and runs the encode steps on all of a tile's vectors together:
//   1. the rows' destinations (slot map), counted by tier and given slots in descending
//      tier order; each row's x enters shared memory as bf16 [slot][channel];
//   2. the projection on the tensor cores: a warp takes 16 slots (one MMA row tile) and half
//      of their coefficient tiles, c = X B as bf16 x bf16 products accumulated in fp32 (within
//      1e-5 |x| of the fp64 projection; the order of the accumulation is the tensor core's),
//      up to the largest rank among its slots (the first slot, by the sort); then the bf16
//      rounding and the coefficient stores (a slot's coefficients past its own rank are
//      neither stored nor kept: they enter its residual as exact zeros), and the fp32
//      projection exported when asked (coeff_dbg);
//   3. residual items of 4 slots, lane = channels lane + 32 m: the fixed-order fma chains
//      over j of step 3 run to the largest rank of the 4 slots; a zero coefficient adds an
//      exact +-0 to an accumulator that started at +0, which leaves it unchanged, so every
//      slot gets the residual of its own-length chain; then steps 4-6 per slot (quantize_store).
// Steps 2 (rounding) to 6 are the same operations in the same order as encode_body's, so the
// stored bytes follow from the exported projection bit for bit.  Three 256-thread blocks fit
// an SM at r_max 64 (~76 KB of shared memory).  The kernel has no waits of its own beyond
// block barriers.
// ------------------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256, 3) encode_kernel(const Geom G, const State S, const AppendCall C,
                                                        const __nv_bfloat16* __restrict__ k_new,
                                                        const __nv_bfloat16* __restrict__ v_new,
                                                        float* __restrict__ coeff_dbg) {
    extern __shared__ __align__(16) uint8_t smem[];
    const EncTileLayout L = enc_tile_layout(G.r_max);
    const int h = blockIdx.y, z = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(smem + L.bs);
    __nv_bfloat16* bt = reinterpret_cast<__nv_bfloat16*>(smem + L.bt);
    __nv_bfloat16* xb = reinterpret_cast<__nv_bfloat16*>(smem + L.xb);
    float* cs = reinterpret_cast<float*>(smem + L.cs);
    uint8_t** sblk = reinterpret_cast<uint8_t**>(smem + L.sblk);
    int* sR = reinterpret_cast<int*>(smem + L.sR);
    int* sprow = reinterpret_cast<int*>(smem + L.sprow);
    int* srow = reinterpret_cast<int*>(smem + L.srow);
    int* rslot = reinterpret_cast<int*>(smem + L.rslot);
    int* cnt = reinterpret_cast<int*>(smem + L.misc);
    int* base = cnt + kMaxTiers;
    int* nvalid_p = base + kMaxTiers;
    float* rstage = reinterpret_cast<float*>(smem + L.cst + warp * kEncStage);
    uint8_t* chstage = reinterpret_cast<uint8_t*>(rstage + kD);
    const int RM = G.r_max, PB = L.PB;

    // ---- this (group, kv-head, K or V) basis: bf16 [kD][PB] and transposed [RP][kEncXB],
    //      the columns past r_max zero
    {
        const __nv_bfloat16* src = (z ? S.basis_v : S.basis_k) + ((size_t)C.g * G.Hkv + h) * kD * RM;
        uint16_t* b16 = reinterpret_cast<uint16_t*>(bs);
        uint16_t* t16 = reinterpret_cast<uint16_t*>(bt);
        const int padc = PB - RM;
        for (int e = tid; e < kD * padc; e += blockDim.x) b16[(e / padc) * PB + RM + e % padc] = 0;
        for (int e = tid; e < (L.RP - RM) * kD; e += blockDim.x) t16[(RM + e / kD) * kEncXB + e % kD] = 0;
        const int nvec = kD * RM / 8;
        for (int e = tid; e < nvec; e += blockDim.x) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + e);
            const int i = (e * 8) / RM, j = (e * 8) % RM;
            uint32_t* dst = reinterpret_cast<uint32_t*>(bs + (size_t)i * PB + j);
            dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                t16[(j + 2 * q) * kEncXB + i] = (uint16_t)(w4[q] & 0xffffu);
                t16[(j + 2 * q + 1) * kEncXB + i] = (uint16_t)(w4[q] >> 16);
            }
        }
    }

    const __nv_bfloat16* xin = z ? v_new : k_new;
    const int ntiles = (C.total + kEncTile - 1) / kEncTile;
    const int trow = tid & (kEncTile - 1), q = tid / kEncTile;      // 4 threads a row, 32 channels each
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        // ---- 1: x into registers (requested first), destinations, tier counts
        const int row = tile * kEncTile + trow;
        const bool in_range = row < C.total;
        uint4 xv[4];
        if (in_range) {
            const uint4* src = reinterpret_cast<const uint4*>(xin + ((size_t)row * G.Hkv + h) * kD + 32 * q);
#pragma unroll
            for (int b = 0; b < 4; ++b) xv[b] = __ldg(src + b);
        }
        if (tid < kMaxTiers) cnt[tid] = 0;
        __syncthreads();                        // counts cleared; the previous tile is done
        Dest d;
        bool ok = false;
        int within = 0;
        if (q == 0 && in_range) {
            const int ci = call_index_of(C, row);
            const int seq = C.seq[ci];
            const int pos = C.pos0[ci] + (row - C.tok0[ci]);
            ok = find_dest(G, S, seq, C.g, C.lig, h, pos, d);
            // a0..a0+na were placed by the placement; a zero entry means placement failed
            // (already reported) or the group never placed this position
            if (!ok && z == 0 && !(pos >= C.a0[ci] && pos < C.a0[ci] + C.na[ci]))
                set_dev_error(S, 5u /*DWKV_DEV_NO_SLOT*/, (uint32_t)seq, (uint32_t)pos);
            if (ok) within = atomicAdd(&cnt[d.k], 1);
        }
        __syncthreads();
        if (tid == 0) {
            int acc = 0;
            for (int k = kMaxTiers - 1; k >= 0; --k) {
                base[k] = acc;
                acc += cnt[k];
            }
            *nvalid_p = acc;
        }
        __syncthreads();
        const int nvalid = *nvalid_p;
        if (q == 0) {
            int slot = -1;
            if (ok) {
                slot = base[d.k] + within;
                sblk[slot] = d.blk + (z ? G.blk_bytes[d.k] : 0u);
                sR[slot] = d.R;
                sprow[slot] = d.row | (d.k << 8);          // row in the page, tier
                srow[slot] = row;
            }
            rslot[trow] = slot;
        }
        if (tid >= nvalid && tid < kEncTile) sR[tid] = 0;          // empty slots
        __syncthreads();
        {
            const int slot = rslot[trow];
            if (slot >= 0) {
                uint4* dst = reinterpret_cast<uint4*>(xb + (size_t)slot * kEncXB + 32 * q);
#pragma unroll
                for (int b = 0; b < 4; ++b) dst[b] = xv[b];
            }
        }
        __syncthreads();

        // ---- 2: projection on the tensor cores, bf16 rounding, coefficient stores
        {
            const int mt = warp & 3, nh = warp >> 2;
            const int Rm = 16 * mt < nvalid ? sR[16 * mt] : 0;
            if (Rm > 0) {
                const int g = lane >> 2, c = lane & 3;
                const uint32_t xaddr = smem_addr(xb + (size_t)(16 * mt + (lane & 15)) * kEncXB + 8 * (lane >> 4));
                const uint32_t baddr = smem_addr(bt + (size_t)(lane & 7) * kEncXB + 8 * ((lane >> 3) & 1));
                const int ntl = Rm / 8;                        // coefficient tiles of 8; this warp: nh, nh + 2, ...
                for (int u0 = nh; u0 < ntl; u0 += 8) {         // up to 4 tiles at a time
                    float dd[4][4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) dd[u][0] = dd[u][1] = dd[u][2] = dd[u][3] = 0.f;
#pragma unroll
                    for (int ks = 0; ks < kD / 16; ++ks) {
                        uint32_t af[4];
                        ldsm_x4(xaddr + 32u * ks, af);
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int nt = u0 + 2 * u;
                            if (nt < ntl) {
                                uint32_t b[2];
                                ldsm_x2(baddr + (uint32_t)(8 * nt) * (kEncXB * 2) + 32u * ks, b);
                                mma_bf16(dd[u], af, b);
                            }
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int nt = u0 + 2 * u;
                        if (nt >= ntl) break;
                        const int j0 = 8 * nt + 2 * c;
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int sl = 16 * mt + g + 8 * hf;
                            const float v0 = dd[u][2 * hf], v1 = dd[u][2 * hf + 1];
                            const bool on = j0 < sR[sl];           // ranks are multiples of 8: j0 + 1 too
                            if (G.c8) {                                // the projections; blocks below
                                cs[j0 * kEncXP + sl] = on ? v0 : 0.f;
                                cs[(j0 + 1) * kEncXP + sl] = on ? v1 : 0.f;
                                if (on && coeff_dbg)
                                    *reinterpret_cast<float2*>(coeff_dbg + (((size_t)srow[sl] * G.Hkv + h) * 2 + z) * RM +
                                                               j0) = make_float2(v0, v1);
                                continue;
                            }
                            const __nv_bfloat16 c0 = __float2bfloat16_rn(v0), c1 = __float2bfloat16_rn(v1);
                            cs[j0 * kEncXP + sl] = on ? __bfloat162float(c0) : 0.f;
                            cs[(j0 + 1) * kEncXP + sl] = on ? __bfloat162float(c1) : 0.f;
                            if (on) {
                                __nv_bfloat162 pr;
                                pr.x = c0;
                                pr.y = c1;
                                *reinterpret_cast<__nv_bfloat162*>(sblk[sl] + (size_t)(j0 >> 3) * 1024 + (sprow[sl] & 0xff) * 16 +
                                                                   (j0 & 7) * 2) = pr;
                                if (coeff_dbg)
                                    *reinterpret_cast<float2*>(coeff_dbg + (((size_t)srow[sl] * G.Hkv + h) * 2 + z) * RM +
                                                               j0) = make_float2(v0, v1);
                            }
                        }
                    }
                }
            }
        }
        __syncthreads();

        // ---- 2 (8-bit coefficients): each half warp quantises one (slot, block of 16) at a
        //      time, the dequantised values replacing the projections in cs
        if (G.c8) {
            const int nbm = L.RP / 16, units = nvalid * nbm, e = lane & 15;
            for (int u0 = 2 * warp; u0 < units; u0 += 2 * (int)(blockDim.x >> 5)) {
                const int u = u0 + (lane >> 4);
                const int sl = u < units ? u / nbm : 0, b = u < units ? u % nbm : 0;
                const bool on = u < units && 16 * b < sR[sl];   // uniform over the half warp
                const int j = 16 * b + e;
                uint16_t sh;
                int qc;
                float cb;
                quantize_coeff8(on ? cs[j * kEncXP + sl] : 0.f, sh, qc, cb);
                if (on) {
                    cs[j * kEncXP + sl] = cb;
                    const int prow = sprow[sl] & 0xff, Rs = sR[sl];
                    sblk[sl][z ? vc8_code_off(j, prow) : kc8_code_off(j, prow)] = (uint8_t)(int8_t)qc;
                    if (e == 0)
                        *reinterpret_cast<uint16_t*>(sblk[sl] + (z ? vc8_scale_off(Rs, b, prow) : kc8_scale_off(Rs, b, prow))) = sh;
                }
            }
            __syncthreads();
        }

        // ---- 3: residual against the stored coefficients, then steps 4-6 per slot; items of
        //      4 slots (16 a tile, taken w, w + 8, ...: a costly item with a cheaper one)
        for (int u = warp; 4 * u < nvalid; u += (int)(blockDim.x >> 5)) {
            const int s0 = 4 * u, Ru = sR[s0];
            float a[4][4];
#pragma unroll
            for (int t = 0; t < 4; ++t)
#pragma unroll
                for (int m = 0; m < 4; ++m) a[t][m] = 0.f;
            for (int j = 0; j < Ru; j += 2) {          // ranks are multiples of 8
                const float4 c0 = *reinterpret_cast<const float4*>(cs + j * kEncXP + s0);
                const float4 c1 = *reinterpret_cast<const float4*>(cs + (j + 1) * kEncXP + s0);
                const float c0v[4] = {c0.x, c0.y, c0.z, c0.w};
                const float c1v[4] = {c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint32_t bb = *reinterpret_cast<const uint32_t*>(bs + (size_t)(lane + 32 * m) * PB + j);
                    const float b0 = __uint_as_float(bb << 16), b1 = __uint_as_float(bb & 0xffff0000u);
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        a[t][m] = __fmaf_rn(b0, c0v[t], a[t][m]);
                        a[t][m] = __fmaf_rn(b1, c1v[t], a[t][m]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int sl = s0 + t;
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    a[t][m] = __fsub_rn(__bfloat162float(xb[(size_t)sl * kEncXB + lane + 32 * m]), a[t][m]);
            }
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const int sl = s0 + t;
                if (sl >= nvalid) break;
                const float r4[4] = {a[t][0], a[t][1], a[t][2], a[t][3]};
                quantize_store<BITS>(r4, sblk[sl], sR[sl], sprow[sl] & 0xff, G.ts[sprow[sl] >> 8], rstage, chstage, G.c8,
                                     C.gate ? C.gate[((size_t)srow[sl] * G.Hkv + h) * 2 + z] : 1.f);
            }
        }
    }
}

// ------------------------------------------------------------------------------------
// The decode's copy of B_K in 8 x 8 tiles (tiled_basis_off), one block per (group, kv-head).
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) tile_basis_kernel(const Geom G, const State S) {
    const size_t base = (size_t)blockIdx.x * kD * G.r_max;
    __nv_bfloat16* dst = const_cast<__nv_bfloat16*>(S.basis_kt) + base;
    for (int e = threadIdx.x; e < kD * G.r_max; e += blockDim.x) {
        const int i = e / G.r_max, j = e % G.r_max;
        dst[tiled_basis_off(i, j, G.r_max)] = S.basis_k[base + e];
    }
}

// ------------------------------------------------------------------------------------
// The kernels' bounded wait, exercised (test support): one thread waits on a shared-memory
// barrier that nothing arrives at; the wait runs out after limit_ns and the kernel records
// DWKV_DEV_TIMEOUT in the device error word, as every kernel does, then returns.
// ------------------------------------------------------------------------------------
__global__ void wait_timeout_kernel(const State S, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_addr(&bar);
    mbar_init(b, 1);
    fence_mbar_init();
    if (!mbar_wait_for(b, 0, limit_ns)) set_dev_error(S, 6u /*DWKV_DEV_TIMEOUT*/, 0xfffffffeu, 0u);
}

// ------------------------------------------------------------------------------------
// Steps 4-6 alone on given residuals (test support): a warp per vector runs quantize_store
// into a page-layout block of its own in `work` (rank 0, row 0), then copies the indices,
// codes (int4 unpacked, sign-extended) and the scale out into plain arrays.
// ------------------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256) quantize_test_kernel(int n, int s, const float* __restrict__ r,
                                                            uint8_t* idx, int8_t* codes, uint16_t* scales,
                                                            uint8_t* work, uint32_t stride) {
    __shared__ __align__(16) uint8_t stage[8 * kEncStage];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int v = blockIdx.x * 8 + warp;
    if (v >= n) return;                         // whole warps
    float rr[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) rr[m] = r[(size_t)v * kD + lane + 32 * m];
    uint8_t* blk = work + (size_t)v * stride;
    float* rstage = reinterpret_cast<float*>(stage + warp * kEncStage);
    quantize_store<BITS>(rr, blk, 0, 0, s, rstage, reinterpret_cast<uint8_t*>(rstage + kD), 0);
    __syncwarp();
    for (int b = lane; b < s; b += 32) {
        idx[(size_t)v * s + b] = blk[off_idx_of(0) + b];
        int c;
        if (BITS == 8) {
            c = (int8_t)blk[off_codes_of(0, s) + b];
        } else {
            const uint32_t byte = blk[off_codes_of(0, s) + (b >> 1)];
            c = (int)(((b & 1) ? byte >> 4 : byte) & 0xfu);
            c = (c ^ 8) - 8;
        }
        codes[(size_t)v * s + b] = (int8_t)c;
    }
    if (lane == 0) scales[v] = *reinterpret_cast<const uint16_t*>(blk + off_scales_of(0, s, BITS));
}

// ------------------------------------------------------------------------------------
// Decode-time append (a few tokens per sequence): one block per (sequence in call, kv-head)
// places the sequence's new positions (when this layer is the group's first to append them)
// and encodes its rows, in one launch.  The bases load while the placement runs.
// ------------------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256) append_small_kernel(const Geom G, const State S, const AppendCall C,
                                                           const uint8_t* __restrict__ tier_idx, int place,
                                                           const __nv_bfloat16* __restrict__ k_new,
                                                           const __nv_bfloat16* __restrict__ v_new,
                                                           float* coeff_dbg) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int i = blockIdx.x, h = blockIdx.y, warp = threadIdx.x >> 5;
    __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(smem);
    // The global round trips overlap: the bases, this warp's unit (x and, when nothing is
    // placed, its destination) and the placement are all in flight together.
    uint4 bv[kBasisRegs];
    bases_issue(G, S, C.g, h, bv);
    const int u0 = 2 * C.tok0[i], u1 = 2 * C.tok0[i + 1];
    const int unit = u0 + warp;                    // at most 4 rows: one unit per warp
    UnitIn in;
    in.ok = false;
    if (!place && unit < u1) in = encode_fetch(G, S, C, k_new, v_new, h, unit, coeff_dbg);
    if (place) place_block(G, S, C, tier_idx, i, h);
    bases_store(G, bv, bs);
    __syncthreads();                         // bases in smem; slots and pages written (block scope)
    if (unit < u1) {
        if (place) in = encode_fetch(G, S, C, k_new, v_new, h, unit, coeff_dbg);
        encode_body<BITS>(G, S, bs, enc_scratch(G, smem, warp), unit, in);
    }
}

// ------------------------------------------------------------------------------------
// Import of already compressed tokens: one warp per token row (keys and values).
// ------------------------------------------------------------------------------------
// Bytes of one coefficient record of the import / export arrays: bf16 [r_max], or int8 codes
// [r_max] then fp16 block scales [r_max / 16].
__host__ __device__ inline size_t coeff_record_bytes(const Geom& G) {
    return G.c8 ? (size_t)G.r_max + G.r_max / 8 : (size_t)2 * G.r_max;
}

template <int BITS>
__global__ void __launch_bounds__(256) import_kernel(const Geom G, const State S, const AppendCall C,
                                                     const uint8_t* __restrict__ coeff,
                                                     const uint8_t* __restrict__ idx,
                                                     const int8_t* __restrict__ codes,
                                                     const __half* __restrict__ scales) {
    const int h = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5, s = G.s, RM = G.r_max;
    for (int row = blockIdx.x * nw + warp; row < C.total; row += gridDim.x * nw) {
        const int ci = call_index_of(C, row);
        const int seq = C.seq[ci];
        const int pos = C.pos0[ci] + (row - C.tok0[ci]);
        Dest dst;
        if (!find_dest(G, S, seq, C.g, C.lig, h, pos, dst)) {
            if (lane == 0 && !(pos >= C.a0[ci] && pos < C.a0[ci] + C.na[ci]))
                set_dev_error(S, 5u, (uint32_t)seq, (uint32_t)pos);
            continue;
        }
        const int R = dst.R, st = G.ts[dst.k];        // the row's tier keeps st <= s entries
        const int c8 = G.c8;
        const size_t crb = coeff_record_bytes(G);
        for (int z = 0; z < 2; ++z) {
            const size_t src = ((size_t)row * G.Hkv + h) * 2 + z;
            uint8_t* blk = dst.blk + (z ? G.blk_bytes[dst.k] : 0u);
            const uint8_t* rec = coeff + src * crb;
            if (c8) {
                for (int j = lane; j < R; j += 32)
                    blk[z ? vc8_code_off(j, dst.row) : kc8_code_off(j, dst.row)] = rec[j];
                for (int b = lane; b < R / 16; b += 32)
                    *reinterpret_cast<uint16_t*>(blk + (z ? vc8_scale_off(R, b, dst.row) : kc8_scale_off(R, b, dst.row))) =
                        *reinterpret_cast<const uint16_t*>(rec + RM + 2 * b);
            } else {
                for (int j = lane; j < R; j += 32)
                    *reinterpret_cast<uint16_t*>(blk + (j >> 3) * 1024 + dst.row * 16 + (j & 7) * 2) =
                        reinterpret_cast<const uint16_t*>(rec)[j];
            }
            for (int e = lane; e < st; e += 32) {
                const uint8_t ch = idx[src * s + e];
                if (ch >= kD) set_dev_error(S, 3u /*DWKV_DEV_BAD_CHANNEL*/, (uint32_t)seq, (uint32_t)pos);
                blk[off_idx_of(R, c8) + dst.row * st + e] = ch;
                if (BITS == 8) blk[off_codes_of(R, st, c8) + dst.row * st + e] = (uint8_t)codes[src * s + e];
            }
            if (BITS == 4) {
                for (int b = lane; b < st / 2; b += 32) {
                    const int c0 = codes[src * s + 2 * b], c1 = codes[src * s + 2 * b + 1];
                    if (c0 < -8 || c0 > 7 || c1 < -8 || c1 > 7)
                        set_dev_error(S, 4u /*DWKV_DEV_BAD_CODE*/, (uint32_t)seq, (uint32_t)pos);
                    blk[off_codes_of(R, st, c8) + dst.row * (st / 2) + b] =
                        (uint8_t)(((uint32_t)c0 & 0xfu) | (((uint32_t)c1 & 0xfu) << 4));
                }
            }
            if (lane == 0 && st)
                *reinterpret_cast<__half*>(blk + off_scales_of(R, st, BITS, c8) + dst.row * 2) = scales[src];
        }
    }
}

// ------------------------------------------------------------------------------------
// Export of positions [t0, t0+n) of (layer, seq), token-ordered.  One warp per (token, h).
// ------------------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256) export_kernel(const Geom G, const State S, int layer, int seq, int t0,
                                                     int n, uint8_t* tier_out, uint8_t* coeff_out,
                                                     uint8_t* idx_out, int8_t* codes_out, __half* scales_out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int g = layer / G.LPG, lig = layer % G.LPG, s = G.s, RM = G.r_max;
    for (int w = blockIdx.x * nw + warp; w < n * G.Hkv; w += gridDim.x * nw) {
        const int t = w / G.Hkv, h = w % G.Hkv;
        Dest dst;
        const bool ok = find_dest(G, S, seq, g, lig, h, t0 + t, dst);
        if (tier_out && lane == 0) tier_out[w] = ok ? (uint8_t)dst.k : (uint8_t)0xff;
        for (int z = 0; z < 2; ++z) {
            const size_t o = (size_t)w * 2 + z;
            const uint8_t* blk = ok ? dst.blk + (z ? G.blk_bytes[dst.k] : 0u) : nullptr;
            const int R = ok ? dst.R : 0, st = ok ? G.ts[dst.k] : 0;   // entries past st read as 0
            const int c8 = G.c8;
            if (coeff_out) {
                uint8_t* rec = coeff_out + o * coeff_record_bytes(G);
                if (c8) {
                    for (int j = lane; j < RM; j += 32)
                        rec[j] = j < R ? blk[z ? vc8_code_off(j, dst.row) : kc8_code_off(j, dst.row)] : 0;
                    for (int b = lane; b < RM / 16; b += 32)
                        *reinterpret_cast<uint16_t*>(rec + RM + 2 * b) =
                            16 * b < R ? *reinterpret_cast<const uint16_t*>(
                                             blk + (z ? vc8_scale_off(R, b, dst.row) : kc8_scale_off(R, b, dst.row)))
                                       : (uint16_t)0;
                } else {
                    for (int j = lane; j < RM; j += 32)
                        reinterpret_cast<uint16_t*>(rec)[j] =
                            j < R ? *reinterpret_cast<const uint16_t*>(blk + (j >> 3) * 1024 + dst.row * 16 + (j & 7) * 2)
                                  : (uint16_t)0;
                }
            }
            for (int e = lane; e < s; e += 32) {
                const bool on = e < st;
                if (idx_out) idx_out[o * s + e] = on ? blk[off_idx_of(R, c8) + dst.row * st + e] : 0;
                if (codes_out) {
                    int c = 0;
                    if (on) {
                        if (BITS == 8) c = (int8_t)blk[off_codes_of(R, st, c8) + dst.row * st + e];
                        else {
                            const uint32_t byte = blk[off_codes_of(R, st, c8) + dst.row * (st / 2) + e / 2];
                            const uint32_t nib = (e & 1) ? (byte >> 4) : (byte & 0xfu);
                            c = (int)(nib ^ 8u) - 8;
                        }
                    }
                    codes_out[o * s + e] = (int8_t)c;
                }
            }
            if (scales_out && lane == 0)
                scales_out[o] = st ? *reinterpret_cast<const __half*>(blk + off_scales_of(R, st, BITS, c8) + dst.row * 2)
                                   : __float2half_rn(0.f);
        }
    }
}

// ------------------------------------------------------------------------------------
// Reset of one sequence: its pages go to the tiers' free rings, its counts go to zero.
// Single block; stream-ordered with every other kernel, so no pop runs concurrently.
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) reset_kernel(const Geom G, const State S, int seq) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ uint32_t s_head, s_tail, s_warp[8], s_total;
    const int pairs = G.G * G.Hkv;
    for (int k = 0; k < G.ntiers; ++k) {
        if (tid == 0) {
            uint32_t hd = S.free_head[k], tl = S.free_tail[k];
            if ((int)(hd - tl) > 0) hd = tl;        // pops overshot: the ring was empty
            s_head = hd;
            s_tail = tl;
        }
        __syncthreads();
        for (int base = 0; base < pairs; base += blockDim.x) {
            const int pr = base + tid;
            uint32_t np = 0;
            int g = 0, h = 0;
            if (pr < pairs) {
                g = pr / G.Hkv;
                h = pr % G.Hkv;
                np = S.owned[cnt_index(G, seq, g, h) + k];
            }
            uint32_t incl = np;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (lane == 31) s_warp[warp] = incl;
            __syncthreads();
            if (tid == 0) {
                uint32_t acc = 0;
                for (int w = 0; w < (int)(blockDim.x >> 5); ++w) { const uint32_t v = s_warp[w]; s_warp[w] = acc; acc += v; }
                s_total = acc;
            }
            __syncthreads();
            const uint32_t excl = s_warp[warp] + incl - np;
            const bool room = (s_tail - s_head) + s_total <= G.free_cap;
            if (pr < pairs && np) {
                if (room) {
                    const size_t pi = page_index(G, seq, g, h, k);
                    for (uint32_t q = 0; q < np; ++q)
                        S.free_list[(size_t)k * G.free_cap + ((s_tail + excl + q) & (G.free_cap - 1))] = S.pages[pi + q];
                } else {
                    set_dev_error(S, 7u /*DWKV_DEV_FREE_LIST*/, (uint32_t)seq, (uint32_t)k);
                }
            }
            __syncthreads();
            if (tid == 0 && room) s_tail += s_total;
            __syncthreads();
        }
        if (tid == 0) {
            S.free_head[k] = s_head;
            S.free_tail[k] = s_tail;
        }
        __syncthreads();
    }
    for (int e = tid; e < pairs * kMaxTiers; e += blockDim.x) {
        S.counts[cnt_index(G, seq, 0, 0) + e] = 0u;
        S.owned[cnt_index(G, seq, 0, 0) + e] = 0u;
    }
}

// ------------------------------------------------------------------------------------
// Re-tiering ("DepthWeave-KV ...", §3, Eq. (2)-(3) paragraphs: the probe's feedback moves the
// router threshold, so a token's rank tier changes).  One block per (sequence in call,
// kv-head) takes the call's tokens of its sequence in order; for each token whose tier
// changes:
//   1. a slot at the end of the new tier (place_one: slot map and page position updated);
//   2. every layer's keys and values re-encoded there from the token's reconstruction, a_i =
//      fma chain over j < r_old of B[i][j] cb_j from +0, plus scale * code on its residual
//      channels, rounded to bf16 (the dense vector is not kept), by the six encode steps at
//      the new rank (encode_body: the same operations as every encoder);
//   3. the old tier's last slot moved into the token's old slot (all layers' rows and the
//      page position; the moved token's slot-map entry follows), and both counts updated.
// Softmax is order-free, so the order of slots within a tier does not matter; a page the old
// tier empties stays with the tier (owned) until retier_release_kernel returns it.
// ------------------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256) retier_kernel(const Geom G, const State S, const RetierCall C,
                                                     const int32_t* __restrict__ positions,
                                                     const uint8_t* __restrict__ new_tier) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int i = blockIdx.x, h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(smem);
    {
        uint4 bv[kBasisRegs];
        bases_issue(G, S, C.g, h, bv);
        bases_store(G, bv, bs);
    }
    __shared__ int s_go, s_kold, s_knew, s_slot, s_last;
    __shared__ uint32_t s_unit_old, s_unit_last;
    __shared__ Dest s_dst;
    const int seq = C.seq[i], P = G.r_max + 2;
    const size_t ci = cnt_index(G, seq, C.g, h);
    for (int t = C.begin[i]; t < C.end[i]; ++t) {
        __syncthreads();                               // the previous token is done
        if (tid == 0) {
            int go = 0;
            const int pos = positions[t];
            const uint32_t knew = new_tier[(size_t)t * G.Hkv + h];
            const uint32_t sm = (pos >= 0 && pos < G.max_context) ? S.slot_map[slot_index(G, seq, C.g, h, pos)] : 0u;
            if (sm == 0u) {
                set_dev_error(S, 5u /*DWKV_DEV_NO_SLOT*/, (uint32_t)seq, (uint32_t)pos);
            } else if (knew >= (uint32_t)G.ntiers) {
                set_dev_error(S, 2u /*DWKV_DEV_BAD_TIER*/, (uint32_t)seq, (uint32_t)pos);
            } else {
                const uint32_t kold = (sm >> 24) - 1u, slot = sm & 0xffffffu;
                Dest d;
                if (kold != knew && place_one(G, S, seq, C.g, h, pos, knew, d, 0)) {
                    const size_t po = page_index(G, seq, C.g, h, (int)kold);
                    const uint32_t last = S.counts[ci + kold] - 1u;
                    s_kold = (int)kold;
                    s_knew = (int)knew;
                    s_slot = (int)slot;
                    s_last = (int)last;
                    s_unit_old = S.pages[po + slot / kPage];
                    s_unit_last = S.pages[po + last / kPage];
                    s_dst = d;
                    go = 1;
                }
            }
            s_go = go;
        }
        __syncthreads();
        if (!s_go) continue;
        const int kold = s_kold, knew = s_knew, slot = s_slot, last = s_last;
        const int Rold = G.tiers[kold], sold = G.ts[kold], row = slot % kPage;
        // ---- 2: re-encode every (layer, K / V) unit of the token, a warp each
        for (int u = warp; u < 2 * G.LPG; u += (int)(blockDim.x >> 5)) {
            const int lig = u >> 1, z = u & 1;
            const uint8_t* ob = S.data + (size_t)s_unit_old * kUnit + (size_t)lig * G.chunk_bytes[kold] +
                                (z ? G.blk_bytes[kold] : 0u);
            const __nv_bfloat16* bz = bs + (size_t)z * kD * P;
            // the token's stored entries read in parallel (lane j holds coefficients j + 32 q
            // and residual entry j), then handed round by shuffles in the chain's order
            float cl[kMaxRank / 32];
#pragma unroll
            for (int q = 0; q < kMaxRank / 32; ++q) {
                const int j = lane + 32 * q;
                cl[q] = j < Rold ? stored_coeff(ob, G.c8, z, Rold, row, j) : 0.f;
            }
            int ch_l = 0;
            float v_l = 0.f;
            if (sold > 0 && lane < sold) stored_resid<BITS>(ob, G.c8, Rold, sold, row, lane, ch_l, v_l);
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j = 0; j < Rold; j += 2) {              // Rold is even: the basis read a pair at a time
                float src = cl[0];
#pragma unroll
                for (int q = 1; q < kMaxRank / 32; ++q) if ((j >> 5) == q) src = cl[q];
                const float cj = __shfl_sync(0xffffffffu, src, j & 31);
                const float cj1 = __shfl_sync(0xffffffffu, src, (j + 1) & 31);   // j + 1 in the same 32
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(bz + (size_t)(lane + 32 * m) * P + j);
                    a[m] = __fmaf_rn(bf16lo(w), cj, a[m]);
                    a[m] = __fmaf_rn(bf16hi(w), cj1, a[m]);
                }
            }
            for (int e = 0; e < sold; ++e) {
                const int ch = __shfl_sync(0xffffffffu, ch_l, e);
                const float v = __shfl_sync(0xffffffffu, v_l, e);
                if ((ch & 31) == lane && ch < kD) {
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        if ((ch >> 5) == m) a[m] = __fadd_rn(a[m], v);
                }
            }
            UnitIn in;
            in.ok = true;
            in.dbg = nullptr;
            in.dst = s_dst;
            in.dst.blk = s_dst.blk + (size_t)lig * G.chunk_bytes[knew];
#pragma unroll
            for (int m = 0; m < 4; ++m) in.xr[m] = __bfloat162float(__float2bfloat16_rn(a[m]));
            encode_body<BITS>(G, S, bs, enc_scratch(G, smem, warp), z, in);
        }
        __syncthreads();
        // ---- 3: the old tier's last slot into the token's old slot
        if (slot != last) {
            const int lrow = last % kPage;
            for (int u = warp; u < 2 * G.LPG; u += (int)(blockDim.x >> 5)) {
                const int lig = u >> 1, z = u & 1;
                const size_t o = (size_t)lig * G.chunk_bytes[kold] + (z ? G.blk_bytes[kold] : 0u);
                move_row<BITS>(S.data + (size_t)s_unit_old * kUnit + o, S.data + (size_t)s_unit_last * kUnit + o, G.c8,
                               z, Rold, sold, row, lrow);
            }
            if (tid == 0) {
                const int32_t* lp = reinterpret_cast<const int32_t*>(S.data + (size_t)s_unit_last * kUnit + pos_block_of(G, kold));
                int32_t* sp = reinterpret_cast<int32_t*>(S.data + (size_t)s_unit_old * kUnit + pos_block_of(G, kold));
                const int32_t moved = lp[lrow];
                sp[row] = moved;
                S.slot_map[slot_index(G, seq, C.g, h, moved)] = ((uint32_t)(kold + 1) << 24) | (uint32_t)slot;
            }
        }
        if (tid == 0) {
            S.counts[ci + kold] = (uint32_t)last;
            S.counts[ci + knew] += 1u;
        }
    }
}

// After re-tiering: the pages a tier holds beyond ceil(count / 64) go back to the tier's free
// ring.  One block for the whole call (no other kernel takes from the rings meanwhile).
__global__ void __launch_bounds__(256) retier_release_kernel(const Geom G, const State S, const RetierCall C) {
    const int tid = threadIdx.x;
    __shared__ uint32_t s_tail[kMaxTiers], s_total[kMaxTiers], s_over[kMaxTiers];
    if (tid < kMaxTiers) {
        s_total[tid] = 0u;
        s_over[tid] = 0u;
        s_tail[tid] = tid < G.ntiers ? S.free_tail[tid] : 0u;
    }
    __syncthreads();
    const int pairs = C.n * G.Hkv;
    // 1: how many pages each tier gives back
    for (int e = tid; e < pairs * G.ntiers; e += blockDim.x) {
        const int k = e % G.ntiers, pr = e / G.ntiers;
        const size_t ci = cnt_index(G, C.seq[pr / G.Hkv], C.g, pr % G.Hkv);
        const uint32_t keep = (S.counts[ci + k] + kPage - 1) / kPage, ow = S.owned[ci + k];
        if (ow > keep) atomicAdd(&s_total[k], ow - keep);
    }
    __syncthreads();
    if (tid < G.ntiers) {
        // pops on an empty ring move the head past the tail; no kernel pops meanwhile, so bring
        // it back before the pushes (as the reset does)
        uint32_t hd = S.free_head[tid];
        if ((int)(hd - s_tail[tid]) > 0) {
            hd = s_tail[tid];
            S.free_head[tid] = hd;
        }
        if ((s_tail[tid] - hd) + s_total[tid] > G.free_cap) {
            s_over[tid] = 1u;
            set_dev_error(S, 7u /*DWKV_DEV_FREE_LIST*/, 0xffffffffu, (uint32_t)tid);
        }
        s_total[tid] = 0u;
    }
    __syncthreads();
    // 2: push them (ring order does not matter)
    for (int e = tid; e < pairs * G.ntiers; e += blockDim.x) {
        const int k = e % G.ntiers, pr = e / G.ntiers;
        const int seq = C.seq[pr / G.Hkv], h = pr % G.Hkv;
        const size_t ci = cnt_index(G, seq, C.g, h);
        const uint32_t keep = (S.counts[ci + k] + kPage - 1) / kPage, ow = S.owned[ci + k];
        if (ow > keep && !s_over[k]) {
            const uint32_t at = atomicAdd(&s_total[k], ow - keep);
            const size_t pi = page_index(G, seq, C.g, h, k);
            for (uint32_t q = keep; q < ow; ++q)
                S.free_list[(size_t)k * G.free_cap + ((s_tail[k] + at + q - keep) & (G.free_cap - 1))] = S.pages[pi + q];
            S.owned[ci + k] = keep;
        }
    }
    __syncthreads();
    if (tid < G.ntiers && !s_over[tid]) S.free_tail[tid] = s_tail[tid] + s_total[tid];
}

}  // namespace dwkv

namespace dwkv {
template __global__ void retier_kernel<8>(const Geom, const State, const RetierCall, const int32_t*, const uint8_t*);
template __global__ void retier_kernel<4>(const Geom, const State, const RetierCall, const int32_t*, const uint8_t*);
template __global__ void encode_kernel<8>(const Geom, const State, const AppendCall, const __nv_bfloat16*,
                                          const __nv_bfloat16*, float*);
template __global__ void encode_kernel<4>(const Geom, const State, const AppendCall, const __nv_bfloat16*,
                                          const __nv_bfloat16*, float*);
template __global__ void quantize_test_kernel<8>(int, int, const float*, uint8_t*, int8_t*, uint16_t*, uint8_t*,
                                                  uint32_t);
template __global__ void quantize_test_kernel<4>(int, int, const float*, uint8_t*, int8_t*, uint16_t*, uint8_t*,
                                                  uint32_t);
template __global__ void append_small_kernel<8>(const Geom, const State, const AppendCall, const uint8_t*, int,
                                                const __nv_bfloat16*, const __nv_bfloat16*, float*);
template __global__ void append_small_kernel<4>(const Geom, const State, const AppendCall, const uint8_t*, int,
                                                const __nv_bfloat16*, const __nv_bfloat16*, float*);
template __global__ void import_kernel<8>(const Geom, const State, const AppendCall, const uint8_t*,
                                          const uint8_t*, const int8_t*, const __half*);
template __global__ void import_kernel<4>(const Geom, const State, const AppendCall, const uint8_t*,
                                          const uint8_t*, const int8_t*, const __half*);
template __global__ void export_kernel<8>(const Geom, const State, int, int, int, int, uint8_t*, uint8_t*,
                                          uint8_t*, int8_t*, __half*);
template __global__ void export_kernel<4>(const Geom, const State, int, int, int, int, uint8_t*, uint8_t*,
                                          uint8_t*, int8_t*, __half*);
}  // namespace dwkv
