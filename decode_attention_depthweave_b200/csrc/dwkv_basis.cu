// dwkv_basis.cu -- online construction of the shared bases ("DepthWeave-KV ...", §3 Method,
// the shared-bases paragraph): the window's channel second moment from dense rows on the
// tensor cores, the basis from a randomized sketch of it (subspace iterations, Gram-Schmidt
// with re-orthogonalisation, a Rayleigh-Ritz step by cyclic Jacobi), the moving-average
// update, and the re-projection of stored tokens onto an updated basis.
//
// Reading (the pages fix none of these numbers): C = sum over the window's layers and rows of
// x x^T per (kv-head, K / V); Y = C Omega (Omega an input test matrix [d][r_max]); Q = GS(Y);
// power_steps times Q = GS(C Q); T = Q^T C Q = U diag(lambda) U^T with lambda descending;
// B = Q U with each column's largest-magnitude entry (lowest channel among equals) positive,
// rounded to bf16.  Update: C <- beta C + (1 - beta) C_new, then Q = GS(C B_old) and the same
// Rayleigh-Ritz step.  Stored tokens: reconstruction on B_old (the re-tiering chain), then the
// six encode steps on B_new at the same tier.
#include <cuda.h>                                  // CUtensorMap

#include "dwkv_encode.cuh"
#include "dwkv_stored.cuh"

namespace dwkv {

// ------------------------------------------------------------------------------------
// Second moment C[w][h][z] += scale * X^T X over the rows of window w's layers (rows = LPG x
// n_rows, layer-major; blockIdx.y = w Hkv + h) on the 5th-generation tensor cores: X^T X is
// one 128 x 128 x 64 product per chunk of 64 rows, accumulated in tensor memory.
//  - A block of 4 warps holds 128 TMEM columns (the fp32 128 x 128 accumulator, row i in lane
//    i) and kGramStages chunk buffers in shared memory.
//  - One thread runs the pipeline: a chunk arrives by two TMA copies (channels 0-63 and 64-127
//    of its 64 rows, through a 4-D tensor map channels x heads x rows x windows; rows past the
//    window's end read as zeros), each 64 rows x 128 bytes in the 128-byte swizzle, which is
//    the MN-major swizzled operand layout: 8-row atoms kGramSbo apart, the two channel halves
//    kGramLbo apart.  A = X^T (M = channels) and B = X (N = channels) are the same bytes under
//    the same descriptor.  The thread issues the chunk's four K = 16 MMAs once its copies have
//    landed and commits them to the buffer's "empty" mbarrier; the buffer is refilled only
//    after that commit has arrived.
//  - After the last chunk each warp reads its 32 rows with tcgen05.ld and adds them into C with
//    fp32 atomics (a row segment of 32 floats an instruction), so the order of the sum is not
//    fixed.
// Every wait is bounded: a wait that runs out records DWKV_DEV_TIMEOUT, waits (bounded) for the
// MMAs issued so far, frees the tensor memory and leaves C unchanged by this block.
// ------------------------------------------------------------------------------------
constexpr int kGramRows = 64;                      // K of a chunk
constexpr int kGramStages = 3;
constexpr uint32_t kGramHalfBytes = (uint32_t)kGramRows * 128u;           // 64 rows x 64 channels
constexpr uint32_t kGramStageBytes = 2u * kGramHalfBytes;                 // 16 KB
constexpr uint32_t kGramSbo = 1024u;               // 8-row atom stride (8 rows x 128 B)
constexpr uint32_t kGramLbo = kGramHalfBytes;      // channel-half stride
constexpr uint32_t kGramTmemCols = 128u;
// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits 4-5 = 1), A and B
// bf16 (bits 7-9 = 1, 10-12 = 1), A and B MN-major (bits 15, 16), N >> 3 = 16 (bits 17-22),
// M >> 4 = 8 (bits 24-28).
constexpr uint32_t kGramIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                ((uint32_t)(kD >> 3) << 17) | ((uint32_t)(kD >> 4) << 24);

// stages (1024-byte aligned for the swizzle, hence the slack), then 2 kGramStages mbarriers and
// the tensor-memory address
size_t gram_smem_bytes() { return (size_t)kGramStages * kGramStageBytes + 1024 + 64; }

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading (channel-half) and
// stride (8-row atom) byte offsets, each >> 4, descriptor version 1 (bits 46-47), layout type
// 2 (bits 61-63).
__device__ __forceinline__ uint64_t gram_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)((kGramLbo >> 4) & 0x3fffu) << 16) |
           ((uint64_t)((kGramSbo >> 4) & 0x3fffu) << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
        "%5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

__global__ void __launch_bounds__(128) gram_kernel(const __grid_constant__ CUtensorMap tmap_k,
                                                   const __grid_constant__ CUtensorMap tmap_v, const Geom G,
                                                   const State S, int n_rows, int rows_per_block,
                                                   float* __restrict__ cacc, float scale) {
    extern __shared__ __align__(1024) uint8_t gsm[];
    __shared__ int s_ok;
    const int h = blockIdx.y % G.Hkv, gw = blockIdx.y / G.Hkv, z = blockIdx.z;   // gw: window within the call
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int total = G.LPG * n_rows;                         // the window's rows (host: < 2^31)
    const int r0 = (int)blockIdx.x * rows_per_block;          // rows_per_block: a multiple of 64
    const int r1 = min(total, r0 + rows_per_block);
    const int nchunks = r1 > r0 ? (r1 - r0 + kGramRows - 1) / kGramRows : 0;
    if (nchunks == 0) return;                                 // uniform over the block
    const uint32_t raw = smem_addr(gsm);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    const uint32_t full = sbase + (uint32_t)kGramStages * kGramStageBytes;   // kGramStages mbarriers
    const uint32_t empty = full + 8u * kGramStages;                          // kGramStages mbarriers
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gsm + (empty + 8u * kGramStages - raw));
    const CUtensorMap* map = z ? &tmap_v : &tmap_k;
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(kGramTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int b = 0; b < kGramStages; ++b) {
            mbar_init(full + 8u * b, 1u);
            mbar_init(empty + 8u * b, 1u);
        }
        fence_mbar_init();
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    if (tid == 0) {
        bool ok = true;
        int issued = 0;                                       // chunks whose MMAs were issued
        for (int q = 0; ok && q < nchunks + kGramStages - 1; ++q) {
            if (q < nchunks) {                                // copies of chunk q
                const int b = q % kGramStages;
                // the buffer held chunk q - stages: its MMAs must have completed
                if (q >= kGramStages && !mbar_wait(empty + 8u * b, (uint32_t)((q / kGramStages - 1) & 1))) {
                    ok = false;
                    break;
                }
                const uint32_t dst = sbase + (uint32_t)b * kGramStageBytes;
                mbar_arrive_expect_tx(full + 8u * b, kGramStageBytes);
                tma_load_4d(dst, map, 0, h, r0 + kGramRows * q, gw, full + 8u * b);
                tma_load_4d(dst + kGramHalfBytes, map, 64, h, r0 + kGramRows * q, gw, full + 8u * b);
            }
            const int c = q - (kGramStages - 1);              // MMAs of chunk c
            if (c >= 0) {
                const int b = c % kGramStages;
                if (!mbar_wait(full + 8u * b, (uint32_t)((c / kGramStages) & 1))) {
                    ok = false;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t buf = sbase + (uint32_t)b * kGramStageBytes;
#pragma unroll
                for (int kk = 0; kk < kGramRows / 16; ++kk) {
                    const uint64_t d = gram_desc(buf + (uint32_t)kk * 2u * kGramSbo);   // rows 16 kk .. 16 kk + 15
                    const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
                    asm volatile(
                        "{\n\t.reg .pred p;\n\t"
                        "setp.ne.b32 p, %4, 0;\n\t"
                        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                        ::"r"(tmem), "l"(d), "l"(d), "r"(kGramIdesc), "r"(acc) : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 empty + 8u * b)
                             : "memory");
                issued = c + 1;
            }
        }
        // the last commit covers every MMA issued (bounded: on a timeout the tensor memory is
        // still freed below, after this wait has given the MMAs its full limit)
        const bool done = issued > 0 && mbar_wait(empty + 8u * (uint32_t)((issued - 1) % kGramStages),
                                                  (uint32_t)(((issued - 1) / kGramStages) & 1));
        s_ok = (ok && done && issued == nchunks) ? 1 : 0;
    }
    __syncthreads();
    if (!s_ok) {
        if (tid == 0) set_dev_error(S, 6u /*DWKV_DEV_TIMEOUT*/, 0x67u, (uint32_t)blockIdx.y);
    } else {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // each 32 x 32 piece goes through the idle stage memory (a 33-float pitch), so that a
        // warp's atomics cover 32 consecutive floats of one row
        float* tile = reinterpret_cast<float*>(gsm + (sbase - raw)) + warp * 32 * 33;
        float* dst = cacc + (size_t)gw * G.Hkv * 2 * kD * kD + ((size_t)h * 2 + z) * kD * kD +
                     (size_t)(32 * warp) * kD + lane;
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += 32) {
            uint32_t v[32];
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
                "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                  "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                  "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                  "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                : "r"(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int j = 0; j < 32; ++j) tile[lane * 33 + j] = __uint_as_float(v[j]);
            __syncwarp();
#pragma unroll 4
            for (int r = 0; r < 32; ++r) atomicAdd(dst + (size_t)r * kD + c0, scale * tile[r * 33 + lane]);
            __syncwarp();
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGramTmemCols) : "memory");
    }
}

// c[e] *= beta over n floats.
__global__ void __launch_bounds__(256) moment_scale_kernel(float* c, size_t n, float beta) {
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (size_t)gridDim.x * blockDim.x)
        c[e] *= beta;
}

// ------------------------------------------------------------------------------------
// The basis of one (kv-head, K / V) of a window from its second moment: one block of 512
// threads, fp64 in shared memory (r_max <= 64).  omega (fp32 [d][r_max]) starts a sketch;
// without it the current basis starts one refresh step.  The [.][r] arrays have a row pitch
// of r + 1 doubles, so the column walks (Gram-Schmidt's dot products, the Jacobi rotations of
// columns) step across banks instead of hitting one.
// ------------------------------------------------------------------------------------
constexpr int kBasisThreads = 512;
size_t basis_smem_bytes(int r) {
    const size_t rp = (size_t)r + 1;
    return (2 * kD * rp + (size_t)r * rp + kD + 2 * (size_t)r + 32) * 8;
}

// Block-wide sum of one double per thread (kBasisThreads threads); every thread gets it.
__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double s = 0.0;
    for (int w = 0; w < kBasisThreads / 32; ++w) s += red[w];
    return s;
}

// W = C Q: C fp32 [d][d] (global), Q, W fp64 [d][r] with row pitch rp (shared).
__device__ void moment_times(const float* __restrict__ cm, const double* q, double* w, int r, int rp) {
    for (int e = threadIdx.x; e < kD * r; e += blockDim.x) {
        const int i = e / r, j = e % r;
        double a = 0.0;
        for (int k = 0; k < kD; ++k) a = fma((double)__ldg(cm + (size_t)i * kD + k), q[k * rp + j], a);
        w[i * rp + j] = a;
    }
    __syncthreads();
}

// Gram-Schmidt of the columns of q [d][r] (row pitch rp) in order, in place, each column
// orthogonalised twice against the previous ones (classical Gram-Schmidt, twice: orthogonal
// to rounding for any conditioning).  Returns false if a column vanishes.
__device__ bool orthonormalize(double* q, int r, int rp, double* dots, double* red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int j = 0; j < r; ++j) {
        for (int pass = 0; pass < 2; ++pass) {
            // dots[i] = q[:, i] . q[:, j] for i < j: a warp per i
            for (int i = warp; i < j; i += kBasisThreads / 32) {
                double a = 0.0;
                for (int row = lane; row < kD; row += 32) a = fma(q[row * rp + i], q[row * rp + j], a);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
                if (lane == 0) dots[i] = a;
            }
            __syncthreads();
            if (tid < kD) {
                double v = q[tid * rp + j];
                for (int i = 0; i < j; ++i) v = fma(-dots[i], q[tid * rp + i], v);
                q[tid * rp + j] = v;
            }
            __syncthreads();
        }
        const double x = tid < kD ? q[tid * rp + j] : 0.0;
        const double n2 = block_sum(x * x, red);
        if (!(n2 > 0.0)) return false;
        if (tid < kD) q[tid * rp + j] = x / sqrt(n2);
        __syncthreads();
    }
    return true;
}

__global__ void __launch_bounds__(kBasisThreads) basis_kernel(const Geom G, const State S, int g,
                                                              const float* __restrict__ moment,
                                                              const float* __restrict__ omega, int power_steps,
                                                              float* __restrict__ eig_out) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int r = G.r_max, rp = r + 1;
    const int h = blockIdx.x >> 1, z = blockIdx.x & 1;
    g += blockIdx.y;                                        // all-windows launches: one row of blocks a window
    moment += (size_t)blockIdx.y * G.Hkv * 2 * kD * kD;
    const int tid = threadIdx.x;
    double* q = reinterpret_cast<double*>(smem);            // [d][rp]
    double* w = q + kD * rp;                                // [d][rp]; later U [r][rp]
    double* t = w + kD * rp;                                // [r][rp]
    double* dots = t + r * rp;                              // [kD]
    double* lam = dots + kD;                                // [r]
    int* order = reinterpret_cast<int*>(lam + r);           // [2r]: Jacobi pairs, then ranks
    double* red = lam + 2 * r;                              // [16]
    const float* cm = moment + ((size_t)h * 2 + z) * kD * kD;
    const size_t boff = ((size_t)g * G.Hkv + h) * kD * r;
    __nv_bfloat16* bz = const_cast<__nv_bfloat16*>(z ? S.basis_v : S.basis_k) + boff;

    // ---- start: Y = C Omega, or C B_old
    for (int e = tid; e < kD * r; e += blockDim.x)
        w[(e / r) * rp + e % r] = omega ? (double)omega[e] : (double)__bfloat162float(bz[e]);
    __syncthreads();
    moment_times(cm, w, q, r, rp);
    bool ok = orthonormalize(q, r, rp, dots, red);
    for (int it = 0; ok && omega && it < power_steps; ++it) {
        moment_times(cm, q, w, r, rp);
        for (int e = tid; e < kD * r; e += blockDim.x) q[(e / r) * rp + e % r] = w[(e / r) * rp + e % r];
        __syncthreads();
        ok = orthonormalize(q, r, rp, dots, red);
    }
    if (!ok) {
        if (tid == 0) set_dev_error(S, 8u /*DWKV_DEV_BASIS*/, (uint32_t)g, (uint32_t)blockIdx.x);
        return;                                            // the basis stays as it was
    }
    // ---- Rayleigh-Ritz: T = Q^T (C Q), symmetric; U = I
    moment_times(cm, q, w, r, rp);
    for (int e = tid; e < r * r; e += blockDim.x) {
        const int a = e / r, b = e % r;
        double s = 0.0;
        for (int i = 0; i < kD; ++i) s = fma(q[i * rp + a], w[i * rp + b], s);
        t[a * rp + b] = s;
    }
    __syncthreads();
    for (int e = tid; e < r * r; e += blockDim.x) {
        const int a = e / r, b = e % r;
        if (a < b) { const double m = 0.5 * (t[a * rp + b] + t[b * rp + a]); t[a * rp + b] = m; t[b * rp + a] = m; }
    }
    double* u = w;                                          // [r][rp]
    for (int e = tid; e < r * r; e += blockDim.x) u[(e / r) * rp + e % r] = (e / r == e % r) ? 1.0 : 0.0;
    __syncthreads();
    // ---- cyclic Jacobi, round-robin pairs (circle method): r / 2 disjoint rotations a round
    double* cs = dots;                                      // [r/2] c, then [r/2] s
    int* pq = order;                                        // [r/2] p, [r/2] q
    const int np = r / 2;
    for (int sweep = 0; sweep < 20; ++sweep) {
        double off = 0.0, fro = 0.0;
        for (int e = tid; e < r * r; e += blockDim.x) {
            const double x = t[(e / r) * rp + e % r];
            fro += x * x;
            if (e / r != e % r) off += x * x;
        }
        off = block_sum(off, red);
        fro = block_sum(fro, red);
        if (!(off > 1e-28 * fro)) break;
        for (int rd = 0; rd < r - 1; ++rd) {
            if (tid < np) {
                int p, qq;
                if (tid == 0) { p = rd; qq = r - 1; }
                else { p = (rd + tid) % (r - 1); qq = (rd - tid + (r - 1)) % (r - 1); }
                if (p > qq) { const int x = p; p = qq; qq = x; }
                const double apq = t[p * rp + qq], app = t[p * rp + p], aqq = t[qq * rp + qq];
                double c = 1.0, sn = 0.0;
                if (apq != 0.0) {
                    const double tau = (aqq - app) / (2.0 * apq);
                    const double tt = tau >= 0.0 ? 1.0 / (tau + sqrt(1.0 + tau * tau)) : -1.0 / (-tau + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + tt * tt);
                    sn = tt * c;
                }
                cs[tid] = c;
                cs[np + tid] = sn;
                pq[tid] = p;
                pq[np + tid] = qq;
            }
            __syncthreads();
            // J^T T J by 2 x 2 blocks: the round's pairs are disjoint and cover every index, so
            // block (pair ka's rows, pair kb's columns) depends on its own four entries alone:
            // its rows are rotated first, then its columns (the operations of a rows pass
            // followed by a columns pass, in that order), in place by one thread
            for (int e = tid; e < np * np; e += blockDim.x) {
                const int ka = e / np, kb = e % np;
                const int pa = pq[ka], qa = pq[np + ka], pb = pq[kb], qb = pq[np + kb];
                const double c1 = cs[ka], s1 = cs[np + ka], c2 = cs[kb], s2 = cs[np + kb];
                const double tpp = t[pa * rp + pb], tpq = t[pa * rp + qb], tqp = t[qa * rp + pb], tqq = t[qa * rp + qb];
                const double rpp = c1 * tpp - s1 * tqp, rqp = s1 * tpp + c1 * tqp;   // rows, column pb
                const double rpq = c1 * tpq - s1 * tqq, rqq = s1 * tpq + c1 * tqq;   // rows, column qb
                t[pa * rp + pb] = c2 * rpp - s2 * rpq;
                t[pa * rp + qb] = s2 * rpp + c2 * rpq;
                t[qa * rp + pb] = c2 * rqp - s2 * rqq;
                t[qa * rp + qb] = s2 * rqp + c2 * rqq;
            }
            for (int e = tid; e < np * r; e += blockDim.x) {    // columns p, q of U: U J
                const int k = e / r, m = e % r, p = pq[k], qq = pq[np + k];
                const double c = cs[k], sn = cs[np + k];
                const double up = u[m * rp + p], uq = u[m * rp + qq];
                u[m * rp + p] = c * up - sn * uq;
                u[m * rp + qq] = sn * up + c * uq;
            }
            __syncthreads();
        }
    }
    // ---- eigenvalues in descending order (ties to the lower index), B = Q U, signs, bf16
    if (tid < r) lam[tid] = t[tid * rp + tid];
    __syncthreads();
    int* ord = order;                                       // ord[rank] = source column
    if (tid < r) {
        int rank = 0;
        for (int b = 0; b < r; ++b) rank += (lam[b] > lam[tid] || (lam[b] == lam[tid] && b < tid)) ? 1 : 0;
        ord[rank] = tid;
    }
    __syncthreads();
    {   // q <- B (unsigned) = Q U[:, ord]: a warp per row, the row's products in registers
        const int lane = tid & 31, warp = tid >> 5;
        const int o0 = lane, o1 = lane + 32;
        const int s0 = o0 < r ? ord[o0] : 0, s1 = o1 < r ? ord[o1] : 0;
        for (int i = warp; i < kD; i += kBasisThreads / 32) {
            double a0 = 0.0, a1 = 0.0;
            for (int j = 0; j < r; ++j) {
                const double qv = q[i * rp + j];
                a0 = fma(qv, u[j * rp + s0], a0);
                a1 = fma(qv, u[j * rp + s1], a1);
            }
            __syncwarp();                                   // every lane has read row i of Q
            if (o0 < r) q[i * rp + o0] = a0;
            if (o1 < r) q[i * rp + o1] = a1;
        }
        __syncthreads();
    }
    // signs: the column's entry of largest magnitude (lowest channel among equals) positive
    if (tid < r) {
        int best = 0;
        double bm = -1.0;
        for (int i = 0; i < kD; ++i) {
            const double m = fabs(q[i * rp + tid]);
            if (m > bm) { bm = m; best = i; }
        }
        dots[tid] = q[best * rp + tid] < 0.0 ? -1.0 : 1.0;
        if (eig_out) eig_out[(((size_t)blockIdx.y * G.Hkv + h) * 2 + z) * r + tid] = (float)lam[ord[tid]];
    }
    __syncthreads();
    __nv_bfloat16* tk = const_cast<__nv_bfloat16*>(S.basis_kt) + boff;
    for (int e = tid; e < kD * r; e += blockDim.x) {
        const int i = e / r, o = e % r;
        const __nv_bfloat16 v = __float2bfloat16_rn((float)(dots[o] * q[i * rp + o]));
        bz[e] = v;
        if (z == 0) tk[tiled_basis_off(i, o, r)] = v;
    }
}

// ------------------------------------------------------------------------------------
// Re-projection of the stored tokens of a window onto its updated basis: gridDim.z blocks per
// (sequence in the list, kv-head), half of them for the keys and half for the values (block z
// index even: keys).  A warp takes a group of up to kRpMaxGroup tokens of one tier and one layer
// of the window on its side (V = min(4, 64 / R) tokens: every lane busy in the projection),
// the groups dealt out over the side's warps.  Each token is reconstructed on the previous
// basis (old_k / old_v: the fixed-order fp32 chain over its rank, plus scale x code on its
// residual channels, rounded to bf16, as a re-tier does) and encoded on the new basis at its own
// tier, in place, by the six encode steps in the encoders' operation order:
//   0    the reconstructions share each basis load; the residual entries are added by a
//        shared-memory scatter (in entry order where a token repeats a channel);
//   1-2  lane (v, p) runs token v's projection chains of coefficients 2p and 2p + 1 over the
//        channels in order (a coefficient pair of the basis one 64-bit load, x four channels
//        a load), then rounds them to bf16 or forms their 8-bit blocks (a block of 16 on 8
//        lanes);
//   3    the residual chains of the group's tokens share each basis load;
//   4-6  quantize_store per token.
// The block's two bases are held as fp32 (the bf16 values exactly).  Slots and counts do not
// change.  Online bases have r_max <= 64.
// ------------------------------------------------------------------------------------
constexpr int kRpMaxGroup = 4;
constexpr int kRpThreads = 384;                    // 12 warps, 2 blocks an SM
constexpr int kRpXPitch = kD + 4;                  // floats: group rows on distinct banks
constexpr uint32_t kRpWarpBytes = (uint32_t)(kRpMaxGroup * kRpXPitch + kRpMaxGroup * 64 + 32) * 4u + 32u +
                                   (uint32_t)kRpMaxGroup * 16u;   // + the group's block addresses and rows

// Dynamic shared memory of reproject_kernel: the side's two bases as fp32 [d][r_max + 2] (the
// bf16 values exactly; a 64-bit load takes a pair of coefficients, and with the row pitch of
// r_max + 2 words a half warp's rows fall on distinct banks), then each warp's group scratch.
size_t reproject_smem_bytes(int r_max, int warps) {
    return (size_t)2 * kD * (r_max + 2) * 4 + (size_t)warps * kRpWarpBytes;
}

template <int BITS, int V>
__device__ __forceinline__ void reproject_group(const Geom& G, int z, int k, int nu, uint8_t* const* blk,
                                                const int* row, const float* bn, const float* bo,
                                                float* xs, float* cs, float* rstage, uint8_t* chstage) {
    const int lane = threadIdx.x & 31;
    const int P = G.r_max + 2, R = G.tiers[k], st = G.ts[k], c8 = G.c8;
    // ---- reconstruction on the previous basis: token u's entries read in parallel (lane j
    //      holds coefficient j and j + 32, residual entry j) and handed round by shuffles
    float cl0[V], cl1[V], v_l[V];
    int ch_l[V];
#pragma unroll
    for (int u = 0; u < V; ++u) {
        const bool on = u < nu;
        const uint8_t* b = blk[u];
        const int rw = row[u];
        cl0[u] = on && lane < R ? stored_coeff(b, c8, z, R, rw, lane) : 0.f;
        cl1[u] = on && lane + 32 < R ? stored_coeff(b, c8, z, R, rw, lane + 32) : 0.f;
        ch_l[u] = kD;
        v_l[u] = 0.f;
        if (on && lane < st) stored_resid<BITS>(b, c8, R, st, rw, lane, ch_l[u], v_l[u]);
    }
    {
        float a[V][4];
#pragma unroll
        for (int u = 0; u < V; ++u)
#pragma unroll
            for (int m = 0; m < 4; ++m) a[u][m] = 0.f;
        for (int j = 0; j < R; j += 2) {                 // R is even: the basis read a pair at a time
            float2 w[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) w[m] = *reinterpret_cast<const float2*>(bo + (size_t)(lane + 32 * m) * P + j);
#pragma unroll
            for (int u = 0; u < V; ++u) {
                const float cj = __shfl_sync(0xffffffffu, j < 32 ? cl0[u] : cl1[u], j & 31);
                const float cj1 = __shfl_sync(0xffffffffu, j + 1 < 32 ? cl0[u] : cl1[u], (j + 1) & 31);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    a[u][m] = __fmaf_rn(w[m].x, cj, a[u][m]);
                    a[u][m] = __fmaf_rn(w[m].y, cj1, a[u][m]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < V; ++u)
#pragma unroll
            for (int m = 0; m < 4; ++m) xs[u * kRpXPitch + lane + 32 * m] = a[u][m];
    }
    __syncwarp();
    // the residual entries: lane e adds entry e to its channel.  A token's channels are
    // distinct, so each channel takes at most one add and their order is free; a token whose
    // channels repeat takes its entries one at a time in entry order.  Channels >= d are
    // ignored.  Then the vector rounds to bf16.
#pragma unroll
    for (int u = 0; u < V; ++u) {
        if (st == 0) break;
        float* xu = xs + u * kRpXPitch;
        const bool has = ch_l[u] < kD;               // only lanes e < st of a live token hold one
        const uint32_t peers = __match_any_sync(0xffffffffu, has ? ch_l[u] : kD + lane);
        if (!__any_sync(0xffffffffu, has && __popc(peers) > 1)) {
            if (has) xu[ch_l[u]] = __fadd_rn(xu[ch_l[u]], v_l[u]);
        } else {
            for (int e = 0; e < st; ++e) {
                const int ch = __shfl_sync(0xffffffffu, ch_l[u], e);
                const float v = __shfl_sync(0xffffffffu, v_l[u], e);
                if (lane == 0 && ch < kD) xu[ch] = __fadd_rn(xu[ch], v);
                __syncwarp();
            }
        }
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < V; ++u)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float* x = xs + u * kRpXPitch + lane + 32 * m;
            *x = __bfloat162float(__float2bfloat16_rn(*x));
        }
    __syncwarp();                                        // every lane has read the old bytes; x in xs
    // ---- 1-2: projection, lane (v, p) = token v, coefficients 2p and 2p + 1
    {
        const int lpv = R >> 1, v = lane / lpv, p = lane - v * lpv, j = 2 * p;
        const bool on = v < V && v < nu;
        const float* xv = xs + (v < V ? v : 0) * kRpXPitch;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 2
        for (int i = 0; i < kD; i += 4) {
            const float4 x4 = *reinterpret_cast<const float4*>(xv + i);
            const float xq[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const float2 w = *reinterpret_cast<const float2*>(bn + (size_t)(i + ii) * P + j);
                acc0 = __fmaf_rn(w.x, xq[ii], acc0);
                acc1 = __fmaf_rn(w.y, xq[ii], acc1);
            }
        }
        float* cv = cs + (v < V ? v : 0) * 64;
        uint8_t* bv = blk[v < V ? v : 0];               // token v's block and row
        const int rv = row[v < V ? v : 0];
        if (c8) {
            // 8-bit blocks: the 16 coefficients of a block on 8 lanes (a pair each), lpv >= 8
            float mx = fmaxf(fabsf(acc0), fabsf(acc1));
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            const __half sh = __float2half_rn(__fdiv_rn(mx, 127.f));
            const float sf = __half2float(sh);
            float q0 = 0.f, q1 = 0.f;
            if (sf != 0.f) {
                q0 = fminf(fmaxf(rintf(__fdiv_rn(acc0, sf)), -127.f), 127.f);
                q1 = fminf(fmaxf(rintf(__fdiv_rn(acc1, sf)), -127.f), 127.f);
            }
            if (on) {
                bv[z ? vc8_code_off(j, rv) : kc8_code_off(j, rv)] = (uint8_t)(int8_t)(int)q0;
                bv[z ? vc8_code_off(j + 1, rv) : kc8_code_off(j + 1, rv)] = (uint8_t)(int8_t)(int)q1;
                if ((j & 15) == 0)
                    *reinterpret_cast<uint16_t*>(bv + (z ? vc8_scale_off(R, j >> 4, rv) : kc8_scale_off(R, j >> 4, rv))) =
                        __half_as_ushort(sh);
                *reinterpret_cast<float2*>(cv + j) = make_float2(q0 * sf, q1 * sf);
            }
        } else if (on) {
            __nv_bfloat162 cb;
            cb.x = __float2bfloat16_rn(acc0);
            cb.y = __float2bfloat16_rn(acc1);
            *reinterpret_cast<float2*>(cv + j) = make_float2(__bfloat162float(cb.x), __bfloat162float(cb.y));
            *reinterpret_cast<__nv_bfloat162*>(bv + (size_t)(j >> 3) * 1024 + rv * 16 + (j & 7) * 2) = cb;
        }
    }
    __syncwarp();
    // ---- 3: residuals against the stored coefficients (fma chain over j from +0), the group's
    //      tokens sharing each basis load
    float r[V][4];
    {
        float a[V][4];
#pragma unroll
        for (int u = 0; u < V; ++u)
#pragma unroll
            for (int m = 0; m < 4; ++m) a[u][m] = 0.f;
        for (int j0 = 0; j0 < R; j0 += 8) {              // R is a multiple of 8
#pragma unroll
            for (int jj = 0; jj < 8; jj += 2) {
                float2 w[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) w[m] = *reinterpret_cast<const float2*>(bn + (size_t)(lane + 32 * m) * P + j0 + jj);
#pragma unroll
                for (int u = 0; u < V; ++u) {
                    const float2 c2 = *reinterpret_cast<const float2*>(cs + u * 64 + j0 + jj);
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        a[u][m] = __fmaf_rn(w[m].x, c2.x, a[u][m]);
                        a[u][m] = __fmaf_rn(w[m].y, c2.y, a[u][m]);
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < V; ++u)
#pragma unroll
            for (int m = 0; m < 4; ++m) r[u][m] = __fsub_rn(xs[u * kRpXPitch + lane + 32 * m], a[u][m]);
    }
    // ---- 4-6 per token
#pragma unroll
    for (int u = 0; u < V; ++u)
        if (u < nu) quantize_store<BITS>(r[u], blk[u], R, row[u], st, rstage, chstage, c8);
    __syncwarp();
}

template <int BITS>
__global__ void __launch_bounds__(kRpThreads, 2) reproject_kernel(const Geom G, const State S, int g, const SeqList L,
                                                                   const __nv_bfloat16* __restrict__ old_k,
                                                                   const __nv_bfloat16* __restrict__ old_v) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int seq = L.seq[blockIdx.x], h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = (int)(blockDim.x >> 5);
    const int z = (int)(blockIdx.z & 1u), part = (int)(blockIdx.z >> 1), nparts = (int)(gridDim.z >> 1);
    const int RM = G.r_max, P = G.r_max + 2;
    float* bn = reinterpret_cast<float*>(smem);                                   // new basis of side z [d][P]
    float* bo = bn + (size_t)kD * P;                                               // previous basis of side z
    uint8_t* ws = smem + (size_t)2 * kD * P * 4 + (size_t)warp * kRpWarpBytes;
    float* xs = reinterpret_cast<float*>(ws);                                     // [group][kRpXPitch]
    float* cs = xs + kRpMaxGroup * kRpXPitch;                                      // [group][64]
    float* rstage = cs + kRpMaxGroup * 64;                                         // [32]
    uint8_t* chstage = reinterpret_cast<uint8_t*>(rstage + 32);                    // [32]
    uint8_t** gblk = reinterpret_cast<uint8_t**>(chstage + 32);                    // [group]
    int* grow = reinterpret_cast<int*>(gblk + kRpMaxGroup);                        // [group]
    {
        const __nv_bfloat16* src_new = (z ? S.basis_v : S.basis_k) + ((size_t)g * G.Hkv + h) * kD * RM;
        const __nv_bfloat16* src_old = (z ? old_v : old_k) + (size_t)h * kD * RM;
        for (int e = tid; e < kD * RM; e += blockDim.x) {
            const int i = e / RM, j = e % RM;
            bn[(size_t)i * P + j] = __bfloat162float(src_new[e]);
            bo[(size_t)i * P + j] = __bfloat162float(src_old[e]);
        }
    }
    // groups of a tier: ceil(count / V) per layer of the window
    __shared__ uint32_t s_cnt[kMaxTiers], s_gbase[kMaxTiers + 1];
    if (tid == 0) {
        uint32_t acc = 0;
        for (int k = 0; k < kMaxTiers; ++k) {
            const uint32_t c = k < G.ntiers ? S.counts[cnt_index(G, seq, g, h) + k] : 0u;
            const uint32_t vk = k < G.ntiers ? (uint32_t)min(kRpMaxGroup, 64 / G.tiers[k]) : 1u;
            s_cnt[k] = c;
            s_gbase[k] = acc;
            acc += (c + vk - 1u) / vk * (uint32_t)G.LPG;
        }
        s_gbase[kMaxTiers] = acc;
    }
    __syncthreads();
    const uint32_t groups = s_gbase[kMaxTiers];
    for (uint32_t gi = (uint32_t)(part * nwarps + warp); gi < groups; gi += (uint32_t)(nwarps * nparts)) {
        int k = 0;
        while (k + 1 < kMaxTiers && gi >= s_gbase[k + 1]) ++k;
        const uint32_t loc = gi - s_gbase[k];
        const int R = G.tiers[k], Vk = min(kRpMaxGroup, 64 / R);
        const uint32_t lig = loc % (uint32_t)G.LPG, first = loc / (uint32_t)G.LPG * (uint32_t)Vk;
        const int nu = (int)min((uint32_t)Vk, s_cnt[k] - first);
        if (lane < kRpMaxGroup) {                        // the group's blocks and rows
            const uint32_t slot = first + (uint32_t)min(lane, nu - 1);
            const uint32_t unit = S.pages[page_index(G, seq, g, h, k) + slot / kPage];
            gblk[lane] = S.data + (size_t)unit * kUnit + (size_t)lig * G.chunk_bytes[k] + (z ? G.blk_bytes[k] : 0u);
            grow[lane] = (int)(slot % kPage);
        }
        __syncwarp();
        if (Vk == 4) reproject_group<BITS, 4>(G, z, k, nu, gblk, grow, bn, bo, xs, cs, rstage, chstage);
        else if (Vk == 2) reproject_group<BITS, 2>(G, z, k, nu, gblk, grow, bn, bo, xs, cs, rstage, chstage);
        else reproject_group<BITS, 1>(G, z, k, nu, gblk, grow, bn, bo, xs, cs, rstage, chstage);
    }
}

template __global__ void reproject_kernel<8>(const Geom, const State, int, const SeqList, const __nv_bfloat16*,
                                             const __nv_bfloat16*);
template __global__ void reproject_kernel<4>(const Geom, const State, int, const SeqList, const __nv_bfloat16*,
                                             const __nv_bfloat16*);

}  // namespace dwkv
