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
#include "dwkv_encode.cuh"
#include "dwkv_stored.cuh"

namespace dwkv {

// ------------------------------------------------------------------------------------
// Second moment C[w][h][z] += scale * X^T X over the rows of window w's layers (rows = LPG x
// n_rows, layer-major; blockIdx.y = w Hkv + h), on the tensor cores.  A block of 8 warps: warp w
// owns channels [16 w, 16 w + 16) of C's rows and all 128 columns (16 n-tiles); chunks of 64
// rows are staged as bf16 [64][136] (a 272-byte pitch: ldmatrix rows on distinct banks).
// Partial sums go to C with fp32 atomics, so the order of the sum is not fixed.
// ------------------------------------------------------------------------------------
constexpr int kGramRows = 64;
constexpr int kGramPitch = kD + 8;
__global__ void __launch_bounds__(256) gram_kernel(const Geom G, int n_rows, const __nv_bfloat16* __restrict__ k_rows,
                                                   const __nv_bfloat16* __restrict__ v_rows, float* __restrict__ cacc,
                                                   float scale) {
    __shared__ __align__(16) __nv_bfloat16 xs[kGramRows * kGramPitch];
    const int h = blockIdx.y % G.Hkv, gw = blockIdx.y / G.Hkv, z = blockIdx.z;   // gw: window within the call
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, c = lane & 3, mi = lane >> 3, rr = lane & 7;
    const __nv_bfloat16* src = (z ? v_rows : k_rows) + (size_t)gw * G.LPG * n_rows * G.Hkv * kD;
    cacc += (size_t)gw * G.Hkv * 2 * kD * kD;
    const long long total = (long long)G.LPG * n_rows;
    const long long per = (total + gridDim.x - 1) / gridDim.x;
    const long long r0 = (long long)blockIdx.x * per, r1 = r0 + per < total ? r0 + per : total;
    float acc[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    const uint32_t xaddr = smem_addr(xs);
    for (long long b0 = r0; b0 < r1; b0 += kGramRows) {
        __syncthreads();
        // stage 64 rows x 128 channels (16-byte loads; rows past the range as zeros)
        for (int e = tid; e < kGramRows * (kD / 8); e += blockDim.x) {
            const int r = e / (kD / 8), q = e % (kD / 8);
            const long long row = b0 + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (row < r1) {
                const long long layer = row / n_rows, t = row % n_rows;
                v = __ldg(reinterpret_cast<const uint4*>(src + ((layer * n_rows + t) * G.Hkv + h) * kD) + q);
            }
            *reinterpret_cast<uint4*>(xs + r * kGramPitch + 8 * q) = v;
        }
        __syncthreads();
#pragma unroll
        for (int ks = 0; ks < kGramRows / 16; ++ks) {
            // A = X^T rows [16 warp, +16) x rows t [16 ks, +16): transposed 8x8 tiles of X
            uint32_t a[4];
            {
                const int t = 16 * ks + 8 * (mi >> 1) + rr, i0 = 16 * warp + 8 * (mi & 1);
                ldsm_x4_t(xaddr + (uint32_t)(t * kGramPitch + i0) * 2u, a);
            }
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                // B = X rows t x channels [16 np, +16): two n-tiles from one x4.trans
                uint32_t b4[4];
                const int t = 16 * ks + 8 * (mi & 1) + rr, j0 = 16 * np + 8 * (mi >> 1);
                ldsm_x4_t(xaddr + (uint32_t)(t * kGramPitch + j0) * 2u, b4);
                const uint32_t b0[2] = {b4[0], b4[1]}, b1[2] = {b4[2], b4[3]};
                mma_bf16(acc[2 * np], a, b0);
                mma_bf16(acc[2 * np + 1], a, b1);
            }
        }
    }
    float* dst = cacc + ((size_t)h * 2 + z) * kD * kD;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int i0 = 16 * warp + g, j0 = 8 * n + 2 * c;
        atomicAdd(dst + (size_t)i0 * kD + j0, scale * acc[n][0]);
        atomicAdd(dst + (size_t)i0 * kD + j0 + 1, scale * acc[n][1]);
        atomicAdd(dst + (size_t)(i0 + 8) * kD + j0, scale * acc[n][2]);
        atomicAdd(dst + (size_t)(i0 + 8) * kD + j0 + 1, scale * acc[n][3]);
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
            for (int e = tid; e < np * r; e += blockDim.x) {    // rows p, q of T: J^T T
                const int k = e / r, m = e % r, p = pq[k], qq = pq[np + k];
                const double c = cs[k], sn = cs[np + k];
                const double xp = t[p * rp + m], xq = t[qq * rp + m];
                t[p * rp + m] = c * xp - sn * xq;
                t[qq * rp + m] = sn * xp + c * xq;
            }
            __syncthreads();
            for (int e = tid; e < np * r; e += blockDim.x) {    // columns p, q of T and U: (.) J
                const int k = e / r, m = e % r, p = pq[k], qq = pq[np + k];
                const double c = cs[k], sn = cs[np + k];
                const double xp = t[m * rp + p], xq = t[m * rp + qq];
                t[m * rp + p] = c * xp - sn * xq;
                t[m * rp + qq] = sn * xp + c * xq;
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
// (sequence in the list, kv-head), a warp per (slot, layer of the window, K / V) unit, the
// units of a (sequence, kv-head) dealt out over its blocks' warps.  Each
// unit is reconstructed on the previous basis (old_k / old_v: the fixed-order fp32 chain over
// its rank, plus scale x code on its residual channels, rounded to bf16, as a re-tier does)
// and encoded on the new basis at its own tier, in place.  Slots and counts do not change.
// ------------------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256) reproject_kernel(const Geom G, const State S, int g, const SeqList L,
                                                        const __nv_bfloat16* __restrict__ old_k,
                                                        const __nv_bfloat16* __restrict__ old_v) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int seq = L.seq[blockIdx.x], h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int RM = G.r_max, P = G.r_max + 2;
    __nv_bfloat16* bs = reinterpret_cast<__nv_bfloat16*>(smem);                   // new [z][d][P]
    __nv_bfloat16* bo = reinterpret_cast<__nv_bfloat16*>(smem + encode_smem_bytes(G.r_max));  // old [z][d][P]
    const size_t boff = ((size_t)g * G.Hkv + h) * kD * RM;
    for (int e = tid; e < 2 * kD * RM; e += blockDim.x) {
        const int zz = e / (kD * RM), ev = e % (kD * RM), i = ev / RM, j = ev % RM;
        bs[(size_t)zz * kD * P + (size_t)i * P + j] = (zz ? S.basis_v : S.basis_k)[boff + ev];
        bo[(size_t)zz * kD * P + (size_t)i * P + j] = (zz ? old_v : old_k)[(size_t)h * kD * RM + ev];
    }
    __shared__ uint32_t s_cnt[kMaxTiers], s_base[kMaxTiers + 1];
    if (tid == 0) {
        uint32_t acc = 0;
        for (int k = 0; k < kMaxTiers; ++k) {
            s_cnt[k] = k < G.ntiers ? S.counts[cnt_index(G, seq, g, h) + k] : 0u;
            s_base[k] = acc;
            acc += s_cnt[k];
        }
        s_base[kMaxTiers] = acc;
    }
    __syncthreads();
    const uint32_t units = s_base[kMaxTiers] * (uint32_t)G.LPG * 2u;
    const uint32_t nw = (blockDim.x >> 5) * gridDim.z;
    for (uint32_t u = blockIdx.z * (blockDim.x >> 5) + warp; u < units; u += nw) {
        const uint32_t z = u & 1u, lig = (u >> 1) % (uint32_t)G.LPG, slotg = (u >> 1) / (uint32_t)G.LPG;
        int k = 0;
        while (k + 1 < kMaxTiers && slotg >= s_base[k + 1]) ++k;
        const uint32_t slot = slotg - s_base[k];
        const int R = G.tiers[k], st = G.ts[k], row = (int)(slot % kPage);
        const uint32_t unit = S.pages[page_index(G, seq, g, h, k) + slot / kPage];
        uint8_t* blk = S.data + (size_t)unit * kUnit + (size_t)lig * G.chunk_bytes[k] + (z ? G.blk_bytes[k] : 0u);
        // reconstruction on the previous basis (fixed fp32 order), rounded to bf16.  The
        // token's coefficients and residual entries are read in parallel (lane j holds entry j
        // and j + 32) and handed round by shuffles: the chain's order is unchanged.
        const __nv_bfloat16* bz = bo + (size_t)z * kD * P;
        const float cl0 = lane < R ? stored_coeff(blk, G.c8, (int)z, R, row, lane) : 0.f;
        const float cl1 = lane + 32 < R ? stored_coeff(blk, G.c8, (int)z, R, row, lane + 32) : 0.f;
        int ch_l = 0;
        float v_l = 0.f;
        if (st > 0 && lane < st) stored_resid<BITS>(blk, G.c8, R, st, row, lane, ch_l, v_l);
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < R; j += 2) {                     // R is even: the basis read a pair at a time
            const float cj = __shfl_sync(0xffffffffu, j < 32 ? cl0 : cl1, j & 31);
            const float cj1 = __shfl_sync(0xffffffffu, j + 1 < 32 ? cl0 : cl1, (j + 1) & 31);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const uint32_t w = *reinterpret_cast<const uint32_t*>(bz + (size_t)(lane + 32 * m) * P + j);
                a[m] = __fmaf_rn(bf16lo(w), cj, a[m]);
                a[m] = __fmaf_rn(bf16hi(w), cj1, a[m]);
            }
        }
        for (int e = 0; e < st; ++e) {
            const int ch = __shfl_sync(0xffffffffu, ch_l, e);
            const float v = __shfl_sync(0xffffffffu, v_l, e);
            if ((ch & 31) == lane && ch < kD) {
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    if ((ch >> 5) == m) a[m] = __fadd_rn(a[m], v);
            }
        }
        __syncwarp();                                        // every lane has read the old bytes
        UnitIn in;
        in.ok = true;
        in.dbg = nullptr;
        in.dst.blk = S.data + (size_t)unit * kUnit + (size_t)lig * G.chunk_bytes[k];
        in.dst.k = k;
        in.dst.row = row;
        in.dst.R = R;
#pragma unroll
        for (int m = 0; m < 4; ++m) in.xr[m] = __bfloat162float(__float2bfloat16_rn(a[m]));
        encode_body<BITS>(G, S, bs, enc_scratch(G, smem, warp), (int)z, in);
    }
}

template __global__ void reproject_kernel<8>(const Geom, const State, int, const SeqList, const __nv_bfloat16*,
                                             const __nv_bfloat16*);
template __global__ void reproject_kernel<4>(const Geom, const State, int, const SeqList, const __nv_bfloat16*,
                                             const __nv_bfloat16*);

}  // namespace dwkv
