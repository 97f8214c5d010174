// dwkv_common.cuh -- geometry, device state and low-level helpers shared by the libdwkv
// kernels and host code.  Product code; no test-only code includes it.
//
// Storage ("DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization for
// Long-Context KV Cache Compression", §3 Method, Eq. (1); tier-bucketed layout of this
// library):
//   * A page holds 64 tokens of ONE rank tier for one (sequence, group, kv-head).  Its
//     bytes are [layer-in-group][K|V] blocks; decode of one layer reads one contiguous
//     chunk (the K block then the V block) per page.
//   * A block of tier rank R with s residual channels and b-bit codes is
//       coeff  [R/8][64][8] bf16     128*R bytes  (8-coefficient columns, 16 B per token:
//                                                  the tcgen05 / ldmatrix "core matrix"
//                                                  order, conflict-free for per-token reads)
//       idx    [64][s]    uint8      64*s
//       codes  [64][s*b/8]           8*s*b        (int4: even slot in the low nibble; the part
//                                                  padded to 128 bytes when shorter)
//       scales [64]       fp16       128
//     Every part is a multiple of 128 bytes, so pages are 128-byte aligned and every page
//     chunk is a legal bulk-copy (TMA) source.
//   * After the layers' chunks a page holds the position of each of its 64 slots (int32), so
//     a slot can be moved within its tier (re-tiering) with its slot-map entry; decode never
//     reads it.
//   * The page pool is handed out in 128-byte units by a device bump pointer plus one
//     free ring per tier (filled by sequence resets).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace dwkv {

constexpr int kPage = 64;          // tokens per page
constexpr int kD = 128;            // head dimension supported by the kernels
constexpr int kGQ = 4;             // query heads per kv head supported by the kernels
constexpr int kUnit = 128;         // page-pool granularity in bytes
constexpr int kMaxTiers = 8;
constexpr int kMaxSeqs = 256;      // sequences per call
constexpr int kMaxRank = 128;      // largest r_max
constexpr int kMaxSplits = 64;     // decode splits per (sequence, kv-head)
constexpr int kConsumerWarps = 12; // each takes half pages (32 tokens) from a shared queue
constexpr int kSlots = 32;          // page chunks in flight at most (one full / empty barrier pair each)
constexpr int kDecodeThreads = 32 * (kConsumerWarps + 1);  // + 1 producer warp
constexpr int kRdBytes = 128 * 32;                         // dense residual tile: 128 ch x 32 tokens int8

struct Geom {
    int L, LPG, G, Hq, Hkv, d, r_max, ntiers, s, bits, max_batch, max_context, max_pages;
    int tiers[kMaxTiers];
    int ts[kMaxTiers];               // residual channels a token of each tier keeps (<= s; s when not routed)
    int routed;                      // 1: per-tier residual counts (every tier at one basis rank)
    int c8;                          // 1: coefficients as 8-bit codes with an fp16 scale per block of 16
    float tau;                       // softmax scale
    uint32_t blk_bytes[kMaxTiers];   // one (layer, K or V) block of a page
    uint32_t chunk_bytes[kMaxTiers]; // one layer of a page: K block + V block
    uint32_t page_units[kMaxTiers];  // whole page, in kUnit
    uint32_t free_cap;               // entries per free ring (power of two)
    uint32_t stage_bytes;            // largest chunk, rounded to 128
};

struct State {
    uint32_t* err;                   // [0] code, [1] info a, [2] info b
    unsigned long long* bump;        // next free pool unit
    uint32_t* free_head;             // [kMaxTiers] ring read index (monotonic)
    uint32_t* free_tail;             // [kMaxTiers] ring write index (monotonic)
    uint32_t* free_list;             // [kMaxTiers][free_cap] page units
    uint32_t* counts;                // [max_batch][G][Hkv][kMaxTiers] slots placed
    uint32_t* owned;                 // [max_batch][G][Hkv][kMaxTiers] pages held (>= ceil(counts / 64);
                                     //   re-tiering can empty a page the tier keeps for reuse)
    uint32_t* pages;                 // [max_batch][G][Hkv][kMaxTiers][max_pages] unit offsets
    uint32_t* slot_map;              // [max_batch][G][Hkv][max_context]: ((tier+1)<<24)|slot
    uint32_t* tickets;               // [max_batch][Hkv] split-combine tickets
    const __nv_bfloat16* basis_k;    // [G][Hkv][d][r_max]
    const __nv_bfloat16* basis_kt;   // the same, per (group, kv-head) as 8 x 8 tiles [d/8][r_max/8][8][8]
    const __nv_bfloat16* basis_v;
    uint8_t* data;                   // page pool
    unsigned long long data_units;
};

// Per-call sequence table of append / import (passed by value as a kernel parameter, so
// captured graphs replay it exactly).
struct AppendCall {
    int n, layer, g, lig, total;
    int seq[kMaxSeqs];
    int pos0[kMaxSeqs];      // first position appended at this layer
    int tok0[kMaxSeqs + 1];  // prefix of n_new: first input row of each sequence
    int a0[kMaxSeqs];        // first position that needs a slot (group's first placement)
    int na[kMaxSeqs];        // positions that need a slot
    const float* gate;       // nullable: residual gate g [total][Hkv][2], folded into the stored scale
};

// One round of a re-tier call: for each listed sequence, the tokens [begin, end) of the call's
// positions / new-tier arrays.
struct RetierCall {
    int n, g;
    int seq[kMaxSeqs];
    int begin[kMaxSeqs];
    int end[kMaxSeqs];
};

// Sequences of a call that touches every stored token of theirs (basis re-projection).
struct SeqList {
    int n;
    int32_t seq[kMaxSeqs];
};

struct DecodeCall {
    int n, layer, g, lig, total_splits, ring_bytes, rec_floats;
    int tok_weight;          // split balance: cost of one token in byte-equivalents
    // One new token per sequence appended in the same launch (0 = plain decode).  The first CTA
    // of each (sequence, kv-head) places and encodes it and attends to it directly; every CTA
    // attends to the pages without it.  `owner_cost` (in the split balance's cost units: bytes
    // plus tok_weight a token) is what that work costs the CTA; it takes that much less.
    int fused;
    uint32_t owner_cost;
    const __nv_bfloat16* k_new;      // [n][Hkv][d] bf16 (fused)
    const __nv_bfloat16* v_new;
    const uint8_t* tier_idx;         // [n][Hkv] tier of the new token (read where it is placed)
    int pos[kMaxSeqs];               // the new token's position (fused)
    uint8_t place[kMaxSeqs];         // 1: this layer places it (its group's first to append it)
    // 1: the tier counts, page tables and page bytes this launch reads are final before it waits
    // on the previous kernel (programmatic dependent launch), so its producer may read them and
    // stream pages at once; 0: it waits first.  The host sets 0 when the previous launch on the
    // handle was a fused step of the same group that still writes them (a placing launch adds
    // its token's count at its end; every fused launch writes its token's bytes of its layer).
    int early;
    int seq[kMaxSeqs];
    int split_begin[kMaxSeqs + 1];
    const __nv_bfloat16* q;  // [n][Hq][d]
    float* out;              // [n][Hq][d]
    float* out_full;         // probe: optional [n][Hq][d]
    float* err;              // probe: [n][Hkv]
    float* ws;               // partial records
};

// ------------------------------------------------------------------------------ layout
// One (layer, K or V) block of a page of tier rank R, 64 token slots:
//   coefficients: bf16 [R/8][64][8] (128 R bytes), or with c8 the 8-bit form (72 R bytes, below)
//   idx u8 [64][s], codes [64][s] (int8, or int4 pairs) padded to 128 bytes, scales fp16 [64].
// The code part rounded up to 128 bytes (only 2 int4 codes a token, 64 bytes, needs it).
__host__ __device__ inline uint32_t code_part_bytes(int s, int bits) { return (8u * s * bits + 127u) & ~127u; }
__host__ __device__ inline uint32_t coeff_part_bytes(int R, int c8) { return c8 ? 72u * R : 128u * R; }
__host__ __device__ inline uint32_t blk_bytes_of(int R, int s, int bits, int c8 = 0) {
    return coeff_part_bytes(R, c8) + 64u * s + code_part_bytes(s, bits) + 128u;
}
__host__ __device__ inline uint32_t off_idx_of(int R, int c8 = 0) { return coeff_part_bytes(R, c8); }
__host__ __device__ inline uint32_t off_codes_of(int R, int s, int c8 = 0) { return coeff_part_bytes(R, c8) + 64u * s; }
__host__ __device__ inline uint32_t off_scales_of(int R, int s, int bits, int c8 = 0) {
    return coeff_part_bytes(R, c8) + 64u * s + code_part_bytes(s, bits);
}
// The 8-bit coefficient form (R a multiple of 16; blocks b of 16 coefficients): codes int8
// [R/16][1024 bytes], then fp16 scales [R/16][128 bytes].
//  keys:   token t's 16 codes of block b are the 16 bytes at b 1024 + 16 t, coefficient 16 b + e
//          at byte kc8_pos(e): bytes 4c..4c+3 hold e = 2c, 2c+1, 2c+8, 2c+9, one lane's two
//          A-operand pairs of an m16n8k16 MMA row.  The scales of tokens t and t + 8 of a
//          16-token tile sit side by side (one 32-bit word for an MMA fragment's two rows).
//  values: coefficient 16 b + e of token t at b 1024 + 64 e + 16 ((t/16) ^ (e/2 mod 4)) + t mod 16:
//          rows of 64 tokens (the A operand of a tokens-deep integer MMA), the 16-byte chunks
//          of a row rotated so that the 8 rows an ldmatrix reads fall in distinct banks.  A
//          token's scales sit together: (R/16) fp16 at (R/16) 1024 + t (R/16) 2.
__host__ __device__ inline uint32_t kc8_pos(int e) {
    return e < 8 ? 4u * (uint32_t)(e >> 1) + (uint32_t)(e & 1) : 4u * (uint32_t)((e - 8) >> 1) + 2u + (uint32_t)(e & 1);
}
__host__ __device__ inline uint32_t kc8_code_off(int j, int t) { return (uint32_t)(j >> 4) * 1024u + 16u * (uint32_t)t + kc8_pos(j & 15); }
__host__ __device__ inline uint32_t kc8_scale_off(int R, int b, int t) {
    return (uint32_t)(R >> 4) * 1024u + (uint32_t)b * 128u + 2u * (16u * (uint32_t)(t >> 4) + 2u * (uint32_t)(t & 7) + (uint32_t)((t >> 3) & 1));
}
__host__ __device__ inline uint32_t vc8_code_off(int j, int t) {
    const int e = j & 15;
    return (uint32_t)(j >> 4) * 1024u + 64u * (uint32_t)e + 16u * (uint32_t)(((t >> 4) ^ (e >> 1)) & 3) + (uint32_t)(t & 15);
}
__host__ __device__ inline uint32_t vc8_scale_off(int R, int b, int t) {
    return (uint32_t)(R >> 4) * 1024u + (uint32_t)t * (uint32_t)(R >> 4) * 2u + 2u * (uint32_t)b;
}
// Element offset of B_K[i][j] in a tiled basis (basis_kt) of rank r_max: 8 x 8 tiles, the tile
// rows 16 contiguous bytes, so that an ldmatrix row set (8 rows of one tile) is one 128-byte line.
__host__ __device__ inline uint32_t tiled_basis_off(int i, int j, int r_max) {
    return ((uint32_t)(i >> 3) * (uint32_t)(r_max >> 3) + (uint32_t)(j >> 3)) * 64u + (uint32_t)(i & 7) * 8u + (uint32_t)(j & 7);
}

// Byte offset of a page's slot-position block (after the layers' chunks).
__host__ __device__ inline uint32_t pos_block_of(const Geom& G, int k) { return (uint32_t)G.LPG * G.chunk_bytes[k]; }
constexpr uint32_t kPosBlockBytes = kPage * 4;

__host__ __device__ inline size_t cnt_index(const Geom& G, int seq, int g, int h) {
    return (((size_t)seq * G.G + g) * G.Hkv + h) * kMaxTiers;
}
__host__ __device__ inline size_t page_index(const Geom& G, int seq, int g, int h, int k) {
    return ((((size_t)seq * G.G + g) * G.Hkv + h) * kMaxTiers + k) * (size_t)G.max_pages;
}
__host__ __device__ inline size_t slot_index(const Geom& G, int seq, int g, int h, int pos) {
    return (((size_t)seq * G.G + g) * G.Hkv + h) * (size_t)G.max_context + pos;
}

// Decode shared-memory layout (identical on host and device).
//   ring    page chunks, packed back to back (a chunk that does not fit before the end
//           starts again at 0); ring_bytes is chosen by the host
//   rd      per consumer warp, one 4 KB residual tile (also holds B_K during the prologue)
//   small   per consumer warp: scores S[32][4] f32, P[32][8] bf16, W [4 heads][48] u16, P2[32][8];
//           with 8-bit coefficients two more weight tiles CW [4 or 8][48] u16 (ping-pong over blocks)
//   qt      q~ = B_K^T q, fp32 [r_max][4];  q  fp32 [d][4];  qh bf16 [d][4];  qb: q~ as MMA
//           B fragments [ks][2][lane];  zero line
//   bars    full[kSlots] empty[kSlots] basis table
//   misc    tier table, page range; warp states; page-id batch; slot offsets
struct DecodeSmem {
    uint32_t ring, rd, small, small_stride, S, P, W, P2, CW, qt, q, qh, qb, zero, bars, misc, tok, total;
};
// The CTA merge reuses the idle ring: the merged sums (at most 6 KB) at 0, B_V at kMergeBvOff.
constexpr uint32_t kMergeBvOff = 8192;
constexpr uint32_t kMiscState = 256;                               // m_state [warps][16]
constexpr uint32_t kMiscFactors = kMiscState + kConsumerWarps * 64; // mf [2][warps][4]
constexpr uint32_t kMiscPages = kMiscFactors + kConsumerWarps * 32; // t_src [32], t_len [32]
constexpr uint32_t kMiscSlots = kMiscPages + 256;                  // slot offsets [kSlots]
constexpr uint32_t kMiscBytes = kMiscSlots + kSlots * 4;
__host__ __device__ inline DecodeSmem decode_smem_layout(const Geom& G, uint32_t ring_bytes, bool probe) {
    DecodeSmem L;
    uint32_t o = 0;
    L.ring = o;    o += ring_bytes;
    L.rd = o;      o += kConsumerWarps * kRdBytes;
    uint32_t w = 0;
    L.S = w;       w += 32 * 16;
    L.P = w;       w += 32 * 16;
    L.W = w;       w += 32 * 16;
    L.P2 = w;      w += probe ? 32 * 16 : 0;
    L.CW = w;      w += G.c8 ? 2 * (probe ? 768 : 384) : 0;
    L.small_stride = w;
    L.small = o;   o += kConsumerWarps * w;
    L.qt = o;      o += (uint32_t)(G.r_max < 16 ? 16 : G.r_max) * 16;
    L.q = o;       o += (uint32_t)G.d * 16;
    L.qh = o;      o += (uint32_t)G.d * 8;
    L.qb = o;      o += 32 * 2 * (kMaxRank / 16) * 4;
    L.zero = o;    o += 128;
    L.bars = o;    o += (2 * kSlots + 2) * 8;
    L.misc = o;    o += (kMiscBytes + 127) & ~127u;
    L.tok = o;     o += 64;                 // the new token's destination (fused append)
    L.total = (o + 127) & ~127u;
    return L;
}

// Floats in one decode partial record: m[4] l[4] (m2[4] l2[4]) o[4][d] (o2[4][d]), where
// o = B_V acc_c + acc_r of the CTA's tokens (relative to m).  The probe layout sizes both.
__host__ __device__ inline int rec_floats_of(const Geom& G, bool probe) {
    return (probe ? 16 : 8) + (probe ? 2 : 1) * kGQ * G.d;
}

// ------------------------------------------------------------------------------ device
#ifdef __CUDACC__
__device__ __forceinline__ void set_dev_error(const State& S, uint32_t code, uint32_t a, uint32_t b) {
    if (atomicCAS(S.err, 0u, code) == 0u) {
        S.err[1] = a;
        S.err[2] = b;
    }
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One poll of the phase of parity `parity`.  The thread may sleep in it for up to
// kWaitSuspendNs until the phase completes: a waiting warp then stops issuing polls, which
// would otherwise compete for the shared-memory pipe with the warps that do the work.
constexpr uint32_t kWaitSuspendNs = 2000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kWaitSuspendNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase of parity `parity` to complete: gives up after limit_ns of wall
// time (checked every 256 polls); the caller then records DWKV_DEV_TIMEOUT and stops
// instead of spinning forever.  The kernels use a 2 s limit.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0u && global_ns() - t0 > limit_ns) return false;
    }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// One bulk (non-tensor) global -> shared copy completing on an mbarrier.  Both addresses
// 16-byte aligned, bytes a multiple of 16.  No cluster multicast.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// An L2 policy under which the loaded lines are the first to be evicted: for data read once
// per launch (the pages), so that the small tables read by every launch stay in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// bulk_g2s with an L2 cache policy.
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Programmatic dependent launch.  A kernel launched with programmatic stream serialisation
// may start while the previous kernel of its stream still runs; grid_dep_wait() returns once
// that kernel has completed and its memory operations are visible (at once when there is no
// such kernel).  grid_dep_launch() lets the next such kernel start once every CTA of this one
// has issued it or exited.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ warp-level MMA pieces (sm_80+ forms)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t (&r)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr));
}
// D (16x8 f32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// D (16x8 f32) += A (16x16 f16, row) * B (16x8 f16, col)
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// Two int8 values (bytes lo, lo + 1 of w when hi == 0, bytes 2, 3 when hi == 1) as an f16 pair,
// exactly: the biased byte (x + 128) in the mantissa of 1024, then 1024 + 128 subtracted.
__device__ __forceinline__ uint32_t s8x2_to_f16x2(uint32_t w, int hi) {
    const uint32_t b = __byte_perm(w ^ 0x80808080u, 0x64646464u, hi ? 0x4342u : 0x4140u);
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(b), "r"(0x64806480u));
    return r;
}

// D (16x8 s32) = A (16x32 s8, row) * B (32x8 u8, col) + C
__device__ __forceinline__ void mma_s8u8(int (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr));
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
#endif

}  // namespace dwkv
