// dwkv_api.cu -- host side of libdwkv: argument checks, arena layout, launch set-up.
// Every public entry point is declared (and documented) in include/dwkv.h.
#include <cuda.h>  // CUtensorMap and its encode function's types (the function itself comes from the driver at run time)

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "dwkv.h"
#include "dwkv_common.cuh"
#include "dwkv_encode.cuh"

namespace dwkv {
__global__ void place_kernel(const Geom, const State, const AppendCall, const uint8_t*);
template <int BITS>
__global__ void encode_kernel(const Geom, const State, const AppendCall, const __nv_bfloat16*, const __nv_bfloat16*,
                              float*);
template <int BITS>
__global__ void quantize_test_kernel(int, int, const float*, uint8_t*, int8_t*, uint16_t*, uint8_t*, uint32_t);
template <int BITS>
__global__ void append_small_kernel(const Geom, const State, const AppendCall, const uint8_t*, int,
                                    const __nv_bfloat16*, const __nv_bfloat16*, float*);
template <int BITS>
__global__ void import_kernel(const Geom, const State, const AppendCall, const uint8_t*, const uint8_t*,
                              const int8_t*, const __half*);
template <int BITS>
__global__ void export_kernel(const Geom, const State, int, int, int, int, uint8_t*, uint8_t*, uint8_t*,
                              int8_t*, __half*);
__global__ void reset_kernel(const Geom, const State, int);
template <int BITS>
__global__ void retier_kernel(const Geom, const State, const RetierCall, const int32_t*, const uint8_t*);
__global__ void retier_release_kernel(const Geom, const State, const RetierCall);
__global__ void wait_timeout_kernel(const State, uint64_t);
__global__ void tile_basis_kernel(const Geom, const State);
__global__ void gram_kernel(const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap, const Geom,
                            const State, int, int, float*, float);
__global__ void moment_scale_kernel(float*, size_t, float);
__global__ void basis_kernel(const Geom, const State, int, const float*, const float*, int, float*);
template <int BITS>
__global__ void reproject_kernel(const Geom, const State, int, const SeqList, const __nv_bfloat16*,
                                 const __nv_bfloat16*);
size_t basis_smem_bytes(int r);
size_t reproject_smem_bytes(int r_max, int warps);
size_t gram_smem_bytes();
template <int BITS, bool PROBE, int RMAX, int S, bool C8>
__global__ void decode_kernel(const Geom, const State, const DecodeCall);
}  // namespace dwkv

using namespace dwkv;

namespace {
thread_local std::string g_err;
}  // namespace

namespace dwkv {
void set_last_error(const char* msg) { g_err = msg; }
}  // namespace dwkv

namespace {

dwkv_status fail(dwkv_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
    return st;
}

dwkv_status cuda_fail(cudaError_t e, const char* what) {
    return fail(DWKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define DWKV_CUDA(call, what)                            \
    do {                                                 \
        cudaError_t e_ = (call);                         \
        if (e_ != cudaSuccess) return cuda_fail(e_, what); \
    } while (0)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

uint32_t next_pow2(uint64_t v) {
    uint64_t p = 1;
    while (p < v) p <<= 1;
    return (uint32_t)std::min<uint64_t>(p, 1ull << 31);
}

bool is_pow2_rank(int r) { return r == 8 || r == 16 || r == 32 || r == 64 || r == 128; }

dwkv_status check_cfg(const dwkv_config* c) {
    if (!c) return fail(DWKV_ERR_INVALID_ARG, "config is NULL");
    if (c->num_layers <= 0 || c->layers_per_group <= 0 || c->num_layers % c->layers_per_group)
        return fail(DWKV_ERR_INVALID_ARG, "num_layers (%d) must be a positive multiple of layers_per_group (%d)",
                    c->num_layers, c->layers_per_group);
    if (c->num_kv_heads <= 0 || c->num_q_heads <= 0 || c->num_q_heads % c->num_kv_heads)
        return fail(DWKV_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                    c->num_q_heads, c->num_kv_heads);
    if (c->head_dim <= 0 || c->head_dim > 256)
        return fail(DWKV_ERR_INVALID_ARG, "head_dim %d out of range", c->head_dim);
    if (c->r_max <= 0 || c->r_max > c->head_dim || c->r_max % 8)
        return fail(DWKV_ERR_INVALID_ARG, "r_max %d must be a multiple of 8 in [8, head_dim]", c->r_max);
    if (c->num_tiers < 1 || c->num_tiers > DWKV_MAX_TIERS)
        return fail(DWKV_ERR_INVALID_ARG, "num_tiers %d out of [1, %d]", c->num_tiers, DWKV_MAX_TIERS);
    if (c->resid_routed != 0 && c->resid_routed != 1)
        return fail(DWKV_ERR_INVALID_ARG, "resid_routed must be 0 or 1 (got %d)", c->resid_routed);
    if (c->coeff_bits != 0 && c->coeff_bits != 16 && c->coeff_bits != 8)
        return fail(DWKV_ERR_INVALID_ARG, "coeff_bits must be 16 (or 0) or 8 (got %d)", c->coeff_bits);
    if (c->coeff_bits == 8 && c->r_max % 16)
        return fail(DWKV_ERR_INVALID_ARG, "with coeff_bits 8, r_max (%d) must be a multiple of 16", c->r_max);
    for (int k = 0; k < c->num_tiers; ++k) {
        if (c->tiers[k] <= 0 || c->tiers[k] % 8 || c->tiers[k] > c->r_max)
            return fail(DWKV_ERR_INVALID_ARG, "tier %d rank %d must be a multiple of 8 in [8, r_max]", k, c->tiers[k]);
        if (c->coeff_bits == 8 && c->tiers[k] % 16)
            return fail(DWKV_ERR_INVALID_ARG, "with coeff_bits 8, tier %d rank %d must be a multiple of 16 (whole blocks)",
                        k, c->tiers[k]);
        if (!c->resid_routed && k && c->tiers[k] <= c->tiers[k - 1])
            return fail(DWKV_ERR_INVALID_ARG, "tiers must be strictly ascending");
        if (c->resid_routed) {
            const int t = c->tier_resid[k];
            if (c->tiers[k] != c->tiers[0])
                return fail(DWKV_ERR_INVALID_ARG, "with resid_routed every tier has the same rank");
            if (t != 0 && t != 2 && t != 4 && t != 8)
                return fail(DWKV_ERR_INVALID_ARG, "tier_resid[%d] = %d must be 0, 2, 4 or 8", k, t);
            if (k && t <= c->tier_resid[k - 1])
                return fail(DWKV_ERR_INVALID_ARG, "tier_resid must be strictly ascending");
        }
    }
    if (c->resid_bits != 8 && c->resid_bits != 4)
        return fail(DWKV_ERR_INVALID_ARG, "resid_bits must be 8 or 4 (got %d)", c->resid_bits);
    if (c->resid_channels < 0 || c->resid_channels > c->head_dim || c->resid_channels % 8)
        return fail(DWKV_ERR_INVALID_ARG, "resid_channels %d must be a multiple of 8 in [0, head_dim]",
                    c->resid_channels);
    if (c->resid_routed && c->resid_channels != 8)
        return fail(DWKV_ERR_INVALID_ARG, "with resid_routed, resid_channels must be 8 (the arrays' stride)");
    if (c->max_batch <= 0 || c->max_context <= 0)
        return fail(DWKV_ERR_INVALID_ARG, "max_batch and max_context must be positive");
    if (c->max_context >= (1 << 24))
        return fail(DWKV_ERR_INVALID_ARG, "max_context must be below 2^24");
    if (!(c->softmax_scale <= 0.f) && !std::isfinite(c->softmax_scale))
        return fail(DWKV_ERR_INVALID_ARG, "softmax_scale must be finite");
    return DWKV_OK;
}

dwkv_status check_supported(const dwkv_config* c) {
    if (c->head_dim != kD) return fail(DWKV_ERR_UNSUPPORTED, "this build has kernels for head_dim 128 only");
    if (c->num_q_heads != kGQ * c->num_kv_heads)
        return fail(DWKV_ERR_UNSUPPORTED, "this build has kernels for 4 query heads per kv head only");
    if (!is_pow2_rank(c->r_max)) return fail(DWKV_ERR_UNSUPPORTED, "r_max must be one of 8, 16, 32, 64, 128");
    if (c->resid_channels != 0 && c->resid_channels != 8 && c->resid_channels != 16 && c->resid_channels != 32)
        return fail(DWKV_ERR_UNSUPPORTED, "this build has kernels for resid_channels 0, 8, 16 or 32");
    for (int k = 0; k < c->num_tiers; ++k)
        if (!is_pow2_rank(c->tiers[k]))
            return fail(DWKV_ERR_UNSUPPORTED, "tier ranks must be among 8, 16, 32, 64, 128");
    return DWKV_OK;
}

struct MetaLayout {
    size_t err, bump, free_head, free_tail, free_list, counts, owned, pages, slot_map, tickets, basis_k, basis_v, basis_kt,
        moment, basis_old, data;
    uint32_t free_cap;
};

Geom make_geom(const dwkv_config* c) {
    Geom G{};
    G.L = c->num_layers;
    G.LPG = c->layers_per_group;
    G.G = c->num_layers / c->layers_per_group;
    G.Hq = c->num_q_heads;
    G.Hkv = c->num_kv_heads;
    G.d = c->head_dim;
    G.r_max = c->r_max;
    G.ntiers = c->num_tiers;
    G.s = c->resid_channels;
    G.routed = c->resid_routed ? 1 : 0;
    G.c8 = c->coeff_bits == 8 ? 1 : 0;
    for (int k = 0; k < kMaxTiers; ++k) G.ts[k] = (k < c->num_tiers && G.routed) ? c->tier_resid[k] : G.s;
    G.bits = c->resid_bits;
    G.max_batch = c->max_batch;
    G.max_context = c->max_context;
    G.max_pages = (c->max_context + kPage - 1) / kPage;
    G.tau = c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / std::sqrt((float)c->head_dim);
    uint32_t stage = 0;
    for (int k = 0; k < kMaxTiers; ++k) {
        if (k < c->num_tiers) {
            G.tiers[k] = c->tiers[k];
            G.blk_bytes[k] = blk_bytes_of(c->tiers[k], G.ts[k], G.bits, G.c8);
            G.chunk_bytes[k] = 2 * G.blk_bytes[k];
            G.page_units[k] = (G.LPG * G.chunk_bytes[k] + kPosBlockBytes) / kUnit;
            stage = std::max(stage, G.chunk_bytes[k]);
        } else {
            G.tiers[k] = 0;
            G.blk_bytes[k] = G.chunk_bytes[k] = G.page_units[k] = 0;
        }
    }
    G.stage_bytes = (uint32_t)align_up(stage, 128);
    G.free_cap = next_pow2((uint64_t)c->max_batch * G.G * G.Hkv * G.max_pages);
    return G;
}

MetaLayout meta_layout(const Geom& G) {
    MetaLayout M{};
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
    M.free_cap = G.free_cap;
    M.err = take(64);
    M.bump = take(8);
    M.free_head = take(4 * kMaxTiers);
    M.free_tail = take(4 * kMaxTiers);
    M.free_list = take((size_t)4 * kMaxTiers * G.free_cap);
    M.counts = take((size_t)4 * G.max_batch * G.G * G.Hkv * kMaxTiers);
    M.owned = take((size_t)4 * G.max_batch * G.G * G.Hkv * kMaxTiers);
    M.pages = take((size_t)4 * G.max_batch * G.G * G.Hkv * kMaxTiers * G.max_pages);
    M.slot_map = take((size_t)4 * G.max_batch * G.G * G.Hkv * G.max_context);
    M.tickets = take((size_t)4 * G.max_batch * G.Hkv);
    M.basis_k = take((size_t)2 * G.G * G.Hkv * G.d * G.r_max);
    M.basis_v = take((size_t)2 * G.G * G.Hkv * G.d * G.r_max);
    M.basis_kt = take((size_t)2 * G.G * G.Hkv * G.d * G.r_max);
    M.moment = take((size_t)4 * G.G * G.Hkv * 2 * G.d * G.d);          // fp32 [G][Hkv][K|V][d][d]
    M.basis_old = take((size_t)2 * 2 * G.G * G.Hkv * G.d * G.r_max);   // bf16 [K|V][G][Hkv][d][r_max]
    M.data = o;
    return M;
}

// Split-K records a decode (probe = false) or probe launch over n_seqs sequences can write:
// at most kMaxSplits per (sequence, kv-head), each rec_floats_of(G, probe) floats.
size_t ws_need(const Geom& G, int n_seqs, bool probe) {
    return (size_t)std::max(n_seqs, 1) * G.Hkv * kMaxSplits * rec_floats_of(G, probe) * sizeof(float);
}

size_t worst_data_bytes(const Geom& G) {
    uint32_t big = 0;
    for (int k = 0; k < G.ntiers; ++k) big = std::max(big, G.page_units[k]);
    const uint64_t pages_per_head = (uint64_t)G.max_pages + G.ntiers - 1;
    return (size_t)G.max_batch * G.G * G.Hkv * pages_per_head * big * kUnit;
}

}  // namespace

struct dwkv_ctx {
    dwkv_config cfg;
    Geom geom;
    State st;
    MetaLayout meta;
    uint8_t* arena;
    size_t arena_bytes;
    int device, num_sms;
    int enc_blocks_per_sm = 1;      // bulk encode kernel occupancy
    size_t smem_optin, smem_per_sm;
    std::vector<int32_t> len;       // [max_batch][L]
    std::vector<int32_t> placed;    // [max_batch][G]
    int dec_ctas_per_sm = 1, dec_waves = 1, dec_stages_req = 0;
    int dec_tok_weight = 1024;      // split balance: byte-equivalent cost of one token
    uint32_t dec_owner_cost = 2500000;  // fused append: the encoding CTA's extra work, in split cost units
    int dec_overlap = 1;            // launch decodes with programmatic stream serialisation
    // The last launch on the handle when it was a fused decode step (else layer -1): a decode
    // launched right after it may start while it runs, and must not read early what it writes.
    int last_fused_layer = -1, last_fused_placed = 0;
};

namespace {

dwkv_status check_handle(dwkv_handle h) {
    if (!h) return fail(DWKV_ERR_INVALID_ARG, "handle is NULL");
    return DWKV_OK;
}

// A launch without programmatic serialisation starts after everything before it on the
// stream has completed, so the next decode may read the cache early again.
void note_plain_launch(dwkv_handle h) { h->last_fused_layer = -1; }

dwkv_status check_layer(dwkv_handle h, int32_t layer) {
    if (layer < 0 || layer >= h->geom.L)
        return fail(DWKV_ERR_INVALID_ARG, "layer %d out of [0, %d)", layer, h->geom.L);
    return DWKV_OK;
}

dwkv_status check_seq_list(dwkv_handle h, int32_t n_seqs, const int32_t* seq_ids) {
    if (n_seqs < 0 || n_seqs > kMaxSeqs)
        return fail(DWKV_ERR_INVALID_ARG, "n_seqs %d out of [0, %d]", n_seqs, kMaxSeqs);
    if (n_seqs && !seq_ids) return fail(DWKV_ERR_INVALID_ARG, "seq_ids is NULL");
    std::vector<char> seen(h->geom.max_batch, 0);
    for (int i = 0; i < n_seqs; ++i) {
        const int s = seq_ids[i];
        if (s < 0 || s >= h->geom.max_batch)
            return fail(DWKV_ERR_INVALID_ARG, "sequence id %d out of [0, %d)", s, h->geom.max_batch);
        if (seen[s]) return fail(DWKV_ERR_INVALID_ARG, "sequence id %d listed twice", s);
        seen[s] = 1;
    }
    return DWKV_OK;
}

State make_state(uint8_t* arena, const MetaLayout& M, size_t arena_bytes) {
    State S{};
    S.err = reinterpret_cast<uint32_t*>(arena + M.err);
    S.bump = reinterpret_cast<unsigned long long*>(arena + M.bump);
    S.free_head = reinterpret_cast<uint32_t*>(arena + M.free_head);
    S.free_tail = reinterpret_cast<uint32_t*>(arena + M.free_tail);
    S.free_list = reinterpret_cast<uint32_t*>(arena + M.free_list);
    S.counts = reinterpret_cast<uint32_t*>(arena + M.counts);
    S.owned = reinterpret_cast<uint32_t*>(arena + M.owned);
    S.pages = reinterpret_cast<uint32_t*>(arena + M.pages);
    S.slot_map = reinterpret_cast<uint32_t*>(arena + M.slot_map);
    S.tickets = reinterpret_cast<uint32_t*>(arena + M.tickets);
    S.basis_k = reinterpret_cast<const __nv_bfloat16*>(arena + M.basis_k);
    S.basis_v = reinterpret_cast<const __nv_bfloat16*>(arena + M.basis_v);
    S.basis_kt = reinterpret_cast<const __nv_bfloat16*>(arena + M.basis_kt);
    S.data = arena + M.data;
    S.data_units = (arena_bytes - M.data) / kUnit;
    return S;
}

size_t encode_smem(const Geom& G) { return encode_smem_bytes(G.r_max); }
size_t encode_tile_smem(const Geom& G) { return enc_tile_layout(G.r_max).total; }

// Bytes of the decode page ring: what the shared-memory budget leaves after the fixed
// regions, capped at dec_stages_req x the largest chunk when that is set (but never below
// the CTA merge's scratch, which reuses it).  0 when fewer than two of the largest chunks fit.
// *smem_out receives the kernel's dynamic shared memory.
uint32_t decode_ring_for(dwkv_handle h, bool probe, size_t* smem_out) {
    const Geom& G = h->geom;
    const size_t budget = h->smem_optin;
    const DecodeSmem L0 = decode_smem_layout(G, 0, probe);
    const size_t scratch = (size_t)kMergeBvOff + (size_t)kD * G.r_max * 2;   // merged sums, then B_V
    const size_t need = std::max(2 * (size_t)G.stage_bytes, scratch);
    if ((size_t)L0.total + need > budget) return 0;
    size_t ring = (budget - L0.total) / 128 * 128;
    if (h->dec_stages_req > 0) ring = std::min(ring, std::max((size_t)h->dec_stages_req * G.stage_bytes, scratch));
    if (ring < need) return 0;
    *smem_out = decode_smem_layout(G, (uint32_t)ring, probe).total;
    return (uint32_t)ring;
}

dwkv_status prepare_call(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                         const int32_t* n_new, AppendCall& C, bool need_tiers, const void* tier_idx) {
    const Geom& G = h->geom;
    dwkv_status st;
    if ((st = check_layer(h, layer)) != DWKV_OK) return st;
    if ((st = check_seq_list(h, n_seqs, seq_ids)) != DWKV_OK) return st;
    if (n_seqs && !n_new) return fail(DWKV_ERR_INVALID_ARG, "n_new is NULL");
    memset(&C, 0, sizeof(C));
    C.n = n_seqs;
    C.layer = layer;
    C.g = layer / G.LPG;
    C.lig = layer % G.LPG;
    long long total = 0;
    bool any_place = false;
    for (int i = 0; i < n_seqs; ++i) {
        const int s = seq_ids[i];
        if (n_new[i] < 0) return fail(DWKV_ERR_INVALID_ARG, "n_new[%d] = %d is negative", i, n_new[i]);
        const int pos0 = h->len[(size_t)s * G.L + layer];
        const long long end = (long long)pos0 + n_new[i];
        if (end > G.max_context)
            return fail(DWKV_ERR_CAPACITY, "sequence %d would hold %lld tokens at layer %d (max_context %d)", s, end,
                        layer, G.max_context);
        const int placed = h->placed[(size_t)s * G.G + C.g];
        C.seq[i] = s;
        C.pos0[i] = pos0;
        C.tok0[i] = (int)total;
        C.a0[i] = std::max(pos0, placed);
        C.na[i] = (int)std::max<long long>(0, end - C.a0[i]);
        any_place |= C.na[i] > 0;
        total += n_new[i];
        if (total > (1ll << 30)) return fail(DWKV_ERR_INVALID_ARG, "too many tokens in one call");
    }
    C.tok0[n_seqs] = (int)total;
    C.total = (int)total;
    if (any_place && need_tiers && !tier_idx)
        return fail(DWKV_ERR_INVALID_ARG, "tier_idx is NULL but layer %d is the first of its group to append "
                                          "some of these positions", layer);
    return DWKV_OK;
}

void commit_call(dwkv_handle h, const AppendCall& C, const int32_t* n_new) {
    const Geom& G = h->geom;
    for (int i = 0; i < C.n; ++i) {
        const int s = C.seq[i];
        const int end = C.pos0[i] + n_new[i];
        h->len[(size_t)s * G.L + C.layer] = end;
        int& pl = h->placed[(size_t)s * G.G + C.g];
        pl = std::max(pl, end);
    }
}

int grid_rows(dwkv_handle h, long long rows) {
    const long long per = 8;  // warps per block
    long long want = (rows + per - 1) / per;
    const long long cap = std::max(1, 4 * h->num_sms / std::max(1, h->geom.Hkv));
    return (int)std::max(1ll, std::min(want, cap));
}

}  // namespace

// =============================================================================== C ABI
extern "C" {

const char* dwkv_version(void) { return "dwkv 0.1 (sm_100a)"; }

const char* dwkv_last_error(void) { return g_err.c_str(); }

dwkv_status dwkv_config_check(const dwkv_config* cfg) {
    dwkv_status st = check_cfg(cfg);
    if (st != DWKV_OK) return st;
    return check_supported(cfg);
}

size_t dwkv_token_bytes(const dwkv_config* cfg, int32_t tier) {
    if (check_cfg(cfg) != DWKV_OK || tier < 0 || tier >= cfg->num_tiers) return 0;
    const int r = cfg->tiers[tier], s = cfg->resid_routed ? cfg->tier_resid[tier] : cfg->resid_channels;
    const int b = cfg->resid_bits;
    const int cb = cfg->coeff_bits == 8 ? r + r / 8 : 2 * r;     // int8 codes + an fp16 scale per 16
    return (size_t)2 * (cb + s + s * b / 8 + 2);
}

size_t dwkv_page_bytes(const dwkv_config* cfg, int32_t tier) {
    if (check_cfg(cfg) != DWKV_OK || tier < 0 || tier >= cfg->num_tiers) return 0;
    const Geom G = make_geom(cfg);
    return (size_t)G.page_units[tier] * kUnit;
}

size_t dwkv_metadata_bytes(const dwkv_config* cfg) {
    if (check_cfg(cfg) != DWKV_OK) return 0;
    return meta_layout(make_geom(cfg)).data;
}

size_t dwkv_arena_bytes(const dwkv_config* cfg) {
    if (check_cfg(cfg) != DWKV_OK) return 0;
    const Geom G = make_geom(cfg);
    return meta_layout(G).data + worst_data_bytes(G);
}

size_t dwkv_arena_bytes_all_tiers(const dwkv_config* cfg) {
    if (check_cfg(cfg) != DWKV_OK) return 0;
    const Geom G = make_geom(cfg);
    size_t per_head = 0;
    for (int k = 0; k < G.ntiers; ++k) per_head += ((size_t)G.max_pages + 1) * G.page_units[k] * kUnit;
    return meta_layout(G).data + (size_t)G.max_batch * G.G * G.Hkv * per_head;
}

size_t dwkv_workspace_bytes(const dwkv_config* cfg, int32_t n_seqs) {
    if (check_cfg(cfg) != DWKV_OK || n_seqs < 0) return 0;
    return ws_need(make_geom(cfg), n_seqs, true);
}

dwkv_status dwkv_create(const dwkv_config* cfg, void* arena, size_t arena_bytes, const void* basis_k,
                        const void* basis_v, void* stream, dwkv_handle* out) {
    dwkv_status st;
    if (!out) return fail(DWKV_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if ((st = dwkv_config_check(cfg)) != DWKV_OK) return st;
    if (!arena || !basis_k || !basis_v) return fail(DWKV_ERR_INVALID_ARG, "arena and bases must be non-NULL");
    if (reinterpret_cast<uintptr_t>(arena) % 256) return fail(DWKV_ERR_INVALID_ARG, "arena must be 256-byte aligned");
    const Geom G = make_geom(cfg);
    const MetaLayout M = meta_layout(G);
    uint32_t big = 0;
    for (int k = 0; k < G.ntiers; ++k) big = std::max(big, G.page_units[k]);
    if (arena_bytes < M.data + (size_t)big * kUnit)
        return fail(DWKV_ERR_CAPACITY, "arena of %zu bytes is below the metadata (%zu) plus one page (%zu)",
                    arena_bytes, M.data, (size_t)big * kUnit);
    if ((arena_bytes - M.data) / kUnit >= (1ull << 32))
        return fail(DWKV_ERR_UNSUPPORTED, "page pool above 512 GiB");
    int dev = 0;
    DWKV_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    cudaPointerAttributes pa{};
    DWKV_CUDA(cudaPointerGetAttributes(&pa, arena), "cudaPointerGetAttributes(arena)");
    if (pa.type != cudaMemoryTypeDevice || pa.device != dev)
        return fail(DWKV_ERR_INVALID_ARG, "arena must be device memory of the current device %d", dev);
    auto* h = new dwkv_ctx();
    h->cfg = *cfg;
    h->geom = G;
    h->meta = M;
    h->arena = static_cast<uint8_t*>(arena);
    h->arena_bytes = arena_bytes;
    h->st = make_state(h->arena, M, arena_bytes);
    h->device = dev;
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    h->num_sms = v > 0 ? v : 1;
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    h->smem_optin = (size_t)v;
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    h->smem_per_sm = (size_t)v;
    h->len.assign((size_t)G.max_batch * G.L, 0);
    h->placed.assign((size_t)G.max_batch * G.G, 0);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t bbytes = (size_t)2 * G.G * G.Hkv * G.d * G.r_max;
    cudaError_t e = cudaMemsetAsync(h->arena, 0, M.basis_k, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(h->arena + M.basis_k, basis_k, bbytes, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(h->arena + M.basis_v, basis_v, bbytes, cudaMemcpyDeviceToDevice, s);
    // the windows' second moments start at zero (an update before any sketch averages from 0)
    if (e == cudaSuccess) e = cudaMemsetAsync(h->arena + M.moment, 0, M.basis_old - M.moment, s);
    if (e == cudaSuccess) {
        tile_basis_kernel<<<G.G * G.Hkv, 256, 0, s>>>(G, h->st);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) {
        const int maxs = (int)h->smem_optin;
        const void* kernels[] = {
#define DWKV_K(B, P, C) (const void*)decode_kernel<B, P, 64, 0, C>, (const void*)decode_kernel<B, P, 64, 8, C>,       \
                     (const void*)decode_kernel<B, P, 64, 16, C>, (const void*)decode_kernel<B, P, 64, 32, C>,     \
                     (const void*)decode_kernel<B, P, 128, 0, C>, (const void*)decode_kernel<B, P, 128, 8, C>,     \
                     (const void*)decode_kernel<B, P, 128, 16, C>, (const void*)decode_kernel<B, P, 128, 32, C>,   \
                     (const void*)decode_kernel<B, P, 64, -1, C>, (const void*)decode_kernel<B, P, 128, -1, C>
            DWKV_K(4, false, false), DWKV_K(4, true, false), DWKV_K(8, false, false), DWKV_K(8, true, false),
            DWKV_K(4, false, true), DWKV_K(4, true, true), DWKV_K(8, false, true), DWKV_K(8, true, true),
#undef DWKV_K
        };
        for (const void* k : kernels)
            if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, maxs);
        // the encode kernels ask for what they use (the fused append also has static smem)
        const int es = (int)encode_smem(G), ets = (int)encode_tile_smem(G);
        const void* enc[] = {(const void*)append_small_kernel<8>, (const void*)append_small_kernel<4>,
                             (const void*)retier_kernel<8>, (const void*)retier_kernel<4>};
        for (const void* k : enc)
            if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, es);
        const void* tiles[] = {(const void*)encode_kernel<8>, (const void*)encode_kernel<4>};
        for (const void* k : tiles)
            if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, ets);
        // bulk encode blocks resident per SM at this geometry's shared memory
        int occ = 0;
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, tiles[G.bits == 8 ? 0 : 1], 256, ets);
        h->enc_blocks_per_sm = std::max(1, occ);
    }
    if (e != cudaSuccess) {
        delete h;
        return cuda_fail(e, "dwkv_create");
    }
    size_t sm = 0;
    if (decode_ring_for(h, true, &sm) == 0) {
        delete h;
        return fail(DWKV_ERR_UNSUPPORTED, "decode pipeline does not fit in shared memory for this geometry");
    }
    *out = h;
    return DWKV_OK;
}

dwkv_status dwkv_destroy(dwkv_handle h) {
    if (!h) return fail(DWKV_ERR_INVALID_ARG, "handle is NULL");
    delete h;
    return DWKV_OK;
}

dwkv_status dwkv_set_decode_tuning(dwkv_handle h, int32_t ctas_per_sm, int32_t waves, int32_t stages) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if (ctas_per_sm != 1 || waves < 1 || waves > 8 || stages < 0 || stages == 1 || stages > 32)
        return fail(DWKV_ERR_INVALID_ARG, "tuning out of range (ctas_per_sm 1, waves 1-8, stages 0 or 2-32)");
    const int oc = h->dec_ctas_per_sm, ow = h->dec_waves, os = h->dec_stages_req;
    h->dec_ctas_per_sm = ctas_per_sm;
    h->dec_waves = waves;
    h->dec_stages_req = stages;
    size_t sm = 0;
    if (decode_ring_for(h, true, &sm) == 0) {
        h->dec_ctas_per_sm = oc; h->dec_waves = ow; h->dec_stages_req = os;
        return fail(DWKV_ERR_INVALID_ARG, "tuning leaves no room for two page chunks");
    }
    return DWKV_OK;
}

dwkv_status dwkv_set_decode_overlap(dwkv_handle h, int32_t enable) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if (enable != 0 && enable != 1) return fail(DWKV_ERR_INVALID_ARG, "enable must be 0 or 1 (got %d)", enable);
    h->dec_overlap = enable;
    return DWKV_OK;
}

// ------------------------------------------------------------------------------------
// Online bases ([DW] §3 Method, the shared-bases paragraph): sketch after prefill, moving-
// average update with re-projection of the stored tokens.
// ------------------------------------------------------------------------------------
namespace {
// Windows [g0, g0 + ng) of a basis call: group >= 0 one window, DWKV_ALL_GROUPS every window.
dwkv_status basis_windows(dwkv_handle h, int32_t group, int* g0, int* ng) {
    const Geom& G = h->geom;
    if (group == DWKV_ALL_GROUPS) { *g0 = 0; *ng = G.G; return DWKV_OK; }
    if (group < 0 || group >= G.G) return fail(DWKV_ERR_INVALID_ARG, "group %d out of [0, %d)", group, G.G);
    *g0 = group;
    *ng = 1;
    return DWKV_OK;
}

dwkv_status check_basis_args(dwkv_handle h, int32_t n_rows, const void* k_rows, const void* v_rows) {
    const Geom& G = h->geom;
    if (G.r_max > 64) return fail(DWKV_ERR_UNSUPPORTED, "online bases are built for r_max <= 64 (got %d)", G.r_max);
    if (n_rows < 0) return fail(DWKV_ERR_INVALID_ARG, "n_rows %d is negative", n_rows);
    if (n_rows > 0 && (!k_rows || !v_rows)) return fail(DWKV_ERR_INVALID_ARG, "k_rows and v_rows must be non-NULL");
    return DWKV_OK;
}

float* moment_of(dwkv_handle h, int g) {
    const Geom& G = h->geom;
    return reinterpret_cast<float*>(h->arena + h->meta.moment) + (size_t)g * G.Hkv * 2 * kD * kD;
}

// cuTensorMapEncodeTiled from the driver through the runtime's entry-point query (the
// library does not link the driver library itself).
using TensorMapEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                       const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                       CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
TensorMapEncodeFn tensor_map_encoder() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return nullptr;
    return reinterpret_cast<TensorMapEncodeFn>(fn);
}

dwkv_status launch_gram(dwkv_handle h, int g0, int ng, int32_t n_rows, const void* k_rows, const void* v_rows,
                        float scale, cudaStream_t s) {
    const Geom& G = h->geom;
    if (n_rows == 0) return DWKV_OK;
    const long long rows = (long long)G.LPG * n_rows;             // a window's rows
    if (rows * G.Hkv * kD >= (1ll << 31) / 2)
        return fail(DWKV_ERR_INVALID_ARG, "n_rows %d: a window's rows exceed the moment kernel's range", n_rows);
    if ((reinterpret_cast<uintptr_t>(k_rows) | reinterpret_cast<uintptr_t>(v_rows)) & 15u)
        return fail(DWKV_ERR_INVALID_ARG, "k_rows and v_rows must be 16-byte aligned");
    // the rows as a 4-D tensor [windows][rows][Hkv][d] for the TMA copies: boxes of 64 channels
    // x 1 head x 64 rows (128-byte swizzle); rows past a window's end read as zeros
    static TensorMapEncodeFn encode = tensor_map_encoder();
    if (!encode) return fail(DWKV_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    CUtensorMap maps[2];
    const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)G.Hkv, (cuuint64_t)rows, (cuuint64_t)ng};
    const cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)G.Hkv * kD * 2, (cuuint64_t)rows * G.Hkv * kD * 2};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    for (int z = 0; z < 2; ++z) {
        const CUresult r = encode(&maps[z], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(z ? v_rows : k_rows),
                                  dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(DWKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    }
    const size_t sm = gram_smem_bytes();
    DWKV_CUDA(cudaFuncSetAttribute(gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm),
              "gram_kernel shared memory");
    // blocks per (window, kv-head, side): about 4 an SM over the call (the most that fit: the
    // stage buffers keep a block's share of an SM's shared memory above a quarter, so the
    // blocks' tensor-memory columns, 128 each, never exceed the SM's 512), each a whole number
    // of 64-row chunks so that only a window's last chunk reaches past its rows
    const long long combos = 2ll * G.Hkv * ng;
    const long long want = std::max(1ll, 4ll * h->num_sms / combos);
    const long long chunks = (rows + 63) / 64;
    const long long per_chunks = (chunks + std::min(want, chunks) - 1) / std::min(want, chunks);
    const int rows_per_block = (int)(per_chunks * 64);
    const int nblk = (int)((chunks + per_chunks - 1) / per_chunks);
    gram_kernel<<<dim3(nblk, G.Hkv * ng, 2), 128, sm, s>>>(maps[0], maps[1], G, h->st, n_rows, rows_per_block,
                                                           moment_of(h, g0), scale);
    DWKV_CUDA(cudaGetLastError(), "gram_kernel launch");
    return DWKV_OK;
}

dwkv_status launch_basis(dwkv_handle h, int g0, int ng, const float* omega, int32_t power_steps, float* eig,
                         cudaStream_t s) {
    const Geom& G = h->geom;
    const size_t sm = basis_smem_bytes(G.r_max);
    DWKV_CUDA(cudaFuncSetAttribute(basis_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm),
              "basis_kernel shared memory");
    basis_kernel<<<dim3(2 * G.Hkv, ng), 512, sm, s>>>(G, h->st, g0, moment_of(h, g0), omega, power_steps, eig);
    DWKV_CUDA(cudaGetLastError(), "basis_kernel launch");
    return DWKV_OK;
}
}  // namespace

dwkv_status dwkv_basis_sketch(dwkv_handle h, int32_t group, int32_t n_rows, const void* k_rows, const void* v_rows,
                              const float* omega, int32_t power_steps, float* eigenvalues, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    int g0 = 0, ng = 0;
    if ((st = basis_windows(h, group, &g0, &ng)) != DWKV_OK) return st;
    if ((st = check_basis_args(h, n_rows, k_rows, v_rows)) != DWKV_OK) return st;
    if (n_rows < 1) return fail(DWKV_ERR_INVALID_ARG, "the sketch needs rows (n_rows = %d)", n_rows);
    if (!omega) return fail(DWKV_ERR_INVALID_ARG, "omega must be non-NULL");
    if (power_steps < 0 || power_steps > 16) return fail(DWKV_ERR_INVALID_ARG, "power_steps %d out of [0, 16]", power_steps);
    const Geom& G = h->geom;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DWKV_CUDA(cudaMemsetAsync(moment_of(h, g0), 0, sizeof(float) * ng * G.Hkv * 2 * kD * kD, s),
              "clear the windows' moments");
    if ((st = launch_gram(h, g0, ng, n_rows, k_rows, v_rows, 1.0f, s)) != DWKV_OK) return st;
    if ((st = launch_basis(h, g0, ng, omega, power_steps, eigenvalues, s)) != DWKV_OK) return st;
    note_plain_launch(h);
    return DWKV_OK;
}

dwkv_status dwkv_basis_update(dwkv_handle h, int32_t group, int32_t n_rows, const void* k_rows, const void* v_rows,
                              float beta, int32_t n_seqs, const int32_t* seq_ids, float* eigenvalues, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    int g0 = 0, ng = 0;
    if ((st = basis_windows(h, group, &g0, &ng)) != DWKV_OK) return st;
    if ((st = check_basis_args(h, n_rows, k_rows, v_rows)) != DWKV_OK) return st;
    if (!(beta >= 0.f && beta <= 1.f)) return fail(DWKV_ERR_INVALID_ARG, "beta must be in [0, 1]");
    if ((st = check_seq_list(h, n_seqs, seq_ids)) != DWKV_OK) return st;
    const Geom& G = h->geom;
    for (int i = 0; i < n_seqs; ++i) {
        const int sq = seq_ids[i];
        for (int g = g0; g < g0 + ng; ++g) {
            const int pl = h->placed[(size_t)sq * G.G + g];
            for (int l = g * G.LPG; l < (g + 1) * G.LPG; ++l)
                if (h->len[(size_t)sq * G.L + l] != pl)
                    return fail(DWKV_ERR_INVALID_ARG, "sequence %d: layer %d holds %d positions but its group placed %d; "
                                                      "update the basis only when every layer of the group holds the "
                                                      "same positions",
                                sq, l, h->len[(size_t)sq * G.L + l], pl);
        }
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    moment_scale_kernel<<<128, 256, 0, s>>>(moment_of(h, g0), (size_t)ng * G.Hkv * 2 * kD * kD, beta);
    DWKV_CUDA(cudaGetLastError(), "moment_scale_kernel launch");
    if ((st = launch_gram(h, g0, ng, n_rows, k_rows, v_rows, 1.0f - beta, s)) != DWKV_OK) return st;
    // the current bases, for the stored tokens' reconstruction: [K|V][window][Hkv][d][r_max]
    const size_t bbytes = (size_t)G.Hkv * kD * G.r_max * 2;
    uint8_t* old = h->arena + h->meta.basis_old;
    DWKV_CUDA(cudaMemcpyAsync(old, h->arena + h->meta.basis_k + (size_t)g0 * bbytes, ng * bbytes,
                              cudaMemcpyDeviceToDevice, s), "save the K bases");
    DWKV_CUDA(cudaMemcpyAsync(old + ng * bbytes, h->arena + h->meta.basis_v + (size_t)g0 * bbytes, ng * bbytes,
                              cudaMemcpyDeviceToDevice, s), "save the V bases");
    if ((st = launch_basis(h, g0, ng, nullptr, 0, eigenvalues, s)) != DWKV_OK) return st;
    const size_t sm = reproject_smem_bytes(G.r_max, 12);
    auto kern = G.bits == 8 ? reproject_kernel<8> : reproject_kernel<4>;
    DWKV_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm),
              "reproject_kernel shared memory");
    int resident = 0;
    DWKV_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kern, 384, sm), "reproject_kernel occupancy");
    resident = std::max(1, resident) * h->num_sms;
    for (int i0 = 0; i0 < n_seqs; i0 += kMaxSeqs) {
        SeqList L;
        memset(&L, 0, sizeof(L));
        L.n = std::min(kMaxSeqs, n_seqs - i0);
        for (int i = 0; i < L.n; ++i) L.seq[i] = seq_ids[i0 + i];
        // blocks per (sequence, kv-head, side): about eight waves of resident blocks over the
        // call, so that blocks finishing at different times leave the SMs evenly loaded (one
        // block's two bases are ~1 % of its work)
        const int per = std::max(1, (8 * resident + 2 * L.n * G.Hkv - 1) / (2 * L.n * G.Hkv));
        for (int g = g0; g < g0 + ng; ++g) {
            const __nv_bfloat16* ok_ = reinterpret_cast<const __nv_bfloat16*>(old + (size_t)(g - g0) * bbytes);
            const __nv_bfloat16* ov_ = reinterpret_cast<const __nv_bfloat16*>(old + (size_t)(ng + g - g0) * bbytes);
            kern<<<dim3(L.n, G.Hkv, 2 * per), 384, sm, s>>>(G, h->st, g, L, ok_, ov_);
            DWKV_CUDA(cudaGetLastError(), "reproject_kernel launch");
        }
    }
    note_plain_launch(h);
    return DWKV_OK;
}

dwkv_status dwkv_get_bases(dwkv_handle h, int32_t group, void* basis_k, void* basis_v, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    const Geom& G = h->geom;
    if (group < 0 || group >= G.G) return fail(DWKV_ERR_INVALID_ARG, "group %d out of [0, %d)", group, G.G);
    if (!basis_k || !basis_v) return fail(DWKV_ERR_INVALID_ARG, "basis_k and basis_v must be non-NULL");
    const size_t bbytes = (size_t)G.Hkv * kD * G.r_max * 2;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DWKV_CUDA(cudaMemcpyAsync(basis_k, h->arena + h->meta.basis_k + (size_t)group * bbytes, bbytes,
                              cudaMemcpyDefault, s), "copy the K basis");
    DWKV_CUDA(cudaMemcpyAsync(basis_v, h->arena + h->meta.basis_v + (size_t)group * bbytes, bbytes,
                              cudaMemcpyDefault, s), "copy the V basis");
    return DWKV_OK;
}

dwkv_status dwkv_get_moment(dwkv_handle h, int32_t group, float* moment, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    const Geom& G = h->geom;
    if (group < 0 || group >= G.G) return fail(DWKV_ERR_INVALID_ARG, "group %d out of [0, %d)", group, G.G);
    if (!moment) return fail(DWKV_ERR_INVALID_ARG, "moment must be non-NULL");
    const size_t nb = sizeof(float) * G.Hkv * 2 * kD * kD;
    DWKV_CUDA(cudaMemcpyAsync(moment, h->arena + h->meta.moment + (size_t)group * nb, nb, cudaMemcpyDefault,
                              static_cast<cudaStream_t>(stream)), "copy the moment");
    return DWKV_OK;
}

dwkv_status dwkv_seq_length(dwkv_handle h, int32_t seq, int32_t layer, int32_t* len) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if ((st = check_layer(h, layer)) != DWKV_OK) return st;
    if (seq < 0 || seq >= h->geom.max_batch) return fail(DWKV_ERR_INVALID_ARG, "sequence id %d out of range", seq);
    if (!len) return fail(DWKV_ERR_INVALID_ARG, "len is NULL");
    *len = h->len[(size_t)seq * h->geom.L + layer];
    return DWKV_OK;
}

dwkv_status dwkv_reset_sequence(dwkv_handle h, int32_t seq, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    const Geom& G = h->geom;
    if (seq < 0 || seq >= G.max_batch) return fail(DWKV_ERR_INVALID_ARG, "sequence id %d out of range", seq);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    reset_kernel<<<1, 256, 0, s>>>(G, h->st, seq);
    DWKV_CUDA(cudaGetLastError(), "reset_kernel launch");
    note_plain_launch(h);
    DWKV_CUDA(cudaMemsetAsync(h->st.slot_map + slot_index(G, seq, 0, 0, 0), 0,
                              (size_t)4 * G.G * G.Hkv * G.max_context, s),
              "cudaMemsetAsync(slot map)");
    std::fill(h->len.begin() + (size_t)seq * G.L, h->len.begin() + (size_t)(seq + 1) * G.L, 0);
    std::fill(h->placed.begin() + (size_t)seq * G.G, h->placed.begin() + (size_t)(seq + 1) * G.G, 0);
    return DWKV_OK;
}

static dwkv_status append_impl(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                               const int32_t* n_new, const void* k_new, const void* v_new,
                               const uint8_t* tier_idx, const float* gate, float* coeff_dbg, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    AppendCall C;
    if ((st = prepare_call(h, layer, n_seqs, seq_ids, n_new, C, true, tier_idx)) != DWKV_OK) return st;
    if (C.total == 0) return DWKV_OK;
    if (!k_new || !v_new) return fail(DWKV_ERR_INVALID_ARG, "k_new and v_new must be non-NULL");
    if ((reinterpret_cast<uintptr_t>(k_new) | reinterpret_cast<uintptr_t>(v_new)) & 15u)
        return fail(DWKV_ERR_INVALID_ARG, "k_new and v_new must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(gate) & 3u) return fail(DWKV_ERR_INVALID_ARG, "gate must be 4-byte aligned");
    C.gate = gate;
    const Geom& G = h->geom;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    bool any = false;
    int most = 0;
    for (int i = 0; i < C.n; ++i) {
        any |= C.na[i] > 0;
        most = std::max(most, n_new[i]);
    }
    const size_t sm = encode_smem(G);
    if (most <= 4) {
        // decode-sized append: placement and encode in one launch, a block per (sequence, kv-head)
        const dim3 grid(C.n, G.Hkv);
        if (G.bits == 8)
            append_small_kernel<8><<<grid, 256, sm, s>>>(G, h->st, C, tier_idx, any ? 1 : 0,
                                                         static_cast<const __nv_bfloat16*>(k_new),
                                                         static_cast<const __nv_bfloat16*>(v_new), coeff_dbg);
        else
            append_small_kernel<4><<<grid, 256, sm, s>>>(G, h->st, C, tier_idx, any ? 1 : 0,
                                                         static_cast<const __nv_bfloat16*>(k_new),
                                                         static_cast<const __nv_bfloat16*>(v_new), coeff_dbg);
        DWKV_CUDA(cudaGetLastError(), "append_small_kernel launch");
        note_plain_launch(h);
        commit_call(h, C, n_new);
        return DWKV_OK;
    }
    if (any) {
        place_kernel<<<dim3(C.n, G.Hkv), 256, 0, s>>>(G, h->st, C, tier_idx);
        DWKV_CUDA(cudaGetLastError(), "place_kernel launch");
        note_plain_launch(h);
    }
    // a block per (kv-head, K or V) and share of the tiles, one wave of resident blocks
    const long long ntiles = (C.total + kEncTile - 1) / kEncTile;
    const long long per = std::max(1, h->enc_blocks_per_sm * h->num_sms / std::max(1, 2 * G.Hkv));
    const dim3 grid((unsigned)std::min(ntiles, per), G.Hkv, 2);
    const size_t tsm = encode_tile_smem(G);
    if (G.bits == 8)
        encode_kernel<8><<<grid, 256, tsm, s>>>(G, h->st, C, static_cast<const __nv_bfloat16*>(k_new),
                                                 static_cast<const __nv_bfloat16*>(v_new), coeff_dbg);
    else
        encode_kernel<4><<<grid, 256, tsm, s>>>(G, h->st, C, static_cast<const __nv_bfloat16*>(k_new),
                                                 static_cast<const __nv_bfloat16*>(v_new), coeff_dbg);
    DWKV_CUDA(cudaGetLastError(), "encode_kernel launch");
    note_plain_launch(h);
    commit_call(h, C, n_new);
    return DWKV_OK;
}

dwkv_status dwkv_append(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids, const int32_t* n_new,
                        const void* k_new, const void* v_new, const uint8_t* tier_idx, float* coeff_dbg,
                        void* stream) {
    return append_impl(h, layer, n_seqs, seq_ids, n_new, k_new, v_new, tier_idx, nullptr, coeff_dbg, stream);
}

dwkv_status dwkv_append_gated(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                              const int32_t* n_new, const void* k_new, const void* v_new, const uint8_t* tier_idx,
                              const float* gate, float* coeff_dbg, void* stream) {
    if (!gate) return fail(DWKV_ERR_INVALID_ARG, "gate is NULL (use dwkv_append)");
    return append_impl(h, layer, n_seqs, seq_ids, n_new, k_new, v_new, tier_idx, gate, coeff_dbg, stream);
}

dwkv_status dwkv_append_compressed(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                                   const int32_t* n_new, const uint8_t* tier_idx, const void* coeff,
                                   const uint8_t* idx, const int8_t* codes, const void* scales, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    AppendCall C;
    if ((st = prepare_call(h, layer, n_seqs, seq_ids, n_new, C, true, tier_idx)) != DWKV_OK) return st;
    if (C.total == 0) return DWKV_OK;
    const Geom& G = h->geom;
    if (!coeff || !scales || (G.s > 0 && (!idx || !codes)))
        return fail(DWKV_ERR_INVALID_ARG, "coeff, idx, codes and scales must be non-NULL");
    if (((uintptr_t)coeff & 1u) || ((uintptr_t)scales & 1u))
        return fail(DWKV_ERR_INVALID_ARG, "coeff and scales must be 2-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    bool any = false;
    for (int i = 0; i < C.n; ++i) any |= C.na[i] > 0;
    if (any) {
        place_kernel<<<dim3(C.n, G.Hkv), 256, 0, s>>>(G, h->st, C, tier_idx);
        DWKV_CUDA(cudaGetLastError(), "place_kernel launch");
        note_plain_launch(h);
    }
    const dim3 grid(grid_rows(h, C.total), G.Hkv);
    if (G.bits == 8)
        import_kernel<8><<<grid, 256, 0, s>>>(G, h->st, C, static_cast<const uint8_t*>(coeff), idx, codes,
                                              static_cast<const __half*>(scales));
    else
        import_kernel<4><<<grid, 256, 0, s>>>(G, h->st, C, static_cast<const uint8_t*>(coeff), idx, codes,
                                              static_cast<const __half*>(scales));
    DWKV_CUDA(cudaGetLastError(), "import_kernel launch");
    note_plain_launch(h);
    commit_call(h, C, n_new);
    return DWKV_OK;
}

// One new token per sequence appended by the decode launch itself (see the decode kernel).
struct FusedAppend {
    const void* k_new;
    const void* v_new;
    const uint8_t* tier_idx;
    const AppendCall* call;          // positions and which sequences this layer places
};

// Shared memory the fused append borrows from the page ring: both bases with padded rows,
// and two encode warps' scratch.
size_t fused_ring_need(const Geom& G) {
    return (size_t)2 * kD * (G.r_max + 2) * 2 + (size_t)2 * (kD + kMaxRank + 32) * 4;
}

// Splits (CTAs per kv-head) of each sequence of a decode launch.  The launch aims at
// SMs x waves CTAs in all, i.e. S = SMs x waves / Hkv splits per kv-head, apportioned to the
// sequences in proportion to the tokens they hold (a sequence's bytes are its tokens times
// the mean bytes of its tiers, which the host does not know; the tiers are i.i.d. across
// sequences, so tokens stand in for bytes) by largest remainders.  Every sequence gets at
// least one split (an empty one writes zeros) and at most min(kMaxSplits, its pages).
void split_counts(dwkv_handle h, int layer, int n_seqs, const int32_t* seq_ids, long long tot, int* sp) {
    const Geom& G = h->geom;
    const long long S = std::max(1ll, (long long)h->num_sms * h->dec_waves / G.Hkv);
    std::vector<long long> len(n_seqs), cap(n_seqs), rem(n_seqs);
    long long used = 0;
    for (int i = 0; i < n_seqs; ++i) {
        len[i] = h->len[(size_t)seq_ids[i] * G.L + layer];
        cap[i] = std::max(1ll, std::min((long long)kMaxSplits, (len[i] + kPage - 1) / kPage));
        const long long q = tot > 0 ? S * len[i] / tot : 0;      // ideal share S len / tot, floored
        rem[i] = tot > 0 ? S * len[i] % tot : 0;
        sp[i] = (int)std::max(1ll, std::min(q, cap[i]));
        used += sp[i];
    }
    // the splits left over go to the largest remainders first (ties to the earlier sequence),
    // then, while some remain (caps cut a share), to the sequence with most tokens per split
    std::vector<int> order(n_seqs);
    for (int i = 0; i < n_seqs; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return rem[a] > rem[b]; });
    for (int i : order) {
        if (used >= S) break;
        if (sp[i] < cap[i]) { ++sp[i]; ++used; }
    }
    while (used < S) {
        int best = -1;
        for (int i = 0; i < n_seqs; ++i)
            if (sp[i] < cap[i] && (best < 0 || len[i] * sp[best] > len[best] * sp[i])) best = i;
        if (best < 0) break;
        ++sp[best];
        ++used;
    }
}

// One decode-kernel launch.  With `overlap` it is launched with programmatic stream
// serialisation: its CTAs may start on SMs the previous kernel of the stream has left, set up
// their pipeline and stream their first pages before waiting for that kernel (the kernel
// waits before it reads q, the new token or anything a decode writes).
cudaError_t launch_decode(void (*k)(const Geom, const State, const DecodeCall), dim3 grid, size_t smem,
                          cudaStream_t s, bool overlap, const Geom& G, const State& St, const DecodeCall& C) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = dim3(kDecodeThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = at;
    lc.numAttrs = overlap ? 1 : 0;
    return cudaLaunchKernelEx(&lc, k, G, St, C);
}

static dwkv_status run_decode(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids, const void* q,
                              float* out, float* err, float* out_full, void* workspace, size_t ws_bytes,
                              void* stream, bool probe, const FusedAppend* fa = nullptr) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if ((st = check_layer(h, layer)) != DWKV_OK) return st;
    if ((st = check_seq_list(h, n_seqs, seq_ids)) != DWKV_OK) return st;
    if (n_seqs == 0) return DWKV_OK;
    const Geom& G = h->geom;
    if (!q) return fail(DWKV_ERR_INVALID_ARG, "q is NULL");
    if (!probe && !out) return fail(DWKV_ERR_INVALID_ARG, "out is NULL");
    if (probe && !err) return fail(DWKV_ERR_INVALID_ARG, "err is NULL");
    if (!workspace) return fail(DWKV_ERR_INVALID_ARG, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(workspace) % 16) return fail(DWKV_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    const size_t need = ws_need(G, n_seqs, probe);
    if (ws_bytes < need) return fail(DWKV_ERR_CAPACITY, "workspace of %zu bytes is below the %zu needed", ws_bytes, need);
    const int g = layer / G.LPG;
    long long tot = 0;
    for (int i = 0; i < n_seqs; ++i) {
        const int s = seq_ids[i];
        const int len = h->len[(size_t)s * G.L + layer], pl = h->placed[(size_t)s * G.G + g];
        if (len != pl)
            return fail(DWKV_ERR_INVALID_ARG, "sequence %d holds %d positions at layer %d but its group placed %d; "
                                              "append every layer of the group before decoding it", s, len, layer, pl);
        tot += len;
    }
    DecodeCall C;
    memset(&C, 0, sizeof(C));
    C.n = n_seqs;
    C.layer = layer;
    C.g = g;
    C.lig = layer % G.LPG;
    size_t smem = 0;
    const uint32_t ring = decode_ring_for(h, probe, &smem);
    if (ring == 0) return fail(DWKV_ERR_UNSUPPORTED, "decode pipeline does not fit in shared memory");
    std::vector<int> sp(n_seqs);
    split_counts(h, layer, n_seqs, seq_ids, tot, sp.data());
    int total = 0;
    for (int i = 0; i < n_seqs; ++i) {
        C.seq[i] = seq_ids[i];
        C.split_begin[i] = total;
        total += sp[i];
    }
    // cache state written by the previous launch, if that was a fused step of this group: a
    // placing launch adds its token's count at its end; every fused launch writes its token's
    // bytes of its layer
    {
        const int pl = h->last_fused_layer;
        const bool same_group = pl >= 0 && pl / G.LPG == g;
        C.early = (same_group && (h->last_fused_placed || pl == layer)) ? 0 : 1;
    }
    C.split_begin[n_seqs] = total;
    C.total_splits = total;
    C.ring_bytes = (int)ring;
    C.rec_floats = rec_floats_of(G, probe);
    C.tok_weight = h->dec_tok_weight;
    C.owner_cost = 0;
    if (fa) {
        C.fused = 1;
        C.owner_cost = h->dec_owner_cost;
        C.k_new = static_cast<const __nv_bfloat16*>(fa->k_new);
        C.v_new = static_cast<const __nv_bfloat16*>(fa->v_new);
        C.tier_idx = fa->tier_idx;
        for (int i = 0; i < n_seqs; ++i) {
            C.pos[i] = fa->call->pos0[i];
            C.place[i] = fa->call->na[i] > 0 ? 1 : 0;
        }
    }
    C.q = static_cast<const __nv_bfloat16*>(q);
    C.out = out;
    C.out_full = out_full;
    C.err = err;
    C.ws = static_cast<float*>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const dim3 grid(total, G.Hkv);
    const bool big = G.r_max > 64;
    cudaError_t lerr = cudaSuccess;
#define DWKV_LAUNCH(B, P, R, SS)                                                                                        \
    lerr = G.c8 ? launch_decode(decode_kernel<B, P, R, SS, true>, grid, smem, s, h->dec_overlap != 0, G, h->st, C)      \
                : launch_decode(decode_kernel<B, P, R, SS, false>, grid, smem, s, h->dec_overlap != 0, G, h->st, C)
#define DWKV_LAUNCH_S(B, P, R)                                  \
    do {                                                        \
        switch (G.routed ? -1 : G.s) {                          \
            case -1: DWKV_LAUNCH(B, P, R, -1); break;           \
            case 0: DWKV_LAUNCH(B, P, R, 0); break;             \
            case 8: DWKV_LAUNCH(B, P, R, 8); break;             \
            case 16: DWKV_LAUNCH(B, P, R, 16); break;           \
            default: DWKV_LAUNCH(B, P, R, 32); break;           \
        }                                                       \
    } while (0)
#define DWKV_LAUNCH_R(B, P) \
    do { if (big) DWKV_LAUNCH_S(B, P, 128); else DWKV_LAUNCH_S(B, P, 64); } while (0)
    if (!probe) {
        if (G.bits == 8) DWKV_LAUNCH_R(8, false);
        else DWKV_LAUNCH_R(4, false);
    } else {
        if (G.bits == 8) DWKV_LAUNCH_R(8, true);
        else DWKV_LAUNCH_R(4, true);
    }
#undef DWKV_LAUNCH_R
#undef DWKV_LAUNCH_S
#undef DWKV_LAUNCH
    if (lerr != cudaSuccess) return cuda_fail(lerr, probe ? "probe kernel launch" : "decode kernel launch");
    DWKV_CUDA(cudaGetLastError(), probe ? "probe kernel launch" : "decode kernel launch");
    h->last_fused_layer = fa ? layer : -1;
    h->last_fused_placed = 0;
    if (fa)
        for (int i = 0; i < n_seqs; ++i) h->last_fused_placed |= C.place[i];
    return DWKV_OK;
}

dwkv_status dwkv_decode_attention(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                                  const void* q, float* out, void* workspace, size_t ws_bytes, void* stream) {
    return run_decode(h, layer, n_seqs, seq_ids, q, out, nullptr, nullptr, workspace, ws_bytes, stream, false);
}

dwkv_status dwkv_append_decode_attention(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                                         const void* k_new, const void* v_new, const uint8_t* tier_idx,
                                         const void* q, float* out, void* workspace, size_t ws_bytes,
                                         void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if ((st = check_layer(h, layer)) != DWKV_OK) return st;
    if (n_seqs < 0 || n_seqs > kMaxSeqs) return fail(DWKV_ERR_INVALID_ARG, "n_seqs %d out of range", n_seqs);
    if (n_seqs == 0) return DWKV_OK;
    if (!k_new || !v_new) return fail(DWKV_ERR_INVALID_ARG, "k_new and v_new must be non-NULL");
    if (!q || !out || !workspace) return fail(DWKV_ERR_INVALID_ARG, "q, out and workspace must be non-NULL");
    if (reinterpret_cast<uintptr_t>(workspace) % 16) return fail(DWKV_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
    const size_t need = ws_need(h->geom, n_seqs, false);
    if (ws_bytes < need) return fail(DWKV_ERR_CAPACITY, "workspace of %zu bytes is below the %zu needed", ws_bytes, need);
    std::vector<int32_t> ones((size_t)n_seqs, 1);
    AppendCall A;
    if ((st = prepare_call(h, layer, n_seqs, seq_ids, ones.data(), A, true, tier_idx)) != DWKV_OK) return st;
    const Geom& G = h->geom;
    size_t smem = 0;
    if (decode_ring_for(h, false, &smem) < fused_ring_need(G)) {
        // the ring is capped below what the fused append borrows: two launches instead
        if ((st = dwkv_append(h, layer, n_seqs, seq_ids, ones.data(), k_new, v_new, tier_idx, nullptr, stream)) !=
            DWKV_OK)
            return st;
        return dwkv_decode_attention(h, layer, n_seqs, seq_ids, q, out, workspace, ws_bytes, stream);
    }
    commit_call(h, A, ones.data());          // the decode below attends to the new positions
    const FusedAppend fa{k_new, v_new, tier_idx, &A};
    return run_decode(h, layer, n_seqs, seq_ids, q, out, nullptr, nullptr, workspace, ws_bytes, stream, false, &fa);
}

dwkv_status dwkv_probe(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids, const void* q,
                       float* err, float* out_full, void* workspace, size_t ws_bytes, void* stream) {
    return run_decode(h, layer, n_seqs, seq_ids, q, nullptr, err, out_full, workspace, ws_bytes, stream, true);
}

dwkv_status dwkv_retier(dwkv_handle h, int32_t group, int32_t n_seqs, const int32_t* seq_ids, const int32_t* n_tok,
                        const int32_t* positions, const uint8_t* new_tier, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    const Geom& G = h->geom;
    if (group < 0 || group >= G.G) return fail(DWKV_ERR_INVALID_ARG, "group %d out of [0, %d)", group, G.G);
    if ((st = check_seq_list(h, n_seqs, seq_ids)) != DWKV_OK) return st;
    if (n_seqs && !n_tok) return fail(DWKV_ERR_INVALID_ARG, "n_tok is NULL");
    std::vector<int> first(n_seqs + 1, 0);
    for (int i = 0; i < n_seqs; ++i) {
        const int s = seq_ids[i];
        const int pl = h->placed[(size_t)s * G.G + group];
        for (int l = group * G.LPG; l < (group + 1) * G.LPG; ++l)
            if (h->len[(size_t)s * G.L + l] != pl)
                return fail(DWKV_ERR_INVALID_ARG, "sequence %d: layer %d holds %d positions but its group placed %d; "
                                                  "re-tier only when every layer of the group holds the same positions",
                            s, l, h->len[(size_t)s * G.L + l], pl);
        if (n_tok[i] < 0 || n_tok[i] > pl)
            return fail(DWKV_ERR_INVALID_ARG, "n_tok[%d] = %d out of [0, %d]", i, n_tok[i], pl);
        first[i + 1] = first[i] + n_tok[i];
    }
    if (first[n_seqs] == 0) return DWKV_OK;
    if (!positions || !new_tier) return fail(DWKV_ERR_INVALID_ARG, "positions and new_tier must be non-NULL");
    // Rounds of at most one page of tokens per sequence, each followed by the release of the
    // pages the moves emptied: a round needs at most a page or two more per tier than the
    // tokens it moves, so a cache sized by dwkv_arena_bytes has room for any number of moves.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t sm = encode_smem(G);
    for (int r0 = 0;; r0 += kPage) {
        RetierCall C;
        memset(&C, 0, sizeof(C));
        C.g = group;
        for (int i = 0; i < n_seqs; ++i) {
            if (n_tok[i] <= r0) continue;
            C.seq[C.n] = seq_ids[i];
            C.begin[C.n] = first[i] + r0;
            C.end[C.n] = first[i] + std::min(n_tok[i], r0 + kPage);
            ++C.n;
        }
        if (C.n == 0) break;
        const dim3 grid(C.n, G.Hkv);
        if (G.bits == 8) retier_kernel<8><<<grid, 256, sm, s>>>(G, h->st, C, positions, new_tier);
        else retier_kernel<4><<<grid, 256, sm, s>>>(G, h->st, C, positions, new_tier);
        DWKV_CUDA(cudaGetLastError(), "retier_kernel launch");
        retier_release_kernel<<<1, 256, 0, s>>>(G, h->st, C);
        DWKV_CUDA(cudaGetLastError(), "retier_release_kernel launch");
    }
    note_plain_launch(h);
    return DWKV_OK;
}

dwkv_status dwkv_export(dwkv_handle h, int32_t layer, int32_t seq, int32_t t0, int32_t n, uint8_t* tier_idx,
                        void* coeff, uint8_t* idx, int8_t* codes, void* scales, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if ((st = check_layer(h, layer)) != DWKV_OK) return st;
    const Geom& G = h->geom;
    if (seq < 0 || seq >= G.max_batch) return fail(DWKV_ERR_INVALID_ARG, "sequence id %d out of range", seq);
    const int len = h->len[(size_t)seq * G.L + layer];
    if (t0 < 0 || n < 0 || (long long)t0 + n > len)
        return fail(DWKV_ERR_INVALID_ARG, "positions [%d, %lld) outside the %d held", t0, (long long)t0 + n, len);
    if (n == 0) return DWKV_OK;
    if (((uintptr_t)coeff & 1u) || ((uintptr_t)scales & 1u))
        return fail(DWKV_ERR_INVALID_ARG, "coeff and scales must be 2-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int grid = (int)std::min<long long>(((long long)n * G.Hkv + 7) / 8, 4096);
    if (G.bits == 8)
        export_kernel<8><<<grid, 256, 0, s>>>(G, h->st, layer, seq, t0, n, tier_idx,
                                              static_cast<uint8_t*>(coeff), idx, codes, static_cast<__half*>(scales));
    else
        export_kernel<4><<<grid, 256, 0, s>>>(G, h->st, layer, seq, t0, n, tier_idx,
                                              static_cast<uint8_t*>(coeff), idx, codes, static_cast<__half*>(scales));
    DWKV_CUDA(cudaGetLastError(), "export_kernel launch");
    note_plain_launch(h);
    return DWKV_OK;
}

dwkv_status dwkv_pool_usage(dwkv_handle h, void* stream, dwkv_pool_stats* out) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if (!out) return fail(DWKV_ERR_INVALID_ARG, "out is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DWKV_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    unsigned long long bump = 0;
    uint32_t hd[kMaxTiers], tl[kMaxTiers];
    DWKV_CUDA(cudaMemcpy(&bump, h->st.bump, 8, cudaMemcpyDeviceToHost), "read pool");
    DWKV_CUDA(cudaMemcpy(hd, h->st.free_head, sizeof(hd), cudaMemcpyDeviceToHost), "read pool");
    DWKV_CUDA(cudaMemcpy(tl, h->st.free_tail, sizeof(tl), cudaMemcpyDeviceToHost), "read pool");
    memset(out, 0, sizeof(*out));
    out->data_bytes_total = (uint64_t)h->st.data_units * kUnit;
    out->data_bytes_reserved = std::min<uint64_t>(bump, h->st.data_units) * kUnit;
    for (int k = 0; k < h->geom.ntiers; ++k) out->free_pages[k] = (int)(tl[k] - hd[k]) > 0 ? tl[k] - hd[k] : 0;
    return DWKV_OK;
}

dwkv_status dwkv_sync_status(dwkv_handle h, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DWKV_CUDA(cudaStreamSynchronize(s), "cudaStreamSynchronize");
    uint32_t w[3] = {0, 0, 0};
    DWKV_CUDA(cudaMemcpy(w, h->st.err, sizeof(w), cudaMemcpyDeviceToHost), "read device error word");
    if (w[0] == 0) return DWKV_OK;
    DWKV_CUDA(cudaMemset(h->st.err, 0, sizeof(w)), "clear device error word");
    static const char* names[] = {"none", "page pool exhausted", "tier index out of range",
                                  "residual channel index out of range", "int4 code outside [-8, 7]",
                                  "position never placed by its group", "bounded wait timed out",
                                  "free-page ring overflow", "basis construction: a sketch column vanished"};
    const char* nm = w[0] < sizeof(names) / sizeof(names[0]) ? names[w[0]] : "unknown";
    return fail(DWKV_ERR_DEVICE_CHECK, "device check failed: %s (code %u, info %u, %u)", nm, w[0], w[1], w[2]);
}

dwkv_status dwkv_check_bounded_wait(dwkv_handle h, uint32_t limit_us, void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if (limit_us < 1 || limit_us > 2000000u)
        return fail(DWKV_ERR_INVALID_ARG, "limit_us = %u must be in 1..2000000", limit_us);
    wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(h->st, (uint64_t)limit_us * 1000ull);
    DWKV_CUDA(cudaGetLastError(), "wait_timeout_kernel launch");
    note_plain_launch(h);
    return DWKV_OK;
}

static uint32_t quantize_stride(int32_t s, int32_t bits) {
    return (off_scales_of(0, s, bits) + 2u + 15u) & ~15u;
}

size_t dwkv_quantize_work_bytes(int32_t n, int32_t s, int32_t bits) {
    if (n < 0 || s < 0 || s > kD || (bits != 8 && bits != 4)) return 0;
    return (size_t)n * quantize_stride(s, bits);
}

dwkv_status dwkv_quantize_residuals(int32_t n, int32_t s, int32_t bits, const float* r, uint8_t* idx,
                                    int8_t* codes, uint16_t* scales, void* work, size_t work_bytes,
                                    void* stream) {
    if (n < 0) return fail(DWKV_ERR_INVALID_ARG, "n = %d must be >= 0", n);
    if (s < 0 || s > kD || s % 8) return fail(DWKV_ERR_INVALID_ARG, "s = %d must be a multiple of 8 in 0..%d", s, kD);
    if (bits != 8 && bits != 4) return fail(DWKV_ERR_INVALID_ARG, "bits = %d must be 8 or 4", bits);
    if (n == 0) return DWKV_OK;
    if (!r || !scales || !work || (s > 0 && (!idx || !codes)))
        return fail(DWKV_ERR_INVALID_ARG, "r, idx, codes, scales and work must be non-NULL");
    if (work_bytes < dwkv_quantize_work_bytes(n, s, bits))
        return fail(DWKV_ERR_INVALID_ARG, "work holds %zu bytes, needs %zu", work_bytes,
                    dwkv_quantize_work_bytes(n, s, bits));
    if (reinterpret_cast<uintptr_t>(work) % 16) return fail(DWKV_ERR_INVALID_ARG, "work must be 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const unsigned grid = (unsigned)((n + 7) / 8);
    if (bits == 8)
        quantize_test_kernel<8><<<grid, 256, 0, st>>>(n, s, r, idx, codes, scales, static_cast<uint8_t*>(work),
                                                       quantize_stride(s, bits));
    else
        quantize_test_kernel<4><<<grid, 256, 0, st>>>(n, s, r, idx, codes, scales, static_cast<uint8_t*>(work),
                                                       quantize_stride(s, bits));
    DWKV_CUDA(cudaGetLastError(), "quantize_test_kernel launch");
    return DWKV_OK;
}

}  // extern "C"

// ============================================================ decode without allocation
// Some callers cannot hand this library any device memory at decode time: plugin hooks of
// an inference engine that run inside the engine's own enqueue path, or serving loops whose
// device memory is entirely reserved by their own pool up front.  For them cudaMalloc is not
// an option (it can synchronise the device, and fails once the pool holds all memory), and
// they may have no workspace buffer to lend.  dwkv_decode_attention_noalloc runs the same
// decode with a fixed scratch area that is part of the library image itself.
namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;   // 8 MiB, held by every GPU that loads the library
constexpr int kNoAllocMaxDevices = 64;

// Split-K partial records of dwkv_decode_attention_noalloc.  Every call on a device uses
// this same array, so calls that overlap on the GPU race on it.  Nothing in it has to start
// at zero: each CTA writes its record before any CTA reads it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

}  // namespace

extern "C" dwkv_status dwkv_decode_attention_noalloc(dwkv_handle h, int32_t layer, int32_t n_seqs,
                                                     const int32_t* seq_ids, const void* q, float* out,
                                                     void* stream) {
    dwkv_status st;
    if ((st = check_handle(h)) != DWKV_OK) return st;
    if (n_seqs < 0 || n_seqs > kMaxSeqs)
        return fail(DWKV_ERR_INVALID_ARG, "n_seqs %d out of [0, %d]", n_seqs, kMaxSeqs);
    const size_t need = ws_need(h->geom, n_seqs, false);
    if (need > kNoAllocScratchBytes)
        return fail(DWKV_ERR_CAPACITY,
                    "dwkv_decode_attention_noalloc: %d sequences need %zu bytes of scratch but the built-in "
                    "scratch holds %zu; decode fewer sequences per call or use dwkv_decode_attention with a "
                    "workspace", n_seqs, need, kNoAllocScratchBytes);
    int dev = -1;
    DWKV_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
    if (dev != h->device)
        return fail(DWKV_ERR_INVALID_ARG, "the handle's device %d must be current (current is %d)", h->device, dev);
    if (dev < 0 || dev >= kNoAllocMaxDevices)
        return fail(DWKV_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kNoAllocMaxDevices - 1);
    void* scratch = nullptr;
    {
        // First call on a device: resolve the device address of the scratch array.  The host
        // name g_noalloc_scratch is only a stand-in; kernels must get this address instead.
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void* ptr = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
            if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
            g_noalloc_ptr[dev] = ptr;
        }
        scratch = g_noalloc_ptr[dev];
    }
    return dwkv_decode_attention(h, layer, n_seqs, seq_ids, q, out, scratch, kNoAllocScratchBytes, stream);
}
