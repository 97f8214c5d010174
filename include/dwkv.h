/*
 * dwkv.h -- C ABI of libdwkv: decode attention read directly from a DepthWeave-KV
 * compressed KV cache, on one NVIDIA B200 (sm_100a).
 *
 * Method: "DepthWeave-KV: Token-Adaptive Cross-Layer Residual Factorization for
 * Long-Context KV Cache Compression" (arXiv 2607.06523), cited as [DW].
 *
 *  - [DW] §3 Method, Eq. (1): the key / value of token t at layer l of depth window m,
 *    kv-head h, is rebuilt as  X^ = A B_{m,h} + g R.  This library stores
 *      * per (group m, kv-head h) a basis B in bf16, d x r_max, column j = basis vector j
 *        (one for keys, one for values; [DW] §3: "independently per head and separately
 *        for keys and values");
 *      * per (layer, kv-head, token) the first r_t coefficients of A in bf16, r_t being the
 *        token's rank tier (the router's output, [DW] §3 Eq. (2));
 *      * per (layer, kv-head, token) a sparse residual R of s channels: channel indices
 *        (uint8), symmetric integer codes (int8, or int4 two's complement with the even
 *        slot in the low nibble) and one fp16 scale.  The gate g is 1.
 *  - [DW] §3, data path paragraph: decode fuses basis lookup, residual dequantisation,
 *    coefficient multiply and the attention score, and never writes the reconstructed
 *    keys / values to memory.  dwkv_decode_attention does that: it projects the query
 *    into basis space once, scores every token from its coefficients plus its residual,
 *    runs an online softmax, accumulates values in coefficient space and residual space,
 *    and applies the value basis once at the end.
 *  - [DW] §3 Eq. (3): the attention-output probe.  dwkv_probe returns, per (sequence,
 *    kv-head), ||o_full - o_nores||_2 / (||o_full||_2 + 1e-6) where o_full uses the
 *    residual and o_nores does not; the norm runs over the kv-head's query heads x d.
 *  - [DW] §3, coefficient paragraph: new keys / values are projected onto the current
 *    basis.  dwkv_append encodes them (projection, residual against the stored bf16
 *    coefficients, s largest |residual| channels with ties to the lower channel,
 *    fp16 scale = amax / qmax, codes = clamp(rint(r / scale))).
 *
 * Conventions for every call:
 *  - Ownership: the caller allocates and owns every buffer (arena, workspace, inputs,
 *    outputs).  The library never allocates or frees device memory.
 *  - Pointers named "device" must be device memory of the handle's GPU; pointers named
 *    "host" are host memory.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *  - All work is stream-ordered and asynchronous.  Arguments are validated on the host
 *    before anything is launched; on any error nothing is launched and the call returns
 *    a non-zero status.  dwkv_last_error() gives a message for the calling thread.
 *  - Checks that need device data (tier indices, residual channels, pool capacity) run
 *    inside the kernels; a failed check sets a device error word instead of faulting and
 *    the affected tokens are skipped.  dwkv_sync_status() reports it.
 *  - A handle is not thread-safe; issue its calls from one thread, on one stream.
 *  - All kernels read the cache state from device memory, so a sequence of calls may be
 *    captured in a CUDA graph and replayed; the host's own per-sequence length mirror
 *    (used only for argument checks) then advances only at capture time.
 */
#ifndef DWKV_H
#define DWKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DWKV_MAX_TIERS 8
#define DWKV_MAX_SEQS_PER_CALL 256
#define DWKV_PAGE_TOKENS 64

typedef struct dwkv_ctx* dwkv_handle;

typedef enum {
    DWKV_OK = 0,
    DWKV_ERR_INVALID_ARG = 1,   /* bad pointer, size, index or call order               */
    DWKV_ERR_CAPACITY = 2,      /* context, arena or workspace too small                */
    DWKV_ERR_CUDA = 3,          /* a CUDA runtime call failed (message has the reason)  */
    DWKV_ERR_DEVICE_CHECK = 4,  /* a kernel-side check failed (see dwkv_sync_status)    */
    DWKV_ERR_UNSUPPORTED = 5    /* valid configuration this build has no kernel for     */
} dwkv_status;

/* Device error codes recorded by kernels (first error wins). */
#define DWKV_DEV_POOL_EXHAUSTED 1   /* no page left in the arena                         */
#define DWKV_DEV_BAD_TIER 2         /* tier index >= num_tiers                           */
#define DWKV_DEV_BAD_CHANNEL 3      /* residual channel index >= head_dim                */
#define DWKV_DEV_BAD_CODE 4         /* code outside the int4 range [-8, 7]                */
#define DWKV_DEV_NO_SLOT 5          /* a layer appended a position its group never placed */
#define DWKV_DEV_TIMEOUT 6          /* a bounded wait in a kernel ran out                 */
#define DWKV_DEV_FREE_LIST 7        /* free-page ring overflow on reset                   */
#define DWKV_DEV_BASIS 8            /* basis construction: a sketch column vanished        */

/* Cache geometry.  Supported by this build: head_dim == 128; num_q_heads == 4 *
 * num_kv_heads; tiers drawn from {8, 16, 32, 64, 128}, strictly ascending, each <= r_max;
 * r_max in {8, 16, 32, 64, 128}; resid_channels s in {0, 8, 16, 32} ([DW] §3 routes at most
 * 8 residual channels per token; s is fixed per cache here); resid_bits 8 or 4; num_layers
 * a multiple of layers_per_group. */
typedef struct {
    int32_t num_layers;        /* L                                                     */
    int32_t layers_per_group;  /* w: adjacent layers sharing one basis ([DW] §3)        */
    int32_t num_q_heads;       /* Hq                                                    */
    int32_t num_kv_heads;      /* Hkv                                                   */
    int32_t head_dim;          /* d                                                     */
    int32_t r_max;             /* basis columns per (group, kv-head, K/V)               */
    int32_t num_tiers;         /* 1..DWKV_MAX_TIERS                                     */
    int32_t tiers[DWKV_MAX_TIERS]; /* coefficient rank of each tier                     */
    int32_t resid_channels;    /* s                                                     */
    int32_t resid_bits;        /* 8 (codes in [-127,127]) or 4 (codes in [-7,7])        */
    int32_t max_batch;         /* sequence slots: ids 0 .. max_batch-1                  */
    int32_t max_context;       /* tokens per sequence                                   */
    float softmax_scale;       /* <= 0 selects 1/sqrt(head_dim)                         */
    /* Residual-count routing ([DW] §3 Eq. (2): the router's level rho is the number of
     * residual channels a token keeps, at a fixed basis rank).  0: every tier keeps
     * resid_channels channels.  1: tier k keeps tier_resid[k] of {0, 2, 4, 8} channels; every
     * tier then has the same rank (tiers[k] all equal), tier_resid strictly ascending, and
     * resid_channels == 8 (the stride of the residual arrays of append_compressed / export). */
    int32_t resid_routed;
    int32_t tier_resid[DWKV_MAX_TIERS];
    /* Coefficient storage ([DW] §3 Method, the shared-bases paragraph: the projection onto the
     * basis is kept in 8-bit blockwise form).  16 (or 0): bf16.  8: int8 codes in blocks of
     * 16 coefficients with one fp16 scale a block, scale = fp16(max |c| / 127) and
     * code = clamp(rint(c / scale), -127, 127); the residual is taken against code * scale.
     * Needs r_max and every tier rank to be multiples of 16.  Re-tiering and the basis
     * update's re-projection re-encode such tokens from code * scale. */
    int32_t coeff_bits;
} dwkv_config;

/* ---- Online bases ([DW] §3 Method, the shared-bases paragraph: "initialized online from
 * the first compressed prefix block" by a randomized low-rank sketch of the cached keys and
 * values after prefill, then "an exponential moving average as generation proceeds", per head
 * and separately for keys and values).  The pages fix no sketch size or update rule; the build
 * reads them as follows, per (window, kv-head, K or V):
 *   C     = sum over the window's layers and rows of x x^T (the channel second moment, fp32);
 *   sketch: Q = GS(C Omega), then power_steps times Q = GS(C Q) (Gram-Schmidt with
 *           re-orthogonalisation, columns in order, fp64);
 *   B     = Q U, U the eigenvectors of Q^T C Q with eigenvalues in descending order (cyclic
 *           Jacobi), each column's largest-magnitude entry (lowest channel among equals)
 *           positive, rounded to bf16: a token of rank r_t uses B's first r_t columns;
 *   update: C <- beta C + (1 - beta) C_rows, then Q = GS(C B) and the same B = Q U.
 * Online bases need r_max <= 64 (else DWKV_ERR_UNSUPPORTED).  The moment reads the rows by
 * TMA: k_rows and v_rows must be 16-byte aligned (else DWKV_ERR_INVALID_ARG), and a driver
 * without cuTensorMapEncodeTiled gives DWKV_ERR_CUDA. */

#define DWKV_ALL_GROUPS (-1)

/* Sketch the bases of window `group` (or of every window: DWKV_ALL_GROUPS, in one launch)
 * from the dense rows of its layers and replace its K and V bases.  k_rows / v_rows: device
 * bf16 [layers][n_rows][num_kv_heads][head_dim] with layers = layers_per_group for one window,
 * num_layers for all (rows of any sequences; n_rows >= 1).  omega: device fp32 [head_dim][r_max] test matrix (the
 * random numbers are the caller's), shared by every head, K and V.  power_steps in [0, 16].
 * eigenvalues (nullable): device fp32 [windows][num_kv_heads][2][r_max], the Rayleigh-Ritz
 * values in the basis' column order.  The window's moment is reset to the rows' C.  Tokens already stored
 * in the window are not re-projected (sketch before storing the window's tokens).  Stream-
 * ordered; a column that vanishes in the sketch leaves the basis as it was and records
 * DWKV_DEV_BASIS. */
dwkv_status dwkv_basis_sketch(dwkv_handle h, int32_t group, int32_t n_rows, const void* k_rows, const void* v_rows,
                              const float* omega, int32_t power_steps, float* eigenvalues, void* stream);

/* Moving-average update of window `group`'s bases (or every window's: DWKV_ALL_GROUPS):
 * C <- beta C + (1 - beta) C_rows over the new
 * dense rows (n_rows >= 0, layout as dwkv_basis_sketch; 0 rows: C is only scaled), the bases
 * refreshed from C, then every stored token of the listed sequences (host seq_ids) re-projected
 * onto them: each (token, layer of the window, K / V) is reconstructed on the previous basis
 * (the fixed-order fp32 chain over its rank plus scale x code, rounded to bf16, as dwkv_retier
 * does, for either coefficient form) and encoded on the new basis at its own tier, in place.  Every layer of the window
 * must hold the same positions for each listed sequence (DWKV_ERR_INVALID_ARG otherwise).
 * beta in [0, 1].  eigenvalues: as dwkv_basis_sketch.  Tokens of sequences not listed keep
 * their bytes and are then stale against the new bases: list every sequence that holds tokens
 * in the window. */
dwkv_status dwkv_basis_update(dwkv_handle h, int32_t group, int32_t n_rows, const void* k_rows, const void* v_rows,
                              float beta, int32_t n_seqs, const int32_t* seq_ids, float* eigenvalues, void* stream);

/* Copies of window `group`'s bases (bf16 [num_kv_heads][head_dim][r_max] each; host or device
 * destinations) and of its second moment (fp32 [num_kv_heads][2][head_dim][head_dim]).
 * Stream-ordered; synchronise before reading a host copy. */
dwkv_status dwkv_get_bases(dwkv_handle h, int32_t group, void* basis_k, void* basis_v, void* stream);
dwkv_status dwkv_get_moment(dwkv_handle h, int32_t group, float* moment, void* stream);

/* Library version string. */
const char* dwkv_version(void);

/* Message of the last failed call on this thread ("" if none). */
const char* dwkv_last_error(void);

/* Validates a configuration without touching the GPU. */
dwkv_status dwkv_config_check(const dwkv_config* cfg);

/* Bytes of one stored token (one layer, one kv-head, keys + values) at tier index
 * `tier`: 2 * (C + s + s*bits/8 + 2), s the tier's residual channels, C = 2 r (bf16
 * coefficients) or r + r/8 (8-bit codes and their block scales).  0 if the arguments are
 * invalid. */
size_t dwkv_token_bytes(const dwkv_config* cfg, int32_t tier);

/* Bytes of one page of tier `tier`: DWKV_PAGE_TOKENS tokens of one (sequence, group,
 * kv-head), all layers of the group, keys and values.  0 if invalid. */
size_t dwkv_page_bytes(const dwkv_config* cfg, int32_t tier);

/* Bytes of the arena's fixed part (bases, page tables, slot maps, counters). */
size_t dwkv_metadata_bytes(const dwkv_config* cfg);

/* Arena bytes that can hold max_batch sequences of max_context tokens in every layer
 * even if every token takes the largest tier.  0 if cfg is invalid.  A smaller arena
 * (at least dwkv_metadata_bytes + one largest page) is accepted: the page pool is then
 * smaller and running out of it is a device-side DWKV_DEV_POOL_EXHAUSTED error. */
size_t dwkv_arena_bytes(const dwkv_config* cfg);

/* Arena bytes for a cache whose tokens change tier (dwkv_retier): a page that moves empty is
 * kept for reuse by its own tier (pages differ in size between tiers), so every tier may hold
 * max_context tokens' worth of pages at once: the metadata plus, for every (sequence, group,
 * kv-head) and tier, (max_pages + 1) pages of that tier.  0 if cfg is invalid. */
size_t dwkv_arena_bytes_all_tiers(const dwkv_config* cfg);

/* Workspace bytes that decode and probe need for a call over n_seqs sequences (the probe's
 * split-K records are twice as large; decode alone accepts a workspace of half this size:
 * n_seqs * Hkv * 64 records of 8 + 4 * head_dim floats). */
size_t dwkv_workspace_bytes(const dwkv_config* cfg, int32_t n_seqs);

/* Creates a cache inside `arena` (device, caller-owned, 256-byte aligned, at least
 * dwkv_metadata_bytes(cfg) + one page) on the current CUDA device.  basis_k / basis_v:
 * device bf16 [G][Hkv][head_dim][r_max] (G = num_layers / layers_per_group), copied into
 * the arena; they need not outlive the call.  The arena's metadata is cleared on
 * `stream`.  Writes the handle to *out. */
dwkv_status dwkv_create(const dwkv_config* cfg, void* arena, size_t arena_bytes,
                        const void* basis_k, const void* basis_v, void* stream,
                        dwkv_handle* out);

/* Releases the host-side handle (no device memory is freed; the arena stays the
 * caller's).  Waits for nothing: finish or synchronise the handle's stream first. */
dwkv_status dwkv_destroy(dwkv_handle h);

/* Empties sequence `seq` in every layer and returns its pages to the free pool. */
dwkv_status dwkv_reset_sequence(dwkv_handle h, int32_t seq, void* stream);

/* Host-side length of `seq` at `layer` (tokens appended so far through this handle). */
dwkv_status dwkv_seq_length(dwkv_handle h, int32_t seq, int32_t layer, int32_t* len);

/* Encodes and appends n_new[i] tokens to each listed sequence at `layer`.
 *   seq_ids, n_new : host int32 [n_seqs]; distinct ids; n_new[i] >= 0
 *   k_new, v_new   : device bf16 [sum(n_new)][Hkv][head_dim], sequences in list order,
 *                    16-byte aligned (DWKV_ERR_INVALID_ARG otherwise)
 *   tier_idx       : device uint8 [sum(n_new)][Hkv], index into cfg.tiers.  A token's
 *                    tier is fixed by the first layer of its group that appends it
 *                    ([DW] §3 Eq. (2): rho_{m,h,t} has no layer index); later layers of
 *                    the group reuse it and ignore this array (which may then be NULL).
 *   coeff_dbg      : NULL, or device fp32 [sum(n_new)][Hkv][2][r_max]: the projection c_j
 *                    (j < r_t; entries past r_t are not written) that the stored bf16
 *                    coefficients round, for checking steps 2-6 against a reference fed the
 *                    same c.  Calls with at most 4 tokens per sequence compute c as an fp32
 *                    fma chain over i = 0..d-1 from +0 (the fused decode step does too); larger
 *                    calls compute it on the tensor cores (bf16 products, fp32 accumulation in
 *                    the tensor core's order), within 1e-5 |x| of the exact projection.
 * Steps 2-6 (bf16 rounding, the residual against the stored coefficients as an fp32 fma
 * chain over j from +0, the top-s selection, scale and codes) are the same operations on
 * every path, so the stored bytes follow from c bit for bit.
 * The positions appended are [len, len + n_new[i]) where len is the sequence's current
 * length at this layer.  Capacity: len + n_new[i] <= max_context. */
dwkv_status dwkv_append(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                        const int32_t* n_new, const void* k_new, const void* v_new,
                        const uint8_t* tier_idx, float* coeff_dbg, void* stream);

/* dwkv_append with the residual gate of [DW] §3 Eq. (1) (X^ = A B + g R, g in [0, 1]) folded
 * into the dequantisation: the token's residual is quantised as in dwkv_append and its stored
 * fp16 scale is fp16_rn(g * scale) (an fp32 product), so decode and probe reconstruct g R.
 *   gate : device fp32 [sum(n_new)][Hkv][2] (K at [..][0], V at [..][1]), 4-byte aligned,
 *          non-NULL; values are used as given.
 * The fused decode step (dwkv_append_decode_attention) appends with g = 1; a re-tiered or
 * re-projected token is re-encoded from its reconstruction (which includes g R) with g = 1. */
dwkv_status dwkv_append_gated(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                              const int32_t* n_new, const void* k_new, const void* v_new,
                              const uint8_t* tier_idx, const float* gate, float* coeff_dbg, void* stream);

/* Appends tokens that are already in compressed form (import of a prepared cache).
 * Same sequence / position rules as dwkv_append.  Device arrays, tokens in list order,
 * K at [..][0][..] and V at [..][1][..]:
 *   coeff  [sum(n_new)][Hkv][2] coefficient records (entries at j >= r_t are ignored):
 *          bf16 [r_max] (coeff_bits 16), or with coeff_bits 8 r_max + r_max/8 bytes,
 *          int8 codes [r_max] then fp16 block scales [r_max/16] (2-byte aligned)
 *   idx    uint8 [sum(n_new)][Hkv][2][s]       (each < head_dim)
 *   codes  int8  [sum(n_new)][Hkv][2][s]       (int4 caches: each in [-8, 7])
 *   scales fp16  [sum(n_new)][Hkv][2] */
dwkv_status dwkv_append_compressed(dwkv_handle h, int32_t layer, int32_t n_seqs,
                                   const int32_t* seq_ids, const int32_t* n_new,
                                   const uint8_t* tier_idx, const void* coeff,
                                   const uint8_t* idx, const int8_t* codes, const void* scales,
                                   void* stream);

/* Decode attention at `layer` for one query token per listed sequence, over every token
 * the sequence holds at that layer ([DW] §3 Eq. (1) inside softmax attention).
 *   seq_ids   : host int32 [n_seqs], distinct
 *   q         : device bf16 [n_seqs][Hq][head_dim]
 *   out       : device fp32 [n_seqs][Hq][head_dim]; an empty sequence gives zeros
 *   workspace : device, 16-byte aligned, >= dwkv_workspace_bytes(cfg, n_seqs) bytes (half of
 *               that suffices for decode, see dwkv_workspace_bytes)
 * Every layer of a group must hold the same positions when one of them is decoded
 * (append each layer of the group before decoding it). */
dwkv_status dwkv_decode_attention(dwkv_handle h, int32_t layer, int32_t n_seqs,
                                  const int32_t* seq_ids, const void* q, float* out,
                                  void* workspace, size_t ws_bytes, void* stream);

/* One decode step of `layer` in a single launch: appends one new token to each listed
 * sequence (exactly as dwkv_append with n_new = 1 each: same placement, same stored bytes)
 * and runs dwkv_decode_attention over every token the sequence then holds, the new one
 * included ([DW] §3: the new token is compressed with the current basis, then attended
 * through Eq. (1) with the rest).  Arguments as dwkv_append and dwkv_decode_attention:
 *   k_new, v_new : device bf16 [n_seqs][Hkv][head_dim]
 *   tier_idx     : device uint8 [n_seqs][Hkv]; read where this layer is the group's first
 *                  to append the position, else may be NULL
 *   q, out, workspace as dwkv_decode_attention.
 * Same errors as the two calls.  When a tuning cap leaves the page ring too small for the
 * launch to stage both bases, it runs the two calls instead (same results). */
dwkv_status dwkv_append_decode_attention(dwkv_handle h, int32_t layer, int32_t n_seqs,
                                         const int32_t* seq_ids, const void* k_new,
                                         const void* v_new, const uint8_t* tier_idx,
                                         const void* q, float* out, void* workspace,
                                         size_t ws_bytes, void* stream);

/* Probe ([DW] §3 Eq. (3), two caches read as with / without the residual) in one pass
 * over the cache.  err: device fp32 [n_seqs][Hkv].  out_full: NULL or device fp32
 * [n_seqs][Hq][head_dim] (the decode output).  Other arguments as decode. */
dwkv_status dwkv_probe(dwkv_handle h, int32_t layer, int32_t n_seqs, const int32_t* seq_ids,
                       const void* q, float* err, float* out_full, void* workspace,
                       size_t ws_bytes, void* stream);

/* Moves stored tokens to other rank tiers ([DW] §3, Eq. (2)-(3) paragraphs: the probe's
 * feedback lowers or raises the router threshold tau_m of a depth window, which changes the
 * rank level its tokens are kept at).  For each listed sequence i, its n_tok[i] positions
 * (device int32 positions[], sequences in list order, distinct within a sequence) and every
 * kv-head h, the token takes tier new_tier[t][h] (device uint8 [sum(n_tok)][Hkv], an index
 * into cfg.tiers) in every layer of `group`, keys and values:
 *   - a token already at its new tier is left as it is;
 *   - otherwise it is re-encoded at the new rank from its reconstruction (Eq. (1), g = 1),
 *     since the dense vector is not kept: a_i = fp32 fma chain over j < r_old of
 *     B[i][j] * c_j from +0 (c_j the stored bf16 coefficient, or with coeff_bits 8 its
 *     code * block scale, exact in fp32), plus scale * code on its residual channels,
 *     rounded to bf16, then the encode steps of dwkv_append; the stored bytes equal
 *     dwkv_append's for that bf16 vector.
 * Every layer of the group must hold the same positions (call between decode steps, not
 * between the layers of one step); DWKV_ERR_INVALID_ARG otherwise.  Positions the group has
 * not placed, or tier indices >= num_tiers, set a device error (DWKV_DEV_NO_SLOT,
 * DWKV_DEV_BAD_TIER) and are skipped.  Decoding after the call sees the new tiers; the
 * sequence's length is unchanged.  Pages a tier empties return to that tier's free ring and
 * serve that tier's later placements; an arena sized by dwkv_arena_bytes_all_tiers has room
 * for any sequence of moves (dwkv_arena_bytes assumes tokens keep their tier). */
dwkv_status dwkv_retier(dwkv_handle h, int32_t group, int32_t n_seqs, const int32_t* seq_ids,
                        const int32_t* n_tok, const int32_t* positions, const uint8_t* new_tier,
                        void* stream);

/* Probe-driven threshold of the router, per depth window ([DW] §3, Eq. (2) and the Eq. (3)
 * paragraph).  Host code only; it holds no device state.
 *  - dwkv_tier_controller_due(c, step): 1 when decode step `step` (>= 0) is a probe step
 *    (every probe_every steps, step 0 included), else 0.
 *  - dwkv_tier_controller_observe(c, group, err, &lowered): one probe interval's result for
 *    the group, err = the largest probe error (dwkv_probe) over its layers and kv-heads.  If
 *    err > tol: tau = max(tau_min, tau - tau_step_down), the quiet count restarts and
 *    *lowered = 1 (the caller may then promote stored tokens, dwkv_retier).  Otherwise the
 *    quiet count grows; when it reaches quiet_intervals, tau = min(tau_max, tau + tau_step_up)
 *    and the count restarts.  NaN err: DWKV_ERR_INVALID_ARG.
 *  - dwkv_tier_controller_route(c, group, n, salience, base_tier, high_tier, tier_out): the
 *    router's two-level rule with the group's current threshold, on host arrays of n tokens:
 *    tier_out[t] = high_tier if salience[t] > tau and base_tier[t] < high_tier, else
 *    base_tier[t].  The salience scores (the router's sigma(u^T phi)) are the caller's.
 *  - dwkv_tier_controller_threshold(c, group, &tau): the group's current threshold. */
typedef struct {
    float tol;                 /* probe error above which tau is lowered                    */
    float tau_init, tau_min, tau_max;
    float tau_step_down, tau_step_up;
    int32_t quiet_intervals;   /* probes in a row at or below tol before tau rises (>= 1)   */
    int32_t probe_every;       /* decode steps between probes (>= 1)                        */
} dwkv_tier_policy;
typedef struct dwkv_tier_ctrl* dwkv_tier_controller;
dwkv_status dwkv_tier_controller_create(const dwkv_tier_policy* policy, int32_t num_groups,
                                        dwkv_tier_controller* out);
dwkv_status dwkv_tier_controller_destroy(dwkv_tier_controller c);
int32_t dwkv_tier_controller_due(dwkv_tier_controller c, int64_t step);
dwkv_status dwkv_tier_controller_threshold(dwkv_tier_controller c, int32_t group, float* tau);
dwkv_status dwkv_tier_controller_observe(dwkv_tier_controller c, int32_t group, float err,
                                         int32_t* lowered);
dwkv_status dwkv_tier_controller_route(dwkv_tier_controller c, int32_t group, int32_t n,
                                       const float* salience, const uint8_t* base_tier,
                                       int32_t high_tier, uint8_t* tier_out);

/* Reads positions [t0, t0 + n) of (layer, seq) back in token order, as stored:
 *   tier_idx uint8 [n][Hkv]; coeff [n][Hkv][2] coefficient records as in
 *   dwkv_append_compressed (zeros at j >= r_t);
 *   idx uint8 [n][Hkv][2][s]; codes int8 [n][Hkv][2][s]; scales fp16 [n][Hkv][2].
 * All device pointers; any of them may be NULL to skip that array. */
dwkv_status dwkv_export(dwkv_handle h, int32_t layer, int32_t seq, int32_t t0, int32_t n,
                        uint8_t* tier_idx, void* coeff, uint8_t* idx, int8_t* codes,
                        void* scales, void* stream);

/* Pool usage, read synchronously (the stream is synchronised first). */
typedef struct {
    uint64_t data_bytes_total;     /* page pool size                                    */
    uint64_t data_bytes_reserved;  /* bytes ever handed out from the pool               */
    uint32_t free_pages[DWKV_MAX_TIERS]; /* pages waiting in each tier's free ring     */
} dwkv_pool_stats;
dwkv_status dwkv_pool_usage(dwkv_handle h, void* stream, dwkv_pool_stats* out);

/* Synchronises `stream`, then returns DWKV_ERR_DEVICE_CHECK if a kernel recorded an
 * error since the last call (the message names it; the word is then cleared), or
 * DWKV_ERR_CUDA if the stream reported a CUDA error. */
dwkv_status dwkv_sync_status(dwkv_handle h, void* stream);

/* Launch tuning (for measurement sweeps): decode CTAs per SM (1 in this build: one
 * 13-warp CTA fills an SM's registers), split waves per decode (1..8) and a cap on the
 * CTA's page ring in units of the largest page chunk (0 = all the shared memory the other
 * regions leave, else 2..32).  Returns DWKV_ERR_INVALID_ARG for values out of range or a
 * ring that cannot hold two chunks. */
dwkv_status dwkv_set_decode_tuning(dwkv_handle h, int32_t ctas_per_sm, int32_t waves,
                                   int32_t stages);

/* Launch overlap of decode and probe (enable 1, the default, or 0).  With it, each launch
 * may start while the previous kernel of its stream still runs: its CTAs take the SMs that
 * kernel leaves, set up and start streaming their pages, and wait for that kernel to
 * complete before they read q, the new token or the tier indices, or write anything.  The
 * cache state they read early is read only once its tier counts show that no earlier
 * decode's placement is still in flight.  Results are the same either way; 0 serialises
 * the launches (for measurement).  DWKV_ERR_INVALID_ARG for other values. */
dwkv_status dwkv_set_decode_overlap(dwkv_handle h, int32_t enable);

/* Decode attention without any caller-provided or library-allocated memory: the same
 * operation as dwkv_decode_attention, but its split-K scratch is a fixed 8 MiB array built
 * into the library (held by every GPU that loads the library until the process exits).
 * There is no counterpart in [DW]; it exists for callers that cannot allocate device memory
 * when they decode (engine plugin hooks, serving loops whose memory pool owns all of HBM) and
 * have no workspace to lend.  Arguments as dwkv_decode_attention without the workspace.
 *  - Calls nothing that allocates (no cudaMalloc / cudaFree).
 *  - Returns DWKV_ERR_CAPACITY when the call's split-K records, n_seqs * Hkv * 64 records of
 *    (8 + 4 * head_dim) floats, exceed 8 MiB (for 8 kv-heads and head_dim 128: up to 7
 *    sequences per call).
 *  - The first call on a device resolves the scratch array's device address (one
 *    cudaGetSymbolAddress); make that first call before any stream capture.  The handle's
 *    device must be current.
 *  - All calls on a device share the one array: calls that overlap on the GPU (other
 *    streams, other handles) race on it.  Nothing in it needs clearing between calls. */
dwkv_status dwkv_decode_attention_noalloc(dwkv_handle h, int32_t layer, int32_t n_seqs,
                                          const int32_t* seq_ids, const void* q, float* out,
                                          void* stream);

/* Test support for the kernels' bounded waits (every wait on a barrier, flag or copy gives up
 * after a time limit, records DWKV_DEV_TIMEOUT in the handle's device error word and returns):
 * launches one thread that waits on a shared-memory barrier nothing arrives at, through the
 * same bounded-wait routine, with a limit of limit_us microseconds (1..2,000,000).  The wait
 * runs out and the kernel returns; the context stays usable, and dwkv_sync_status then reports
 * DWKV_ERR_DEVICE_CHECK ("bounded wait timed out") and clears the word. */
dwkv_status dwkv_check_bounded_wait(dwkv_handle h, uint32_t limit_us, void* stream);

/* Test support: encode steps 4-6 on given residuals ([DW] §3: the residual is kept only on the
 * routed channels, quantised), through the same device code the encoders use.  For each of n
 * vectors: the s channels with the largest |r_i| (ties to the lower channel) in ascending
 * channel order, the fp16 scale round(max |r_sel| / qmax) (qmax 127 or 7) and the codes
 * clamp(rint(r_i / scale), -qmax, qmax) (all 0 when the scale is 0).
 *   r      : device fp32 [n][head_dim] (head_dim = 128)
 *   s      : 0..128, a multiple of 8;  bits : 8 or 4
 *   idx    : device uint8 [n][s];  codes : device int8 [n][s] (one code per byte, int4 too)
 *   scales : device fp16 bits [n]
 *   work   : device scratch of at least dwkv_quantize_work_bytes(n, s, bits) bytes
 * DWKV_ERR_INVALID_ARG for arguments out of range or NULL pointers (n > 0 and s > 0). */
size_t dwkv_quantize_work_bytes(int32_t n, int32_t s, int32_t bits);
dwkv_status dwkv_quantize_residuals(int32_t n, int32_t s, int32_t bits, const float* r, uint8_t* idx,
                                    int8_t* codes, uint16_t* scales, void* work, size_t work_bytes,
                                    void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DWKV_H */
