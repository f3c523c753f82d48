/*
 * patch.h -- C ABI of the B200 (sm_100a) tile-hybrid sparse linear layer.
 *
 * A weight matrix W[N,K] is cut into tile_n x tile_k tiles.  A per-tile map
 * marks each tile dense or 2:4-sparse, so the overall sparsity is anywhere
 * between 0% and 50% ("PATCH: Learnable Tile-level Hybrid Sparsity for LLMs",
 * section 2, core mechanism).  Inside a 2:4 tile every group of 4 consecutive
 * input channels keeps the 2 weights with the highest Wanda score
 * |W_ij| * ||X_:,j||_2 over calibration tokens ("SparseGPT vs Wanda: one-shot
 * LLM pruning without retraining", section on Wanda), ties going to the lower
 * index.  The product Y = X * W_eff^T then runs as one kernel over the mixed
 * tiles (PATCH page, section 2, inference and deployment: dense tiles on the
 * dense tensor-core path, 2:4 tiles on the sparse one).
 *
 * Conventions for every call:
 *   - All array pointers are DEVICE pointers on the current CUDA device,
 *     unless a comment says otherwise.  The caller owns them.
 *   - bf16 arrays are row-major with the last index contiguous.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued on it; no call synchronises the host except
 *     where its comment says so.
 *   - Errors are returned, never thrown.  An asynchronous kernel fault
 *     surfaces as PATCH_ERR_CUDA on a later call.  Calls on different
 *     handles may run concurrently; calls on one handle must not.
 *
 * Layouts:
 *   meta  uint32 [N, K/32]: group g of row i (columns 4g..4g+3) is the 4-bit
 *         code idx0 | (idx1 << 2) of its two kept positions (idx0 < idx1), at
 *         bits 4*(g%8) of word [i, g/8].  Codes are written for every group,
 *         dense tiles included (dense tiles simply ignore them).
 *   map   uint32 [ceil(n_tiles/32)]: tile t = (i/tile_n)*(K/tile_k) + j/tile_k
 *         is 2:4 iff bit t%32 of word t/32 is 1.  Unused high bits are 0.
 *   colsq fp64 [K]: s_j = sum_t x_tj^2 over calibration tokens, added in a
 *         fixed order: chunks of 128 consecutive tokens, each summed token
 *         by token from 0.0, then the chunk sums added chunk by chunk from
 *         0.0.  The result is therefore bit-reproducible.
 *   tile_loss fp64 [n_tiles]: Wanda score removed by 2:4 pruning of the tile,
 *         added in a fixed order: inside each 32-column word of a row the
 *         pruned scores left to right; the row's words left to right; the
 *         tile's row sums as a balanced binary tree ((0,1), (2,3), ..., then
 *         pairs of those, ...).
 */
#ifndef PATCH_B200_H
#define PATCH_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PATCH_OK = 0,
    PATCH_ERR_INVALID_ARG = 1, /* null pointer, misalignment, bad shape     */
    PATCH_ERR_UNSUPPORTED = 2, /* tile size not in {64,128}, not sm_100     */
    PATCH_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed          */
    PATCH_ERR_OOM = 4,         /* device allocation failed                   */
    PATCH_ERR_TIMEOUT = 5      /* a bounded device wait ran out (see below)  */
} patch_status;

typedef struct {
    int64_t N;      /* output features (rows of W)                          */
    int64_t K;      /* input features (columns of W)                        */
    int32_t tile_n; /* tile rows, 64 or 128                                 */
    int32_t tile_k; /* tile columns, 64 or 128                              */
} patch_shape;

/* Opaque packed weight, owned by the library (patch_pack / patch_free). */
typedef struct patch_packed patch_packed;

/*
 * Wanda 2:4 mask builder and tile map.
 *
 * Follows the Wanda criterion (SparseGPT-vs-Wanda page, section on Wanda:
 * weight magnitude times the activation of its input channel, lowest
 * pruned) restricted to 2:4 groups (PATCH page, section 1: semi-structured
 * 2:4, two nonzeros per four; section 2: one of six patterns per group),
 * plus the per-tile dense / 2:4 decision (PATCH page, section 2, core
 * mechanism).  PATCH learns that decision; this call either takes it from
 * `map_in` or, when `map_in` is NULL, marks as 2:4 the floor(f * n_tiles)
 * tiles of least tile_loss (ties to the lower tile index).
 *
 *   W_bf16      [N,K] bf16, 16-byte aligned.
 *   Xcal_bf16   [T,K] bf16 calibration activations, 16-byte aligned; may be
 *               NULL when colsq_in is given.
 *   T           calibration tokens (>= 1 when Xcal_bf16 is used).
 *   colsq_in    optional [K] fp64 sums of squares to reuse (matrices that
 *               share an input, e.g. q/k/v); NULL = compute from Xcal.
 *   shp         N % tile_n == 0, K % tile_k == 0; tiles in {64,128}.
 *   sparse_tile_fraction  f in [0,1], used only when map_in is NULL.
 *   map_in      optional caller map (copied to map_out).
 *   meta_out    [N, K/32] uint32 (written).
 *   map_out     [ceil(n_tiles/32)] uint32 (written).
 *   colsq_out   optional [K] fp64 (written when non-NULL).
 *   tile_loss_out optional [n_tiles] fp64 (written when non-NULL).
 *
 * Temporary device memory (chunk partials of the column sums, 8*K*ceil(T/128)
 * bytes, plus 8*K bytes of norms) is taken from the stream-ordered pool and
 * released on the same stream.  Errors: INVALID_ARG for null/misaligned
 * pointers or bad shapes; UNSUPPORTED for other tile sizes; OOM; CUDA.
 */
patch_status patch_score_mask(const void *W_bf16, const void *Xcal_bf16, int64_t T,
                              const double *colsq_in, patch_shape shp,
                              double sparse_tile_fraction, const uint32_t *map_in,
                              uint32_t *meta_out, uint32_t *map_out, double *colsq_out,
                              double *tile_loss_out, void *stream);

/*
 * The mask builder for another N:M pattern ("PATCH: Learnable Tile-level
 * Hybrid Sparsity for LLMs", section 5, significance: the tile scheme is not
 * tied to 2:4 and extends to patterns such as 4:8).  (n_keep, m_group) =
 * (2, 4) is exactly patch_score_mask; (4, 8): inside a sparse tile every
 * group of 8 consecutive input channels keeps the 4 weights with the highest
 * Wanda score (ties to the lower index).  Arguments, outputs, tile loss order
 * and map rule as patch_score_mask, except the codes:
 *   meta [N, K/32] uint32: group g of row i (columns 8g..8g+7) is an 8-bit
 *        keep mask (bit q set for a kept position q; four bits set) at bits
 *        8*(g%4) of word [i, g/4].
 * Errors as patch_score_mask; PATCH_ERR_UNSUPPORTED for other (n, m).
 */
patch_status patch_score_mask_nm(const void *W_bf16, const void *Xcal_bf16, int64_t T,
                                 const double *colsq_in, patch_shape shp, int32_t n_keep,
                                 int32_t m_group, double sparse_tile_fraction, const uint32_t *map_in,
                                 uint32_t *meta_out, uint32_t *map_out, double *colsq_out,
                                 double *tile_loss_out, void *stream);

/*
 * Column sums of squares of calibration activations alone: the activation
 * term of the Wanda score (SparseGPT-vs-Wanda page, section on Wanda: the
 * weight magnitude is weighed by the input activation of its channel; here
 * ||X_:,j||_2^2 over the calibration tokens).  colsq_out [K] fp64 receives
 * exactly what patch_score_mask writes to colsq_out for the same Xcal (the
 * fixed order above), ready for its colsq_in: one call per distinct layer
 * input, shared by the matrices that read it.
 *   Xcal_bf16 [T,K] bf16, 16-byte aligned; T >= 1; K a multiple of 64.
 * Scratch (8*K*ceil(T/128) bytes of chunk partials) comes from the library's
 * pool, released on the stream.  Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA.
 */
patch_status patch_colsq(const void *Xcal_bf16, int64_t T, int64_t K, double *colsq_out,
                         void *stream);

/*
 * The two halves of patch_colsq, for callers that hold the calibration tokens
 * in pieces (e.g. one piece per GPU, each a multiple of 128 tokens except the
 * last).
 *   patch_colsq_partials: partials_out [ceil(T/128), K] fp64 (16-byte
 *     aligned, written): row c is the sum of x_tj^2 over tokens 128c ..
 *     128c+127 of this Xcal, added token by token from 0.0.
 *   patch_colsq_fold: colsq_out[j] = the rows of partials [chunks, K]
 *     (16-byte aligned) added row by row from 0.0.
 * The partials of consecutive pieces, stacked in token order and folded, give
 * bit for bit patch_colsq's result for the whole set.  No scratch.  Errors:
 * INVALID_ARG (null pointers, T or chunks < 1, K not a multiple of 64,
 * misalignment), UNSUPPORTED, CUDA.
 */
patch_status patch_colsq_partials(const void *Xcal_bf16, int64_t T, int64_t K,
                                  double *partials_out, void *stream);
patch_status patch_colsq_fold(const double *partials, int64_t chunks, int64_t K, double *colsq_out,
                              void *stream);

/*
 * Allocation-free variant of patch_score_mask.  The pages have no
 * counterpart: this entry point exists for callers that may not allocate
 * device memory at all, e.g. code running inside a framework whose caching
 * allocator owns the whole GPU (a cudaMalloc behind its back would fail or
 * fragment its pool), embedded runtimes that reserve every byte up front, or
 * paths with hard latency limits where an allocation (which can synchronise
 * the device) is not allowed.
 *
 * Same arguments, outputs and results as patch_score_mask.  The temporary
 * values (chunk partials of the column sums, norms, and the loss / rank
 * counters when the caller does not ask for them) live in one fixed array of
 * device memory inside this library, 16 MiB per device
 * (patch_score_mask_noalloc_capacity()), held on each device from the first
 * call there (see Set-up) until the process exits.  A call needs
 * 8*K*ceil(T/128) + 8*K + 8*n_tiles + 4*n_tiles bytes of it (plus alignment;
 * the last two terms only when tile_loss_out is NULL / map_in is NULL);
 * larger problems return PATCH_ERR_UNSUPPORTED without launching anything.
 * It calls no cudaMalloc / cudaFree / pool allocation.
 *
 * All calls on a device share the array and it keeps what the last call left
 * in it; each call writes every value before reading it.  Calls whose GPU
 * work overlaps (different streams without ordering between them) race on the
 * array and give wrong results: order them on one stream or with events.
 *
 * Set-up.  The array's device address belongs to a CUDA context; the first
 * call in each context looks it up (cudaGetSymbolAddress, with the device
 * current) and caches it under the context's id, so a device reset or a new
 * primary context is looked up afresh.  Under lazy module loading (the CUDA
 * default) that first lookup is also what loads this library's module on
 * the device, i.e. when the 16 MiB are reserved: a caller whose allocator
 * takes the GPU's memory up front should make one call (any small problem)
 * at initialisation, before that reservation and before any stream capture.
 */
patch_status patch_score_mask_noalloc(const void *W_bf16, const void *Xcal_bf16, int64_t T,
                                      const double *colsq_in, patch_shape shp,
                                      double sparse_tile_fraction, const uint32_t *map_in,
                                      uint32_t *meta_out, uint32_t *map_out, double *colsq_out,
                                      double *tile_loss_out, void *stream);

/* Bytes of the fixed scratch array patch_score_mask_noalloc works in. */
size_t patch_score_mask_noalloc_capacity(void);

/*
 * Diagnostics: bytes of the library's stream-ordered device pool (current
 * device) in use now, and the high-water mark of that use.  reset_high != 0
 * first restarts the mark from the current use, so a later reading above
 * `used_now` shows that something took pool memory in between.  Host
 * pointers, either may be NULL.  No device work.  Errors: CUDA.
 */
patch_status patch_pool_usage(uint64_t *used_now, uint64_t *used_high, int32_t reset_high);

/*
 * Global tile allocation over several matrices of one block (the ablation in
 * section 4 of "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs": a
 * single sparsity target for the block, which lets each layer's share vary,
 * beats the same target in every layer).  The pages learn the allocation by
 * training; this is its data-free stand-in with Wanda tile losses: of all the
 * tiles of the `count` matrices, the floor(fraction * total) with the least
 * pruned-score loss become 2:4.  Ties in loss go to the lower global index,
 * where the matrices are taken in the order given (tile t of matrix m has
 * index n_tiles[0] + ... + n_tiles[m-1] + t).
 *
 * losses[m]   DEVICE fp64 [n_tiles[m]]: matrix m's tile losses, as written by
 *             patch_score_mask's tile_loss_out (the caller owns them).
 * n_tiles[m]  HOST: tile count of matrix m (>= 1).
 * count       1..64 matrices.  With count = 1 the result equals the map
 *             patch_score_mask selects for the same fraction.
 * fraction    0..1 of ALL tiles.
 * maps_out[m] DEVICE uint32 [ceil(n_tiles[m] / 32)]: matrix m's bitmap (bit
 *             t % 32 of word t / 32 set for a 2:4 tile), for patch_score_mask's
 *             map_in and patch_pack.
 * Stream-ordered on `stream`; scratch comes from the library's pool.
 * Errors: PATCH_ERR_INVALID_ARG for null pointers, count outside 1..64, a
 * zero tile count or fraction outside [0, 1]; PATCH_ERR_UNSUPPORTED above
 * 65535 * 256 tiles in all.
 */
patch_status patch_select_maps_global(const double *const *losses, const int64_t *n_tiles,
                                      int32_t count, double fraction, uint32_t *const *maps_out,
                                      void *stream);

/*
 * Compressor: lay the dense tiles and the 2:4-compressed tiles (kept values +
 * metadata) out for the hybrid GEMM.  Compressed storage is what turns
 * zeros into speed (SparseGPT-vs-Wanda page, section on structured vs
 * unstructured sparsity); the layout is this library's own.
 *
 *   W_bf16  [N,K] bf16 (16-byte aligned); meta, map as produced above.
 *   shp     as above, and additionally N % 128 == 0, K % 128 == 0 and
 *           K <= 28672.
 *   out     receives the new handle (host pointer to a library object).
 *   packed_bytes  optional host pointer: compressed weight bytes (values +
 *           metadata, excluding the k-step table).
 *
 * Packed format (normative).  Geometry: bands of 128 rows, k-steps of 64
 * columns, k-pairs of 128 columns.
 *   - k-step (band b, step c) is stored 2:4-compressed iff every map tile
 *     overlapping rows [128b,128b+128) x cols [64c,64c+64) is 2:4; otherwise
 *     dense, holding W_eff (W with pruned entries of 2:4 tiles set to +0).
 *   - bands one after another; inside a band, k-steps in order.
 *   - dense k-step: 16384 bytes; element (r,k), r<128, k<64, at byte
 *     (r/8)*1024 + (r%8)*128 + ((k/8) ^ (r%8))*16 + (k%8)*2
 *     (the tensor-core K-major 128-byte-swizzled layout).
 *   - 2:4 k-step: 8192 bytes of kept values; kept value v (v<32, column
 *     order, two per group) of row r at byte
 *     (r/8)*512 + (r%8)*64 + ((v/8) ^ ((r%8)/2))*16 + (v%8)*2
 *     (K-major 64-byte-swizzled).
 *   - metadata block: 2048 bytes per (band, k-pair) holding at least one 2:4
 *     k-step, placed right before the values of the pair's first 2:4
 *     k-step.  Row m = m0+8*m1+16*m2 (m0<8,m1<2,m2<8), pair column
 *     k = k0+16*k1+32*k2 (k0<16,k1<2,k2<4): the code bit of column k is in
 *     16-byte line m0+8*k1+16*m2 at bit 32*k2+16*m1+k0 (a group's 4-bit code
 *     over its four columns, least significant bit first).  Bits of a dense
 *     k-step are 0.  This is the tensor-memory metadata layout of the
 *     sm_100 sparse MMA for 16-bit inputs, one 16-byte line per TMEM lane.
 *   - table[b*(K/64)+c] (uint64): bits 0..47 byte offset of the k-step's
 *     data, bit 62 = 2:4, bit 63 = the pair's metadata block precedes it.
 *
 * Synchronises the stream once: the layout is planned on the device from the
 * map (k-step table and decode chunk descriptors written there), and only a
 * small summary (total bytes, the first chunk descriptors) and the per-band
 * k-pair byte prefix (the prefill kernels' work balance) are read back, in
 * that one wait, to size the packed allocation exactly.
 * Errors: INVALID_ARG, UNSUPPORTED, OOM, CUDA.
 */
patch_status patch_pack(const void *W_bf16, const uint32_t *meta, const uint32_t *map,
                        patch_shape shp, patch_packed **out, size_t *packed_bytes,
                        void *stream);

/*
 * patch_pack for several matrices with ONE wait (no counterpart on the pages:
 * the compressor above, batched).  Matrix i is (Ws_bf16[i], metas[i],
 * maps[i], shps[i]), each under patch_pack's preconditions; shapes may
 * differ.  Every layout is planned in one launch (a block per matrix), the
 * plan summaries and k-pair prefixes are read back in one wait of `stream`,
 * then every packed buffer is allocated and packed.  Each outs[i] is then
 * exactly the handle patch_pack would give for matrix i (the same packed
 * bytes and tables).
 *   count         1..8.
 *   outs          count handle slots (host array); all null on any error.
 *   packed_bytes  optional host array of count: compressed bytes per handle.
 * Errors: as patch_pack, for any member (every member's arguments are
 * checked before anything is allocated); on an error no handle is left.
 */
patch_status patch_pack_group(const void *const *Ws_bf16, const uint32_t *const *metas,
                              const uint32_t *const *maps, const patch_shape *shps, int32_t count,
                              patch_packed **outs, size_t *packed_bytes, void *stream);

/*
 * Compressor for another N:M pattern (see patch_score_mask_nm).  (2, 4) is
 * exactly patch_pack.  (4, 8): the 4:8 handle's packed format (normative):
 *   - bands of 128 rows, k-steps of 64 columns; a k-step is 4:8-compressed
 *     iff every map tile overlapping it is 4:8, otherwise dense (the dense
 *     layout above, holding W_eff: pruned entries of 4:8 tiles +0);
 *   - 4:8 k-step: 9216 bytes: kept value v (v < 32, column order, four per
 *     group of 8) of row r at byte r*64 + v*2; the keep mask of group g
 *     (g < 8) of row r at byte 8192 + r*8 + g;
 *   - table[b*(K/64)+c] (uint64): bits 0..47 byte offset; bit 60 = 4:8.
 * The tensor cores have no 4:8 mode for 16-bit inputs: patch_hybrid_gemm on
 * a 4:8 handle expands each 4:8 k-step in shared memory into the dense tile
 * and issues dense MMAs (the compressed bytes are what it reads from memory).
 * Errors as patch_pack; PATCH_ERR_UNSUPPORTED for other (n, m).
 */
patch_status patch_pack_nm(const void *W_bf16, const uint32_t *meta, const uint32_t *map,
                           patch_shape shp, int32_t n_keep, int32_t m_group, patch_packed **out,
                           size_t *packed_bytes, void *stream);

/*
 * FP8 values inside dense and 2:4 tiles ("SparseGPT vs Wanda: one-shot LLM
 * pruning without retraining", FAQ: pruning combines with quantisation,
 * prune first, then quantise).  The Wanda 2:4 codes and the tile map come
 * from patch_score_mask as for bf16; W_eff is then quantised to e4m3 with one
 * fp32 scale per output row, and patch_hybrid_gemm on the handle quantises X
 * with one fp32 scale per token (each call: into the handle's own scratch for
 * M <= 64, else into pool scratch of M*K + 4*M bytes) and computes
 *     Y[m,n] = sx[m] * sw[n] * sum_k dec(qx[m,k]) * dec(qw[n,k])
 * on the tensor cores (tcgen05 kind::f8f6f4: dense MMAs for dense k-steps,
 * the sparse MMA for 2:4 k-steps), fp32 accumulation, one rounding.  M <= 64
 * with an even number of 128-column k-steps runs the split-K configuration
 * (chunk partials added in a fixed order, scales applied at the end); the
 * handle then also holds the chunk descriptors and partial slots.
 * Quantisation of a row: s = amax / 448 in fp32 (1 for an all-zero row);
 * q = e4m3(x / s) with the quotient in fp32, rounded to nearest with ties to
 * the even code, saturating at +-448.
 *
 * patch_pack_fp8: W_bf16, meta, map, shp as patch_pack (K a multiple of 128).
 * Synchronises once (it reads the map back to plan the layout).  Packed
 * format (normative): bands of 128 rows, k-steps of 128 columns; a k-step is
 * 2:4 iff every map tile overlapping it is 2:4, otherwise dense (codes of
 * W_eff);
 *   - dense k-step: 16384 bytes, code (r,k) at
 *     (r/8)*1024 + (r%8)*128 + ((k/16) ^ (r%8))*16 + k%16;
 *   - 2:4 k-step: a 2048-byte metadata block (16-byte line m holds row m's
 *     code bits, bit k = bit k%4 of the 4-bit code of column group k/4: the
 *     row's four meta words for these columns), then 8192 bytes of kept
 *     codes, kept code v (v < 64, column order) of row r at
 *     (r/8)*512 + (r%8)*64 + ((v/16) ^ ((r%8)/2))*16 + v%16;
 *   - table[b*(K/128)+c] (uint64): bits 0..47 offset of the k-step's codes,
 *     bit 62 = 2:4.
 * With an even band count the handle also holds a prefill table for the
 * two-SM kernel (not exported): bands 2p and 2p+1 take one kind at every
 * k-step, a 2:4 k-step whose partner band's is dense pointing to a dense
 * side copy of its W_eff codes (16384 bytes each, after the packed bytes).
 * Errors as patch_pack.
 */
patch_status patch_pack_fp8(const void *W_bf16, const uint32_t *meta, const uint32_t *map,
                            patch_shape shp, patch_packed **out, size_t *packed_bytes,
                            void *stream);

/*
 * The per-row e4m3 quantisation above, on its own: X_bf16 [R,C] (16-byte
 * aligned, C a multiple of 8) -> codes_out [R,C] uint8 (8-byte aligned) and
 * scales_out [R] fp32.  Stream-ordered, no scratch.  Errors: INVALID_ARG,
 * UNSUPPORTED, CUDA.
 */
patch_status patch_quantize_fp8(const void *X_bf16, int64_t R, int64_t C, uint8_t *codes_out,
                                float *scales_out, void *stream);

/* Copy an FP8 handle's W_eff row scales ([N] fp32) to scales_dst (device),
 * stream-ordered.  INVALID_ARG for other handles. */
patch_status patch_packed_fp8_scales(const patch_packed *Wp, float *scales_dst, void *stream);

/*
 * Hybrid product Y[M,N] = X[M,K] * W_eff^T with fp32 accumulation in tensor
 * memory and one rounding at the end (PATCH page, section 2, inference and
 * deployment: one kernel over mixed dense / 2:4 tiles).  Dense k-steps issue
 * the dense tcgen05 MMA, 2:4 k-steps the sparse tcgen05 MMA, into one
 * accumulator.  M <= 16, and M <= 64 where K <= 8192, run the split-K
 * configuration (the weights read once, spread over every SM, with 16-, 32-
 * or 64-token tiles and an in-order fix-up of the chunk partials); larger M
 * the prefill configuration.  The call only enqueues work: it never waits for the
 * device (everything it needs from the device was read back by patch_pack).
 *
 *   Wp      handle from patch_pack.
 *   X_bf16  [M,K] bf16, 16-byte aligned.
 *   M       tokens, >= 0 (any value; a ragged last token tile is masked;
 *           M == 0 returns PATCH_OK without touching X or Y).
 *   Y       [M,N]: bf16 (y_is_fp32 = 0) or fp32 (y_is_fp32 = 1), 16-byte
 *           aligned.
 *
 * Every device wait inside the kernel is bounded (2 s); a wait that runs out
 * sets the handle's status word and the kernel returns early (Y undefined);
 * while the word is set, later calls on the handle skip their work.
 * Errors: INVALID_ARG, CUDA; PATCH_ERR_TIMEOUT is reported by
 * patch_get_status, not here (the call does not synchronise).
 */
patch_status patch_hybrid_gemm(const patch_packed *Wp, const void *X_bf16, int64_t M, void *Y,
                               int32_t y_is_fp32, void *stream);

/*
 * Several hybrid products that read the same activations, in one launch:
 * Ys[i][M, N_i] = X[M, K] * W_eff_i^T for i < count, each exactly as
 * patch_hybrid_gemm computes it (bit for bit: the same chunks, added in the
 * same order).  The layers of a decoder block that share an input (q, k and
 * v; gate and up) are each one hybrid linear layer of the PATCH page
 * (section 2, inference and deployment); the pages say nothing about
 * launching them together.  This entry point exists because at decode token
 * counts a product is bound by reading its weights once, and the fixed cost
 * of a launch (its start, the first copies' latency, the tail and the fix-up)
 * weighs most on the smaller matrices: one launch over the group pays it
 * once and spreads all the group's chunks over every SM.
 *
 *   Wps     count (1..8) handles from patch_pack on the current device, all
 *           with the same K.
 *   X_bf16  [M,K] bf16, 16-byte aligned, the input of every product.
 *   M       tokens, >= 0 (M == 0 returns PATCH_OK without touching anything).
 *   Ys      count outputs, Ys[i] [M, N_i] bf16 or fp32 (y_is_fp32), 16-byte
 *           aligned, not overlapping one another or X.
 *
 * One launch is made when every handle is bf16 2:4 and M is in the split-K
 * range (M <= 16, or M <= 64 with K <= 8192), or when every handle is FP8
 * with an even number of 128-column k-steps and M <= 64 (X is then quantised
 * once, into the first handle's scratch), or, above 128 tokens, when every
 * handle is bf16 2:4 with an even band count and K <= 28672, or every handle
 * is FP8 with an even band count and an even number of 128-column k-steps
 * (at most 224; X quantised once, into a pool allocation of M*K + 4*M bytes
 * freed on the stream), and the library estimates one two-SM launch over all
 * their band pairs to finish no later than their own launches; otherwise
 * (mixed kinds, 4:8 handles, 64 < M <= 128) the products are enqueued one
 * after another, as count calls of patch_hybrid_gemm would.  In the split-K launches each output is
 * bit-identical to its single call; the grouped prefill launch may tile the
 * tokens differently from a single call, which changes fp32 rounding order
 * only.  Partial slots come from the library's
 * stream-ordered pool for the call; the first handle's claim counter serves
 * the launch, so calls that use a handle must not run concurrently on
 * different streams (the rule of patch_hybrid_gemm).  A wait that runs out
 * raises every handle's status word; a raised word on any handle makes the
 * whole launch skip its work.  The call never waits for the device.
 * Handles that cannot share a launch (another pattern or K) are not an
 * error: their products are enqueued one by one.  Errors: INVALID_ARG (null
 * pointers, count out of range, misalignment, y_is_fp32 not 0 / 1), CUDA.
 */
patch_status patch_hybrid_gemm_group(const patch_packed *const *Wps, int32_t count, const void *X_bf16,
                                     int64_t M, void *const *Ys, int32_t y_is_fp32, void *stream);

/*
 * Failure-detection test hook: while `on` is non-zero, the first CTA of every
 * later patch_hybrid_gemm never loads its first k-step, so that CTA's bounded
 * wait runs out on purpose and patch_get_status reports PATCH_ERR_TIMEOUT.
 * Off by default (the environment variable PATCH_B200_TEST_STALL=1, read once
 * when the library loads, turns it on from the start).  Tests only.
 */
void patch_test_stall_first_kstep(int32_t on);

/*
 * Test hook: the prefill kernel every later patch_hybrid_gemm with M > 16
 * uses.  0 = chosen by the library (the default), 1 = one band per CTA
 * (64-token tiles up to M = 64),
 * 2 = two bands per CTA sharing each token tile, 3 = two-SM (CTA pair)
 * kernel, 4 = two-SM kernel with two bands per SM; 3 and 4 only where the
 * band count is even (else as 0).  FP8 handles: 1 = one band per CTA, 3 =
 * the two-SM kernel (even band count and an even number of 128-column
 * k-steps, else as 1), anything else = chosen by the library.  Results are
 * the same up to fp32 rounding order; this only lets tests reach each kernel.
 */
void patch_test_prefill_kernel(int32_t which);

/* Release a handle's device memory (stream-ordered on `stream`).  NULL ok. */
void patch_free(patch_packed *Wp, void *stream);

/*
 * Read and clear the handle's device status word (synchronises the device).
 * PATCH_OK, PATCH_ERR_TIMEOUT (a bounded wait ran out in an earlier
 * patch_hybrid_gemm), or PATCH_ERR_CUDA / INVALID_ARG.
 */
patch_status patch_get_status(const patch_packed *Wp);

/* Read-only view of a handle, for inspection and tests. */
typedef struct {
    const void *packed;     /* device: packed bytes                         */
    const uint64_t *table;  /* device: k-step table, (N/128)*(K/64) entries */
    size_t packed_bytes;    /* bytes at `packed`                            */
    int64_t N, K;
    int32_t tile_n, tile_k;
    int64_t sparse_ksteps;  /* k-steps stored 2:4                           */
    int64_t meta_blocks;    /* 2048-byte metadata blocks                    */
} patch_packed_view;

patch_status patch_packed_info(const patch_packed *Wp, patch_packed_view *view);

/*
 * Copy a handle's packed bytes (view.packed_bytes) and k-step table
 * ((N/128)*(K/64) uint64; (N/128)*(K/128) for FP8 handles) into caller-owned
 * DEVICE buffers, stream-ordered.
 * Either destination may be NULL to skip it.  For inspection and tests.
 */
patch_status patch_packed_export(const patch_packed *Wp, void *packed_dst, uint64_t *table_dst,
                                 void *stream);

/*
 * Number of kernels this library has enqueued in this process, on any stream
 * and device (a monotonically increasing count; read it before and after a
 * region to count that region's launches).  Diagnostics only; no device work.
 */
uint64_t patch_launch_count(void);

/* Human-readable name of a status code (static string). */
const char *patch_status_string(patch_status s);

#ifdef __cplusplus
}
#endif

#endif /* PATCH_B200_H */
