// Launchers shared between the translation units of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace patchk {

// Counts kernels enqueued by the library (exported as patch_launch_count).
void note_launches(int n);

// Column sums of squares: chunk partials [ceil(T/128), K] (chunk c = tokens
// 128c .. 128c+127 added in token order from 0.0), the in-order fold of the
// partials (colsq_out and / or norm_out = sqrt, either may be null), or both.
cudaError_t launch_colsq_partials(const void *Xcal, int64_t T, int64_t K, double *partial,
                                  cudaStream_t stream);
cudaError_t launch_colsq_fold(const double *partial, int64_t chunks, int64_t K, double *colsq_out,
                              double *norm_out, cudaStream_t stream);
cudaError_t launch_colsq(const void *Xcal, int64_t T, int64_t K, double *partial,
                         double *colsq_out, double *norm_out, cudaStream_t stream);
cudaError_t launch_norms_from_colsq(const double *colsq_in, int64_t K, double *colsq_out,
                                    double *norm_out, cudaStream_t stream);
// `rank` / `done` (may be null when no map is selected) are zeroed here for
// launch_select_map, which must follow on the same stream.  pattern 2: 2:4
// groups (4-bit codes); 4: 4:8 groups (8-bit keep masks).
cudaError_t launch_score_mask(const void *W, const double *norm, int64_t N, int64_t K, int tn,
                              int tk, uint32_t *meta, double *loss, int32_t *rank, uint32_t *done,
                              cudaStream_t stream, int pattern = 2);
cudaError_t launch_select_map(const double *loss, int64_t n_tiles, int64_t n_sparse, int32_t *rank,
                              uint32_t *done, uint32_t *map, cudaStream_t stream);

// Global tile allocation over up to kMaxGlobalMatrices matrices: `loss_cat`
// holds their tile losses concatenated, `rank` (zeroed, one per tile) is
// scratch; writes each matrix's bitmap to maps[m].
constexpr int kMaxGlobalMatrices = 64;
// the rank kernel's grid.y counts 256-tile slices of all tiles (<= 65535)
constexpr int64_t kMaxGlobalTiles = 65535LL * 256;
cudaError_t launch_select_maps_global(const double *loss_cat, const int64_t *n_tiles, int count,
                                      int64_t n_sparse, int32_t *rank, uint32_t *const *maps,
                                      cudaStream_t stream);

// `ptable` (may be null) adds the dense copies of the prefill table's side
// entries, written after the packed bytes.
cudaError_t launch_pack(const void *W, const uint32_t *meta, const uint32_t *map, int64_t N,
                        int64_t K, int tn, int tk, const uint64_t *table, const uint64_t *ptable,
                        uint8_t *out, cudaStream_t stream, int pattern = 2);
// Sets each handle's ready flag (zeroed, in the handle) to 1 with release
// semantics once the kernels queued before it on the stream (the packs) have
// completed; up to kPlanMaxGroup flags, one launch.
cudaError_t launch_publish_ready(uint32_t *const *ready, int count, cudaStream_t stream);
void preload_pack_kernels();

// Split-K decode kernel: CTAs whose first chunks travel in the kernel
// parameters, at most.
constexpr int kDecMaxCtas = 160;
constexpr int kDecMaxGroup = 8;  // matrices sharing X in one split-K launch

// Layout plan of a packed matrix, computed on the device from the tile map
// (plan_pack_kernel) and read back once by patch_pack.
struct PackPlan {
    uint64_t packed_bytes;
    uint64_t sparse_ksteps;
    uint64_t meta_blocks;
    uint32_t duo_ok;          // the band count is even: the prefill table pairs bands 2p, 2p+1
    uint32_t max_pair_bytes;  // largest packed k-pair
    uint64_t side_bytes;      // dense copies after the packed bytes (prefill table)
    uint32_t pair_max_bytes;  // largest k-pair the prefill table points to
    uint32_t pad_;
    uint64_t first_desc[2 * kDecMaxCtas];  // decode chunk descriptors 0 .. 2*kDecMaxCtas-1
};
// Plans the packed layout of up to kPlanMaxGroup matrices, one block each:
// writes each matrix's k-step table [bands][nsteps], decode chunk
// descriptors [bands][cpb], per-band cumulative k-pair bytes
// [bands][nsteps/2 + 1], the first byte of each band (scratch [bands]), the
// prefill table [bands][nsteps] with the side-region offsets of its dense
// copies (scratch side_start [bands]) and the plan summary.
constexpr int kPlanMaxGroup = 8;
struct PlanArgs {
    const uint32_t *map;
    int64_t N, K;
    int tn, tk, cp, cpb;
    uint64_t *table, *chunk_desc;
    int64_t *pair_prefix;
    uint64_t *band_start, *ptable, *side_start;
    PackPlan *plan;
    int pattern;
    uint32_t *status;  // the handle's kStatusWords status words (zeroed by the plan launch), or null
};
constexpr int kStatusWords = 64;
cudaError_t launch_plan_pack_group(const PlanArgs *args, int count, cudaStream_t stream);

struct GemmLaunch {
    const uint8_t *packed;
    const uint64_t *table;
    int64_t N, K;
    const void *X;
    int64_t M;
    void *Y;
    int y_fp32;
    float *workspace;        // stream-K partials owned by the handle (may be null)
    size_t workspace_bytes;  // capacity of `workspace`
    cudaMemPool_t pool;      // for larger stream-K partials
    uint32_t *status;
    const uint32_t *ready;   // set by the pack kernel when the packed bytes are final
    // decode chunking (see plan_decode_chunks)
    const uint64_t *chunk_desc;       // device [dec_nchunks]
    const uint64_t *chunk_desc_host;  // host copy
    int dec_cp, dec_cpb, dec_nchunks;
    uint32_t *counter;                // device: chunks claimed, zero between calls
    uint64_t packed_rows;             // (packed bytes + side copies) / 128
    const uint64_t *ptable;           // prefill table: bands 2p, 2p+1 agree in type at every k-step
    int duo_ok;                       // the prefill table pairs every band (even band count)
    int max_pair_bytes;               // largest k-pair the prefill table points to
    int num_sms;
    int stall_first_kstep;   // failure-detection test hook (see patch_hybrid_gemm)
    int force_kernel;        // test hook: 0 auto, 1 one-band, 2 band-pair, 3 two-SM, 4 two-SM four-band (M > 16)
    int pattern;             // 2: dense / 2:4 tiles; 4: dense / 4:8 tiles
    const int64_t *pair_prefix;  // host: per band, cumulative packed bytes of its k-pairs
    // FP8 handles (split-K path only): X holds the e4m3 codes, Y = acc * sw[n] * sx[m]
    const float *f8_sw;      // [N] W_eff row scales
    const float *f8_sx;      // [M] token scales
};

// Picks the configuration (token tile, schedule) for M and launches.
cudaError_t launch_hybrid_gemm(const GemmLaunch &g, cudaStream_t stream);

// Band-pair prefill GEMM (csrc/prefill_gemm.cu): token tile, grid and
// shared-memory plan for a matrix of N rows and M tokens.
struct PairPlan {
    int bn;           // tokens per tile (multiple of 16, 128..240)
    int ttiles;       // ceil(M / bn)
    int items;        // band pairs x token tiles
    int waves;        // ceil(items / SMs)
    int stages;       // k-steps in flight
    int stage_bytes;
    int smem;         // dynamic shared memory per CTA
    double cost;      // waves x estimated cycles per k-step of an item
};
// Estimated cycles of one dense k-step of a band-pair item with BN tokens.
double pair_kstep_cycles(int bn);
PairPlan plan_pair_gemm(int64_t N, int64_t M, int num_sms);
cudaError_t launch_pair_gemm(const GemmLaunch &g, const PairPlan &plan, cudaStream_t stream);

// Two-SM prefill GEMM (csrc/prefill_duo.cu) for matrices whose bands 2p and
// 2p+1 agree in tile type at every k-step.
struct DuoPlan {
    int bn;           // tokens per tile (each CTA of the pair holds bn / 2)
    int ttiles, items;
    int clusters;     // CTA pairs launched
    int stages, stage_bytes, smem;
    int aslot;        // weight slot of a stage (the largest k-pair, rounded to 1 KB)
    double cost;      // waves x estimated cycles per k-step of an item
};
DuoPlan plan_duo_gemm(int64_t N, int64_t M, int num_sms, int max_pair_bytes);
cudaError_t launch_duo_gemm(const GemmLaunch &g, const DuoPlan &plan, cudaStream_t stream);
// One launch over up to kDuoGroupMax matrices that read the same X (same K,
// M and output type); the plan is made for the sum of their N.
constexpr int kDuoGroupMax = 8;
cudaError_t launch_duo_group(const GemmLaunch *gs, int count, const DuoPlan &plan, cudaStream_t stream);
// Whether one two-SM launch over the group (bf16 2:4 handles with paired
// band types, the same X, more than 128 tokens) is estimated to finish before
// the matrices' own launches one after another; fills *plan when it is.
bool plan_hybrid_group(const GemmLaunch *gs, int count, DuoPlan *plan);
double duo_kstep_cycles(int bn);

// Two-SM, four-band prefill GEMM (csrc/prefill_quad.cu): each SM of a CTA
// pair holds two bands (pairs 2p, 2p+1 of the prefill table) sharing its half
// of the token tile.
struct QuadPlan {
    int bn;           // tokens per tile (each CTA of the pair holds bn / 2)
    int ttiles, items;
    int clusters;     // CTA pairs launched
    int stages, stage_bytes, smem;
    double cost;      // waves x estimated cycles per k-step of an item
};
QuadPlan plan_quad_gemm(int64_t N, int64_t M, int num_sms);
cudaError_t launch_quad_gemm(const GemmLaunch &g, const QuadPlan &plan, cudaStream_t stream);
double quad_kstep_cycles(int bn);

// Load every GEMM kernel of the library in the current context (each file
// its own).  Under lazy module loading the first launch of a kernel loads it,
// which waits for the device; the pack calls, which synchronise anyway, run
// these once per context so that no GEMM call ever does.
void preload_hybrid_kernels();
void preload_decode_kernels();
void preload_pair_kernels();
void preload_duo_kernels();
void preload_quad_kernels();
void preload_fp8_gemm_kernels();
void preload_duo_fp8_kernels();
void preload_fp8_quantize_kernels();

// Split-K GEMV / skinny GEMM for M <= kDecodeMaxM (csrc/decode_gemm.cu):
// token tiles of 16, 32 or 64 rows.
constexpr int64_t kDecodeMaxM = 64;
// above 16 tokens the split-K kernel serves K up to this (longer K: the
// one-band stream-K kernel)
constexpr int64_t kSplitKMaxK = 8192;
// whether a bf16 2:4 product of M tokens runs the split-K kernel (test hook
// `force_kernel` set: only M <= 16 does)
inline bool takes_split_k(int64_t M, int64_t K, int force_kernel) {
    return M <= 16 || (M <= kDecodeMaxM && K <= kSplitKMaxK && force_kernel == 0);
}
cudaError_t launch_decode_gemm(const GemmLaunch &g, cudaStream_t stream);
// One split-K launch over `count` (1..kDecMaxGroup) matrices that read the
// same X: the same K, M, X, output type and chunking; each member its own
// handle fields and Y.  The first member's counter (and workspace, when large
// enough) serve the launch.
cudaError_t launch_decode_group(const GemmLaunch *gs, int count, cudaStream_t stream);
// The same split-K kernel on FP8 handles (one matrix, or a group reading the
// same X): 128-column e4m3 k-steps taken two per "pair", kind::f8f6f4 MMAs,
// the fix-up applying each matrix's row scales and the token scales.  X holds
// the e4m3 code matrix [M, K] (the same for every member, as is f8_sx),
// M <= kDecodeMaxM.
cudaError_t launch_decode_f8(const GemmLaunch *gs, int count, cudaStream_t stream);
// Chunking of a packed matrix for the decode GEMV: `cp` k-pairs per chunk,
// `cpb` chunks per band.
void plan_decode_chunks(int64_t bands, int64_t nsteps, int num_sms, int *cp, int *cpb, int *nchunks);
// Descriptor of the chunk holding pairs [pr0, pr0 + np) of a band whose
// k-step table starts at `band_table`: first byte | 2:4 flags << 40 | np << 56.
uint64_t decode_chunk_desc(const uint64_t *band_table, int64_t nsteps, int pr0, int np);
// fp32 partial bytes of the decode GEMV (one bn x 128 slot per chunk).
size_t decode_workspace_bytes(int nchunks, int bn = 16);

// FP8 handles (csrc/fp8_kernels.cu, csrc/fp8_gemm.cu).
// Per-row e4m3 quantisation of a bf16 matrix [R, C]: scale[r] = amax / 448
// (1 for a zero row), q = e4m3(x / scale) (fp32 quotient, round to nearest,
// saturating).
cudaError_t launch_fp8_quantize_rows(const void *x, int64_t R, int64_t C, uint8_t *q, float *scale,
                                     cudaStream_t stream);
// W_eff row scales into `scale` [N] and the packed k-steps at the table's offsets.
// ptable (nullable): the prefill table; its side entries (kEntrySide) get
// dense copies of their k-steps' W_eff codes
cudaError_t launch_pack_fp8(const void *W, const uint32_t *meta, const uint32_t *map, int64_t N,
                            int64_t K, int tn, int tk, const uint64_t *table, const uint64_t *ptable,
                            float *scale, uint8_t *out, uint32_t *ready, cudaStream_t stream);
struct Fp8Launch {
    const uint8_t *packed;
    const uint64_t *table;   // [N/128][K/128]
    const uint64_t *ptable;  // prefill table (even band counts), else null
    uint64_t packed_bytes;   // packed k-steps + side copies
    int all_sparse;          // every k-step 2:4 (no dense weight slot needed)
    const float *sw;         // [N]
    const uint8_t *xq;       // [M, K] e4m3 codes of X
    const float *sx;         // [M]
    int64_t N, K, M;
    void *Y;
    int y_fp32;
    uint32_t *status;
    int num_sms;
    int force_kernel;        // test hook: 1 = one band per CTA, 3 = two-SM kernel, 0 = chosen here
    cudaMemPool_t pool;      // split-K partials of the one-band kernel (null: no split)
};
cudaError_t launch_fp8_gemm(const Fp8Launch &g, cudaStream_t stream);

// Two-SM FP8 prefill GEMM (csrc/prefill_duo_fp8.cu): bands 2p, 2p+1 of the
// prefill table on a CTA pair, two 128-column k-steps per stage.
struct DuoFp8Plan {
    int bn;           // tokens per tile (each CTA of the pair holds bn / 2)
    int ttiles, items;
    int clusters;     // CTA pairs launched
    int stages, stage_bytes, smem;
    int aslot;        // weight slot of a stage (two k-steps)
    int aslot_step;   // its half for one k-step
    double cost;      // waves x estimated cycles per k-step of an item
};
DuoFp8Plan plan_duo_fp8(int64_t N, int64_t M, int num_sms, bool all_sparse);
cudaError_t launch_duo_fp8(const Fp8Launch &g, const DuoFp8Plan &plan, cudaStream_t stream);
// One launch over up to kDuoGroupMax FP8 matrices that read the same X codes
// and scales (same K, M and output type); the plan is made for the sum of
// their N, with all_sparse only if every matrix is.
cudaError_t launch_duo_fp8_group(const Fp8Launch *gs, int count, const DuoFp8Plan &plan, cudaStream_t stream);

// The library's stream-ordered memory pool for the current device (cached
// memory is kept, not returned to the system between calls).
cudaError_t device_pool(cudaMemPool_t *pool);

}  // namespace patchk
