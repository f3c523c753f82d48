// Split-K hybrid GEMV / skinny GEMM for decode token counts (M <= 64; token
// tiles of 16, 32 or 64 rows) on the sm_100a tensor cores.
//
// Same product as the prefill kernel, Y = X * W_eff^T with dense k-steps on
// tcgen05.mma and 2:4 k-steps on tcgen05.mma.sp ("PATCH: Learnable Tile-level
// Hybrid Sparsity for LLMs", section 2, inference and deployment), shaped for
// the case where the weights are read once and the run is bound by HBM.  The
// same kernel serves FP8 handles (e4m3 codes, kind::f8f6f4, scales applied by
// the fix-up) and launches over several matrices that read one X.
//
// Work.  Every 128-row band of W is cut into chunks of `cp` consecutive
// k-pairs (128 input columns each).  CTA c first runs chunks c and c + G (G
// CTAs), then claims further chunks from an atomic counter, so SMs that
// stream faster take more chunks and no CTA's static share decides the end
// of the kernel.  A claim is made one chunk ahead, while the current chunk's
// copies are in flight, so its round trip is off the copy path.  Each
// chunk leaves its BN x 128 fp32 partial in its own slot; a fix-up kernel adds
// the chunks of a band in chunk order, so Y does not depend on which CTA ran
// which chunk.  No CTA ever waits for another.
//
// Copies.  A chunk's pairs are contiguous in the packed buffer; the chunk
// descriptor (byte offset + the 2:4 flags of its k-steps) is enough to place
// every k-step, so no table is read: the descriptors of the CTAs' first
// chunks travel in the kernel parameters and the first copies start at once.
// A pipeline stage holds two consecutive k-pairs of a chunk (a k-quad, 256
// input columns): one bulk copy of their packed bytes (36-64 KB) and one 3-D
// TMA load of their four X tiles (BN rows, rows past M read as zero).  Few,
// large copies matter: an SM's copy engine spends about as long on a small
// copy as on a 16 KB one.
//
// Issue.  On B200 each tcgen05.mma costs the issuing thread about 75 cycles
// whatever N is (N = 16 measured), a metadata copy about 180 and a commit about
// 140, while instructions from two threads overlap.  So two issuer warps
// share the work: ring positions alternate between them, each with its own
// accumulator per chunk (a chunk's two stages always land on different
// issuers), and the epilogue adds the two.  An issuer derives the k-step
// layout of a stage from the stage's word in registers, builds descriptors by
// adding offsets to per-stage bases, and commits once per stage.
//
// Launch.  A programmatic dependent of the previous kernel: once the packer's
// ready flag is seen, the first stages' weight copies are issued before
// `griddepcontrol.wait`; X, Y, the partials and the chunk counter are touched
// only after it.  The fix-up kernel resets the counter for the next call.
//
// Roles (224 threads): warp 0 lane 0 producer, lane 0 of warps 1 and 6 MMA
// issuers (even and odd ring positions), warps 2..5 epilogue (tcgen05.ld of
// the BN-column accumulators, fp32 partial stores).  Two accumulator sets
// alternate between consecutive chunks.  Every mbarrier wait is bounded by
// %globaltimer.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "patch_common.cuh"
#include "patch_internal.h"

namespace patchk {

namespace {

constexpr int kDecThreads = 224;
constexpr int kDecChunkPairs = 4;                         // k-pairs per chunk, at most
constexpr int kDecWBytes = 4 * kDenseStepBytes;           // two packed k-pairs, at most
constexpr uint64_t kDecWaitLimitNs = 2000000000ull;       // 2 s per wait

// Per token-tile width BN (the MMA's N: 16, 32 or 64 token rows).  A stage is
// the packed bytes of two k-pairs plus their four X tiles; three stages fit
// at BN = 16 (72 KB each), two at 32 and 64 (80 / 96 KB).  Tensor memory:
// 2 chunks x 2 issuers x BN accumulator columns, then 2 issuers x 2 k-pairs
// x 4 metadata columns.
template <int BN>
struct DecCfg {
    static_assert(BN == 16 || BN == 32 || BN == 64, "decode token tile");
    static constexpr int kXStepBytes = BN * kStep * 2;     // one k-step of X: BN rows x 64
    static constexpr int kXBytes = 4 * kXStepBytes;        // the stage's four X tiles
    static constexpr int kStageBytes = kDecWBytes + kXBytes;
    static constexpr int kStages = BN == 16 ? 3 : 2;
    static constexpr uint32_t kEcol = 4 * BN;
    // metadata: per issuer 2 pairs x 2 k-steps x 4 columns (FP8 k-steps each
    // carry their own block; bf16 pairs use the first 4 of each 8)
    static constexpr int kCols = 4 * BN + 32;
    static constexpr int kTmemCols = kCols <= 128 ? 128 : kCols <= 256 ? 256 : 512;
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 512;
    static_assert(kStageBytes % 1024 == 0, "stage regions stay 1024-B aligned");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kStages <= 4, "stage words and drained counters share the control block");
};

// chunk descriptor: first byte (40 bits) | 2:4 flag of each k-step (16) | pairs (4)
constexpr uint64_t kDescOffsetMask = (1ull << 40) - 1;
constexpr int kDescFlagsShift = 40;
constexpr int kDescPairsShift = 56;

// stage word: chunk (29 bits) | no more work (bit 31) | pairs in the stage (1
// or 2) << 32 | the chunk has two stages (bit 34) | k-step 2:4 flags << 36 |
// ordinal of the chunk in this CTA (16 bits; for the done word: chunks in
// all) << 40 | ring position (low 8 bits) << 56
constexpr uint64_t kStageChunk = (1ull << 29) - 1;
constexpr uint64_t kStageDone = 1ull << 31;
constexpr int kStagePairsShift = 32;
constexpr uint64_t kStageTwo = 1ull << 34;
constexpr int kStageFlagsShift = 36;
constexpr int kStageOrdShift = 40;
constexpr int kStagePosShift = 56;
constexpr int kDecMaxChunksPerCta = 65535;

// One launch covers one matrix, or several that read the same X (the same K,
// hence the same chunking): their bands are numbered one after another
// (matrix i holds global bands band0[i] .. band0[i+1]-1), chunk j belongs to
// global band j / cpb, and each matrix keeps its own packed bytes, chunk
// descriptors, output, status and ready words.
struct DecodeParams {
    int64_t K, M;
    int cpb;      // chunks per band (the same for every matrix of the launch)
    int cp;       // k-pairs per chunk (the last chunk of a band may hold fewer)
    int nchunks;  // all matrices
    int nmat;     // 1 .. kDecMaxGroup
    int32_t band0[kDecMaxGroup + 1];
    const uint8_t *packed[kDecMaxGroup];
    const uint64_t *chunk_desc[kDecMaxGroup];  // [bands * cpb] of each matrix
    void *Y[kDecMaxGroup];
    int64_t N[kDecMaxGroup];
    uint32_t *status[kDecMaxGroup];
    const uint32_t *ready[kDecMaxGroup];
    int y_fp32;
    const float *f8_sw[kDecMaxGroup];  // FP8: [N] row scales of each matrix
    const float *f8_sx;                // FP8: [M] token scales (the shared X)
    float *partial[kDecMaxGroup];  // per matrix: [its chunks][BN][128]
    uint32_t *counter;  // chunks claimed beyond the first 2 * gridDim.x; zero between calls
    int stall_first_kstep;  // failure-detection test hook
    uint64_t first_desc[kDecMaxCtas];   // descriptor of chunk c for c < gridDim.x
    uint64_t second_desc[kDecMaxCtas];  // of chunk c + gridDim.x where that exists
};

// matrix holding global band gb
__device__ __forceinline__ int dec_mat_of_band(const DecodeParams &p, int gb) {
    int i = 0;
    while (i + 1 < p.nmat && p.band0[i + 1] <= gb) ++i;
    return i;
}

// a wait that ran out: every matrix of the launch reports it
__device__ __forceinline__ void dec_raise_timeout(const DecodeParams &p) {
    for (int i = 0; i < p.nmat; ++i) atomicOr(p.status[i], kStatusTimeout);
}

// Bytes of pair i of a chunk whose k-step flags are `flags`, and whether its
// metadata block is present.  Mirrors the packer: a 2 KB metadata block
// precedes the first 2:4 k-step of every k-pair.
// FP8 (e4m3): every 2:4 k-step carries its own 2 KB metadata block.
template <bool F8>
__device__ __forceinline__ uint32_t pair_bytes(uint32_t flags, int i) {
    const uint32_t f = (flags >> (2 * i)) & 3u;
    if constexpr (F8) {
        const uint32_t sp = kMetaBlockBytes + kSparseStepBytes;
        return ((f & 1u) ? sp : kDenseStepBytes) + ((f & 2u) ? sp : kDenseStepBytes);
    }
    return (f == 0u) ? 2u * kDenseStepBytes
                     : (f == 3u) ? kMetaBlockBytes + 2u * kSparseStepBytes
                                 : kMetaBlockBytes + kDenseStepBytes + kSparseStepBytes;
}

// Wait until each of four shared counters (chunks drained by each epilogue
// warp; the warps run independently, so a sum could hide a lagging one)
// reaches `target`.  Counters have no phase aliasing; the issuers may trail
// or lead one another by a chunk.
__device__ __forceinline__ bool drained_all(volatile uint32_t *ctr, uint32_t target) {
    return ctr[0] >= target && ctr[1] >= target && ctr[2] >= target && ctr[3] >= target;
}
__device__ __forceinline__ bool wait_count_bounded(volatile uint32_t *ctr, uint32_t target,
                                                   volatile uint32_t *abort_flag, uint64_t limit_ns) {
    if (drained_all(ctr, target)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (drained_all(ctr, target)) return true;
        if ((i & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > limit_ns) return false;
        }
    }
}

__device__ __forceinline__ void store_out(const DecodeParams &p, int mi, int64_t idx, float v) {
    if (p.y_fp32)
        static_cast<float *>(p.Y[mi])[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(p.Y[mi])[idx] = __float2bfloat16_rn(v);
}

template <int BN, bool F8>
__global__ void __launch_bounds__(kDecThreads, 1)
decode_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ DecodeParams p) {
    using C = DecCfg<BN>;
    constexpr int kDecStages = C::kStages;
    constexpr int kDecStageBytes = C::kStageBytes;
    constexpr int kDecXBytes = C::kXBytes;
    constexpr int kDecXStepBytes = C::kXStepBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kDecStages * kDecStageBytes);
    uint64_t *empty = full + kDecStages;
    uint64_t *acc_full = empty + kDecStages;  // [2] four arrivals from the issuers per chunk
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 2);
    volatile uint32_t *abort_flag = tmem_slot + 1;  // raised by any role that gives up
    volatile uint32_t *never_flag = tmem_slot + 2;  // stays 0: time-only bounded waits
    volatile int32_t *acc_chunk = reinterpret_cast<volatile int32_t *>(tmem_slot + 4);  // [2]
    volatile uint32_t *acc_mask = tmem_slot + 6;  // [2] issuers holding a part of the chunk
    volatile uint32_t *drained = tmem_slot + 16;  // [4] chunks drained by each epilogue quarter
    uint64_t *stage_word = reinterpret_cast<uint64_t *>(tmem_slot + 8);                 // [STAGES]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    bool waited = true;  // thread 0: past griddepcontrol.wait

    if (threadIdx.x == 0) {
        pdl_trigger();
        // the packed bytes are final once the ready flag is seen; otherwise
        // (the packer may be the kernel just before) wait first
        bool all_ready = true;
        for (int i = 0; i < p.nmat; ++i) all_ready = all_ready && ld_acquire_gpu(p.ready[i]) != 0u;
        if (!all_ready) pdl_wait();
        else waited = false;
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&acc_full[b], 4);
        *never_flag = 0u;
        for (int w = 0; w < 4; ++w) drained[w] = 0u;
        // a matrix whose status is raised skips the whole launch
        uint32_t raised = 0u;
        for (int i = 0; i < p.nmat; ++i) raised |= *reinterpret_cast<volatile uint32_t *>(p.status[i]);
        *abort_flag = (raised & kStatusTimeout) ? 1u : 0u;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmap_x);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;

    if (warp == 0) {
        if (lane == 0 && !skip) {
            // ------------------------------------------------------ producer
            int it = 0;  // stages armed so far (ring position)
            uint64_t cord = 0;  // chunks armed so far
            bool ok = true;
            int pend_s[kDecStages], pend_k[kDecStages];  // X loads of stages armed before the wait
            int npend = 0;
            auto flush_x = [&]() {
                pdl_wait();
                waited = true;
                for (int q = 0; q < npend; ++q)
                    tma_load_3d(smem + pend_s[q] * kDecStageBytes + kDecWBytes, &tmap_x, 0, 0, pend_k[q],
                                &full[pend_s[q]]);
                npend = 0;
            };
            // chunks j (current) and jn (next) are known; the one after jn is
            // claimed during chunk j, once the counter may be touched (the
            // previous call's fix-up resets it)
            const int G = static_cast<int>(gridDim.x);
            int j = blockIdx.x;
            uint64_t d = p.first_desc[blockIdx.x];
            int jn = blockIdx.x + G;
            uint64_t dn = (jn < p.nchunks) ? p.second_desc[blockIdx.x] : 0ull;
            bool have_tk = false;
            uint32_t tk = 0;
            while (ok && j < p.nchunks) {
                const int pr0 = (j % p.cpb) * p.cp;
                const int np = static_cast<int>((d >> kDescPairsShift) & 0xFu);
                const uint32_t flags = static_cast<uint32_t>((d >> kDescFlagsShift) & 0xFFFFu);
                uint64_t cur = d & kDescOffsetMask;
                for (int i = 0; i < np; i += 2) {
                    const int s = it % kDecStages;
                    const uint32_t ph = (it / kDecStages) & 1u;
                    if (!waited && it >= kDecStages) flush_x();
                    if (it >= kDecStages &&
                        !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kDecWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    const int sp = min(2, np - i);
                    const uint32_t bytes = pair_bytes<F8>(flags, i) + (sp == 2 ? pair_bytes<F8>(flags, i + 1) : 0u);
                    const uint32_t sflags = (flags >> (2 * i)) & (sp == 2 ? 0xFu : 0x3u);
                    stage_word[s] = static_cast<uint64_t>(j) | (np > 2 ? kStageTwo : 0ull) |
                                    (static_cast<uint64_t>(sp) << kStagePairsShift) |
                                    (static_cast<uint64_t>(sflags) << kStageFlagsShift) |
                                    (cord << kStageOrdShift) |
                                    (static_cast<uint64_t>(it & 0xFF) << kStagePosShift);
                    ++it;
                    const uint64_t src = cur;
                    cur += bytes;
                    if (!(p.stall_first_kstep && blockIdx.x == 0 && it == 1)) {  // else never lands
                        uint8_t *st = smem + s * kDecStageBytes;
                        mbar_arrive_expect_tx(&full[s], bytes + kDecXBytes);
                        bulk_g2s(st, p.packed[dec_mat_of_band(p, j / p.cpb)] + src, bytes, &full[s]);
                        if (waited) {
                            tma_load_3d(st + kDecWBytes, &tmap_x, 0, 0, 2 * (pr0 + i), &full[s]);
                        } else {
                            pend_s[npend] = s;
                            pend_k[npend] = 2 * (pr0 + i);
                            ++npend;
                        }
                    }
                    // the result is first read at the end of the chunk
                    if (waited && !have_tk && jn < p.nchunks) {
                        tk = atomicAdd(p.counter, 1u);
                        have_tk = true;
                    }
                }
                if (!ok) break;
                ++cord;
                int jnn = p.nchunks;
                uint64_t dnn = 0;
                if (jn < p.nchunks) {
                    if (!have_tk) {
                        if (!waited) flush_x();
                        tk = atomicAdd(p.counter, 1u);
                    }
                    have_tk = false;
                    jnn = 2 * G + static_cast<int>(tk);
                    if (jnn < p.nchunks) {
                        const int mi = dec_mat_of_band(p, jnn / p.cpb);
                        dnn = __ldcg(p.chunk_desc[mi] + (jnn - p.band0[mi] * p.cpb));
                    }
                }
                j = jn;
                d = dn;
                jn = jnn;
                dn = dnn;
            }
            if (!waited) flush_x();
            // no more chunks: a stage carrying the done flag (plain arrive)
            // for each issuer, with the chunk count
            for (int q = 0; q < 2 && ok; ++q) {
                const int s = it % kDecStages;
                const uint32_t ph = (it / kDecStages) & 1u;
                if (it >= kDecStages &&
                    !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kDecWaitLimitNs)) {
                    ok = false;
                } else {
                    stage_word[s] = kStageDone | (cord << kStageOrdShift) |
                                    (static_cast<uint64_t>(it & 0xFF) << kStagePosShift);
                    mbar_arrive(&full[s]);
                    ++it;
                }
            }
            if (!ok) {
                *abort_flag = 1u;
                dec_raise_timeout(p);
            }
            // Drain: the last phase armed on every stage must have landed
            // before the CTA exits (a no-op when the MMA thread consumed all).
            for (int q = (it > kDecStages ? it - kDecStages : 0); q < it; ++q) {
                if (p.stall_first_kstep && blockIdx.x == 0 && q == 0) continue;  // never armed
                mbar_wait_bounded(&full[q % kDecStages], (q / kDecStages) & 1u, never_flag,
                                  kDecWaitLimitNs / 4);
            }
        }
    } else if (warp == 1 || warp == 6) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------------- MMA
            const int q = warp == 6 ? 1 : 0;  // ring positions q, q + 2, ...
            // Descriptors: a template per layout plus the operand's shared
            // address in 16-byte units (all addresses here are below 256 KB,
            // so the 14-bit address field never carries into other fields).
            constexpr uint32_t kIdDense = F8 ? idesc_e4m3(BN, false) : idesc_bf16(BN, false);
            constexpr uint32_t kIdSp0 = F8 ? idesc_e4m3(BN, true) : idesc_bf16(BN, true, 0);
            constexpr uint32_t kIdSp1 = idesc_bf16(BN, true, 1);
            const uint64_t t_sw128 = smem_desc(0, 16, 1024, kSwizzle128B);  // dense A, X
            const uint64_t t_sw64 = smem_desc(0, 16, 512, kSwizzle64B);     // 2:4 A
            const uint64_t t_meta = smem_desc(0, 16, 128, kSwizzleNone);    // metadata
            const uint32_t e_tmem = tmem_base + C::kEcol + 16 * q;
            const uint32_t smem0 = smem_u32(smem);
            int it = q;       // ring position
            int nch = 0;      // chunks of this CTA (from the done word)
            bool ok = true;
            for (;; it += 2) {
                const int s = it % kDecStages;
                const uint32_t ph = (it / kDecStages) & 1u;
                // The slot's previous phase belongs to the other issuer and may
                // still be in flight, when a parity wait for ours passes at once:
                // so the stage is ours only once the wait passes AND the word
                // carries our position (the producer writes it only after the
                // previous phase was consumed, and the next phase needs our
                // commit, so the two together are exact).
                uint64_t w = 0;
                {
                    const uint64_t t0 = globaltimer_ns();
                    for (uint32_t n = 0;; ++n) {
                        if (mbar_try_wait(&full[s], ph)) {
                            w = *reinterpret_cast<volatile uint64_t *>(&stage_word[s]);
                            if (((w >> kStagePosShift) & 0xFFu) == static_cast<uint64_t>(it & 0xFF)) break;
                        }
                        if ((n & 63u) == 63u &&
                            (*abort_flag || globaltimer_ns() - t0 > kDecWaitLimitNs)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!ok) break;
                }
                tc_fence_after();
                const int c = static_cast<int>((w >> kStageOrdShift) & 0xFFFFu);
                if (w & kStageDone) {
                    nch = c;
                    break;
                }
                // this issuer holds at most one stage of chunk c: its accumulator
                // is free once the epilogue has drained chunks up to c - 2
                const int buf = c & 1;
                if (c >= 2 && !wait_count_bounded(drained, static_cast<uint32_t>(c - 1), abort_flag,
                                                  kDecWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (2 * buf + q) * BN;
                const uint32_t st16 = (smem0 + s * kDecStageBytes) >> 4;  // stage, 16-byte units
                const uint64_t x16 = t_sw128 + st16 + (kDecWBytes >> 4);
                const int sp = static_cast<int>((w >> kStagePairsShift) & 3u);
                const uint32_t fl = static_cast<uint32_t>(w >> kStageFlagsShift) & 0xFu;
                uint32_t off16 = 0;  // running offset in the stage, 16-byte units
                uint32_t acc = 0u;  // the stage starts this issuer's part of the chunk
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (t >= sp) break;
                    const uint32_t f = (fl >> (2 * t)) & 3u;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t bx = x16 + (2 * t + h) * (kDecXStepBytes >> 4);
                        if constexpr (F8) {
                            // a 128-column e4m3 k-step: the byte shape of a bf16
                            // 64-column one (128-byte rows dense, 64-byte rows of
                            // kept codes), K32 dense / K64 sparse per MMA; a 2:4
                            // k-step's own metadata block precedes it, sparse MMA
                            // j reads columns e + 2j with selector 0
                            if ((f >> h) & 1u) {
                                const uint32_t e = e_tmem + 8 * t + 4 * h;
                                tmem_cp_128x128b(e, t_meta + st16 + off16);
                                off16 += kMetaBlockBytes >> 4;
                                const uint64_t a = t_sw64 + st16 + off16;
                                mma_f8_sparse(d_tmem, a, bx, e, kIdSp0, acc);
                                mma_f8_sparse(d_tmem, a + 2, bx + 4, e + 2, kIdSp0, 1u);
                                off16 += kSparseStepBytes >> 4;
                            } else {
                                const uint64_t a = t_sw128 + st16 + off16;
                                mma_f8(d_tmem, a, bx, kIdDense, acc);
                                mma_f8(d_tmem, a + 2, bx + 2, kIdDense, 1u);
                                mma_f8(d_tmem, a + 4, bx + 4, kIdDense, 1u);
                                mma_f8(d_tmem, a + 6, bx + 6, kIdDense, 1u);
                                off16 += kDenseStepBytes >> 4;
                            }
                        } else {
                            if ((f >> h) & 1u) {
                                // the pair's metadata block precedes its first 2:4 k-step
                                if (h == 0 || !(f & 1u)) {
                                    tmem_cp_128x128b(e_tmem + 8 * t, t_meta + st16 + off16);
                                    off16 += kMetaBlockBytes >> 4;
                                }
                                const uint64_t a = t_sw64 + st16 + off16;
                                const uint32_t e = e_tmem + 8 * t + 2 * h;
                                mma_sparse(d_tmem, a, bx, e, kIdSp0, acc);
                                mma_sparse(d_tmem, a + 2, bx + 4, e, kIdSp1, 1u);
                                off16 += kSparseStepBytes >> 4;
                            } else {
                                const uint64_t a = t_sw128 + st16 + off16;
                                mma_dense(d_tmem, a, bx, kIdDense, acc);
                                mma_dense(d_tmem, a + 2, bx + 2, kIdDense, 1u);
                                mma_dense(d_tmem, a + 4, bx + 4, kIdDense, 1u);
                                mma_dense(d_tmem, a + 6, bx + 6, kIdDense, 1u);
                                off16 += kDenseStepBytes >> 4;
                            }
                        }
                        acc = 1u;
                    }
                }
                tc_commit(&empty[s]);
                // acc_full[buf] takes four arrivals per chunk: a commit and an
                // arrive from each of two issuers, or a commit and three from one
                const bool two = (w & kStageTwo) != 0;
                acc_chunk[buf] = static_cast<int32_t>(w & kStageChunk);
                acc_mask[buf] = two ? 3u : (1u << q);
                tc_commit(&acc_full[buf]);
                mbar_arrive_cnt(&acc_full[buf], two ? 1u : 3u);  // publishes acc_chunk, acc_mask
            }
            if (!ok) {
                *abort_flag = 1u;
                dec_raise_timeout(p);
            }
            // End of work for the epilogue: a phase whose chunk is -1, one
            // commit and one arrive from each issuer.  The commits fire once
            // every MMA issued has completed, so TMEM is never freed under a
            // running MMA.  (After a timeout the chunk count is unknown and the
            // epilogue gives up on its own bounded wait.)
            if (ok) {
                const int buf = nch & 1;
                if (nch >= 2)
                    wait_count_bounded(drained, static_cast<uint32_t>(nch - 1), never_flag, kDecWaitLimitNs);
                acc_chunk[buf] = -1;
                tc_commit(&acc_full[buf]);
                mbar_arrive(&acc_full[buf]);
            }
        }
    } else if (!skip) {
        // ------------------------------------------------------- epilogue
        pdl_wait();  // the partial slots may still be read by an earlier fix-up
        const int quad = warp % 4;  // TMEM lanes 32*quad .. 32*quad+31
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        for (int ci = 0;; ++ci) {
            const int buf = ci & 1;
            const bool ok = mbar_wait_bounded(&acc_full[buf], (ci >> 1) & 1u, never_flag, kDecWaitLimitNs);
            tc_fence_after();
            if (!ok) {
                *abort_flag = 1u;
                dec_raise_timeout(p);
                break;
            }
            const int j = acc_chunk[buf];
            if (j < 0) break;
            const uint32_t mask = acc_mask[buf];  // the same for every lane
            // 16 token columns at a time (columns past M are never stored)
#pragma unroll 1
            for (int c0 = 0; c0 < BN && c0 < p.M; c0 += 16) {
                uint32_t r0[16], r1[16];
                if (mask & 1u) tmem_ld_32x32b_x16(lane_base + (2 * buf) * BN + c0, r0);
                if (mask & 2u) tmem_ld_32x32b_x16(lane_base + (2 * buf + 1) * BN + c0, r1);
                tmem_ld_wait();
                if (*abort_flag == 0) {
                    const int mi = dec_mat_of_band(p, j / p.cpb);
                    const int64_t lj = j - static_cast<int64_t>(p.band0[mi]) * p.cpb;  // chunk of matrix mi
                    float *part = p.partial[mi] + (lj * BN + c0) * kBand + row;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float v = (mask == 3u) ? __fadd_rn(__uint_as_float(r0[q]), __uint_as_float(r1[q]))
                                                     : __uint_as_float(mask & 1u ? r0[q] : r1[q]);
                        if (c0 + q < p.M) part[q * kBand] = v;
                    }
                }
            }
            // the accumulator may be reused as soon as every lane has read it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                drained[quad] = static_cast<uint32_t>(ci + 1);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// Fix-up: Y[m, band*128 + row] = the band's chunk partials added in chunk
// order.  Block (band, m), one thread per row.  Launched as a programmatic
// dependent of the GEMM; resets the chunk counter once the GEMM is complete.
template <int BN, bool F8>
__global__ void __launch_bounds__(kBand)
decode_reduce_kernel(const __grid_constant__ DecodeParams p) {
    if (threadIdx.x == 0) pdl_trigger();  // the next GEMM may start its prologue
    pdl_wait();
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.counter = 0u;
    const int band = blockIdx.x, m = blockIdx.y, row = threadIdx.x;
    const int mi = dec_mat_of_band(p, band);
    const float *src = p.partial[mi] + (static_cast<int64_t>(band - p.band0[mi]) * p.cpb * BN + m) * kBand + row;
    float acc = 0.0f;
    for (int c0 = 0; c0 < p.cpb; c0 += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            v[q] = (c0 + q < p.cpb) ? __ldcg(src + static_cast<int64_t>(c0 + q) * BN * kBand) : 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (c0 + q < p.cpb) acc = __fadd_rn(acc, v[q]);
    }
    const int64_t n = static_cast<int64_t>(band - p.band0[mi]) * kBand + row;
    if constexpr (F8) acc = acc * __ldg(p.f8_sw[mi] + n) * __ldg(p.f8_sx + m);
    store_out(p, mi, static_cast<int64_t>(m) * p.N[mi] + n, acc);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

}  // namespace

void plan_decode_chunks(int64_t bands, int64_t nsteps, int num_sms, int *cp, int *cpb, int *nchunks) {
    const int64_t Q = nsteps / 2;
    // four k-pairs (about 100 KB at half 2:4) per chunk: measured on B200
    // against 1, 2, 6 and 8 for the Llama-7B shapes; smaller chunks cost more
    // partials and claims than they gain in balance, larger ones lose balance
    (void)num_sms;
    const int64_t c = std::min<int64_t>(kDecChunkPairs, Q);
    *cp = static_cast<int>(c);
    *cpb = static_cast<int>((Q + c - 1) / c);
    *nchunks = static_cast<int>(bands * *cpb);
}

uint64_t decode_chunk_desc(const uint64_t *band_table, int64_t nsteps, int pr0, int np) {
    const uint64_t e = band_table[2 * pr0];
    const uint64_t off = (e & kEntryOffsetMask) - ((e & kEntryMeta) ? kMetaBlockBytes : 0);
    uint64_t flags = 0;
    for (int i = 0; i < 2 * np; ++i)
        if (band_table[2 * pr0 + i] & kEntrySparse) flags |= 1ull << i;
    (void)nsteps;
    return (off & kDescOffsetMask) | (flags << kDescFlagsShift) |
           (static_cast<uint64_t>(np) << kDescPairsShift);
}

size_t decode_workspace_bytes(int nchunks, int bn) {
    return sizeof(float) * static_cast<size_t>(nchunks) * bn * kBand;
}

namespace {

template <int BN, bool F8>
cudaError_t launch_decode(const GemmLaunch *gs, int count, cudaStream_t stream) {
    using C = DecCfg<BN>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(decode_gemm_kernel<BN, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    if (count < 1 || count > kDecMaxGroup) return cudaErrorInvalidValue;
    const GemmLaunch &g = gs[0];
    if (F8 && !g.f8_sx) return cudaErrorInvalidValue;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    // X [M,K] viewed as (128-byte column blocks, M rows, K-steps): 64 bf16
    // columns or 128 e4m3 codes per k-step; box = the four k-steps of a
    // stage, BN rows, 128-byte swizzle, rows past M and k-steps past K read
    // as zero
    const int64_t kstep_cols = F8 ? 128 : kStep, elem = F8 ? 1 : 2;
    CUtensorMap map;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kstep_cols), static_cast<cuuint64_t>(g.M),
                                static_cast<cuuint64_t>(g.K / kstep_cols)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(g.K * elem), static_cast<cuuint64_t>(kstep_cols * elem)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kstep_cols), static_cast<cuuint32_t>(BN), 4};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&map, F8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void *>(g.X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    if (!g.counter) return cudaErrorInvalidValue;
    if (g.dec_cp < 1 || g.dec_cp > kDecChunkPairs || g.dec_cpb < 1) return cudaErrorInvalidValue;

    DecodeParams p;
    p.K = g.K;
    p.M = g.M;
    p.cpb = g.dec_cpb;
    p.cp = g.dec_cp;
    p.nmat = count;
    p.y_fp32 = g.y_fp32;
    p.f8_sx = g.f8_sx;
    p.counter = g.counter;
    p.stall_first_kstep = g.stall_first_kstep;
    int64_t bands = 0;
    for (int i = 0; i < kDecMaxGroup; ++i) {
        p.packed[i] = nullptr;
        p.f8_sw[i] = nullptr;
        p.chunk_desc[i] = nullptr;
        p.Y[i] = nullptr;
        p.N[i] = 0;
        p.status[i] = nullptr;
        p.ready[i] = nullptr;
    }
    for (int i = 0; i < count; ++i) {
        const GemmLaunch &m = gs[i];
        // one chunking, one X, one output type for the whole launch
        if (m.K != g.K || m.M != g.M || m.X != g.X || m.y_fp32 != g.y_fp32 || m.dec_cp != g.dec_cp ||
            m.dec_cpb != g.dec_cpb || m.N % kBand != 0 || m.dec_nchunks != (m.N / kBand) * g.dec_cpb ||
            !m.chunk_desc || !m.chunk_desc_host || !m.packed || !m.Y || !m.status || !m.ready ||
            (F8 && (!m.f8_sw || m.f8_sx != g.f8_sx)))
            return cudaErrorInvalidValue;
        p.band0[i] = static_cast<int32_t>(bands);
        p.packed[i] = m.packed;
        p.f8_sw[i] = m.f8_sw;
        p.chunk_desc[i] = m.chunk_desc;
        p.Y[i] = m.Y;
        p.N[i] = m.N;
        p.status[i] = m.status;
        p.ready[i] = m.ready;
        bands += m.N / kBand;
    }
    for (int i = count; i <= kDecMaxGroup; ++i) p.band0[i] = static_cast<int32_t>(bands);
    const int64_t nchunks = bands * g.dec_cpb;
    // a CTA's chunk ordinals travel in 16 bits (dynamic claiming could in
    // principle hand one CTA every chunk); chunk numbers in 29 bits
    if (nchunks > kDecMaxChunksPerCta) return cudaErrorInvalidValue;
    p.nchunks = static_cast<int>(nchunks);
    const int grid = static_cast<int>(std::min<int64_t>(std::min<int64_t>(g.num_sms, nchunks), kDecMaxCtas));
    // host copy of chunk c's descriptor
    auto desc_of = [&](int64_t c) {
        int i = 0;
        while (i + 1 < count && p.band0[i + 1] * static_cast<int64_t>(g.dec_cpb) <= c) ++i;
        return gs[i].chunk_desc_host[c - static_cast<int64_t>(p.band0[i]) * g.dec_cpb];
    };
    for (int c = 0; c < kDecMaxCtas; ++c) {
        p.first_desc[c] = c < grid ? desc_of(c) : 0ull;
        p.second_desc[c] = (c < grid && c + grid < nchunks) ? desc_of(c + grid) : 0ull;
    }
    // partials: each handle's own slots (16 token rows per chunk) where they
    // are large enough; otherwise one block from the stream-ordered pool for
    // the call, cut per matrix
    bool own = true;
    for (int i = 0; i < count; ++i)
        own = own && gs[i].workspace &&
              decode_workspace_bytes(gs[i].dec_nchunks, BN) <= gs[i].workspace_bytes;
    float *ws = nullptr;
    if (!own) {
        const cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws),
                                                      decode_workspace_bytes(p.nchunks, BN), g.pool, stream);
        if (e != cudaSuccess) return e;
    }
    for (int i = 0; i < kDecMaxGroup; ++i)
        p.partial[i] = i >= count ? nullptr
                       : own ? gs[i].workspace
                             : ws + static_cast<int64_t>(p.band0[i]) * g.dec_cpb * BN * kBand;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, decode_gemm_kernel<BN, F8>, map, p);
    if (err == cudaSuccess) {
        note_launches(1);
        cfg.gridDim = dim3(static_cast<unsigned>(bands), static_cast<unsigned>(g.M));
        cfg.blockDim = dim3(kBand);
        cfg.dynamicSmemBytes = 0;
        err = cudaLaunchKernelEx(&cfg, decode_reduce_kernel<BN, F8>, p);
        if (err == cudaSuccess) note_launches(1);
    }
    if (ws) {
        const cudaError_t e2 = cudaFreeAsync(ws, stream);
        if (err == cudaSuccess) err = e2;
    }
    return err;
}

}  // namespace

void preload_decode_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, decode_gemm_kernel<16, false>);
    (void)cudaFuncGetAttributes(&a, decode_gemm_kernel<32, false>);
    (void)cudaFuncGetAttributes(&a, decode_gemm_kernel<64, false>);
    (void)cudaFuncGetAttributes(&a, decode_reduce_kernel<16, false>);
    (void)cudaFuncGetAttributes(&a, decode_reduce_kernel<32, false>);
    (void)cudaFuncGetAttributes(&a, decode_reduce_kernel<64, false>);
    (void)cudaFuncGetAttributes(&a, decode_gemm_kernel<16, true>);
    (void)cudaFuncGetAttributes(&a, decode_gemm_kernel<32, true>);
    (void)cudaFuncGetAttributes(&a, decode_gemm_kernel<64, true>);
    (void)cudaFuncGetAttributes(&a, decode_reduce_kernel<16, true>);
    (void)cudaFuncGetAttributes(&a, decode_reduce_kernel<32, true>);
    (void)cudaFuncGetAttributes(&a, decode_reduce_kernel<64, true>);
}

cudaError_t launch_decode_group(const GemmLaunch *gs, int count, cudaStream_t stream) {
    if (count < 1) return cudaErrorInvalidValue;
    const int64_t M = gs[0].M;
    if (M <= 16) return launch_decode<16, false>(gs, count, stream);
    if (M <= 32) return launch_decode<32, false>(gs, count, stream);
    if (M <= kDecodeMaxM) return launch_decode<64, false>(gs, count, stream);
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode_gemm(const GemmLaunch &g, cudaStream_t stream) {
    return launch_decode_group(&g, 1, stream);
}

cudaError_t launch_decode_f8(const GemmLaunch *gs, int count, cudaStream_t stream) {
    if (count < 1) return cudaErrorInvalidValue;
    const int64_t M = gs[0].M;
    if (M <= 16) return launch_decode<16, true>(gs, count, stream);
    if (M <= 32) return launch_decode<32, true>(gs, count, stream);
    if (M <= kDecodeMaxM) return launch_decode<64, true>(gs, count, stream);
    return cudaErrorInvalidValue;
}

}  // namespace patchk
