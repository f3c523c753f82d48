// Two-SM FP8 hybrid GEMM for prefill: tcgen05 kind::f8f6f4 with
// cta_group::2 (sm_100a).  Y = diag(sx) (QX QW^T) diag(sw), the product of
// the FP8 path ("SparseGPT vs Wanda: one-shot LLM pruning without
// retraining", FAQ: prune first, then quantise; the tile scheme of "PATCH:
// Learnable Tile-level Hybrid Sparsity for LLMs", section 2).
//
// Why.  The tensor core reads its operands from shared memory and the TMA
// copies write there too, about 128 B per cycle per SM in all.  With one CTA
// per MMA every SM writes and reads the whole token tile; with cta_group::2 a
// CTA pair runs M = 256 MMAs (one 128-row band per SM) and each SM holds
// HALF of the token tile, which cuts an SM's shared-memory bytes per
// 128-column k-step from 92 KB to 62 KB at 240 tokens.
//
// Work item = (band pair, token tile of BN tokens); clusters of two CTAs take
// items c, c + C, ...; CTA rank r owns band 2p + r and tokens [r BN/2,
// (r+1) BN/2) of the tile.  Stage = two 128-column k-steps: this SM's band
// (one TMA load per k-step of 16 KB dense or 2 KB metadata + 8 KB codes,
// through tensor maps over the packed buffer in 2 KB rows, each into a fixed
// half of the weight slot) and its half of the X codes for both k-steps (ONE
// 3-D TMA load, 128-byte swizzle, rows past M zero), from a weight and an X
// producer thread.  Both CTAs' loads complete on the leader's stage mbarrier.
// The bands of a pair take one kind at every k-step through the prefill table
// (a 2:4 k-step whose partner is dense points to a dense side copy).  The
// leader's MMA thread issues 4 dense K32 or 2 sparse K64 M256 x BN MMAs per
// k-step (the 2:4 metadata of k-step h, sparse MMA q at tensor-memory column
// e + 4h + 2q): two k-steps per stage halve the per-stage work of the issuing
// thread against the MMAs'.  A commit with a CTA mask frees the stage in both
// CTAs and hands each accumulator to both epilogues, which scale by sw[n]
// sx[m] and round once.  Two accumulators alternate between items (2 x BN + 8
// metadata columns).
//
// Every mbarrier wait is bounded by %globaltimer; a CTA that gives up raises
// its own and its peer's abort flag, drains its copies and still meets its
// peer at the final cluster barrier, so both CTAs free tensor memory together.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "patch_cluster.cuh"
#include "patch_common.cuh"
#include "patch_internal.h"

namespace patchk {

namespace {

constexpr int kD8Threads = 352;   // warps 0 weights, 1 MMA, 6 X; 2-5 and 7-10 the two epilogue groups
constexpr int kD8Step = 128;      // columns (code bytes) per k-step
constexpr int kD8MaxStages = 8;
constexpr int kD8TabSteps = 224;  // k-steps per band (K <= 28672)
constexpr int kD8TabBytes = 2 * kD8TabSteps * 8;
constexpr int kD8TmemCols = 512;
constexpr int kD8SmemLimit = 232448;
constexpr int kD8TailBytes = 1024 + kD8TabBytes + 512;
constexpr uint64_t kD8WaitLimitNs = 2000000000ull;

constexpr int kD8MaxGroup = kDuoGroupMax;  // matrices sharing X in one launch

// One launch covers one matrix, or several that read the same X codes (the
// same K): their band pairs are numbered one after another (matrix i holds
// global pairs pair0[i] .. pair0[i+1]-1) and each keeps its own prefill
// table, packed bytes (tensor maps), row scales, output and status word.
struct D8Params {
    const uint64_t *table[kD8MaxGroup];  // prefill tables [bands][steps]
    const float *sw[kD8MaxGroup];
    int64_t N[kD8MaxGroup];
    void *Y[kD8MaxGroup];
    uint32_t *status[kD8MaxGroup];
    int32_t pair0[kD8MaxGroup + 1];
    int nmat;
    const float *sx;
    int64_t K, M;
    int steps, ttiles, items;
    int bn, half, stages, stage_bytes, aslot;
    int aslot_step;          // weight bytes reserved per k-step in a stage (aslot = 2 x this)
    int y_fp32;
};

// matrix holding global band pair gp
__device__ __forceinline__ int d8_mat_of_pair(const D8Params &p, int gp) {
    int i = 0;
    while (i + 1 < p.nmat && p.pair0[i + 1] <= gp) ++i;
    return i;
}

// Tensor maps over each packed buffer as rows of 2 KB: one k-step (8 rows
// dense, 5 rows 2:4) or two contiguous k-steps (16, 13 or 10 rows).
struct D8Maps {
    CUtensorMap x;
    CUtensorMap a_dense[kD8MaxGroup], a_sparse[kD8MaxGroup], a_dd[kD8MaxGroup], a_mixed[kD8MaxGroup],
        a_ss[kD8MaxGroup];
};

// one k-step's MMAs back to back: four dense K32, or two 2:4 K64 with the
// metadata columns e0 and e1; `accumulate` applies to the first only
__device__ __forceinline__ void mma_f8_pair_x4(uint32_t d_tmem, uint64_t a0, uint64_t a1, uint64_t a2, uint64_t a3,
                                               uint64_t b0, uint64_t b1, uint64_t b2, uint64_t b3, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        "setp.ne.b32 p, %10, 0;\n\t"
        "setp.eq.b32 t, %9, %9;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %5, %9, p;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %2, %6, %9, t;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %3, %7, %9, t;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %4, %8, %9, t;\n\t}\n" ::"r"(d_tmem),
        "l"(a0), "l"(a1), "l"(a2), "l"(a3), "l"(b0), "l"(b1), "l"(b2), "l"(b3), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_f8_sparse_pair_x2(uint32_t d_tmem, uint64_t a0, uint64_t a1, uint64_t b0,
                                                      uint64_t b1, uint32_t e0, uint32_t e1, uint32_t idesc,
                                                      uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        "setp.ne.b32 p, %8, 0;\n\t"
        "setp.eq.b32 t, %7, %7;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::f8f6f4 [%0], %1, %3, [%5], %7, p;\n\t"
        "tcgen05.mma.sp.cta_group::2.kind::f8f6f4 [%0], %2, %4, [%6], %7, t;\n\t}\n" ::"r"(d_tmem),
        "l"(a0), "l"(a1), "l"(b0), "l"(b1), "r"(e0), "r"(e1), "r"(idesc), "r"(accumulate)
        : "memory");
}

// kind::f8f6f4 instruction descriptor: A and B e4m3 (format 0), K-major, fp32
// D, M = 256, the given N; `sparse` sets the 2:4 flag (selector 0).
__host__ __device__ constexpr uint32_t idesc_e4m3_pair(int n, bool sparse) {
    return (sparse ? (1u << 2) : 0u) | (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(256 >> 4) << 24);
}

__device__ __forceinline__ void store_y(const D8Params &p, int mi, int64_t idx, float v) {
    if (p.y_fp32)
        static_cast<float *>(p.Y[mi])[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(p.Y[mi])[idx] = __float2bfloat16_rn(v);
}

__global__ void __launch_bounds__(kD8Threads, 1)
duo_fp8_kernel(const __grid_constant__ D8Maps maps, const __grid_constant__ D8Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = p.stages;
    uint64_t *tab_buf = reinterpret_cast<uint64_t *>(smem + S * p.stage_bytes);  // [2][224]
    uint64_t *full = tab_buf + 2 * kD8TabSteps;  // leader: all loads of both CTAs
    uint64_t *empty = full + kD8MaxStages;        // both: freed by the leader's commit
    uint64_t *acc_full = empty + kD8MaxStages;    // [2] both
    uint64_t *acc_empty = acc_full + 2;           // [2] leader: 4 warps x 2 CTAs
    uint64_t *tab_full = acc_empty + 2;           // [2] own table copies
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tab_full + 2);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    volatile uint32_t *never_flag = tmem_slot + 2;
    // [S]: bit h = k-step h of the stage is 2:4; bits 2-12 = where k-step 1's
    // bytes start in the weight slot (16-byte units)
    uint32_t *stage_word = tmem_slot + 4;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_rank();
    const int cl = blockIdx.x / 2, C = gridDim.x / 2;
    const int bn = p.bn, half = p.half;

    auto fetch_table = [&](int item, int buf) {
        const int gp = item / p.ttiles, mi = d8_mat_of_pair(p, gp);
        const int band = 2 * (gp - p.pair0[mi]) + static_cast<int>(rank);
        const uint32_t nb = static_cast<uint32_t>(p.steps) * 8u;
        mbar_arrive_expect_tx(&tab_full[buf], nb);
        bulk_g2s(tab_buf + buf * kD8TabSteps, p.table[mi] + static_cast<int64_t>(band) * p.steps, nb,
                 &tab_full[buf]);
    };
    auto give_up = [&]() {
        *abort_flag = 1u;
        st_cluster_u32(map_to_rank(const_cast<uint32_t *>(abort_flag), rank ^ 1u), 1u);
        for (int i = 0; i < p.nmat; ++i) atomicOr(p.status[i], kStatusTimeout);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kD8MaxStages; ++s) {
            mbar_init(&full[s], 2);  // the leader's weight and X producers
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 16);  // 8 epilogue warps x 2 CTAs
            mbar_init(&tab_full[b], 1);
        }
        *never_flag = 0u;
        // a matrix whose status is raised skips the whole launch
        uint32_t raised = 0u;
        for (int i = 0; i < p.nmat; ++i) raised |= *reinterpret_cast<volatile uint32_t *>(p.status[i]);
        *abort_flag = (raised & kStatusTimeout) ? 1u : 0u;
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kD8TmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.x);
        for (int i = 0; i < p.nmat; ++i) {
            prefetch_tmap(&maps.a_dense[i]);
            prefetch_tmap(&maps.a_sparse[i]);
            prefetch_tmap(&maps.a_dd[i]);
            prefetch_tmap(&maps.a_mixed[i]);
            prefetch_tmap(&maps.a_ss[i]);
        }
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers and tensor memory exist from here on
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;
    if (threadIdx.x == 0 && !skip) {
        for (int i = 0; i < 2 && cl + i * C < p.items; ++i) fetch_table(cl + i * C, i);
    }
    const int pairs = p.steps / 2;

    if (warp == 0) {
        if (lane == 0 && !skip) {
            // ----------------------------------------------- weight producer
            int it = 0;
            bool ok = true;
            int tabs = 0;
            for (int i = 0; i < 2 && cl + i * C < p.items; ++i) ++tabs;
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int buf = i & 1;
                if (!mbar_wait_bounded(&tab_full[buf], (i >> 1) & 1u, abort_flag, kD8WaitLimitNs)) {
                    ok = false;
                    break;
                }
                const uint64_t *tab = tab_buf + buf * kD8TabSteps;
                const int mi = d8_mat_of_pair(p, item / p.ttiles);  // the item's matrix
                for (int pr = 0; pr < pairs; ++pr) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kD8WaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    ++it;
                    const uint64_t e0 = tab[2 * pr], e1 = tab[2 * pr + 1];
                    const bool sp0 = (e0 & kEntrySparse) != 0, sp1 = (e1 & kEntrySparse) != 0;
                    const uint32_t b0 = sp0 ? kMetaBlockBytes + kSparseStepBytes : kDenseStepBytes;
                    const uint32_t b1 = sp1 ? kMetaBlockBytes + kSparseStepBytes : kDenseStepBytes;
                    const uint64_t f0 = (e0 & kEntryOffsetMask) - (sp0 ? kMetaBlockBytes : 0);
                    const uint64_t f1 = (e1 & kEntryOffsetMask) - (sp1 ? kMetaBlockBytes : 0);
                    // k-step 1 right behind k-step 0 in the slot; both bands of
                    // the pair agree in kinds and, the packer pairing their
                    // side copies too, in this placement
                    stage_word[s] = (sp0 ? 1u : 0u) | (sp1 ? 2u : 0u) | ((b0 >> 4) << 2);
                    // the leader arms its barrier for both CTAs' weight bytes
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (b0 + b1));
                    uint8_t *st = smem + s * p.stage_bytes;
                    if (f1 == f0 + b0) {
                        // contiguous: one copy of both k-steps
                        const CUtensorMap *am = (sp0 && sp1) ? &maps.a_ss[mi]
                                              : ((sp0 || sp1) ? &maps.a_mixed[mi] : &maps.a_dd[mi]);
                        tma2d_pair(st, am, 0, static_cast<int32_t>(f0 / 2048), map_to_rank(&full[s], 0));
                    } else {
                        tma2d_pair(st, sp0 ? &maps.a_sparse[mi] : &maps.a_dense[mi], 0,
                                   static_cast<int32_t>(f0 / 2048), map_to_rank(&full[s], 0));
                        tma2d_pair(st + b0, sp1 ? &maps.a_sparse[mi] : &maps.a_dense[mi], 0,
                                   static_cast<int32_t>(f1 / 2048), map_to_rank(&full[s], 0));
                    }
                }
                if (ok && cl + (i + 2) * C < p.items) {
                    fetch_table(cl + (i + 2) * C, buf);
                    ++tabs;
                }
            }
            for (int q = (tabs > 2 ? tabs - 2 : 0); q < tabs; ++q)
                mbar_wait_bounded(&tab_full[q & 1], (q >> 1) & 1u, never_flag, kD8WaitLimitNs / 4);
            if (!ok) give_up();
            // drain: the leader waits for the last phase of every stage (its
            // barrier counts both CTAs' loads); the peer until the leader's
            // MMAs have released each of its stages, or gives up
            for (int q = (it > S ? it - S : 0); q < it; ++q) {
                if (rank == 0)
                    mbar_wait_bounded(&full[q % S], (q / S) & 1u, never_flag, kD8WaitLimitNs / 4);
                else
                    mbar_wait_bounded(&empty[q % S], (q / S) & 1u, never_flag, kD8WaitLimitNs / 4);
            }
        }
    } else if (warp == 6) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------- X producer
            const uint32_t x_bytes = 2u * 2u * static_cast<uint32_t>(half) * kD8Step;  // both CTAs, 2 k-steps
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int tt = item % p.ttiles;
                for (int pr = 0; pr < pairs; ++pr) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kD8WaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    ++it;
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], x_bytes);
                    tma3d_pair(smem + s * p.stage_bytes + p.aslot, &maps.x, 0,
                               tt * bn + static_cast<int>(rank) * half, 2 * pr, map_to_rank(&full[s], 0));
                }
            }
            if (!ok) give_up();
        }
    } else if (warp == 1) {
        if (lane == 0 && !skip && rank == 0) {
            // ------------------------------------------------- MMA (leader)
            const uint32_t e_tmem = tmem_base + static_cast<uint32_t>(2 * bn);  // 4 columns per k-step
            const uint32_t id_dense = idesc_e4m3_pair(bn, false), id_sparse = idesc_e4m3_pair(bn, true);
            constexpr DescBase kDescDenseA = smem_desc_base(16, 1024, kSwizzle128B);
            constexpr DescBase kDescSparseA = smem_desc_base(16, 512, kSwizzle64B);
            constexpr DescBase kDescX = smem_desc_base(16, 1024, kSwizzle128B);
            constexpr DescBase kDescMeta = smem_desc_base(16, 128, kSwizzleNone);
            // the stage and its phase advance without division; addresses
            // in 16-byte units
            const uint32_t smem16 = smem_u32(smem) >> 4;
            const uint32_t stage16 = static_cast<uint32_t>(p.stage_bytes) >> 4;
            const uint32_t aslot16 = static_cast<uint32_t>(p.aslot) >> 4;
            const uint32_t xk16 = static_cast<uint32_t>(half * kD8Step) >> 4;  // one k-step of X rows
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int buf = i & 1;
                if (i >= 2 &&
                    !mbar_wait_bounded(&acc_empty[buf], ((i >> 1) & 1u) ^ 1u, abort_flag, kD8WaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * bn);
                for (int pr = 0; pr < pairs; ++pr) {
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, kD8WaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t w = stage_word[s];
                    const uint32_t slot16 = smem16 + static_cast<uint32_t>(s) * stage16;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t a16 = slot16 + (h ? ((w >> 2) & 0x7FFu) : 0u);
                        const uint32_t b16 = slot16 + aslot16 + static_cast<uint32_t>(h) * xk16;
                        const uint32_t acc = (pr == 0 && h == 0) ? 0u : 1u;
                        if (w & (1u << h)) {
                            const uint32_t e = e_tmem + 4u * static_cast<uint32_t>(h);
                            tmem_cp_pair_128x128b(e, desc_at(kDescMeta, a16));
                            const uint32_t v16 = a16 + kMetaBlockBytes / 16;
                            mma_f8_sparse_pair_x2(d_tmem, desc_at(kDescSparseA, v16), desc_at(kDescSparseA, v16 + 2),
                                                  desc_at(kDescX, b16), desc_at(kDescX, b16 + 4), e, e + 2, id_sparse,
                                                  acc);
                        } else {
                            mma_f8_pair_x4(d_tmem, desc_at(kDescDenseA, a16), desc_at(kDescDenseA, a16 + 2),
                                           desc_at(kDescDenseA, a16 + 4), desc_at(kDescDenseA, a16 + 6),
                                           desc_at(kDescX, b16), desc_at(kDescX, b16 + 2), desc_at(kDescX, b16 + 4),
                                           desc_at(kDescX, b16 + 6), id_dense, acc);
                        }
                    }
                    tc_commit_pair(&empty[s]);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                // fires once every MMA of the item has completed (also after a
                // failure, so no epilogue frees tensor memory under a running MMA)
                tc_commit_pair(&acc_full[buf]);
            }
            if (!ok) give_up();
        }
    } else if (!skip) {
        // ---------------------------------------------- epilogue (both CTAs)
        // two groups of four warps (one warp per TMEM lane quarter each)
        // take alternate 16-column chunks of an accumulator
        const int quad = warp % 4;
        const int grp = warp >= 7 ? 1 : 0;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        for (int i = 0;; ++i) {
            const int item = cl + i * C;
            if (item >= p.items) break;
            const int gp = item / p.ttiles, tt = item % p.ttiles;
            const int mi = d8_mat_of_pair(p, gp);
            const int bp = gp - p.pair0[mi];
            const int buf = i & 1;
            const bool ok = mbar_wait_bounded(&acc_full[buf], (i >> 1) & 1u, never_flag, kD8WaitLimitNs);
            tc_fence_after();
            if (!ok) {
                give_up();
                break;
            }
            const int64_t n = static_cast<int64_t>(2 * bp + static_cast<int>(rank)) * kBand + row;
            const int64_t m_base = static_cast<int64_t>(tt) * bn;
            const int m_valid = static_cast<int>(min(static_cast<int64_t>(bn), p.M - m_base));
            const float swn = __ldg(p.sw[mi] + n);
            const int64_t ld = p.N[mi];
            if (*abort_flag == 0) {
#pragma unroll 1
                for (int c0 = 16 * grp; c0 < m_valid; c0 += 32) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(buf * bn + c0), r);
                    // token scales of the chunk: lane l holds column l % 16's
                    const int ml = c0 + (lane & 15);
                    const float sxl = ml < m_valid ? __ldg(p.sx + m_base + ml) : 0.0f;
                    tmem_ld_wait();
                    int64_t idx = (m_base + c0) * ld + n;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const float sq = __shfl_sync(0xFFFFFFFFu, sxl, q);
                        if (c0 + q < m_valid) store_y(p, mi, idx, __uint_as_float(r[q]) * swn * sq);
                        idx += ld;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(map_to_rank(&acc_empty[buf], 0));
        }
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // the peer's MMAs and remote arrivals are all done
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kD8TmemCols);
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
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// the packed buffer as rows of 2 KB (256 x 8-byte elements), box of `box_rows`
bool encode_rows(EncodeTiledFn enc, CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    const cuuint64_t dims[2] = {256, rows};
    const cuuint64_t strides[1] = {2048};
    const cuuint32_t box[2] = {256, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t ensure_attributes() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(duo_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kD8SmemLimit);
    });
    return attr_err;
}

// clusters of two CTAs that fit on the device at once with `smem` bytes each
int max_clusters(int smem) {
    if (ensure_attributes() != cudaSuccess) return 0;
    static std::mutex mu;
    static int cached_smem = -1, cached = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cached_smem == smem) return cached;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kD8Threads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, duo_fp8_kernel, &cfg) != cudaSuccess) n = 0;
    cached_smem = smem;
    cached = n;
    return n;
}

}  // namespace

void preload_duo_fp8_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, duo_fp8_kernel);
}

DuoFp8Plan plan_duo_fp8(int64_t N, int64_t M, int num_sms, bool all_sparse) {
    DuoFp8Plan best{};
    const int64_t bpairs = (N / kBand) / 2;
    // shared memory per stage (two k-steps): the weight slot (two dense
    // k-steps, or metadata + codes twice when no k-step of the matrix is
    // dense) + BN/2 X rows of 128 B per k-step
    const int aslot_step = all_sparse ? kMetaBlockBytes + kSparseStepBytes : kDenseStepBytes;
    const int aslot = 2 * aslot_step;
    auto smem_for = [aslot](int bn, int *stages, int *stage_bytes) {
        *stage_bytes = aslot + 2 * (bn / 2) * kD8Step;
        *stages = std::min(kD8MaxStages, (kD8SmemLimit - kD8TailBytes) / *stage_bytes);
        return *stages * *stage_bytes + kD8TailBytes;
    };
    int st = 0, sb = 0;
    const int clusters_cap = max_clusters(smem_for(128, &st, &sb));
    if (clusters_cap < 1) return best;
    const int clusters = std::min(clusters_cap, num_sms / 2);
    // per SM per dense k-step: max(MMA cycles (4 x BN/2), shared-memory bytes
    // (weights and X half written by the copies and read by the MMAs) at
    // 128 B per cycle); the last wave counts whole
    double best_cost = 0;
    for (int bn = 240; bn >= 128; bn -= 16) {
        const int64_t tt = (M + bn - 1) / bn;
        const int64_t items = bpairs * tt;
        if (items > INT32_MAX) continue;  // items are counted in 32 bits
        const int64_t waves = (items + clusters - 1) / clusters;
        const double kstep = std::max(2.0 * bn, 2.0 * (aslot + 64.0 * bn) / 128.0);
        const double cost = static_cast<double>(waves) * kstep;
        if (best.bn == 0 || cost < best_cost) {
            best_cost = cost;
            best.bn = bn;
            best.ttiles = static_cast<int>(tt);
            best.items = static_cast<int>(items);
            best.clusters = static_cast<int>(std::min<int64_t>(clusters, items));
        }
    }
    best.smem = smem_for(best.bn, &best.stages, &best.stage_bytes);
    best.aslot = aslot;
    best.aslot_step = aslot_step;
    best.cost = best_cost;
    return best;
}

cudaError_t launch_duo_fp8_group(const Fp8Launch *gs, int count, const DuoFp8Plan &plan, cudaStream_t stream) {
    const cudaError_t attr_err = ensure_attributes();
    if (attr_err != cudaSuccess) return attr_err;
    if (count < 1 || count > kD8MaxGroup) return cudaErrorInvalidValue;
    const Fp8Launch &g = gs[0];
    const int64_t steps = g.K / kD8Step;
    if (plan.bn < 128 || plan.stages < 2 || plan.smem > kD8SmemLimit || plan.clusters < 1)
        return cudaErrorInvalidValue;
    if (steps % 2 != 0 || steps > kD8TabSteps) return cudaErrorInvalidValue;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    D8Maps maps;
    // X codes [M, K] uint8 row-major, viewed as (128 bytes, M rows, K/128
    // k-steps): box = this CTA's half of the token tile for both k-steps of a
    // stage, 128-byte swizzle, rows past M read as zero
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD8Step), static_cast<cuuint64_t>(g.M),
                                static_cast<cuuint64_t>(g.K / kD8Step)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(g.K), static_cast<cuuint64_t>(kD8Step)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kD8Step), static_cast<cuuint32_t>(plan.bn / 2), 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t *>(g.xq), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    constexpr uint32_t kRowsD = kDenseStepBytes / 2048, kRowsS = (kMetaBlockBytes + kSparseStepBytes) / 2048;
    D8Params p;
    int64_t pairs = 0;
    for (int i = 0; i < count; ++i) {
        const Fp8Launch &m = gs[i];
        // one X (codes and scales), one K, one output type; every matrix pairs its bands
        if (m.K != g.K || m.M != g.M || m.xq != g.xq || m.sx != g.sx || m.y_fp32 != g.y_fp32 ||
            (m.N / kBand) % 2 != 0 || !m.ptable || !m.packed_bytes || !m.sw || !m.Y || !m.status)
            return cudaErrorInvalidValue;
        // a matrix without dense k-steps only fits a plan sized for that
        if (!m.all_sparse && plan.aslot_step != kDenseStepBytes) return cudaErrorInvalidValue;
        const uint64_t rows = m.packed_bytes / 2048;  // packed + side copies, in 2 KB rows
        if (!encode_rows(enc, &maps.a_dense[i], m.packed, rows, kRowsD) ||
            !encode_rows(enc, &maps.a_sparse[i], m.packed, rows, kRowsS) ||
            !encode_rows(enc, &maps.a_dd[i], m.packed, rows, 2 * kRowsD) ||
            !encode_rows(enc, &maps.a_mixed[i], m.packed, rows, kRowsD + kRowsS) ||
            !encode_rows(enc, &maps.a_ss[i], m.packed, rows, 2 * kRowsS))
            return cudaErrorInvalidValue;
        p.table[i] = m.ptable;
        p.sw[i] = m.sw;
        p.N[i] = m.N;
        p.Y[i] = m.Y;
        p.status[i] = m.status;
        p.pair0[i] = static_cast<int32_t>(pairs);
        pairs += m.N / (2 * kBand);
    }
    for (int i = count; i < kD8MaxGroup; ++i) {
        maps.a_dense[i] = maps.a_dense[0];
        maps.a_sparse[i] = maps.a_sparse[0];
        maps.a_dd[i] = maps.a_dd[0];
        maps.a_mixed[i] = maps.a_mixed[0];
        maps.a_ss[i] = maps.a_ss[0];
        p.table[i] = nullptr;
        p.sw[i] = nullptr;
        p.N[i] = 0;
        p.Y[i] = nullptr;
        p.status[i] = nullptr;
    }
    for (int i = count; i <= kD8MaxGroup; ++i) p.pair0[i] = static_cast<int32_t>(pairs);
    if (static_cast<int64_t>(plan.items) != pairs * plan.ttiles) return cudaErrorInvalidValue;
    p.nmat = count;
    p.sx = g.sx;
    p.K = g.K;
    p.M = g.M;
    p.steps = static_cast<int>(steps);
    p.ttiles = plan.ttiles;
    p.items = plan.items;
    p.bn = plan.bn;
    p.half = plan.bn / 2;
    p.stages = plan.stages;
    p.stage_bytes = plan.stage_bytes;
    p.aslot = plan.aslot;
    p.aslot_step = plan.aslot_step;
    p.y_fp32 = g.y_fp32;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * plan.clusters));
    cfg.blockDim = dim3(kD8Threads);
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, duo_fp8_kernel, maps, p);
    if (err == cudaSuccess) note_launches(1);
    return err;
}

cudaError_t launch_duo_fp8(const Fp8Launch &g, const DuoFp8Plan &plan, cudaStream_t stream) {
    return launch_duo_fp8_group(&g, 1, plan, stream);
}

}  // namespace patchk
