// Two-SM hybrid GEMM for prefill: tcgen05 with cta_group::2 (sm_100a).
//
// Same product as the other GEMM paths, Y = X * W_eff^T ("PATCH: Learnable
// Tile-level Hybrid Sparsity for LLMs", section 2, inference and deployment),
// for matrices whose paired bands agree in tile type at every k-step (every
// tile dense, every tile 2:4, or any map whose bands 2p and 2p+1 match).
//
// Why.  The tensor core reads its operands from shared memory and the copies
// write there too, about 128 B per cycle per SM in all.  With one CTA per MMA
// every SM must hold the whole token tile; with cta_group::2 a CTA pair runs
// M = 256 MMAs (one 128-row band per SM) and each SM holds HALF of the token
// tile: per dense 64-column k-step an SM moves 32 KB + 128 B per token
// (copies in + operand reads) for 2 x BN MMA cycles, about 97 % of the MMA rate
// at BN = 240, and a 2:4 k-step about 64 % of the sparse rate.  Both bands of
// an instruction must be of one kind, hence the matching requirement.
//
// Work item = (band pair, token tile of BN tokens); clusters of two CTAs take
// items c, c + C, ...; CTA rank r owns band 2p + r and tokens
// [r BN/2, (r+1) BN/2) of the tile.  Stage = one k-pair (128 columns): this
// SM's band (ONE TMA load of the pair's 18-32 KB, through tensor maps over
// the packed buffer in 2 KB rows) and its half of the X tile for both k-steps
// (ONE 3-D TMA load, 128-byte swizzle, rows past M zero).  Few, large copies:
// a copy costs ~0.16 us of issue-to-issue time whatever its size up to 16 KB.  All loads of both CTAs complete on the
// leader's stage mbarrier (TMA .cta_group::2); the weights and the X tiles
// are issued by two threads in different warps, since the copies one thread
// issues are processed largely one after another.  The leader's single MMA thread
// issues tcgen05.mma(.sp).cta_group::2 M256 x BN; tcgen05.commit with a CTA
// mask frees the stage in both CTAs and hands the accumulator to both
// epilogues.  Each SM holds its band's 128 x BN fp32 accumulator; two
// accumulators alternate between items (2 x 240 + 4 metadata columns).
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

constexpr int kDuoMaxGroup = kDuoGroupMax;     // matrices sharing X in one launch
constexpr int kDuoThreads = 352;   // warps 0 weights, 1 MMA, 6 X tiles; 2-5 and 7-10 the two epilogue groups
constexpr int kDuoMaxStages = 8;
constexpr int kDuoTabSteps = 448;                      // k-steps per band (K <= 28672)
constexpr int kDuoTabBytes = 2 * kDuoTabSteps * 8;     // two items of one band
constexpr int kDuoAslotMax = 2 * kDenseStepBytes;  // one k-pair of weights, at most
constexpr int kDuoTmemCols = 512;
constexpr int kDuoSmemLimit = 232448;
constexpr int kDuoTailBytes = 1024 + kDuoTabBytes + 512;
constexpr uint64_t kDuoWaitLimitNs = 2000000000ull;

// One launch covers one matrix, or several that read the same X (the same K):
// their band pairs are numbered one after another (matrix i holds global
// pairs pair0[i] .. pair0[i+1]-1) and each keeps its own prefill table,
// packed bytes (tensor maps), output, status and ready words.
struct DuoParams {
    const uint64_t *table[kDuoMaxGroup];  // prefill tables
    int64_t N[kDuoMaxGroup];
    void *Y[kDuoMaxGroup];
    uint32_t *status[kDuoMaxGroup];
    const uint32_t *ready[kDuoMaxGroup];
    int32_t pair0[kDuoMaxGroup + 1];
    int nmat;
    int64_t K, M;
    int nsteps, ttiles, items;
    int bn, half, stages, stage_bytes;
    int aslot;  // bytes of a stage's weight slot: the largest k-pair of the matrices
    int y_fp32;
    int stall_first_kstep;  // failure-detection test hook
};

// matrix holding global band pair gp
__device__ __forceinline__ int duo_mat_of_pair(const DuoParams &p, int gp) {
    int i = 0;
    while (i + 1 < p.nmat && p.pair0[i + 1] <= gp) ++i;
    return i;
}

__device__ __forceinline__ void store_y(const DuoParams &p, int mi, int64_t idx, float v) {
    if (p.y_fp32)
        static_cast<float *>(p.Y[mi])[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(p.Y[mi])[idx] = __float2bfloat16_rn(v);
}

// Tensor maps over the packed buffer viewed as rows of 2 KB (256 x 8-byte
// elements); the box is one packed k-pair: 16 rows (two dense k-steps), 13
// (one dense + metadata + one 2:4) or 9 (metadata + two 2:4).  X is viewed
// as (64 columns, M rows, K/64 k-steps) with a box of both k-steps of a pair.
struct DuoMaps {
    CUtensorMap x;
    CUtensorMap a_dd[kDuoMaxGroup], a_mixed[kDuoMaxGroup], a_ss[kDuoMaxGroup];
};

__global__ void __launch_bounds__(kDuoThreads, 1)
duo_gemm_kernel(const __grid_constant__ DuoMaps maps, const __grid_constant__ DuoParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = p.stages;
    uint64_t *tab_buf = reinterpret_cast<uint64_t *>(smem + S * p.stage_bytes);  // [2][448]
    uint64_t *full = tab_buf + 2 * kDuoTabSteps;  // leader: all loads of both CTAs
    uint64_t *empty = full + kDuoMaxStages;        // both: freed by the leader's commit
    uint64_t *acc_full = empty + kDuoMaxStages;    // [2] both
    uint64_t *acc_empty = acc_full + 2;            // [2] leader: 4 warps x 2 CTAs
    uint64_t *tab_full = acc_empty + 2;            // [2] own table copies
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tab_full + 2);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    volatile uint32_t *never_flag = tmem_slot + 2;
    // [S]: the stage's k-pair for the MMA thread, packed by the weight producer:
    // bits 0-10 / 11-21 = k-step 0 / 1 values' offset in the stage (16-byte
    // units), bits 22 / 23 = k-step 0 / 1 is 2:4, bits 24 / 25 = its
    // metadata block precedes it
    uint32_t *stage_word = tmem_slot + 4;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_rank();
    const int cl = blockIdx.x / 2, C = gridDim.x / 2;
    const int bn = p.bn, half = p.half;

    auto fetch_table = [&](int item, int buf) {
        const int gp = item / p.ttiles, mi = duo_mat_of_pair(p, gp);
        const int band = 2 * (gp - p.pair0[mi]) + static_cast<int>(rank);
        const uint32_t nb = static_cast<uint32_t>(p.nsteps) * 8u;
        mbar_arrive_expect_tx(&tab_full[buf], nb);
        bulk_g2s(tab_buf + buf * kDuoTabSteps, p.table[mi] + static_cast<int64_t>(band) * p.nsteps, nb,
                 &tab_full[buf]);
    };
    auto give_up = [&]() {
        *abort_flag = 1u;
        st_cluster_u32(map_to_rank(const_cast<uint32_t *>(abort_flag), rank ^ 1u), 1u);
        for (int i = 0; i < p.nmat; ++i) atomicOr(p.status[i], kStatusTimeout);
    };

    if (threadIdx.x == 0) {
        pdl_trigger();
        // weights are final once the packer's ready flag is seen; otherwise
        // (the packer may be the kernel just before) wait first
        bool all_ready = true;
        for (int i = 0; i < p.nmat; ++i) all_ready = all_ready && ld_acquire_gpu(p.ready[i]) != 0u;
        if (!all_ready) pdl_wait();
        for (int s = 0; s < kDuoMaxStages; ++s) {
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
        tmem_alloc_pair(tmem_slot, kDuoTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.x);
        for (int i = 0; i < p.nmat; ++i) {
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
    // a CTA that starts with its status raised skips all work but still meets
    // its peer at the end; the peer's waits then run out and it does the same
    const bool skip = *abort_flag != 0;
    if (threadIdx.x == 0 && !skip) {
        for (int i = 0; i < 2 && cl + i * C < p.items; ++i) fetch_table(cl + i * C, i);
    }

    if (warp == 0) {
        if (lane == 0 && !skip) {
            // ------------------------------------------------------ producer
            // (both CTAs; every load completes on the LEADER's stage barrier)
            int it = 0;
            bool ok = true;
            int tabs = 0;
            for (int i = 0; i < 2 && cl + i * C < p.items; ++i) ++tabs;
            // weights need no wait once the packer's ready flag was seen;
            // otherwise thread 0 already passed griddepcontrol.wait
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int buf = i & 1;
                if (!mbar_wait_bounded(&tab_full[buf], (i >> 1) & 1u, abort_flag, kDuoWaitLimitNs)) {
                    ok = false;
                    break;
                }
                const uint64_t *tab = tab_buf + buf * kDuoTabSteps;
                const int mi = duo_mat_of_pair(p, item / p.ttiles);  // the item's matrix
                for (int pr = 0; pr < p.nsteps / 2; ++pr) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kDuoWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    const uint64_t e0 = tab[2 * pr], e1 = tab[2 * pr + 1];
                    const uint64_t first = (e0 & kEntryOffsetMask) - ((e0 & kEntryMeta) ? kMetaBlockBytes : 0);
                    const uint64_t end = (e1 & kEntryOffsetMask) +
                                         ((e1 & kEntrySparse) ? kSparseStepBytes : kDenseStepBytes);
                    const uint32_t a_bytes = static_cast<uint32_t>(end - first);  // 32, 26 or 18 KB
                    stage_word[s] = static_cast<uint32_t>(((e0 & kEntryOffsetMask) - first) >> 4) |
                                    (static_cast<uint32_t>(((e1 & kEntryOffsetMask) - first) >> 4) << 11) |
                                    ((e0 & kEntrySparse) ? 1u << 22 : 0u) | ((e1 & kEntrySparse) ? 1u << 23 : 0u) |
                                    ((e0 & kEntryMeta) ? 1u << 24 : 0u) | ((e1 & kEntryMeta) ? 1u << 25 : 0u);
                    ++it;
                    if (p.stall_first_kstep && blockIdx.x == 0 && it == 1) continue;  // never lands
                    // the two bands of a pair agree in kind and metadata placement,
                    // so the leader arms the barrier for both CTAs' weight bytes
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * a_bytes);
                    const CUtensorMap *am = a_bytes == 2u * kDenseStepBytes ? &maps.a_dd[mi]
                                          : (a_bytes == 2u * kSparseStepBytes + kMetaBlockBytes ? &maps.a_ss[mi]
                                                                                               : &maps.a_mixed[mi]);
                    tma2d_pair(smem + s * p.stage_bytes, am, 0, static_cast<int32_t>(first / 2048),
                               map_to_rank(&full[s], 0));
                }
                if (ok && cl + (i + 2) * C < p.items) {
                    fetch_table(cl + (i + 2) * C, buf);
                    ++tabs;
                }
            }
            for (int q = (tabs > 2 ? tabs - 2 : 0); q < tabs; ++q)
                mbar_wait_bounded(&tab_full[q & 1], (q >> 1) & 1u, never_flag, kDuoWaitLimitNs / 4);
            if (!ok) give_up();
            // Drain.  The leader waits for the last phase of every stage (its
            // barrier counts both CTAs' loads); the peer waits until the
            // leader's MMA has released each of its stages, or gives up.
            for (int q = (it > S ? it - S : 0); q < it; ++q) {
                if (p.stall_first_kstep && blockIdx.x == 0 && q == 0) continue;  // never armed
                if (rank == 0)
                    mbar_wait_bounded(&full[q % S], (q / S) & 1u, never_flag, kDuoWaitLimitNs / 4);
                else
                    mbar_wait_bounded(&empty[q % S], (q / S) & 1u, never_flag, kDuoWaitLimitNs / 4);
            }
        }
    } else if (warp == 6) {
        if (lane == 0 && !skip) {
            // ------------------------------------------------ X producer
            // (both CTAs; a second issuing thread: copies from one thread
            // are processed largely one after another)
            pdl_wait();  // X may still be written by the kernel before
            const uint32_t x_bytes = 2u * 2u * static_cast<uint32_t>(half) * kStep * 2u;  // both CTAs, 2 k-steps
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int tt = item % p.ttiles;
                for (int pr = 0; pr < p.nsteps / 2; ++pr) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kDuoWaitLimitNs)) {
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
            const uint32_t e_tmem = tmem_base + static_cast<uint32_t>(2 * bn);
            const uint32_t idesc_dense = idesc_pair(bn, false);
            const uint32_t idesc_sparse[2] = {idesc_pair(bn, true, 0), idesc_pair(bn, true, 1)};
            constexpr DescBase kDescDenseA = smem_desc_base(16, 1024, kSwizzle128B);
            constexpr DescBase kDescSparseA = smem_desc_base(16, 512, kSwizzle64B);
            constexpr DescBase kDescX = smem_desc_base(16, 1024, kSwizzle128B);
            constexpr DescBase kDescMeta = smem_desc_base(16, 128, kSwizzleNone);
            // the stage and its phase advance without division; a stage's
            // shared-memory addresses in 16-byte units
            const uint32_t smem16 = smem_u32(smem) >> 4;
            const uint32_t stage16 = static_cast<uint32_t>(p.stage_bytes) >> 4;
            const uint32_t aslot16 = static_cast<uint32_t>(p.aslot) >> 4;
            const uint32_t xk16 = static_cast<uint32_t>(half * kStep * 2) >> 4;  // one k-step of X rows
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int buf = i & 1;
                if (i >= 2 &&
                    !mbar_wait_bounded(&acc_empty[buf], ((i >> 1) & 1u) ^ 1u, abort_flag, kDuoWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * bn);
                for (int pr = 0; pr < p.nsteps / 2; ++pr) {
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, kDuoWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t w = stage_word[s];
                    const uint32_t slot16 = smem16 + static_cast<uint32_t>(s) * stage16;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint32_t a16 = slot16 + ((w >> (11 * h)) & 0x7FFu);
                        const uint32_t b16 = slot16 + aslot16 + static_cast<uint32_t>(h) * xk16;
                        const bool fresh = pr == 0 && h == 0;
                        if (w & (1u << (22 + h))) {
                            if (w & (1u << (24 + h)))
                                tmem_cp_pair_128x128b(e_tmem, desc_at(kDescMeta, a16 - kMetaBlockBytes / 16));
                            mma_sparse_pair_x2(d_tmem, desc_at(kDescSparseA, a16), desc_at(kDescSparseA, a16 + 2),
                                               desc_at(kDescX, b16), desc_at(kDescX, b16 + 4), e_tmem + 2 * h,
                                               idesc_sparse[0], idesc_sparse[1], fresh ? 0u : 1u);
                        } else {
                            mma_dense_pair_x4(d_tmem, desc_at(kDescDenseA, a16), desc_at(kDescDenseA, a16 + 2),
                                              desc_at(kDescDenseA, a16 + 4), desc_at(kDescDenseA, a16 + 6),
                                              desc_at(kDescX, b16), desc_at(kDescX, b16 + 2), desc_at(kDescX, b16 + 4),
                                              desc_at(kDescX, b16 + 6), idesc_dense, fresh ? 0u : 1u);
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
        pdl_wait();  // Y may still be read by an earlier kernel
        const int quad = warp % 4;
        const int grp = warp >= 7 ? 1 : 0;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        for (int i = 0;; ++i) {
            const int item = cl + i * C;
            if (item >= p.items) break;
            const int gp = item / p.ttiles, tt = item % p.ttiles;
            const int mi = duo_mat_of_pair(p, gp);
            const int bp = gp - p.pair0[mi];
            const int buf = i & 1;
            const bool ok = mbar_wait_bounded(&acc_full[buf], (i >> 1) & 1u, never_flag, kDuoWaitLimitNs);
            tc_fence_after();
            if (!ok) {
                give_up();
                break;
            }
            const int64_t n = static_cast<int64_t>(2 * bp + static_cast<int>(rank)) * kBand + row;
            const int64_t m_base = static_cast<int64_t>(tt) * bn;
            const int m_valid = static_cast<int>(min(static_cast<int64_t>(bn), p.M - m_base));
            if (*abort_flag == 0) {
#pragma unroll 1
                for (int c0 = 16 * grp; c0 < m_valid; c0 += 32) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(buf * bn + c0), r);
                    tmem_ld_wait();
                    const int64_t ld = p.N[mi];
                    int64_t idx = (m_base + c0) * ld + n;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        if (c0 + q < m_valid) store_y(p, mi, idx, __uint_as_float(r[q]));
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
    if (warp == 1) tmem_dealloc_pair(tmem_base, kDuoTmemCols);
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

// the packed buffer as rows of 2 KB (256 x 8-byte elements), box of `box_rows`
bool encode_rows(EncodeTiledFn enc, CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    const cuuint64_t dims[2] = {256, rows};
    const cuuint64_t strides[1] = {2048};
    const cuuint32_t box[2] = {256, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t ensure_duo_attributes() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(duo_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kDuoSmemLimit);
    });
    return attr_err;
}

// clusters of two CTAs that fit on the device at once with `smem` bytes each
int duo_max_clusters(int smem) {
    if (ensure_duo_attributes() != cudaSuccess) return 0;
    static std::mutex mu;
    static int cached_smem = -1, cached = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cached_smem == smem) return cached;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kDuoThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, duo_gemm_kernel, &cfg) != cudaSuccess) n = 0;
    cached_smem = smem;
    cached = n;
    return n;
}

}  // namespace

double duo_kstep_cycles(int bn) {
    // per SM per dense k-step: max(MMA 2 BN cycles, shared-memory traffic
    // (16 KB + 64 B per token in, the same again read) at 128 B per cycle)
    return std::max(2.0 * bn, 256.0 + bn);
}

void preload_duo_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, duo_gemm_kernel);
}

DuoPlan plan_duo_gemm(int64_t N, int64_t M, int num_sms, int max_pair_bytes) {
    DuoPlan best{};
    const int64_t bpairs = (N / kBand) / 2;
    // shared memory per stage: 16 KB of weights + BN/2 tokens x 128 B
    // a matrix without dense k-pairs needs only an 18 KB weight slot, which
    // leaves room for one more stage
    const int aslot = std::min(kDuoAslotMax, (std::max(max_pair_bytes, 2048) + 1023) / 1024 * 1024);
    auto smem_for = [aslot](int bn, int *stages, int *stage_bytes) {
        *stage_bytes = aslot + 2 * (bn / 2) * kStep * 2;
        *stages = std::min(kDuoMaxStages, (kDuoSmemLimit - kDuoTailBytes) / *stage_bytes);
        return *stages * *stage_bytes + kDuoTailBytes;
    };
    int st = 0, sb = 0;
    const int clusters_cap = duo_max_clusters(smem_for(240, &st, &sb));
    if (clusters_cap < 1) return best;  // bn = 0: not usable
    const int clusters = std::min(clusters_cap, num_sms / 2);
    double best_cost = 0;
    for (int bn = 240; bn >= 128; bn -= 16) {
        const int64_t tt = (M + bn - 1) / bn;
        const int64_t items = bpairs * tt;
        if (items > INT32_MAX) continue;  // items are counted in 32 bits
        const int64_t waves = (items + clusters - 1) / clusters;
        const double cost = static_cast<double>(waves) * duo_kstep_cycles(bn);
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
    // the same work in per-SM units as the band-pair kernel's estimate: a
    // cluster item covers two SMs, so compare per-SM cycles
    best.cost = best_cost;
    return best;
}

cudaError_t launch_duo_group(const GemmLaunch *gs, int count, const DuoPlan &plan, cudaStream_t stream) {
    const cudaError_t attr_err = ensure_duo_attributes();
    if (attr_err != cudaSuccess) return attr_err;
    if (count < 1 || count > kDuoMaxGroup) return cudaErrorInvalidValue;
    if (plan.stages < 2 || plan.smem > kDuoSmemLimit || plan.clusters < 1) return cudaErrorInvalidValue;
    const GemmLaunch &g = gs[0];
    if (g.K / kStep > kDuoTabSteps) return cudaErrorInvalidValue;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    DuoMaps maps;
    // X [M,K] as (64 columns, M rows, K/64 k-steps); box = this CTA's half of
    // the token tile for both k-steps of a pair; rows past M read as zero
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kStep), static_cast<cuuint64_t>(g.M),
                                static_cast<cuuint64_t>(g.K / kStep)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(g.K) * 2, static_cast<cuuint64_t>(kStep) * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kStep), static_cast<cuuint32_t>(plan.bn / 2), 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(g.X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    DuoParams p;
    int64_t pairs = 0;
    for (int i = 0; i < count; ++i) {
        const GemmLaunch &m = gs[i];
        // one X, one K, one output type; every matrix pairs its bands
        if (m.K != g.K || m.M != g.M || m.X != g.X || m.y_fp32 != g.y_fp32 || (m.N / kBand) % 2 != 0 ||
            !m.packed_rows || !m.ptable || !m.Y || !m.status || !m.ready)
            return cudaErrorInvalidValue;
        const uint64_t rows = m.packed_rows / 16;  // 2 KB rows
        if (!encode_rows(enc, &maps.a_dd[i], m.packed, rows, 2 * kDenseStepBytes / 2048) ||
            !encode_rows(enc, &maps.a_mixed[i], m.packed, rows,
                         (kDenseStepBytes + kMetaBlockBytes + kSparseStepBytes) / 2048) ||
            !encode_rows(enc, &maps.a_ss[i], m.packed, rows, (kMetaBlockBytes + 2 * kSparseStepBytes) / 2048))
            return cudaErrorInvalidValue;
        p.table[i] = m.ptable;  // the prefill table: the bands of every pair agree in type
        p.N[i] = m.N;
        p.Y[i] = m.Y;
        p.status[i] = m.status;
        p.ready[i] = m.ready;
        p.pair0[i] = static_cast<int32_t>(pairs);
        pairs += m.N / (2 * kBand);
    }
    for (int i = count; i < kDuoMaxGroup; ++i) {
        maps.a_dd[i] = maps.a_dd[0];
        maps.a_mixed[i] = maps.a_mixed[0];
        maps.a_ss[i] = maps.a_ss[0];
        p.table[i] = nullptr;
        p.N[i] = 0;
        p.Y[i] = nullptr;
        p.status[i] = nullptr;
        p.ready[i] = nullptr;
    }
    for (int i = count; i <= kDuoMaxGroup; ++i) p.pair0[i] = static_cast<int32_t>(pairs);
    p.nmat = count;
    p.K = g.K;
    p.M = g.M;
    p.nsteps = static_cast<int>(g.K / kStep);
    p.ttiles = plan.ttiles;
    p.items = plan.items;
    if (static_cast<int64_t>(p.items) != pairs * plan.ttiles) return cudaErrorInvalidValue;
    p.bn = plan.bn;
    p.half = plan.bn / 2;
    p.stages = plan.stages;
    p.stage_bytes = plan.stage_bytes;
    p.aslot = plan.aslot;
    p.y_fp32 = g.y_fp32;
    p.stall_first_kstep = g.stall_first_kstep;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * plan.clusters));
    cfg.blockDim = dim3(kDuoThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaError_t err = cudaLaunchKernelEx(&cfg, duo_gemm_kernel, maps, p);
    if (err == cudaSuccess) note_launches(1);
    return err;
}

cudaError_t launch_duo_gemm(const GemmLaunch &g, const DuoPlan &plan, cudaStream_t stream) {
    return launch_duo_group(&g, 1, plan, stream);
}

}  // namespace patchk
