// Two-SM, four-band hybrid GEMM for prefill: tcgen05 with cta_group::2 (sm_100a).
//
// Same product as the other GEMM paths, Y = X * W_eff^T ("PATCH: Learnable
// Tile-level Hybrid Sparsity for LLMs", section 2, inference and deployment:
// dense tiles on the dense tensor-core path, 2:4 tiles on the sparse one).
//
// Why.  The tensor core reads its operands from shared memory and the copies
// write there too, about 128 B per cycle per SM in all.  In the two-SM kernel
// (csrc/prefill_duo.cu) each SM holds one band and half of a token tile; per
// 64-column k-step it moves 32 KB of weights and 128 B per token of X for
// 2 x BN MMA cycles (dense), and a 2:4 k-step, at half the MMA time, is bound
// by that traffic.  Here each SM holds TWO bands that share its half of the
// token tile: two M = 256 instructions per k-step (bands 4q+2j on the leader
// and 4q+2j+1 on its peer, j = 0, 1) read the same X half, so per dense
// k-step an SM moves 64 KB of weights + 192 B per token for 4 x BN MMA
// cycles (MMA-bound at BN = 240), and a 2:4 k-step about 36 KB + 192 B per
// token for 2 x BN cycles (about 0.75 of the sparse rate instead of about
// 0.6).
//
// Work item = (band quad q, token tile of BN tokens); clusters of two CTAs
// take items c, c + C, ...; CTA rank r owns bands 4q + r (pair 0) and
// 4q + 2 + r (pair 1) and tokens [r BN/2, (r+1) BN/2) of the tile.  The bands
// of a pair come from the PREFILL table, whose pairs (2p, 2p+1) agree in type
// at every k-step (the packer gives a band a dense copy of a k-pair where its
// partner differs), so one instruction kind serves both CTAs.  A stage is one
// k-step: each CTA loads its two bands' k-step (TMA over the packed buffer in
// 2 KB rows: 16 KB dense, 2 KB metadata + 8 KB kept values, or 8 KB) and its
// half of the X tile (TMA, 128-byte swizzle, rows past M zero); every load of
// both CTAs completes on the leader's stage mbarrier (TMA .cta_group::2).
// Each band slot and X have an issuing thread of their own (warps 0, 3, 2):
// the copies one thread issues are processed largely one after another, at
// about 0.16 us each, which for two weight copies per k-step from one thread
// would exceed a 2:4 k-step's MMA time.  The leader's
// MMA thread issues, per pair, 4 dense M256 x BN x K16 or 2 sparse
// M256 x BN x K32 (after one tcgen05.cp of the pair's metadata block into 4
// TMEM columns when the k-pair starts); tcgen05.commit with a CTA mask frees
// the stage in both CTAs and hands the accumulators to both epilogues.  Each
// SM holds two 128 x BN fp32 accumulators (one per pair; 2 x BN + 8 of the
// 512 TMEM columns), drained by 8 epilogue warps before the next item.
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

constexpr int kQdThreads = 384;     // 12 warps: producers 0, 3 (weights) and 2 (X), MMA 1, epilogue 4..11
constexpr int kQdMaxStages = 6;
constexpr int kQdTabSteps = 448;                           // k-steps per band (K <= 28672)
constexpr int kQdTabBytes = 2 * 2 * kQdTabSteps * 8;       // two items x two bands
constexpr int kQdAslot = kDenseStepBytes;                  // one band's k-step, at most
constexpr int kQdTmemCols = 512;
constexpr int kQdSmemLimit = 232448;
constexpr int kQdTailBytes = 1024 + kQdTabBytes + 512;
constexpr int kQdEpiWarps = 8;
constexpr uint64_t kQdWaitLimitNs = 2000000000ull;

struct QuadParams {
    const uint64_t *ptable;
    int64_t N, K, M;
    int nsteps, bands, quads, ttiles, items;
    int bn, half, stages, stage_bytes;
    void *Y;
    int y_fp32;
    uint32_t *status;
    const uint32_t *ready;
    int stall_first_kstep;  // failure-detection test hook
};

// Tensor maps over the packed buffer viewed as rows of 2 KB; the box is one
// band's k-step: 8 rows (dense), 5 (metadata + kept values), 4 (kept values).
struct QuadMaps {
    CUtensorMap x, a_dense, a_meta, a_sparse;
};

__device__ __forceinline__ void store_y(const QuadParams &p, int64_t idx, float v) {
    if (p.y_fp32)
        static_cast<float *>(p.Y)[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(p.Y)[idx] = __float2bfloat16_rn(v);
}

// bytes a band's k-step occupies in its stage slot, and its first packed byte
__device__ __forceinline__ uint32_t kstep_bytes(uint64_t e) {
    return (e & kEntrySparse) ? kSparseStepBytes + ((e & kEntryMeta) ? kMetaBlockBytes : 0u)
                              : static_cast<uint32_t>(kDenseStepBytes);
}
__device__ __forceinline__ uint64_t kstep_first(uint64_t e) {
    return (e & kEntryOffsetMask) - ((e & kEntryMeta) ? kMetaBlockBytes : 0u);
}

__global__ void __launch_bounds__(kQdThreads, 1)
quad_gemm_kernel(const __grid_constant__ QuadMaps maps, const __grid_constant__ QuadParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = p.stages;
    uint64_t *tab_buf = reinterpret_cast<uint64_t *>(smem + S * p.stage_bytes);  // [2 items][2 bands][448]
    uint64_t *full = tab_buf + 2 * 2 * kQdTabSteps;  // leader: all loads of both CTAs
    uint64_t *empty = full + kQdMaxStages;            // both: freed by the leader's commit
    uint64_t *acc_full = empty + kQdMaxStages;        // both
    uint64_t *acc_empty = acc_full + 1;               // leader: 8 warps x 2 CTAs
    uint64_t *tab_full = acc_empty + 1;               // [2 buffers][2 slots] own table copies
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tab_full + 4);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    volatile uint32_t *never_flag = tmem_slot + 2;
    uint64_t *stage_info = reinterpret_cast<uint64_t *>(tmem_slot + 4);  // [S][2]: the leader's entries

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t rank = cluster_rank();
    const int cl = blockIdx.x / 2, C = gridDim.x / 2;
    const int bn = p.bn, half = p.half;

    // pairs of an item: pair 1 is absent in a last quad of only two bands
    auto pairs_of = [&](int item) { return (4 * (item / p.ttiles) + 3 < p.bands) ? 2 : 1; };
    auto band_of = [&](int item, int j) { return 4 * (item / p.ttiles) + 2 * j + static_cast<int>(rank); };
    // slot j's table of an item (nothing for an absent pair: a plain arrival)
    auto fetch_table = [&](int item, int buf, int j) {
        uint64_t *bar = &tab_full[buf * 2 + j];
        if (j >= pairs_of(item)) {
            mbar_arrive(bar);
            return;
        }
        const uint32_t nb = static_cast<uint32_t>(p.nsteps) * 8u;
        mbar_arrive_expect_tx(bar, nb);
        bulk_g2s(tab_buf + (buf * 2 + j) * kQdTabSteps,
                 p.ptable + static_cast<int64_t>(band_of(item, j)) * p.nsteps, nb, bar);
    };
    auto give_up = [&]() {
        *abort_flag = 1u;
        st_cluster_u32(map_to_rank(const_cast<uint32_t *>(abort_flag), rank ^ 1u), 1u);
        atomicOr(p.status, kStatusTimeout);
    };

    if (threadIdx.x == 0) {
        pdl_trigger();
        // weights are final once the packer's ready flag is seen; otherwise
        // (the packer may be the kernel just before) wait first
        if (ld_acquire_gpu(p.ready) == 0u) pdl_wait();
        for (int s = 0; s < kQdMaxStages; ++s) {
            mbar_init(&full[s], 3);  // the leader's two weight producers and its X producer
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * kQdEpiWarps);
        for (int b = 0; b < 4; ++b) mbar_init(&tab_full[b], 1);
        *never_flag = 0u;
        *abort_flag = (*reinterpret_cast<volatile uint32_t *>(p.status) & kStatusTimeout) ? 1u : 0u;
        fence_mbar_init_cluster();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kQdTmemCols);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&maps.x);
        prefetch_tmap(&maps.a_dense);
        prefetch_tmap(&maps.a_meta);
        prefetch_tmap(&maps.a_sparse);
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers and tensor memory exist from here on
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // a CTA that starts with its status raised skips all work but still meets
    // its peer at the end; the peer's waits then run out and it does the same
    const bool skip = *abort_flag != 0;

    if (warp == 0 || warp == 3) {
        if (lane == 0 && !skip) {
            // ---------------------------------------- weight producer, slot j
            // (both CTAs; every load completes on the LEADER's stage barrier)
            const int j = warp == 0 ? 0 : 1;
            int it = 0;
            bool ok = true;
            int tabs = 0;
            for (int i = 0; i < 2 && cl + i * C < p.items; ++i) {
                fetch_table(cl + i * C, i, j);
                ++tabs;
            }
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int buf = i & 1;
                const bool live = j < pairs_of(item);
                if (!mbar_wait_bounded(&tab_full[buf * 2 + j], (i >> 1) & 1u, abort_flag, kQdWaitLimitNs)) {
                    ok = false;
                    break;
                }
                const uint64_t *tab = tab_buf + (buf * 2 + j) * kQdTabSteps;
                for (int c = 0; c < p.nsteps; ++c) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kQdWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    const uint64_t e = live ? tab[c] : 0ull;
                    stage_info[2 * s + j] = e;
                    ++it;
                    if (p.stall_first_kstep && blockIdx.x == 0 && it == 1) continue;  // never lands
                    const uint32_t bytes = live ? kstep_bytes(e) : 0u;
                    // the bands of a pair agree in kind and metadata placement,
                    // so the leader arms the barrier for both CTAs' bytes
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * bytes);
                    if (live) {
                        const CUtensorMap *am = bytes == kDenseStepBytes ? &maps.a_dense
                                              : (bytes == kSparseStepBytes ? &maps.a_sparse : &maps.a_meta);
                        tma2d_pair(smem + s * p.stage_bytes + j * kQdAslot, am, 0,
                                   static_cast<int32_t>(kstep_first(e) / 2048), map_to_rank(&full[s], 0));
                    }
                }
                if (ok && cl + (i + 2) * C < p.items) {
                    fetch_table(cl + (i + 2) * C, buf, j);
                    ++tabs;
                }
            }
            for (int q = (tabs > 2 ? tabs - 2 : 0); q < tabs; ++q)
                mbar_wait_bounded(&tab_full[(q & 1) * 2 + j], (q >> 1) & 1u, never_flag, kQdWaitLimitNs / 4);
            if (!ok) give_up();
            // Drain.  The leader waits for the last phase of every stage (its
            // barrier counts both CTAs' loads); the peer waits until the
            // leader's MMA has released each of its stages, or gives up.
            for (int q = (it > S ? it - S : 0); q < it; ++q) {
                if (p.stall_first_kstep && blockIdx.x == 0 && q == 0) continue;  // never armed
                if (rank == 0)
                    mbar_wait_bounded(&full[q % S], (q / S) & 1u, never_flag, kQdWaitLimitNs / 4);
                else
                    mbar_wait_bounded(&empty[q % S], (q / S) & 1u, never_flag, kQdWaitLimitNs / 4);
            }
        }
    } else if (warp == 2) {
        if (lane == 0 && !skip) {
            // ----------------------------------------------------- X producer
            // (both CTAs; a second issuing thread: copies from one thread are
            // processed largely one after another)
            pdl_wait();  // X may still be written by the kernel before
            const uint32_t x_bytes = 2u * static_cast<uint32_t>(half) * kStep * 2u;  // both CTAs
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int tt = item % p.ttiles;
                for (int c = 0; c < p.nsteps; ++c) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kQdWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    ++it;
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], x_bytes);
                    tma2d_pair(smem + s * p.stage_bytes + 2 * kQdAslot, &maps.x, c * kStep,
                               tt * bn + static_cast<int>(rank) * half, map_to_rank(&full[s], 0));
                }
            }
            if (!ok) give_up();
        }
    } else if (warp == 1) {
        if (lane == 0 && !skip && rank == 0) {
            // ------------------------------------------------- MMA (leader)
            const uint32_t idesc_dense = idesc_pair(bn, false);
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cl + i * C;
                if (item >= p.items) break;
                const int np = pairs_of(item);
                // both accumulators drained by both CTAs' epilogues
                if (i >= 1 && !mbar_wait_bounded(acc_empty, (i - 1) & 1u, abort_flag, kQdWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int c = 0; c < p.nsteps; ++c, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, kQdWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = smem + s * p.stage_bytes;
                    const uint32_t b_addr = smem_u32(st + 2 * kQdAslot);
                    const int h = c & 1;  // k-step within its metadata pair
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        if (j >= np) break;
                        const uint64_t e = stage_info[2 * s + j];
                        const uint32_t slot = smem_u32(st + j * kQdAslot);
                        const uint32_t a_addr = slot + ((e & kEntryMeta) ? kMetaBlockBytes : 0u);
                        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(j * bn);
                        const uint32_t e_tmem = tmem_base + static_cast<uint32_t>(2 * bn + 4 * j);
                        if (e & kEntrySparse) {
                            if (e & kEntryMeta)
                                tmem_cp_pair_128x128b(e_tmem, smem_desc(slot, 16, 128, kSwizzleNone));
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const uint64_t ad = smem_desc(a_addr + q * 32, 16, 512, kSwizzle64B);
                                const uint64_t bd = smem_desc(b_addr + q * 64, 16, 1024, kSwizzle128B);
                                mma_sparse_pair(d_tmem, ad, bd, e_tmem + 2 * h, idesc_pair(bn, true, q),
                                                (c == 0 && q == 0) ? 0u : 1u);
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint64_t ad = smem_desc(a_addr + q * 32, 16, 1024, kSwizzle128B);
                                const uint64_t bd = smem_desc(b_addr + q * 32, 16, 1024, kSwizzle128B);
                                mma_dense_pair(d_tmem, ad, bd, idesc_dense, (c == 0 && q == 0) ? 0u : 1u);
                            }
                        }
                    }
                    tc_commit_pair(&empty[s]);
                }
                // fires once every MMA of the item has completed (also after a
                // failure, so no epilogue frees tensor memory under a running MMA)
                tc_commit_pair(acc_full);
            }
            if (!ok) give_up();
        }
    } else if (warp >= 4 && !skip) {
        // ---------------------------------------------- epilogue (both CTAs)
        pdl_wait();  // Y may still be read by an earlier kernel
        const int j = (warp - 4) / 4;   // accumulator (pair) this warp drains
        const int quad = warp % 4;      // TMEM lanes 32*quad .. 32*quad+31
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                   static_cast<uint32_t>(j * bn);
        for (int i = 0;; ++i) {
            const int item = cl + i * C;
            if (item >= p.items) break;
            const int tt = item % p.ttiles;
            const bool ok = mbar_wait_bounded(acc_full, i & 1u, never_flag, kQdWaitLimitNs);
            tc_fence_after();
            if (!ok) {
                give_up();
                break;
            }
            const int64_t n = static_cast<int64_t>(band_of(item, j)) * kBand + row;
            const int64_t m_base = static_cast<int64_t>(tt) * bn;
            const int m_valid = static_cast<int>(min(static_cast<int64_t>(bn), p.M - m_base));
            if (*abort_flag == 0 && j < pairs_of(item)) {
#pragma unroll 1
                for (int c0 = 0; c0 < m_valid; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(c0), r);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c0 + q < m_valid) store_y(p, (m_base + c0 + q) * p.N + n, __uint_as_float(r[q]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(map_to_rank(acc_empty, 0));
        }
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // the peer's MMAs and remote arrivals are all done
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kQdTmemCols);
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

cudaError_t ensure_quad_attributes() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(quad_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kQdSmemLimit);
    });
    return attr_err;
}

// clusters of two CTAs that fit on the device at once with `smem` bytes each
int quad_max_clusters(int smem) {
    if (ensure_quad_attributes() != cudaSuccess) return 0;
    static std::mutex mu;
    static int cached_smem = -1, cached = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (cached_smem == smem) return cached;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kQdThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, quad_gemm_kernel, &cfg) != cudaSuccess) n = 0;
    cached_smem = smem;
    cached = n;
    return n;
}

int quad_smem(int bn, int *stages, int *stage_bytes) {
    *stage_bytes = 2 * kQdAslot + (bn / 2) * kStep * 2;
    *stages = std::min(kQdMaxStages, (kQdSmemLimit - kQdTailBytes) / *stage_bytes);
    return *stages * *stage_bytes + kQdTailBytes;
}

}  // namespace

double quad_kstep_cycles(int bn) {
    // per SM per dense k-step: max(MMA 4 BN cycles (two M = 256 x BN x K64
    // instructions' halves), shared-memory traffic (32 KB of weights in and
    // read, BN/2 tokens x 128 B in and read twice) at 128 B per cycle)
    return std::max(4.0 * bn, 512.0 + 1.5 * bn);
}

void preload_quad_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, quad_gemm_kernel);
}

QuadPlan plan_quad_gemm(int64_t N, int64_t M, int num_sms) {
    QuadPlan best{};
    const int64_t bands = N / kBand;
    const int64_t quads = (bands + 3) / 4;
    int st = 0, sb = 0;
    const int clusters_cap = quad_max_clusters(quad_smem(240, &st, &sb));
    if (clusters_cap < 1 || bands % 2 != 0) return best;  // bn = 0: not usable
    const int clusters = std::min(clusters_cap, num_sms / 2);
    double best_cost = 0;
    for (int bn = 240; bn >= 128; bn -= 16) {
        const int64_t tt = (M + bn - 1) / bn;
        const int64_t items = quads * tt;
        const int64_t waves = (items + clusters - 1) / clusters;
        const double cost = static_cast<double>(waves) * quad_kstep_cycles(bn);
        if (best.bn == 0 || cost < best_cost) {
            best_cost = cost;
            best.bn = bn;
            best.ttiles = static_cast<int>(tt);
            best.items = static_cast<int>(items);
            best.clusters = static_cast<int>(std::min<int64_t>(clusters, items));
        }
    }
    best.smem = quad_smem(best.bn, &best.stages, &best.stage_bytes);
    best.cost = best_cost;
    return best;
}

cudaError_t launch_quad_gemm(const GemmLaunch &g, const QuadPlan &plan, cudaStream_t stream) {
    const cudaError_t attr_err = ensure_quad_attributes();
    if (attr_err != cudaSuccess) return attr_err;
    if (plan.bn < 16 || plan.stages < 2 || plan.smem > kQdSmemLimit || plan.clusters < 1)
        return cudaErrorInvalidValue;
    if ((g.N / kBand) % 2 != 0 || g.K / kStep > kQdTabSteps || !g.packed_rows || !g.ptable)
        return cudaErrorInvalidValue;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    QuadMaps maps;
    // X [M,K] bf16 row-major: box = 64 columns x this CTA's BN/2 tokens,
    // 128-byte swizzle, rows past M read as zero
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(g.K), static_cast<cuuint64_t>(g.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(g.K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kStep), static_cast<cuuint32_t>(plan.bn / 2)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(g.X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const uint64_t rows = g.packed_rows / 16;  // 2 KB rows of packed bytes + side copies
    if (!encode_rows(enc, &maps.a_dense, g.packed, rows, kDenseStepBytes / 2048) ||
        !encode_rows(enc, &maps.a_meta, g.packed, rows, (kMetaBlockBytes + kSparseStepBytes) / 2048) ||
        !encode_rows(enc, &maps.a_sparse, g.packed, rows, kSparseStepBytes / 2048))
        return cudaErrorInvalidValue;
    QuadParams p;
    p.ptable = g.ptable;
    p.N = g.N;
    p.K = g.K;
    p.M = g.M;
    p.nsteps = static_cast<int>(g.K / kStep);
    p.bands = static_cast<int>(g.N / kBand);
    p.quads = (p.bands + 3) / 4;
    p.ttiles = plan.ttiles;
    p.items = plan.items;
    p.bn = plan.bn;
    p.half = plan.bn / 2;
    p.stages = plan.stages;
    p.stage_bytes = plan.stage_bytes;
    p.Y = g.Y;
    p.y_fp32 = g.y_fp32;
    p.status = g.status;
    p.ready = g.ready;
    p.stall_first_kstep = g.stall_first_kstep;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * plan.clusters));
    cfg.blockDim = dim3(kQdThreads);
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
    cudaError_t err = cudaLaunchKernelEx(&cfg, quad_gemm_kernel, maps, p);
    if (err == cudaSuccess) note_launches(1);
    return err;
}

}  // namespace patchk
