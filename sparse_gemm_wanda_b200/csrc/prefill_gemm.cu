// Band-pair hybrid GEMM for prefill on the sm_100a tensor cores.
//
// Same product as the other GEMM paths, Y = X * W_eff^T, dense k-steps on
// tcgen05.mma and 2:4 k-steps on tcgen05.mma.sp ("PATCH: Learnable
// Tile-level Hybrid Sparsity for LLMs", section 2, inference and deployment).
//
// Why a second prefill kernel.  The tensor core reads its operands from
// shared memory, and the copies that fill it write there too: measured on
// B200, the two together saturate at about 128 B per cycle per SM.  A one-band
// CTA with a 160-token tile moves 72 KB per dense 64-column k-step (36 KB in,
// 36 KB of operand reads) for 320 cycles of MMA, so the tensor pipe runs at
// about 55 %, and a 2:4 k-step moves 57 KB for 160 cycles (about 36 % of the
// sparse rate).  Here a CTA owns TWO bands that share one X tile of up to 240
// tokens, in two TMEM accumulators of 128 x BN fp32 (2 x 240 + 8 metadata
// columns of the 512): a dense k-step moves 64 KB + 384 B per token for
// 4 x BN cycles (80 % at BN = 240), a 2:4 one 124 KB for 480 cycles.  The two
// bands are independent MMAs, so a dense tile next to a 2:4 tile costs
// nothing extra: each band issues its own kind per k-step.
//
// Work item = (band pair, token tile); persistent CTAs take items c, c + P,
// ...  A stage is one k-step: one bulk copy per band (16 KB dense, or the 2 KB
// metadata block + 8 KB kept values) and one 2-D TMA load of the X tile
// (128-byte swizzle, rows past M read as zero).
//
// Roles (352 threads): warp 0 lane 0 weight producer, warp 10 lane 0 X
// producer (copies one thread issues are processed largely one after another,
// so the two streams get a thread each), warp 1 lane 0 MMA issuer, warps 2..9
// epilogue (warps 2..5 drain band 0, warps 6..9 band 1; each warp its 32-lane
// TMEM quarter).  Launched as a programmatic dependent: with the packer's
// ready flag seen, the table and the weights are fetched before
// `griddepcontrol.wait`; X and Y only after it.  Every mbarrier
// wait is bounded by %globaltimer.
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

constexpr int kPgThreads = 352;   // + warp 10: the X-tile producer
constexpr int kPgEpiWarps = 8;
constexpr int kPgMaxStages = 6;
constexpr int kPgTabSteps = 448;                 // k-steps per band (K <= 28672)
constexpr int kPgTabBytes = 2 * 2 * kPgTabSteps * 8;  // two items x two bands
constexpr int kPgAslot = kDenseStepBytes;        // per band per stage
constexpr int kPgTmemCols = 512;
constexpr int kPgSmemLimit = 232448;             // 227 KB per CTA
constexpr int kPgTailBytes = 1024 + kPgTabBytes + 512;
constexpr uint64_t kPgWaitLimitNs = 2000000000ull;

struct PairParams {
    const uint8_t *packed;
    const uint64_t *table;
    int64_t N, K, M;
    int nsteps, bands, bpairs, ttiles, items;
    int bn, stages, stage_bytes;
    void *Y;
    int y_fp32;
    uint32_t *status;
    const uint32_t *ready;
    int stall_first_kstep;  // failure-detection test hook
};

__device__ __forceinline__ void store_y(const PairParams &p, int64_t idx, float v) {
    if (p.y_fp32)
        static_cast<float *>(p.Y)[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(p.Y)[idx] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ void tma_load_2d_x(void *dst, const void *tmap, int32_t x, int32_t y,
                                              uint64_t *bar) {
    tma_load_2d(dst, tmap, x, y, bar);
}

__global__ void __launch_bounds__(kPgThreads, 1)
pair_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ PairParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int S = p.stages;
    uint64_t *tab_buf = reinterpret_cast<uint64_t *>(smem + S * p.stage_bytes);  // [2][2][448]
    uint64_t *full = tab_buf + 2 * 2 * kPgTabSteps;
    uint64_t *empty = full + kPgMaxStages;
    uint64_t *acc_full = empty + kPgMaxStages;
    uint64_t *acc_empty = acc_full + 1;
    uint64_t *tab_full = acc_empty + 1;  // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tab_full + 2);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    volatile uint32_t *never_flag = tmem_slot + 2;
    uint64_t *stage_info = reinterpret_cast<uint64_t *>(tmem_slot + 4);  // [S][2]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cta = blockIdx.x, P = gridDim.x;

    auto item_bands = [&](int item, int &bp, int &tt, bool &two) {
        bp = item / p.ttiles;
        tt = item % p.ttiles;
        two = 2 * bp + 1 < p.bands;
    };
    auto fetch_table = [&](int item, int buf) {
        int bp, tt;
        bool two;
        item_bands(item, bp, tt, two);
        const uint32_t nb = static_cast<uint32_t>(p.nsteps) * 8u;
        mbar_arrive_expect_tx(&tab_full[buf], two ? 2 * nb : nb);
        uint64_t *dst = tab_buf + buf * 2 * kPgTabSteps;
        bulk_g2s(dst, p.table + static_cast<int64_t>(2 * bp) * p.nsteps, nb, &tab_full[buf]);
        if (two)
            bulk_g2s(dst + kPgTabSteps, p.table + static_cast<int64_t>(2 * bp + 1) * p.nsteps, nb,
                     &tab_full[buf]);
    };

    if (threadIdx.x == 0) {
        pdl_trigger();
        // weights are final once the packer's ready flag is seen; otherwise
        // (the packer may be the kernel just before) wait first
        if (ld_acquire_gpu(p.ready) == 0u) pdl_wait();
        for (int s = 0; s < kPgMaxStages; ++s) {
            mbar_init(&full[s], 2);  // weight producer + X producer
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kPgEpiWarps);
        mbar_init(&tab_full[0], 1);
        mbar_init(&tab_full[1], 1);
        *never_flag = 0u;
        *abort_flag = (*reinterpret_cast<volatile uint32_t *>(p.status) & kStatusTimeout) ? 1u : 0u;
        fence_mbar_init();
        if (!*abort_flag) {
            for (int i = 0; i < 2 && cta + i * P < p.items; ++i) fetch_table(cta + i * P, i);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kPgTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmap_x);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;
    const int bn = p.bn;

    if (warp == 0) {
        if (lane == 0 && !skip) {
            // ------------------------------------------------------ producer
            int it = 0;  // stages armed so far
            bool ok = true;
            int tabs = 0;  // table copies issued
            for (int i = 0; i < 2 && cta + i * P < p.items; ++i) ++tabs;
            for (int i = 0; ok; ++i) {
                const int item = cta + i * P;
                if (item >= p.items) break;
                int bp, tt;
                bool two;
                item_bands(item, bp, tt, two);
                const int buf = i & 1;
                if (!mbar_wait_bounded(&tab_full[buf], (i >> 1) & 1u, abort_flag, kPgWaitLimitNs)) {
                    ok = false;
                    break;
                }
                const uint64_t *tab = tab_buf + buf * 2 * kPgTabSteps;
                for (int c = 0; c < p.nsteps; ++c) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kPgWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    const uint64_t e0 = tab[c];
                    const uint64_t e1 = two ? tab[kPgTabSteps + c] : 0ull;
                    stage_info[2 * s + 0] = e0;
                    stage_info[2 * s + 1] = e1;
                    ++it;
                    if (p.stall_first_kstep && cta == 0 && it == 1) continue;  // never lands
                    uint32_t bytes = 0;
                    uint64_t f0 = 0, f1 = 0;
                    uint32_t b0 = 0, b1 = 0;
                    {
                        const bool sp = (e0 & kEntrySparse) != 0, me = (e0 & kEntryMeta) != 0;
                        f0 = (e0 & kEntryOffsetMask) - (me ? kMetaBlockBytes : 0);
                        b0 = (me ? kMetaBlockBytes : 0) + (sp ? kSparseStepBytes : kDenseStepBytes);
                        bytes += b0;
                    }
                    if (two) {
                        const bool sp = (e1 & kEntrySparse) != 0, me = (e1 & kEntryMeta) != 0;
                        f1 = (e1 & kEntryOffsetMask) - (me ? kMetaBlockBytes : 0);
                        b1 = (me ? kMetaBlockBytes : 0) + (sp ? kSparseStepBytes : kDenseStepBytes);
                        bytes += b1;
                    }
                    uint8_t *st = smem + s * p.stage_bytes;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    bulk_g2s(st, p.packed + f0, b0, &full[s]);
                    if (two) bulk_g2s(st + kPgAslot, p.packed + f1, b1, &full[s]);
                }
                // this table buffer is free again: fetch the table of item i + 2
                if (ok && cta + (i + 2) * P < p.items) {
                    fetch_table(cta + (i + 2) * P, buf);
                    ++tabs;
                }
            }
            for (int q = (tabs > 2 ? tabs - 2 : 0); q < tabs; ++q)
                mbar_wait_bounded(&tab_full[q & 1], (q >> 1) & 1u, never_flag, kPgWaitLimitNs / 4);
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
            for (int q = (it > S ? it - S : 0); q < it; ++q) {
                if (p.stall_first_kstep && cta == 0 && q == 0) continue;  // never armed
                mbar_wait_bounded(&full[q % S], (q / S) & 1u, never_flag, kPgWaitLimitNs / 4);
            }
        }
    } else if (warp == 10) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------- X producer
            // a second issuing thread: copies one thread issues are processed
            // largely one after another
            pdl_wait();  // X may still be written by the kernel before
            const uint32_t x_bytes = static_cast<uint32_t>(bn) * kStep * 2u;
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cta + i * P;
                if (item >= p.items) break;
                const int tt = item % p.ttiles;
                for (int c = 0; c < p.nsteps; ++c) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kPgWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    ++it;
                    mbar_arrive_expect_tx(&full[s], x_bytes);
                    tma_load_2d_x(smem + s * p.stage_bytes + 2 * kPgAslot, &tmap_x, c * kStep, tt * bn,
                                  &full[s]);
                }
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
            // drain: the last phase of every stage this thread armed
            for (int q = (it > S ? it - S : 0); q < it; ++q)
                mbar_wait_bounded(&full[q % S], (q / S) & 1u, never_flag, kPgWaitLimitNs / 4);
        }
    } else if (warp == 1) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------------- MMA
            const uint32_t idesc_dense = idesc_bf16(bn, false);
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int item = cta + i * P;
                if (item >= p.items) break;
                int bp, tt;
                bool two;
                item_bands(item, bp, tt, two);
                if (i >= 1 && !mbar_wait_bounded(acc_empty, (i - 1) & 1u, abort_flag, kPgWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int c = 0; c < p.nsteps; ++c, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, kPgWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t *st = smem + s * p.stage_bytes;
                    const uint32_t b_addr = smem_u32(st + 2 * kPgAslot);
                    const int h = c & 1;  // k-step within its metadata pair
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        if (j == 1 && !two) break;
                        const uint64_t e = stage_info[2 * s + j];
                        const uint32_t slot = smem_u32(st + j * kPgAslot);
                        const uint32_t a_addr = slot + ((e & kEntryMeta) ? kMetaBlockBytes : 0u);
                        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(j * bn);
                        const uint32_t e_tmem = tmem_base + static_cast<uint32_t>(2 * bn + 4 * j);
                        if (e & kEntrySparse) {
                            if (e & kEntryMeta)
                                tmem_cp_128x128b(e_tmem, smem_desc(slot, 16, 128, kSwizzleNone));
#pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const uint64_t ad = smem_desc(a_addr + q * 32, 16, 512, kSwizzle64B);
                                const uint64_t bd = smem_desc(b_addr + q * 64, 16, 1024, kSwizzle128B);
                                mma_sparse(d_tmem, ad, bd, e_tmem + 2 * h, idesc_bf16(bn, true, q),
                                           (c == 0 && q == 0) ? 0u : 1u);
                            }
                        } else {
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const uint64_t ad = smem_desc(a_addr + q * 32, 16, 1024, kSwizzle128B);
                                const uint64_t bd = smem_desc(b_addr + q * 32, 16, 1024, kSwizzle128B);
                                mma_dense(d_tmem, ad, bd, idesc_dense, (c == 0 && q == 0) ? 0u : 1u);
                            }
                        }
                    }
                    tc_commit(&empty[s]);
                }
                // fires once every MMA of the item has completed (also after a
                // failure, so the epilogue never frees TMEM under a running MMA)
                tc_commit(acc_full);
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
        }
    } else if (!skip) {
        // ------------------------------------------------------- epilogue
        pdl_wait();  // Y may still be read by an earlier kernel
        const int w = warp - 2;          // 0..7
        const int j = w / 4;             // band of the pair
        const int quad = warp % 4;       // TMEM lanes 32*quad .. 32*quad+31
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                   static_cast<uint32_t>(j * bn);
        for (int i = 0;; ++i) {
            const int item = cta + i * P;
            if (item >= p.items) break;
            int bp, tt;
            bool two;
            item_bands(item, bp, tt, two);
            const bool ok = mbar_wait_bounded(acc_full, i & 1u, never_flag, kPgWaitLimitNs);
            tc_fence_after();
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
                break;
            }
            const bool live = *abort_flag == 0 && (j == 0 || two);
            const int64_t n = static_cast<int64_t>(2 * bp + j) * kBand + row;
            const int64_t m_base = static_cast<int64_t>(tt) * bn;
            const int m_valid = static_cast<int>(min(static_cast<int64_t>(bn), p.M - m_base));
            if (live) {
#pragma unroll 1
                for (int c0 = 0; c0 < m_valid; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(lane_base + c0, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c0 + q < m_valid) store_y(p, (m_base + c0 + q) * p.N + n, __uint_as_float(r[q]));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kPgTmemCols);
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

double pair_kstep_cycles(int bn) { return 512.0 + 3.0 * bn; }

void preload_pair_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, pair_gemm_kernel);
}

PairPlan plan_pair_gemm(int64_t N, int64_t M, int num_sms) {
    // Token tile: the multiple of 16 in [128, 240] that minimises
    // waves x time per item (the last wave counts whole).  A dense k-step of
    // an item is bound by shared-memory traffic, 64 KB + 384 B per token of
    // copies in and operand reads at 128 B per cycle: 512 + 3 BN cycles.
    // Ties go to the wider tile.
    PairPlan best{};
    const int64_t bands = N / kBand, bpairs = (bands + 1) / 2;
    double best_cost = 0;
    for (int bn = 240; bn >= 128; bn -= 16) {
        const int64_t tt = (M + bn - 1) / bn;
        const int64_t items = bpairs * tt;
        const int64_t waves = (items + num_sms - 1) / num_sms;
        const double cost = static_cast<double>(waves) * pair_kstep_cycles(bn);
        if (best.bn == 0 || cost < best_cost) {
            best_cost = cost;
            best.bn = bn;
            best.ttiles = static_cast<int>(tt);
            best.items = static_cast<int>(items);
            best.waves = static_cast<int>(waves);
        }
    }
    const int stage_bytes = 2 * kPgAslot + best.bn * kStep * 2;
    best.stages = std::min(kPgMaxStages, (kPgSmemLimit - kPgTailBytes) / stage_bytes);
    best.stage_bytes = stage_bytes;
    best.smem = best.stages * stage_bytes + kPgTailBytes;
    best.cost = best_cost;
    return best;
}

cudaError_t launch_pair_gemm(const GemmLaunch &g, const PairPlan &plan, cudaStream_t stream) {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(pair_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kPgSmemLimit);
    });
    if (attr_err != cudaSuccess) return attr_err;
    if (plan.stages < 2 || plan.smem > kPgSmemLimit) return cudaErrorInvalidValue;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    // X [M,K] bf16 row-major: box = 64 columns x BN rows, 128-byte swizzle,
    // rows past M read as zero
    CUtensorMap map;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(g.K), static_cast<cuuint64_t>(g.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(g.K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kStep), static_cast<cuuint32_t>(plan.bn)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(g.X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    PairParams p;
    p.packed = g.packed;
    p.table = g.table;
    p.N = g.N;
    p.K = g.K;
    p.M = g.M;
    p.nsteps = static_cast<int>(g.K / kStep);
    p.bands = static_cast<int>(g.N / kBand);
    p.bpairs = (p.bands + 1) / 2;
    p.ttiles = plan.ttiles;
    p.items = plan.items;
    p.bn = plan.bn;
    p.stages = plan.stages;
    p.stage_bytes = plan.stage_bytes;
    p.Y = g.Y;
    p.y_fp32 = g.y_fp32;
    p.status = g.status;
    p.ready = g.ready;
    p.stall_first_kstep = g.stall_first_kstep;
    if (p.nsteps > kPgTabSteps) return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min(g.num_sms, plan.items)));
    cfg.blockDim = dim3(kPgThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, pair_gemm_kernel, map, p);
    if (err == cudaSuccess) note_launches(1);
    return err;
}

}  // namespace patchk
