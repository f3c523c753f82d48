// FP8 hybrid GEMM on the sm_100a tensor cores: Y = diag(sx) (QX QW^T) diag(sw).
//
// FP8 values inside dense and 2:4 tiles ("SparseGPT vs Wanda: one-shot LLM
// pruning without retraining", FAQ: prune first, then quantise; the tile
// scheme of "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section
// 2): dense k-steps issue tcgen05.mma kind::f8f6f4 (4 x M128 N=BN K32 per
// 128-column k-step), 2:4 k-steps tcgen05.mma.sp kind::f8f6f4 (2 x M128 N=BN
// K64, after one tcgen05.cp of the k-step's metadata block into 4 TMEM
// columns; the metadata of sparse MMA q sits at TMEM column 2q with selector
// 0).  Both e4m3, fp32 accumulation in tensor memory; the epilogue multiplies
// by the token's and the output row's fp32 scales and rounds once.
//
// Work: an output tile is one 128-row band x BN tokens; persistent CTAs take
// tiles c, c + P, ...; two accumulators alternate so one tile's epilogue
// overlaps the next tile's main loop.  With at most half as many tiles as SMs
// (decode token counts on smaller matrices) each tile's k-steps are cut into
// `ksplit` equal ranges, the
// work items are (tile, range), each item leaves its fp32 accumulator in its
// own slot, and a fix-up kernel adds a tile's slots in range order and
// applies the scales, so the result does not depend on timing.  A stage is one k-step: one bulk copy of
// its packed bytes (16 KB dense, or 2 KB metadata + 8 KB kept codes) and one
// TMA load of the BN x 128-byte X tile (128-byte swizzle, rows past M zero).
// Roles (224 threads): warp 0 lane 0 weight producer, warp 6 lane 0 X
// producer (the copies one thread issues are processed largely one after
// another, so the two streams go through two threads), warp 1 lane 0 MMA
// (warp 1 also allocates tensor memory), warps 2..5 epilogue.  Every mbarrier
// wait is bounded by %globaltimer; a wait that runs out raises the handle's
// status.
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

constexpr int kF8Threads = 224;
constexpr int kF8Step = 128;                 // columns (bytes of codes) per k-step
constexpr int kF8Aslot = kDenseStepBytes;    // 16 KB: a dense k-step, or metadata + kept codes
constexpr int kF8SmemLimit = 232448;
constexpr int kF8MaxStages = 8;
constexpr uint64_t kF8WaitLimitNs = 2000000000ull;

struct F8Params {
    const uint8_t *packed;
    const uint64_t *table;   // [bands][K/128]
    const float *sw;         // [N] weight row scales
    const float *sx;         // [M] token scales
    int64_t N, K, M;
    int steps, bands, ttiles, tiles;
    int ksplit;      // k-step ranges per tile (1: no split)
    int kper;        // k-steps per range (the last range may hold fewer)
    int items;       // tiles * ksplit
    float *partial;  // ksplit > 1: [items][BN][128] fp32, unscaled
    void *Y;
    int y_fp32;
    uint32_t *status;
};

// Work item w: tile w / ksplit, k-steps [c0, c1) of it.
__device__ __forceinline__ void f8_item(const F8Params &p, int w, int &tile, int &c0, int &c1) {
    tile = w / p.ksplit;
    c0 = (w % p.ksplit) * p.kper;
    c1 = min(p.steps, c0 + p.kper);
}

__device__ __forceinline__ void store_y(const F8Params &p, int64_t idx, float v) {
    if (p.y_fp32)
        static_cast<float *>(p.Y)[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(p.Y)[idx] = __float2bfloat16_rn(v);
}

template <int BN>
struct F8Cfg {
    static constexpr int kXBytes = BN * kF8Step;
    static constexpr int kStageBytes = kF8Aslot + kXBytes;
    static constexpr int kTail = 1024 + 512;
    static constexpr int kStages = std::min(kF8MaxStages, (kF8SmemLimit - kTail) / kStageBytes);
    static constexpr int kSmem = kStages * kStageBytes + kTail;
    static constexpr int kCols = 2 * BN + 4;
    static constexpr int kTmemCols = kCols <= 128 ? 128 : (kCols <= 256 ? 256 : 512);
    static_assert(kStages >= 2, "at least two stages");
    static_assert(kXBytes % 1024 == 0, "stage regions stay 1024-B aligned");
    static_assert(kCols <= 512, "tensor memory holds 512 columns");
};

template <int BN>
__global__ void __launch_bounds__(kF8Threads, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ F8Params p) {
    using C = F8Cfg<BN>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + S * C::kStageBytes);
    uint64_t *empty = full + S;
    uint64_t *acc_full = empty + S;   // [2]
    uint64_t *acc_empty = acc_full + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_empty + 2);
    volatile uint32_t *abort_flag = tmem_slot + 1;
    volatile uint32_t *never_flag = tmem_slot + 2;
    uint64_t *stage_info = reinterpret_cast<uint64_t *>(tmem_slot + 4);  // [S]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cta = blockIdx.x, P = gridDim.x;

    if (threadIdx.x == 0) {
        pdl_trigger();  // the fix-up (or the next kernel) may start its prologue
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 2);  // the weight and X producers
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        *never_flag = 0u;
        *abort_flag = (*reinterpret_cast<volatile uint32_t *>(p.status) & kStatusTimeout) ? 1u : 0u;
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
            pdl_wait();  // launched as a programmatic dependent: global memory after the wait
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int w = cta + i * P;
                if (w >= p.items) break;
                int tile, c0, c1;
                f8_item(p, w, tile, c0, c1);
                const int band = tile / p.ttiles;
                const uint64_t *tab = p.table + static_cast<int64_t>(band) * p.steps;
                for (int c = c0; c < c1; ++c) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kF8WaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    const uint64_t e = __ldg(tab + c);
                    const bool sp = (e & kEntrySparse) != 0;
                    const uint64_t first = (e & kEntryOffsetMask) - (sp ? kMetaBlockBytes : 0);
                    const uint32_t bytes = sp ? kMetaBlockBytes + kSparseStepBytes : kDenseStepBytes;
                    stage_info[s] = e;
                    ++it;
                    uint8_t *st = smem + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    bulk_g2s(st, p.packed + first, bytes, &full[s]);
                }
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
            // the last phase issued on every stage lands before the CTA exits
            for (int q = (it > S ? it - S : 0); q < it; ++q)
                mbar_wait_bounded(&full[q % S], (q / S) & 1u, never_flag, kF8WaitLimitNs / 4);
        }
    } else if (warp == 6) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------- X producer
            pdl_wait();  // the codes are written by the kernel just before
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int w = cta + i * P;
                if (w >= p.items) break;
                int tile, c0, c1;
                f8_item(p, w, tile, c0, c1);
                const int tt = tile % p.ttiles;
                for (int c = c0; c < c1; ++c) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (it >= S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kF8WaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    ++it;
                    mbar_arrive_expect_tx(&full[s], C::kXBytes);
                    tma_load_2d(smem + s * C::kStageBytes + kF8Aslot, &tmap_x, c * kF8Step, tt * BN, &full[s]);
                }
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------------- MMA
            const uint32_t e_tmem = tmem_base + static_cast<uint32_t>(2 * BN);
            constexpr uint32_t kIdDense = idesc_e4m3(BN, false);
            constexpr uint32_t kIdSparse = idesc_e4m3(BN, true);
            int it = 0;
            bool ok = true;
            for (int i = 0; ok; ++i) {
                const int w = cta + i * P;
                if (w >= p.items) break;
                int tile, c0, c1;
                f8_item(p, w, tile, c0, c1);
                const int buf = i & 1;
                if (i >= 2 &&
                    !mbar_wait_bounded(&acc_empty[buf], ((i >> 1) & 1u) ^ 1u, abort_flag, kF8WaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int c = c0; c < c1; ++c, ++it) {
                    const int s = it % S;
                    const uint32_t ph = (it / S) & 1u;
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, kF8WaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t slot = smem_u32(smem + s * C::kStageBytes);
                    const uint32_t b_addr = slot + kF8Aslot;
                    if (stage_info[s] & kEntrySparse) {
                        tmem_cp_128x128b(e_tmem, smem_desc(slot, 16, 128, kSwizzleNone));
#pragma unroll
                        for (int q = 0; q < 2; ++q) {
                            const uint64_t ad = smem_desc(slot + kMetaBlockBytes + q * 32, 16, 512, kSwizzle64B);
                            const uint64_t bd = smem_desc(b_addr + q * 64, 16, 1024, kSwizzle128B);
                            mma_f8_sparse(d_tmem, ad, bd, e_tmem + 2 * q, kIdSparse, (c == c0 && q == 0) ? 0u : 1u);
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint64_t ad = smem_desc(slot + q * 32, 16, 1024, kSwizzle128B);
                            const uint64_t bd = smem_desc(b_addr + q * 32, 16, 1024, kSwizzle128B);
                            mma_f8(d_tmem, ad, bd, kIdDense, (c == c0 && q == 0) ? 0u : 1u);
                        }
                    }
                    tc_commit(&empty[s]);
                }
                // fires once every MMA of the tile has completed (also after a
                // failure, so the epilogue never frees TMEM under a running MMA)
                tc_commit(&acc_full[buf]);
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
        }
    } else if (!skip) {
        // ------------------------------------------------------- epilogue
        pdl_wait();  // Y and the partial slots may still be used by earlier kernels
        const int quad = warp % 4;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        for (int i = 0;; ++i) {
            const int w = cta + i * P;
            if (w >= p.items) break;
            const int tile = w / p.ksplit;
            const int buf = i & 1;
            const bool ok = mbar_wait_bounded(&acc_full[buf], (i >> 1) & 1u, never_flag, kF8WaitLimitNs);
            tc_fence_after();
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
                break;
            }
            const int band = tile / p.ttiles, tt = tile % p.ttiles;
            const int64_t n = static_cast<int64_t>(band) * kBand + row;
            const int64_t m_base = static_cast<int64_t>(tt) * BN;
            const int m_valid = static_cast<int>(min(static_cast<int64_t>(BN), p.M - m_base));
            const float swn = __ldg(p.sw + n);
            if (*abort_flag == 0 && p.ksplit > 1) {
                // this range's accumulator, unscaled, into the item's slot
                float *part = p.partial + static_cast<int64_t>(w) * BN * kBand + row;
#pragma unroll 1
                for (int c0 = 0; c0 < m_valid; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(buf * BN + c0), r);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c0 + q < m_valid) part[(c0 + q) * kBand] = __uint_as_float(r[q]);
                }
            } else if (*abort_flag == 0) {
#pragma unroll 1
                for (int c0 = 0; c0 < m_valid; c0 += 16) {
                    uint32_t r[16];
                    tmem_ld_32x32b_x16(lane_base + static_cast<uint32_t>(buf * BN + c0), r);
                    tmem_ld_wait();
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c0 + q < m_valid) {
                            const int64_t m = m_base + c0 + q;
                            store_y(p, m * p.N + n, __uint_as_float(r[q]) * swn * __ldg(p.sx + m));
                        }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// Split-K fix-up: Y[m, n] = (the tile's range accumulators added in range
// order, from zero) * sw[n] * sx[m].  Block (tile, token of the tile), one
// thread per row of the band.  Launched as a programmatic dependent of the
// GEMM; waits for it.
template <int BN>
__global__ void __launch_bounds__(kBand)
fp8_splitk_reduce_kernel(const __grid_constant__ F8Params p) {
    if (threadIdx.x == 0) pdl_trigger();
    pdl_wait();
    const int tile = blockIdx.x, ml = blockIdx.y, row = threadIdx.x;
    const int band = tile / p.ttiles, tt = tile % p.ttiles;
    const int64_t m = static_cast<int64_t>(tt) * BN + ml;
    if (m >= p.M) return;
    const float *src = p.partial + (static_cast<int64_t>(tile) * p.ksplit * BN + ml) * kBand + row;
    float acc = 0.0f;
    for (int k0 = 0; k0 < p.ksplit; k0 += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            v[q] = (k0 + q < p.ksplit) ? __ldcg(src + static_cast<int64_t>(k0 + q) * BN * kBand) : 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (k0 + q < p.ksplit) acc = __fadd_rn(acc, v[q]);
    }
    const int64_t n = static_cast<int64_t>(band) * kBand + row;
    store_y(p, m * p.N + n, acc * __ldg(p.sw + n) * __ldg(p.sx + m));
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

template <int BN>
cudaError_t run_fp8(const Fp8Launch &g, cudaStream_t stream) {
    using C = F8Cfg<BN>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(fp8_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::kSmem);
    });
    if (attr_err != cudaSuccess) return attr_err;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorInvalidValue;
    // X codes [M, K] uint8 row-major: box = 128 bytes x BN rows, 128-byte
    // swizzle, rows past M read as zero
    CUtensorMap map;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(g.K), static_cast<cuuint64_t>(g.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(g.K)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kF8Step), static_cast<cuuint32_t>(BN)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(g.xq), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    F8Params p;
    p.packed = g.packed;
    p.table = g.table;
    p.sw = g.sw;
    p.sx = g.sx;
    p.N = g.N;
    p.K = g.K;
    p.M = g.M;
    p.steps = static_cast<int>(g.K / kF8Step);
    p.bands = static_cast<int>(g.N / kBand);
    p.ttiles = static_cast<int>((g.M + BN - 1) / BN);
    p.tiles = p.bands * p.ttiles;
    p.Y = g.Y;
    p.y_fp32 = g.y_fp32;
    p.status = g.status;
    // at most half as many tiles as SMs: split each tile's k-steps so that
    // about two work items fall on every SM (ranges of equal length, none
    // empty); with more tiles the partials and the fix-up cost more than the
    // idle SMs (measured on 11008x4096: 86 tiles, 22.3 us split against 17.3)
    p.ksplit = 1;
    p.kper = p.steps;
    if (2 * p.tiles <= g.num_sms && g.pool) {
        const int want = std::min(p.steps, std::min(16, (2 * g.num_sms + p.tiles - 1) / p.tiles));
        if (want > 1) {
            p.kper = (p.steps + want - 1) / want;
            p.ksplit = (p.steps + p.kper - 1) / p.kper;
        }
    }
    p.items = p.tiles * p.ksplit;
    p.partial = nullptr;
    float *ws = nullptr;
    if (p.ksplit > 1) {
        const size_t bytes = sizeof(float) * static_cast<size_t>(p.items) * BN * kBand;
        const cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), bytes, g.pool, stream);
        if (e != cudaSuccess) return e;
        p.partial = ws;
    }
    const int grid = std::min(g.num_sms, p.items);
    // programmatic dependent of the X quantisation before it (see the roles)
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t kcfg = {};
    kcfg.gridDim = dim3(static_cast<unsigned>(grid));
    kcfg.blockDim = dim3(kF8Threads);
    kcfg.dynamicSmemBytes = C::kSmem;
    kcfg.stream = stream;
    kcfg.attrs = attr;
    kcfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&kcfg, fp8_gemm_kernel<BN>, map, p);
    if (err == cudaSuccess) note_launches(1);
    if (err == cudaSuccess && p.ksplit > 1) {
        cudaLaunchConfig_t cfg = {};
        // blocks only for the tokens a tile holds
        cfg.gridDim = dim3(static_cast<unsigned>(p.tiles), static_cast<unsigned>(std::min<int64_t>(BN, g.M)));
        cfg.blockDim = dim3(kBand);
        cfg.stream = stream;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        err = cudaLaunchKernelEx(&cfg, fp8_splitk_reduce_kernel<BN>, p);
        if (err == cudaSuccess) note_launches(1);
    }
    if (ws) {
        const cudaError_t e2 = cudaFreeAsync(ws, stream);
        if (err == cudaSuccess) err = e2;
    }
    return err;
}

}  // namespace

void preload_fp8_gemm_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, fp8_gemm_kernel<64>);
    (void)cudaFuncGetAttributes(&a, fp8_gemm_kernel<128>);
    (void)cudaFuncGetAttributes(&a, fp8_gemm_kernel<240>);
    (void)cudaFuncGetAttributes(&a, fp8_splitk_reduce_kernel<64>);
    (void)cudaFuncGetAttributes(&a, fp8_splitk_reduce_kernel<128>);
    (void)cudaFuncGetAttributes(&a, fp8_splitk_reduce_kernel<240>);
}

cudaError_t launch_fp8_gemm(const Fp8Launch &g, cudaStream_t stream) {
    if (g.K % kF8Step != 0 || g.N % kBand != 0 || g.M < 1) return cudaErrorInvalidValue;
    // more than one token tile: the two-SM kernel, where the bands pair up
    // (prefill table) and the k-step count is even
    const bool duo_ok = g.ptable && (g.N / kBand) % 2 == 0 && (g.K / kF8Step) % 2 == 0 && g.K / kF8Step <= 224;
    if (duo_ok && g.force_kernel != 1 && (g.M > 128 || g.force_kernel == 3)) {
        const DuoFp8Plan dp = plan_duo_fp8(g.N, g.M, g.num_sms, g.all_sparse != 0);
        if (dp.bn > 0) return launch_duo_fp8(g, dp, stream);
    }
    if (g.M <= 64) return run_fp8<64>(g, stream);
    if (g.M <= 128) return run_fp8<128>(g, stream);
    return run_fp8<240>(g, stream);
}

}  // namespace patchk
