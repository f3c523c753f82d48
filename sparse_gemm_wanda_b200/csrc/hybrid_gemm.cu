// Hybrid dense / 2:4 GEMM on the sm_100a tensor cores: Y = X * W_eff^T.
//
// "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section 2
// (inference and deployment): dense tiles run on the dense tensor-core path,
// 2:4 tiles on the sparse one, inside one kernel over the mixed tiles.  The
// page's kernels came from a Triton autotuner on Ampere-class GPUs; this is a
// hand-written Blackwell design:
//
//   * one CTA = one 128-row band of W x one tile of BN tokens (x one split-K
//     slice for decode).  D^T[128 x BN] lives in tensor memory (fp32).
//   * warp 0 (one thread): producer.  Per 64-column k-step it reads the
//     k-step's table entry and moves the packed weights with ONE bulk copy
//     (16 KB dense, or 8 KB kept values + the 2 KB metadata block of the pair
//     when it starts there) and the activations X with one TMA tensor load
//     (128-byte swizzle), all completing on the stage's mbarrier.
//   * warp 1 (one thread): MMA issuer.  Dense k-step: 4 x tcgen05.mma
//     (M128 N=BN K16).  2:4 k-step: tcgen05.cp of the metadata block into 4
//     TMEM columns when the pair starts, then 2 x tcgen05.mma.sp (M128 N=BN
//     K32).  Both accumulate into the same TMEM accumulator.  tcgen05.commit
//     frees the stage.
//   * warps 2..5: epilogue.  tcgen05.ld of the accumulator (each warp its
//     32-lane quarter), one rounding to bf16 (or fp32 out), stores to Y, or
//     fp32 split-K partials that a second kernel adds in slice order.
//
// Every mbarrier wait is bounded by %globaltimer; when one runs out the CTA
// raises the status word, drains its copies in flight and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "patch_common.cuh"
#include "patch_internal.h"

namespace patchk {

constexpr int kGemmThreads = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

template <int BN, int STAGES>
struct GemmCfg {
    static constexpr int kABytes = kDenseStepBytes;  // room for a dense k-step
    static constexpr int kBBytes = BN * kStep * 2;   // BN tokens x 64 columns
    static constexpr int kEBytes = kMetaBlockBytes;
    static constexpr int kStageBytes = kABytes + kBBytes + kEBytes;
    static constexpr int kTmemCols = (BN + 4 <= 32) ? 32 : (BN + 4 <= 64) ? 64
                                     : (BN + 4 <= 128) ? 128 : (BN + 4 <= 256) ? 256 : 512;
    static constexpr int kEcol = BN;  // metadata columns follow the accumulator
    static constexpr int kBarBytes = 8 * (2 * STAGES + 1) + 16;
    static constexpr int kSmemBytes = STAGES * kStageBytes + 1024 + kBarBytes;
    static_assert(kBBytes % 1024 == 0, "stage regions must stay 1024-B aligned");
};

struct GemmParams {
    const uint8_t *packed;
    const uint64_t *table;
    int64_t N, K, M;
    int nsteps;            // K / 64
    int steps_per_split;   // even, so a split never starts inside a k-pair
    void *Y;
    int y_fp32;
    float *partial;        // [splits][M][N] when gridDim.z > 1
    uint32_t *status;
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
hybrid_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const GemmParams p) {
    using C = GemmCfg<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::kStageBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *accf = empty + STAGES;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accf + 1);
    volatile uint32_t *abort_flag = tmem_slot + 1;   // raised by any role that gives up
    volatile uint32_t *never_flag = tmem_slot + 2;   // stays 0: time-only bounded waits

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int band = blockIdx.x, ttile = blockIdx.y, split = blockIdx.z;
    const int ks_begin = split * p.steps_per_split;
    const int ks_end = min(p.nsteps, ks_begin + p.steps_per_split);
    const int nks = ks_end - ks_begin;
    const uint64_t *tab = p.table + static_cast<int64_t>(band) * p.nsteps + ks_begin;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accf, 1);
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
    const bool skip = (*abort_flag != 0) || nks <= 0;

    if (warp == 0) {
        if (lane == 0 && !skip) {
            // ------------------------------------------------------ producer
            int issued = 0;
            bool ok = true;
            for (int i = 0; i < nks; ++i) {
                const int s = i % STAGES;
                const uint32_t ph = (i / STAGES) & 1u;
                if (i >= STAGES && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                const uint64_t e = tab[i];
                const bool sp = (e & kEntrySparse) != 0, has_e = (e & kEntryMeta) != 0;
                const uint32_t a_bytes = sp ? kSparseStepBytes : kDenseStepBytes;
                uint8_t *st = smem + s * C::kStageBytes;
                const uint8_t *src = p.packed + (e & kEntryOffsetMask);
                mbar_arrive_expect_tx(&full[s], a_bytes + C::kBBytes + (has_e ? C::kEBytes : 0));
                bulk_g2s(st, src, a_bytes, &full[s]);
                if (has_e) bulk_g2s(st + C::kABytes + C::kBBytes, src - C::kEBytes, C::kEBytes, &full[s]);
                tma_load_2d(st + C::kABytes, &tmap_x, (ks_begin + i) * kStep, ttile * BN, &full[s]);
                ++issued;
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
            // Drain: the last phase issued on every stage must have landed
            // before the CTA exits (a no-op when the MMA thread consumed all).
            for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
                mbar_wait_bounded(&full[i % STAGES], (i / STAGES) & 1u, never_flag,
                                  kWaitLimitNs / 4);
        }
    } else if (warp == 1) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------------- MMA
            const uint32_t d_tmem = tmem_base;
            const uint32_t e_tmem = tmem_base + C::kEcol;
            constexpr uint32_t kIdescDense = idesc_bf16(BN, false);
            bool ok = true;
            for (int i = 0; i < nks; ++i) {
                const int s = i % STAGES;
                const uint32_t ph = (i / STAGES) & 1u;
                if (!mbar_wait_bounded(&full[s], ph, abort_flag, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t e = tab[i];
                uint8_t *st = smem + s * C::kStageBytes;
                const uint32_t a_addr = smem_u32(st), b_addr = smem_u32(st + C::kABytes);
                if (e & kEntrySparse) {
                    if (e & kEntryMeta)
                        tmem_cp_128x128b(e_tmem, smem_desc(smem_u32(st + C::kABytes + C::kBBytes),
                                                           16, 128, kSwizzleNone));
                    const uint32_t half = static_cast<uint32_t>((ks_begin + i) & 1);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const uint64_t ad = smem_desc(a_addr + j * 32, 16, 512, kSwizzle64B);
                        const uint64_t bd = smem_desc(b_addr + j * 64, 16, 1024, kSwizzle128B);
                        mma_sparse(d_tmem, ad, bd, e_tmem + 2 * half, idesc_bf16(BN, true, j),
                                   (i > 0 || j > 0) ? 1u : 0u);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint64_t ad = smem_desc(a_addr + j * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = smem_desc(b_addr + j * 32, 16, 1024, kSwizzle128B);
                        mma_dense(d_tmem, ad, bd, kIdescDense, (i > 0 || j > 0) ? 1u : 0u);
                    }
                }
                tc_commit(&empty[s]);
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
            tc_commit(accf);  // fires once every MMA issued above has completed
        }
    } else if (!skip) {
        // ------------------------------------------------------- epilogue
        // The MMA thread always commits accf, also when it gave up, so this
        // wait is bounded by time only: no MMA may be in flight at dealloc.
        const bool ok = mbar_wait_bounded(accf, 0u, never_flag, kWaitLimitNs);
        tc_fence_after();
        if (!ok) {
            *abort_flag = 1u;
            atomicOr(p.status, kStatusTimeout);
        } else if (*abort_flag == 0) {
            const int quad = warp % 4;  // TMEM lanes 32*quad .. 32*quad+31
            const int64_t n = static_cast<int64_t>(band) * kBand + quad * 32 + lane;
            const int64_t m_base = static_cast<int64_t>(ttile) * BN;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + c0, r);
                tmem_ld_wait();
                if (gridDim.z > 1) {
                    float *dst = p.partial + static_cast<int64_t>(split) * p.M * p.N;
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int64_t m = m_base + c0 + q;
                        if (m < p.M) dst[m * p.N + n] = __uint_as_float(r[q]);
                    }
                } else if (p.y_fp32) {
                    float *y = static_cast<float *>(p.Y);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int64_t m = m_base + c0 + q;
                        if (m < p.M) y[m * p.N + n] = __uint_as_float(r[q]);
                    }
                } else {
                    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(p.Y);
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const int64_t m = m_base + c0 + q;
                        if (m < p.M) y[m * p.N + n] = __float2bfloat16_rn(__uint_as_float(r[q]));
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::kTmemCols);
}

// Y[m,n] = sum over split slices s (in order) of partial[s][m][n].
__global__ void splitk_reduce_kernel(const float *__restrict__ partial, int splits, int64_t M,
                                     int64_t N, void *Y, int y_fp32) {
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t total = M * N;
    if (idx >= total) return;
    float acc = 0.0f;
    for (int s = 0; s < splits; ++s) acc = __fadd_rn(acc, __ldg(partial + s * total + idx));
    if (y_fp32)
        static_cast<float *>(Y)[idx] = acc;
    else
        static_cast<__nv_bfloat16 *>(Y)[idx] = __float2bfloat16_rn(acc);
}

// ------------------------------------------------------------------- host
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
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

// X [M,K] bf16 row-major, box = 64 columns x BN rows, 128-byte swizzle;
// rows past M read as zero.
bool make_x_map(CUtensorMap *map, const void *X, int64_t M, int64_t K, int bn) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kStep), static_cast<cuuint32_t>(bn)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES>
cudaError_t run(const GemmLaunch &g, int splits, int steps_per_split, cudaStream_t stream) {
    using C = GemmCfg<BN, STAGES>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(hybrid_gemm_kernel<BN, STAGES>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err != cudaSuccess) return attr_err;
    CUtensorMap map;
    if (!make_x_map(&map, g.X, g.M, g.K, BN)) return cudaErrorInvalidValue;
    GemmParams p;
    p.packed = g.packed;
    p.table = g.table;
    p.N = g.N;
    p.K = g.K;
    p.M = g.M;
    p.nsteps = static_cast<int>(g.K / kStep);
    p.steps_per_split = steps_per_split;
    p.Y = g.Y;
    p.y_fp32 = g.y_fp32;
    p.partial = splits > 1 ? g.workspace : nullptr;
    p.status = g.status;
    dim3 grid(static_cast<unsigned>(g.N / kBand), static_cast<unsigned>((g.M + BN - 1) / BN),
              static_cast<unsigned>(splits));
    hybrid_gemm_kernel<BN, STAGES><<<grid, kGemmThreads, C::kSmemBytes, stream>>>(map, p);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess || splits == 1) return err;
    const int64_t total = g.M * g.N;
    splitk_reduce_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
        g.workspace, splits, g.M, g.N, g.Y, g.y_fp32);
    return cudaGetLastError();
}

}  // namespace

int decode_splits(int64_t N, int64_t K, int num_sms) {
    const int64_t bands = N / kBand;
    const int64_t pairs = K / (2 * kStep);
    // aim at two resident CTAs per SM
    int64_t s = (2 * static_cast<int64_t>(num_sms) + bands - 1) / bands;
    if (s > pairs) s = pairs;
    if (s > 16) s = 16;
    if (s < 1) s = 1;
    // balance: slices of ceil(pairs / s) pairs, drop empty trailing slices
    const int64_t per = (pairs + s - 1) / s;
    return static_cast<int>((pairs + per - 1) / per);
}

cudaError_t launch_hybrid_gemm(const GemmLaunch &g, cudaStream_t stream) {
    const int nsteps = static_cast<int>(g.K / kStep);
    if (g.M <= 16 && g.workspace != nullptr) {
        int splits = decode_splits(g.N, g.K, g.num_sms);
        const int pairs = nsteps / 2;
        const int per_pairs = (pairs + splits - 1) / splits;
        if (static_cast<int64_t>(splits) * g.M * g.N > g.workspace_floats) splits = 1;
        const int steps = splits > 1 ? 2 * per_pairs : nsteps;
        return run<16, 5>(g, splits, steps, stream);
    }
    if (g.M <= 64) return run<64, 6>(g, 1, nsteps, stream);
    if (g.M <= 128) return run<128, 6>(g, 1, nsteps, stream);
    return run<256, 4>(g, 1, nsteps, stream);
}

}  // namespace patchk
