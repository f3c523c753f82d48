// Column sums of squares of the calibration activations (sm_100a): the
// activation term of the Wanda score, s_j = sum_t x_tj^2, whose square root
// weighs |W_ij| ("SparseGPT vs Wanda: one-shot LLM pruning without
// retraining", section on Wanda: weight magnitude times the activation of its
// input channel).
//
// Fixed order, so s is bit-reproducible for any launch shape and any split of
// the tokens at multiples of 128: tokens are cut into chunks of 128, each
// chunk summed token by token from 0.0 (colsq_partial_kernel), then the chunk
// sums are added chunk by chunk from 0.0 (colsq_final_kernel).  A bf16 value
// squared is exact in fp64, so only the additions round.
//
// Both kernels stream HBM: the partial kernel reads every calibration byte
// once with 16-byte loads (a warp reads 512 contiguous bytes of a token row),
// the fold reads the chunk partials (1/32 of the calibration bytes) once,
// several stages deep.
#include <cuda_runtime.h>
#include <stdint.h>

#include "patch_internal.h"

namespace patchk {

constexpr int kColsqChunk = 128;   // tokens per fixed-order chunk
constexpr int kColsqThreads = 128;  // a block: 128 threads x 8 columns = 1024 columns
constexpr int kColsqUnroll = 4;     // token rows in flight per thread (4, 8 and 16 measured: 4 best)
constexpr int kFoldCols = 32;       // columns per fold block (one warp folds them)
constexpr int kFoldRows = 32;       // chunk partials per stage (8 KB)
constexpr int kFoldStages = 6;      // ring of stages: 48 KB of shared memory
constexpr int kFoldThreads = 256;

// One thread = 8 consecutive columns x one 128-token chunk, the chunk's tokens
// in order.  Every token row is read with one 16-byte load per thread, so a
// warp reads 512 contiguous bytes of each row; kColsqUnroll rows are in flight
// before the first is used.  Per column the sum is the same chain of fp64
// additions as a one-column loop: a = 0; a = a + x_t^2 for t in the chunk.
// x_t^2 is exact in fp64 (an 8-bit significand squared), so one fused
// multiply-add per element rounds exactly as the multiply and then the add.
__global__ void __launch_bounds__(kColsqThreads)
colsq_partial_kernel(const uint16_t *__restrict__ X, int64_t T, int64_t K,
                     double *__restrict__ partial) {
    // grid.x: chunks (no limit that matters for T), grid.y: 1024-column blocks
    const int64_t cg = static_cast<int64_t>(blockIdx.y) * kColsqThreads + threadIdx.x;
    if (cg * 8 >= K) return;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kColsqChunk;
    const int64_t t1 = min(T, t0 + kColsqChunk);
    const uint4 *src = reinterpret_cast<const uint4 *>(X + t0 * K) + cg;
    const int64_t row16 = K / 8;  // 16-byte words per token row
    double a[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) a[q] = 0.0;
    auto add_row = [&](const uint4 v) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const double lo = static_cast<double>(__uint_as_float(w[h] << 16));
            const double hi = static_cast<double>(__uint_as_float(w[h] & 0xFFFF0000u));
            a[2 * h] = __fma_rn(lo, lo, a[2 * h]);
            a[2 * h + 1] = __fma_rn(hi, hi, a[2 * h + 1]);
        }
    };
    int64_t t = t0;
    for (; t + kColsqUnroll <= t1; t += kColsqUnroll) {
        uint4 v[kColsqUnroll];
#pragma unroll
        for (int u = 0; u < kColsqUnroll; ++u) v[u] = __ldcs(src + u * row16);
#pragma unroll
        for (int u = 0; u < kColsqUnroll; ++u) add_row(v[u]);
        src += kColsqUnroll * row16;
    }
    for (; t < t1; ++t) {
        add_row(__ldcs(src));
        src += row16;
    }
    double2 *dst = reinterpret_cast<double2 *>(partial + static_cast<int64_t>(blockIdx.x) * K + cg * 8);
#pragma unroll
    for (int q = 0; q < 4; ++q) dst[q] = make_double2(a[2 * q], a[2 * q + 1]);
}

// 16-byte asynchronous copy global -> shared (L2 only); commit this thread's
// copies as one group; wait until at most N of its groups are pending.
__device__ __forceinline__ void fold_cp16(void *smem_dst, const void *gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
                 "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void fold_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void fold_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// s_j = chunk sums added in chunk order; n_j = sqrt(s_j).  A block owns 32
// columns (a 256-byte run of every partial row).  Its threads copy stages of
// kFoldRows partial rows into a ring of kFoldStages shared-memory buffers with
// 16-byte asynchronous copies (kFoldStages - 1 stages in flight), and warp 0
// adds each landed stage, lane j to column j, row by row in chunk order.  The
// chain of fp64 additions per column (one per 128-token chunk) is what bounds
// it: 2048 chunks take about 30 us however deep the ring (measured on B200).
__global__ void __launch_bounds__(kFoldThreads)
colsq_final_kernel(const double *__restrict__ partial, int64_t chunks, int64_t K,
                   double *__restrict__ colsq_out, double *__restrict__ norm_out) {
    __shared__ __align__(16) double ring[kFoldStages][kFoldRows][kFoldCols];
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int64_t j0 = static_cast<int64_t>(blockIdx.x) * kFoldCols;
    const int64_t j = j0 + lane;
    const int64_t nstages = (chunks + kFoldRows - 1) / kFoldRows;
    // stage g into buffer g % kFoldStages: row r, 16-byte chunk c of the run
    auto issue = [&](int64_t g) {
        if (g < nstages) {
#pragma unroll
            for (int k = 0; k < kFoldRows * (kFoldCols / 2) / kFoldThreads; ++k) {
                const int q = k * kFoldThreads + tid;
                const int r = q / (kFoldCols / 2), c = q % (kFoldCols / 2);
                const int64_t row = g * kFoldRows + r, col = j0 + 2 * c;
                if (row < chunks && col < K)  // K is even: a copied pair is whole
                    fold_cp16(&ring[g % kFoldStages][r][2 * c], partial + row * K + col);
            }
        }
        fold_commit();  // one group per stage, empty or not
    };
    for (int g = 0; g < kFoldStages - 1; ++g) issue(g);
    double s = 0.0;
    for (int64_t g = 0; g < nstages; ++g) {
        fold_wait<kFoldStages - 2>();  // this thread's copies of stage g have landed
        __syncthreads();               // everyone's have
        if (warp == 0) {
            const int n = static_cast<int>(min(static_cast<int64_t>(kFoldRows), chunks - g * kFoldRows));
            const double(*t)[kFoldCols] = ring[g % kFoldStages];
            for (int r = 0; r < n; ++r) s = __dadd_rn(s, t[r][lane]);
        }
        __syncthreads();  // buffer g % kFoldStages is free again
        issue(g + kFoldStages - 1);
    }
    fold_wait<0>();
    if (warp == 0 && j < K) {
        if (colsq_out) colsq_out[j] = s;
        if (norm_out) norm_out[j] = __dsqrt_rn(s);
    }
}

cudaError_t launch_colsq_partials(const void *Xcal, int64_t T, int64_t K, double *partial,
                                  cudaStream_t stream) {
    const int64_t chunks = (T + kColsqChunk - 1) / kColsqChunk;
    const int64_t col_blocks = (K / 8 + kColsqThreads - 1) / kColsqThreads;
    if (T < 1 || K < 8 || K % 8 != 0 || col_blocks > 65535 || chunks > 0x7FFFFFFF)
        return cudaErrorInvalidValue;
    dim3 grid(static_cast<unsigned>(chunks), static_cast<unsigned>(col_blocks));
    colsq_partial_kernel<<<grid, kColsqThreads, 0, stream>>>(static_cast<const uint16_t *>(Xcal), T,
                                                             K, partial);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_colsq_fold(const double *partial, int64_t chunks, int64_t K, double *colsq_out,
                              double *norm_out, cudaStream_t stream) {
    if (chunks < 1 || K < 1 || (K + kFoldCols - 1) / kFoldCols > 0x7FFFFFFF) return cudaErrorInvalidValue;
    colsq_final_kernel<<<static_cast<unsigned>((K + kFoldCols - 1) / kFoldCols), kFoldThreads, 0, stream>>>(
        partial, chunks, K, colsq_out, norm_out);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_colsq(const void *Xcal, int64_t T, int64_t K, double *partial,
                         double *colsq_out, double *norm_out, cudaStream_t stream) {
    cudaError_t e = launch_colsq_partials(Xcal, T, K, partial, stream);
    if (e != cudaSuccess) return e;
    return launch_colsq_fold(partial, (T + kColsqChunk - 1) / kColsqChunk, K, colsq_out, norm_out, stream);
}

}  // namespace patchk
