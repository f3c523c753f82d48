// Wanda 2:4 mask builder for the tile-hybrid sparse linear layer (sm_100a).
//
// Steps (each a kernel, all HBM-streaming):
//   1. colsq_partial / colsq_final: s_j = sum_t x_tj^2 over calibration tokens
//      in a fixed order (128-token chunks summed token by token, chunk sums
//      added chunk by chunk), so s is bit-reproducible for any launch shape;
//      n_j = sqrt(s_j) (IEEE round-to-nearest).
//   2. score_mask: per tile, Wanda scores |W_ij| * n_j (one fp64 multiply),
//      top-2-of-4 per group (score descending, lower index on ties), the 4-bit
//      code idx0 | idx1 << 2, and the tile's pruned-score loss (rows left to
//      right, then rows top to bottom).
//   3. select_map: tiles ranked by (loss ascending, index ascending); the
//      first floor(f * n_tiles) become 2:4.
//
// Sources: the Wanda criterion (weight magnitude times the activation of its
// input channel) is from "SparseGPT vs Wanda: one-shot LLM pruning without
// retraining", section on Wanda; 2:4 groups and the dense / 2:4 tile choice
// are from "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", sections 1
// and 2 (core mechanism).  PATCH learns the tile choice; ranking tiles by the
// Wanda score that 2:4 pruning would remove is this library's data-free
// stand-in for it.
#include <cuda_runtime.h>
#include <stdint.h>

#include "patch_internal.h"

namespace patchk {

constexpr int kColsqChunk = 128;   // tokens per fixed-order chunk
constexpr int kColsqThreads = 256;
constexpr int kColsqUnroll = 16;

__device__ __forceinline__ double bf16_lo_to_f64(uint32_t v) {
    return static_cast<double>(__uint_as_float(v << 16));
}
__device__ __forceinline__ double bf16_hi_to_f64(uint32_t v) {
    return static_cast<double>(__uint_as_float(v & 0xFFFF0000u));
}

// One thread = two adjacent columns x one 128-token chunk.  Reads are 4-byte
// per thread, 128 contiguous bytes per warp and row.
__global__ void __launch_bounds__(kColsqThreads)
colsq_partial_kernel(const uint32_t *__restrict__ X2, int64_t T, int64_t K,
                     double *__restrict__ partial) {
    const int64_t pairs = K / 2;
    const int64_t p = static_cast<int64_t>(blockIdx.x) * kColsqThreads + threadIdx.x;
    if (p >= pairs) return;
    const int64_t t0 = static_cast<int64_t>(blockIdx.y) * kColsqChunk;
    const int64_t t1 = min(T, t0 + kColsqChunk);
    const uint32_t *src = X2 + t0 * pairs + p;
    double a = 0.0, b = 0.0;
    int64_t t = t0;
    for (; t + kColsqUnroll <= t1; t += kColsqUnroll) {
        uint32_t v[kColsqUnroll];
#pragma unroll
        for (int u = 0; u < kColsqUnroll; ++u) v[u] = __ldg(src + u * pairs);
#pragma unroll
        for (int u = 0; u < kColsqUnroll; ++u) {
            const double x0 = bf16_lo_to_f64(v[u]), x1 = bf16_hi_to_f64(v[u]);
            a = __dadd_rn(a, __dmul_rn(x0, x0));
            b = __dadd_rn(b, __dmul_rn(x1, x1));
        }
        src += kColsqUnroll * pairs;
    }
    for (; t < t1; ++t) {
        const uint32_t v = __ldg(src);
        const double x0 = bf16_lo_to_f64(v), x1 = bf16_hi_to_f64(v);
        a = __dadd_rn(a, __dmul_rn(x0, x0));
        b = __dadd_rn(b, __dmul_rn(x1, x1));
        src += pairs;
    }
    reinterpret_cast<double2 *>(partial + blockIdx.y * K)[p] = make_double2(a, b);
}

// s_j = chunk sums added in chunk order; n_j = sqrt(s_j).
__global__ void __launch_bounds__(256)
colsq_final_kernel(const double *__restrict__ partial, int64_t chunks, int64_t K,
                   double *__restrict__ colsq_out, double *__restrict__ norm_out) {
    const int64_t j = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
    if (j >= K) return;
    double s = 0.0;
    int64_t c = 0;
    constexpr int U = 16;
    for (; c + U <= chunks; c += U) {
        double v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) v[u] = __ldg(partial + (c + u) * K + j);
#pragma unroll
        for (int u = 0; u < U; ++u) s = __dadd_rn(s, v[u]);
    }
    for (; c < chunks; ++c) s = __dadd_rn(s, __ldg(partial + c * K + j));
    if (colsq_out) colsq_out[j] = s;
    norm_out[j] = __dsqrt_rn(s);
}

// Norms from caller-provided sums of squares (shared-input matrices).
__global__ void norms_from_colsq_kernel(const double *__restrict__ colsq_in, int64_t K,
                                        double *__restrict__ colsq_out,
                                        double *__restrict__ norm_out) {
    const int64_t j = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
    if (j >= K) return;
    const double s = colsq_in[j];
    if (colsq_out) colsq_out[j] = s;
    norm_out[j] = __dsqrt_rn(s);
}

// ----------------------------------------------------------------- scoring
constexpr int kScoreThreads = 128;

// Select the two kept positions of one group: q is kept iff fewer than two
// other candidates come before it in the order (score desc, index asc).
__device__ __forceinline__ uint32_t top2_code(const double s[4]) {
    // For p < q, p precedes q iff s_p >= s_q (a tie goes to the lower index).
    const int b01 = s[0] >= s[1], b02 = s[0] >= s[2], b03 = s[0] >= s[3];
    const int b12 = s[1] >= s[2], b13 = s[1] >= s[3], b23 = s[2] >= s[3];
    const int r0 = (1 - b01) + (1 - b02) + (1 - b03);
    const int r1 = b01 + (1 - b12) + (1 - b13);
    const int r2 = b02 + b12 + (1 - b23);
    const int r3 = b03 + b13 + b23;
    const int k0 = r0 < 2, k1 = r1 < 2, k2 = r2 < 2, k3 = r3 < 2;
    // lowest and highest kept positions
    const uint32_t lo = k0 ? 0u : (k1 ? 1u : 2u);
    const uint32_t hi = k3 ? 3u : (k2 ? 2u : 1u);
    return lo | (hi << 2);
}

// One CTA per tile.  The tile is staged in shared memory with coalesced 16-B
// loads (rows padded by 16 B); then thread r owns row r of the tile, so the
// row's pruned-score sum runs left to right in one thread.
template <int TN, int TK>
__global__ void __launch_bounds__(kScoreThreads)
score_mask_kernel(const uint16_t *__restrict__ W, const double *__restrict__ norm, int64_t N,
                  int64_t K, uint32_t *__restrict__ meta, double *__restrict__ loss) {
    constexpr int kRowElems = TK + 8;       // padded row (bf16 elements)
    constexpr int kChunksPerRow = TK / 8;   // 16-byte chunks per tile row
    constexpr int kWordsPerRow = TK / 32;   // meta words per tile row
    __shared__ __align__(16) uint16_t ws[TN * kRowElems];
    __shared__ double ns[TK];
    __shared__ double rows[TN];
    __shared__ uint32_t ms[TN * kWordsPerRow];

    const int64_t tiles_k = K / TK;
    const int64_t t = blockIdx.x;
    const int64_t i0 = (t / tiles_k) * TN, j0 = (t % tiles_k) * TK;
    const int tid = threadIdx.x;

    for (int u = tid; u < TN * kChunksPerRow; u += kScoreThreads) {
        const int r = u / kChunksPerRow, c = u % kChunksPerRow;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(W + (i0 + r) * K + j0) + c);
        *reinterpret_cast<uint4 *>(ws + r * kRowElems + c * 8) = v;
    }
    for (int u = tid; u < TK; u += kScoreThreads) ns[u] = __ldg(norm + j0 + u);
    __syncthreads();

    if (tid < TN) {
        const uint16_t *row = ws + tid * kRowElems;
        double rsum = 0.0;
#pragma unroll 1
        for (int w = 0; w < kWordsPerRow; ++w) {
            uint32_t word = 0;
#pragma unroll
            for (int h = 0; h < 4; ++h) {  // 4 x 8 columns = one 32-column word
                const uint4 v = *reinterpret_cast<const uint4 *>(row + w * 32 + h * 8);
                const uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int gg = 0; gg < 2; ++gg) {
                    const int col = w * 32 + h * 8 + gg * 4;
                    double s[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t pairbits = e[gg * 2 + q / 2];
                        const uint32_t bits = (q & 1) ? (pairbits >> 16) : (pairbits & 0xFFFFu);
                        const double mag = static_cast<double>(__uint_as_float((bits & 0x7FFFu) << 16));
                        s[q] = __dmul_rn(mag, ns[col + q]);
                    }
                    const uint32_t code = top2_code(s);
                    const uint32_t lo = code & 3u, hi = code >> 2;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (q != static_cast<int>(lo) && q != static_cast<int>(hi))
                            rsum = __dadd_rn(rsum, s[q]);
                    word |= code << (4 * (h * 2 + gg));
                }
            }
            ms[tid * kWordsPerRow + w] = word;
        }
        rows[tid] = rsum;
    }
    __syncthreads();

    const int64_t words_k = K / 32;
    for (int u = tid; u < TN * kWordsPerRow; u += kScoreThreads) {
        const int r = u / kWordsPerRow, w = u % kWordsPerRow;
        meta[(i0 + r) * words_k + j0 / 32 + w] = ms[u];
    }
    if (tid == 0) {
        double total = 0.0;
        for (int r = 0; r < TN; ++r) total = __dadd_rn(total, rows[r]);
        loss[t] = total;
    }
}

// ------------------------------------------------------------- tile ranking
constexpr int kRankThreads = 128;
constexpr int kRankSlice = 256;

// rank[t] += #{u in this block's slice : (L_u, u) < (L_t, t)}.  Integer
// counts, so the accumulated rank does not depend on the order of atomics.
__global__ void __launch_bounds__(kRankThreads)
rank_tiles_kernel(const double *__restrict__ loss, int64_t n_tiles, int32_t *__restrict__ rank) {
    __shared__ double sl[kRankSlice];
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kRankThreads + threadIdx.x;
    const int64_t u0 = static_cast<int64_t>(blockIdx.y) * kRankSlice;
    const int64_t u1 = min(n_tiles, u0 + kRankSlice);
    for (int64_t u = u0 + threadIdx.x; u < u1; u += kRankThreads) sl[u - u0] = loss[u];
    __syncthreads();
    if (t >= n_tiles) return;
    const double lt = loss[t];
    int32_t r = 0;
    for (int64_t u = u0; u < u1; ++u) {
        const double lu = sl[u - u0];
        r += (lu < lt) || (lu == lt && u < t);
    }
    atomicAdd(rank + t, r);
}

// Bit t of the map is set iff rank[t] < n_sparse.  One warp per 32 tiles.
__global__ void map_from_rank_kernel(const int32_t *__restrict__ rank, int64_t n_tiles,
                                     int64_t n_sparse, uint32_t *__restrict__ map) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t words = (n_tiles + 31) / 32;
    if (t / 32 >= words) return;
    const bool bit = t < n_tiles && rank[t] < n_sparse;
    const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, bit);
    if ((threadIdx.x & 31) == 0) map[t / 32] = ballot;
}

// ------------------------------------------------------------------ launch
cudaError_t launch_colsq(const void *Xcal, int64_t T, int64_t K, double *partial,
                         double *colsq_out, double *norm_out, cudaStream_t stream) {
    const int64_t chunks = (T + kColsqChunk - 1) / kColsqChunk;
    const int64_t pairs = K / 2;
    dim3 grid(static_cast<unsigned>((pairs + kColsqThreads - 1) / kColsqThreads),
              static_cast<unsigned>(chunks));
    colsq_partial_kernel<<<grid, kColsqThreads, 0, stream>>>(static_cast<const uint32_t *>(Xcal), T,
                                                             K, partial);
    colsq_final_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, stream>>>(
        partial, chunks, K, colsq_out, norm_out);
    return cudaGetLastError();
}

cudaError_t launch_norms_from_colsq(const double *colsq_in, int64_t K, double *colsq_out,
                                    double *norm_out, cudaStream_t stream) {
    norms_from_colsq_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, stream>>>(
        colsq_in, K, colsq_out, norm_out);
    return cudaGetLastError();
}

cudaError_t launch_score_mask(const void *W, const double *norm, int64_t N, int64_t K, int tn,
                              int tk, uint32_t *meta, double *loss, cudaStream_t stream) {
    const int64_t n_tiles = (N / tn) * (K / tk);
    const uint16_t *w = static_cast<const uint16_t *>(W);
    const unsigned g = static_cast<unsigned>(n_tiles);
    if (tn == 128 && tk == 128)
        score_mask_kernel<128, 128><<<g, kScoreThreads, 0, stream>>>(w, norm, N, K, meta, loss);
    else if (tn == 128 && tk == 64)
        score_mask_kernel<128, 64><<<g, kScoreThreads, 0, stream>>>(w, norm, N, K, meta, loss);
    else if (tn == 64 && tk == 128)
        score_mask_kernel<64, 128><<<g, kScoreThreads, 0, stream>>>(w, norm, N, K, meta, loss);
    else if (tn == 64 && tk == 64)
        score_mask_kernel<64, 64><<<g, kScoreThreads, 0, stream>>>(w, norm, N, K, meta, loss);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

cudaError_t launch_select_map(const double *loss, int64_t n_tiles, int64_t n_sparse, int32_t *rank,
                              uint32_t *map, cudaStream_t stream) {
    cudaError_t err = cudaMemsetAsync(rank, 0, sizeof(int32_t) * n_tiles, stream);
    if (err != cudaSuccess) return err;
    dim3 grid(static_cast<unsigned>((n_tiles + kRankThreads - 1) / kRankThreads),
              static_cast<unsigned>((n_tiles + kRankSlice - 1) / kRankSlice));
    rank_tiles_kernel<<<grid, kRankThreads, 0, stream>>>(loss, n_tiles, rank);
    const int64_t words = (n_tiles + 31) / 32;
    const int64_t threads = words * 32;
    map_from_rank_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        rank, n_tiles, n_sparse, map);
    return cudaGetLastError();
}

}  // namespace patchk
