// Wanda 2:4 mask builder for the tile-hybrid sparse linear layer (sm_100a).
//
// Steps (each a kernel, all HBM-streaming):
//   1. column sums of squares of the calibration set: csrc/colsq_kernels.cu;
//      here only n_j = sqrt(s_j) from caller-given sums.
//   2. score_mask: per tile, Wanda scores |W_ij| * n_j (one fp64 multiply),
//      top-2-of-4 per group (score descending, lower index on ties), the 4-bit
//      code idx0 | idx1 << 2, and the tile's pruned-score loss (32-column words
//      left to right, a row's words left to right, rows as a pairwise tree).
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
// Select the two kept positions of one group: q is kept iff fewer than two
// other candidates come before it in the order (score desc, index asc); for
// p < q, p precedes q iff s_p >= s_q (a tie goes to the lower index).  As a
// table over the six comparison bits
// i = [s0>=s1] | [s0>=s2]<<1 | [s0>=s3]<<2 | [s1>=s2]<<3 | [s1>=s3]<<4 | [s2>=s3]<<5:
// low nibble the 4-bit code (lowest | highest kept position << 2), high
// nibble the pruned positions (those not in the code).  Every one of the 64
// patterns gets the value of the rank formula, reachable or not.
__host__ __device__ constexpr uint8_t top2_entry(int i) {
    const int b01 = i & 1, b02 = (i >> 1) & 1, b03 = (i >> 2) & 1;
    const int b12 = (i >> 3) & 1, b13 = (i >> 4) & 1, b23 = (i >> 5) & 1;
    const int r0 = (1 - b01) + (1 - b02) + (1 - b03);
    const int r1 = b01 + (1 - b12) + (1 - b13);
    const int r2 = b02 + b12 + (1 - b23);
    const int r3 = b03 + b13 + b23;
    const int k0 = r0 < 2, k1 = r1 < 2, k2 = r2 < 2, k3 = r3 < 2;
    const int lo = k0 ? 0 : (k1 ? 1 : 2);
    const int hi = k3 ? 3 : (k2 ? 2 : 1);
    const int pruned = 0xF & ~((1 << lo) | (1 << hi));
    return static_cast<uint8_t>(lo | (hi << 2) | (pruned << 4));
}
struct Top2Table {
    uint32_t w[16];  // entry i in byte i % 4 of word i / 4
};
__host__ __device__ constexpr Top2Table make_top2_table() {
    Top2Table t{};
    for (int i = 0; i < 64; ++i) t.w[i / 4] |= static_cast<uint32_t>(top2_entry(i)) << (8 * (i % 4));
    return t;
}
__constant__ Top2Table kTop2Table = make_top2_table();

// 4:8 groups: q is kept iff fewer than four other candidates come before it
// in the order (score desc, index asc); returns the 8-bit keep mask.
__device__ __forceinline__ uint32_t top4_mask(const double s[8]) {
    int r[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) r[q] = 0;
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = a + 1; b < 8; ++b) {
            // a < b: a precedes b iff s_a >= s_b (a tie goes to the lower index)
            const int ab = s[a] >= s[b];
            r[b] += ab;
            r[a] += 1 - ab;
        }
    uint32_t m = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) m |= static_cast<uint32_t>(r[q] < 4) << q;
    return m;
}

// |w| of a bf16 bit pattern, exactly, as a double (sign cleared: -0 -> +0).
// Normal values are rebuilt with integer operations (exponent rebias 127 ->
// 1023, mantissa moved up); zero and subnormals take the conversion path.
__device__ __forceinline__ double bf16_abs_f64(uint32_t bits16) {
    const uint32_t e8 = (bits16 >> 7) & 0xFFu, m7 = bits16 & 0x7Fu;
    if (e8 != 0u) return __hiloint2double(static_cast<int>(((e8 + 896u) << 20) | (m7 << 13)), 0);
    return static_cast<double>(__uint_as_float((bits16 & 0x7FFFu) << 16));
}

// One CTA per tile, one thread per (row, 32-column word) of the tile.  A
// thread reads its 64 bytes of W with coalesced 16-byte loads (a warp covers
// whole rows), scores its groups (PAT = 2: eight 2:4 groups, 4-bit codes;
// PAT = 4: four 4:8 groups, 8-bit keep masks), writes the meta word and the
// word's pruned-score sum (left to right).  The CTA then adds each row's
// words left to right and the rows as a balanced pairwise tree.
template <int TN, int TK, int PAT>
__global__ void __launch_bounds__(TN *(TK / 32), PAT == 2 ? 2048 / (TN * (TK / 32)) : 1)
score_mask_kernel(const uint16_t *__restrict__ W, const double *__restrict__ norm, int64_t N,
                  int64_t K, uint32_t *__restrict__ meta, double *__restrict__ loss,
                  int32_t *__restrict__ rank, uint32_t *__restrict__ done) {
    constexpr int WPR = TK / 32;      // words per tile row
    constexpr int kNormStride = 34;   // padded: the words' norms sit in different banks (16-B rows)
    constexpr int kWarps = TN / 32;   // warps holding the tile's row sums
    __shared__ __align__(16) double ns[WPR * kNormStride];
    __shared__ uint32_t top2[16];
    __shared__ double wsum[TN * WPR];
    __shared__ double warp_sum[kWarps];
    const int64_t tiles_k = K / TK;
    const int64_t t = blockIdx.x;
    const int64_t i0 = (t / tiles_k) * TN, j0 = (t % tiles_k) * TK;
    const int tid = threadIdx.x;
    const int r = tid / WPR, w = tid % WPR;

    for (int u = tid; u < TK; u += TN * WPR) ns[(u / 32) * kNormStride + u % 32] = __ldg(norm + j0 + u);
    if (PAT == 2 && tid < 16) top2[tid] = kTop2Table.w[tid];
    const uint4 *src = reinterpret_cast<const uint4 *>(W + (i0 + r) * K + j0 + 32 * w);
    uint4 v[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) v[h] = __ldg(src + h);
    __syncthreads();

    const double *nw = ns + w * kNormStride;
    double acc = 0.0;
    uint32_t word = 0;
    if constexpr (PAT == 4) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // group h: columns 8h .. 8h+7 of the word
            const uint32_t e[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
            double sc[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t bits = (q & 1) ? (e[q / 2] >> 16) : (e[q / 2] & 0xFFFFu);
                sc[q] = __dmul_rn(bf16_abs_f64(bits), nw[8 * h + q]);
            }
            const uint32_t m = top4_mask(sc);
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (!((m >> q) & 1u)) acc = __dadd_rn(acc, sc[q]);
            word |= m << (8 * h);
        }
    } else {
        const uint8_t *tab = reinterpret_cast<const uint8_t *>(top2);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const uint32_t e[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int col = h * 8 + gg * 4;
                const double2 n01 = *reinterpret_cast<const double2 *>(nw + col);
                const double2 n23 = *reinterpret_cast<const double2 *>(nw + col + 2);
                // |w| exactly: bf16 -> fp32 (the bits moved up), sign cleared
                // for both halves of a word at once, fp32 -> fp64 exact
                const uint32_t a01 = e[gg * 2] & 0x7FFF7FFFu, a23 = e[gg * 2 + 1] & 0x7FFF7FFFu;
                double sc[4];
                sc[0] = __dmul_rn(static_cast<double>(__uint_as_float(a01 << 16)), n01.x);
                sc[1] = __dmul_rn(static_cast<double>(__uint_as_float(a01 & 0xFFFF0000u)), n01.y);
                sc[2] = __dmul_rn(static_cast<double>(__uint_as_float(a23 << 16)), n23.x);
                sc[3] = __dmul_rn(static_cast<double>(__uint_as_float(a23 & 0xFFFF0000u)), n23.y);
                const uint32_t idx = static_cast<uint32_t>(sc[0] >= sc[1]) | (static_cast<uint32_t>(sc[0] >= sc[2]) << 1) |
                                     (static_cast<uint32_t>(sc[0] >= sc[3]) << 2) |
                                     (static_cast<uint32_t>(sc[1] >= sc[2]) << 3) |
                                     (static_cast<uint32_t>(sc[1] >= sc[3]) << 4) |
                                     (static_cast<uint32_t>(sc[2] >= sc[3]) << 5);
                const uint32_t ent = tab[idx];
                // the pruned scores, left to right
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if ((ent >> (4 + q)) & 1u) acc = __dadd_rn(acc, sc[q]);
                word |= (ent & 0xFu) << (4 * (h * 2 + gg));
            }
        }
    }
    meta[(i0 + r) * (K / 32) + j0 / 32 + w] = word;
    wsum[tid] = acc;
    __syncthreads();
    if (tid < TN) {
        // row sum: the row's words left to right
        double row = 0.0;
#pragma unroll
        for (int q = 0; q < WPR; ++q) row = __dadd_rn(row, wsum[tid * WPR + q]);
        // balanced pairwise tree over rows: levels 1..5 inside the warp (node q
        // of level k lives in lane q * 2^k), then across the warps
#pragma unroll
        for (int off = 1; off < 32; off *= 2) {
            const double other = __shfl_down_sync(0xFFFFFFFFu, row, off);
            row = __dadd_rn(row, other);
        }
        if ((tid & 31) == 0) warp_sum[tid / 32] = row;
    }
    __syncthreads();
    if (tid == 0 && rank) {  // counters of the ranking step that follows
        rank[t] = 0;
        if (t == 0) *done = 0u;
    }
    if (tid == 0) {
        double x[kWarps];
#pragma unroll
        for (int q = 0; q < kWarps; ++q) x[q] = warp_sum[q];
#pragma unroll
        for (int n = kWarps; n > 1; n /= 2)
#pragma unroll
            for (int q = 0; q < n / 2; ++q) x[q] = __dadd_rn(x[2 * q], x[2 * q + 1]);
        loss[t] = x[0];
    }
}

// ------------------------------------------------------------- tile ranking
constexpr int kRankThreads = 128;
constexpr int kRankPerThread = 2;                           // tiles t per thread
constexpr int kRankTiles = kRankThreads * kRankPerThread;   // tiles t per block
constexpr int kRankSlice = 256;                             // tiles u per block, at most

// slice of u per block: narrower for few tiles, so the comparisons spread over
// enough blocks to fill the device
inline int rank_slice(int64_t n_tiles) { return n_tiles <= 4096 ? 64 : kRankSlice; }

// rank[t] += #{u in this block's slice : (L_u, u) < (L_t, t)}.  Integer
// counts, so the accumulated rank does not depend on the order of atomics.
// The last block to finish writes the bitmap: bit t set iff rank[t] < n_sparse.
// For u < t the pair order is L_u <= L_t, for u > t it is L_u < L_t; a slice
// wholly below or above a thread's tiles takes the one comparison.
__global__ void __launch_bounds__(kRankThreads)
rank_tiles_kernel(const double *__restrict__ loss, int64_t n_tiles, int64_t n_sparse, int slice,
                  int32_t *__restrict__ rank, uint32_t *__restrict__ done, uint32_t *__restrict__ map) {
    __shared__ double sl[kRankSlice];
    __shared__ bool last;
    const int64_t tb = static_cast<int64_t>(blockIdx.x) * kRankTiles + threadIdx.x;
    const int64_t u0 = static_cast<int64_t>(blockIdx.y) * slice;
    const int64_t u1 = min(n_tiles, u0 + slice);
    for (int64_t u = u0 + threadIdx.x; u < u1; u += kRankThreads) sl[u - u0] = loss[u];
    __syncthreads();
    double lt[kRankPerThread];
    int32_t cnt[kRankPerThread];
#pragma unroll
    for (int j = 0; j < kRankPerThread; ++j) {
        const int64_t t = tb + j * kRankThreads;
        lt[j] = t < n_tiles ? loss[t] : 0.0;
        cnt[j] = 0;
    }
    const int len = static_cast<int>(u1 - u0);
    const int64_t t_first = tb, t_last = tb + (kRankPerThread - 1) * kRankThreads;
    if (u1 <= t_first) {
        for (int i = 0; i < len; ++i) {
            const double lu = sl[i];
#pragma unroll
            for (int j = 0; j < kRankPerThread; ++j) cnt[j] += lu <= lt[j];
        }
    } else if (u0 > t_last) {
        for (int i = 0; i < len; ++i) {
            const double lu = sl[i];
#pragma unroll
            for (int j = 0; j < kRankPerThread; ++j) cnt[j] += lu < lt[j];
        }
    } else {
        for (int i = 0; i < len; ++i) {
            const double lu = sl[i];
            const int64_t u = u0 + i;
#pragma unroll
            for (int j = 0; j < kRankPerThread; ++j) {
                const int64_t t = tb + j * kRankThreads;
                cnt[j] += (lu < lt[j]) || (lu == lt[j] && u < t);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kRankPerThread; ++j) {
        const int64_t t = tb + j * kRankThreads;
        if (t < n_tiles) atomicAdd(rank + t, cnt[j]);
    }
    if (!map) return;  // the caller turns ranks into bitmaps itself
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        last = atomicAdd(done, 1u) == gridDim.x * gridDim.y - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    const int64_t words = (n_tiles + 31) / 32;
    for (int64_t wd = threadIdx.x; wd < words; wd += kRankThreads) {
        uint32_t bits = 0;
#pragma unroll
        for (int q = 0; q < 32; ++q) {
            const int64_t tt = wd * 32 + q;
            if (tt < n_tiles && __ldcg(rank + tt) < n_sparse) bits |= 1u << q;
        }
        map[wd] = bits;
    }
}

// Global tile allocation: bit t of matrix m's bitmap is set iff the tile's
// rank over all matrices (concatenated, matrix m starting at offset[m]) is
// below n_sparse.  One thread per output word.
struct GlobalMaps {
    uint32_t *map[kMaxGlobalMatrices];
    int64_t offset[kMaxGlobalMatrices + 1];  // first global tile of each matrix; [count] = total
    int64_t word0[kMaxGlobalMatrices + 1];   // first output word of each matrix (prefix)
    int count;
};

__global__ void __launch_bounds__(128)
split_maps_kernel(const int32_t *__restrict__ rank, int64_t n_sparse, const __grid_constant__ GlobalMaps g) {
    const int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (w >= g.word0[g.count]) return;
    int m = 0;
    while (m + 1 < g.count && g.word0[m + 1] <= w) ++m;
    const int64_t lw = w - g.word0[m];
    const int64_t n = g.offset[m + 1] - g.offset[m];
    uint32_t bits = 0;
    for (int q = 0; q < 32; ++q) {
        const int64_t t = lw * 32 + q;
        if (t < n && rank[g.offset[m] + t] < n_sparse) bits |= 1u << q;
    }
    g.map[m][lw] = bits;
}

cudaError_t launch_select_maps_global(const double *loss_cat, const int64_t *n_tiles, int count,
                                      int64_t n_sparse, int32_t *rank, uint32_t *const *maps,
                                      cudaStream_t stream) {
    if (count < 1 || count > kMaxGlobalMatrices) return cudaErrorInvalidValue;
    GlobalMaps g;
    g.count = count;
    g.offset[0] = 0;
    g.word0[0] = 0;
    for (int m = 0; m < count; ++m) {
        g.map[m] = maps[m];
        g.offset[m + 1] = g.offset[m] + n_tiles[m];
        g.word0[m + 1] = g.word0[m] + (n_tiles[m] + 31) / 32;
    }
    const int64_t total = g.offset[count];
    const int slice = rank_slice(total);
    dim3 grid(static_cast<unsigned>((total + kRankTiles - 1) / kRankTiles),
              static_cast<unsigned>((total + slice - 1) / slice));
    rank_tiles_kernel<<<grid, kRankThreads, 0, stream>>>(loss_cat, total, n_sparse, slice, rank, nullptr,
                                                         nullptr);
    split_maps_kernel<<<static_cast<unsigned>((g.word0[count] + 127) / 128), 128, 0, stream>>>(rank, n_sparse, g);
    note_launches(2);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ launch
cudaError_t launch_norms_from_colsq(const double *colsq_in, int64_t K, double *colsq_out,
                                    double *norm_out, cudaStream_t stream) {
    norms_from_colsq_kernel<<<static_cast<unsigned>((K + 255) / 256), 256, 0, stream>>>(
        colsq_in, K, colsq_out, norm_out);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_score_mask(const void *W, const double *norm, int64_t N, int64_t K, int tn,
                              int tk, uint32_t *meta, double *loss, int32_t *rank, uint32_t *done,
                              cudaStream_t stream, int pattern) {
    const int64_t n_tiles = (N / tn) * (K / tk);
    const uint16_t *w = static_cast<const uint16_t *>(W);
    const unsigned g = static_cast<unsigned>(n_tiles);
#define PATCH_SCORE_LAUNCH(TN, TK)                                                                  \
    if (tn == TN && tk == TK) {                                                                     \
        if (pattern == 4)                                                                           \
            score_mask_kernel<TN, TK, 4><<<g, TN *(TK / 32), 0, stream>>>(w, norm, N, K, meta, loss, \
                                                                        rank, done);               \
        else                                                                                        \
            score_mask_kernel<TN, TK, 2><<<g, TN *(TK / 32), 0, stream>>>(w, norm, N, K, meta, loss, \
                                                                        rank, done);               \
        note_launches(1);                                                                           \
        return cudaGetLastError();                                                                  \
    }
    if (pattern != 2 && pattern != 4) return cudaErrorInvalidValue;
    PATCH_SCORE_LAUNCH(128, 128)
    PATCH_SCORE_LAUNCH(128, 64)
    PATCH_SCORE_LAUNCH(64, 128)
    PATCH_SCORE_LAUNCH(64, 64)
#undef PATCH_SCORE_LAUNCH
    return cudaErrorInvalidValue;
}

cudaError_t launch_select_map(const double *loss, int64_t n_tiles, int64_t n_sparse, int32_t *rank,
                              uint32_t *done, uint32_t *map, cudaStream_t stream) {
    const int slice = rank_slice(n_tiles);
    dim3 grid(static_cast<unsigned>((n_tiles + kRankTiles - 1) / kRankTiles),
              static_cast<unsigned>((n_tiles + slice - 1) / slice));
    rank_tiles_kernel<<<grid, kRankThreads, 0, stream>>>(loss, n_tiles, n_sparse, slice, rank, done, map);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace patchk
