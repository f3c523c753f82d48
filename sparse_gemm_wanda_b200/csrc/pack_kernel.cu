// Compressor: lays each (band, k-step) of W_eff out for the hybrid GEMM.
//
// Compressed storage is what turns zeroed weights into speed ("SparseGPT vs
// Wanda: one-shot LLM pruning without retraining", section on structured vs
// unstructured sparsity); dense and 2:4 tiles side by side are the PATCH
// format ("PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section 2).
// The byte layout is this library's own (stated normatively in patch.h):
//   dense k-step  128 x 64 bf16, K-major, 128-byte swizzle   (16384 B)
//   2:4 k-step    128 x 32 kept bf16, K-major, 64-byte swizzle (8192 B)
//   metadata      128 lines x 16 B per k-pair, the sparse-MMA TMEM layout
// so the GEMM moves each piece with one bulk copy and no reshuffling.
#include <cuda_runtime.h>
#include <stdint.h>

#include "patch_common.cuh"
#include "patch_internal.h"

namespace patchk {

constexpr int kPackThreads = 128;

// One CTA per (band, k-step).  The 128 x 64 block of W is staged in shared
// memory with coalesced loads, thread r rewrites row r, and the result leaves
// through coalesced 16-byte stores in the swizzled order.
__global__ void __launch_bounds__(kPackThreads)
pack_kernel(const uint16_t *__restrict__ W, const uint32_t *__restrict__ meta,
            const uint32_t *__restrict__ map, int64_t N, int64_t K, int tn, int tk,
            const uint64_t *__restrict__ table, uint8_t *__restrict__ out) {
    constexpr int kRow = kStep + 8;  // padded smem row (bf16)
    __shared__ __align__(16) uint16_t ws[kBand * kRow];
    __shared__ __align__(16) uint16_t cs[kBand * 40];  // compressed rows (32 used)
    __shared__ uint32_t ms[kBand * 2];

    const int64_t nsteps = K / kStep;
    const int64_t b = blockIdx.x / nsteps, c = blockIdx.x % nsteps;
    const uint64_t entry = table[blockIdx.x];
    const int64_t off = static_cast<int64_t>(entry & kEntryOffsetMask);
    const bool sparse = (entry & kEntrySparse) != 0;
    const int tid = threadIdx.x;
    const int64_t row0 = b * kBand, col0 = c * kStep;
    const int64_t words_k = K / 32;

    for (int u = tid; u < kBand * 8; u += kPackThreads) {
        const int r = u / 8, q = u % 8;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(W + (row0 + r) * K + col0) + q);
        *reinterpret_cast<uint4 *>(ws + r * kRow + q * 8) = v;
    }
    for (int u = tid; u < kBand * 2; u += kPackThreads) {
        const int r = u / 2, q = u % 2;
        ms[u] = __ldg(meta + (row0 + r) * words_k + col0 / 32 + q);
    }
    __syncthreads();

    {
        const int r = tid;
        uint16_t *row = ws + r * kRow;
        const uint32_t m0 = ms[2 * r], m1 = ms[2 * r + 1];
        if (!sparse) {
            // Dense storage: W_eff, i.e. W with pruned entries of 2:4 tiles at +0
            // (a k-step falls in exactly one tile column since tk >= 64).
            const int64_t tile = ((row0 + r) / tn) * (K / tk) + col0 / tk;
            if ((__ldg(map + tile / 32) >> (tile % 32)) & 1u) {
                for (int g = 0; g < 16; ++g) {
                    const uint32_t code = ((g < 8 ? m0 : m1) >> (4 * (g % 8))) & 0xFu;
                    for (int q = 0; q < 4; ++q)
                        if (q != static_cast<int>(code & 3u) && q != static_cast<int>(code >> 2))
                            row[4 * g + q] = 0;
                }
            }
        } else {
            uint16_t *crow = cs + r * 40;
            for (int g = 0; g < 16; ++g) {
                const uint32_t code = ((g < 8 ? m0 : m1) >> (4 * (g % 8))) & 0xFu;
                crow[2 * g] = row[4 * g + (code & 3u)];
                crow[2 * g + 1] = row[4 * g + (code >> 2)];
            }
        }
    }
    __syncthreads();

    if (!sparse) {
        // output 16-B chunk u = r*8 + ((k/8) ^ (r%8))
        for (int u = tid; u < kBand * 8; u += kPackThreads) {
            const int r = u / 8, cc = u % 8, src = cc ^ (r % 8);
            const uint4 v = *reinterpret_cast<const uint4 *>(ws + r * kRow + src * 8);
            reinterpret_cast<uint4 *>(out + off)[u] = v;
        }
        return;
    }
    // output 16-B chunk u = r*4 + ((v/8) ^ ((r%8)/2))
    for (int u = tid; u < kBand * 4; u += kPackThreads) {
        const int r = u / 4, cc = u % 4, src = cc ^ ((r % 8) / 2);
        const uint4 v = *reinterpret_cast<const uint4 *>(cs + r * 40 + src * 8);
        reinterpret_cast<uint4 *>(out + off)[u] = v;
    }
    if (entry & kEntryMeta) {
        // The metadata block of k-pair p: line l = m0 + 8*k1 + 16*m2 holds, in
        // 32-bit word k2, the 16 code bits of rows (m0 + 16*m2) [low half] and
        // (m0 + 8 + 16*m2) [high half] for pair columns 32*k2 + 16*k1 + [0,16).
        const int64_t p = c / 2;
        const int l = tid;
        const int m0i = l % 8, k1 = (l / 8) % 2, m2 = l / 16;
        const int64_t ra = row0 + m0i + 16 * m2, rb = ra + 8;
        uint32_t wv[4];
        for (int k2 = 0; k2 < 4; ++k2) {
            const int64_t ks = 2 * p + k2 / 2;
            const bool sp = (table[b * nsteps + ks] & kEntrySparse) != 0;
            const uint32_t lo = (__ldg(meta + ra * words_k + 4 * p + k2) >> (16 * k1)) & 0xFFFFu;
            const uint32_t hi = (__ldg(meta + rb * words_k + 4 * p + k2) >> (16 * k1)) & 0xFFFFu;
            wv[k2] = sp ? (lo | (hi << 16)) : 0u;
        }
        reinterpret_cast<uint4 *>(out + off - kMetaBlockBytes)[l] =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
    }
}

cudaError_t launch_pack(const void *W, const uint32_t *meta, const uint32_t *map, int64_t N,
                        int64_t K, int tn, int tk, const uint64_t *table, uint8_t *out,
                        cudaStream_t stream) {
    const int64_t blocks = (N / kBand) * (K / kStep);
    pack_kernel<<<static_cast<unsigned>(blocks), kPackThreads, 0, stream>>>(
        static_cast<const uint16_t *>(W), meta, map, N, K, tn, tk, table, out);
    return cudaGetLastError();
}

}  // namespace patchk
