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

// Keep the two entries of each group that its 4-bit code names, zero the
// others, for 8 consecutive bf16 values (two groups) held in a uint4.
__device__ __forceinline__ uint4 mask_two_groups(uint4 v, uint32_t codes8) {
    uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int g = 0; g < 2; ++g) {
        const uint32_t code = (codes8 >> (4 * g)) & 0xFu;
        const uint32_t lo = code & 3u, hi = code >> 2;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (q == static_cast<int>(lo) || q == static_cast<int>(hi)) continue;
            e[2 * g + q / 2] &= (q & 1) ? 0x0000FFFFu : 0xFFFF0000u;
        }
    }
    return make_uint4(e[0], e[1], e[2], e[3]);
}

// The two kept values of one group (4 bf16 in the 32-bit words a, b) as one
// 32-bit word, lower position first.
__device__ __forceinline__ uint32_t kept_pair(uint32_t a, uint32_t b, uint32_t code) {
    const uint32_t w0 = a & 0xFFFFu, w1 = a >> 16, w2 = b & 0xFFFFu, w3 = b >> 16;
    const uint32_t lo = code & 3u, hi = code >> 2;  // lo in {0,1,2}, hi in {1,2,3}
    const uint32_t x0 = lo == 0 ? w0 : (lo == 1 ? w1 : w2);
    const uint32_t x1 = hi == 3 ? w3 : (hi == 2 ? w2 : w1);
    return x0 | (x1 << 16);
}

// One CTA per (band, k-step); every thread writes whole 16-byte chunks of the
// swizzled output straight from global W (no shared-memory staging).
__global__ void __launch_bounds__(kPackThreads)
pack_kernel(const uint16_t *__restrict__ W, const uint32_t *__restrict__ meta,
            const uint32_t *__restrict__ map, int64_t N, int64_t K, int tn, int tk,
            const uint64_t *__restrict__ table, uint8_t *__restrict__ out,
            uint32_t *__restrict__ done, uint32_t *__restrict__ ready) {
    const int64_t nsteps = K / kStep;
    const int64_t b = blockIdx.x / nsteps, c = blockIdx.x % nsteps;
    const uint64_t entry = table[blockIdx.x];
    const int64_t off = static_cast<int64_t>(entry & kEntryOffsetMask);
    const int tid = threadIdx.x;
    const int64_t row0 = b * kBand, col0 = c * kStep;
    const int64_t words_k = K / 32;

    if (!(entry & kEntrySparse)) {
        // dense: chunk u = r*8 + ((k/8) ^ (r%8)); W_eff, i.e. pruned entries of
        // a 2:4 tile (64-row tiles sharing a band with a dense tile) are zeroed
#pragma unroll 4
        for (int u = tid; u < kBand * 8; u += kPackThreads) {
            const int r = u / 8, k8 = (u % 8) ^ (r % 8);
            const int64_t i = row0 + r, j = col0 + 8 * k8;
            uint4 v = __ldg(reinterpret_cast<const uint4 *>(W + i * K + j));
            const int64_t tile = (i / tn) * (K / tk) + j / tk;
            if ((__ldg(map + tile / 32) >> (tile % 32)) & 1u) {
                const uint32_t mw = __ldg(meta + i * words_k + j / 32);
                v = mask_two_groups(v, mw >> (4 * ((j % 32) / 4)));
            }
            reinterpret_cast<uint4 *>(out + off)[u] = v;
        }
    } else {
        // 2:4: chunk u = r*4 + ((v/8) ^ ((r%8)/2)) holds the kept values of groups
        // 4*(v/8) .. 4*(v/8)+3 of the row, two per group in column order
#pragma unroll 4
        for (int u = tid; u < kBand * 4; u += kPackThreads) {
            const int r = u / 4, v8 = (u % 4) ^ ((r % 8) / 2);
            const int64_t i = row0 + r, j = col0 + 16 * v8;
            const uint4 *src = reinterpret_cast<const uint4 *>(W + i * K + j);
            const uint4 a = __ldg(src), bq = __ldg(src + 1);
            const uint32_t e[8] = {a.x, a.y, a.z, a.w, bq.x, bq.y, bq.z, bq.w};
            const uint32_t codes = __ldg(meta + i * words_k + j / 32) >> (4 * ((j % 32) / 4));
            uint32_t o[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) o[g] = kept_pair(e[2 * g], e[2 * g + 1], (codes >> (4 * g)) & 0xFu);
            reinterpret_cast<uint4 *>(out + off)[u] = make_uint4(o[0], o[1], o[2], o[3]);
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
#pragma unroll
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
    // completion: every thread's stores are ordered before the block's ticket;
    // the last block publishes the ready flag the GEMM reads before its
    // griddepcontrol.wait
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t v = atomicAdd(done, 1u);
        if (v == gridDim.x - 1) {
            __threadfence();
            st_release_gpu(ready, 1u);
        }
    }
}

cudaError_t launch_pack(const void *W, const uint32_t *meta, const uint32_t *map, int64_t N,
                        int64_t K, int tn, int tk, const uint64_t *table, uint8_t *out,
                        uint32_t *done, uint32_t *ready, cudaStream_t stream) {
    const int64_t blocks = (N / kBand) * (K / kStep);
    pack_kernel<<<static_cast<unsigned>(blocks), kPackThreads, 0, stream>>>(
        static_cast<const uint16_t *>(W), meta, map, N, K, tn, tk, table, out, done, ready);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace patchk
