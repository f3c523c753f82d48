// FP8 (e4m3) values inside dense and 2:4 tiles: quantisation and packing (sm_100a).
//
// Prune first, then quantise ("SparseGPT vs Wanda: one-shot LLM pruning
// without retraining", FAQ on combining pruning with quantisation): the Wanda
// 2:4 codes and the tile map are decided on the bf16 weights as for the
// 16-bit handles; W_eff is then quantised to e4m3 with one fp32 scale per
// output row, and the activations with one fp32 scale per token:
//     s = amax / 448 (1 for an all-zero row),  q = e4m3(x / s)
// with the quotient in fp32 (round to nearest) and the conversion rounding to
// nearest even, saturating at 448 (cvt.rn.satfinite through cuda_fp8.h).
//
// Packed layout (normative statement in include/patch.h): bands of 128 rows,
// k-steps of 128 columns (128 bytes of codes per row); a dense k-step is
// 16 KB in the K-major 128-byte-swizzled layout, a 2:4 k-step a 2 KB
// metadata block (line m = row m's 128 code bits, the tensor-memory layout of
// the 8-bit sparse MMA) followed by 8 KB of kept codes, K-major 64-byte
// swizzled.
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "patch_common.cuh"
#include "patch_internal.h"

namespace patchk {

namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__device__ __forceinline__ uint32_t e4m3(float x, float s) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(__fdiv_rn(x, s), __NV_SATFINITE, __NV_E4M3));
}

// Four e4m3 codes of bf16 values a[0..3] (packed two per word) in one word.
__device__ __forceinline__ uint32_t e4m3x4(uint32_t w01, uint32_t w23, float s) {
    return e4m3(bf16_to_f32(w01 & 0xFFFFu), s) | (e4m3(bf16_to_f32(w01 >> 16), s) << 8) |
           (e4m3(bf16_to_f32(w23 & 0xFFFFu), s) << 16) | (e4m3(bf16_to_f32(w23 >> 16), s) << 24);
}

__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < static_cast<int>(blockDim.x / 32) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    return red[0];
}

// One block per row of a bf16 matrix [R, C] (C a multiple of 8): scale and codes.
// Launched as a programmatic dependent: it lets the next kernel (the FP8 GEMM)
// start its prologue at once, and touches memory only after the kernel
// before it has completed.
__global__ void __launch_bounds__(kQuantThreads)
fp8_quantize_rows_kernel(const uint16_t *__restrict__ x, int64_t C, uint8_t *__restrict__ q,
                         float *__restrict__ scale) {
    __shared__ float red[kQuantThreads / 32];
    if (threadIdx.x == 0) pdl_trigger();
    pdl_wait();
    const int64_t r = blockIdx.x;
    const uint4 *row = reinterpret_cast<const uint4 *>(x + r * C);
    const int64_t chunks = C / 8;
    float amax = 0.0f;
    for (int64_t i = threadIdx.x; i < chunks; i += kQuantThreads) {
        const uint4 v = __ldg(row + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_to_f32(w[h] & 0xFFFFu)), fabsf(bf16_to_f32(w[h] >> 16))));
    }
    amax = block_max(amax, red);
    const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (threadIdx.x == 0) scale[r] = s;
    uint2 *out = reinterpret_cast<uint2 *>(q + r * C);
    for (int64_t i = threadIdx.x; i < chunks; i += kQuantThreads) {
        const uint4 v = __ldg(row + i);
        out[i] = make_uint2(e4m3x4(v.x, v.y, s), e4m3x4(v.z, v.w, s));
    }
}

// Keep the entries of 8 bf16 values (two 2:4 groups, codes in `codes8`).
__device__ __forceinline__ uint4 keep_two_groups(uint4 v, uint32_t codes8) {
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

__device__ __forceinline__ bool tile_sparse(const uint32_t *map, int64_t i, int64_t j, int tn, int tk,
                                            int64_t K) {
    const int64_t t = (i / tn) * (K / tk) + j / tk;
    return (__ldg(map + t / 32) >> (t % 32)) & 1u;
}

// One block per row of W: the row's W_eff scale (amax of the kept and dense entries / 448).
__global__ void __launch_bounds__(kQuantThreads)
fp8_weff_scales_kernel(const uint16_t *__restrict__ W, const uint32_t *__restrict__ meta,
                       const uint32_t *__restrict__ map, int64_t K, int tn, int tk,
                       float *__restrict__ scale) {
    __shared__ float red[kQuantThreads / 32];
    const int64_t i = blockIdx.x;
    const uint4 *row = reinterpret_cast<const uint4 *>(W + i * K);
    float amax = 0.0f;
    for (int64_t u = threadIdx.x; u < K / 8; u += kQuantThreads) {
        const int64_t j = u * 8;
        uint4 v = __ldg(row + u);
        if (tile_sparse(map, i, j, tn, tk, K))
            v = keep_two_groups(v, __ldg(meta + i * (K / 32) + j / 32) >> (4 * ((j % 32) / 4)));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int h = 0; h < 4; ++h)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_to_f32(w[h] & 0xFFFFu)), fabsf(bf16_to_f32(w[h] >> 16))));
    }
    amax = block_max(amax, red);
    if (threadIdx.x == 0) scale[i] = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

// One block per (band, 128-column k-step), 128 threads; with a prefill
// table, a second set of blocks writes the dense side copies it names.
__global__ void __launch_bounds__(128)
pack_fp8_kernel(const uint16_t *__restrict__ W, const uint32_t *__restrict__ meta,
                const uint32_t *__restrict__ map, int64_t K, int tn, int tk,
                const float *__restrict__ scale, const uint64_t *__restrict__ table,
                const uint64_t *__restrict__ ptable, int64_t units, uint8_t *__restrict__ out) {
    const int64_t steps = K / 128;
    const bool side = blockIdx.x >= units;
    const int64_t unit = side ? blockIdx.x - units : blockIdx.x;
    const int64_t b = unit / steps, c = unit % steps;
    uint64_t entry = table[unit];
    if (side) {
        entry = ptable[unit];
        if (!(entry & kEntrySide)) return;
        entry &= kEntryOffsetMask;  // a dense k-step at the side offset
    }
    uint8_t *dst = out + (entry & kEntryOffsetMask);
    const int64_t row0 = b * kBand, col0 = c * 128, words_k = K / 32;
    const int tid = threadIdx.x;
    if (!(entry & kEntrySparse)) {
        // chunk u: row r, physical 16-byte chunk p holds logical columns 16 * (p ^ (r % 8))
        for (int u = tid; u < kBand * 8; u += 128) {
            const int r = u / 8, kc = (u % 8) ^ (r % 8);
            const int64_t i = row0 + r, j = col0 + 16 * kc;
            const uint4 *src = reinterpret_cast<const uint4 *>(W + i * K + j);
            uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
            if (tile_sparse(map, i, j, tn, tk, K)) {
                const uint32_t mw = __ldg(meta + i * words_k + j / 32) >> (4 * ((j % 32) / 4));
                v0 = keep_two_groups(v0, mw & 0xFFu);
                v1 = keep_two_groups(v1, (mw >> 8) & 0xFFu);
            }
            const float s = __ldg(scale + i);
            reinterpret_cast<uint4 *>(dst)[u] =
                make_uint4(e4m3x4(v0.x, v0.y, s), e4m3x4(v0.z, v0.w, s), e4m3x4(v1.x, v1.y, s),
                           e4m3x4(v1.z, v1.w, s));
        }
        return;
    }
    // metadata block (2 KB before the codes): line m = row m's four meta words
    {
        const int m = tid;
        const uint4 mw = *reinterpret_cast<const uint4 *>(meta + (row0 + m) * words_k + col0 / 32);
        reinterpret_cast<uint4 *>(dst - kMetaBlockBytes)[m] = mw;
    }
    // kept codes: chunk u = row r, physical chunk p (of 4) holds kept codes
    // 16 * (p ^ ((r % 8) / 2)) .. +15, i.e. groups of columns 32 * that .. +31
    for (int u = tid; u < kBand * 4; u += 128) {
        const int r = u / 4, vc = (u % 4) ^ ((r % 8) / 2);
        const int64_t i = row0 + r, j = col0 + 32 * vc;
        const uint4 *src = reinterpret_cast<const uint4 *>(W + i * K + j);
        const uint32_t codes = __ldg(meta + i * words_k + j / 32);
        const float s = __ldg(scale + i);
        uint32_t outw[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // 8 columns (two groups) -> 4 kept codes
            const uint4 v = __ldg(src + h);
            const uint32_t e[4] = {v.x, v.y, v.z, v.w};
            uint32_t word = 0;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const uint32_t code = (codes >> (4 * (2 * h + g))) & 0xFu;
                const uint32_t lo = code & 3u, hi = code >> 2;
                const uint32_t a = e[2 * g], bb = e[2 * g + 1];
                const uint32_t x0 = lo == 0 ? (a & 0xFFFFu) : (lo == 1 ? (a >> 16) : (bb & 0xFFFFu));
                const uint32_t x1 = hi == 3 ? (bb >> 16) : (hi == 2 ? (bb & 0xFFFFu) : (a >> 16));
                word |= (e4m3(bf16_to_f32(x0), s) | (e4m3(bf16_to_f32(x1), s) << 8)) << (16 * g);
            }
            outw[h] = word;
        }
        reinterpret_cast<uint4 *>(dst)[u] = make_uint4(outw[0], outw[1], outw[2], outw[3]);
    }
}

}  // namespace

__global__ void publish_ready_kernel(uint32_t *ready) { st_release_gpu(ready, 1u); }

void preload_fp8_quantize_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, fp8_quantize_rows_kernel);
    (void)cudaFuncGetAttributes(&a, publish_ready_kernel);
}

cudaError_t launch_fp8_quantize_rows(const void *x, int64_t R, int64_t C, uint8_t *q, float *scale,
                                     cudaStream_t stream) {
    if (R < 1 || C < 8 || C % 8 != 0 || R > 0x7FFFFFFF) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(R));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, fp8_quantize_rows_kernel, static_cast<const uint16_t *>(x), C,
                                             q, scale);
    if (e == cudaSuccess) note_launches(1);
    return e;
}

cudaError_t launch_pack_fp8(const void *W, const uint32_t *meta, const uint32_t *map, int64_t N,
                            int64_t K, int tn, int tk, const uint64_t *table, const uint64_t *ptable,
                            float *scale, uint8_t *out, uint32_t *ready, cudaStream_t stream) {
    if (N % kBand != 0 || K % 128 != 0 || N > 0x7FFFFFFF) return cudaErrorInvalidValue;
    fp8_weff_scales_kernel<<<static_cast<unsigned>(N), kQuantThreads, 0, stream>>>(
        static_cast<const uint16_t *>(W), meta, map, K, tn, tk, scale);
    const int64_t units = (N / kBand) * (K / 128);
    pack_fp8_kernel<<<static_cast<unsigned>(ptable ? 2 * units : units), 128, 0, stream>>>(
        static_cast<const uint16_t *>(W), meta, map, K, tn, tk, scale, table, ptable, units, out);
    note_launches(2);
    // the packed codes and scales are final once the kernels above have
    // completed (stream order): the split-K GEMM may then fetch them ahead of
    // its griddepcontrol.wait
    if (ready) {
        publish_ready_kernel<<<1, 1, 0, stream>>>(ready);
        note_launches(1);
    }
    return cudaGetLastError();
}

}  // namespace patchk
