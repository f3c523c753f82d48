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

// Keep the entries of one 4:8 group (8 bf16 in a uint4) whose mask bits are set.
__device__ __forceinline__ uint4 mask_eight(uint4 v, uint32_t m) {
    uint32_t e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 8; ++q)
        if (!((m >> q) & 1u)) e[q / 2] &= (q & 1) ? 0x0000FFFFu : 0xFFFF0000u;
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
// swizzled output straight from global W (no shared-memory staging), its
// loads issued before its stores.  Where the prefill table points the k-step
// to a dense side copy (bands of a pair that differ in type), the same CTA
// also writes that copy: the k-step's W_eff in the dense layout.
__global__ void __launch_bounds__(kPackThreads, 8)
pack_kernel(const uint16_t *__restrict__ W, const uint32_t *__restrict__ meta,
            const uint32_t *__restrict__ map, int64_t N, int64_t K, int tn, int tk,
            const uint64_t *__restrict__ table, const uint64_t *__restrict__ ptable,
            uint8_t *__restrict__ out, int pattern) {
    const int64_t nsteps = K / kStep;
    const int64_t steps_all = (N / kBand) * nsteps;
    (void)steps_all;
    const int64_t idx = blockIdx.x;
    const int64_t b = idx / nsteps, c = idx % nsteps;
    const uint64_t entry = table[idx];
    const int64_t off = static_cast<int64_t>(entry & kEntryOffsetMask);
    // the dense side copy of this k-step, if the prefill table has one
    const uint64_t sentry = ptable ? ptable[idx] : 0ull;
    const bool side = (sentry & kEntrySide) != 0;
    const int64_t soff = static_cast<int64_t>(sentry & kEntryOffsetMask);
    const int tid = threadIdx.x;
    const int64_t row0 = b * kBand, col0 = c * kStep;
    const int64_t words_k = K / 32;

    if (entry & kEntryNM48) {
        // 4:8: thread = row; its 32 kept values (in column order, four per
        // group of 8) at r*64, its 8 keep masks at 8192 + r*8
        const int r = tid;
        const int64_t i = row0 + r;
        const uint4 *src = reinterpret_cast<const uint4 *>(W + i * K + col0);
        const uint32_t m0 = __ldg(meta + i * words_k + col0 / 32), m1 = __ldg(meta + i * words_k + col0 / 32 + 1);
        uint32_t vals[16];
        uint32_t masks[2] = {0u, 0u};
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const uint4 q4 = __ldg(src + g);
            const uint32_t e[4] = {q4.x, q4.y, q4.z, q4.w};
            const uint32_t m = ((g < 4 ? m0 : m1) >> (8 * (g % 4))) & 0xFFu;
            masks[g / 4] |= m << (8 * (g % 4));
            // exactly four kept per group: slots k[0..3] in column order
            uint32_t k[4] = {0u, 0u, 0u, 0u};
            int c = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t h = (q & 1) ? (e[q / 2] >> 16) : (e[q / 2] & 0xFFFFu);
                const bool keep = (m >> q) & 1u;
#pragma unroll
                for (int t = 0; t < 4; ++t) k[t] = (keep && c == t) ? h : k[t];
                c += keep ? 1 : 0;
            }
            vals[2 * g] = k[0] | (k[1] << 16);
            vals[2 * g + 1] = k[2] | (k[3] << 16);
        }
        uint4 *dst = reinterpret_cast<uint4 *>(out + off + r * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(vals[4 * q], vals[4 * q + 1], vals[4 * q + 2], vals[4 * q + 3]);
        *reinterpret_cast<uint2 *>(out + off + 8192 + r * 8) = make_uint2(masks[0], masks[1]);
    } else if (!(entry & kEntrySparse)) {
        // dense: chunk u = r*8 + ((k/8) ^ (r%8)); W_eff, i.e. pruned entries of
        // a 2:4 tile (64-row tiles sharing a band with a dense tile) are zeroed
        constexpr int kPer = kBand * 8 / kPackThreads;
        uint4 v[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int u = tid + q * kPackThreads;
            const int r = u / 8, k8 = (u % 8) ^ (r % 8);
            v[q] = __ldg(reinterpret_cast<const uint4 *>(W + (row0 + r) * K + col0 + 8 * k8));
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int u = tid + q * kPackThreads;
            const int r = u / 8, k8 = (u % 8) ^ (r % 8);
            const int64_t i = row0 + r, j = col0 + 8 * k8;
            const int64_t tile = (i / tn) * (K / tk) + j / tk;
            if ((__ldg(map + tile / 32) >> (tile % 32)) & 1u) {
                const uint32_t mw = __ldg(meta + i * words_k + j / 32);
                if (pattern == 4)
                    v[q] = mask_eight(v[q], (mw >> (8 * ((j % 32) / 8))) & 0xFFu);
                else
                    v[q] = mask_two_groups(v[q], mw >> (4 * ((j % 32) / 4)));
            }
            reinterpret_cast<uint4 *>(out + off)[u] = v[q];
            if (side) reinterpret_cast<uint4 *>(out + soff)[u] = v[q];
        }
    } else {
        // 2:4: chunk u = r*4 + ((v/8) ^ ((r%8)/2)) holds the kept values of groups
        // 4*(v/8) .. 4*(v/8)+3 of the row, two per group in column order
        constexpr int kPer = kBand * 4 / kPackThreads;
        uint4 a[kPer], bq[kPer];
        uint32_t mw[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int u = tid + q * kPackThreads;
            const int r = u / 4, v8 = (u % 4) ^ ((r % 8) / 2);
            const int64_t i = row0 + r, j = col0 + 16 * v8;
            const uint4 *src = reinterpret_cast<const uint4 *>(W + i * K + j);
            a[q] = __ldg(src);
            bq[q] = __ldg(src + 1);
            mw[q] = __ldg(meta + i * words_k + j / 32);
        }
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int u = tid + q * kPackThreads;
            const int r = u / 4, v8 = (u % 4) ^ ((r % 8) / 2);
            const int64_t j = col0 + 16 * v8;
            const uint32_t e[8] = {a[q].x, a[q].y, a[q].z, a[q].w, bq[q].x, bq[q].y, bq[q].z, bq[q].w};
            const uint32_t codes = mw[q] >> (4 * ((j % 32) / 4));
            uint32_t o[4];
#pragma unroll
            for (int g = 0; g < 4; ++g) o[g] = kept_pair(e[2 * g], e[2 * g + 1], (codes >> (4 * g)) & 0xFu);
            reinterpret_cast<uint4 *>(out + off)[u] = make_uint4(o[0], o[1], o[2], o[3]);
            if (side) {
                // the same 16 columns as W_eff in the dense layout: chunks
                // 2 v8 and 2 v8 + 1 of row r, at (k8 ^ (r % 8))
                uint4 *d = reinterpret_cast<uint4 *>(out + soff) + r * 8;
                d[(2 * v8) ^ (r % 8)] = mask_two_groups(a[q], codes);
                d[(2 * v8 + 1) ^ (r % 8)] = mask_two_groups(bq[q], codes >> 8);
            }
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
}

// The ready flags of up to kPlanMaxGroup handles, set (release) by one
// thread each once every kernel before this one on the stream has completed:
// the packed bytes are then final, and a GEMM that reads its flag as set may
// fetch weights before its griddepcontrol.wait.
struct ReadyList {
    uint32_t *ready[kPlanMaxGroup];
};
__global__ void publish_ready_list_kernel(const __grid_constant__ ReadyList list, int count) {
    if (static_cast<int>(threadIdx.x) < count) st_release_gpu(list.ready[threadIdx.x], 1u);
}

// ------------------------------------------------------------------- plan
// The layout of every band: per k-step its type (2:4 iff the one or two tiles
// covering its 128 rows are 2:4) and byte offset, a 2 KB metadata block
// before the first 2:4 k-step of each k-pair; bands follow one another.  A
// k-pair's size depends only on its two k-step types (32, 26 or 18 KB), so
// offsets are prefix sums.  One block of 32 warps: a warp takes a band at a
// time, gathers its k-step types into bit words in shared memory (one ballot
// per 32 k-steps), then sizes its k-pairs with a k-pair per lane; the block
// scans the band sizes; the warps write the entries and the decode chunk
// descriptors.  All index arithmetic is 32-bit with shifts (tile sides are
// powers of two).
constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kPlanMaxWords = 14;  // 448 k-steps (K <= 28672) / 32
// bands whose k-step types the planner keeps in shared memory after its first
// pass (the later passes then read them there instead of the map again)
constexpr int kPlanCacheBands = 512;

// Bit c % 32 of word c / 32 of `bits`: k-step c of band b is 2:4.
__device__ __forceinline__ void band_types(const uint32_t *__restrict__ map, int b, int nsteps,
                                           int log_tn, int log_tk, int tiles_k, int lane,
                                           uint32_t *bits) {
    const int rows_tiles = kBand >> log_tn;  // 1 or 2
    const int ti0 = (b * kBand) >> log_tn;
    for (int c0 = 0; c0 < nsteps; c0 += 32) {
        const int c = c0 + lane;
        bool sp = false;
        if (c < nsteps) {
            const int tj = (c * kStep) >> log_tk;
            int t = ti0 * tiles_k + tj;
            sp = (__ldg(map + (t >> 5)) >> (t & 31)) & 1u;
            if (rows_tiles == 2) {
                t += tiles_k;
                sp = sp && ((__ldg(map + (t >> 5)) >> (t & 31)) & 1u);
            }
        }
        const uint32_t w = __ballot_sync(0xFFFFFFFFu, sp);
        if (lane == 0) bits[c0 >> 5] = w;
    }
    __syncwarp();
}

__device__ __forceinline__ bool bit_of(const uint32_t *bits, int c) { return (bits[c >> 5] >> (c & 31)) & 1u; }

__device__ __forceinline__ uint32_t kpair_bytes(bool s0, bool s1, int pattern = 2) {
    if (pattern == 4)
        return (s0 ? kNM48StepBytes : kDenseStepBytes) + (s1 ? kNM48StepBytes : kDenseStepBytes);
    return (s0 ? kMetaBlockBytes + kSparseStepBytes : kDenseStepBytes) +
           (s1 ? (s0 ? 0 : kMetaBlockBytes) + kSparseStepBytes : kDenseStepBytes);
}

// The plans of up to kPlanMaxGroup matrices, one block each.
struct PlanGroup {
    const uint32_t *map[kPlanMaxGroup];
    int bands[kPlanMaxGroup], nsteps[kPlanMaxGroup], log_tn[kPlanMaxGroup], log_tk[kPlanMaxGroup];
    int cp[kPlanMaxGroup], cpb[kPlanMaxGroup];
    uint64_t *table[kPlanMaxGroup], *chunk_desc[kPlanMaxGroup];
    int64_t *pair_prefix[kPlanMaxGroup];
    uint64_t *band_start[kPlanMaxGroup], *ptable[kPlanMaxGroup], *side_start[kPlanMaxGroup];
    PackPlan *plan[kPlanMaxGroup];
    uint32_t *status[kPlanMaxGroup];  // the handle's 64 status words, zeroed here
    int pattern[kPlanMaxGroup];
};

__global__ void __launch_bounds__(kPlanThreads, 1) plan_pack_kernel(const __grid_constant__ PlanGroup grp) {
    // this block's matrix
    const int gi = blockIdx.x;
    const uint32_t *__restrict__ map = grp.map[gi];
    const int bands = grp.bands[gi], nsteps = grp.nsteps[gi], log_tn = grp.log_tn[gi], log_tk = grp.log_tk[gi];
    const int cp = grp.cp[gi], cpb = grp.cpb[gi], pattern = grp.pattern[gi];
    uint64_t *__restrict__ table = grp.table[gi];
    uint64_t *__restrict__ chunk_desc = grp.chunk_desc[gi];
    int64_t *__restrict__ pair_prefix = grp.pair_prefix[gi];
    uint64_t *__restrict__ band_start = grp.band_start[gi];
    uint64_t *__restrict__ ptable = grp.ptable[gi];
    uint64_t *__restrict__ side_start = grp.side_start[gi];
    PackPlan *__restrict__ plan = grp.plan[gi];
    if (grp.status[gi] && threadIdx.x < kStatusWords) grp.status[gi][threadIdx.x] = 0u;
    __shared__ unsigned long long warp_sum[kPlanWarps];
    __shared__ uint32_t types[kPlanWarps][2][kPlanMaxWords];
    __shared__ uint32_t tcache[kPlanCacheBands * kPlanMaxWords];
    __shared__ unsigned long long carry, n_sparse, n_meta, side_carry;
    __shared__ unsigned int duo_ok, max_pair, pmax_pair;
    const int tid = threadIdx.x, lane = tid % 32, wid = tid / 32;
    const int Q = nsteps / 2, tiles_k = (nsteps * kStep) >> log_tk;
    uint32_t *mine = types[wid][0], *next = types[wid][1];
    const bool cached = bands <= kPlanCacheBands;
    const int words = (nsteps + 31) / 32;
    // band b's k-step types: the cache after pass 1, else gathered into buf
    auto types_of = [&](int b, uint32_t *buf) -> const uint32_t * {
        if (cached) return tcache + b * kPlanMaxWords;
        band_types(map, b, nsteps, log_tn, log_tk, tiles_k, lane, buf);
        return buf;
    };
    if (tid == 0) {
        carry = 0;
        n_sparse = 0;
        n_meta = 0;
        duo_ok = (bands % 2 == 0 && pattern == 2) ? 1u : 0u;
        max_pair = 0;
        pmax_pair = 0;
        side_carry = 0;
    }
    __syncthreads();
    // pass 1: k-pair sizes and their prefix within each band
    {
        unsigned long long ns = 0, nm = 0;
        unsigned int mp = 0;
        for (int b = wid; b < bands; b += kPlanWarps) {
            band_types(map, b, nsteps, log_tn, log_tk, tiles_k, lane, mine);
            if (cached && lane < words) tcache[b * kPlanMaxWords + lane] = mine[lane];
            int64_t *pre = pair_prefix + static_cast<int64_t>(b) * (Q + 1);
            if (lane == 0) pre[0] = 0;
            unsigned long long run = 0;
            for (int q0 = 0; q0 < Q; q0 += 32) {
                const int q = q0 + lane;
                uint32_t bytes = 0;
                if (q < Q) {
                    const bool s0 = bit_of(mine, 2 * q), s1 = bit_of(mine, 2 * q + 1);
                    bytes = kpair_bytes(s0, s1, pattern);
                    ns += s0 + s1;
                    nm += (pattern == 2 && (s0 || s1)) ? 1 : 0;
                    mp = max(mp, bytes);
                }
                unsigned long long incl = bytes;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += v;
                }
                if (q < Q) pre[q + 1] = static_cast<int64_t>(run + incl);
                run += __shfl_sync(0xFFFFFFFFu, incl, 31);
            }
            __syncwarp();
        }
        // one shared-memory atomic per warp (1024 contending 64-bit atomics on
        // one address serialise for tens of microseconds)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ns += __shfl_xor_sync(0xFFFFFFFFu, ns, o);
            nm += __shfl_xor_sync(0xFFFFFFFFu, nm, o);
            mp = max(mp, __shfl_xor_sync(0xFFFFFFFFu, mp, o));
        }
        if (lane == 0) {
            atomicAdd(&n_sparse, ns);
            atomicAdd(&n_meta, nm);
            atomicMax(&max_pair, mp);
        }
    }
    __syncthreads();
    // pass 2: the first byte of every band (block-wide exclusive scan)
    for (int base = 0; base < bands; base += kPlanThreads) {
        const int b = base + tid;
        const unsigned long long bytes =
            b < bands ? static_cast<unsigned long long>(pair_prefix[static_cast<int64_t>(b) * (Q + 1) + Q]) : 0ull;
        unsigned long long incl = bytes;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_sum[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            unsigned long long w = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, w, o);
                if (lane >= o) w += v;
            }
            warp_sum[lane] = w;  // inclusive over warps
        }
        __syncthreads();
        if (b < bands) band_start[b] = carry + (wid > 0 ? warp_sum[wid - 1] : 0ull) + (incl - bytes);
        __syncthreads();
        if (tid == 0) carry += warp_sum[kPlanWarps - 1];
        __syncthreads();
    }
    // pass 3: k-step entries and decode chunk descriptors
    for (int b = wid; b < bands; b += kPlanWarps) {
        const uint32_t *tb = types_of(b, mine);
        const uint64_t start = band_start[b];
        const int64_t *pre = pair_prefix + static_cast<int64_t>(b) * (Q + 1);
        uint64_t *row = table + static_cast<int64_t>(b) * nsteps;
        for (int q = lane; q < Q; q += 32) {
            const bool s0 = bit_of(tb, 2 * q), s1 = bit_of(tb, 2 * q + 1);
            uint64_t off = start + static_cast<uint64_t>(pre[q]);
            uint64_t e0, e1;
            if (pattern == 4) {
                e0 = off | (s0 ? kEntryNM48 : 0ull);
                off += s0 ? kNM48StepBytes : kDenseStepBytes;
                row[2 * q] = e0;
                row[2 * q + 1] = off | (s1 ? kEntryNM48 : 0ull);
                continue;
            }
            if (s0) {
                off += kMetaBlockBytes;
                e0 = kEntrySparse | kEntryMeta | off;
                off += kSparseStepBytes;
            } else {
                e0 = off;
                off += kDenseStepBytes;
            }
            if (s1) {
                uint64_t m = 0;
                if (!s0) {
                    off += kMetaBlockBytes;
                    m = kEntryMeta;
                }
                e1 = kEntrySparse | m | off;
            } else {
                e1 = off;
            }
            row[2 * q] = e0;
            row[2 * q + 1] = e1;
        }
        for (int q = lane; q < cpb; q += 32) {
            const int pr0 = q * cp;
            const int np = min(cp, Q - pr0);
            uint64_t flags = 0;
            for (int i = 0; i < 2 * np; ++i)
                if (bit_of(tb, 2 * pr0 + i)) flags |= 1ull << i;
            const uint64_t first = start + static_cast<uint64_t>(pre[pr0]);
            chunk_desc[static_cast<int64_t>(b) * cpb + q] =
                (first & ((1ull << 40) - 1)) | (flags << 40) | (static_cast<uint64_t>(np) << 56);
        }
        __syncwarp();
    }
    __syncthreads();
    // pass 4: the prefill table.  The two-SM prefill kernel runs bands 2p and
    // 2p+1 through one M = 256 instruction, which must be of one kind.  Where
    // the pair's k-pair types differ, each band of it holding a 2:4 k-step
    // gets a dense copy of that k-pair (W_eff, 32 KB) in a side region after
    // the packed bytes; elsewhere the prefill table repeats the packed entry.
    // 4a: densified k-pairs per band (counted into side_start)
    for (int pb = wid; 2 * pb < bands; pb += kPlanWarps) {
        const int b = 2 * pb;
        const bool paired = b + 1 < bands && pattern == 2;
        const uint32_t *tb = types_of(b, mine);
        const uint32_t *tn1 = paired ? types_of(b + 1, next) : next;
        unsigned int n0 = 0, n1 = 0, mp = 0;
        for (int q0 = 0; q0 < Q; q0 += 32) {
            const int q = q0 + lane;
            bool d0 = false, d1 = false;
            if (q < Q) {
                const bool s0 = bit_of(tb, 2 * q), s1 = bit_of(tb, 2 * q + 1);
                const bool t0 = paired && bit_of(tn1, 2 * q), t1 = paired && bit_of(tn1, 2 * q + 1);
                const bool mis = paired && (s0 != t0 || s1 != t1);
                d0 = mis && (s0 || s1);
                d1 = mis && (t0 || t1);
                mp = max(mp, d0 || d1 ? static_cast<unsigned int>(kSidePairBytes)
                                      : max(kpair_bytes(s0, s1, pattern),
                                            paired ? kpair_bytes(t0, t1, pattern) : 0u));
            }
            n0 += __popc(__ballot_sync(0xFFFFFFFFu, d0));
            n1 += __popc(__ballot_sync(0xFFFFFFFFu, d1));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mp = max(mp, __shfl_xor_sync(0xFFFFFFFFu, mp, o));
        if (lane == 0) {
            // every band's count is written (a band without a partner, or of a
            // handle without a prefill table, densifies nothing)
            side_start[b] = n0;
            if (b + 1 < bands) side_start[b + 1] = paired ? n1 : 0u;
            atomicMax(&pmax_pair, mp);
        }
        __syncwarp();
    }
    __syncthreads();
    // 4b: side offsets, an exclusive scan of 32 KB per densified k-pair
    for (int base = 0; base < bands; base += kPlanThreads) {
        const int b = base + tid;
        const unsigned long long bytes = b < bands ? side_start[b] * static_cast<unsigned long long>(kSidePairBytes) : 0ull;
        unsigned long long incl = bytes;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) warp_sum[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            unsigned long long w = warp_sum[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, w, o);
                if (lane >= o) w += v;
            }
            warp_sum[lane] = w;
        }
        __syncthreads();
        if (b < bands) side_start[b] = carry + side_carry + (wid > 0 ? warp_sum[wid - 1] : 0ull) + (incl - bytes);
        __syncthreads();
        if (tid == 0) side_carry += warp_sum[kPlanWarps - 1];
        __syncthreads();
    }
    // 4c: the entries; densified k-pairs are numbered in order within a band
    for (int b = wid; b < bands; b += kPlanWarps) {
        const int partner = b ^ 1;
        const bool paired = partner < bands && pattern == 2;
        const uint32_t *tb = types_of(b, mine);
        const uint32_t *tp = paired ? types_of(partner, next) : next;
        const uint64_t *row = table + static_cast<int64_t>(b) * nsteps;
        uint64_t *prow = ptable + static_cast<int64_t>(b) * nsteps;
        unsigned int run = 0;
        for (int q0 = 0; q0 < Q; q0 += 32) {
            const int q = q0 + lane;
            bool d = false;
            if (q < Q) {
                const bool s0 = bit_of(tb, 2 * q), s1 = bit_of(tb, 2 * q + 1);
                const bool t0 = paired && bit_of(tp, 2 * q), t1 = paired && bit_of(tp, 2 * q + 1);
                d = paired && (s0 != t0 || s1 != t1) && (s0 || s1);
            }
            const uint32_t ball = __ballot_sync(0xFFFFFFFFu, d);
            if (q < Q) {
                if (d) {
                    const unsigned int k = run + __popc(ball & ((1u << lane) - 1u));
                    const uint64_t off = side_start[b] + static_cast<uint64_t>(k) * kSidePairBytes;
                    prow[2 * q] = kEntrySide | off;
                    prow[2 * q + 1] = kEntrySide | (off + kDenseStepBytes);
                } else {
                    prow[2 * q] = row[2 * q];
                    prow[2 * q + 1] = row[2 * q + 1];
                }
            }
            run += __popc(ball);
        }
        __syncwarp();
    }
    __syncthreads();
    // the first chunk descriptors, written above by other warps of the block
    const int64_t nchunks = static_cast<int64_t>(bands) * cpb;
    for (int64_t j = tid; j < 2 * kDecMaxCtas; j += kPlanThreads)
        plan->first_desc[j] = j < nchunks ? chunk_desc[j] : 0ull;
    if (tid == 0) {
        plan->packed_bytes = carry;
        plan->sparse_ksteps = n_sparse;
        plan->meta_blocks = n_meta;
        plan->duo_ok = duo_ok;
        plan->max_pair_bytes = max_pair;
        plan->side_bytes = side_carry;
        plan->pair_max_bytes = pmax_pair;
    }
}

cudaError_t launch_plan_pack_group(const PlanArgs *args, int count, cudaStream_t stream) {
    if (count < 1 || count > kPlanMaxGroup) return cudaErrorInvalidValue;
    PlanGroup grp{};
    for (int i = 0; i < count; ++i) {
        const PlanArgs &a = args[i];
        const int64_t nsteps = a.K / kStep;
        if (nsteps > 32 * kPlanMaxWords || (a.N / kBand) > (int64_t(1) << 24)) return cudaErrorInvalidValue;
        if (a.pattern != 2 && a.pattern != 4) return cudaErrorInvalidValue;
        grp.map[i] = a.map;
        grp.bands[i] = static_cast<int>(a.N / kBand);
        grp.nsteps[i] = static_cast<int>(nsteps);
        grp.log_tn[i] = a.tn == 64 ? 6 : 7;
        grp.log_tk[i] = a.tk == 64 ? 6 : 7;
        grp.cp[i] = a.cp;
        grp.cpb[i] = a.cpb;
        grp.table[i] = a.table;
        grp.chunk_desc[i] = a.chunk_desc;
        grp.pair_prefix[i] = a.pair_prefix;
        grp.band_start[i] = a.band_start;
        grp.ptable[i] = a.ptable;
        grp.side_start[i] = a.side_start;
        grp.plan[i] = a.plan;
        grp.status[i] = a.status;
        grp.pattern[i] = a.pattern;
    }
    plan_pack_kernel<<<count, kPlanThreads, 0, stream>>>(grp);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_pack(const void *W, const uint32_t *meta, const uint32_t *map, int64_t N,
                        int64_t K, int tn, int tk, const uint64_t *table, const uint64_t *ptable,
                        uint8_t *out, cudaStream_t stream, int pattern) {
    const int64_t blocks = (N / kBand) * (K / kStep);
    if (blocks > 0x7FFFFFFF || (pattern != 2 && pattern != 4)) return cudaErrorInvalidValue;
    pack_kernel<<<static_cast<unsigned>(blocks), kPackThreads, 0, stream>>>(
        static_cast<const uint16_t *>(W), meta, map, N, K, tn, tk, table, ptable, out, pattern);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_publish_ready(uint32_t *const *ready, int count, cudaStream_t stream) {
    if (count < 1 || count > kPlanMaxGroup) return cudaErrorInvalidValue;
    ReadyList list{};
    for (int i = 0; i < count; ++i) list.ready[i] = ready[i];
    publish_ready_list_kernel<<<1, 32, 0, stream>>>(list, count);
    note_launches(1);
    return cudaGetLastError();
}

void preload_pack_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, pack_kernel);
    (void)cudaFuncGetAttributes(&a, publish_ready_list_kernel);
}

}  // namespace patchk
