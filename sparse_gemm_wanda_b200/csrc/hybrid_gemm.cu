// Hybrid dense / 2:4 GEMM on the sm_100a tensor cores: Y = X * W_eff^T.
//
// "PATCH: Learnable Tile-level Hybrid Sparsity for LLMs", section 2
// (inference and deployment): dense tiles run on the dense tensor-core path,
// 2:4 tiles on the sparse one, inside one kernel over the mixed tiles.  The
// page's kernels came from a Triton autotuner on Ampere-class GPUs; this is a
// hand-written Blackwell design.
//
// Work.  An output tile is one 128-row band of W x BN tokens; D^T[128 x BN]
// accumulates in tensor memory (fp32).  CTAs are persistent.  Two schedules:
//   * whole tiles: tile c, c + P, c + 2P, ... (many tiles per CTA);
//   * stream-K: the (tile, k-pair) units are cut into P contiguous ranges of
//     (nearly) equal bytes, one per CTA.  A tile covered by several CTAs leaves fp32
//     partials; a fix-up kernel, launched as a programmatic dependent, adds
//     them in CTA order and stores Y, so the result does not depend on timing.
//     No CTA ever waits for another.
//
// Launch.  The kernel is launched as a programmatic dependent of the previous
// kernel of the stream and lets its own successor be scheduled at once.
// Before `griddepcontrol.wait` it touches only what no earlier kernel can be
// writing: once the packer has published the handle's ready flag (release /
// acquire at device scope), the k-step table and the first STAGES pairs of
// packed weights are fetched ahead of the wait, so the weight stream of one
// GEMM overlaps the tail of the kernel before it.  X, Y and the partials are
// touched only after the wait.
//
// Roles (192 threads):
//   * warp 0, one thread: producer.  Per 64-column k-step it reads the table
//     entry and moves the packed weights with ONE bulk copy (16 KB dense, or
//     8 KB kept values, plus the 2 KB metadata block where a pair starts) and
//     the activations X with one TMA tensor load (128-byte swizzle), all
//     completing on the stage's mbarrier.
//   * warp 1, one thread: MMA issuer.  Dense k-step: 4 x tcgen05.mma kind::f16
//     (M128 N=BN K16).  2:4 k-step: tcgen05.cp of the metadata block into 4
//     TMEM columns when the pair starts, then 2 x tcgen05.mma.sp (M128 N=BN
//     K32).  Both accumulate into the same accumulator; two accumulators
//     alternate between consecutive tiles so the epilogue of one overlaps the
//     main loop of the next.
//   * warps 2..5: epilogue.  tcgen05.ld (each warp its 32-lane quarter), one
//     rounding to bf16 (or fp32 out), stores to Y, or partials.
//   * 4:8 handles only (NM = true, 448 threads): warps 6..13, converters.  The
//     tensor core has no 4:8 sparse mode for 16-bit inputs, so a 4:8 k-step
//     (kept values + 8-bit keep masks, 9 KB) lands in its stage's 16 KB region
//     and the converters rewrite it in place as the dense 128-byte-swizzled
//     tile: two threads per row, each reads its 4 groups' 16 values and 4
//     masks, all eight warps meet on an mbarrier (reads before writes), then
//     each writes its 4 chunks of 16 B, built with two byte permutes per
//     32-bit word from a 256-entry table (selectors and zero masks per keep
//     mask) in shared memory; a fence to the async proxy, and the stage goes
//     to the MMA thread, which issues dense MMAs.
//
// Every mbarrier wait is bounded by %globaltimer; when one runs out the CTA
// raises the status word, drains its copies in flight and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "patch_common.cuh"
#include "patch_internal.h"

namespace patchk {

constexpr int kGemmThreads = 192;
constexpr int kGemmThreadsNM = 448;  // + 8 converter warps for 4:8 handles
constexpr int kConvWarps = 8;
constexpr int kLutBytes = 256 * 32;  // per keep mask: 4 byte-permute selectors, 4 zero masks
// k-steps of one segment whose table entries are staged in shared memory
// (K <= 28672)
constexpr int kMaxTableSteps = 448;
// stream-K CTAs whose unit boundaries travel in the kernel parameters
constexpr int kMaxStreamKCtas = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

template <int BN, int STAGES>
struct GemmCfg {
    // One stage = one k-pair (128 columns): the pair's packed weights (at most
    // two dense k-steps, 32 KB; the metadata block travels inside) and the two
    // 64-column X tiles.
    static constexpr int kABytes = 2 * kDenseStepBytes;
    static constexpr int kBTileBytes = BN * kStep * 2;  // BN tokens x 64 columns
    static constexpr int kBBytes = 2 * kBTileBytes;
    static constexpr int kStageBytes = kABytes + kBBytes;
    static constexpr int kCols = 2 * BN + 4;            // two accumulators + metadata
    static constexpr int kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128
                                     : kCols <= 256 ? 256 : 512;
    static constexpr int kEcol = 2 * BN;
    static constexpr int kBarBytes = 8 * (4 * STAGES + 6) + 32 + 24 * STAGES;
    static constexpr int kTabBytes = 2 * kMaxTableSteps * 8;  // two segments of table entries
    static constexpr int kSmemBytes = STAGES * kStageBytes + kTabBytes + 1024 + kBarBytes;
    static_assert(kBTileBytes % 1024 == 0, "stage regions must stay 1024-B aligned");
    static_assert(kCols <= 512, "tensor memory holds 512 columns");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

struct GemmParams {
    const uint8_t *packed;
    const uint64_t *table;
    int64_t N, K, M;
    int nsteps;      // K / 64
    int bands;       // N / 128
    int ttiles;      // ceil(M / BN)
    int stream_k;    // 0: whole tiles, 1: stream-K units
    int64_t units;   // stream-K: tiles * pairs
    void *Y;
    int y_fp32;
    float *partial;  // stream-K: [2 * gridDim.x][BN][128]
    uint32_t *status;
    const uint32_t *ready;  // set (release) by the packer once the packed bytes are final
    int stall_first_kstep;  // failure-detection test hook: CTA 0 never loads its first k-step
    int32_t u0[kMaxStreamKCtas + 1];  // stream-K: first unit of every CTA (u0[P] = units)
};

// One piece of work of a CTA: k-steps [ks0, ks1) of tile (band, ttile).
struct Segment {
    int tile, band, ttile, ks0, ks1;
    int nsegs;   // CTAs sharing the tile (1 = store Y directly)
    int slot;    // partial slot of this CTA for this tile
};

// CTA whose unit range holds unit x: the largest c with u0[c] <= x.
__device__ __forceinline__ int sk_cta_of(const int32_t *u0, int P, int64_t x) {
    int lo = 0, hi = P - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (u0[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ bool get_segment(const GemmParams &p, int c, int i, Segment &s) {
    const int P = gridDim.x;
    const int tiles = p.bands * p.ttiles;
    if (!p.stream_k) {
        const int64_t t = static_cast<int64_t>(c) + static_cast<int64_t>(i) * P;
        if (t >= tiles) return false;
        s.tile = static_cast<int>(t);
        s.ks0 = 0;
        s.ks1 = p.nsteps;
        s.nsegs = 1;
        s.slot = -1;
    } else {
        const int Q = p.nsteps / 2;
        const int64_t u0 = p.u0[c], u1 = p.u0[c + 1];
        if (u0 >= u1) return false;
        const int64_t t0 = u0 / Q;
        const int64_t t = t0 + i;
        if (t * Q >= u1) return false;
        const int64_t a = max(u0, t * Q), b = min(u1, (t + 1) * Q);
        s.tile = static_cast<int>(t);
        s.ks0 = static_cast<int>(2 * (a - t * Q));
        s.ks1 = static_cast<int>(2 * (b - t * Q));
        const int64_t cf = sk_cta_of(p.u0, P, t * Q), cl = sk_cta_of(p.u0, P, (t + 1) * Q - 1);
        s.nsegs = static_cast<int>(cl - cf + 1);
        s.slot = 2 * c + (t == t0 ? 0 : 1);
    }
    s.band = s.tile / p.ttiles;
    s.ttile = s.tile % p.ttiles;
    return true;
}

__device__ __forceinline__ void store_y(const GemmParams &p, int64_t idx, float v) {
    if (p.y_fp32)
        static_cast<float *>(p.Y)[idx] = v;
    else
        static_cast<__nv_bfloat16 *>(p.Y)[idx] = __float2bfloat16_rn(v);
}

// 4:8 expansion.  A stage region holds a 4:8 k-step as 128 rows x (32 kept
// bf16 at r*64, 8 keep masks at 8192 + r*8); in place it becomes 128 x 64 bf16
// in the K-major 128-byte-swizzled layout (row r, 16-byte chunk g at
// r*128 + (g ^ (r%8))*16).  Thread (row, hv) handles groups 4hv .. 4hv+3.
//
// The table entry of keep mask m (two uint4): for each 32-bit output word w
// (positions 2w, 2w+1 of the group) the byte-permute selector that picks the
// kept values' bytes out of {k01, k23} (the group's four kept values), and the
// mask that zeroes the pruned half-words.
__device__ __forceinline__ void nm48_lut_entry(uint32_t m, uint4 *lut) {
    uint32_t sel[4], zm[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const uint32_t i0 = __popc(m & ((1u << (2 * w)) - 1u)) & 3u;
        const uint32_t i1 = __popc(m & ((1u << (2 * w + 1)) - 1u)) & 3u;
        sel[w] = (2 * i0) | ((2 * i0 + 1) << 4) | ((2 * i1) << 8) | ((2 * i1 + 1) << 12);
        zm[w] = (((m >> (2 * w)) & 1u) ? 0x0000FFFFu : 0u) | (((m >> (2 * w + 1)) & 1u) ? 0xFFFF0000u : 0u);
    }
    lut[2 * m] = make_uint4(sel[0] | (sel[1] << 16), sel[2] | (sel[3] << 16), zm[0], zm[1]);
    lut[2 * m + 1] = make_uint4(zm[2], zm[3], 0u, 0u);
}
__device__ __forceinline__ void nm48_read(const uint8_t *region, int row, int hv, uint32_t (&v)[8],
                                          uint32_t &m) {
    const uint4 *src = reinterpret_cast<const uint4 *>(region + row * 64 + hv * 32);
    const uint4 a = src[0], b = src[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    m = *reinterpret_cast<const uint32_t *>(region + 8192 + row * 8 + hv * 4);
}
__device__ __forceinline__ void nm48_write(uint8_t *region, int row, int hv, const uint32_t (&v)[8],
                                           uint32_t m, const uint4 *lut) {
#pragma unroll
    for (int gg = 0; gg < 4; ++gg) {
        const uint32_t mask = (m >> (8 * gg)) & 0xFFu;
        const uint4 e0 = lut[2 * mask], e1 = lut[2 * mask + 1];
        const uint32_t k01 = v[2 * gg], k23 = v[2 * gg + 1];
        const uint4 o = make_uint4(__byte_perm(k01, k23, e0.x & 0xFFFFu) & e0.z,
                                   __byte_perm(k01, k23, e0.x >> 16) & e0.w,
                                   __byte_perm(k01, k23, e0.y & 0xFFFFu) & e1.x,
                                   __byte_perm(k01, k23, e0.y >> 16) & e1.y);
        const int g = 4 * hv + gg;
        *reinterpret_cast<uint4 *>(region + row * 128 + ((g ^ (row % 8)) * 16)) = o;
    }
}

__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int BN, int STAGES, bool NM>
__global__ void __launch_bounds__(NM ? kGemmThreadsNM : kGemmThreads, 1)
hybrid_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ GemmParams p) {
    using C = GemmCfg<BN, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t *tab_buf = reinterpret_cast<uint64_t *>(smem + STAGES * C::kStageBytes);  // [2][kMaxTableSteps]
    // 4:8: the expansion table, between the table entries and the barriers
    uint4 *lut = reinterpret_cast<uint4 *>(smem + STAGES * C::kStageBytes + C::kTabBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * C::kStageBytes + C::kTabBytes +
                                                  (NM ? kLutBytes : 0));
    uint64_t *empty = full + STAGES;
    uint64_t *acc_full = empty + STAGES;   // [2]
    uint64_t *acc_empty = acc_full + 2;    // [2]
    uint64_t *tab_full = acc_empty + 2;    // [2]
    uint64_t *conv = tab_full + 2;         // [STAGES] 4:8: stage converted (8 warps)
    uint64_t *cread = conv + STAGES;       // [STAGES] 4:8: inputs read (8 warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(cread + STAGES);
    volatile uint32_t *abort_flag = tmem_slot + 1;  // raised by any role that gives up
    volatile uint32_t *never_flag = tmem_slot + 2;  // stays 0: time-only bounded waits
    // per stage, written by the producer before it arms the stage: the pair's two
    // table entries and the stream offset of its first byte
    uint64_t *stage_info = reinterpret_cast<uint64_t *>(tmem_slot + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int cta = blockIdx.x;
    // thread 0 (the producer) knows whether it has passed griddepcontrol.wait
    bool waited = true;

    if (threadIdx.x == 0) {
        pdl_trigger();
        // the packed weights and table are final once the ready flag is seen;
        // otherwise (the packer may be the kernel just before) wait first
        if (ld_acquire_gpu(p.ready) == 0u) pdl_wait();
        else waited = false;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&conv[s], kConvWarps);
            mbar_init(&cread[s], kConvWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
            mbar_init(&tab_full[b], 1);
        }
        *never_flag = 0u;
        *abort_flag = (*reinterpret_cast<volatile uint32_t *>(p.status) & kStatusTimeout) ? 1u : 0u;
        fence_mbar_init();
        // the first two segments' table entries start moving before anything else
        if (!*abort_flag) {
            Segment g0;
            for (int i = 0; i < 2 && get_segment(p, cta, i, g0); ++i) {
                const uint32_t nbytes = static_cast<uint32_t>(g0.ks1 - g0.ks0) * 8u;
                mbar_arrive_expect_tx(&tab_full[i], nbytes);
                bulk_g2s(tab_buf + i * kMaxTableSteps,
                         p.table + static_cast<int64_t>(g0.band) * p.nsteps + g0.ks0, nbytes, &tab_full[i]);
            }
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmap_x);
    if constexpr (NM) {
        for (int m = static_cast<int>(threadIdx.x) - 192; m >= 0 && m < 256; m += kConvWarps * 32)
            nm48_lut_entry(static_cast<uint32_t>(m), lut);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const bool skip = *abort_flag != 0;

    if (warp == 0) {
        if (lane == 0 && !skip) {
            // ------------------------------------------------------ producer
            int it = 0;  // k-pairs issued so far (stage ring position)
            bool ok = true;
            // The table entries of a segment reach shared memory through one
            // bulk copy issued a whole segment ahead (two buffers), so no table
            // read waits behind the weight stream in the memory queues.
            Segment sg, nx;
            auto fetch_table = [&](const Segment &g, int buf) {
                const uint32_t nbytes = static_cast<uint32_t>(g.ks1 - g.ks0) * 8u;
                mbar_arrive_expect_tx(&tab_full[buf], nbytes);
                bulk_g2s(tab_buf + buf * kMaxTableSteps,
                         p.table + static_cast<int64_t>(g.band) * p.nsteps + g.ks0, nbytes, &tab_full[buf]);
            };
            bool have = get_segment(p, cta, 0, sg);  // tables 0 and 1 were fetched at start
            bool have_nx = have && get_segment(p, cta, 1, nx);
            int tabs_issued = (have ? 1 : 0) + (have_nx ? 1 : 0);
            // X tiles of the stages armed before griddepcontrol.wait
            int pend_s[STAGES], pend_t[STAGES], pend_pr[STAGES];
            int npend = 0;
            auto flush_pending = [&]() {
                pdl_wait();
                waited = true;
                for (int j = 0; j < npend; ++j)
                    tma_load_3d(smem + pend_s[j] * C::kStageBytes + C::kABytes, &tmap_x, 0,
                                pend_t[j] * BN, 2 * pend_pr[j], &full[pend_s[j]]);
                npend = 0;
            };
            for (int i = 0; ok && have; ++i) {
                const int buf = i & 1;
                if (!mbar_wait_bounded(&tab_full[buf], (i >> 1) & 1u, abort_flag, kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                const uint64_t *tab = tab_buf + buf * kMaxTableSteps;
                for (int pr = sg.ks0 / 2; pr < sg.ks1 / 2; ++pr) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!waited && it >= STAGES) flush_pending();
                    if (it >= STAGES && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    const uint64_t c0 = tab[2 * pr - sg.ks0], c1 = tab[2 * pr + 1 - sg.ks0];
                    const uint64_t first = (c0 & kEntryOffsetMask) - ((c0 & kEntryMeta) ? kMetaBlockBytes : 0);
                    const uint64_t end = (c1 & kEntryOffsetMask) +
                                         ((c1 & kEntrySparse) ? kSparseStepBytes : kDenseStepBytes);
                    const uint32_t bytes = static_cast<uint32_t>(end - first);
                    stage_info[3 * s + 0] = c0;
                    stage_info[3 * s + 1] = c1;
                    stage_info[3 * s + 2] = first;
                    ++it;
                    if (p.stall_first_kstep && cta == 0 && it == 1) continue;  // never lands
                    uint8_t *st = smem + s * C::kStageBytes;
                    if constexpr (NM) {
                        // 4:8 handle: each k-step into its own 16 KB region,
                        // where the converters expand a 4:8 one in place
                        const uint32_t b0 = (c0 & kEntryNM48) ? kNM48StepBytes : kDenseStepBytes;
                        const uint32_t b1 = (c1 & kEntryNM48) ? kNM48StepBytes : kDenseStepBytes;
                        mbar_arrive_expect_tx(&full[s], b0 + b1 + C::kBBytes);
                        bulk_g2s(st, p.packed + (c0 & kEntryOffsetMask), b0, &full[s]);
                        bulk_g2s(st + kDenseStepBytes, p.packed + (c1 & kEntryOffsetMask), b1, &full[s]);
                    } else {
                        mbar_arrive_expect_tx(&full[s], bytes + C::kBBytes);
                        bulk_g2s(st, p.packed + first, bytes, &full[s]);
                    }
                    if (waited) {
                        tma_load_3d(st + C::kABytes, &tmap_x, 0, sg.ttile * BN, 2 * pr, &full[s]);
                    } else {
                        pend_s[npend] = s;
                        pend_t[npend] = sg.ttile;
                        pend_pr[npend] = pr;
                        ++npend;
                    }
                }
                // this buffer is free again: fetch the table of segment i + 2
                sg = nx;
                have = have_nx;
                if (have) {
                    Segment n2;
                    have_nx = get_segment(p, cta, i + 2, n2);
                    if (have_nx) {
                        fetch_table(n2, buf);
                        ++tabs_issued;
                        nx = n2;
                    }
                }
            }
            if (!waited) flush_pending();
            // table copies still in flight must land before the CTA exits (the
            // latest phase of each buffer)
            for (int j = (tabs_issued > 2 ? tabs_issued - 2 : 0); j < tabs_issued; ++j)
                mbar_wait_bounded(&tab_full[j & 1], (j >> 1) & 1u, never_flag, kWaitLimitNs / 4);
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
            // Drain: the last phase issued on every stage must have landed
            // before the CTA exits (a no-op when the MMA thread consumed all).
            for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j) {
                if (p.stall_first_kstep && cta == 0 && j == 0) continue;  // never issued
                mbar_wait_bounded(&full[j % STAGES], (j / STAGES) & 1u, never_flag, kWaitLimitNs / 4);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && !skip) {
            // ---------------------------------------------------------- MMA
            const uint32_t e_tmem = tmem_base + C::kEcol;
            constexpr uint32_t kIdescDense = idesc_bf16(BN, false);
            int it = 0;
            bool ok = true;
            Segment sg;
            for (int i = 0; ok && get_segment(p, cta, i, sg); ++i) {
                const int buf = i & 1;
                if (i >= 2 && !mbar_wait_bounded(&acc_empty[buf], ((i >> 1) & 1u) ^ 1u, abort_flag,
                                                 kWaitLimitNs)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * BN;
                for (int pr = sg.ks0 / 2; pr < sg.ks1 / 2; ++pr, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    // 4:8 handle: the converters have rewritten the stage as dense tiles
                    if (NM && !mbar_wait_bounded(&conv[s], ph, abort_flag, kWaitLimitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t first = stage_info[3 * s + 2];
                    uint8_t *st = smem + s * C::kStageBytes;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint64_t e = NM ? 0ull : stage_info[3 * s + h];  // 4:8: all dense now
                        const uint32_t a_addr =
                            NM ? smem_u32(st + h * kDenseStepBytes)
                               : smem_u32(st + static_cast<uint32_t>((e & kEntryOffsetMask) - first));
                        const uint32_t b_addr = smem_u32(st + C::kABytes + h * C::kBTileBytes);
                        const bool first_step = (pr == sg.ks0 / 2) && h == 0;
                        if (e & kEntrySparse) {
                            if (e & kEntryMeta)
                                tmem_cp_128x128b(e_tmem, smem_desc(a_addr - kMetaBlockBytes, 16, 128,
                                                                   kSwizzleNone));
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const uint64_t ad = smem_desc(a_addr + j * 32, 16, 512, kSwizzle64B);
                                const uint64_t bd = smem_desc(b_addr + j * 64, 16, 1024, kSwizzle128B);
                                mma_sparse(d_tmem, ad, bd, e_tmem + 2 * h, idesc_bf16(BN, true, j),
                                           (first_step && j == 0) ? 0u : 1u);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const uint64_t ad = smem_desc(a_addr + j * 32, 16, 1024, kSwizzle128B);
                                const uint64_t bd = smem_desc(b_addr + j * 32, 16, 1024, kSwizzle128B);
                                mma_dense(d_tmem, ad, bd, kIdescDense, (first_step && j == 0) ? 0u : 1u);
                            }
                        }
                    }
                    tc_commit(&empty[s]);
                }
                // fires once every MMA of this tile has completed (also after a
                // failure, so the epilogue never deallocates under a running MMA)
                tc_commit(&acc_full[buf]);
            }
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
            }
        }
    } else if (warp >= 6) {
        if constexpr (NM) {
            if (!skip) {
                // -------------------------------------------- 4:8 converters
                // every stage in the MMA's order; a 4:8 k-step is rewritten in
                // place, so all rows are read (all eight warps meet on `cread`)
                // before any row is written
                const int t = (warp - 6) * 32 + lane;
                const int row = t >> 1, hv = t & 1;
                int it = 0;
                bool ok = true;
                Segment sg;
                for (int i = 0; ok && get_segment(p, cta, i, sg); ++i) {
                    for (int pr = sg.ks0 / 2; pr < sg.ks1 / 2; ++pr, ++it) {
                        const int s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1u;
                        if (!mbar_wait_bounded(&full[s], ph, abort_flag, kWaitLimitNs)) {
                            ok = false;
                            break;
                        }
                        uint8_t *st = smem + s * C::kStageBytes;
                        const bool c0 = (stage_info[3 * s + 0] & kEntryNM48) != 0;
                        const bool c1 = (stage_info[3 * s + 1] & kEntryNM48) != 0;
                        uint32_t v0[8], v1[8], m0 = 0, m1 = 0;
                        if (c0) nm48_read(st, row, hv, v0, m0);
                        if (c1) nm48_read(st + kDenseStepBytes, row, hv, v1, m1);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&cread[s]);
                        if (!mbar_wait_bounded(&cread[s], ph, abort_flag, kWaitLimitNs)) {
                            ok = false;
                            break;
                        }
                        if (c0) nm48_write(st, row, hv, v0, m0, lut);
                        if (c1) nm48_write(st + kDenseStepBytes, row, hv, v1, m1, lut);
                        fence_async_shared();  // the generic-proxy writes, visible to the MMA
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&conv[s]);
                    }
                }
                if (!ok) {
                    *abort_flag = 1u;
                    atomicOr(p.status, kStatusTimeout);
                }
            }
        }
    } else if (!skip) {
        // ------------------------------------------------------- epilogue
        pdl_wait();  // Y and the partials may still be in use by earlier kernels
        const int quad = warp % 4;  // TMEM lanes 32*quad .. 32*quad+31
        const int row = quad * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        Segment sg;
        for (int i = 0; get_segment(p, cta, i, sg); ++i) {
            const int buf = i & 1;
            // bounded by time only: the MMA thread commits acc_full even when
            // it gave up, so no MMA can be in flight at deallocation
            const bool ok = mbar_wait_bounded(&acc_full[buf], (i >> 1) & 1u, never_flag, kWaitLimitNs);
            tc_fence_after();
            if (!ok) {
                *abort_flag = 1u;
                atomicOr(p.status, kStatusTimeout);
                break;
            }
            const bool live = *abort_flag == 0;
            const int64_t n = static_cast<int64_t>(sg.band) * kBand + row;
            const int64_t m_base = static_cast<int64_t>(sg.ttile) * BN;
            const int m_valid = static_cast<int>(min(static_cast<int64_t>(BN), p.M - m_base));
            float *part = (sg.nsegs > 1) ? p.partial + static_cast<int64_t>(sg.slot) * BN * kBand
                                         : nullptr;
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 16) {
                uint32_t r[16];
                tmem_ld_32x32b_x16(lane_base + buf * BN + c0, r);
                tmem_ld_wait();
                if (!live) continue;
                if (part) {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c0 + q < m_valid) part[(c0 + q) * kBand + row] = __uint_as_float(r[q]);
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        if (c0 + q < m_valid)
                            store_y(p, (m_base + c0 + q) * p.N + n, __uint_as_float(r[q]));
                }
            }
            // the accumulator may be reused as soon as every lane has read it
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

// Stream-K fix-up: for every tile shared by several CTAs, Y = the partials of
// its CTAs added in CTA order (fixed order: the result does not depend on
// timing).  Launched as a programmatic dependent of the GEMM; waits for it.
template <int BN>
__global__ void __launch_bounds__(256)
streamk_reduce_kernel(const float *__restrict__ partial, const __grid_constant__ GemmParams p,
                      int P) {
    const int Q = p.nsteps / 2, ttiles = p.ttiles;
    const int64_t M = p.M, N = p.N;
    void *Y = p.Y;
    const int y_fp32 = p.y_fp32;
    // block (tile t, chunk): one output per thread, 256 outputs per block
    __shared__ int slots[64];
    __shared__ int nslots;
    const int64_t t = blockIdx.y;
    if (threadIdx.x == 0) {
        const int64_t cf = sk_cta_of(p.u0, P, t * Q), cl = sk_cta_of(p.u0, P, (t + 1) * Q - 1);
        int n = 0;
        if (cf != cl) {  // a tile with one CTA was stored directly
            for (int64_t cc = cf; cc <= cl && n < 64; ++cc)
                slots[n++] = static_cast<int>(2 * cc + ((p.u0[cc] / Q == t) ? 0 : 1));
        }
        nslots = n;
    }
    __syncthreads();
    const int ns = nslots;
    if (threadIdx.x == 0) pdl_trigger();  // the next GEMM may start its prologue
    pdl_wait();
    if (ns == 0) return;
    const int band = static_cast<int>(t / ttiles), ttile = static_cast<int>(t % ttiles);
    const int64_t m_base = static_cast<int64_t>(ttile) * BN;
    const int m_valid = static_cast<int>(min(static_cast<int64_t>(BN), M - m_base));
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= m_valid * kBand) return;
    const int m = e / kBand, row = e % kBand;
    const float *src = partial + m * kBand + row;
    float acc = 0.0f;
    for (int j0 = 0; j0 < ns; j0 += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            v[q] = (j0 + q < ns) ? __ldcg(src + static_cast<int64_t>(slots[j0 + q]) * BN * kBand) : 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q)
            if (j0 + q < ns) acc = __fadd_rn(acc, v[q]);
    }
    const int64_t yi = (m_base + m) * N + static_cast<int64_t>(band) * kBand + row;
    if (y_fp32)
        static_cast<float *>(Y)[yi] = acc;
    else
        static_cast<__nv_bfloat16 *>(Y)[yi] = __float2bfloat16_rn(acc);
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

// X [M,K] bf16 row-major viewed as (64 columns, M rows, K/64 k-steps); one box
// = both 64-column tiles of a k-pair for BN rows, 128-byte swizzle; rows past
// M read as zero.
bool make_x_map(CUtensorMap *map, const void *X, int64_t M, int64_t K, int bn) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kStep), static_cast<cuuint64_t>(M),
                                static_cast<cuuint64_t>(K / kStep)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(kStep) * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kStep), static_cast<cuuint32_t>(bn), 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(X), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Stream-K boundaries: unit u = tile * Q + pair (tile = band * ttiles + ttile)
// costs its packed bytes plus the bytes of its two X tiles; CTA c starts at the
// first unit whose cumulative cost reaches c / P of the total.
void streamk_bounds(const GemmLaunch &g, GemmParams &p, int bn, int P) {
    const int Q = p.nsteps / 2;
    const int64_t tiles = static_cast<int64_t>(p.bands) * p.ttiles;
    const int64_t xb = 2LL * bn * kStep * 2;  // X bytes per pair
    if (!g.pair_prefix) {  // equal unit counts
        for (int c = 0; c <= P; ++c) p.u0[c] = static_cast<int32_t>((c * p.units) / P);
        return;
    }
    auto pair_cum = [&](int band, int q) {  // cost of pairs [0, q) of a band
        return g.pair_prefix[static_cast<int64_t>(band) * (Q + 1) + q] + xb * q;
    };
    std::vector<int64_t> tile_cum(static_cast<size_t>(tiles + 1), 0);
    for (int64_t t = 0; t < tiles; ++t)
        tile_cum[t + 1] = tile_cum[t] + pair_cum(static_cast<int>(t / p.ttiles), Q);
    const int64_t total = tile_cum[tiles];
    p.u0[0] = 0;
    p.u0[P] = static_cast<int32_t>(p.units);
    for (int c = 1; c < P; ++c) {
        const int64_t target = (total * c) / P;
        // the tile holding the target, then the first pair boundary at or past it
        int64_t t = std::upper_bound(tile_cum.begin(), tile_cum.end(), target) - tile_cum.begin() - 1;
        if (t >= tiles) t = tiles - 1;
        const int band = static_cast<int>(t / p.ttiles);
        int q = 0;
        while (q < Q && tile_cum[t] + pair_cum(band, q) < target) ++q;
        int64_t u = t * Q + q;
        if (u < p.u0[c - 1]) u = p.u0[c - 1];
        p.u0[c] = static_cast<int32_t>(u);
    }
    // every CTA keeps at least one unit (P <= units)
    for (int c = 1; c < P; ++c)
        if (p.u0[c] <= p.u0[c - 1]) p.u0[c] = p.u0[c - 1] + 1;
    p.u0[P] = static_cast<int32_t>(p.units);
    for (int c = P - 1; c >= 1; --c)
        if (p.u0[c] >= p.u0[c + 1]) p.u0[c] = p.u0[c + 1] - 1;
}

template <int BN, int STAGES, bool NM = false>
cudaError_t run(const GemmLaunch &g, int ctas_per_sm, cudaStream_t stream) {
    using C = GemmCfg<BN, STAGES>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    constexpr int kSmem = C::kSmemBytes + (NM ? kLutBytes : 0);
    static_assert(kSmem <= 232448, "shared memory per CTA");
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(hybrid_gemm_kernel<BN, STAGES, NM>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
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
    p.bands = static_cast<int>(g.N / kBand);
    p.ttiles = static_cast<int>((g.M + BN - 1) / BN);
    p.Y = g.Y;
    p.y_fp32 = g.y_fp32;
    p.status = g.status;
    p.ready = g.ready;
    p.stall_first_kstep = g.stall_first_kstep;
    const int64_t tiles = static_cast<int64_t>(p.bands) * p.ttiles;
    const int64_t slots = static_cast<int64_t>(g.num_sms) * ctas_per_sm;
    // whole tiles when there are at least two waves of them, stream-K otherwise
    const bool sk = tiles < 2 * slots;
    p.stream_k = sk ? 1 : 0;
    p.units = tiles * (p.nsteps / 2);
    // stream-K: at most 62 CTAs per tile, so a tile's partials fit the fix-up's slot list
    const int64_t grid = sk ? std::min<int64_t>(std::min<int64_t>(std::min<int64_t>(slots, p.units),
                                                                   62 * tiles),
                                                kMaxStreamKCtas)
                            : std::min<int64_t>(slots, tiles);
    if (sk) streamk_bounds(g, p, BN, static_cast<int>(grid));
    float *ws = nullptr;
    if (sk) {
        const size_t bytes = sizeof(float) * static_cast<size_t>(2 * grid) * BN * kBand;
        if (g.workspace && bytes <= g.workspace_bytes) {
            ws = g.workspace;
        } else {
            cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), bytes, g.pool, stream);
            if (e != cudaSuccess) return e;
        }
    }
    p.partial = ws;
    // programmatic dependent launch: the prologue and the first weight copies
    // overlap the previous kernel (see the kernel's comment on what it reads
    // before griddepcontrol.wait)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(NM ? kGemmThreadsNM : kGemmThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, hybrid_gemm_kernel<BN, STAGES, NM>, map, p);
    if (err == cudaSuccess) note_launches(1);
    if (err == cudaSuccess && sk) {
        cfg.gridDim = dim3(static_cast<unsigned>((BN * kBand + 255) / 256), static_cast<unsigned>(tiles));
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = 0;
        err = cudaLaunchKernelEx(&cfg, streamk_reduce_kernel<BN>, static_cast<const float *>(ws), p,
                                 static_cast<int>(grid));
        if (err == cudaSuccess) note_launches(1);
    }
    if (ws && ws != g.workspace) {
        cudaError_t e2 = cudaFreeAsync(ws, stream);
        if (err == cudaSuccess) err = e2;
    }
    return err;
}

}  // namespace

void preload_hybrid_kernels() {
    cudaFuncAttributes a;
    (void)cudaFuncGetAttributes(&a, hybrid_gemm_kernel<64, 4, false>);
    (void)cudaFuncGetAttributes(&a, hybrid_gemm_kernel<128, 3, false>);
    (void)cudaFuncGetAttributes(&a, hybrid_gemm_kernel<160, 3, false>);
    (void)cudaFuncGetAttributes(&a, hybrid_gemm_kernel<64, 4, true>);
    (void)cudaFuncGetAttributes(&a, hybrid_gemm_kernel<128, 3, true>);
    (void)cudaFuncGetAttributes(&a, streamk_reduce_kernel<64>);
    (void)cudaFuncGetAttributes(&a, streamk_reduce_kernel<128>);
    (void)cudaFuncGetAttributes(&a, streamk_reduce_kernel<160>);
}

cudaError_t launch_hybrid_gemm(const GemmLaunch &g, cudaStream_t stream) {
    if (g.pattern == 4) {
        // 4:8 handles: the one-band kernel with converter warps, every M
        // (stream-K over (tile, k-pair) units when tiles are few)
        if (g.M <= 64) return run<64, 4, true>(g, 1, stream);
        return run<128, 3, true>(g, 1, stream);
    }
    if (g.M <= 16) return launch_decode_gemm(g, stream);  // split-K GEMV, csrc/decode_gemm.cu
    // test hook: one prefill kernel for every M > 16 (parity of each kernel)
    if (g.force_kernel == 1) return g.M <= 64 ? run<64, 4>(g, 1, stream) : run<160, 3>(g, 1, stream);
    if (g.force_kernel == 2 && g.K / kStep <= 448) return launch_pair_gemm(g, plan_pair_gemm(g.N, g.M, g.num_sms), stream);
    if (g.force_kernel == 3 && g.duo_ok && g.K / kStep <= 448) {
        const DuoPlan dp = plan_duo_gemm(g.N, g.M, g.num_sms, g.max_pair_bytes);
        if (dp.bn > 0) return launch_duo_gemm(g, dp, stream);
    }
    if (g.force_kernel == 4 && g.duo_ok && g.K / kStep <= 448) {
        const QuadPlan qp = plan_quad_gemm(g.N, g.M, g.num_sms);
        if (qp.bn > 0) return launch_quad_gemm(g, qp, stream);
    }
    // up to 64 tokens: the split-K kernel of csrc/decode_gemm.cu (32- or
    // 64-token tiles, four k-pairs per chunk, every chunk's partial added in
    // order by the fix-up) while a band has at most 16 chunks; for longer K
    // this file's stream-K kernel, with two partials per CTA, is faster.
    // Measured on B200, back-to-back calls on the Llama-7B block shapes at
    // f = 0.6: 4096x4096 M = 32 / 64: 11.6 / 12.5 us against 14.4 / 14.5;
    // 11008x4096: 20.7 / 24.9 against 24.1 / 25.2; 4096x11008: 21.7 / 23.2
    // against 20.6 / 21.2.
    if (takes_split_k(g.M, g.K, 0)) return launch_decode_gemm(g, stream);
    if (g.M <= 64) return run<64, 4>(g, 1, stream);   // 48 KB stages
    if (g.M <= 128) return run<128, 3>(g, 1, stream); // 64 KB stages
    // larger token counts: the band-pair kernel (two bands share each X tile)
    // unless its items fall into so few waves that this kernel's finer tiles
    // finish first.  Both estimated per k-step from shared-memory traffic
    // (copies in + tensor-core operand reads at 128 B per cycle): a 160-token
    // one-band item moves 72 KB per dense k-step, 576 cycles.
    const PairPlan pp = plan_pair_gemm(g.N, g.M, g.num_sms);
    const int64_t items1 = (g.N / kBand) * ((g.M + 159) / 160);
    const int64_t waves1 = (items1 + g.num_sms - 1) / g.num_sms;
    const double t_one = static_cast<double>(waves1) * 576.0;
    if (g.duo_ok && g.K / kStep <= 448) {
        // two-SM MMAs (through the prefill table, whose band pairs agree in
        // type) when their estimate is lowest.  The four-band variant
        // (prefill_quad.cu) measured slower than this one on the 7B and 13B
        // MLP shapes (latency-bound at about a third of the tensor pipe), so
        // it is reached only through the test hook.
        const DuoPlan dp = plan_duo_gemm(g.N, g.M, g.num_sms, g.max_pair_bytes);
        if (dp.bn > 0 && dp.cost <= pp.cost && dp.cost <= t_one) return launch_duo_gemm(g, dp, stream);
    }
    if (pp.cost <= t_one && g.K / kStep <= 448)
        return launch_pair_gemm(g, pp, stream);
    return run<160, 3>(g, 1, stream);                 // 72 KB stages
}

namespace {

// The estimate launch_hybrid_gemm acts on for one bf16 2:4 matrix above 128
// tokens: the lowest of the one-band, band-pair and two-SM estimates.
double own_prefill_cost(const GemmLaunch &g) {
    const PairPlan pp = plan_pair_gemm(g.N, g.M, g.num_sms);
    const int64_t items1 = (g.N / kBand) * ((g.M + 159) / 160);
    double cost = static_cast<double>((items1 + g.num_sms - 1) / g.num_sms) * 576.0;
    if (g.K / kStep <= 448) cost = std::min(cost, pp.cost);
    if (g.duo_ok && g.K / kStep <= 448) {
        const DuoPlan dp = plan_duo_gemm(g.N, g.M, g.num_sms, g.max_pair_bytes);
        if (dp.bn > 0) cost = std::min(cost, dp.cost);
    }
    return cost;
}

}  // namespace

bool plan_hybrid_group(const GemmLaunch *gs, int count, DuoPlan *plan) {
    if (count < 2 || count > kDuoGroupMax) return false;
    const GemmLaunch &g = gs[0];
    if (g.M <= 128 || g.K / kStep > 448) return false;
    int64_t sum_n = 0;
    int max_pair = 0;
    double own = 0;
    for (int i = 0; i < count; ++i) {
        const GemmLaunch &m = gs[i];
        if (m.pattern != 2 || !m.duo_ok || m.K != g.K || m.M != g.M || m.num_sms != g.num_sms ||
            m.force_kernel != g.force_kernel || (m.N / kBand) % 2 != 0)
            return false;
        sum_n += m.N;
        max_pair = std::max(max_pair, m.max_pair_bytes);
        own += own_prefill_cost(m);
    }
    // test hook 3 (two-SM kernel for every M) takes the grouped launch too
    if (g.force_kernel != 0 && g.force_kernel != 3) return false;
    const DuoPlan dp = plan_duo_gemm(sum_n, g.M, g.num_sms, max_pair);
    if (dp.bn == 0) return false;
    if (g.force_kernel == 0 && dp.cost > own) return false;
    *plan = dp;
    return true;
}

}  // namespace patchk
