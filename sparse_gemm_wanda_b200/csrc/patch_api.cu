// C ABI of the tile-hybrid sparse linear layer: argument checks, planning of
// the packed layout, device memory of the packed handle, kernel launches.
// Declarations and the normative description of every call: include/patch.h.
#include <atomic>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <set>
#include <mutex>
#include <new>
#include <vector>

#include "patch.h"
#include "patch_common.cuh"
#include "patch_internal.h"

struct patch_packed {
    int device;
    int pattern;               // 2: dense / 2:4 tiles; 4: dense / 4:8 tiles; 8: FP8 dense / 2:4
    float *fp8_scale;          // FP8 handles: W_eff row scales [N]
    uint8_t *fp8_xscratch;     // FP8 handles: X codes and token scales of calls with M <= kFp8ScratchRows
    uint8_t *base;             // pool allocation: table, descriptors, prefix, plan, workspace, status
    patch_shape shp;
    uint8_t *packed;           // packed k-steps, then the side copies (a pool allocation of its own, exact size)
    size_t packed_bytes;       // the packed k-steps (the normative format)
    size_t side_bytes;         // dense k-pair copies after them, for the prefill table
    uint64_t *table;           // (N/128) * (K/64) entries
    uint64_t *ptable;          // prefill table: (N/128) * (K/64) entries
    int64_t sparse_ksteps;
    int64_t meta_blocks;
    float *workspace;          // decode partials (one slot per chunk); reused by stream-K
    size_t workspace_bytes;
    uint64_t *chunk_desc;      // device: decode chunk descriptors
    std::vector<uint64_t> chunk_desc_host;
    int dec_cp, dec_cpb, dec_nchunks;
    int duo_ok;                // even band count: the prefill table pairs bands 2p, 2p+1
    int max_pair_bytes;        // largest k-pair the prefill table points to
    uint32_t *status;          // device: status word, pack counter, ready flag
    int num_sms;
    cudaMemPool_t pool;
    int64_t bands;
    int64_t *pair_prefix_dev;  // device: per band, cumulative packed bytes of its k-pairs
    // host copy of pair_prefix, read back by patch_pack
    std::vector<int64_t> pair_prefix;
};

namespace {

using patchk::kBand;
using patchk::kStep;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool tile_ok(int32_t t) { return t == 64 || t == 128; }

patch_status check_shape(const patch_shape &s) {
    if (s.N <= 0 || s.K <= 0) return PATCH_ERR_INVALID_ARG;
    if (!tile_ok(s.tile_n) || !tile_ok(s.tile_k)) return PATCH_ERR_UNSUPPORTED;
    if (s.N % s.tile_n != 0 || s.K % s.tile_k != 0) return PATCH_ERR_INVALID_ARG;
    if (s.K % 64 != 0) return PATCH_ERR_INVALID_ARG;
    if (s.N > (int64_t(1) << 31) || s.K > (int64_t(1) << 31)) return PATCH_ERR_INVALID_ARG;
    return PATCH_OK;
}

struct DevInfo {
    int major = 0, minor = 0, sms = 0;
};

// Compute capability and SM count of the current device (queried once).
patch_status check_device(int *num_sms) {
    static std::mutex mu;
    static std::map<int, DevInfo> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PATCH_ERR_CUDA;
    DevInfo info;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(dev);
        if (it != cache.end()) {
            info = it->second;
        } else {
            if (cudaDeviceGetAttribute(&info.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&info.minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
                cudaDeviceGetAttribute(&info.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return PATCH_ERR_CUDA;
            cache[dev] = info;
        }
    }
    if (info.major != 10 || info.minor != 0) return PATCH_ERR_UNSUPPORTED;
    if (num_sms) *num_sms = info.sms;
    return PATCH_OK;
}

// The plan summaries written by plan_pack_kernel and each matrix's per-band
// k-pair prefix (the prefill kernels balance their work with it), read back
// into one page-locked buffer per device (grown on demand, held under the
// lock until the copies landed) and from there into `dst` and `prefix[i]`.
// Every copy is asynchronous; the stream is waited for once, here, and no
// later call on the handles waits.
cudaError_t read_plans(const patchk::PackPlan *const *src, patchk::PackPlan *dst, const int64_t *const *prefix_src,
                       std::vector<int64_t> *const *prefix, int count, cudaStream_t stream) {
    static std::mutex mu;
    static std::map<int, std::pair<uint8_t *, size_t>> bufs;
    if (count < 1 || count > patchk::kPlanMaxGroup) return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    size_t need = sizeof(patchk::PackPlan) * static_cast<size_t>(count);
    for (int i = 0; i < count; ++i) need += sizeof(int64_t) * prefix[i]->size();
    std::lock_guard<std::mutex> lock(mu);
    std::pair<uint8_t *, size_t> &buf = bufs[dev];
    if (buf.second < need) {
        if (buf.first) cudaFreeHost(buf.first);  // no copy into it is in flight: each call waits for its own
        buf = {nullptr, 0};
        e = cudaMallocHost(reinterpret_cast<void **>(&buf.first), need);
        if (e != cudaSuccess) {
            buf = {nullptr, 0};
            return e;
        }
        buf.second = need;
    }
    patchk::PackPlan *plans = reinterpret_cast<patchk::PackPlan *>(buf.first);
    int64_t *pre = reinterpret_cast<int64_t *>(buf.first + sizeof(patchk::PackPlan) * static_cast<size_t>(count));
    size_t at = 0;
    for (int i = 0; i < count && e == cudaSuccess; ++i) {
        e = cudaMemcpyAsync(plans + i, src[i], sizeof(patchk::PackPlan), cudaMemcpyDeviceToHost, stream);
        if (e == cudaSuccess && !prefix[i]->empty())
            e = cudaMemcpyAsync(pre + at, prefix_src[i], sizeof(int64_t) * prefix[i]->size(), cudaMemcpyDeviceToHost,
                                stream);
        at += prefix[i]->size();
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return e;
    at = 0;
    for (int i = 0; i < count; ++i) {
        dst[i] = plans[i];
        std::copy(pre + at, pre + at + prefix[i]->size(), prefix[i]->begin());
        at += prefix[i]->size();
    }
    return cudaSuccess;
}

// Failure-detection test hook (see patch_test_stall_first_kstep): read from
// the environment once, when the library is loaded; changed only by the
// exported setter.
std::atomic<int> g_test_kernel{0};  // patch_test_prefill_kernel

std::atomic<int> g_test_stall{[] {
    const char *v = getenv("PATCH_B200_TEST_STALL");
    return (v && v[0] == '1') ? 1 : 0;
}()};

patch_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return PATCH_OK;
    if (e == cudaErrorMemoryAllocation) return PATCH_ERR_OOM;
    return PATCH_ERR_CUDA;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace

namespace patchk {

cudaError_t device_pool(cudaMemPool_t *pool) {
    static std::mutex mu;
    static std::map<int, cudaMemPool_t> pools;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = pools.find(dev);
    if (it != pools.end()) {
        *pool = it->second;
        return cudaSuccess;
    }
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t p = nullptr;
    e = cudaMemPoolCreate(&p, &props);
    if (e != cudaSuccess) return e;
    uint64_t keep = UINT64_MAX;  // keep freed blocks cached across synchronisations
    e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &keep);
    if (e != cudaSuccess) return e;
    pools[dev] = p;
    *pool = p;
    return cudaSuccess;
}

}  // namespace patchk

namespace patchk {
namespace {
std::atomic<uint64_t> g_launches{0};
}  // namespace
void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
}  // namespace patchk

extern "C" {

const char *patch_status_string(patch_status s) {
    switch (s) {
        case PATCH_OK: return "ok";
        case PATCH_ERR_INVALID_ARG: return "invalid argument";
        case PATCH_ERR_UNSUPPORTED: return "unsupported";
        case PATCH_ERR_CUDA: return "cuda error";
        case PATCH_ERR_OOM: return "out of device memory";
        case PATCH_ERR_TIMEOUT: return "bounded device wait ran out";
    }
    return "unknown status";
}

static patch_status score_mask_impl(const void *W_bf16, const void *Xcal_bf16, int64_t T,
                                    const double *colsq_in, patch_shape shp,
                                    double sparse_tile_fraction, const uint32_t *map_in,
                                    uint32_t *meta_out, uint32_t *map_out, double *colsq_out,
                                    double *tile_loss_out, void *stream_v, int pattern) {
    patch_status st = check_shape(shp);
    if (st != PATCH_OK) return st;
    if (!W_bf16 || !meta_out || !map_out || !aligned16(W_bf16)) return PATCH_ERR_INVALID_ARG;
    if (!colsq_in && (!Xcal_bf16 || T < 1 || !aligned16(Xcal_bf16))) return PATCH_ERR_INVALID_ARG;
    if (!map_in && !(sparse_tile_fraction >= 0.0 && sparse_tile_fraction <= 1.0))
        return PATCH_ERR_INVALID_ARG;
    st = check_device(nullptr);
    if (st != PATCH_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);

    const int64_t N = shp.N, K = shp.K;
    const int64_t n_tiles = (N / shp.tile_n) * (K / shp.tile_k);
    const int64_t chunks = colsq_in ? 0 : (T + 127) / 128;

    // one stream-ordered scratch allocation: chunk partials, norms, loss, rank
    size_t off_partial = 0;
    size_t off_norm = round_up(off_partial + sizeof(double) * chunks * K, 256);
    size_t off_loss = round_up(off_norm + sizeof(double) * K, 256);
    size_t off_rank = round_up(off_loss + (tile_loss_out ? 0 : sizeof(double) * n_tiles), 256);
    size_t off_done = round_up(off_rank + (map_in ? 0 : sizeof(int32_t) * n_tiles), 256);
    size_t total = off_done + 256;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = patchk::device_pool(&pool);
    if (e != cudaSuccess) return from_cuda(e);
    uint8_t *scratch = nullptr;
    e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&scratch), total, pool, stream);
    if (e != cudaSuccess) return from_cuda(e);
    double *partial = reinterpret_cast<double *>(scratch + off_partial);
    double *norm = reinterpret_cast<double *>(scratch + off_norm);
    double *loss = tile_loss_out ? tile_loss_out : reinterpret_cast<double *>(scratch + off_loss);
    int32_t *rank = map_in ? nullptr : reinterpret_cast<int32_t *>(scratch + off_rank);
    uint32_t *done = reinterpret_cast<uint32_t *>(scratch + off_done);

    if (colsq_in)
        e = patchk::launch_norms_from_colsq(colsq_in, K, colsq_out, norm, stream);
    else
        e = patchk::launch_colsq(Xcal_bf16, T, K, partial, colsq_out, norm, stream);
    if (e == cudaSuccess)
        e = patchk::launch_score_mask(W_bf16, norm, N, K, shp.tile_n, shp.tile_k, meta_out, loss,
                                      rank, done, stream, pattern);
    if (e == cudaSuccess) {
        if (map_in) {
            e = cudaMemcpyAsync(map_out, map_in, sizeof(uint32_t) * ((n_tiles + 31) / 32),
                                cudaMemcpyDeviceToDevice, stream);
        } else {
            const int64_t n_sp =
                static_cast<int64_t>(floor(sparse_tile_fraction * static_cast<double>(n_tiles)));
            e = patchk::launch_select_map(loss, n_tiles, n_sp, rank, done, map_out, stream);
        }
    }
    cudaError_t e2 = cudaFreeAsync(scratch, stream);
    return from_cuda(e != cudaSuccess ? e : e2);
}

// (n_keep, m_group) -> pattern code: 2 for 2:4, 4 for 4:8, 0 otherwise
static int pattern_of(int32_t n_keep, int32_t m_group) {
    if (n_keep == 2 && m_group == 4) return 2;
    if (n_keep == 4 && m_group == 8) return 4;
    return 0;
}

patch_status patch_score_mask(const void *W_bf16, const void *Xcal_bf16, int64_t T,
                              const double *colsq_in, patch_shape shp,
                              double sparse_tile_fraction, const uint32_t *map_in,
                              uint32_t *meta_out, uint32_t *map_out, double *colsq_out,
                              double *tile_loss_out, void *stream_v) {
    return score_mask_impl(W_bf16, Xcal_bf16, T, colsq_in, shp, sparse_tile_fraction, map_in, meta_out,
                           map_out, colsq_out, tile_loss_out, stream_v, 2);
}

patch_status patch_score_mask_nm(const void *W_bf16, const void *Xcal_bf16, int64_t T,
                                 const double *colsq_in, patch_shape shp, int32_t n_keep,
                                 int32_t m_group, double sparse_tile_fraction, const uint32_t *map_in,
                                 uint32_t *meta_out, uint32_t *map_out, double *colsq_out,
                                 double *tile_loss_out, void *stream_v) {
    const int pattern = pattern_of(n_keep, m_group);
    if (!pattern) return PATCH_ERR_UNSUPPORTED;
    return score_mask_impl(W_bf16, Xcal_bf16, T, colsq_in, shp, sparse_tile_fraction, map_in, meta_out,
                           map_out, colsq_out, tile_loss_out, stream_v, pattern);
}

patch_status patch_colsq(const void *Xcal_bf16, int64_t T, int64_t K, double *colsq_out,
                         void *stream_v) {
    if (!Xcal_bf16 || !colsq_out || T < 1 || K < 64 || K % 64 != 0 || !aligned16(Xcal_bf16))
        return PATCH_ERR_INVALID_ARG;
    patch_status st = check_device(nullptr);
    if (st != PATCH_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    const int64_t chunks = (T + 127) / 128;
    cudaMemPool_t pool = nullptr;
    cudaError_t e = patchk::device_pool(&pool);
    if (e != cudaSuccess) return from_cuda(e);
    double *partial = nullptr;
    e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&partial),
                                sizeof(double) * static_cast<size_t>(chunks * K), pool, stream);
    if (e != cudaSuccess) return from_cuda(e);
    e = patchk::launch_colsq(Xcal_bf16, T, K, partial, colsq_out, nullptr, stream);
    cudaError_t e2 = cudaFreeAsync(partial, stream);
    return from_cuda(e != cudaSuccess ? e : e2);
}

patch_status patch_colsq_partials(const void *Xcal_bf16, int64_t T, int64_t K,
                                  double *partials_out, void *stream_v) {
    if (!Xcal_bf16 || !partials_out || T < 1 || K < 64 || K % 64 != 0 || !aligned16(Xcal_bf16) ||
        !aligned16(partials_out))
        return PATCH_ERR_INVALID_ARG;
    patch_status st = check_device(nullptr);
    if (st != PATCH_OK) return st;
    return from_cuda(patchk::launch_colsq_partials(Xcal_bf16, T, K, partials_out,
                                                   static_cast<cudaStream_t>(stream_v)));
}

patch_status patch_colsq_fold(const double *partials, int64_t chunks, int64_t K, double *colsq_out,
                              void *stream_v) {
    if (!partials || !colsq_out || chunks < 1 || K < 64 || K % 64 != 0 || !aligned16(partials))
        return PATCH_ERR_INVALID_ARG;
    patch_status st = check_device(nullptr);
    if (st != PATCH_OK) return st;
    return from_cuda(patchk::launch_colsq_fold(partials, chunks, K, colsq_out, nullptr,
                                               static_cast<cudaStream_t>(stream_v)));
}

// ------------------------------------------------------ allocation-free mask
// Scratch of patch_score_mask_noalloc: a fixed array in device memory that
// every device loading this library holds until the process exits.  Host code
// must not pass the symbol itself to a kernel (on the host it is only a
// stand-in); its device address is looked up once per device below.
constexpr size_t kNoallocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

// Driver entry points for the current context and its process-unique id,
// fetched through the runtime (the library links no driver stub).
using CtxGetCurrentFn = int (*)(void **);
using CtxGetIdFn = int (*)(void *, unsigned long long *);

static bool current_context_id(unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    void *ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != 0 || !ctx) return false;
    return get_id(ctx, id) == 0;
}

// Device address of the scratch array in the current context.  The address
// belongs to a context (a device reset or a new primary context maps the
// module again, elsewhere), so it is cached per context id, never per device
// ordinal.  A miss, or a context the driver cannot name, looks it up with
// cudaGetSymbolAddress; under lazy module loading that first lookup loads
// this library's module on the device, which is when the array is reserved.
static cudaError_t noalloc_scratch_address(uint8_t **ptr) {
    static std::mutex mu;
    static std::map<unsigned long long, uint8_t *> addr;
    std::lock_guard<std::mutex> lock(mu);
    unsigned long long id = 0;
    const bool named = current_context_id(&id);
    if (named) {
        auto it = addr.find(id);
        if (it != addr.end()) {
            *ptr = it->second;
            return cudaSuccess;
        }
    }
    void *p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // with the device current
    if (e != cudaSuccess) return e;
    // the lookup made the runtime's context current if none was: cache under it
    if (current_context_id(&id)) addr[id] = static_cast<uint8_t *>(p);
    *ptr = static_cast<uint8_t *>(p);
    return cudaSuccess;
}

// The GEMM kernels, loaded once per context (see preload_* in
// patch_internal.h); a context the driver cannot name loads them every time
// (cheap once loaded).
static void preload_gemm_kernels() {
    static std::mutex mu;
    static std::set<unsigned long long> done;
    unsigned long long id = 0;
    const bool named = current_context_id(&id);
    std::lock_guard<std::mutex> lock(mu);
    if (named && done.count(id)) return;
    patchk::preload_hybrid_kernels();
    patchk::preload_decode_kernels();
    patchk::preload_pair_kernels();
    patchk::preload_duo_kernels();
    patchk::preload_quad_kernels();
    patchk::preload_fp8_gemm_kernels();
    patchk::preload_duo_fp8_kernels();
    patchk::preload_fp8_quantize_kernels();
    patchk::preload_pack_kernels();
    if (named) done.insert(id);
}

patch_status patch_score_mask_noalloc(const void *W_bf16, const void *Xcal_bf16, int64_t T,
                                      const double *colsq_in, patch_shape shp,
                                      double sparse_tile_fraction, const uint32_t *map_in,
                                      uint32_t *meta_out, uint32_t *map_out, double *colsq_out,
                                      double *tile_loss_out, void *stream_v) {
    patch_status st = check_shape(shp);
    if (st != PATCH_OK) return st;
    if (!W_bf16 || !meta_out || !map_out || !aligned16(W_bf16)) return PATCH_ERR_INVALID_ARG;
    if (!colsq_in && (!Xcal_bf16 || T < 1 || !aligned16(Xcal_bf16))) return PATCH_ERR_INVALID_ARG;
    if (!map_in && !(sparse_tile_fraction >= 0.0 && sparse_tile_fraction <= 1.0))
        return PATCH_ERR_INVALID_ARG;
    const int64_t N = shp.N, K = shp.K;
    const int64_t n_tiles = (N / shp.tile_n) * (K / shp.tile_k);
    const int64_t chunks = colsq_in ? 0 : (T + 127) / 128;
    // same scratch layout as patch_score_mask, inside the fixed array
    const size_t off_norm = round_up(sizeof(double) * static_cast<size_t>(chunks * K), 256);
    const size_t off_loss = round_up(off_norm + sizeof(double) * K, 256);
    const size_t off_rank = round_up(off_loss + (tile_loss_out ? 0 : sizeof(double) * n_tiles), 256);
    const size_t off_done = round_up(off_rank + (map_in ? 0 : sizeof(int32_t) * n_tiles), 256);
    const size_t total = off_done + 256;
    if (total > kNoallocScratchBytes) return PATCH_ERR_UNSUPPORTED;  // beyond the fixed scratch
    st = check_device(nullptr);
    if (st != PATCH_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    uint8_t *scratch = nullptr;
    cudaError_t e = noalloc_scratch_address(&scratch);
    if (e != cudaSuccess) return from_cuda(e);
    double *partial = reinterpret_cast<double *>(scratch);
    double *norm = reinterpret_cast<double *>(scratch + off_norm);
    double *loss = tile_loss_out ? tile_loss_out : reinterpret_cast<double *>(scratch + off_loss);
    int32_t *rank = map_in ? nullptr : reinterpret_cast<int32_t *>(scratch + off_rank);
    uint32_t *done = reinterpret_cast<uint32_t *>(scratch + off_done);
    // every scratch value is written before it is read in this call (the
    // score kernel zeroes the rank counters), so leftovers of the previous
    // call do not matter
    if (colsq_in)
        e = patchk::launch_norms_from_colsq(colsq_in, K, colsq_out, norm, stream);
    else
        e = patchk::launch_colsq(Xcal_bf16, T, K, partial, colsq_out, norm, stream);
    if (e == cudaSuccess)
        e = patchk::launch_score_mask(W_bf16, norm, N, K, shp.tile_n, shp.tile_k, meta_out, loss,
                                      rank, done, stream);
    if (e == cudaSuccess) {
        if (map_in) {
            e = cudaMemcpyAsync(map_out, map_in, sizeof(uint32_t) * ((n_tiles + 31) / 32),
                                cudaMemcpyDeviceToDevice, stream);
        } else {
            const int64_t n_sp =
                static_cast<int64_t>(floor(sparse_tile_fraction * static_cast<double>(n_tiles)));
            e = patchk::launch_select_map(loss, n_tiles, n_sp, rank, done, map_out, stream);
        }
    }
    return from_cuda(e);
}

size_t patch_score_mask_noalloc_capacity(void) { return kNoallocScratchBytes; }

patch_status patch_pool_usage(uint64_t *used_now, uint64_t *used_high, int32_t reset_high) {
    cudaMemPool_t pool = nullptr;
    cudaError_t e = patchk::device_pool(&pool);
    if (e != cudaSuccess) return from_cuda(e);
    if (reset_high) {
        uint64_t zero = 0;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &zero);
        if (e != cudaSuccess) return from_cuda(e);
    }
    uint64_t now = 0, high = 0;
    e = cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemCurrent, &now);
    if (e == cudaSuccess) e = cudaMemPoolGetAttribute(pool, cudaMemPoolAttrUsedMemHigh, &high);
    if (e != cudaSuccess) return from_cuda(e);
    if (used_now) *used_now = now;
    if (used_high) *used_high = high;
    return PATCH_OK;
}

patch_status patch_select_maps_global(const double *const *losses, const int64_t *n_tiles,
                                      int32_t count, double fraction, uint32_t *const *maps_out,
                                      void *stream_v) {
    if (!losses || !n_tiles || !maps_out || count < 1 || count > patchk::kMaxGlobalMatrices)
        return PATCH_ERR_INVALID_ARG;
    if (!(fraction >= 0.0 && fraction <= 1.0)) return PATCH_ERR_INVALID_ARG;
    int64_t total = 0;
    for (int32_t m = 0; m < count; ++m) {
        if (!losses[m] || !maps_out[m] || n_tiles[m] < 1) return PATCH_ERR_INVALID_ARG;
        total += n_tiles[m];
    }
    if (total > patchk::kMaxGlobalTiles) return PATCH_ERR_UNSUPPORTED;
    patch_status st = check_device(nullptr);
    if (st != PATCH_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    // scratch: the losses concatenated | a rank counter per tile
    const size_t off_rank = round_up(sizeof(double) * static_cast<size_t>(total), 256);
    const size_t bytes = off_rank + sizeof(int32_t) * static_cast<size_t>(total);
    cudaMemPool_t pool = nullptr;
    cudaError_t e = patchk::device_pool(&pool);
    if (e != cudaSuccess) return from_cuda(e);
    uint8_t *scratch = nullptr;
    e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&scratch), bytes, pool, stream);
    if (e != cudaSuccess) return from_cuda(e);
    double *cat = reinterpret_cast<double *>(scratch);
    int32_t *rank = reinterpret_cast<int32_t *>(scratch + off_rank);
    int64_t off = 0;
    for (int32_t m = 0; m < count && e == cudaSuccess; ++m) {
        e = cudaMemcpyAsync(cat + off, losses[m], sizeof(double) * static_cast<size_t>(n_tiles[m]),
                            cudaMemcpyDeviceToDevice, stream);
        off += n_tiles[m];
    }
    if (e == cudaSuccess) e = cudaMemsetAsync(rank, 0, sizeof(int32_t) * static_cast<size_t>(total), stream);
    if (e == cudaSuccess) {
        const int64_t n_sp = static_cast<int64_t>(floor(fraction * static_cast<double>(total)));
        e = patchk::launch_select_maps_global(cat, n_tiles, count, n_sp, rank, maps_out, stream);
    }
    cudaError_t e2 = cudaFreeAsync(scratch, stream);
    return from_cuda(e != cudaSuccess ? e : e2);
}

uint64_t patch_launch_count(void) { return patchk::g_launches.load(std::memory_order_relaxed); }

void patch_test_stall_first_kstep(int32_t on) { g_test_stall.store(on ? 1 : 0, std::memory_order_relaxed); }

void patch_test_prefill_kernel(int32_t which) {
    g_test_kernel.store((which >= 0 && which <= 4) ? which : 0, std::memory_order_relaxed);
}

// Up to kPlanMaxGroup matrices packed with one wait: every handle is made and
// its plan launched (one plan launch for all), the plans are read back in one
// wait, then every packed buffer is allocated and packed.  On an error no
// handle is left: those made so far are freed and every out[i] is null.
static patch_status pack_group_impl(const void *const *Ws, const uint32_t *const *metas,
                                    const uint32_t *const *maps, const patch_shape *shps, int count,
                                    patch_packed **outs, size_t *packed_bytes, void *stream_v, int pattern) {
    if (!outs || count < 1 || count > patchk::kPlanMaxGroup) return PATCH_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i) outs[i] = nullptr;
    if (!Ws || !metas || !maps || !shps) return PATCH_ERR_INVALID_ARG;
    // every argument is checked before anything is allocated
    for (int i = 0; i < count; ++i) {
        const patch_status st = check_shape(shps[i]);
        if (st != PATCH_OK) return st;
        if (shps[i].N % kBand != 0 || shps[i].K % (2 * kStep) != 0) return PATCH_ERR_INVALID_ARG;
        if (shps[i].K > 28672) return PATCH_ERR_INVALID_ARG;  // one segment's table must fit on chip
        if (!Ws[i] || !metas[i] || !maps[i] || !aligned16(Ws[i])) return PATCH_ERR_INVALID_ARG;
    }
    int num_sms = 0;
    patch_status st = check_device(&num_sms);
    if (st != PATCH_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);

    patch_packed *hs[patchk::kPlanMaxGroup] = {};
    patchk::PlanArgs pa[patchk::kPlanMaxGroup];
    const patchk::PackPlan *plan_dev[patchk::kPlanMaxGroup];
    const int64_t *prefix_dev[patchk::kPlanMaxGroup];
    std::vector<int64_t> *prefix_host[patchk::kPlanMaxGroup];
    auto fail = [&](patch_status why) {
        for (int i = 0; i < count; ++i)
            if (hs[i]) patch_free(hs[i], stream_v);
        return why;
    };
    for (int i = 0; i < count; ++i) {
        const patch_shape shp = shps[i];
        const int64_t N = shp.N, K = shp.K;
        const int64_t bands = N / kBand, nsteps = K / kStep, Q = nsteps / 2;
        patch_packed *h = new (std::nothrow) patch_packed();
        if (!h) return fail(PATCH_ERR_OOM);
        hs[i] = h;
        cudaGetDevice(&h->device);
        h->pattern = pattern;
        h->shp = shp;
        h->num_sms = num_sms;
        h->bands = bands;
        patchk::plan_decode_chunks(bands, nsteps, num_sms, &h->dec_cp, &h->dec_cpb, &h->dec_nchunks);
        h->workspace_bytes = patchk::decode_workspace_bytes(h->dec_nchunks);

        // The layout is planned on the device from the map (no map read-back,
        // no table upload); only the plan summary comes back, to size the
        // packed buffer.  Allocation 1: table | chunk descriptors | k-pair
        // prefix | band starts | plan | workspace | status.  Allocation 2: the
        // packed bytes.
        const size_t off_table = 0;
        const size_t off_chunks = off_table + sizeof(uint64_t) * static_cast<size_t>(bands * nsteps);
        const size_t off_prefix = round_up(off_chunks + sizeof(uint64_t) * static_cast<size_t>(h->dec_nchunks), 256);
        const size_t off_bstart = round_up(off_prefix + sizeof(int64_t) * static_cast<size_t>(bands * (Q + 1)), 256);
        const size_t off_ptable = round_up(off_bstart + sizeof(uint64_t) * static_cast<size_t>(bands), 256);
        const size_t off_sstart = round_up(off_ptable + sizeof(uint64_t) * static_cast<size_t>(bands * nsteps), 256);
        const size_t off_plan = round_up(off_sstart + sizeof(uint64_t) * static_cast<size_t>(bands), 256);
        const size_t off_ws = round_up(off_plan + sizeof(patchk::PackPlan), 256);
        const size_t off_status = round_up(off_ws + h->workspace_bytes, 256);
        const size_t status_bytes = sizeof(uint32_t) * patchk::kStatusWords;
        const size_t total = off_status + status_bytes;
        cudaError_t e = patchk::device_pool(&h->pool);
        if (e == cudaSuccess)
            e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&h->base), total, h->pool, stream);
        if (e != cudaSuccess) return fail(from_cuda(e));
        h->table = reinterpret_cast<uint64_t *>(h->base + off_table);
        h->chunk_desc = reinterpret_cast<uint64_t *>(h->base + off_chunks);
        h->pair_prefix_dev = reinterpret_cast<int64_t *>(h->base + off_prefix);
        h->ptable = reinterpret_cast<uint64_t *>(h->base + off_ptable);
        patchk::PackPlan *pd = reinterpret_cast<patchk::PackPlan *>(h->base + off_plan);
        h->workspace = reinterpret_cast<float *>(h->base + off_ws);
        // status word | (unused) | ready flag | decode chunk counter
        // (zeroed by the plan launch, before any kernel reads them)
        h->status = reinterpret_cast<uint32_t *>(h->base + off_status);
        pa[i] = patchk::PlanArgs{maps[i], N, K, static_cast<int>(shp.tile_n), static_cast<int>(shp.tile_k),
                                 h->dec_cp, h->dec_cpb, h->table, h->chunk_desc, h->pair_prefix_dev,
                                 reinterpret_cast<uint64_t *>(h->base + off_bstart), h->ptable,
                                 reinterpret_cast<uint64_t *>(h->base + off_sstart), pd, pattern, h->status};
        plan_dev[i] = pd;
        prefix_dev[i] = h->pair_prefix_dev;
        h->pair_prefix.assign(static_cast<size_t>(bands * (Q + 1)), 0);
        prefix_host[i] = &h->pair_prefix;
    }
    cudaError_t e = patchk::launch_plan_pack_group(pa, count, stream);
    preload_gemm_kernels();  // this call waits for the device below in any case
    patchk::PackPlan plans[patchk::kPlanMaxGroup];
    if (e == cudaSuccess) e = read_plans(plan_dev, plans, prefix_dev, prefix_host, count, stream);
    if (e != cudaSuccess) return fail(from_cuda(e));
    for (int i = 0; i < count; ++i) {
        patch_packed *h = hs[i];
        const patchk::PackPlan &plan = plans[i];
        h->packed_bytes = static_cast<size_t>(plan.packed_bytes);
        h->side_bytes = static_cast<size_t>(plan.side_bytes);
        if (plan.packed_bytes >= (1ull << 40) || plan.packed_bytes + plan.side_bytes >= (1ull << 47))
            return fail(PATCH_ERR_UNSUPPORTED);  // chunk descriptors hold 40-bit offsets, table entries 48-bit ones
        h->sparse_ksteps = static_cast<int64_t>(plan.sparse_ksteps);
        h->meta_blocks = static_cast<int64_t>(plan.meta_blocks);
        h->duo_ok = plan.duo_ok ? 1 : 0;
        h->max_pair_bytes = static_cast<int>(plan.pair_max_bytes);
        h->chunk_desc_host.assign(plan.first_desc,
                                  plan.first_desc + std::min<int64_t>(h->dec_nchunks, 2 * patchk::kDecMaxCtas));
        e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&h->packed),
                                    std::max<size_t>(h->packed_bytes + h->side_bytes, 16), h->pool, stream);
        if (e == cudaSuccess)
            e = patchk::launch_pack(Ws[i], metas[i], maps[i], h->shp.N, h->shp.K, static_cast<int>(h->shp.tile_n),
                                    static_cast<int>(h->shp.tile_k), h->table, h->side_bytes ? h->ptable : nullptr,
                                    h->packed, stream, pattern);
        if (e != cudaSuccess) return fail(from_cuda(e));
    }
    // every handle's ready flag (status word 2), once all the packs above completed
    uint32_t *ready[patchk::kPlanMaxGroup];
    for (int i = 0; i < count; ++i) ready[i] = hs[i]->status + 2;
    e = patchk::launch_publish_ready(ready, count, stream);
    if (e != cudaSuccess) return fail(from_cuda(e));
    for (int i = 0; i < count; ++i) {
        if (packed_bytes) packed_bytes[i] = hs[i]->packed_bytes;
        outs[i] = hs[i];
    }
    return PATCH_OK;
}

static patch_status pack_impl(const void *W_bf16, const uint32_t *meta, const uint32_t *map,
                              patch_shape shp, patch_packed **out, size_t *packed_bytes,
                              void *stream_v, int pattern) {
    if (!out) return PATCH_ERR_INVALID_ARG;
    return pack_group_impl(&W_bf16, &meta, &map, &shp, 1, out, packed_bytes, stream_v, pattern);
}

patch_status patch_pack(const void *W_bf16, const uint32_t *meta, const uint32_t *map,
                        patch_shape shp, patch_packed **out, size_t *packed_bytes, void *stream_v) {
    return pack_impl(W_bf16, meta, map, shp, out, packed_bytes, stream_v, 2);
}

patch_status patch_pack_group(const void *const *Ws_bf16, const uint32_t *const *metas,
                              const uint32_t *const *maps, const patch_shape *shps, int32_t count,
                              patch_packed **outs, size_t *packed_bytes, void *stream_v) {
    return pack_group_impl(Ws_bf16, metas, maps, shps, count, outs, packed_bytes, stream_v, 2);
}

patch_status patch_pack_nm(const void *W_bf16, const uint32_t *meta, const uint32_t *map,
                           patch_shape shp, int32_t n_keep, int32_t m_group, patch_packed **out,
                           size_t *packed_bytes, void *stream_v) {
    if (out) *out = nullptr;
    const int pattern = pattern_of(n_keep, m_group);
    if (!pattern) return PATCH_ERR_UNSUPPORTED;
    return pack_impl(W_bf16, meta, map, shp, out, packed_bytes, stream_v, pattern);
}

patch_status patch_quantize_fp8(const void *X_bf16, int64_t R, int64_t C, uint8_t *codes_out,
                                float *scales_out, void *stream_v) {
    if (!X_bf16 || !codes_out || !scales_out || R < 1 || C < 8 || C % 8 != 0 || !aligned16(X_bf16) ||
        (reinterpret_cast<uintptr_t>(codes_out) & 7u) != 0 || R > 0x7FFFFFFF)
        return PATCH_ERR_INVALID_ARG;
    patch_status st = check_device(nullptr);
    if (st != PATCH_OK) return st;
    return from_cuda(patchk::launch_fp8_quantize_rows(X_bf16, R, C, codes_out, scales_out,
                                                      static_cast<cudaStream_t>(stream_v)));
}

// Decode-sized FP8 calls quantise X into the handle's own scratch (no pool
// allocation on the call); larger ones take a pool block for the call.
constexpr int64_t kFp8ScratchRows = 64;
static size_t fp8_xscratch_bytes(int64_t rows, int64_t K) {
    return round_up(static_cast<size_t>(rows * K), 256) + sizeof(float) * static_cast<size_t>(rows);
}

patch_status patch_pack_fp8(const void *W_bf16, const uint32_t *meta, const uint32_t *map,
                            patch_shape shp, patch_packed **out, size_t *packed_bytes,
                            void *stream_v) {
    if (!out) return PATCH_ERR_INVALID_ARG;
    *out = nullptr;
    patch_status st = check_shape(shp);
    if (st != PATCH_OK) return st;
    if (shp.N % kBand != 0 || shp.K % 128 != 0 || shp.K > 28672) return PATCH_ERR_INVALID_ARG;
    if (!W_bf16 || !meta || !map || !aligned16(W_bf16) || !aligned16(meta)) return PATCH_ERR_INVALID_ARG;
    int num_sms = 0;
    st = check_device(&num_sms);
    if (st != PATCH_OK) return st;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    const int64_t N = shp.N, K = shp.K, tn = shp.tile_n, tk = shp.tile_k;
    const int64_t bands = N / kBand, steps = K / 128, tiles_k = K / tk;
    const int64_t n_tiles = (N / tn) * tiles_k;
    // the layout is planned on the host from the map (read back in the one
    // wait of this call): a k-step is 2:4 iff every tile it overlaps is
    std::vector<uint32_t> hmap(static_cast<size_t>((n_tiles + 31) / 32));
    preload_gemm_kernels();  // this call waits for the device below in any case
    cudaError_t e = cudaMemcpyAsync(hmap.data(), map, sizeof(uint32_t) * hmap.size(), cudaMemcpyDeviceToHost,
                                    stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return from_cuda(e);
    auto sparse_tile = [&](int64_t t) { return (hmap[static_cast<size_t>(t / 32)] >> (t % 32)) & 1u; };
    std::vector<uint64_t> table(static_cast<size_t>(bands * steps));
    uint64_t off = 0, n_sparse = 0;
    for (int64_t b = 0; b < bands; ++b)
        for (int64_t c = 0; c < steps; ++c) {
            bool sp = true;
            for (int64_t ti = (b * kBand) / tn; ti <= (b * kBand + kBand - 1) / tn; ++ti)
                for (int64_t tj = (c * 128) / tk; tj <= (c * 128 + 127) / tk; ++tj)
                    if (!sparse_tile(ti * tiles_k + tj)) sp = false;
            if (sp) {
                table[static_cast<size_t>(b * steps + c)] = (off + patchk::kMetaBlockBytes) | patchk::kEntrySparse;
                off += patchk::kMetaBlockBytes + patchk::kSparseStepBytes;
                ++n_sparse;
            } else {
                table[static_cast<size_t>(b * steps + c)] = off;
                off += patchk::kDenseStepBytes;
            }
        }
    // prefill table for the two-SM kernel (even band counts): bands 2p and
    // 2p+1 take the same kind at every k-step; where one is 2:4 and the other
    // dense, the 2:4 band's k-step gets a dense side copy of its W_eff codes
    // after the packed bytes
    const bool duo = bands % 2 == 0;
    std::vector<uint64_t> ptable(duo ? table.size() : 0);
    uint64_t side = 0;
    if (duo)
        for (int64_t bp = 0; bp < bands / 2; ++bp)
            for (int64_t c = 0; c < steps; ++c) {
                const size_t i0 = static_cast<size_t>(2 * bp * steps + c), i1 = i0 + static_cast<size_t>(steps);
                ptable[i0] = table[i0];
                ptable[i1] = table[i1];
                const bool s0 = (table[i0] & patchk::kEntrySparse) != 0, s1 = (table[i1] & patchk::kEntrySparse) != 0;
                if (s0 != s1) {
                    ptable[s0 ? i0 : i1] = (off + side) | patchk::kEntrySide;
                    side += patchk::kDenseStepBytes;
                }
            }
    // split-K chunks for decode token counts (an even k-step count: two
    // 128-column k-steps per pair): per chunk the first byte (a 2:4 k-step's
    // metadata block precedes it), each k-step's 2:4 flag and the pair count
    int dec_cp = 0, dec_cpb = 0, dec_nchunks = 0;
    std::vector<uint64_t> chunk_desc;
    if (steps % 2 == 0) {
        patchk::plan_decode_chunks(bands, steps, num_sms, &dec_cp, &dec_cpb, &dec_nchunks);
        chunk_desc.resize(static_cast<size_t>(dec_nchunks));
        const int64_t Q = steps / 2;
        for (int64_t b = 0; b < bands; ++b)
            for (int64_t q = 0; q < dec_cpb; ++q) {
                const int64_t pr0 = q * dec_cp, np = std::min<int64_t>(dec_cp, Q - pr0);
                const uint64_t e0 = table[static_cast<size_t>(b * steps + 2 * pr0)];
                const uint64_t first = (e0 & patchk::kEntryOffsetMask) -
                                       ((e0 & patchk::kEntrySparse) ? patchk::kMetaBlockBytes : 0);
                uint64_t flags = 0;
                for (int64_t i = 0; i < 2 * np; ++i)
                    if (table[static_cast<size_t>(b * steps + 2 * pr0 + i)] & patchk::kEntrySparse) flags |= 1ull << i;
                chunk_desc[static_cast<size_t>(b * dec_cpb + q)] =
                    (first & ((1ull << 40) - 1)) | (flags << 40) | (static_cast<uint64_t>(np) << 56);
            }
        if (off >= (1ull << 40)) dec_nchunks = 0;  // descriptors hold 40-bit offsets
    }
    patch_packed *h = new (std::nothrow) patch_packed();
    if (!h) return PATCH_ERR_OOM;
    cudaGetDevice(&h->device);
    h->pattern = 8;
    h->shp = shp;
    h->num_sms = num_sms;
    h->bands = bands;
    h->packed_bytes = off;
    h->side_bytes = side;
    h->duo_ok = duo ? 1 : 0;
    h->sparse_ksteps = static_cast<int64_t>(n_sparse);
    h->meta_blocks = static_cast<int64_t>(n_sparse);
    // allocation 1: table | prefill table | row scales | X scratch of
    // decode-sized calls | status; allocation 2: the packed bytes, then the
    // side copies
    const size_t ws_bytes = dec_nchunks ? patchk::decode_workspace_bytes(dec_nchunks) : 0;
    const size_t off_ptable = round_up(sizeof(uint64_t) * table.size(), 256);
    const size_t off_scale = round_up(off_ptable + sizeof(uint64_t) * ptable.size(), 256);
    const size_t off_xs = round_up(off_scale + sizeof(float) * static_cast<size_t>(N), 256);
    const size_t off_chunks = round_up(off_xs + fp8_xscratch_bytes(kFp8ScratchRows, K), 256);
    const size_t off_ws = round_up(off_chunks + sizeof(uint64_t) * chunk_desc.size(), 256);
    const size_t off_status = round_up(off_ws + ws_bytes, 256);
    const size_t total = off_status + 256;
    e = patchk::device_pool(&h->pool);
    if (e == cudaSuccess) e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&h->base), total, h->pool, stream);
    if (e != cudaSuccess) {
        delete h;
        return from_cuda(e);
    }
    h->table = reinterpret_cast<uint64_t *>(h->base);
    h->ptable = duo ? reinterpret_cast<uint64_t *>(h->base + off_ptable) : nullptr;
    h->fp8_scale = reinterpret_cast<float *>(h->base + off_scale);
    h->fp8_xscratch = h->base + off_xs;
    h->status = reinterpret_cast<uint32_t *>(h->base + off_status);
    if (dec_nchunks) {
        h->dec_cp = dec_cp;
        h->dec_cpb = dec_cpb;
        h->dec_nchunks = dec_nchunks;
        h->chunk_desc = reinterpret_cast<uint64_t *>(h->base + off_chunks);
        h->chunk_desc_host.assign(chunk_desc.begin(),
                                  chunk_desc.begin() + std::min<int64_t>(dec_nchunks, 2 * patchk::kDecMaxCtas));
        h->workspace = reinterpret_cast<float *>(h->base + off_ws);
        h->workspace_bytes = ws_bytes;
    }
    e = cudaMemsetAsync(h->status, 0, 256, stream);
    if (e == cudaSuccess)
        e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&h->packed), std::max<size_t>(off + side, 16),
                                    h->pool, stream);
    // pageable sources: the call returns once the tables have been staged
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(h->table, table.data(), sizeof(uint64_t) * table.size(), cudaMemcpyHostToDevice,
                            stream);
    if (e == cudaSuccess && duo)
        e = cudaMemcpyAsync(h->ptable, ptable.data(), sizeof(uint64_t) * ptable.size(), cudaMemcpyHostToDevice,
                            stream);
    if (e == cudaSuccess && dec_nchunks)
        e = cudaMemcpyAsync(h->chunk_desc, chunk_desc.data(), sizeof(uint64_t) * chunk_desc.size(),
                            cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess)
        e = patchk::launch_pack_fp8(W_bf16, meta, map, N, K, static_cast<int>(tn), static_cast<int>(tk),
                                    h->table, h->ptable, h->fp8_scale, h->packed, h->status + 2, stream);
    if (e != cudaSuccess) {
        patch_free(h, stream_v);
        return from_cuda(e);
    }
    if (packed_bytes) *packed_bytes = h->packed_bytes;
    *out = h;
    return PATCH_OK;
}

patch_status patch_packed_fp8_scales(const patch_packed *Wp, float *scales_dst, void *stream_v) {
    if (!Wp || !scales_dst || Wp->pattern != 8) return PATCH_ERR_INVALID_ARG;
    return from_cuda(cudaMemcpyAsync(scales_dst, Wp->fp8_scale, sizeof(float) * static_cast<size_t>(Wp->shp.N),
                                     cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream_v)));
}

// The split-K launch description of one FP8 handle's product on X codes xq
// with token scales sx.
static patchk::GemmLaunch fp8_split_launch(const patch_packed *Wp, const uint8_t *xq, const float *sx, int64_t M,
                                           void *Y, int32_t y_is_fp32) {
    patchk::GemmLaunch g = {};
    g.packed = Wp->packed;
    g.table = Wp->table;
    g.N = Wp->shp.N;
    g.K = Wp->shp.K;
    g.X = xq;
    g.M = M;
    g.Y = Y;
    g.y_fp32 = y_is_fp32;
    g.workspace = Wp->workspace;
    g.workspace_bytes = Wp->workspace_bytes;
    g.pool = Wp->pool;
    g.status = Wp->status;
    g.ready = Wp->status + 2;  // raised once the pack's kernels have completed
    g.counter = Wp->status + 3;
    g.chunk_desc = Wp->chunk_desc;
    g.chunk_desc_host = Wp->chunk_desc_host.data();
    g.dec_cp = Wp->dec_cp;
    g.dec_cpb = Wp->dec_cpb;
    g.dec_nchunks = Wp->dec_nchunks;
    g.num_sms = Wp->num_sms;
    g.stall_first_kstep = g_test_stall.load(std::memory_order_relaxed);
    g.f8_sw = Wp->fp8_scale;
    g.f8_sx = sx;
    return g;
}

// the launch description of one FP8 handle's product on quantised X
static patchk::Fp8Launch fp8_launch(const patch_packed *Wp, const uint8_t *xq, const float *sx, int64_t M,
                                    void *Y, int32_t y_is_fp32) {
    patchk::Fp8Launch g;
    g.packed = Wp->packed;
    g.table = Wp->table;
    g.ptable = Wp->ptable;
    g.packed_bytes = Wp->packed_bytes + Wp->side_bytes;
    g.all_sparse = Wp->sparse_ksteps == Wp->bands * (Wp->shp.K / 128) ? 1 : 0;
    g.force_kernel = g_test_kernel.load(std::memory_order_relaxed);
    g.sw = Wp->fp8_scale;
    g.xq = xq;
    g.sx = sx;
    g.N = Wp->shp.N;
    g.K = Wp->shp.K;
    g.M = M;
    g.Y = Y;
    g.y_fp32 = y_is_fp32;
    g.status = Wp->status;
    g.num_sms = Wp->num_sms;
    g.pool = Wp->pool;
    return g;
}

static patch_status fp8_gemm(const patch_packed *Wp, const void *X_bf16, int64_t M, void *Y,
                             int32_t y_is_fp32, cudaStream_t stream) {
    const int64_t K = Wp->shp.K;
    // the activations' codes and token scales
    const size_t off_sx = round_up(static_cast<size_t>(M * K), 256);
    const size_t bytes = off_sx + sizeof(float) * static_cast<size_t>(M);
    uint8_t *ws = nullptr;
    const bool own = M <= kFp8ScratchRows && Wp->fp8_xscratch;
    cudaError_t e = cudaSuccess;
    if (own)
        ws = Wp->fp8_xscratch;
    else
        e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), bytes, Wp->pool, stream);
    if (e != cudaSuccess) return from_cuda(e);
    float *sx = reinterpret_cast<float *>(ws + off_sx);
    e = patchk::launch_fp8_quantize_rows(X_bf16, M, K, ws, sx, stream);
    const int force = g_test_kernel.load(std::memory_order_relaxed);
    if (e == cudaSuccess && M <= patchk::kDecodeMaxM && Wp->dec_nchunks > 0 && force == 0) {
        // decode token counts: the split-K kernel on the e4m3 codes, the weights
        // read once over every SM; the fix-up applies the row and token scales
        const patchk::GemmLaunch g = fp8_split_launch(Wp, ws, sx, M, Y, y_is_fp32);
        e = patchk::launch_decode_f8(&g, 1, stream);
    } else if (e == cudaSuccess) {
        e = patchk::launch_fp8_gemm(fp8_launch(Wp, ws, sx, M, Y, y_is_fp32), stream);
    }
    const cudaError_t e2 = own ? cudaSuccess : cudaFreeAsync(ws, stream);
    return from_cuda(e != cudaSuccess ? e : e2);
}

// the launch description of one bf16 handle's product
static patchk::GemmLaunch gemm_launch(const patch_packed *Wp, const void *X_bf16, int64_t M, void *Y,
                                      int32_t y_is_fp32) {
    patchk::GemmLaunch g;
    g.packed = Wp->packed;
    g.table = Wp->table;
    g.N = Wp->shp.N;
    g.K = Wp->shp.K;
    g.X = X_bf16;
    g.M = M;
    g.Y = Y;
    g.y_fp32 = y_is_fp32;
    g.workspace = Wp->workspace;
    g.workspace_bytes = Wp->workspace_bytes;
    g.pool = Wp->pool;
    g.status = Wp->status;
    g.ready = Wp->status + 2;
    g.counter = Wp->status + 3;
    g.chunk_desc = Wp->chunk_desc;
    g.chunk_desc_host = Wp->chunk_desc_host.data();
    g.dec_cp = Wp->dec_cp;
    g.dec_cpb = Wp->dec_cpb;
    g.dec_nchunks = Wp->dec_nchunks;
    g.packed_rows = (Wp->packed_bytes + Wp->side_bytes) / 128;
    g.ptable = Wp->ptable;
    g.duo_ok = Wp->duo_ok;
    g.max_pair_bytes = Wp->max_pair_bytes;
    g.num_sms = Wp->num_sms;
    // the stream-K balance of the prefill kernels uses the k-pair prefix,
    // read back once by patch_pack: nothing here waits for the device
    g.pair_prefix = Wp->pair_prefix.empty() ? nullptr : Wp->pair_prefix.data();
    g.stall_first_kstep = g_test_stall.load(std::memory_order_relaxed);
    g.force_kernel = g_test_kernel.load(std::memory_order_relaxed);
    g.pattern = Wp->pattern;
    return g;
}

patch_status patch_hybrid_gemm(const patch_packed *Wp, const void *X_bf16, int64_t M, void *Y,
                               int32_t y_is_fp32, void *stream_v) {
    if (!Wp || M < 0) return PATCH_ERR_INVALID_ARG;
    if (M == 0) return PATCH_OK;  // empty batch: nothing to do
    if (!X_bf16 || !Y) return PATCH_ERR_INVALID_ARG;
    if (!aligned16(X_bf16) || !aligned16(Y)) return PATCH_ERR_INVALID_ARG;
    if (y_is_fp32 != 0 && y_is_fp32 != 1) return PATCH_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31)) return PATCH_ERR_INVALID_ARG;
    if (Wp->pattern == 8) return fp8_gemm(Wp, X_bf16, M, Y, y_is_fp32, static_cast<cudaStream_t>(stream_v));
    const patchk::GemmLaunch g = gemm_launch(Wp, X_bf16, M, Y, y_is_fp32);
    return from_cuda(patchk::launch_hybrid_gemm(g, static_cast<cudaStream_t>(stream_v)));
}

patch_status patch_hybrid_gemm_group(const patch_packed *const *Wps, int32_t count, const void *X_bf16,
                                     int64_t M, void *const *Ys, int32_t y_is_fp32, void *stream_v) {
    if (!Wps || !Ys || count < 1 || count > patchk::kDecMaxGroup || M < 0) return PATCH_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i)
        if (!Wps[i]) return PATCH_ERR_INVALID_ARG;
    if (M == 0) return PATCH_OK;
    if (!X_bf16 || !aligned16(X_bf16)) return PATCH_ERR_INVALID_ARG;
    for (int i = 0; i < count; ++i)
        if (!Ys[i] || !aligned16(Ys[i])) return PATCH_ERR_INVALID_ARG;
    if (y_is_fp32 != 0 && y_is_fp32 != 1) return PATCH_ERR_INVALID_ARG;
    if (M > (int64_t(1) << 31)) return PATCH_ERR_INVALID_ARG;
    const int64_t K = Wps[0]->shp.K;
    const int force = g_test_kernel.load(std::memory_order_relaxed);
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    // FP8 handles: X is quantised once (into the first handle's scratch) and
    // the group's products run as one split-K launch on the codes
    bool f8_group = count > 1 && M <= kFp8ScratchRows && M <= patchk::kDecodeMaxM && force == 0;
    for (int i = 0; i < count && f8_group; ++i)
        f8_group = Wps[i]->pattern == 8 && Wps[i]->shp.K == K && Wps[i]->dec_nchunks > 0 &&
                   Wps[i]->num_sms == Wps[0]->num_sms && Wps[0]->fp8_xscratch;
    if (f8_group) {
        uint8_t *xq = Wps[0]->fp8_xscratch;
        float *sx = reinterpret_cast<float *>(xq + round_up(static_cast<size_t>(M * K), 256));
        cudaError_t e = patchk::launch_fp8_quantize_rows(X_bf16, M, K, xq, sx, stream);
        if (e != cudaSuccess) return from_cuda(e);
        patchk::GemmLaunch gs[patchk::kDecMaxGroup];
        for (int i = 0; i < count; ++i) gs[i] = fp8_split_launch(Wps[i], xq, sx, M, Ys[i], y_is_fp32);
        return from_cuda(patchk::launch_decode_f8(gs, count, stream));
    }
    if (count > 1 && M > 128 && (force == 0 || force == 3)) {
        // FP8 prefill: X quantised once, then one two-SM launch over every
        // matrix's band pairs when the estimate says it finishes first
        const int64_t steps = K / 128;
        bool ok = steps % 2 == 0 && steps <= 224;
        bool all_sparse = true;
        int64_t sum_n = 0;
        double own = 0;
        for (int i = 0; i < count && ok; ++i) {
            const patch_packed *h = Wps[i];
            ok = h->pattern == 8 && h->shp.K == K && h->ptable && (h->shp.N / 128) % 2 == 0 &&
                 h->num_sms == Wps[0]->num_sms;
            if (!ok) break;
            const bool sp = h->sparse_ksteps == h->bands * steps;
            all_sparse = all_sparse && sp;
            sum_n += h->shp.N;
            const patchk::DuoFp8Plan one = patchk::plan_duo_fp8(h->shp.N, M, h->num_sms, sp);
            ok = one.bn > 0;
            own += one.cost;
        }
        patchk::DuoFp8Plan dp{};
        if (ok) dp = patchk::plan_duo_fp8(sum_n, M, Wps[0]->num_sms, all_sparse);
        if (ok && dp.bn > 0 && (force == 3 || dp.cost <= own)) {
            const size_t off_sx = round_up(static_cast<size_t>(M * K), 256);
            uint8_t *ws = nullptr;
            cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws),
                                                    off_sx + sizeof(float) * static_cast<size_t>(M),
                                                    Wps[0]->pool, stream);
            if (e != cudaSuccess) return from_cuda(e);
            float *sx = reinterpret_cast<float *>(ws + off_sx);
            e = patchk::launch_fp8_quantize_rows(X_bf16, M, K, ws, sx, stream);
            if (e == cudaSuccess) {
                patchk::Fp8Launch gs[patchk::kDecMaxGroup];
                for (int i = 0; i < count; ++i) gs[i] = fp8_launch(Wps[i], ws, sx, M, Ys[i], y_is_fp32);
                e = patchk::launch_duo_fp8_group(gs, count, dp, stream);
            }
            const cudaError_t e2 = cudaFreeAsync(ws, stream);
            return from_cuda(e != cudaSuccess ? e : e2);
        }
    }
    if (count > 1 && M > 128 && !patchk::takes_split_k(M, K, force)) {
        // prefill: one two-SM launch over every matrix's band pairs when the
        // estimate says it finishes first (fills the SMs that one matrix's
        // items leave idle in its last wave)
        bool same = true;
        for (int i = 0; i < count && same; ++i) same = Wps[i]->shp.K == K;
        if (same) {
            patchk::GemmLaunch gs[patchk::kDecMaxGroup];
            for (int i = 0; i < count; ++i) gs[i] = gemm_launch(Wps[i], X_bf16, M, Ys[i], y_is_fp32);
            patchk::DuoPlan dp;
            if (patchk::plan_hybrid_group(gs, count, &dp)) return from_cuda(patchk::launch_duo_group(gs, count, dp, stream));
        }
    }
    bool one_launch = count > 1 && patchk::takes_split_k(M, K, force);
    for (int i = 0; i < count && one_launch; ++i)
        one_launch = Wps[i]->pattern == 2 && Wps[i]->shp.K == K && Wps[i]->num_sms == Wps[0]->num_sms;
    if (!one_launch) {
        // the products one after another on the stream (the same results)
        for (int i = 0; i < count; ++i) {
            const patch_status st = patch_hybrid_gemm(Wps[i], X_bf16, M, Ys[i], y_is_fp32, stream_v);
            if (st != PATCH_OK) return st;
        }
        return PATCH_OK;
    }
    patchk::GemmLaunch gs[patchk::kDecMaxGroup];
    for (int i = 0; i < count; ++i) gs[i] = gemm_launch(Wps[i], X_bf16, M, Ys[i], y_is_fp32);
    return from_cuda(patchk::launch_decode_group(gs, count, stream));
}

void patch_free(patch_packed *Wp, void *stream_v) {
    if (!Wp) return;
    if (Wp->packed) cudaFreeAsync(Wp->packed, static_cast<cudaStream_t>(stream_v));
    if (Wp->base) cudaFreeAsync(Wp->base, static_cast<cudaStream_t>(stream_v));
    delete Wp;
}

patch_status patch_get_status(const patch_packed *Wp) {
    if (!Wp) return PATCH_ERR_INVALID_ARG;
    uint32_t word = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(&word, Wp->status, sizeof(word), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && word != 0) e = cudaMemset(Wp->status, 0, sizeof(uint32_t));
    // a call that gave up may have left decode chunks claimed
    if (e == cudaSuccess && word != 0) e = cudaMemset(Wp->status + 3, 0, sizeof(uint32_t));
    if (e != cudaSuccess) return from_cuda(e);
    return (word & patchk::kStatusTimeout) ? PATCH_ERR_TIMEOUT : PATCH_OK;
}

patch_status patch_packed_info(const patch_packed *Wp, patch_packed_view *view) {
    if (!Wp || !view) return PATCH_ERR_INVALID_ARG;
    view->packed = Wp->packed;
    view->table = Wp->table;
    view->packed_bytes = Wp->packed_bytes;
    view->N = Wp->shp.N;
    view->K = Wp->shp.K;
    view->tile_n = Wp->shp.tile_n;
    view->tile_k = Wp->shp.tile_k;
    view->sparse_ksteps = Wp->sparse_ksteps;
    view->meta_blocks = Wp->meta_blocks;
    return PATCH_OK;
}

patch_status patch_packed_export(const patch_packed *Wp, void *packed_dst, uint64_t *table_dst,
                                 void *stream_v) {
    if (!Wp) return PATCH_ERR_INVALID_ARG;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_v);
    cudaError_t e = cudaSuccess;
    if (packed_dst && Wp->packed_bytes)
        e = cudaMemcpyAsync(packed_dst, Wp->packed, Wp->packed_bytes, cudaMemcpyDeviceToDevice,
                            stream);
    if (e == cudaSuccess && table_dst)
        e = cudaMemcpyAsync(table_dst, Wp->table,
                            sizeof(uint64_t) * (Wp->shp.N / kBand) *
                                (Wp->shp.K / (Wp->pattern == 8 ? 128 : kStep)),
                            cudaMemcpyDeviceToDevice, stream);
    return from_cuda(e);
}

}  // extern "C"
