// noalloc.cu -- kvc_index_topk_noalloc: the indexer top-K with its scratch in
// a fixed device array inside the library, for callers that cannot allocate.
//
// Some callers cannot call cudaMalloc (or any allocator): a plugin hosted by a
// framework that owns every device allocation and hands the plugin only its
// inputs and outputs, or a latency-critical path where cudaMalloc's implicit
// device-wide synchronisation is not allowed.  This entry point runs the same
// kernels as kvc_index_topk, but its scratch -- the per-entry scores, the
// per-sequence histograms and counters, the candidate lists -- lives in the
// file-scope array below, sized for at most kNoAllocMaxBatch sequences and
// kNoAllocMaxRows = batch x capacity entries.  Every GPU that loads the library
// holds the array (about 10.5 MiB) until the process exits.
#include <mutex>

#include "kvc_internal.cuh"

namespace kvc {
namespace {

constexpr int kNoAllocMaxBatch = 64;
constexpr long long kNoAllocMaxRows = 1ll << 19;
// tiles of the top-K selection over the whole batch: each sequence rounds up
constexpr size_t kMaxTiles = (size_t)(kNoAllocMaxRows / kSelTile) + kNoAllocMaxBatch;
constexpr size_t kScoresBytes = (size_t)kNoAllocMaxRows * 4;
constexpr size_t kCounterBytes = ((size_t)kNoAllocMaxBatch * (kBins + 2) * 4 + 255) / 256 * 256;
constexpr size_t kThrBytes = 512;
constexpr size_t kTileCountBytes = (kMaxTiles * 4 + 255) / 256 * 256;
constexpr size_t kCandBytes = kMaxTiles * kSelTile * 8;
constexpr size_t kScratchBytes = kScoresBytes + kCounterBytes + kThrBytes + kTileCountBytes + kCandBytes;

static __device__ __align__(256) unsigned char g_topk_scratch[kScratchBytes];

// Device address of g_topk_scratch per device.  In host code the symbol's name
// is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress with that device current; it is looked up once per
// device, on the first call made on it, and kept for the life of the process.
// Anything that destroys the device's primary context (cudaDeviceReset, a
// framework tearing the context down) leaves that address dangling: the entry
// point must not be called on that device afterwards.
std::mutex g_mu;
void* g_addr[64] = {};

kvc_status scratch_for_current_device(unsigned char** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KVC_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        int major = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            major != 10)
            return KVC_ERR_DEVICE;
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess || !p) return KVC_ERR_CUDA;
        g_addr[dev] = p;
    }
    *out = static_cast<unsigned char*>(g_addr[dev]);
    return KVC_OK;
}

bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace kvc

using namespace kvc;

extern "C" kvc_status kvc_index_topk_noalloc(const kvc_config* cfg, const int8_t* idx_q,
                                             const kvc_cache* cache, int32_t* topk_idx,
                                             int32_t* scores, uint32_t* dev_status,
                                             void* stream) {
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    if (sh.idx_fmt != 0) return KVC_ERR_UNSUPPORTED;
    if (!cache || !cache->records || !cache->idx_k || !cache->n_entries) return KVC_ERR_INVALID;
    if (cache->batch < 0 || cache->capacity < 0) return KVC_ERR_INVALID;
    if (!aligned_to(cache->idx_k, 16) || !aligned_to(cache->n_entries, 4)) return KVC_ERR_INVALID;
    if (cache->batch == 0) return KVC_OK;
    if (!idx_q || !topk_idx || !aligned_to(idx_q, 16) || !aligned_to(topk_idx, 4))
        return KVC_ERR_INVALID;
    if (scores && !aligned_to(scores, 4)) return KVC_ERR_INVALID;
    // the fixed scratch bounds the problem size
    if (cache->batch > kNoAllocMaxBatch ||
        (long long)cache->batch * cache->capacity > kNoAllocMaxRows)
        return KVC_ERR_CAPACITY;
    unsigned char* ws = nullptr;
    kvc_status st = scratch_for_current_device(&ws);
    if (st != KVC_OK) return st;
    TopkArgs a = {};
    a.idx_q = idx_q;
    a.idx_k = cache->idx_k;
    a.n_entries = cache->n_entries;
    a.batch = cache->batch;
    a.capacity = cache->capacity;
    a.idx_capacity = cache->capacity;
    a.topk = cfg->topk;
    a.di = cfg->idx_dim;
    a.topk_idx = topk_idx;
    a.scores = scores ? scores : reinterpret_cast<int32_t*>(ws);
    unsigned char* p = ws + kScoresBytes;
    // zero when the library loads (a static array); the kernels' last CTAs
    // leave them at zero after every call that did not time out
    a.counters = reinterpret_cast<int32_t*>(p);
    p += kCounterBytes;
    a.thr = reinterpret_cast<int32_t*>(p);
    p += kThrBytes;
    a.tile_count = reinterpret_cast<int32_t*>(p);
    p += kTileCountBytes;
    a.cands = reinterpret_cast<unsigned long long*>(p);
    a.status = dev_status;
    return launch_index_topk(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KVC_OK
                                                                                 : KVC_ERR_CUDA;
}
