// kvc_api.cu -- the C ABI of libkvc.so: argument validation, workspace
// layout, CSA2 layer-group orchestration, tracing and the format codecs.
// Every entry point validates on the host and then only enqueues kernels on
// the caller's stream; nothing here allocates device memory or synchronises.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>
#include <atomic>

#include <nvtx3/nvToolsExt.h>

#include "kvc_internal.cuh"

namespace kvc {

bool derive_shape(const kvc_config* c, Shape* s) {
    if (!c) return false;
    if (c->latent_dim <= 0 || c->latent_dim % 8 || c->rope_dim < 0 || c->rope_dim % 8) return false;
    const int D = c->latent_dim + c->rope_dim;
    if (D > 1024) return false;
    const int G = c->group;
    if (G < 8 || G > 256 || (G & (G - 1)) || c->latent_dim % G) return false;
    if (c->scale_fmt != KVC_SCALE_F32 && c->scale_fmt != KVC_SCALE_UE4M3) return false;
    const int di = c->idx_dim;
    if (di != 16 && di != 32 && di != 64 && di != 128 && di != 256) return false;
    if (c->topk < 1 || c->topk > 2048) return false;
    if (c->window < 0 || c->window > 65536) return false;
    if (c->n_heads < 1 || c->n_heads > 256) return false;
    if (!(c->sm_scale > 0.f) || !(c->sm_scale < 1e30f)) return false;
    if (c->act_dtype != KVC_F32 && c->act_dtype != KVC_BF16) return false;
    if (c->ratio != 0 && c->ratio != 2 && c->ratio != 4) return false;
    if (c->idx_fmt != 0 && c->idx_fmt != 1) return false;
    s->D = D;
    s->Dv = c->latent_dim;
    s->G = G;
    s->lpg = G / 8;
    s->n_groups = (c->latent_dim + G - 1) / G + (c->rope_dim + G - 1) / G;
    s->code_bytes = D / 2;
    s->scale_bytes = c->scale_fmt == KVC_SCALE_UE4M3 ? 1 : 4;
    s->rec_unpadded = s->code_bytes + s->n_groups * s->scale_bytes;
    s->rb = (s->rec_unpadded + 15) / 16 * 16;
    s->act_bytes = c->act_dtype == KVC_BF16 ? 2 : 4;
    s->idx_fmt = c->idx_fmt;
    s->idx_rb = c->idx_fmt == 1 ? di / 2 + di / 16 : di;
    return true;
}

// ------------------------------------------------------------------ tracing
namespace {
struct TraceState {
    std::mutex mu;
    bool on = false;
    int max = 0;
    std::vector<cudaEvent_t> ev;  // 2 per launch
    std::vector<std::string> name;
    int used = 0;
    int open = -1;
};
TraceState& trace() {
    static TraceState t;
    return t;
}
std::atomic<uint64_t> g_launches{0};
}  // namespace

// Inside stream capture a plain event record only marks a dependency; an
// external record becomes a graph node that records the event on replay.
static void record(cudaEvent_t e, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
    else
        cudaEventRecord(e, s);
}

void trace_before(const char* name, cudaStream_t s) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    TraceState& t = trace();
    std::lock_guard<std::mutex> lk(t.mu);
    t.open = -1;
    if (!t.on || t.used >= t.max) return;
    t.open = t.used++;
    t.name[t.open] = name;
    record(t.ev[2 * t.open], s);
}

void trace_after(cudaStream_t s) {
    TraceState& t = trace();
    std::lock_guard<std::mutex> lk(t.mu);
    if (t.open >= 0) record(t.ev[2 * t.open + 1], s);
    t.open = -1;
}

// ------------------------------------------------------------------ codecs
namespace {
__global__ void codec_kernel(const float* __restrict__ x, int64_t n, uint8_t* __restrict__ out,
                             int e4m3) {
    pdl_wait();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = x[i];
        uint32_t r;
        if (e4m3) {
            r = e4m3_from_f32(v);
        } else {
            float w[8] = {fminf(fmaxf(v, -6.f), 6.f), 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            r = e2m1x8_from_f32(w) & 15u;
        }
        out[i] = (uint8_t)r;
    }
}
}  // namespace

cudaError_t launch_fp4_codec(const float* x, int64_t n, uint8_t* out, int e4m3, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    trace_before("fp4_codec", s);
    const cudaError_t e = launch_pdl(codec_kernel, (unsigned)blocks, 256, 0, s, x, n, out, e4m3);
    trace_after(s);
    return e;
}

namespace {
// ------------------------------------------------------------------ workspace
constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct WsLayout {
    size_t scores, counters, thr, tile_count, cands, part_o, part_ml;
    size_t bscore, nblk, pool_blocks, pool_n;  // hierarchical indexer (0 when off)
    size_t total;
};
// hier_blocks > 0 adds the hierarchical indexer's block scores and pool.
WsLayout ws_layout(const kvc_config& c, const Shape& sh, int batch, int cap,
                   int hier_blocks = 0, int hier_block = 0) {
    WsLayout w = {};
    size_t off = 0;
    const size_t tiles = (size_t)batch * sel_tiles(cap);
    w.scores = off;  // int32 scores, or the FP4 keys' candidate slots (as many bytes per tile)
    off = up(off + (c.idx_fmt == 1 ? tiles * kFp4TileCands * 8 : (size_t)batch * cap * 4));
    w.counters = off;  // histograms [B][kBins], finished scan CTAs [B], finished select CTAs [B]
    off = up(off + topk_counter_words(batch) * 4);
    w.thr = off;
    off = up(off + (size_t)batch * 2 * 4);
    w.tile_count = off;
    off = up(off + tiles * 4);
    w.cands = off;
    off = up(off + tiles * kSelTile * 8);
    w.part_o = off;
    off = up(off + (size_t)batch * c.n_heads * kMaxSplit * sh.Dv * 4);
    w.part_ml = off;
    off = up(off + (size_t)batch * c.n_heads * kMaxSplit * 2 * 4);
    if (hier_blocks > 0) {
        const size_t cap_blk = ((size_t)cap + hier_block - 1) / hier_block;
        w.bscore = off;
        off = up(off + (size_t)batch * cap_blk * 4);
        w.nblk = off;
        off = up(off + (size_t)batch * 4);
        w.pool_blocks = off;
        off = up(off + (size_t)batch * hier_blocks * 4);
        w.pool_n = off;
        off = up(off + (size_t)batch * 4);
    }
    w.total = off;
    return w;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool device_ok() {
    static int checked[64] = {};  // 0 unknown, 1 ok, 2 bad
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    if (checked[dev] == 0) {
        int major = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        checked[dev] = major == 10 ? 1 : 2;
    }
    return checked[dev] == 1;
}

kvc_status check_cache(const kvc_cache* cache, const Shape& sh) {
    if (!cache || !cache->records || !cache->idx_k || !cache->n_entries) return KVC_ERR_INVALID;
    if (cache->batch < 0 || cache->capacity < 0) return KVC_ERR_INVALID;
    if (cache->batch > 65535) return KVC_ERR_CAPACITY;  // batch is a grid dimension
    if (!aligned(cache->records, 16) || !aligned(cache->idx_k, 16) || !aligned(cache->n_entries, 4))
        return KVC_ERR_INVALID;
    if ((int64_t)cache->capacity * sh.rb > ((int64_t)1 << 40)) return KVC_ERR_CAPACITY;
    return KVC_OK;
}

// Batched scoring: one block per query holding that query's scores, counters,
// thresholds and candidates (the same regions as the single-query layout).
struct BatchWs {
    size_t scores, counters, thr, tile_count, cands, block;
};
BatchWs batch_ws_layout(int batch, int cap) {
    BatchWs w = {};
    size_t off = 0;
    w.scores = off;
    off = up(off + (size_t)batch * cap * 4);
    w.counters = off;
    off = up(off + topk_counter_words(batch) * 4);
    w.thr = off;
    off = up(off + (size_t)batch * 2 * 4);
    w.tile_count = off;
    off = up(off + (size_t)batch * sel_tiles(cap) * 4);
    w.cands = off;
    off = up(off + (size_t)batch * sel_tiles(cap) * kSelTile * 8);
    w.block = off;
    return w;
}

kvc_status check_ws(void* ws, size_t ws_bytes, const kvc_config& c, const Shape& sh, int batch,
                    int cap, WsLayout* w, int hier_blocks = 0, int hier_block = 0) {
    *w = ws_layout(c, sh, batch, cap, hier_blocks, hier_block);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < w->total) return KVC_ERR_WORKSPACE;
    return KVC_OK;
}

kvc_status run_topk(const kvc_config& c, const int8_t* idx_q, const kvc_cache* cache,
                    int32_t* topk, int32_t* scores, unsigned char* ws, const WsLayout& w,
                    uint32_t* st, cudaStream_t s) {
    if (cache->capacity > kMaxTopkCapacity) return KVC_ERR_CAPACITY;
    if (c.idx_fmt == 1 && scores) return KVC_ERR_UNSUPPORTED;
    TopkArgs a = {};
    a.idx_q = idx_q;
    a.idx_k = cache->idx_k;
    a.n_entries = cache->n_entries;
    a.batch = cache->batch;
    a.capacity = cache->capacity;
    a.idx_capacity = cache->capacity;
    a.topk = c.topk;
    a.di = c.idx_dim;
    a.topk_idx = topk;
    a.scores = scores ? scores : reinterpret_cast<int32_t*>(ws + w.scores);
    a.counters = reinterpret_cast<int32_t*>(ws + w.counters);
    a.thr = reinterpret_cast<int32_t*>(ws + w.thr);
    a.tile_count = reinterpret_cast<int32_t*>(ws + w.tile_count);
    a.cands = reinterpret_cast<unsigned long long*>(ws + w.cands);
    a.status = st;
    if (c.idx_fmt == 1) {  // exact 64-bit scores in the candidate region (unused here)
        const int rb = c.idx_dim / 2 + c.idx_dim / 16;
        return launch_index_topk_fp4(a, rb, reinterpret_cast<long long*>(ws + w.cands), s) ==
                       cudaSuccess
                   ? KVC_OK
                   : KVC_ERR_CUDA;
    }
    return launch_index_topk(a, s) == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

// Hierarchical indexer: the block pool of a Full layer (its scores are in
// the workspace after run_topk).
kvc_status run_block_pool(const kvc_config& c, const kvc_cache* cache, int keep, int block,
                          unsigned char* ws, const WsLayout& w, uint32_t* st, cudaStream_t s) {
    HierArgs h = {};
    h.scores = reinterpret_cast<const int32_t*>(ws + w.scores);
    h.n_entries = cache->n_entries;
    h.batch = cache->batch;
    h.capacity = cache->capacity;
    h.block = block;
    h.keep = keep;
    h.di = c.idx_dim;
    h.bscore = reinterpret_cast<int32_t*>(ws + w.bscore);
    h.nblk = reinterpret_cast<int32_t*>(ws + w.nblk);
    h.pool_blocks = reinterpret_cast<int32_t*>(ws + w.pool_blocks);
    h.pool_n = reinterpret_cast<int32_t*>(ws + w.pool_n);
    h.counters = reinterpret_cast<int32_t*>(ws + w.counters);
    h.thr = reinterpret_cast<int32_t*>(ws + w.thr);
    h.tile_count = reinterpret_cast<int32_t*>(ws + w.tile_count);
    h.cands = reinterpret_cast<unsigned long long*>(ws + w.cands);
    h.status = st;
    return launch_block_pool(h, s) == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

// A Reindex layer over the pool: its indexer query scores the pool's rows only.
kvc_status run_pool_topk(const kvc_config& c, const int8_t* idx_q, const kvc_cache* cache,
                         int keep, int block, int32_t* topk, unsigned char* ws,
                         const WsLayout& w, uint32_t* st, cudaStream_t s) {
    TopkArgs a = {};
    a.idx_q = idx_q;
    a.idx_k = cache->idx_k;
    a.n_entries = reinterpret_cast<const int32_t*>(ws + w.pool_n);
    a.batch = cache->batch;
    a.capacity = (int)std::min<long long>((long long)keep * block, cache->capacity);
    a.idx_capacity = cache->capacity;
    a.topk = c.topk;
    a.di = c.idx_dim;
    a.topk_idx = topk;
    a.scores = reinterpret_cast<int32_t*>(ws + w.scores);
    a.counters = reinterpret_cast<int32_t*>(ws + w.counters);
    a.thr = reinterpret_cast<int32_t*>(ws + w.thr);
    a.tile_count = reinterpret_cast<int32_t*>(ws + w.tile_count);
    a.cands = reinterpret_cast<unsigned long long*>(ws + w.cands);
    a.status = st;
    a.pool_blocks = reinterpret_cast<const int32_t*>(ws + w.pool_blocks);
    a.pool_keep = keep;
    a.pool_block = block;
    return launch_index_topk(a, s) == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}

kvc_status run_attn(const kvc_config& c, const Shape& sh, const void* q, const kvc_cache* cache,
                    const int32_t* topk, const void* window, int window_len, float* out,
                    float* lse, unsigned char* ws, const WsLayout& w, uint32_t* st,
                    cudaStream_t s, int32_t* topk_copy = nullptr,
                    const uint8_t* win_fp8 = nullptr, const float* win_scale = nullptr,
                    bool q_ready = false) {
    AttnArgs a = {};
    a.q_ready = q_ready ? 1 : 0;
    a.topk_copy = topk_copy;
    a.win_fp8 = win_fp8;
    a.win_scale = win_scale;
    a.q = q;
    a.records = static_cast<const uint8_t*>(cache->records);
    a.n_entries = cache->n_entries;
    a.topk_idx = topk;
    a.window = window;
    a.window_len = window_len;
    a.window_stride = c.window;
    a.batch = cache->batch;
    a.capacity = cache->capacity;
    a.out = out;
    a.lse = lse;
    a.part_o = reinterpret_cast<float*>(ws + w.part_o);
    a.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
    a.status = st;
    return launch_attention(c, sh, a, s) == cudaSuccess ? KVC_OK : KVC_ERR_CUDA;
}
}  // namespace

}  // namespace kvc

namespace kvc {
// An NVTX range around every enqueuing entry point, so a profiler's timeline
// shows each C-ABI call over the kernels it launched (free when no tool is
// attached).
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};
}  // namespace kvc

using namespace kvc;

extern "C" {

size_t kvc_record_bytes(const kvc_config* cfg) {
    Shape sh;
    return derive_shape(cfg, &sh) ? (size_t)sh.rb : 0;
}

size_t kvc_idx_row_bytes(const kvc_config* cfg) {
    Shape sh;
    return derive_shape(cfg, &sh) ? (size_t)sh.idx_rb : 0;
}

size_t kvc_bytes_resident(const kvc_config* cfg, int64_t entries, int n_layers, int padded) {
    Shape sh;
    if (!derive_shape(cfg, &sh) || entries < 0 || n_layers < 0) return 0;
    const int64_t rec = padded ? sh.rb : sh.rec_unpadded;
    return (size_t)(entries * rec + entries * sh.idx_rb +
                    (int64_t)n_layers * cfg->window * sh.D * sh.act_bytes);
}

size_t kvc_workspace_bytes(const kvc_config* cfg, int batch, int capacity) {
    Shape sh;
    if (!derive_shape(cfg, &sh) || batch < 0 || capacity < 0) return 0;
    return ws_layout(*cfg, sh, batch, capacity).total;
}

static bool hier_ok(int hier_blocks, int hier_block) {
    return hier_blocks == 0 ||
           (hier_blocks > 0 && hier_blocks <= 65536 && hier_block >= 1 && hier_block <= 256);
}

size_t kvc_workspace_bytes_hier(const kvc_config* cfg, int batch, int capacity, int hier_blocks,
                                int hier_block) {
    Shape sh;
    if (!derive_shape(cfg, &sh) || batch < 0 || capacity < 0 || !hier_ok(hier_blocks, hier_block))
        return 0;
    return ws_layout(*cfg, sh, batch, capacity, hier_blocks, hier_block).total;
}

kvc_status kvc_pack(const kvc_config* cfg, const void* tokens, int n_new, const float* gate,
                    const int8_t* idx_k_new, const kvc_cache* cache, uint32_t* dev_status,
                    void* stream) {
    const NvtxRange nvtx_range("kvc_pack");
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    kvc_status st = check_cache(cache, sh);
    if (st != KVC_OK) return st;
    const int r = cfg->ratio == 4 ? 4 : 2;
    if (n_new < 0 || n_new % r) return KVC_ERR_INVALID;
    if (n_new == 0 || cache->batch == 0) return KVC_OK;
    if (n_new / r > cache->capacity) return KVC_ERR_CAPACITY;
    if (!tokens || !gate || !idx_k_new) return KVC_ERR_INVALID;
    if (!aligned(tokens, 16) || !aligned(gate, 16) || !aligned(idx_k_new, 16)) return KVC_ERR_INVALID;
    if (!device_ok()) return KVC_ERR_DEVICE;
    PackArgs a;
    a.tokens = tokens;
    a.n_new = n_new;
    a.batch = cache->batch;
    a.capacity = cache->capacity;
    a.gate = gate;
    a.idx_k_new = idx_k_new;
    a.records = static_cast<uint8_t*>(cache->records);
    a.idx_k = cache->idx_k;
    a.n_entries = cache->n_entries;
    a.status = dev_status;
    return launch_pack(*cfg, sh, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? KVC_OK
                                                                                     : KVC_ERR_CUDA;
}

kvc_status kvc_index_topk(const kvc_config* cfg, const int8_t* idx_q, const kvc_cache* cache,
                          int32_t* topk_idx, int32_t* scores, void* ws, size_t ws_bytes,
                          uint32_t* dev_status, void* stream) {
    const NvtxRange nvtx_range("kvc_index_topk");
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    kvc_status st = check_cache(cache, sh);
    if (st != KVC_OK) return st;
    if (cache->batch == 0) return KVC_OK;
    if (!idx_q || !topk_idx || !aligned(idx_q, 16) || !aligned(topk_idx, 4)) return KVC_ERR_INVALID;
    if (scores && !aligned(scores, 4)) return KVC_ERR_INVALID;
    if (scores && sh.idx_fmt == 1) return KVC_ERR_UNSUPPORTED;  // FP4 keys: 64-bit scores
    if (cache->capacity > kMaxTopkCapacity) return KVC_ERR_CAPACITY;
    WsLayout w;
    if ((st = check_ws(ws, ws_bytes, *cfg, sh, cache->batch, cache->capacity, &w)) != KVC_OK) return st;
    if (!device_ok()) return KVC_ERR_DEVICE;
    return run_topk(*cfg, idx_q, cache, topk_idx, scores, static_cast<unsigned char*>(ws), w,
                    dev_status, static_cast<cudaStream_t>(stream));
}

kvc_status kvc_sparse_decode_attn(const kvc_config* cfg, const void* q, const kvc_cache* cache,
                                  const int32_t* topk_idx, const void* window, int window_len,
                                  float* out, float* lse, void* ws, size_t ws_bytes,
                                  uint32_t* dev_status, void* stream) {
    const NvtxRange nvtx_range("kvc_sparse_decode_attn");
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    kvc_status st = check_cache(cache, sh);
    if (st != KVC_OK) return st;
    if (cache->batch == 0) return KVC_OK;
    if (window_len < 0 || window_len > cfg->window) return KVC_ERR_INVALID;
    if (!q || !topk_idx || !out || (window_len > 0 && !window)) return KVC_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(topk_idx, 4) ||
        (window && !aligned(window, 16)) || (lse && !aligned(lse, 4)))
        return KVC_ERR_INVALID;
    WsLayout w;
    if ((st = check_ws(ws, ws_bytes, *cfg, sh, cache->batch, cache->capacity, &w)) != KVC_OK) return st;
    if (!device_ok()) return KVC_ERR_DEVICE;
    return run_attn(*cfg, sh, q, cache, topk_idx, window, window_len, out, lse,
                    static_cast<unsigned char*>(ws), w, dev_status, static_cast<cudaStream_t>(stream));
}

kvc_status kvc_sparse_decode_attn_fp8win(const kvc_config* cfg, const void* q,
                                         const kvc_cache* cache, const int32_t* topk_idx,
                                         const uint8_t* win_codes, const float* win_scales,
                                         int window_len, float* out, float* lse, void* ws,
                                         size_t ws_bytes, uint32_t* dev_status, void* stream) {
    const NvtxRange nvtx_range("kvc_sparse_decode_attn_fp8win");
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    kvc_status st = check_cache(cache, sh);
    if (st != KVC_OK) return st;
    if (cache->batch == 0) return KVC_OK;
    if (window_len < 0 || window_len > cfg->window) return KVC_ERR_INVALID;
    if (!q || !topk_idx || !out || (window_len > 0 && (!win_codes || !win_scales)))
        return KVC_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(topk_idx, 4) ||
        (win_codes && !aligned(win_codes, 16)) || (win_scales && !aligned(win_scales, 4)) ||
        (lse && !aligned(lse, 4)) || sh.D % 16)
        return KVC_ERR_INVALID;
    WsLayout w;
    if ((st = check_ws(ws, ws_bytes, *cfg, sh, cache->batch, cache->capacity, &w)) != KVC_OK) return st;
    if (!device_ok()) return KVC_ERR_DEVICE;
    // a non-null code pointer selects the FP8 window in the kernels
    const uint8_t* codes = window_len > 0 ? win_codes : nullptr;
    return run_attn(*cfg, sh, q, cache, topk_idx, nullptr, window_len, out, lse,
                    static_cast<unsigned char*>(ws), w, dev_status,
                    static_cast<cudaStream_t>(stream), nullptr, codes, win_scales);
}

kvc_status kvc_pack_window_fp8(const kvc_config* cfg, const void* rows, int64_t n_rows,
                               uint8_t* codes, float* scales, uint32_t* dev_status,
                               void* stream) {
    const NvtxRange nvtx_range("kvc_pack_window_fp8");
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    if (n_rows < 0 || (n_rows > 0 && (!rows || !codes || !scales))) return KVC_ERR_INVALID;
    if (n_rows == 0) return KVC_OK;
    if (!aligned(rows, 16) || !aligned(codes, 8) || !aligned(scales, 4)) return KVC_ERR_INVALID;
    if (!device_ok()) return KVC_ERR_DEVICE;
    return launch_window_fp8(*cfg, sh, rows, n_rows, codes, scales, dev_status,
                             static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KVC_OK
               : KVC_ERR_CUDA;
}

kvc_status kvc_layer_group_step(const kvc_config* cfg, int n_layers, const int32_t* modes,
                                const void* q, const int8_t* idx_q, const void* windows,
                                int window_len, const kvc_cache* cache, float* out, float* lse,
                                int32_t* topk, void* ws, size_t ws_bytes, uint32_t* dev_status,
                                void* stream) {
    const NvtxRange nvtx_range("kvc_layer_group_step");
    return kvc_layer_group_step_hier(cfg, 0, 0, n_layers, modes, q, idx_q, windows, window_len,
                                     cache, out, lse, topk, ws, ws_bytes, dev_status, stream);
}

kvc_status kvc_layer_group_step_hier(const kvc_config* cfg, int hier_blocks, int hier_block,
                                     int n_layers, const int32_t* modes, const void* q,
                                     const int8_t* idx_q, const void* windows, int window_len,
                                     const kvc_cache* cache, float* out, float* lse,
                                     int32_t* topk, void* ws, size_t ws_bytes,
                                     uint32_t* dev_status, void* stream) {
    const NvtxRange nvtx_range("kvc_layer_group_step_hier");
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    if (!hier_ok(hier_blocks, hier_block)) return KVC_ERR_INVALID;
    if (hier_blocks > 0 && sh.idx_fmt != 0) return KVC_ERR_UNSUPPORTED;
    kvc_status st = check_cache(cache, sh);
    if (st != KVC_OK) return st;
    if (n_layers < 1 || !modes) return KVC_ERR_INVALID;
    for (int l = 0; l < n_layers; ++l)
        if (modes[l] != KVC_FULL && modes[l] != KVC_REINDEX && modes[l] != KVC_REUSE)
            return KVC_ERR_INVALID;
    if (modes[0] == KVC_REUSE) return KVC_ERR_INVALID;
    if (cache->batch == 0) return KVC_OK;
    if (window_len < 0 || window_len > cfg->window) return KVC_ERR_INVALID;
    if (!q || !idx_q || !out || !topk || (window_len > 0 && !windows)) return KVC_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(idx_q, 16) || !aligned(out, 16) || !aligned(topk, 4) ||
        (windows && !aligned(windows, 16)) || (lse && !aligned(lse, 4)))
        return KVC_ERR_INVALID;
    const size_t B = (size_t)cache->batch, H = (size_t)cfg->n_heads;
    const size_t q_stride = B * H * sh.D * sh.act_bytes;
    const size_t w_stride = B * (size_t)cfg->window * sh.D * sh.act_bytes;
    if (q_stride % 16 || (w_stride % 16) || (B * cfg->idx_dim) % 16) return KVC_ERR_INVALID;
    if (cache->capacity > kMaxTopkCapacity) return KVC_ERR_CAPACITY;
    WsLayout w;
    if ((st = check_ws(ws, ws_bytes, *cfg, sh, cache->batch, cache->capacity, &w, hier_blocks,
                       hier_block)) != KVC_OK)
        return st;
    if (!device_ok()) return KVC_ERR_DEVICE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    const size_t K = (size_t)cfg->topk;
    int head = -1;
    bool have_pool = false;
    for (int l = 0; l < n_layers; ++l) {
        int32_t* tk = topk + (size_t)l * B * K;
        const int8_t* iq = idx_q + (size_t)l * B * cfg->idx_dim;
        if (modes[l] == KVC_FULL || (modes[l] == KVC_REINDEX && !have_pool)) {
            // Full scores its stored cache; Reindex rescores the same stored
            // (Full layer's) cache with its own indexer query.
            st = run_topk(*cfg, iq, cache, tk, nullptr, wsb, w, dev_status, s);
            if (st != KVC_OK) return st;
            if (hier_blocks > 0 && modes[l] == KVC_FULL) {
                // hierarchical indexer: later Reindex layers score only the
                // pool of this layer's best blocks
                st = run_block_pool(*cfg, cache, hier_blocks, hier_block, wsb, w, dev_status, s);
                if (st != KVC_OK) return st;
                have_pool = true;
            }
            head = l;
        } else if (modes[l] == KVC_REINDEX) {
            st = run_pool_topk(*cfg, iq, cache, hier_blocks, hier_block, tk, wsb, w, dev_status,
                               s);
            if (st != KVC_OK) return st;
            head = l;
        }
        // a Reuse layer attends over its head's top-K; the attention launch
        // also writes the layer's own copy of those indices
        const bool reuse = modes[l] == KVC_REUSE;
        st = run_attn(*cfg, sh, static_cast<const unsigned char*>(q) + l * q_stride, cache,
                      reuse ? topk + (size_t)head * B * K : tk,
                      windows ? static_cast<const unsigned char*>(windows) + l * w_stride : nullptr,
                      window_len, out + (size_t)l * B * H * sh.Dv, lse ? lse + (size_t)l * B * H : nullptr,
                      wsb, w, dev_status, s, reuse ? tk : nullptr, nullptr, nullptr,
                      /*q_ready=*/true);  // only this step's own kernels ran since the call
        if (st != KVC_OK) return st;
    }
    return KVC_OK;
}

size_t kvc_workspace_bytes_batched(const kvc_config* cfg, int nq, int batch, int capacity) {
    Shape sh;
    if (!derive_shape(cfg, &sh) || nq < 1 || nq > kMaxBatchQ || batch < 0 || capacity < 0)
        return 0;
    return (size_t)nq * batch_ws_layout(batch, capacity).block;
}

kvc_status kvc_index_topk_batched(const kvc_config* cfg, int nq, const int8_t* idx_q,
                                  const kvc_cache* cache, int32_t* topk_idx, void* ws,
                                  size_t ws_bytes, uint32_t* dev_status, void* stream) {
    const NvtxRange nvtx_range("kvc_index_topk_batched");
    Shape sh;
    if (!derive_shape(cfg, &sh)) return KVC_ERR_INVALID;
    if (nq < 1 || nq > kMaxBatchQ) return KVC_ERR_INVALID;
    if (cfg->idx_dim != 128 || sh.idx_fmt != 0) return KVC_ERR_UNSUPPORTED;
    kvc_status st = check_cache(cache, sh);
    if (st != KVC_OK) return st;
    if (cache->batch == 0) return KVC_OK;
    if (!idx_q || !topk_idx || !aligned(idx_q, 16) || !aligned(topk_idx, 4))
        return KVC_ERR_INVALID;
    if (cache->capacity > kMaxTopkCapacity) return KVC_ERR_CAPACITY;
    const BatchWs w = batch_ws_layout(cache->batch, cache->capacity);
    if (!ws || !aligned(ws, kAlign) || ws_bytes < (size_t)nq * w.block) return KVC_ERR_WORKSPACE;
    if (!device_ok()) return KVC_ERR_DEVICE;
    unsigned char* wsb = static_cast<unsigned char*>(ws);
    BatchTopkArgs ba = {};
    ba.nq = nq;
    const size_t B = (size_t)cache->batch, K = (size_t)cfg->topk;
    for (int q = 0; q < nq; ++q) {
        TopkArgs& a = ba.q[q];
        unsigned char* blk = wsb + (size_t)q * w.block;
        a.idx_q = idx_q + (size_t)q * B * cfg->idx_dim;
        a.idx_k = cache->idx_k;
        a.n_entries = cache->n_entries;
        a.batch = cache->batch;
        a.capacity = cache->capacity;
        a.idx_capacity = cache->capacity;
        a.topk = cfg->topk;
        a.di = cfg->idx_dim;
        a.topk_idx = topk_idx + (size_t)q * B * K;
        a.scores = reinterpret_cast<int32_t*>(blk + w.scores);
        a.counters = reinterpret_cast<int32_t*>(blk + w.counters);
        a.thr = reinterpret_cast<int32_t*>(blk + w.thr);
        a.tile_count = reinterpret_cast<int32_t*>(blk + w.tile_count);
        a.cands = reinterpret_cast<unsigned long long*>(blk + w.cands);
        a.status = dev_status;
    }
    return launch_index_topk_batched(ba, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KVC_OK
               : KVC_ERR_CUDA;
}

kvc_status kvc_e2m1_encode(const float* x, int64_t n, uint8_t* codes, void* stream) {
    const NvtxRange nvtx_range("kvc_e2m1_encode");
    if (n < 0 || (n > 0 && (!x || !codes))) return KVC_ERR_INVALID;
    if (n > 0 && !device_ok()) return KVC_ERR_DEVICE;
    return launch_fp4_codec(x, n, codes, 0, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KVC_OK
               : KVC_ERR_CUDA;
}

kvc_status kvc_e4m3_encode(const float* x, int64_t n, uint8_t* bytes, void* stream) {
    const NvtxRange nvtx_range("kvc_e4m3_encode");
    if (n < 0 || (n > 0 && (!x || !bytes))) return KVC_ERR_INVALID;
    if (n > 0 && !device_ok()) return KVC_ERR_DEVICE;
    return launch_fp4_codec(x, n, bytes, 1, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KVC_OK
               : KVC_ERR_CUDA;
}

kvc_status kvc_trace_begin(int max_launches) {
    if (max_launches < 1 || max_launches > (1 << 20)) return KVC_ERR_INVALID;
    TraceState& t = trace();
    std::lock_guard<std::mutex> lk(t.mu);
    for (cudaEvent_t e : t.ev) cudaEventDestroy(e);
    t.ev.assign(2 * (size_t)max_launches, nullptr);
    for (auto& e : t.ev)
        if (cudaEventCreate(&e) != cudaSuccess) {
            t.on = false;
            return KVC_ERR_CUDA;
        }
    t.name.assign(max_launches, std::string());
    t.max = max_launches;
    t.used = 0;
    t.on = true;
    return KVC_OK;
}

kvc_status kvc_trace_end(void) {
    TraceState& t = trace();
    std::lock_guard<std::mutex> lk(t.mu);
    t.on = false;
    return KVC_OK;
}

kvc_status kvc_trace_kernel(const char* name, int* launches, double* total_ms) {
    if (!name || !launches || !total_ms) return KVC_ERR_INVALID;
    TraceState& t = trace();
    std::lock_guard<std::mutex> lk(t.mu);
    int cnt = 0;
    double sum = 0.0;
    for (int i = 0; i < t.used; ++i) {
        if (t.name[i] != name) continue;
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, t.ev[2 * i], t.ev[2 * i + 1]) != cudaSuccess) return KVC_ERR_CUDA;
        ++cnt;
        sum += ms;
    }
    *launches = cnt;
    *total_ms = sum;
    return KVC_OK;
}

uint64_t kvc_launch_count(void) { return g_launches.load(); }

kvc_status kvc_debug_set_wait_limit_ns(uint64_t ns) {
    set_device_wait_limit_ns(ns);
    return KVC_OK;
}

const char* kvc_status_string(kvc_status s) {
    switch (s) {
        case KVC_OK: return "ok";
        case KVC_ERR_INVALID: return "invalid argument or configuration";
        case KVC_ERR_CAPACITY: return "size exceeds capacity";
        case KVC_ERR_CUDA: return "CUDA launch or runtime error";
        case KVC_ERR_UNSUPPORTED: return "unsupported shape";
        case KVC_ERR_TIMEOUT: return "bounded wait timed out";
        case KVC_ERR_DEVICE: return "no sm_100 device current";
        case KVC_ERR_WORKSPACE: return "workspace null, misaligned or too small";
    }
    return "unknown status";
}

const char* kvc_version(void) { return "kvc 0.1 sm_100a"; }

}  // extern "C"
