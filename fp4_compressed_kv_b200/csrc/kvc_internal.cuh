// kvc_internal.cuh -- declarations shared by the kernels and the C ABI of
// libkvc.so.  Not installed; the public interface is include/kvc.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvc.h"

namespace kvc {

// Indexer histogram: 2048 bins over the biased int8 x int8 score range.
constexpr int kBins = 2048;
// Top-K selection: scores are cut into tiles of kSelTile entries; each tile
// keeps its candidate keys (in index order) in its own slot of the candidate
// array.  A sequence holds at most kMaxSelTiles tiles (8,388,608 entries).
constexpr int kSelTile = 8192;
constexpr int kMaxSelTiles = 1024;
constexpr long long kMaxTopkCapacity = (long long)kSelTile * kMaxSelTiles;
// Candidates of the threshold bin kept for the in-shared-memory finish.
constexpr int kMaxTies = 4096;
// FP4 indexer keys: candidate slots (64-bit keys) per select tile, in the
// workspace's score region (sized [B][sel_tiles(cap)][kFp4TileCands] keys).
constexpr int kFp4TileCands = kSelTile / 2;
__host__ __device__ inline int sel_tiles(int capacity) { return (capacity + kSelTile - 1) / kSelTile; }
// Per-call counters of the top-K: histograms [B][kBins], finished scan CTAs
// [B] and finished select CTAs [B], adjacent so one memset clears them.
inline size_t topk_counter_words(int batch) { return (size_t)batch * (kBins + 2); }
// Upper bound on the number of key splits of one attention problem.
constexpr int kMaxSplit = 16;

// Shape facts derived once from a kvc_config.
struct Shape {
    int D;          // latent + rope
    int Dv;         // latent
    int G;          // group size
    int lpg;        // lanes (8-channel chunks) per group: G / 8
    int n_groups;   // latent groups + rope groups
    int code_bytes; // D / 2
    int scale_bytes;// 1 (UE4M3) or 4 (fp32)
    int rec_unpadded;
    int rb;         // record stride (padded to 16)
    int act_bytes;  // 2 (bf16) or 4 (fp32)
    int idx_fmt;    // 0 int8 indexer rows, 1 FP4 indexer rows
    int idx_rb;     // bytes of one indexer row
};

bool derive_shape(const kvc_config* c, Shape* s);

// Score bias and histogram shift for indexer width di: every int8 x int8 dot
// of width di lies in [-di*127*128, di*128*128]; adding di*127*128 makes it
// non-negative and below 2^(log2(di)+15), so >> (log2(di)+4) gives a bin in
// [0, 2048).
inline int score_shift(int di) {
    int l = 0;
    while ((1 << l) < di) ++l;
    return l + 4;
}
inline int score_bias(int di) { return di * 127 * 128; }

// ------------------------------------------------------------------ tracing
void trace_before(const char* name, cudaStream_t s);
void trace_after(cudaStream_t s);

// Bound on one device wait of a kernel launched from now on (nanoseconds of
// %globaltimer; 2 s unless a test lowered it through
// kvc_debug_set_wait_limit_ns).
unsigned long long device_wait_limit_ns();
void set_device_wait_limit_ns(unsigned long long ns);
// Bound of the clean-up waits that follow a timeout (never lowered).
constexpr unsigned long long kCleanupWaitNs = 2000000000ull;

// ------------------------------------------------------------------ launchers
struct PackArgs {
    const void* tokens;
    int n_new, batch, capacity;
    const float* gate;
    const int8_t* idx_k_new;
    uint8_t* records;
    int8_t* idx_k;
    int32_t* n_entries;
    uint32_t* status;
};
cudaError_t launch_pack(const kvc_config& c, const Shape& sh, const PackArgs& a,
                        cudaStream_t s);

struct TopkArgs {
    const int8_t* idx_q;   // [B][Di]
    const int8_t* idx_k;   // [B][cap][Di]
    const int32_t* n_entries;
    int batch, capacity, topk, di;
    int32_t* topk_idx;     // [B][K]
    int32_t* scores;       // [B][cap] (user buffer or workspace)
    int32_t* counters;     // topk_counter_words(B) ints: zero before the call (a zero-filled
                           // workspace); the kernels' last CTAs leave them at zero again,
                           // except after a timeout, which leaves them dirty
    int32_t* thr;          // [B][2] threshold bin, entries above it (written by the scan)
    int32_t* tile_count;   // [B][sel_tiles(cap)] candidates per tile
    unsigned long long* cands;  // [B][sel_tiles(cap) * kSelTile]
    uint32_t* status;
    int idx_capacity;      // row stride (entries) of idx_k per sequence
    // Pool mode (hierarchical indexer): when pool_blocks is set, row r of
    // sequence b is entry pool_blocks[b][r / pool_block] * pool_block +
    // r % pool_block of idx_k; capacity and n_entries then describe the pool
    // and the top-K is written as entry indices.
    const int32_t* pool_blocks;  // [B][pool_keep] ascending, or null
    int pool_keep, pool_block;
    // Block stage of the hierarchical indexer (selecting blocks): when set,
    // the finish also writes each sequence's pool length, from the entries
    // pool_src_n (capacity pool_src_cap) cut into blocks of pool_src_block.
    int32_t* pool_len_out;
    const int32_t* pool_src_n;
    int pool_src_cap, pool_src_block;
    // bound on one device wait (set by the launcher from the library's
    // current limit; 0 = a single non-blocking poll, the timeout test hook)
    unsigned long long wait_ns;
};
cudaError_t launch_index_topk(const TopkArgs& a, cudaStream_t s);
// FP4 indexer keys: exact 64-bit scores (scores64 [B][capacity]) and the
// top-K by a radix selection; idx_k rows of idx_rb bytes.
cudaError_t launch_index_topk_fp4(const TopkArgs& a, int idx_rb, long long* scores64,
                                  cudaStream_t s);
// The selection alone, from scores and threshold bins already in the scratch.
cudaError_t launch_select(const TopkArgs& a, int bias, int shift, cudaStream_t s);

// Several indexer queries per sequence scored in one pass over the shared
// indexer cache on the tensor cores (kind::i8), then one selection per query.
// All queries share idx_k / n_entries / batch / capacity / topk / di (= 128);
// each has its own idx_q, output and scratch.
constexpr int kMaxBatchQ = 8;
struct BatchTopkArgs {
    TopkArgs q[kMaxBatchQ];
    int nq;
};
cudaError_t launch_index_topk_batched(const BatchTopkArgs& ba, cudaStream_t s);

// Hierarchical indexer, block stage: from a Full layer's entry scores
// ([B][capacity]), the blocks of `block` consecutive entries are scored by
// their best entry and the best `keep` blocks of every sequence are written
// ascending to pool_blocks [B][keep] (-1 padded); pool_n [B] receives the
// number of pool entries.  Scratch regions as in TopkArgs, sized for
// ceil(capacity / block) block scores.
struct HierArgs {
    const int32_t* scores;     // [B][capacity] entry scores
    const int32_t* n_entries;  // [B]
    int batch, capacity, block, keep, di;
    int32_t* bscore;           // [B][ceil(capacity / block)]
    int32_t* nblk;             // [B]
    int32_t* pool_blocks;      // [B][keep]
    int32_t* pool_n;           // [B]
    int32_t* counters;         // topk_counter_words(B)
    int32_t* thr;              // [B][2]
    int32_t* tile_count;       // [B][sel_tiles(ceil(capacity / block))]
    unsigned long long* cands; // [B][sel_tiles(...) * kSelTile]
    uint32_t* status;
};
cudaError_t launch_block_pool(const HierArgs& h, cudaStream_t s);

struct AttnArgs {
    const void* q;          // [B][H][D]
    const uint8_t* records; // [B][cap][rb]
    const int32_t* n_entries;
    const int32_t* topk_idx;// [B][K]
    const void* window;     // [B][W][D]
    int window_len, window_stride, batch, capacity;
    float* out;             // [B][H][Dv]
    float* lse;             // [B][H] or null
    float* part_o;          // [B][H][kMaxSplit][Dv]
    float* part_ml;         // [B][H][kMaxSplit][2]
    uint32_t* status;
    int32_t* topk_copy;     // [B][K]: receives a copy of topk_idx (a Reuse layer's), or null
    // FP8 window: when set, the window rows are signed E4M3 codes
    // [B][W][D] with one fp32 scale per row [B][W] (window is then unused)
    const uint8_t* win_fp8;
    const float* win_scale;
    // set when nothing launched between the caller's last write of q and
    // this call writes q (a layer-group step): q is then read while the
    // previous kernel still drains, before griddepcontrol.wait
    int q_ready;
};
cudaError_t launch_attention(const kvc_config& c, const Shape& sh, const AttnArgs& a,
                             cudaStream_t s);

// FP8 window rows: rows [n][D] act_dtype -> codes [n][D] signed E4M3, one
// fp32 scale per row (absmax / 448).
cudaError_t launch_window_fp8(const kvc_config& c, const Shape& sh, const void* rows, long long n,
                              uint8_t* codes, float* scales, uint32_t* status, cudaStream_t s);

cudaError_t launch_fp4_codec(const float* x, int64_t n, uint8_t* out, int e4m3,
                             cudaStream_t s);

// Every library kernel is launched with programmatic stream serialization:
// the long kernels signal griddepcontrol.launch_dependents once their main
// loop is done, the pack of a few tokens as it starts, so the next kernel's
// CTAs are scheduled while they run or drain (the selection does not: the
// attention's clusters are placed best on SMs freed all at once);
// each kernel does only local set-up (shared memory, tensor memory,
// barriers, and inputs no library kernel writes) before waiting for its
// predecessor with griddepcontrol.wait, which returns once the predecessor
// -- and so every kernel before it -- has completed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ device helpers
#ifdef __CUDACC__
// Lets the next kernel on the stream be scheduled (it still waits for this
// one to complete before it reads anything this one writes).
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;\n");
}
// Waits until the previous kernel on the stream has completed and its writes
// are visible (returns at once when it was not launched as a dependent).
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void set_status(uint32_t* st, uint32_t bit) {
    if (st) atomicOr(st, bit);
}

// Round-to-nearest-even, saturating conversion of a non-negative fp32 to an
// E4M3 byte (hardware cvt; the value sits in the low byte).
__device__ __forceinline__ uint32_t e4m3_from_f32(float s) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
    return r & 0xFFu;
}

// Exact decode of an E4M3 byte (sign ignored: scales are unsigned).
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
    const uint32_t e = (b >> 3) & 15u, m = b & 7u;
    if (e == 0) return (float)m * 0x1.0p-9f;
    return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Signed E4M3 decode (exact).
__device__ __forceinline__ float e4m3s_to_f32(uint32_t b) {
    const float v = e4m3_to_f32(b & 0x7Fu);
    return (b & 0x80u) ? -v : v;
}
// Four fp32 values -> four signed E4M3 bytes (value t in byte t), round to
// nearest even, saturating; codes of magnitude 0 lose their sign.
__device__ __forceinline__ uint32_t e4m3x4_from_f32(float a0, float a1, float a2, float a3) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(a1), "f"(a0));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(a3), "f"(a2));
    const uint32_t w = (uint32_t)lo | ((uint32_t)hi << 16);
    const uint32_t nonzero = ((w & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) & 0x80808080u;
    return w & (0x7F7F7F7Fu | nonzero);
}

// Eight fp32 values already in [-6, 6] -> eight E2M1 codes in one word,
// value 2t in the low nibble of byte t; codes of magnitude 0 lose their sign.
__device__ __forceinline__ uint32_t e2m1x8_from_f32(const float v[8]) {
    uint32_t w;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(w)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    const uint32_t mag = w & 0x77777777u;
    const uint32_t nonzero = (mag + 0x77777777u) & 0x88888888u;
    return w & (0x77777777u | nonzero);
}
#endif

}  // namespace kvc
