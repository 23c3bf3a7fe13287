// index_topk.cu -- lightweight-indexer scoring and exact top-K selection.
//
// Method: "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
// 压缩到 890 B的？" (acejoy.com) part 3 breakthrough 4 (a lightweight indexer
// scores every history entry; only the 512 best are attended) and part 4
// "CSA2：三种模式" (Full and Reindex layers score the whole stored context).
// Scores are int8 x int8 dot products accumulated in int32 (exact).  The
// order is (score descending, index ascending); the output lists the chosen
// indices in ascending order, padded with -1.
//
// Design (B200): the scan is a pure HBM stream of 128-byte int8 rows.
//  1. index_scan: a grid of CTAs tiles every sequence's visible entries;
//     Di/16 lanes share a row, each loading 16 bytes (coalesced 512-byte warp
//     loads, 4 rows in flight per lane), dp4a + xor-shuffle reduce to the
//     score.  Each score is stored (4 bytes beside the 128 read) and counted
//     in a 2048-bin shared-memory histogram of its biased value; the CTA then
//     adds its non-zero bins to the sequence's global histogram.
//  2. topk_collect: every CTA rebuilds the threshold bin t from the global
//     histogram (the highest bin whose suffix count reaches K) and appends
//     the (score, index) keys of entries in bins >= t to a candidate list
//     (warp-aggregated atomics).  Typically K + a few dozen candidates.
//  3. topk_finalize: one CTA per sequence.  Entries above bin t are all in;
//     the r = K - count(bins > t) best of bin t are chosen by exact ranking
//     of 64-bit keys (score, ~index); the K winners are then placed in index
//     order by rank counting.  If more than kMaxCand candidates reached the
//     list (heavy ties), a slower exact path finds the threshold score and
//     the index cut-off with a second histogram and compacts the scores in
//     index order.
// No kernel waits on another CTA: the three launches are stream-ordered.
#include "kvc_internal.cuh"

namespace kvc {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ int score_bin(int s, int bias, int shift) {
    return (s + bias) >> shift;
}

__device__ __forceinline__ unsigned long long make_key(int s, int idx, int bias) {
    return ((unsigned long long)(uint32_t)(s + bias) << 32) | (uint32_t)(~(uint32_t)idx);
}
__device__ __forceinline__ int key_index(unsigned long long k) {
    return (int)(~(uint32_t)(k & 0xffffffffull));
}

// Block-wide: threshold bin t = the highest bin whose suffix count >= K, and
// the count of entries in bins above t.  Requires total >= K.  blockDim.x
// must be a multiple of 32 and divide kBins.
__device__ void find_threshold(const int32_t* __restrict__ hist, int K, int* t_out,
                               int* above_out, int* sh_warp) {
    const int nt = blockDim.x, tid = threadIdx.x;
    const int per = kBins / nt;
    if (tid == 0) {
        *t_out = 0;
        *above_out = 0;
    }
    // thread tid covers bins [kBins - (tid+1)*per, kBins - tid*per): thread 0 the top
    const int hi = kBins - tid * per, lo = hi - per;
    int local = 0;
    for (int b = lo; b < hi; ++b) local += hist[b];
    // inclusive prefix over threads (top bins first)
    int v = local;
    const int lane = tid & 31, w = tid >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    if (lane == 31) sh_warp[w] = v;
    __syncthreads();
    int warp_prefix = 0;
    for (int i = 0; i < w; ++i) warp_prefix += sh_warp[i];
    const int incl = v + warp_prefix;
    const int excl = incl - local;  // count strictly above bin hi-1
    if (excl < K && incl >= K) {
        int run = excl;
        for (int b = hi - 1; b >= lo; --b) {
            if (run + hist[b] >= K) {
                *t_out = b;
                *above_out = run;
                break;
            }
            run += hist[b];
        }
    }
    __syncthreads();
}

template <int DI>
__global__ void __launch_bounds__(kThreads)
index_scan_kernel(TopkArgs a, int tile, int bias, int shift) {
    __shared__ int hist[kBins];
    constexpr int TPR = DI / 16;   // lanes per row
    constexpr int RPW = 32 / TPR;  // rows per warp step
    constexpr int UNROLL = 4;
    const int b = blockIdx.y;
    const int n = a.n_entries[b];
    if (n < 0 || n > a.capacity) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_status(a.status, KVC_DEV_BAD_LENGTH);
        return;
    }
    const int start = blockIdx.x * tile;
    if (start >= n) return;
    const int end = min(start + tile, n);
    for (int i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0;
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int sub = lane % TPR, rloc = lane / TPR;
    const int4 qv = __ldg(reinterpret_cast<const int4*>(a.idx_q + (size_t)b * DI) + sub);
    const int8_t* kb = a.idx_k + (size_t)b * a.capacity * DI;
    int32_t* sc = a.scores + (size_t)b * a.capacity;
    constexpr int kStep = (kThreads / 32) * RPW;  // rows per CTA step
    for (int r0 = start + warp * RPW; r0 < end; r0 += kStep * UNROLL) {
        int4 kv[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int row = r0 + u * kStep + rloc;
            if (row < end)
                kv[u] = __ldcs(reinterpret_cast<const int4*>(kb + (size_t)row * DI) + sub);
            else
                kv[u] = make_int4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            int s = __dp4a(kv[u].x, qv.x, 0);
            s = __dp4a(kv[u].y, qv.y, s);
            s = __dp4a(kv[u].z, qv.z, s);
            s = __dp4a(kv[u].w, qv.w, s);
#pragma unroll
            for (int o = 1; o < TPR; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            const int row = r0 + u * kStep + rloc;
            if (sub == 0 && row < end) {
                sc[row] = s;
                atomicAdd(&hist[score_bin(s, bias, shift)], 1);
            }
        }
    }
    __syncthreads();
    int32_t* gh = a.hist + (size_t)b * kBins;
    for (int i = threadIdx.x; i < kBins; i += kThreads)
        if (hist[i]) atomicAdd(&gh[i], hist[i]);
}

__global__ void __launch_bounds__(kThreads)
topk_collect_kernel(TopkArgs a, int tile, int bias, int shift) {
    __shared__ int sh_warp[kThreads / 32];
    __shared__ int s_t, s_above;
    const int b = blockIdx.y;
    const int n = a.n_entries[b];
    if (n < 0 || n > a.capacity || n <= a.topk) return;
    const int start = blockIdx.x * tile;
    if (start >= n) return;
    const int end = min(start + tile, n);
    find_threshold(a.hist + (size_t)b * kBins, a.topk, &s_t, &s_above, sh_warp);
    const int t = s_t;
    const int32_t* sc = a.scores + (size_t)b * a.capacity;
    unsigned long long* cand = a.cands + (size_t)b * kMaxCand;
    const int lane = threadIdx.x & 31;
    for (int base = start; base < end; base += kThreads) {
        const int j = base + threadIdx.x;
        int s = 0;
        bool take = false;
        if (j < end) {
            s = __ldcg(sc + j);
            take = score_bin(s, bias, shift) >= t;
        }
        const unsigned m = __ballot_sync(0xffffffffu, take);
        if (m) {
            int first = 0;
            if (lane == 0) first = atomicAdd(&a.cand_count[b], __popc(m));
            first = __shfl_sync(0xffffffffu, first, 0);
            if (take) {
                const int pos = first + __popc(m & ((1u << lane) - 1u));
                if (pos < kMaxCand) cand[pos] = make_key(s, j, bias);
            }
        }
    }
}

// Block-wide exclusive prefix sum of one int per thread; returns the block total.
__device__ int block_excl_scan(int v, int* excl, int* sh_warp) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += u;
    }
    __syncthreads();
    if (lane == 31) sh_warp[w] = x;
    __syncthreads();
    int pre = 0, total = 0;
    for (int i = 0; i < nw; ++i) {
        if (i < w) pre += sh_warp[i];
        total += sh_warp[i];
    }
    *excl = pre + x - v;
    return total;
}

constexpr int kFinThreads = 1024;

__global__ void __launch_bounds__(kFinThreads)
topk_finalize_kernel(TopkArgs a, int bias, int shift) {
    extern __shared__ __align__(16) unsigned char smem[];
    unsigned long long* keys = reinterpret_cast<unsigned long long*>(smem);  // kMaxCand
    int* tie = reinterpret_cast<int*>(keys + kMaxCand);                      // kMaxCand
    int* sel = tie + kMaxCand;                                               // <= K
    __shared__ int sh_warp[kFinThreads / 32];
    __shared__ int s_t, s_above, s_ntie, s_nsel, s_low, s_gt;

    const int b = blockIdx.x, K = a.topk;
    int32_t* out = a.topk_idx + (size_t)b * K;
    const int n = a.n_entries[b];
    if (n < 0 || n > a.capacity) {
        for (int i = threadIdx.x; i < K; i += blockDim.x) out[i] = -1;
        return;
    }
    if (n <= K) {
        for (int i = threadIdx.x; i < K; i += blockDim.x) out[i] = i < n ? i : -1;
        return;
    }
    const int32_t* hist = a.hist + (size_t)b * kBins;
    find_threshold(hist, K, &s_t, &s_above, sh_warp);
    const int t = s_t, r = K - s_above;  // take r entries of bin t
    const int M = __ldcg(a.cand_count + b);

    if (M <= kMaxCand) {
        if (threadIdx.x == 0) s_ntie = s_nsel = 0;
        __syncthreads();
        const unsigned long long* cand = a.cands + (size_t)b * kMaxCand;
        for (int i = threadIdx.x; i < M; i += blockDim.x) {
            const unsigned long long k = __ldcg(cand + i);
            keys[i] = k;
            const int bin = (int)((k >> 32) >> shift);
            if (bin == t) {
                tie[atomicAdd(&s_ntie, 1)] = i;
            } else {
                const int p = atomicAdd(&s_nsel, 1);
                if (p < K) sel[p] = key_index(k);
            }
        }
        __syncthreads();
        const int nt = s_ntie;
        for (int i = threadIdx.x; i < nt; i += blockDim.x) {
            const unsigned long long k = keys[tie[i]];
            int rank = 0;
            for (int j = 0; j < nt; ++j) rank += keys[tie[j]] > k;
            if (rank < r) {
                const int p = atomicAdd(&s_nsel, 1);
                if (p < K) sel[p] = key_index(k);
            }
        }
        __syncthreads();
        // s_nsel == K here; place winners in ascending index order
        for (int i = threadIdx.x; i < K; i += blockDim.x) {
            const int v = sel[i];
            int pos = 0;
            for (int j = 0; j < K; ++j) pos += sel[j] < v;
            out[pos] = v;
        }
        return;
    }

    // Heavy ties: exact threshold score inside bin t from a second histogram
    // over the low `shift` bits (<= 4096 bins), then an index-order pass.
    int* h2 = reinterpret_cast<int*>(smem);  // 1 << shift ints (<= 16 KB)
    const int nb2 = 1 << shift;
    for (int i = threadIdx.x; i < nb2; i += blockDim.x) h2[i] = 0;
    __syncthreads();
    const int32_t* sc = a.scores + (size_t)b * a.capacity;
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
        const int v = __ldcg(sc + j) + bias;
        if ((v >> shift) == t) atomicAdd(&h2[v & (nb2 - 1)], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0, low = 0;
        for (int i = nb2 - 1; i >= 0; --i) {
            if (run + h2[i] >= r) {
                low = i;
                break;
            }
            run += h2[i];
        }
        s_low = low;       // threshold score = (t << shift | low) - bias
        s_gt = run;        // entries of bin t above the threshold score
    }
    __syncthreads();
    const int thr = ((t << shift) | s_low) - bias;
    const int need_eq = r - s_gt;  // entries equal to thr to take, lowest index first
    int taken = 0, eq_seen = 0;
    for (int base = 0; base < n; base += blockDim.x) {
        const int j = base + threadIdx.x;
        const int s = j < n ? __ldcg(sc + j) : INT32_MIN;
        const int is_eq = (j < n && s == thr) ? 1 : 0;
        int eq_before;
        const int eq_total = block_excl_scan(is_eq, &eq_before, sh_warp);
        const int take = (j < n) && (s > thr || (is_eq && eq_seen + eq_before < need_eq));
        int pos_before;
        const int take_total = block_excl_scan(take, &pos_before, sh_warp);
        if (take && taken + pos_before < K) out[taken + pos_before] = j;
        taken += take_total;
        eq_seen += eq_total;
    }
    for (int i = taken + threadIdx.x; i < K; i += blockDim.x) out[i] = -1;
}

template <int DI>
cudaError_t launch_scan(const TopkArgs& a, int tile, int bias, int shift, cudaStream_t s) {
    dim3 grid((a.capacity + tile - 1) / tile, a.batch);
    index_scan_kernel<DI><<<grid, kThreads, 0, s>>>(a, tile, bias, shift);
    return cudaGetLastError();
}

size_t finalize_smem() {
    return (size_t)kMaxCand * 8 + (size_t)kMaxCand * 4 + 2048 * 4;
}

}  // namespace

cudaError_t launch_index_topk(const TopkArgs& a, cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    const int bias = score_bias(a.di), shift = score_shift(a.di);
    // zero the histograms and candidate counters (adjacent in the workspace)
    cudaError_t err = cudaMemsetAsync(a.hist, 0, (size_t)a.batch * (kBins + 1) * sizeof(int32_t), s);
    if (err != cudaSuccess) return err;
    // scan tile: aim for about 4 CTAs per SM over the whole batch
    const long long rows = (long long)a.batch * a.capacity;
    long long tile = (rows + 4 * 148 - 1) / (4 * 148);
    tile = (tile + 255) / 256 * 256;
    if (tile < 256) tile = 256;
    if (tile > 16384) tile = 16384;
    trace_before("index_scan", s);
    switch (a.di) {
        case 16: err = launch_scan<16>(a, (int)tile, bias, shift, s); break;
        case 32: err = launch_scan<32>(a, (int)tile, bias, shift, s); break;
        case 64: err = launch_scan<64>(a, (int)tile, bias, shift, s); break;
        case 128: err = launch_scan<128>(a, (int)tile, bias, shift, s); break;
        default: err = launch_scan<256>(a, (int)tile, bias, shift, s); break;
    }
    trace_after(s);
    if (err != cudaSuccess) return err;
    {
        const int ctile = 16384;
        dim3 grid((a.capacity + ctile - 1) / ctile, a.batch);
        trace_before("topk_collect", s);
        topk_collect_kernel<<<grid, kThreads, 0, s>>>(a, ctile, bias, shift);
        trace_after(s);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        err = cudaFuncSetAttribute(topk_finalize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)finalize_smem());
        if (err != cudaSuccess) return err;
        attr_set[dev] = true;
    }
    trace_before("topk_finalize", s);
    topk_finalize_kernel<<<a.batch, kFinThreads, finalize_smem(), s>>>(a, bias, shift);
    trace_after(s);
    return cudaGetLastError();
}

}  // namespace kvc
