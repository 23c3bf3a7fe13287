// topk_select.cu -- exact top-K selection from the indexer scores.
//
// Method: "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
// 压缩到 890 B的？" (acejoy.com) part 3 breakthrough 4 (only the 512 best
// entries by indexer score are attended).  The order is (score descending,
// index ascending); the output lists the chosen indices in ascending order,
// padded with -1.  The scan (index_topk.cu) has stored every score and found,
// per sequence, the threshold bin t of a 2048-bin histogram (the highest bin
// whose suffix count reaches K) and the count `above` of entries in higher
// bins, so exactly r = K - above entries of bin t are taken.
//
// topk_select_kernel: a CTA per tile of 8,192 scores compacts the (score,
// index) keys of its entries in bins >= t, in index order, into the tile's
// own slot (a warp per 1,024 scores, ballot prefix sums).  The sequence's
// last tile CTA (a fenced counter) then completes the selection without
// sorting the output: it stages every candidate key in shared memory in
// index order (one round of parallel loads), takes the r best keys of bin t
// (a bitonic sort of the few tie candidates) as the cut-off key k*, and a
// block prefix sum over the candidates with key >= k* places the winners in
// index order.  If more than kMaxTies entries share bin t, an exact slower
// path finds the threshold score and the index cut-off with a second
// histogram and compacts the scores.
#include <algorithm>
#include <climits>

#include "topk_common.cuh"

namespace kvc {
namespace {

// In-place block bitonic sort of p (a power of two) keys; descending when
// `desc`.  Every thread of the block must call it.
template <typename Key>
__device__ void block_bitonic(Key* k, int p, bool desc) {
    for (int size = 2; size <= p; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < p; i += blockDim.x) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool up = ((i & size) == 0) != desc;  // ascending run
                    const Key x = k[i], y = k[j];
                    if ((x > y) == up) {
                        k[i] = y;
                        k[j] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Candidate keys of one sequence staged in shared memory for the finish.
// One warp sorts up to 64 keys descending (lane l holds positions l and l+32;
// padding must be 0).  Ascending bitonic network on ~key, shuffles only.
__device__ __forceinline__ void warp_sort64_desc(unsigned long long& x0, unsigned long long& x1,
                                                 int lane) {
    x0 = ~x0;
    x1 = ~x1;
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j == 32) {  // partner is the lane's other element; k == 64: ascending
                const unsigned long long lo = x0 < x1 ? x0 : x1, hi = x0 < x1 ? x1 : x0;
                x0 = lo;
                x1 = hi;
            } else {
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    unsigned long long& x = r ? x1 : x0;
                    const int e = lane + 32 * r;
                    const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j);
                    const bool asc = (e & k) == 0;
                    const bool keep_min = ((e & j) == 0) == asc;
                    x = keep_min ? (x < y ? x : y) : (x < y ? y : x);
                }
            }
        }
    }
    x0 = ~x0;
    x1 = ~x1;
}

constexpr int kStageKeys = 6144;
constexpr size_t kFinishSmem =
    (size_t)kStageKeys * 8 + (size_t)kMaxTies * 8 + (size_t)kMaxSelTiles * 4 * 2;

// One CTA per sequence finishes the selection from the tiles' candidates.
__device__ void finish_body(const TopkArgs& a, int b, int bias, int shift, unsigned char* smem);

// Hierarchical block stage: the pool length of sequence b (whole kept blocks,
// the sequence's last block counting only its visible entries), given
// whether the last block was kept.
__device__ void store_pool_len(const TopkArgs& a, int b, bool last_kept) {
    const int nb = a.n_entries[b];  // blocks of the sequence
    const int n0 = a.pool_src_n[b];
    const int n = (n0 >= 0 && n0 <= a.pool_src_cap) ? n0 : 0;
    const int kept = (nb >= 0 && nb <= a.capacity) ? min(a.topk, nb) : 0;
    int len = kept * a.pool_src_block;
    if (kept > 0 && last_kept) len -= nb * a.pool_src_block - n;
    a.pool_len_out[b] = len;
}

// Finishes sequence b, and in the hierarchical block stage its pool length.
__device__ void finish_sequence(const TopkArgs& a, int b, int bias, int shift,
                                unsigned char* smem) {
    finish_body(a, b, bias, shift, smem);
    if (!a.pool_len_out) return;
    __syncthreads();  // this CTA's output writes are visible to its threads
    if (threadIdx.x == 0) {
        const int nb = a.n_entries[b];
        const int kept = (nb >= 0 && nb <= a.capacity) ? min(a.topk, nb) : 0;
        store_pool_len(a, b,
                       kept > 0 && __ldcg(a.topk_idx + (size_t)b * a.topk + kept - 1) == nb - 1);
    }
}

// Heavy ties: the exact threshold score inside bin t from a second histogram
// over the low `shift` bits (<= 4096 bins), then an index-order pass over
// every score.  One CTA; r = entries of bin t to take.
__device__ void finish_heavy(const TopkArgs& a, int b, int bias, int shift, int t, int r,
                             unsigned char* smem) {
    __shared__ int sh_warp[kThreads / 32];
    __shared__ int s_low, s_gt;
    const int K = a.topk, tid = threadIdx.x;
    const int n = a.n_entries[b];
    int32_t* out = a.topk_idx + (size_t)b * K;
    const int32_t* sc = a.scores + (size_t)b * a.capacity;
    int* h2 = reinterpret_cast<int*>(smem);
    const int nb2 = 1 << shift;
    for (int i = tid; i < nb2; i += kThreads) h2[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += kThreads) {
        const int v = __ldcg(sc + j) + bias;
        if ((v >> shift) == t) atomicAdd(&h2[v & (nb2 - 1)], 1);
    }
    __syncthreads();
    if (tid == 0) {
        int run = 0, low = 0;
        for (int i = nb2 - 1; i >= 0; --i) {
            if (run + h2[i] >= r) {
                low = i;
                break;
            }
            run += h2[i];
        }
        s_low = low;  // threshold score = (t << shift | low) - bias
        s_gt = run;   // entries of bin t above the threshold score
    }
    __syncthreads();
    const int thr = ((t << shift) | s_low) - bias;
    const int need_eq = r - s_gt;  // entries equal to thr to take, lowest index first
    int taken = 0, eq_seen = 0;
    for (int base = 0; base < n; base += kThreads) {
        const int j = base + tid;
        const int s = j < n ? __ldcg(sc + j) : INT32_MIN;
        const int is_eq = (j < n && s == thr) ? 1 : 0;
        int eq_before;
        const int eq_total = block_excl_scan(is_eq, &eq_before, sh_warp);
        const int take = (j < n) && (s > thr || (is_eq && eq_seen + eq_before < need_eq));
        int pos_before;
        const int take_total = block_excl_scan(take, &pos_before, sh_warp);
        if (take && taken + pos_before < K) out[taken + pos_before] = out_index(a, b, j);
        taken += take_total;
        eq_seen += eq_total;
    }
    for (int i = taken + tid; i < K; i += kThreads) out[i] = -1;
}

__device__ void finish_body(const TopkArgs& a, int b, int bias, int shift, unsigned char* smem) {
    unsigned long long* stage = reinterpret_cast<unsigned long long*>(smem);  // kStageKeys
    unsigned long long* ties = stage + kStageKeys;                            // kMaxTies
    int* cnt = reinterpret_cast<int*>(ties + kMaxTies);                       // per tile
    int* off = cnt + kMaxSelTiles;                                            // per tile
    __shared__ int sh_warp[kThreads / 32];
    __shared__ int s_nt;
    __shared__ unsigned long long s_kstar;
    const int K = a.topk, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int n = a.n_entries[b];
    int32_t* out = a.topk_idx + (size_t)b * K;
    if (n < 0 || n > a.capacity) {
        for (int i = tid; i < K; i += kThreads) out[i] = -1;
        return;
    }
    if (n <= K) {
        for (int i = tid; i < K; i += kThreads) out[i] = i < n ? out_index(a, b, i) : -1;
        return;
    }
    const int ntiles = (n + kSelTile - 1) / kSelTile;
    const int t = __ldcg(a.thr + 2 * b), above = __ldcg(a.thr + 2 * b + 1);
    const int ctiles = sel_tiles(a.capacity);
    const unsigned long long* cb = a.cands + (size_t)b * ctiles * kSelTile;
    // tile counts and their exclusive prefix
    int M = 0;
    for (int base = 0; base < ntiles; base += kThreads) {
        const int i = base + tid;
        const int c = i < ntiles ? __ldcg(a.tile_count + (size_t)b * ctiles + i) : 0;
        int ex;
        const int tot = block_excl_scan(c, &ex, sh_warp);
        if (i < ntiles) {
            cnt[i] = c;
            off[i] = M + ex;
        }
        M += tot;
    }
    if (tid == 0) s_nt = 0;
    __syncthreads();
    const int r = K - above;  // entries to take from bin t
    if (M <= kStageKeys) {
        // every candidate key, in index order: all loads in flight at once,
        // then the keys of bin t gathered from shared memory
#pragma unroll 4
        for (int p = tid; p < M; p += kThreads) {
            int lo = 0, hi = ntiles - 1;  // last tile with off <= p
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (off[mid] <= p) lo = mid; else hi = mid - 1;
            }
            stage[p] = __ldcg(cb + (size_t)lo * kSelTile + (p - off[lo]));
        }
        __syncthreads();
        for (int p = tid; p < M; p += kThreads) {
            const unsigned long long k = stage[p];
            if ((int)((k >> 32) >> shift) == t) {
                const int q = atomicAdd(&s_nt, 1);
                if (q < kMaxTies) ties[q] = k;
            }
        }
        __syncthreads();
        const int nt = s_nt;
        if (nt <= kMaxTies) {
            if (nt <= 64) {  // the common case: one warp, no block barriers
                if (warp == 0) {
                    unsigned long long x0 = lane < nt ? ties[lane] : 0ull;
                    unsigned long long x1 = lane + 32 < nt ? ties[lane + 32] : 0ull;
                    warp_sort64_desc(x0, x1, lane);
                    const int want = r - 1;  // r-th best key of bin t
                    const unsigned long long k =
                        __shfl_sync(0xffffffffu, want < 32 ? x0 : x1, want & 31);
                    if (lane == 0) s_kstar = (r >= 1 && r <= nt) ? k : ~0ull;
                }
            } else {
                int p2 = 1;
                while (p2 < nt) p2 <<= 1;
                for (int i = nt + tid; i < p2; i += kThreads) ties[i] = 0ull;  // sorts last
                __syncthreads();
                block_bitonic(ties, p2, true);
                if (tid == 0) s_kstar = (r >= 1 && r <= nt) ? ties[r - 1] : ~0ull;
            }
            __syncthreads();
            const unsigned long long kstar = s_kstar;
            int run = 0;
            for (int base = 0; base < M; base += kThreads) {
                const int p = base + tid;
                const bool sel = p < M && stage[p] >= kstar;
                int ex;
                const int tot = block_excl_scan(sel ? 1 : 0, &ex, sh_warp);
                if (sel && run + ex < K) out[run + ex] = out_index(a, b, key_index(stage[p]));
                run += tot;
            }
            for (int i = run + tid; i < K; i += kThreads) out[i] = -1;  // only if inconsistent
            return;
        }
    } else {
        // too many candidates to stage: the tie keys straight from the tiles
        for (int ti = warp; ti < ntiles; ti += kThreads / 32) {
            const unsigned long long* ct = cb + (size_t)ti * kSelTile;
            for (int i = lane; i < cnt[ti]; i += 32) {
                const unsigned long long k = __ldcg(ct + i);
                if ((int)((k >> 32) >> shift) == t) {
                    const int q = atomicAdd(&s_nt, 1);
                    if (q < kMaxTies) ties[q] = k;
                }
            }
        }
        __syncthreads();
        const int nt = s_nt;
        if (nt <= kMaxTies) {
            int p2 = 1;
            while (p2 < nt) p2 <<= 1;
            for (int i = nt + tid; i < p2; i += kThreads) ties[i] = 0ull;
            __syncthreads();
            block_bitonic(ties, p2, true);
            if (tid == 0) s_kstar = (r >= 1 && r <= nt) ? ties[r - 1] : ~0ull;
            __syncthreads();
            const unsigned long long kstar = s_kstar;
            // winners per tile, prefix over tiles, then write in index order
            for (int ti = warp; ti < ntiles; ti += kThreads / 32) {
                const unsigned long long* ct = cb + (size_t)ti * kSelTile;
                int c = 0;
                for (int i = lane; i < cnt[ti]; i += 32) c += __ldcg(ct + i) >= kstar;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
                if (lane == 0) off[ti] = c;
            }
            __syncthreads();
            int run = 0;
            for (int base = 0; base < ntiles; base += kThreads) {
                const int i = base + tid;
                const int c = i < ntiles ? off[i] : 0;
                int ex;
                const int tot = block_excl_scan(c, &ex, sh_warp);
                if (i < ntiles) off[i] = run + ex;
                run += tot;
                __syncthreads();
            }
            for (int ti = warp; ti < ntiles; ti += kThreads / 32) {
                const unsigned long long* ct = cb + (size_t)ti * kSelTile;
                int o = off[ti];
                for (int i0 = 0; i0 < cnt[ti]; i0 += 32) {
                    const int i = i0 + lane;
                    const unsigned long long k = i < cnt[ti] ? __ldcg(ct + i) : 0ull;
                    const bool sel = i < cnt[ti] && k >= kstar;
                    const unsigned m = __ballot_sync(0xffffffffu, sel);
                    const int p = o + __popc(m & ((1u << lane) - 1u));
                    if (sel && p < K) out[p] = out_index(a, b, key_index(k));
                    o += __popc(m);
                }
            }
            __syncthreads();
            for (int i = run + tid; i < K; i += kThreads) out[i] = -1;  // only if inconsistent
            return;
        }
    }

    finish_heavy(a, b, bias, shift, t, r, smem);
}

// A score read from L2 that the compiler may neither drop nor issue again
// later (keeping it in a register instead of re-reading it where it is used).
__device__ __forceinline__ int ld_score(const int32_t* p) {
    int v;
    asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__global__ void __launch_bounds__(kThreads)
topk_select_kernel(TopkArgs a, int bias, int shift) {
    extern __shared__ __align__(16) unsigned char fsmem[];
    __shared__ int sh_warp[kThreads / 32];
    __shared__ int s_last;
    constexpr int PER = kSelTile / kThreads;     // scores per thread (32)
    constexpr int WROWS = kSelTile / (kThreads / 32);  // rows per warp (1024)
    pdl_wait();
    const int b = blockIdx.y, K = a.topk, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int n = a.n_entries[b];
    if (n < 0 || n > a.capacity || n <= K) {  // nothing to select: all or nothing
        if (blockIdx.x == 0) finish_sequence(a, b, bias, shift, fsmem);
        return;
    }
    const int ntiles = (n + kSelTile - 1) / kSelTile;
    const int tile = blockIdx.x;
    if (tile >= ntiles) return;
    const int t = __ldcg(a.thr + 2 * b);
    const int32_t* sc = a.scores + (size_t)b * a.capacity;
    const int ctiles = sel_tiles(a.capacity);
    unsigned long long* cand = a.cands + ((size_t)b * ctiles + tile) * kSelTile;
    // warp w owns rows [w*1024, (w+1)*1024) of the tile; lane l reads rows
    // i*32 + l, so every load of the warp is one contiguous 128-byte line
    const int r0 = tile * kSelTile + warp * WROWS + lane;
    int v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = (r0 + 32 * i < n) ? ld_score(sc + r0 + 32 * i) : 0;
    unsigned take = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i)
        if (r0 + 32 * i < n && score_bin(v[i], bias, shift) >= t) take |= 1u << i;
    int wc = __popc(take);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) wc += __shfl_xor_sync(0xffffffffu, wc, o);
    if (lane == 0) sh_warp[warp] = wc;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        base += w < warp ? sh_warp[w] : 0;
        total += sh_warp[w];
    }
    // compact in index order: row-major over (i, lane) inside the warp
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const unsigned m = __ballot_sync(0xffffffffu, (take >> i) & 1u);
        if ((take >> i) & 1u) cand[base + __popc(m & lt)] = make_key(v[i], r0 + 32 * i, bias);
        base += __popc(m);
    }
    if (tid == 0) a.tile_count[(size_t)b * ctiles + tile] = total;
    // the sequence's last tile CTA (a fenced counter; nobody waits) finishes it
    __threadfence();
    __syncthreads();
    if (tid == 0)
        s_last = atomicAdd(a.counters + (size_t)a.batch * (kBins + 1) + b, 1) == ntiles - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) a.counters[(size_t)a.batch * (kBins + 1) + b] = 0;  // zeroed for the next call
    finish_sequence(a, b, bias, shift, fsmem);
}


// ---- selection inside one thread-block cluster per sequence
//
// When a sequence's scores span at most kClusterTiles tiles of 256 x PER
// scores, its tile CTAs form one cluster and finish the selection together,
// without a second pass through global memory or a last-CTA hand-off:
//  a. each CTA compacts its keys of bins >= t, in index order, into its own
//     shared memory (a tile with more than kCandCap of them writes them to its
//     global candidate slot instead) and stores its counts and up to
//     kTieSlots keys of bin t into every CTA of the cluster (distributed
//     shared memory: a slot per tile);
//  b. after one cluster barrier every CTA holds every count and tie key in
//     its own shared memory and derives the same cut-off key k* (the tie of
//     rank r - 1 among all ties, each tie's rank counted by one thread), and
//     with it how many winners the lower tiles hold;
//  c. each CTA writes its own winners (keys >= k*: every key above bin t, and
//     the ties from k* up) at that offset, in index order.
// More than kTieSlots ties in the sequence: every CTA gathers the bin-t keys
// of all tiles and sorts them in a block; more than kMaxTies: the first CTA
// runs the second-histogram pass over the stored scores alone.
constexpr int kClusterTiles = 8;
constexpr int kTieSlots = 128;
constexpr int kCandCap = 4096;
constexpr size_t kClusterSmem = (size_t)kCandCap * 8 + (size_t)kMaxTies * 8 +
                                (size_t)kClusterTiles * kTieSlots * 8;

__device__ __forceinline__ uint32_t cta_smem(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
// Address of the same shared variable in cluster CTA `rank`.
__device__ __forceinline__ uint32_t peer_smem(uint32_t addr, int rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ unsigned long long ld_peer_u64(uint32_t addr) {
    unsigned long long v;
    asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_peer_s32(uint32_t addr, int v) {
    asm volatile("st.shared::cluster.s32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_peer_u64(uint32_t addr, unsigned long long v) {
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}
// Cluster barrier halves.  Every thread of every CTA of the cluster executes
// each the same number of times, in arrive/wait pairs.
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int PER>
__global__ void __launch_bounds__(kThreads, PER <= 32 ? 3 : 2)
topk_select_cluster_kernel(TopkArgs a, int bias, int shift) {
    extern __shared__ __align__(16) unsigned char csmem[];
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(csmem);  // kCandCap
    unsigned long long* ties = cand + kCandCap;                                // kMaxTies
    unsigned long long* inbox = ties + kMaxTies;  // [kClusterTiles][kTieSlots]: tiles' ties
    __shared__ int sh_warp[kThreads / 32];
    __shared__ int in_cnt[kClusterTiles], in_nt[kClusterTiles];  // written by every tile
    __shared__ int s_nt, s_ng, s_lo, s_all;
    __shared__ unsigned long long s_kstar;
    constexpr int TILE = kThreads * PER;          // scores per CTA
    constexpr int WROWS = TILE / (kThreads / 32);  // rows per warp
    pdl_wait();
    const int b = blockIdx.y, K = a.topk, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int tile = blockIdx.x, ranks = gridDim.x;  // one cluster spans gridDim.x tiles
    const int32_t* sc = a.scores + (size_t)b * a.capacity;
    // this tile's scores (a warp per WROWS rows, lane l reading rows i*32 + l),
    // requested together with the sequence's length and threshold
    const int r0 = tile * TILE + warp * WROWS + lane;
    int v[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = (r0 + 32 * i < a.capacity) ? ld_score(sc + r0 + 32 * i) : 0;
    const int n = a.n_entries[b];
    const int t = __ldcg(a.thr + 2 * b), above = __ldcg(a.thr + 2 * b + 1);
    if (n < 0 || n > a.capacity || n <= K) {  // the same for the whole cluster: no barrier
        if (tile == 0) finish_sequence(a, b, bias, shift, csmem);
        return;
    }
    // every CTA of the cluster has started once this barrier completes (it is
    // awaited just before the first store into another CTA's memory)
    cluster_arrive_relaxed();
    const int r = K - above;  // entries of bin t to take
    int32_t* out = a.topk_idx + (size_t)b * K;
    // this sequence's global candidate region (sized for the whole capacity)
    unsigned long long* gcand = a.cands + (size_t)b * sel_tiles(a.capacity) * kSelTile;
    if (tid == 0) {
        s_nt = 0;
        s_ng = 0;
        s_lo = 0;
        s_all = 0;
    }

    // a. this tile's keys of bins >= t in index order; its ties to every CTA
    unsigned long long take = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i)
        if (r0 + 32 * i < n && score_bin(v[i], bias, shift) >= t) take |= 1ull << i;
    int wc = __popcll(take);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) wc += __shfl_xor_sync(0xffffffffu, wc, o);
    if (lane == 0) sh_warp[warp] = wc;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        base += w < warp ? sh_warp[w] : 0;
        total += sh_warp[w];
    }
    const unsigned lt = (1u << lane) - 1u;
    const bool spill = total > kCandCap;  // too many for shared memory: the global slot
    unsigned long long* gslot = gcand + (size_t)tile * TILE;
    const uint32_t a_inbox = cta_smem(inbox + tile * kTieSlots);
    // rows i that no lane of the warp takes (nearly all of them) cost one test
    const unsigned long long any =
        (unsigned long long)__reduce_or_sync(0xffffffffu, (unsigned)(take >> 32)) << 32 |
        __reduce_or_sync(0xffffffffu, (unsigned)take);
    cluster_wait_acquire();  // (the start barrier)
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (!((any >> i) & 1ull)) continue;  // warp-uniform
        const bool tk = (take >> i) & 1ull;
        const unsigned m = __ballot_sync(0xffffffffu, tk);
        if (tk) {
            const unsigned long long key = make_key(v[i], r0 + 32 * i, bias);
            const int pos = base + __popc(m & lt);
            if (spill) gslot[pos] = key;
            else cand[pos] = key;
        }
        base += __popc(m);
    }
    if (spill) __threadfence();
    __syncthreads();
    // this tile's keys of bin t, staged (any order) to be sent below in one
    // round: one shared-memory atomic per warp and pass
    {
        const unsigned long long* mine = spill ? gslot : cand;
        for (int p0 = 0; p0 < total; p0 += kThreads) {
            const int p = p0 + tid;
            const unsigned long long key = p < total ? mine[p] : 0ull;
            const bool tie = p < total && (int)((key >> 32) >> shift) == t;
            const unsigned m = __ballot_sync(0xffffffffu, tie);
            int q0 = 0;
            if (lane == 0 && m) q0 = atomicAdd(&s_nt, __popc(m));
            q0 = __shfl_sync(0xffffffffu, q0, 0);
            const int q = q0 + __popc(m & lt);
            if (tie && q < kTieSlots) ties[q] = key;
        }
    }
    __syncthreads();
    {  // this tile's counts and ties into every CTA (one store per thread)
        const int nt = s_nt, sent = min(nt, kTieSlots);
        for (int x = tid; x < ranks * (sent + 2); x += kThreads) {
            const int j = x % ranks, q = x / ranks;
            if (q < sent) st_peer_u64(peer_smem(a_inbox + 8u * q, j), ties[q]);
            else if (q == sent) st_peer_s32(peer_smem(cta_smem(in_cnt + tile), j), total);
            else st_peer_s32(peer_smem(cta_smem(in_nt + tile), j), nt);
        }
    }
    __syncthreads();
    cluster_arrive_release();  // every tile's counts and ties are in every CTA
    cluster_wait_acquire();

    // b. in every CTA: the cut-off key k*, the winners in lower tiles (this
    // CTA's output offset) and in all tiles
    int nt_all = 0, above_lo = 0, above_all = 0;
    for (int j = 0; j < ranks; ++j) {
        const int cj = in_cnt[j], nj = in_nt[j];
        nt_all += nj;
        above_all += cj - nj;
        if (j < tile) above_lo += cj - nj;
    }
    unsigned long long kstar = ~0ull;
    if (nt_all <= kTieSlots) {
        // thread i < nt_all takes tie i (tile j's slot i - (ties of tiles < j))
        // into a dense list, then counts the ties above it: the one with
        // r - 1 above is k*
        unsigned long long mine = 0ull;
        int src = 0;
        if (tid < nt_all) {
            int first = 0;
            while (tid >= first + in_nt[src]) first += in_nt[src++];
            mine = inbox[src * kTieSlots + (tid - first)];
            ties[tid] = mine;
        }
        for (int i = nt_all + tid; i < ((nt_all + 7) & ~7); i += kThreads) ties[i] = 0ull;
        __syncthreads();
        if (tid < nt_all) {
            int above_me = 0;
            for (int s2 = 0; s2 < nt_all; s2 += 8) {  // padding 0 counts nowhere
#pragma unroll
                for (int u = 0; u < 8; ++u) above_me += ties[s2 + u] > mine;
            }
            if (above_me == r - 1) s_kstar = mine;
            if (above_me < r) {
                atomicAdd(&s_all, 1);
                if (src < tile) atomicAdd(&s_lo, 1);
            }
        }
        __syncthreads();
        if (r >= 1 && r <= nt_all) kstar = s_kstar;
    } else if (nt_all <= kMaxTies) {
        // many ties: every CTA gathers the bin-t keys of all tiles and sorts them
        const uint32_t a_cand = cta_smem(cand);
        for (int j = 0; j < ranks; ++j) {
            const int cj = in_cnt[j];
            const uint32_t src = peer_smem(a_cand, j);
            const unsigned long long* gsrc = gcand + (size_t)j * TILE;
            for (int i = tid; i < cj; i += kThreads) {
                const unsigned long long key =
                    cj > kCandCap ? __ldcg(gsrc + i) : ld_peer_u64(src + 8u * (uint32_t)i);
                if ((int)((key >> 32) >> shift) == t) {
                    const int q = atomicAdd(&s_ng, 1);
                    if (q < kMaxTies) ties[q] = key;
                }
            }
        }
        __syncthreads();
        cluster_arrive_relaxed();  // no reads of the other CTAs' memory after this
        int p2 = 1;
        while (p2 < nt_all) p2 <<= 1;
        for (int i = nt_all + tid; i < p2; i += kThreads) ties[i] = 0ull;  // sorts last
        __syncthreads();
        block_bitonic(ties, p2, true);
        if (r >= 1 && r <= nt_all) kstar = ties[r - 1];
        int lo = 0, all = 0;
        for (int i = tid; i < nt_all; i += kThreads) {
            if (ties[i] >= kstar) {
                ++all;
                if (key_index(ties[i]) / TILE < tile) ++lo;
            }
        }
        if (lo) atomicAdd(&s_lo, lo);
        if (all) atomicAdd(&s_all, all);
        __syncthreads();
        cluster_wait_acquire();  // the other CTAs are done with this CTA's memory
    }
    if (nt_all > kMaxTies) {
        // heavy ties: the first CTA selects from the stored scores alone
        if (tile == 0) {
            finish_heavy(a, b, bias, shift, t, r, reinterpret_cast<unsigned char*>(ties));
            if (a.pool_len_out) {
                __syncthreads();
                if (tid == 0) store_pool_len(a, b, __ldcg(out + K - 1) == n - 1);
            }
        }
        return;
    }
    // c. this tile's winners (keys >= k*) in index order at its offset
    const int cnt = total;
    const unsigned long long* mine = spill ? gslot : cand;
    int run = above_lo + s_lo;
    for (int p0 = 0; p0 < cnt; p0 += kThreads) {
        const int p = p0 + tid;
        const unsigned long long key = p < cnt ? mine[p] : 0ull;
        const bool sel = p < cnt && key >= kstar;
        int ex;
        const int tot = block_excl_scan(sel ? 1 : 0, &ex, sh_warp);
        if (sel && run + ex < K) out[run + ex] = out_index(a, b, key_index(key));
        run += tot;
    }
    if (tile == 0) {  // only if the threshold was inconsistent: nothing chosen past `written`
        const int written = kstar == ~0ull ? 0 : above_all + s_all;
        for (int i = written + tid; i < K; i += kThreads) out[i] = -1;
    }
    if (a.pool_len_out && tile == (n - 1) / TILE && tid == 0) {
        const bool last = cnt > 0 && key_index(mine[cnt - 1]) == n - 1 && mine[cnt - 1] >= kstar;
        store_pool_len(a, b, last);
    }
}

}  // namespace

namespace {
template <int PER>
cudaError_t launch_cluster_select(const TopkArgs& a, int bias, int shift, int ranks,
                                  cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ranks, a.batch);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kClusterSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = ranks;  // the tiles of a sequence form one cluster
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, topk_select_cluster_kernel<PER>, a, bias, shift);
}
}  // namespace

cudaError_t launch_select(const TopkArgs& a, int bias, int shift, cudaStream_t s) {
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_set[64] = {};
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(
            topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFinishSmem);
        if (e != cudaSuccess) return e;
        void (*const ks[4])(TopkArgs, int, int) = {
            topk_select_cluster_kernel<32>, topk_select_cluster_kernel<40>,
            topk_select_cluster_kernel<48>, topk_select_cluster_kernel<64>};
        for (auto k : ks) {
            e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kClusterSmem);
            if (e != cudaSuccess) return e;
        }
        attr_set[dev] = true;
    }
    // one cluster per sequence when its tiles of 256 x PER scores number at
    // most 8: the smallest such PER of 32, 40, 48, 64
    const long long cap = a.capacity;
    auto tiles = [&](int per) {
        return std::max(1, (int)((cap + (long long)per * kThreads - 1) / ((long long)per * kThreads)));
    };
    trace_before("topk_select", s);
    cudaError_t err;
    if (tiles(32) <= kClusterTiles)
        err = launch_cluster_select<32>(a, bias, shift, tiles(32), s);
    else if (tiles(40) <= kClusterTiles)
        err = launch_cluster_select<40>(a, bias, shift, tiles(40), s);
    else if (tiles(48) <= kClusterTiles)
        err = launch_cluster_select<48>(a, bias, shift, tiles(48), s);
    else if (tiles(64) <= kClusterTiles)
        err = launch_cluster_select<64>(a, bias, shift, tiles(64), s);
    else
        err = launch_pdl(topk_select_kernel, dim3(std::max(1, sel_tiles(a.capacity)), a.batch), kThreads,
                         kFinishSmem, s, a, bias, shift);
    trace_after(s);
    return err;
}

}  // namespace kvc
