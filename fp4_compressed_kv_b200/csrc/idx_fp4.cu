// idx_fp4.cu -- indexer scoring and exact top-K over FP4 indexer keys.
//
// Method: "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
// 压缩到 890 B的？" (acejoy.com) part 3 breakthrough 4 (a lightweight indexer
// scores every history entry; the 512 best are attended) with the pages' FP4
// indexer K ("890 字节是怎么算出来的": 128 dims x 0.5 B plus 8 scales = 72 B).
// A key row holds di/2 E2M1 code bytes (channel 2c in the low nibble of byte
// c), then di/16 UE4M3 scales, one per 16 channels.  The score of an entry is
// the exact value of q . dequant(k): per group of 16, the integer sum of q_d
// times twice the E2M1 value (-12..12), times the group's scale times 2^9 (an
// integer for every UE4M3 value), summed over the groups -- the score times
// 2^10, in 64 bits (|.| < 2^39 for di <= 256).  So the selection stays exact.
//
// 128- and 256-channel keys (the fast path, the pages' 72-byte row and its
// double):
//  1. idx_fp4_scan_fast: CTA (x, b) scores 4096 rows of sequence b; a warp
//     stages blocks of 32 rows with coalesced 8-byte loads (the next block's
//     in flight) and each lane scores one row: byte permutes turn eight codes
//     into eight signed twice-values for two dp4a with the query; the group sum
//     times the scale's table value accumulates in 64 bits.  The row's 64-bit
//     key (score, then index) is stored and its bin -- 16 per octave of |S| --
//     counted; the sequence's last CTA derives the threshold bin.
//  2. idx_fp4_select_tiles: per tile of 8192 keys, those of bins >= t go to
//     candidate slots in index order.
//  3. idx_fp4_select_finish: per sequence, the candidates in index order, the
//     cut-off key among those of the threshold bin (ranked by counting, or
//     sorted), and the winners' rows in index order; an exact radix selection
//     over all keys when the candidates overflow.
// Other widths (16, 32, 64 channels) take a direct design: a thread per entry
// (byte loads) writes the score, then a CTA of 1024 threads per sequence finds
// the K-th best score by a radix selection over the 40-bit value score + 2^39
// (4 passes of 10 bits: a 1024-bin histogram of the entries that match the
// digits found so far, then a block prefix sum over the bins from the top),
// and one pass in index order takes the entries above that value and, lowest
// index first, as many equal to it as the K still need.
#include <algorithm>

#include "topk_common.cuh"

namespace kvc {
namespace {

constexpr int kSelThreads = 1024;  // one bin of the 1024-bin histogram per thread

// Twice the E2M1 value of a 4-bit code: magnitudes 0, 1, 2, 3, 4, 6, 8, 12.
__device__ __forceinline__ int e2m1_twice(int code) {
    const int m = code & 7;
    const int mag = m < 5 ? m : (m == 5 ? 6 : (m == 6 ? 8 : 12));
    return (code & 8) ? -mag : mag;
}

// 2^9 times the value of a UE4M3 byte (4 exponent bits, bias 7; 3 mantissa
// bits): m for exponent 0, (8 + m) 2^(e - 1) otherwise.
__device__ __forceinline__ long long ue4m3_times_512(int byte) {
    const int e = (byte >> 3) & 15, m = byte & 7;
    return e == 0 ? (long long)m : (long long)(8 + m) << (e - 1);
}

__global__ void __launch_bounds__(256)
idx_fp4_scan_direct_kernel(const int8_t* __restrict__ q, const uint8_t* __restrict__ rows,
                    const int32_t* __restrict__ n_entries, int batch, int capacity, int di,
                    int rb, long long* __restrict__ scores, uint32_t* status) {
    pdl_wait();
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;  // b * capacity + j
    if (t >= (long long)batch * capacity) return;
    const int b = (int)(t / capacity), j = (int)(t % capacity);
    const int n = n_entries[b];
    if (n < 0 || n > capacity) {
        if (j == 0) set_status(status, KVC_DEV_BAD_LENGTH);
        return;
    }
    if (j >= n) return;
    const uint8_t* row = rows + t * rb;
    const int8_t* qb = q + (long long)b * di;
    long long total = 0;
    for (int g = 0; g < di / 16; ++g) {
        int part = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int byte = __ldg(row + 8 * g + u);
            part += (int)__ldg(qb + 16 * g + 2 * u) * e2m1_twice(byte & 15) +
                    (int)__ldg(qb + 16 * g + 2 * u + 1) * e2m1_twice(byte >> 4);
        }
        total += (long long)part * ue4m3_times_512(__ldg(row + di / 2 + g));
    }
    scores[t] = total;
}

__global__ void __launch_bounds__(kSelThreads)
idx_fp4_select_direct_kernel(const long long* __restrict__ scores, const int32_t* __restrict__ n_entries,
                      int capacity, int K, int32_t* __restrict__ topk) {
    __shared__ int hist[kSelThreads];
    __shared__ int sh_warp[kSelThreads / 32];
    __shared__ int s_digit, s_above;
    pdl_wait();
    const int b = blockIdx.x, tid = threadIdx.x;
    const int n = n_entries[b];
    int32_t* out = topk + (long long)b * K;
    if (n < 0 || n > capacity) {
        for (int i = tid; i < K; i += kSelThreads) out[i] = -1;
        return;
    }
    if (n <= K) {  // every entry, then -1
        for (int i = tid; i < K; i += kSelThreads) out[i] = i < n ? i : -1;
        return;
    }
    const long long* sc = scores + (long long)b * capacity;
    const long long kBias = 1LL << 39;  // score + 2^39 lies in [0, 2^40)
    unsigned long long prefix = 0, mask = 0;
    int remaining = K;  // entries still to take among those matching the prefix
    for (int p = 0; p < 4; ++p) {
        const int shift = 30 - 10 * p;
        hist[tid] = 0;
        if (tid == 0) {
            s_digit = 0;
            s_above = 0;
        }
        __syncthreads();
        for (int j = tid; j < n; j += kSelThreads) {
            const unsigned long long v = (unsigned long long)(sc[j] + kBias);
            if ((v & mask) == prefix) atomicAdd(&hist[(v >> shift) & 1023], 1);
        }
        __syncthreads();
        // thread t owns bin 1023 - t: the exclusive sum counts the higher bins
        const int cnt = hist[kSelThreads - 1 - tid];
        int excl;
        block_excl_scan(cnt, &excl, sh_warp);
        if (excl < remaining && remaining <= excl + cnt) {
            s_digit = kSelThreads - 1 - tid;
            s_above = excl;
        }
        __syncthreads();
        remaining -= s_above;
        prefix |= (unsigned long long)s_digit << shift;
        mask |= 1023ull << shift;
        __syncthreads();  // every thread has read the histogram and the digit
    }
    // the K-th best value is `prefix`; `remaining` entries equal to it are taken
    const unsigned long long vt = prefix;
    const int need = remaining;
    int taken = 0, eq_seen = 0;
    for (int base = 0; base < n; base += kSelThreads) {
        const int j = base + tid;
        const unsigned long long v = j < n ? (unsigned long long)(sc[j] + kBias) : 0ull;
        const int is_eq = (j < n && v == vt) ? 1 : 0;
        int eq_before;
        const int eq_total = block_excl_scan(is_eq, &eq_before, sh_warp);
        const int take = (j < n) && (v > vt || (is_eq && eq_seen + eq_before < need));
        int pos;
        const int take_total = block_excl_scan(take, &pos, sh_warp);
        if (take && taken + pos < K) out[taken + pos] = j;
        taken += take_total;
        eq_seen += eq_total;
    }
    for (int i = taken + tid; i < K; i += kSelThreads) out[i] = -1;  // only if inconsistent
}

// ======================================================================
// Fast path (128- and 256-channel keys, rows of 72 / 144 bytes).
//
// Keys: the exact score S (the score times 2^10, |S| < 2^39) and the row j
// pack into one 64-bit key, (S + 2^39) << 24 | (2^24 - 1 - j), so a larger key
// is a better entry (score descending, index ascending) and no two are equal.
// Bins: an 11-bit function of S that never decreases as S grows -- sign,
// binary exponent of |S| and 4 bits below its leading one (16 bins per
// octave) -- so the K best keys lie in the bins at or above the threshold bin
// t of a 2048-bin histogram, and bin t holds a few hundred of them at most for
// any spread-out score distribution.
constexpr int kScanTile = 4096;        // rows per scan CTA: 8 warps x 16 blocks of 32
constexpr int kFinishCap = kSelTile;  // candidates the finish stages in shared memory
constexpr int kTileCands = kFp4TileCands;  // candidate slots per select tile
constexpr long long kKeyBias = 1LL << 39;

__device__ __forceinline__ int fp4_bin(long long S) {
    // |S| truncated to fp32 (never rounds up, so the bin never decreases as
    // |S| grows): its exponent and the 4 mantissa bits below the leading one;
    // 0 for S = 0, 16 .. 639 otherwise (|S| < 2^39)
    const uint32_t fb = __float_as_uint(__ll2float_rz(S < 0 ? -S : S));
    const int v = max(0, (int)(fb >> 19) - (127 << 4) + 16);
    return S < 0 ? 1023 - v : 1024 + v;
}
__device__ __forceinline__ unsigned long long fp4_key(long long S, int j) {
    return ((unsigned long long)(S + kKeyBias) << 24) | (unsigned long long)(0xFFFFFFu - (uint32_t)j);
}
__device__ __forceinline__ long long key_score(unsigned long long k) {
    return (long long)(k >> 24) - kKeyBias;
}
__device__ __forceinline__ int key_row(unsigned long long k) {
    return (int)(0xFFFFFFu - (uint32_t)(k & 0xFFFFFFull));
}

// Eight E2M1 codes (channel i in nibble i of w) as eight signed int8
// twice-values, channels 0-3 in lo and 4-7 in hi, by byte permutes: the
// magnitude index picks from a table of twice-magnitudes {0,1,2,3,4,6,8,12}
// and from its negation, then each byte comes from one or the other by its
// sign bit.  prmt.b32 in its default mode reads its selector from the low 16
// bits (bit 3 of a nibble would replicate the byte's sign, so every selector
// here has it clear); the high half's selectors are the shared masks shifted.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ void e2m1x8_twice(uint32_t w, uint32_t& lo, uint32_t& hi) {
    const uint32_t sel = w & 0x77777777u;                          // magnitude indexes
    const uint32_t pick = ((w >> 1) & 0x44444444u) | 0x32103210u;  // byte i or byte 4 + i
    const uint32_t sel_h = sel >> 16, pick_h = pick >> 16;
    lo = prmt(prmt(0x03020100u, 0x0C080604u, sel), prmt(0xFDFEFF00u, 0xF4F8FAFCu, sel), pick);
    hi = prmt(prmt(0x03020100u, 0x0C080604u, sel_h), prmt(0xFDFEFF00u, 0xF4F8FAFCu, sel_h),
              pick_h);
}

// idx_fp4_scan_fast: CTA (x, b) scores rows [4096 x, 4096 x + 4096) of
// sequence b.  A warp takes blocks of 32 rows: coalesced 8-byte loads (the
// next block's in flight during the arithmetic) into its shared-memory stage,
// then lane l scores row l from there -- per group of 16 channels four dp4a of
// decoded twice-values with the query (held in registers), times 2^9 times
// the group's UE4M3 scale, summed in 64 bits.  It stores the row's key and
// counts its bin; the sequence's last CTA (a fenced counter; nobody waits)
// derives the threshold bin t and the count above it.
template <int DI>
__global__ void __launch_bounds__(kThreads, DI == 128 ? 5 : 2)
idx_fp4_scan_fast(TopkArgs a, unsigned long long* __restrict__ keys) {
    constexpr int RB = DI / 2 + DI / 16;  // row bytes
    constexpr int RW = RB / 8;            // 8-byte words per row
    constexpr int NG = DI / 16;           // channel groups (one code word each)
    __shared__ __align__(16) unsigned long long stage[kThreads / 32][32 * RW];
    __shared__ __align__(16) uint32_t qs[DI / 4];
    __shared__ int s512[256];  // 2^9 times the value of each UE4M3 byte
    __shared__ int hist[kBins];
    __shared__ int sh_warp[kThreads / 32];
    __shared__ int s_last, s_t, s_above;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.y, cap = a.capacity;
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0;
    s512[tid] = (int)ue4m3_times_512(tid);  // kThreads = 256 bytes
    pdl_wait();
    const int n = a.n_entries[b];
    if (n < 0 || n > cap) {
        if (blockIdx.x == 0 && tid == 0) set_status(a.status, KVC_DEV_BAD_LENGTH);
        return;
    }
    const int r0 = blockIdx.x * kScanTile;
    if (r0 >= n) return;  // the sequence's CTAs are the first ceil(n / 4096)
    const int rend = min(r0 + kScanTile, n);
    if (tid < DI / 4) qs[tid] = __ldg(reinterpret_cast<const uint32_t*>(a.idx_q + (size_t)b * DI) + tid);
    __syncthreads();  // histogram zeroed, tables and query staged
    const unsigned long long* src =
        reinterpret_cast<const unsigned long long*>(a.idx_k + (size_t)b * a.idx_capacity * RB);
    unsigned long long pre[RW];
    auto fetch = [&](int rb0) {  // rows [rb0, rb0 + 32): word k * 32 + lane of the block
        if (rb0 + 32 <= rend) {
#pragma unroll
            for (int k = 0; k < RW; ++k) pre[k] = __ldcs(src + (size_t)rb0 * RW + k * 32 + lane);
        } else {
#pragma unroll
            for (int k = 0; k < RW; ++k) {
                const int w = k * 32 + lane;
                pre[k] = rb0 + w / RW < rend ? __ldcs(src + (size_t)rb0 * RW + w) : 0ull;
            }
        }
    };
    unsigned long long* st = stage[warp];
    int blk = r0 + 32 * warp;
    if (blk < rend) fetch(blk);
    for (; blk < rend; blk += 32 * (kThreads / 32)) {
#pragma unroll
        for (int k = 0; k < RW; ++k) st[k * 32 + lane] = pre[k];
        __syncwarp();
        if (blk + 256 < rend) fetch(blk + 256);
        const int j = blk + lane;
        if (j < rend) {
            const uint2* row = reinterpret_cast<const uint2*>(st + lane * RW);
            long long S = 0;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const uint2 cw = row[g];
                const uint4 qg = reinterpret_cast<const uint4*>(qs)[g];  // (broadcast)
                uint32_t c0, c1, c2, c3;
                e2m1x8_twice(cw.x, c0, c1);
                e2m1x8_twice(cw.y, c2, c3);
                int part = __dp4a((int)c0, (int)qg.x, 0);
                part = __dp4a((int)c1, (int)qg.y, part);
                part = __dp4a((int)c2, (int)qg.z, part);
                part = __dp4a((int)c3, (int)qg.w, part);
                const uint2 sw = row[NG + (g >> 3)];
                const uint32_t sword = (g & 4) ? sw.y : sw.x;
                S += (long long)part * s512[(sword >> (8 * (g & 3))) & 0xFFu];
            }
            keys[(size_t)b * cap + j] = fp4_key(S, j);
            atomicAdd(&hist[fp4_bin(S)], 1);
        }
        __syncwarp();  // the stage is rewritten by the next block
    }
    __syncthreads();
    if (n > a.topk) {
        int32_t* gh = a.counters + (size_t)b * kBins;
        for (int i = tid; i < kBins; i += kThreads)
            if (hist[i]) atomicAdd(&gh[i], hist[i]);
        __threadfence();
        __syncthreads();
        const int ntiles = (n + kScanTile - 1) / kScanTile;
        if (tid == 0)
            s_last = atomicAdd(a.counters + (size_t)a.batch * kBins + b, 1) == ntiles - 1;
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int i = tid; i < kBins; i += kThreads) {
                hist[i] = __ldcg(gh + i);
                gh[i] = 0;  // left zeroed for the next call
            }
            if (tid == 0) {
                a.counters[(size_t)a.batch * kBins + b] = 0;
                s_t = s_above = 0;
            }
            __syncthreads();
            find_threshold(hist, a.topk, &s_t, &s_above, sh_warp);
            if (tid == 0) {
                a.thr[2 * b] = s_t;
                a.thr[2 * b + 1] = s_above;
            }
        }
    }
    pdl_trigger();
}

// Descending bitonic sort of p (a power of two) keys in shared memory; every
// thread of the block calls it.
__device__ __forceinline__ void bitonic_desc(unsigned long long* k, int p) {
    for (int size = 2; size <= p; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = threadIdx.x; i < p; i += blockDim.x) {
                const int j = i ^ stride;
                if (j > i) {
                    const bool desc = (i & size) == 0;
                    const unsigned long long x = k[i], y = k[j];
                    if ((x < y) == desc) {
                        k[i] = y;
                        k[j] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// idx_fp4_select_tiles: CTA (x, b) takes tile x (8192 keys) of sequence b:
// the keys of bins >= t go, in index order, to the tile's candidate slots (at
// most kTileCands; a warp per 1024 keys, ballot prefix sums), and their count
// (-1: too many) to tile_count.
__global__ void __launch_bounds__(kThreads)
idx_fp4_select_tiles(TopkArgs a, const unsigned long long* __restrict__ keys) {
    extern __shared__ __align__(16) unsigned long long sk[];  // [kSelTile]
    __shared__ int sh_warp[kThreads / 32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.y, tile = blockIdx.x, cap = a.capacity, K = a.topk;
    pdl_wait();
    const int n = a.n_entries[b];
    if (n < 0 || n > cap || n <= K) return;  // (the finish writes these outputs)
    const int ntiles = (n + kSelTile - 1) / kSelTile;
    if (tile >= ntiles) return;
    const int t = a.thr[2 * b];
    const unsigned long long* tk = keys + (size_t)b * cap + (size_t)tile * kSelTile;
    const int tiles = sel_tiles(cap);
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(a.scores) +
                               ((size_t)b * tiles + tile) * kTileCands;
    const int tn = min(kSelTile, n - tile * kSelTile);
    uint32_t take = 0;
    for (int r0 = 0; r0 < 32; r0 += 16) {  // 16 loads in flight per lane
        unsigned long long kv[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int i = warp * 1024 + (r0 + u) * 32 + lane;
            kv[u] = i < tn ? __ldcg(tk + i) : 0ull;
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            const int i = warp * 1024 + (r0 + u) * 32 + lane;
            if (i < tn) {
                sk[i] = kv[u];
                if (fp4_bin(key_score(kv[u])) >= t) take |= 1u << (r0 + u);
            }
        }
    }
    int cnt = 0;
    for (int r = 0; r < 32; ++r) cnt += __popc(__ballot_sync(0xffffffffu, (take >> r) & 1u));
    if (lane == 0) sh_warp[warp] = cnt;  // the warps' counts: offsets and total
    __syncthreads();
    int wbase = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        const int c = sh_warp[w];
        wbase += w < warp ? c : 0;
        total += c;
    }
    if (total <= kTileCands) {
        const uint32_t lt = (1u << lane) - 1u;
        int pos = wbase;
        for (int r = 0; r < 32; ++r) {
            const uint32_t bal = __ballot_sync(0xffffffffu, (take >> r) & 1u);
            if ((take >> r) & 1u) cand[pos + __popc(bal & lt)] = sk[warp * 1024 + r * 32 + lane];
            pos += __popc(bal);
        }
    }
    if (tid == 0) a.tile_count[(size_t)b * tiles + tile] = total <= kTileCands ? total : -1;
    pdl_trigger();
}

// idx_fp4_select_finish: CTA b gathers sequence b's candidates, tile by tile
// (so in index order), into shared memory, finds the cut-off key k* -- the
// (K - above)-th best of the candidates in bin t, by counting larger keys for
// up to 1024 of them, else by a bitonic sort -- and writes the rows of the
// keys >= k* in index order.  A tile with too many candidates, more than
// kFinishCap in all or more than kMaxTies in bin t: the exact radix selection
// over all the sequence's keys instead.
__global__ void __launch_bounds__(kThreads)
idx_fp4_select_finish(TopkArgs a, const unsigned long long* __restrict__ keys) {
    extern __shared__ __align__(16) unsigned long long sk[];  // [kSelTile] | ties [kMaxTies]
    unsigned long long* tie = sk + kSelTile;
    __shared__ int sh_warp[kThreads / 32];
    __shared__ int hist[256];
    __shared__ int s_digit, s_above;
    const int tid = threadIdx.x;
    const int b = blockIdx.x, cap = a.capacity, K = a.topk;
    pdl_wait();
    const int n = a.n_entries[b];
    int32_t* out = a.topk_idx + (size_t)b * K;
    if (n < 0 || n > cap || n <= K) {  // a bad length: -1s; at most K entries: all of them
        for (int i = tid; i < K; i += kThreads) out[i] = (n >= 0 && n <= cap && i < n) ? i : -1;
        return;
    }
    const int ntiles = (n + kSelTile - 1) / kSelTile, tiles = sel_tiles(cap);
    const int t = a.thr[2 * b], above = a.thr[2 * b + 1];
    const unsigned long long* seq = keys + (size_t)b * cap;
    const int32_t* tcnt = a.tile_count + (size_t)b * tiles;
    int* cnt_s = reinterpret_cast<int*>(tie);  // tile counts, then offsets (ntiles <= 1024)
    for (int i = tid; i < ntiles; i += kThreads) cnt_s[i] = __ldcg(tcnt + i);
    __syncthreads();
    int tot = 0;
    bool exact = false;
    for (int i = 0; i < ntiles; ++i) {
        const int c = cnt_s[i];
        exact |= c < 0;
        tot += c;
    }
    unsigned long long kstar = 0;
    exact |= tot > kFinishCap;
    if (!exact) {
        int off = 0;
        const unsigned long long* sc =
            reinterpret_cast<const unsigned long long*>(a.scores) + (size_t)b * tiles * kTileCands;
        for (int i = 0; i < ntiles; ++i) {  // (independent loads: no global value steers them)
            const int c = cnt_s[i];
            for (int k = tid; k < c; k += kThreads) sk[off + k] = __ldcg(sc + (size_t)i * kTileCands + k);
            off += c;
        }
        __syncthreads();  // (also: every thread has read the counts before tie[] is reused)
        int m = 0;  // candidates of bin t, in index order, into tie[]
        for (int base = 0; base < tot; base += kThreads) {
            const int i = base + tid;
            const int f = (i < tot && fp4_bin(key_score(sk[i])) == t) ? 1 : 0;
            int ex;
            const int ft = block_excl_scan(f, &ex, sh_warp);
            if (f && m + ex < kMaxTies) tie[m + ex] = sk[i];
            m += ft;
        }
        const int r = K - above;  // entries of bin t taken
        exact = m > kMaxTies || r < 1 || r > m;
        if (!exact && m <= 1024) {
            // the key with exactly r - 1 larger ones among the m (distinct) keys
            __syncthreads();
            if (tid == 0) s_digit = 0;
            __syncthreads();
            for (int i = tid; i < m; i += kThreads) {
                const unsigned long long x = tie[i];
                int larger = 0;
                for (int k = 0; k < m; ++k) larger += tie[k] > x;
                if (larger == r - 1) {
                    tie[kMaxTies - 1] = x;  // (m <= 1024: the slot is free)
                    s_digit = 1;
                }
            }
            __syncthreads();
            kstar = tie[kMaxTies - 1];
        } else if (!exact) {
            int P = 1;
            while (P < m) P <<= 1;
            for (int i = m + tid; i < P; i += kThreads) tie[i] = 0ull;  // below every key
            __syncthreads();
            bitonic_desc(tie, P);
            kstar = tie[r - 1];
        }
    }
    // ---- exact path: the K-th largest of the n distinct keys by a radix
    // selection over the 64 key bits, 8 at a time (a 256-bin histogram of the
    // keys that match the digits found so far, then a prefix sum over the bins
    // from the top)
    if (exact) {
        unsigned long long prefix = 0, mask = 0;
        int remaining = K;
        for (int p = 7; p >= 0; --p) {
            const int shift = 8 * p;
            hist[tid] = 0;
            __syncthreads();
            for (int j = tid; j < n; j += kThreads) {
                const unsigned long long k = __ldcg(seq + j);
                if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255], 1);
            }
            __syncthreads();
            const int cnt = hist[255 - tid];  // thread t owns bin 255 - t: higher bins first
            int excl;
            block_excl_scan(cnt, &excl, sh_warp);
            if (excl < remaining && remaining <= excl + cnt) {
                s_digit = 255 - tid;
                s_above = excl;
            }
            __syncthreads();
            remaining -= s_above;
            prefix |= (unsigned long long)s_digit << shift;
            mask |= 255ull << shift;
            __syncthreads();  // every thread has read the digit before the next pass
        }
        kstar = prefix;
    }
    // the winners, keys >= k*, in index order (a key's row is its index)
    const unsigned long long* src = exact ? seq : sk;
    const int len = exact ? n : tot;
    int taken = 0;
    for (int base = 0; base < len; base += kThreads) {
        const int i = base + tid;
        const unsigned long long k = i < len ? src[i] : 0ull;
        const int w = (i < len && k >= kstar) ? 1 : 0;
        int ex;
        const int wt = block_excl_scan(w, &ex, sh_warp);
        if (w && taken + ex < K) out[taken + ex] = key_row(k);
        taken += wt;
    }
    for (int i = taken + tid; i < K; i += kThreads) out[i] = -1;
}
}  // namespace

cudaError_t launch_index_topk_fp4(const TopkArgs& a, int idx_rb, long long* scores64,
                                  cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    const long long rows = (long long)a.batch * a.capacity;
    cudaError_t err;
    if (a.di == 128 || a.di == 256) {  // the fast path: keys and the threshold bins
        unsigned long long* keys = reinterpret_cast<unsigned long long*>(scores64);
        if (rows > 0) {
            const dim3 g((unsigned)((a.capacity + kScanTile - 1) / kScanTile), (unsigned)a.batch);
            trace_before("index_scan_fp4", s);
            err = a.di == 128 ? launch_pdl(idx_fp4_scan_fast<128>, g, kThreads, 0, s, a, keys)
                              : launch_pdl(idx_fp4_scan_fast<256>, g, kThreads, 0, s, a, keys);
            trace_after(s);
            if (err != cudaSuccess) return err;
        }
        const size_t smem_t = (size_t)kSelTile * sizeof(unsigned long long);
        const size_t smem_f = (size_t)(kSelTile + kMaxTies) * sizeof(unsigned long long);
        err = cudaFuncSetAttribute(idx_fp4_select_tiles,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_t);
        if (err != cudaSuccess) return err;
        err = cudaFuncSetAttribute(idx_fp4_select_finish,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_f);
        if (err != cudaSuccess) return err;
        const dim3 g((unsigned)std::max(1, sel_tiles(a.capacity)), (unsigned)a.batch);
        trace_before("topk_select_fp4", s);
        err = launch_pdl(idx_fp4_select_tiles, g, kThreads, smem_t, s, a,
                         static_cast<const unsigned long long*>(keys));
        if (err == cudaSuccess)
            err = launch_pdl(idx_fp4_select_finish, (unsigned)a.batch, kThreads, smem_f, s, a,
                             static_cast<const unsigned long long*>(keys));
        trace_after(s);
        return err;
    }
    if (rows > 0) {
        trace_before("index_scan_fp4", s);
        err = launch_pdl(idx_fp4_scan_direct_kernel, (unsigned)((rows + 255) / 256), 256, 0, s,
                         a.idx_q, reinterpret_cast<const uint8_t*>(a.idx_k), a.n_entries,
                         a.batch, a.capacity, a.di, idx_rb, scores64, a.status);
        trace_after(s);
        if (err != cudaSuccess) return err;
    }
    trace_before("topk_select_fp4", s);
    err = launch_pdl(idx_fp4_select_direct_kernel, (unsigned)a.batch, kSelThreads, 0, s,
                     static_cast<const long long*>(scores64), a.n_entries, a.capacity, a.topk,
                     a.topk_idx);
    trace_after(s);
    return err;
}

}  // namespace kvc
