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
// A first, direct design:
//  1. idx_fp4_scan: a thread per entry reads its row (byte loads: a row need
//     not be 4-byte aligned) and the sequence's query, and writes the score.
//  2. idx_fp4_select: a CTA of 1024 threads per sequence finds the K-th best
//     score by a radix selection over the 40-bit value score + 2^39 (4 passes
//     of 10 bits: a 1024-bin histogram of the entries that match the digits
//     found so far, then a block prefix sum over the bins from the top), and
//     one pass in index order takes the entries above that value and, lowest
//     index first, as many equal to it as the K still need.
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
idx_fp4_scan_kernel(const int8_t* __restrict__ q, const uint8_t* __restrict__ rows,
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
idx_fp4_select_kernel(const long long* __restrict__ scores, const int32_t* __restrict__ n_entries,
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

}  // namespace

cudaError_t launch_index_topk_fp4(const TopkArgs& a, int idx_rb, long long* scores64,
                                  cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    const long long rows = (long long)a.batch * a.capacity;
    cudaError_t err;
    if (rows > 0) {
        trace_before("index_scan_fp4", s);
        err = launch_pdl(idx_fp4_scan_kernel, (unsigned)((rows + 255) / 256), 256, 0, s, a.idx_q,
                         reinterpret_cast<const uint8_t*>(a.idx_k), a.n_entries, a.batch,
                         a.capacity, a.di, idx_rb, scores64, a.status);
        trace_after(s);
        if (err != cudaSuccess) return err;
    }
    trace_before("topk_select_fp4", s);
    err = launch_pdl(idx_fp4_select_kernel, (unsigned)a.batch, kSelThreads, 0, s,
                     static_cast<const long long*>(scores64), a.n_entries, a.capacity, a.topk,
                     a.topk_idx);
    trace_after(s);
    return err;
}

}  // namespace kvc
