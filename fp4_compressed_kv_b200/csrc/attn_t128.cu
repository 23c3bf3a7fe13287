// attn_t128.cu -- sparse decode attention on the 5th-generation tensor cores
// for the MLA shape: 64 query heads sharing 576-channel entries (512 latent +
// 64 RoPE), values = the latent channels.
//
// Method: "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
// 压缩到 890 B的？" (acejoy.com) part 3 breakthrough 2 (every head reads the
// same latent entry, up-projections absorbed), breakthrough 4 (the 512
// selected entries plus a 128-token window), part 4 "P4 main KV" (FP4 is
// dequantised before attention).  One softmax runs jointly over the selected
// entries and the window keys.
//
// The key axis is the MMA's M dimension: a chunk of 128 keys against all 64
// heads is one M = 128, N = 64 product, with no padding rows.
//  1. A CTA owns either record chunks or the window chunk of one sequence.
//     Record chunks run with f16 operands: every dequantised entry is exact in
//     f16, and each head's query row is scaled by a power of two into the f16
//     range (the softmax undoes it).  The window chunk runs with bf16
//     operands: its query tile and key rows arrive by TMA (128B-swizzled
//     boxes) without passing through registers.  FP8 window rows are decoded
//     to their exact E4M3 values; each row's scale is applied to its logits
//     and to its probabilities, not to the stored tile.
//  2. A record chunk's keys are written into a 128B-swizzled K tile (9 atoms
//     of 64 channels x 128 keys): the selected records are loaded into
//     registers (16-byte loads, all in flight while the query tile is
//     converted), their E2M1 codes converted in hardware and multiplied by
//     the f16 group scale.  Thread = (key, half row): a warp's 16-byte stores
//     cover 8 swizzle slots x 4 rows, the minimum 4 wavefronts.
//  3. One thread issues S^T = K Q^T: 36 tcgen05.mma (M = 128 keys, N = 64
//     heads, K = 16) into tensor memory.
//  4. Warps 0-3 (thread = key = tensor-memory lane) read their key's 64
//     scores, take each head's chunk maximum with warp max-reductions, move a
//     head's reference only when its maximum passes it by more than 2^8 (the
//     accumulated O^T is rescaled in tensor memory then), and write P^T (key
//     rows of 64 heads) over the RoPE atom of the K tile, which the QK product
//     no longer reads.  Row sums are column sums of that same rounded P^T.
//  5. One thread issues O^T += V^T P^T: the latent atoms of the K tile read as
//     an MN-major operand, 4 x 8 tcgen05.mma (M = 128 channels, N = 64 heads,
//     K = 16 keys) into tensor memory.  A second record chunk's loads are in
//     flight while this product runs.
//  6. The CTAs of a sequence (at most 8) form a thread-block cluster; CTA r
//     owns heads [r*HG/n, (r+1)*HG/n) of the group.  After a cluster barrier
//     each CTA stores its unnormalised O columns (from tensor memory) and its
//     (m, l) straight into the owners' freed K tiles over distributed shared
//     memory; after a second barrier every owner weights the rows by
//     2^(m - max m), sums them in split order and writes the normalised
//     output.  More CTAs per sequence: attn_merge.
// Every wait on an mbarrier is bounded; on expiry the CTA sets
// KVC_DEV_TIMEOUT, waits (bounded) for the copies and products it issued,
// frees its tensor memory and returns.
#include <algorithm>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <mutex>

#include "kvc_internal.cuh"
#include "tc05_common.cuh"

namespace kvc {
namespace t128 {

using namespace tc;

constexpr int H = 64, D = 576, DV = 512, CK = 128, NT = 256;
constexpr int NATOM = D / 64;                        // 9 channel atoms of 64
constexpr uint32_t Q_ATOM = H * 128;                 // 64 rows x 128 B
constexpr uint32_t K_ATOM = CK * 128;                // 128 rows x 128 B
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + NATOM * Q_ATOM;   // 73,728
constexpr uint32_t OFF_P = OFF_K + 8 * K_ATOM;       // the RoPE atom, P^T after QK
constexpr uint32_t OFF_MISC = OFF_K + NATOM * K_ATOM;  // 221,184
// misc: kidx[128] i32 | qs[64] | mref[64] | lrun[64] | fac[64] | wmax[4][64] |
//       lpart[8][64] | ks[128] | bars[4] u64 | tmem slot | flags | ones (2 KB)
constexpr uint32_t M_KIDX = 0, M_QS = 512, M_MREF = 768, M_LRUN = 1024, M_FAC = 1280,
                   M_WMAX = 1536, M_LPART = 2560, M_KS = 4608, M_BARS = 5120, M_TSLOT = 5152,
                   M_FLAGS = 5168, M_ONES = 5248, MISC_BYTES = 7296;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0, L_COL = 64, O_COL = 256;  // S^T, L^T: 64 cols; O^T: 4 x 64
constexpr float kRescaleSlack = 8.0f;                // log2 units
enum { BAR_S = 0, BAR_O = 1, BAR_Q = 2, BAR_W = 3 };

// ---- TMA and bulk copies (non-multicast, into this CTA's shared memory)
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// The query tile of a record CTA, landed by TMA as bf16, converted in place to
// f16 with a per-head power of two that puts the row maximum in [2^14,
// 2^15); the head's softmax multiplier qs[h] absorbs it.  Thread t: head t/4,
// channels [144 (t%4), +144) as 18 16-byte pieces (the same swizzled
// positions the TMA wrote; a warp's accesses take the minimum 4 wavefronts).
__device__ __forceinline__ void convert_q_f16(const AttnArgs& a, float sm_log2, uint32_t sQ,
                                              uint32_t q_atom, float* qs, int tid) {
    const int h = tid >> 2, qq = tid & 3;
    uint4 v[18];
#pragma unroll
    for (int i = 0; i < 18; ++i) {
        const int c16 = 18 * qq + i;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                     : "=r"(v[i].x), "=r"(v[i].y), "=r"(v[i].z), "=r"(v[i].w)
                     : "r"(sQ + (c16 >> 3) * q_atom + swz(h, c16 & 7)));
    }
    uint32_t amax = 0;  // max |x| as fp32 bits (integer order = float order)
#pragma unroll
    for (int i = 0; i < 18; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            amax = max(amax, (w[k] << 16) & 0x7FFFFFFFu);
            amax = max(amax, w[k] & 0x7FFF0000u);
        }
    }
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int k = 0;
    if (amax >= 0x7F800000u) {
        if (qq == 0) set_status(a.status, KVC_DEV_NONFINITE);
    } else if (amax != 0) {
        const int e = (int)(amax >> 23) - 127;  // floor(log2 amax) for normal values
        k = min(max(e - 14, -60), 113);
    }
    const float mul = __uint_as_float((uint32_t)(127 - k) << 23);
    if (qq == 0) qs[h] = sm_log2 * __uint_as_float((uint32_t)(127 + k) << 23);
#pragma unroll
    for (int i = 0; i < 18; ++i) {
        const int c16 = 18 * qq + i;
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            o[j] = pack_f16(__uint_as_float(w[j] << 16) * mul,
                            __uint_as_float(w[j] & 0xFFFF0000u) * mul);
        sts128(sQ + (c16 >> 3) * q_atom + swz(h, c16 & 7), o[0], o[1], o[2], o[3]);
    }
}

// Scale byte index of 8-channel piece (item i, word u) for groups of G:
// latent items 0..15, RoPE items 16..17 (groups restart at channel 512).
template <int G>
__device__ __host__ constexpr int scale_index(int i, int u) {
    return i < 16 ? (32 * i + 8 * u) / G : 512 / G + (32 * (i - 16) + 8 * u) / G;
}
template <int G>
constexpr int scale_vecs() {  // 16-byte loads covering the scale bytes
    return (512 / G + (64 + G - 1) / G + 15) / 16;
}

// Scale word (4 bytes at record offset 288 + 4 w) holding every scale of
// 32-channel item i: for groups of 8..128 channels an item's scales share
// one aligned word.
template <int G>
__device__ __host__ constexpr int scale_word(int i) {
    return scale_index<G>(i, 0) >> 2;
}
// A chunk's records, 8 threads per key: thread t = 8 q + sub takes keys
// q, q + 32, q + 64, q + 96 and of each the 32-channel items sub, sub + 8
// and (sub < 2) sub + 16 -- 16-byte loads where 8 adjacent lanes read 128
// contiguous bytes of one record -- with the scale word of each item.
struct RecRegs {
    uint4 cw[4][3];
    uint32_t sw[4][3];
};
template <int G>
__device__ __forceinline__ void load_records(const uint8_t* base, int rb, const int* kidx, int tid,
                                             RecRegs& r) {
    const int sub = tid & 7, q = tid >> 3;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int k = kidx[q + 32 * p];
        if (k < 0) continue;
        const uint8_t* rec = base + (size_t)k * rb;
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            const int i = sub + 8 * u;
            if (u == 2 && sub >= 2) break;
            r.cw[p][u] = ldg_nc(rec + 16 * i);
            r.sw[p][u] = __ldg(reinterpret_cast<const uint32_t*>(rec + 288) + scale_word<G>(i));
        }
    }
}
// ... dequantised into the K tile: codes times the f16 group scale (exact),
// or zeros for a masked key.  Key j = q + 32 p has j & 7 = q & 7 and item i =
// sub + 8 u has i & 1 = sub & 1, so a thread's 16-byte slots are fixed: only
// the atom and the 4 KB row block move.  A warp's stores (4 keys x 8 items)
// cover 8 swizzle slots x 4 atoms: the minimum 4 wavefronts.
template <int G>
__device__ __forceinline__ void store_records(const RecRegs& r, const int* kidx, uint32_t sK,
                                              int tid) {
    const int sub = tid & 7, q = tid >> 3;
    const uint32_t x7 = q & 7;
    const uint32_t base = sK + (uint32_t)(sub >> 1) * K_ATOM + (uint32_t)(q >> 3) * 1024u + x7 * 128u;
    uint32_t slot[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) slot[k] = ((4u * (sub & 1) + k) ^ x7) << 4;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const bool live = kidx[q + 32 * p] >= 0;
#pragma unroll
        for (int u = 0; u < 3; ++u) {
            if (u == 2 && sub >= 2) break;
            const int i = sub + 8 * u;
            const uint32_t row = base + (uint32_t)(4 * u) * K_ATOM + (uint32_t)p * 4096u;
            const uint32_t words[4] = {r.cw[p][u].x, r.cw[p][u].y, r.cw[p][u].z, r.cw[p][u].w};
            const int s0 = scale_index<G>(i, 0) & 3;  // the item's first scale byte
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t w[4] = {0u, 0u, 0u, 0u};
                if (live) {
                    const int sb = G >= 32 ? s0 : (s0 + (8 * k) / G);
                    const uint32_t byte = (r.sw[p][u] >> (8 * sb)) & 0xFFu;
                    e2m1x8_scaled(words[k], ue4m3_f16x2(byte), w);
                }
                sts128(row + slot[k], w[0], w[1], w[2], w[3]);
            }
        }
    }
}
__device__ __forceinline__ void zero_row_half(uint32_t sK, int s, int half) {
#pragma unroll 1
    for (int c16 = 36 * half; c16 < 36 * half + 36; ++c16)
        sts128(sK + (uint32_t)(c16 >> 3) * K_ATOM + swz(s, c16 & 7), 0u, 0u, 0u, 0u);
}

// The all-ones A operand of the row-sum product (128 rows x 16 keys), in the
// non-swizzled K-major layout: two 8x8 core matrices of 128 B along K, every
// 8-row group reading the same two (stride 0).  L^T = ONES x P^T puts each
// head's sum of its rounded weights in every lane of one tensor-memory tile.
__device__ __forceinline__ uint64_t ones_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | (1ull << 46);
}

template <int G>
__global__ void __launch_bounds__(NT, 1)
attn_t128_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_w,
                 const __grid_constant__ CUtensorMap tm_wr, AttnArgs a, Shape sh, int K,
                 float sm_log2, int rsplit, int cpr, int nsplit, int cluster, int HG, int WR,
                 unsigned long long wait_ns) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;  // 1024-byte alignment for the swizzle
    unsigned char* smem = smem_raw + (base - raw_base);
    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sP = base + OFF_P;
    unsigned char* misc = smem + OFF_MISC;
    int* kidx = reinterpret_cast<int*>(misc + M_KIDX);
    float* qs = reinterpret_cast<float*>(misc + M_QS);
    float* mref = reinterpret_cast<float*>(misc + M_MREF);
    float* lrun = reinterpret_cast<float*>(misc + M_LRUN);
    float* fac = reinterpret_cast<float*>(misc + M_FAC);
    int* wmax = reinterpret_cast<int*>(misc + M_WMAX);
    float* lpart = reinterpret_cast<float*>(misc + M_LPART);
    float* ks = reinterpret_cast<float*>(misc + M_KS);  // FP8 window: scale of each key row
    uint64_t* bars = reinterpret_cast<uint64_t*>(misc + M_BARS);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + M_TSLOT);
    int* flags = reinterpret_cast<int*>(misc + M_FLAGS);
    const uint32_t sOnes = base + OFF_MISC + M_ONES;
    const uint32_t bS = smem_u32(&bars[BAR_S]), bO = smem_u32(&bars[BAR_O]),
                   bQ = smem_u32(&bars[BAR_Q]), bW = smem_u32(&bars[BAR_W]);

    const int split = blockIdx.x, hg0 = blockIdx.y * HG, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int W = a.window_len;
    const int rc = (K + CK - 1) / CK;
    const uint32_t q_atom = (uint32_t)HG * 128u;  // Q atoms of HG rows, packed
    // this CTA's chunks: record chunks [c0, c1) or window chunk split - rsplit
    const bool win = split >= rsplit;
    const bool fp8 = win && a.win_fp8 != nullptr;
    const bool lmma = !fp8;  // row sums by the tensor core (FP8 rows: column sums)
    const int c0 = win ? split - rsplit : split * cpr;
    const int c1 = win ? min(c0 + 1, (W + CK - 1) / CK) : min(c0 + cpr, rc);
    const uint32_t idQK = idesc_f16(128, HG, win ? 1 : 0, 0, 0);
    const uint32_t idPV = idesc_f16(128, 64, win ? 1 : 0, 1, 1);
    const uint32_t idL = idesc_f16(128, 64, win ? 1 : 0, 0, 1);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars[i]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (tid < H) {
        mref[tid] = -INFINITY;
        lrun[tid] = 0.f;
        if (win) qs[tid] = sm_log2;
    }
    {  // the ones block (2 KB, read 256 B) of 1.0 in the chunk's operand type
        const uint32_t one = win ? 0x3F803F80u : 0x3C003C00u;
        asm volatile("st.shared.v2.u32 [%0], {%1, %1};\n" ::"r"(sOnes + 8 * tid), "r"(one));
    }
    __syncthreads();  // barriers initialised before any copy arrives on them
    // The query rows of this head group (bf16) by TMA: issued before the wait
    // when no kernel launched since the caller wrote q (inside a layer-group
    // step), else after it.  Record CTAs convert them in place.
    auto tma_q = [&]() {
        mbar_expect_tx(bQ, NATOM * q_atom);
        for (int at = 0; at < NATOM; ++at)
            tma_load_2d(sQ + at * q_atom, &tm_q, 64 * at, b * H + hg0, bQ);
    };
    if (a.q_ready && tid == 0) tma_q();
    pdl_wait();
    const int n = a.n_entries[b];
    const bool len_ok = n >= 0 && n <= a.capacity;
    if (!a.q_ready && tid == 0) tma_q();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;
    int nqk = 0, npv = 0, nw = 0;  // commits / copies issued (for the cleanup waits)
    int nq = 1;                    // query-tile copies issued on bQ
    const int s = tid & (CK - 1), half = tid >> 7;  // key and half row (window paths)
    const uint8_t* recs = a.records + (size_t)b * a.capacity * sh.rb;
    // ---- slot table of chunk c: record index, window row, or -1 (masked)
    auto slot_table = [&](int c) {
        if (tid < CK) {
            int k = -1;
            if (!win) {
                const int j = c * CK + tid;
                if (j < K) {
                    const int idx = a.topk_idx[(size_t)b * K + j];
                    if (a.topk_copy && hg0 == 0) a.topk_copy[(size_t)b * K + j] = idx;
                    if (len_ok && idx >= 0 && idx < n)
                        k = idx;
                    else if (idx != -1 && len_ok && hg0 == 0)
                        set_status(a.status, KVC_DEV_BAD_INDEX);
                }
            } else {
                const int r = c * CK + tid;
                if (r < W) k = r;
                if (fp8) ks[tid] = k >= 0 ? __ldg(a.win_scale + (size_t)b * a.window_stride + r) : 0.f;
            }
            kidx[tid] = k;
        }
        __syncthreads();
        return kidx[s];
    };
    // ---- a record chunk's rows into registers: in flight while the query
    // rows land and are converted (first chunk) or while the previous chunk's
    // PV runs
    RecRegs rr;
    int k = -1;
    if (c0 < c1) {
        k = slot_table(c0);
        if (!win) load_records<G>(recs, sh.rb, kidx, tid, rr);
    }
    if (!win && c0 < c1) {
        const bool got = warp == 0 ? mbar_wait(bQ, 0, wait_ns) : true;
        ok = __syncthreads_and(got) != 0;
        if (ok && tid < 4 * HG) convert_q_f16(a, sm_log2, sQ, q_atom, qs, tid);
    }

    for (int c = c0; c < c1 && ok; ++c) {
        const int it = c - c0;
        if (it > 0) {
            k = slot_table(c);
            if (!win) load_records<G>(recs, sh.rb, kidx, tid, rr);
        }
        if (win && !fp8) {
            // the window rows of this chunk by TMA: 9 boxes of 64 channels x 128 rows
            if (tid == 0) {
                mbar_expect_tx(bW, NATOM * K_ATOM);
                for (int at = 0; at < NATOM; ++at)
                    tma_load_2d(sK + at * K_ATOM, &tm_w, 64 * at, b * a.window_stride + c * CK, bW);
            }
            ++nw;
        }
        // ---- the K tile is free once the previous chunk's PV is done
        if (it > 0) {
            const bool got = warp == 0 ? mbar_wait(bO, (it - 1) & 1, wait_ns) : true;
            ok = __syncthreads_and(got) != 0;
            if (!ok) break;
            tc_fence_after();
        }
        // ---- fill the K tile
        if (!win) {
            store_records<G>(rr, kidx, sK, tid);
        } else if (fp8) {
            // signed E4M3 codes decoded exactly to bf16 (the row scale is
            // applied to the logits and to the probabilities)
            if (k < 0) {
                zero_row_half(sK, s, half);
            } else {
                const uint8_t* src = a.win_fp8 + ((size_t)b * a.window_stride + k) * D + 288 * half;
                uint4 v[18];
#pragma unroll
                for (int u = 0; u < 18; ++u) v[u] = ldg_nc(src + 16 * u);
#pragma unroll
                for (int u = 0; u < 18; ++u) {
                    const uint32_t words[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                    uint32_t o[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t h0, h1;
                        asm("{\n\t.reg .b16 lo, hi;\n\t"
                            "mov.b32 {lo, hi}, %2;\n\t"
                            "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
                            "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
                            : "=r"(h0), "=r"(h1)
                            : "r"(words[q]));
                        const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
                        const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
                        o[2 * q] = pack_bf16(f0.x, f0.y);  // exact: E4M3 has 4 significant bits
                        o[2 * q + 1] = pack_bf16(f1.x, f1.y);
                    }
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const int c16 = 36 * half + 2 * u + p;
                        sts128(sK + (uint32_t)(c16 >> 3) * K_ATOM + swz(s, c16 & 7), o[4 * p],
                               o[4 * p + 1], o[4 * p + 2], o[4 * p + 3]);
                    }
                }
            }
        } else {
            // the TMA rows must have landed; masked rows are then zeroed (a
            // box past the window reads other rows, or zeros past the tensor)
            const bool got = warp == 0 ? mbar_wait(bW, (nw - 1) & 1, wait_ns) : true;
            ok = __syncthreads_and(got) != 0;
            if (!ok) break;
            if (k < 0) zero_row_half(sK, s, half);
        }
        if (win && it == 0) {  // the query rows' TMA
            const bool got = warp == 0 ? mbar_wait(bQ, 0, wait_ns) : true;
            ok = __syncthreads_and(got) != 0;
            if (!ok) break;
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ---- S^T = K Q^T (one thread issues)
        if (tid == 0) {
            tc_fence_after();
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t at = kk >> 2, koff = (kk & 3) * 32;
                mma_f16(tmem + S_COL, sdesc(sK + at * K_ATOM + koff, 16, 1024),
                        sdesc(sQ + at * q_atom + koff, 16, 1024), idQK, kk > 0);
            }
            mma_commit(bS);
        }
        ++nqk;
        {
            const bool got = warp == 0 ? mbar_wait(bS, it & 1, wait_ns) : true;
            ok = __syncthreads_and(got) != 0;
        }
        tc_fence_after();
        if (!ok) break;
        // folded window: the last record product has read the f16 query tile;
        // its bf16 original comes back by TMA while softmax and PV run
        if (WR > 0 && !win && c == c1 - 1) {
            if (tid == 0) tma_q();
            nq = 2;
        }

        // ---- softmax, all 8 warps: thread = key = tensor-memory lane (warp w
        // reads lane quadrant w & 3) and warp w takes head columns [c_lo,
        // c_hi) = half (w >> 2) of the group, 8 at a time.  y is the raw logit
        // (times the FP8 row scale); x = y * qs[h] in log2 units.  Scores are
        // read twice (maxima, then weights), in rolled loops.
        const bool valid = k >= 0;
        const float kf = fp8 ? ks[s] : 1.f;
        const uint32_t ta_s = tmem + ((uint32_t)((warp & 3) * 32) << 16) + S_COL;
        const int c8_lo = (warp >> 2) * (HG / 16), c8_hi = c8_lo + HG / 16;
        {
#pragma unroll 1
            for (int c8 = c8_lo; c8 < c8_hi; ++c8) {
                uint32_t r[8];
                tmem_ld8(ta_s + 8 * c8, r);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float y = valid ? __uint_as_float(r[i]) * kf : -INFINITY;
                    const int m = __reduce_max_sync(0xffffffffu, f32_ord(y));
                    if (lane == ((8 * c8 + i) & 31)) wmax[(warp & 3) * 64 + 8 * c8 + i] = m;
                }
            }
        }
        if (tid == 0) flags[0] = 0;
        __syncthreads();
        if (tid < HG) {
            float my = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) my = fmaxf(my, ord_f32(wmax[w * 64 + tid]));
            const float mc = my * qs[tid];  // qs > 0
            const float mo = mref[tid];
            const float mn = (mo == -INFINITY || mc > mo + kRescaleSlack) ? mc : mo;
            const float f = mo == -INFINITY ? 0.f : ex2(mo - mn);  // 1 when unchanged
            fac[tid] = f;
            mref[tid] = mn;
            if (it > 0 && f != 1.f) flags[0] = 1;
        }
        __syncthreads();
        {
#pragma unroll 1
            for (int c8 = c8_lo; c8 < c8_hi; ++c8) {
                uint32_t r[8];
                tmem_ld8(ta_s + 8 * c8, r);
                tmem_wait_ld();
                uint32_t w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int h = 8 * c8 + 2 * u;
                    const float m0 = mref[h], m1 = mref[h + 1];
                    const float y0 = valid ? __uint_as_float(r[2 * u]) * kf : -INFINITY;
                    const float y1 = valid ? __uint_as_float(r[2 * u + 1]) * kf : -INFINITY;
                    float p0 = m0 == -INFINITY ? 0.f : ex2(fmaf(y0, qs[h], -m0));
                    float p1 = m1 == -INFINITY ? 0.f : ex2(fmaf(y1, qs[h + 1], -m1));
                    if (fp8) {  // v = scale x E4M3 row: the scale moves onto p
                        p0 *= kf;
                        p1 *= kf;
                    }
                    w[u] = win ? pack_bf16(p0, p1) : pack_f16(p0, p1);
                }
                sts128(sP + swz(s, c8), w[0], w[1], w[2], w[3]);
            }
        }
        if (!lmma) {
            // FP8 rows: column sums of the rounded P^T divided by the row
            // scale (warp w adds keys [16 w, 16 w + 16) for its lane's pair)
            __syncthreads();
            float s0 = 0.f, s1 = 0.f;
            if (2 * lane < HG) {
#pragma unroll 4
                for (int jj = 0; jj < 16; ++jj) {
                    const int j = 16 * warp + jj;
                    uint32_t v;
                    asm volatile("ld.shared.u32 %0, [%1];\n"
                                 : "=r"(v)
                                 : "r"(sP + swz(j, lane >> 2) + (lane & 3) * 4));
                    const float sj = ks[j];
                    const float inv = sj > 0.f ? __frcp_rn(sj) : 0.f;
                    s0 += __uint_as_float(v << 16) * inv;
                    s1 += __uint_as_float(v & 0xFFFF0000u) * inv;
                }
            }
            lpart[warp * 64 + 2 * lane] = s0;
            lpart[warp * 64 + 2 * lane + 1] = s1;
        }
        fence_async_smem();  // P^T stores before the PV product reads them
        tc_fence_before();
        __syncthreads();
        if (!lmma && tid < HG) {
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < 8; ++w) sum += lpart[w * 64 + tid];
            lrun[tid] = lrun[tid] * fac[tid] + sum;
        }
        // ---- rare: a head's reference moved after O^T (and L) hold earlier chunks
        if (flags[0]) {
            tc_fence_after();
            const int g = warp & 3;
            for (int t = 0; t < 3; ++t) {
                const int mt = (warp >> 2) * 3 + t;  // O^T tiles 0-3, L tile (4), spare (5)
                if (mt > 4) break;
                const uint32_t col = mt < 4 ? O_COL + 64 * mt : L_COL;
                for (int h0 = 0; h0 < HG; h0 += 32) {
                    const uint32_t ta = tmem + ((uint32_t)(g * 32) << 16) + col + h0;
                    uint32_t r[32];
                    tmem_ld32(ta, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (h0 + i < HG) r[i] = __float_as_uint(__uint_as_float(r[i]) * fac[h0 + i]);
                    tmem_st32(ta, r);
                }
            }
            tc_fence_before();
            __syncthreads();
        }
        // ---- O^T += V^T P^T and L^T += ONES P^T (one thread issues)
        if (tid == 0) {
            tc_fence_after();
            for (int mt = 0; mt < DV / 128; ++mt)
                for (int kk = 0; kk < CK / 16; ++kk)
                    mma_f16(tmem + O_COL + 64 * mt,
                            sdesc(sK + (2 * mt) * K_ATOM + kk * 2048u, K_ATOM, 1024),
                            sdesc(sP + kk * 2048u, K_ATOM, 1024), idPV, (it > 0 || kk > 0) ? 1u : 0u);
            if (lmma)
                for (int kk = 0; kk < CK / 16; ++kk)
                    mma_f16(tmem + L_COL, ones_desc(sOnes), sdesc(sP + kk * 2048u, K_ATOM, 1024),
                            idL, (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bO);
        }
        ++npv;
    }
    // ---- folded window: with WR > 0 the window chunk has no CTA of its own;
    // record CTA r also attends over window rows [r WR, r WR + WR) for every
    // head of its group (bf16 operands), updating the running softmax and O^T
    // in place.  The rows land by TMA as packed atoms of WR rows in the freed
    // K tile (the product's A operand reads 128 rows from each atom start; the
    // logits of rows past WR are masked), P^T after them.
    if (WR > 0 && !win && !a.win_fp8 && ok && c0 < c1) {  // (bf16 window rows only)
        const int r0 = split * WR;
        const uint32_t w_atom = (uint32_t)WR * 128u;
        const uint32_t sPw = sK + 9 * w_atom + 16384u;
        {  // the K tile and P^T are free once the last record PV is done
            const bool got = warp == 0 ? mbar_wait(bO, (npv - 1) & 1, wait_ns) : true;
            ok = __syncthreads_and(got) != 0;
        }
        tc_fence_after();
        if (ok) {
            if (tid < CK) kidx[tid] = (tid < WR && r0 + tid < W) ? r0 + tid : -1;
            if (tid == 0) {
                mbar_expect_tx(bW, NATOM * w_atom);
                for (int at = 0; at < NATOM; ++at)
                    tma_load_2d(sK + at * w_atom, &tm_wr, 64 * at, b * a.window_stride + r0, bW);
            }
            ++nw;
            // the ones block in bf16 for the window's row sums
            asm volatile("st.shared.v2.u32 [%0], {%1, %1};\n" ::"r"(sOnes + 8 * tid),
                         "r"(0x3F803F80u));
            const bool got =
                warp == 0 ? (mbar_wait(bW, 0, wait_ns) && mbar_wait(bQ, 1, wait_ns)) : true;
            ok = __syncthreads_and(got) != 0;
        }
        if (ok) {
            const int kw = kidx[s];
            if (s < WR && kw < 0) {  // rows past the window (read as other rows or zeros)
#pragma unroll 1
                for (int c16 = 36 * half; c16 < 36 * half + 36; ++c16)
                    sts128(sK + (uint32_t)(c16 >> 3) * w_atom + swz(s, c16 & 7), 0u, 0u, 0u, 0u);
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
                const uint32_t idQKw = idesc_f16(128, HG, 1, 0, 0);
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t at = kk >> 2, koff = (kk & 3) * 32;
                    mma_f16(tmem + S_COL, sdesc(sK + at * w_atom + koff, 16, 1024),
                            sdesc(sQ + at * q_atom + koff, 16, 1024), idQKw, kk > 0);
                }
                mma_commit(bS);
            }
            ++nqk;
            const bool got = warp == 0 ? mbar_wait(bS, (nqk - 1) & 1, wait_ns) : true;
            ok = __syncthreads_and(got) != 0;
            tc_fence_after();
            const bool valid = kw >= 0;
            const uint32_t ta_s = tmem + ((uint32_t)((warp & 3) * 32) << 16) + S_COL;
            // (heads split in halves between warps w and w + 4; quadrants
            // without window rows report -inf maxima)
            const bool rows_here = (warp & 3) * 32 < WR;
            const int c8_lo = (warp >> 2) * (HG / 16), c8_hi = c8_lo + HG / 16;
            if (ok) {
#pragma unroll 1
                for (int c8 = c8_lo; c8 < c8_hi; ++c8) {
                    uint32_t r[8];
                    tmem_ld8(ta_s + 8 * c8, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float y = valid ? __uint_as_float(r[i]) : -INFINITY;
                        const int m = __reduce_max_sync(0xffffffffu, f32_ord(y));
                        if (lane == ((8 * c8 + i) & 31)) wmax[(warp & 3) * 64 + 8 * c8 + i] = m;
                    }
                }
            }
            if (tid == 0) flags[0] = 0;
            __syncthreads();
            if (ok && tid < HG) {
                float my = -INFINITY;
#pragma unroll
                for (int w = 0; w < 4; ++w) my = fmaxf(my, ord_f32(wmax[w * 64 + tid]));
                const float mc = my * sm_log2;
                const float mo = mref[tid];
                const float mn = (mo == -INFINITY || mc > mo + kRescaleSlack) ? mc : mo;
                const float f = mo == -INFINITY ? 0.f : ex2(mo - mn);
                fac[tid] = f;
                mref[tid] = mn;
                if (f != 1.f) flags[0] = 1;
            }
            __syncthreads();
            // P^T rows of this CTA's window keys, by whole warps (the tensor-memory
            // load is warp-collective; rows WR..31 of a quadrant come out as
            // zeros, unread)
            if (ok && rows_here) {
#pragma unroll 1
                for (int c8 = c8_lo; c8 < c8_hi; ++c8) {
                    uint32_t r[8];
                    tmem_ld8(ta_s + 8 * c8, r);
                    tmem_wait_ld();
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int h = 8 * c8 + 2 * u;
                        const float m0 = mref[h], m1 = mref[h + 1];
                        const float y0 = valid ? __uint_as_float(r[2 * u]) : -INFINITY;
                        const float y1 = valid ? __uint_as_float(r[2 * u + 1]) : -INFINITY;
                        const float p0 = m0 == -INFINITY ? 0.f : ex2(fmaf(y0, sm_log2, -m0));
                        const float p1 = m1 == -INFINITY ? 0.f : ex2(fmaf(y1, sm_log2, -m1));
                        w[u] = pack_bf16(p0, p1);
                    }
                    sts128(sPw + swz(s, c8), w[0], w[1], w[2], w[3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            if (ok && flags[0]) {  // heads whose reference moved: rescale O^T and L
                tc_fence_after();
                const int g = warp & 3;
                for (int t = 0; t < 3; ++t) {
                    const int mt = (warp >> 2) * 3 + t;
                    if (mt > 4) break;
                    const uint32_t col = mt < 4 ? O_COL + 64 * mt : L_COL;
                    for (int h0 = 0; h0 < HG; h0 += 32) {
                        const uint32_t ta = tmem + ((uint32_t)(g * 32) << 16) + col + h0;
                        uint32_t r[32];
                        tmem_ld32(ta, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (h0 + i < HG)
                                r[i] = __float_as_uint(__uint_as_float(r[i]) * fac[h0 + i]);
                        tmem_st32(ta, r);
                    }
                }
                tc_fence_before();
                __syncthreads();
            }
            if (ok && tid == 0) {
                tc_fence_after();
                const uint32_t idPVw = idesc_f16(128, 64, 1, 1, 1);
                const uint32_t idLw = idesc_f16(128, 64, 1, 0, 1);
                for (int mt = 0; mt < DV / 128; ++mt)
                    for (int kk = 0; kk < WR / 16; ++kk)
                        mma_f16(tmem + O_COL + 64 * mt,
                                sdesc(sK + (2 * mt) * w_atom + kk * 2048u, w_atom, 1024),
                                sdesc(sPw + kk * 2048u, w_atom, 1024), idPVw, 1u);
                for (int kk = 0; kk < WR / 16; ++kk)
                    mma_f16(tmem + L_COL, ones_desc(sOnes), sdesc(sPw + kk * 2048u, w_atom, 1024),
                            idLw, 1u);
                mma_commit(bO);
            }
            if (ok) ++npv;
        }
    }

    // the last PV must be complete before O^T is read
    if (ok && c1 > c0) {
        const bool got = warp == 0 ? mbar_wait(bO, (npv - 1) & 1, wait_ns) : true;
        ok = __syncthreads_and(got) != 0;
        tc_fence_after();
        if (ok && lmma && warp == 0) {  // the row sums: every lane of the L tile holds them
            for (int h0 = 0; h0 < HG; h0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + L_COL + h0, r);
                tmem_wait_ld();
                if (lane == 0)
                    for (int i = 0; i < 32; ++i)
                        if (h0 + i < HG) lrun[h0 + i] = __uint_as_float(r[i]);
            }
        }
        __syncthreads();
    }

    pdl_trigger();  // only the epilogue is left: let the next kernel be scheduled

    const bool mine = ok && c0 < c1;
    if (cluster) {
        // ---- the nsplit CTAs of this sequence and head group form one
        // cluster; CTA r owns heads [r*hpc, (r+1)*hpc) of the group.  Once
        // every CTA's products are done (cluster barrier), each CTA stores its
        // unnormalised O columns (from tensor memory, a lane per channel) and
        // its (m, l) straight into the owners' shared memory -- rows [src][hh]
        // of 2 KB in the owner's freed K tile -- and after a second cluster
        // barrier every owner combines its rows locally and writes the output.
        const int hpc = (HG + nsplit - 1) / nsplit;
        const int h_lo = split * hpc, nh = max(0, min(HG, h_lo + hpc) - h_lo);
        uint32_t* dst_off = reinterpret_cast<uint32_t*>(misc + M_KS);  // [HG] owner row addresses
        float* mlx = lpart;                                            // [nsplit][nh][2]
        float* wts = reinterpret_cast<float*>(wmax);                   // [nh][nsplit]
        if (tid < HG) {
            const int r = tid / hpc, hh = tid - r * hpc;
            const int nh_r = min(hpc, HG - r * hpc);
            uint32_t rk, rm;
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rk) : "r"(sK), "r"(r));
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                         : "=r"(rm)
                         : "r"(smem_u32(mlx)), "r"(r));
            dst_off[tid] = rk + (uint32_t)(split * nh_r + hh) * DV * 4;
            ks[64 + tid] = __uint_as_float(rm + (uint32_t)(split * nh_r + hh) * 8);
        }
        tc_fence_before();
        cluster_sync();  // every CTA of the cluster is past its last product
        tc_fence_after();
        if (tid < HG) {
            const float m = mine ? mref[tid] : -INFINITY, l = mine ? lrun[tid] : 0.f;
            asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(
                             __float_as_uint(ks[64 + tid])),
                         "f"(m), "f"(l)
                         : "memory");
        }
        if (mine) {
            const int g = warp & 3;
            for (int t = 0; t < 2; ++t) {
                const int mt = (warp >> 2) * 2 + t;
                const uint32_t d4 = (mt * 128 + g * 32 + lane) * 4;
                // both 32-head blocks of the tile loaded before one wait (HG <= 64)
                uint32_t r[2][32];
                const uint32_t ta = tmem + ((uint32_t)(g * 32) << 16) + O_COL + 64 * mt;
                tmem_ld32(ta, r[0]);
                if (HG > 32) tmem_ld32(ta + 32, r[1]);
                tmem_wait_ld();
#pragma unroll
                for (int hb = 0; hb < 2; ++hb)
                    if (hb * 32 < HG) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (hb * 32 + i < HG)
                                asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(
                                                 dst_off[hb * 32 + i] + d4),
                                             "r"(r[hb][i])
                                             : "memory");
                    }
            }
        }
        cluster_sync();  // every row and (m, l) has arrived
        if (tid < nh) {
            // every split's (m, l) loaded at once (at most 8 splits)
            float2 ml[8];
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2)
                if (s2 < nsplit) ml[s2] = reinterpret_cast<const float2*>(mlx)[s2 * nh + tid];
            float M = -INFINITY;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2)
                if (s2 < nsplit) M = fmaxf(M, ml[s2].x);
            float L = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2)
                if (s2 < nsplit) {
                    const float m = ml[s2].x, l = ml[s2].y;
                    const float w = (M == -INFINITY || m == -INFINITY) ? 0.f : ex2(m - M);
                    wts[tid * nsplit + s2] = w;
                    L += w * l;
                }
            fac[tid] = L > 0.f ? 1.f / L : 0.f;
            if (a.lse)
                a.lse[(size_t)b * H + hg0 + h_lo + tid] =
                    L > 0.f ? (M + __log2f(L)) * 0.6931471805599453f : -INFINITY;
        }
        __syncthreads();
        const float* rows = reinterpret_cast<const float*>(smem + OFF_K);
#pragma unroll 2
        for (int it2 = tid; it2 < nh * (DV / 4); it2 += NT) {
            const int hh = it2 / (DV / 4), q4 = it2 - hh * (DV / 4);
            // every split's weight and row loaded at once (a cluster holds at
            // most 8 CTAs); a split with weight 0 pushed no row: its value is
            // selected away, never multiplied
            float w[8];
            float4 v[8];
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2)
                if (s2 < nsplit) {
                    w[s2] = wts[hh * nsplit + s2];
                    v[s2] = reinterpret_cast<const float4*>(rows + (s2 * nh + hh) * DV)[q4];
                }
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2)
                if (s2 < nsplit && w[s2] != 0.f) {
                    acc.x = fmaf(w[s2], v[s2].x, acc.x);
                    acc.y = fmaf(w[s2], v[s2].y, acc.y);
                    acc.z = fmaf(w[s2], v[s2].z, acc.z);
                    acc.w = fmaf(w[s2], v[s2].w, acc.w);
                }
            const float inv = fac[hh];
            *reinterpret_cast<float4*>(a.out + ((size_t)b * H + hg0 + h_lo + hh) * DV + 4 * q4) =
                make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        }
    } else if (nsplit == 1 || mine) {
        // ---- thread = one latent channel of a tile, 32 heads per load
        const int g = warp & 3;
        for (int t = 0; t < 2; ++t) {
            const int mt = (warp >> 2) * 2 + t;
            const int d = mt * 128 + g * 32 + lane;
            for (int h0 = 0; h0 < HG; h0 += 32) {
                uint32_t r[32] = {};
                if (mine) {
                    tmem_ld32(tmem + ((uint32_t)(g * 32) << 16) + O_COL + 64 * mt + h0, r);
                    tmem_wait_ld();
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (h0 + i >= HG) break;
                    const int h = hg0 + h0 + i;
                    if (nsplit == 1) {
                        const float l = mine ? lrun[h0 + i] : 0.f;
                        a.out[((size_t)b * H + h) * DV + d] = l > 0.f ? __uint_as_float(r[i]) / l : 0.f;
                    } else {
                        a.part_o[(((size_t)b * H + h) * kMaxSplit + split) * DV + d] =
                            __uint_as_float(r[i]);
                    }
                }
            }
        }
    }
    if (!cluster && tid < HG) {
        const float m = mine ? mref[tid] : -INFINITY, l = mine ? lrun[tid] : 0.f;
        const int h = hg0 + tid;
        if (nsplit == 1) {
            if (a.lse)
                a.lse[(size_t)b * H + h] = l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
        } else {
            const size_t row = ((size_t)b * H + h) * kMaxSplit + split;
            a.part_ml[row * 2] = m;
            a.part_ml[row * 2 + 1] = l;
        }
    }
    if (!ok && tid == 0) {
        // a bounded wait gave up: flag it, give the copies and products this
        // CTA issued one more bounded wait each, then free the tensor memory
        set_status(a.status, KVC_DEV_TIMEOUT);
        if (nqk > 0) mbar_wait(bS, (nqk - 1) & 1, kCleanupWaitNs);
        if (npv > 0) mbar_wait(bO, (npv - 1) & 1, kCleanupWaitNs);
        if (nw > 0) mbar_wait(bW, (nw - 1) & 1, kCleanupWaitNs);
    }
    // the query rows' TMA must have landed before the CTA exits (a CTA with
    // no chunk never waited for it)
    if (tid == 0 && (!ok || c0 >= c1)) mbar_wait(bQ, (nq - 1) & 1, kCleanupWaitNs);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                     "r"(TMEM_COLS));
    }
}

}  // namespace t128

bool t128_supported(const kvc_config& c, const Shape& sh) {
    const bool g_ok = sh.G == 8 || sh.G == 16 || sh.G == 32 || sh.G == 64 || sh.G == 128;
    return c.act_dtype == KVC_BF16 && c.scale_fmt == KVC_SCALE_UE4M3 && c.n_heads == t128::H &&
           sh.D == t128::D && sh.Dv == t128::DV && g_ok;
}

namespace {
unsigned long long g_wait_ns = 2000000000ull;  // bound on one device wait

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}
// 2-D bf16 tensor [rows][576] (row stride 1152 B), boxes of 64 channels x
// box_rows rows, 128-byte swizzle, zero fill past the end.
bool encode_rows(CUtensorMap* m, const void* base, unsigned long long rows, unsigned box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)t128::D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)t128::D * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace
unsigned long long device_wait_limit_ns() { return g_wait_ns; }
void set_device_wait_limit_ns(unsigned long long ns) { g_wait_ns = ns; }

template <int G>
static cudaError_t launch_g(const CUtensorMap& tq, const CUtensorMap& tw, const CUtensorMap& twr,
                            const dim3& grid, int cluster_x, const AttnArgs& a, const Shape& sh,
                            int K, float sm_log2, int rsplit, int cpr, int nsplit, int cluster,
                            int HG, int WR, cudaStream_t s) {
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(t128::attn_t128_kernel<G>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)t128::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(t128::NT);
    cfg.dynamicSmemBytes = t128::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, t128::attn_t128_kernel<G>, tq, tw, twr, a, sh, K, sm_log2,
                              rsplit, cpr, nsplit, cluster, HG, WR, g_wait_ns);
}

// Clusters of `size` CTAs of this kernel that can be resident at once on the
// current device (cached per device and size; 0 when the query fails).
template <int G>
static int max_clusters(int size) {
    static int cache[64][9] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || size < 1 || size > 8) return 0;
    if (cache[dev][size]) return cache[dev][size] > 0 ? cache[dev][size] : 0;
    cudaFuncSetAttribute(t128::attn_t128_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)t128::SMEM_BYTES);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(size, 1);
    cfg.blockDim = dim3(t128::NT);
    cfg.dynamicSmemBytes = t128::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = size;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, t128::attn_t128_kernel<G>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cache[dev][size] = n > 0 ? n : -1;
    return n > 0 ? n : 0;
}

template <int G>
static int launch_t128_g(const kvc_config& c, const AttnArgs& a, const Shape& sh, cudaStream_t s) {
    const int K = c.topk;
    const int rc = (K + t128::CK - 1) / t128::CK;
    const int wc = (a.window_len + t128::CK - 1) / t128::CK;
    // Work split: the key chunks of a sequence go to one cluster of CTAs (one
    // record chunk each while that fits in 8, else cpr), and the 64 heads to
    // 64 / HG such clusters.  Fewest chunks per CTA first, then the most
    // clusters (smallest head group) that can all be resident at once;
    // without one, the largest head group with the fewest chunks per CTA.
    int cpr = 0, HG = 64;
    for (int cp = 1; cp <= std::max(rc, 1) && !cpr; ++cp) {
        const int ns = (rc + cp - 1) / cp + wc;
        if (ns > 8) continue;
        for (int hg = 16; hg <= 64; hg *= 2) {
            const long long clusters = (long long)a.batch * (64 / hg);
            if (ns == 1 || max_clusters<G>(ns) >= clusters) {
                cpr = cp;
                HG = hg;
                break;
            }
        }
    }
    if (!cpr) {
        cpr = 1;
        while (rc > 0 && cpr < rc && (rc + cpr - 1) / cpr + wc > 8) ++cpr;
        HG = 64;
    }
    // When that split needs two or more record chunks per CTA, a window of
    // one chunk can instead be folded into the record CTAs (each takes 128 /
    // rc of the window rows, for all its heads) if every sequence's cluster
    // of rc CTAs can then be resident: one chunk and a window slice per CTA.
    int WR = 0;
    if (cpr > 1 && wc == 1 && (rc == 2 || rc == 4 || rc == 8) && !a.win_fp8) {
        for (int hg = 16; hg <= 64; hg *= 2) {
            if (max_clusters<G>(rc) >= (long long)a.batch * (64 / hg)) {
                cpr = 1;
                HG = hg;
                WR = t128::CK / rc;
                break;
            }
        }
    }
    const int wsplit = WR ? 0 : wc;  // window chunks with a CTA of their own
    int rsplit = rc == 0 ? 0 : (rc + cpr - 1) / cpr;
    int nsplit = rsplit + wsplit;
    if (nsplit == 0) {  // nothing to attend: one CTA per head group writes zeros and -inf
        rsplit = 1;
        nsplit = 1;
    }
    if (nsplit > kMaxSplit) return -1;
    const int cluster = (nsplit > 1 && nsplit <= 8) ? 1 : 0;
    // every CTA's query rows arrive by TMA (boxes of HG rows); so do bf16
    // window rows (boxes of a chunk, or of WR rows when folded)
    CUtensorMap tq = {}, tw = {}, twr = {};
    if (!encode_rows(&tq, a.q, (unsigned long long)a.batch * t128::H, HG)) return -1;
    if (wc > 0 && !a.win_fp8 &&
        !encode_rows(&tw, a.window, (unsigned long long)a.batch * a.window_stride, t128::CK))
        return -1;
    if (WR && !encode_rows(&twr, a.window, (unsigned long long)a.batch * a.window_stride, WR))
        return -1;
    const float sm_log2 = c.sm_scale * 1.4426950408889634f;
    trace_before("attn_t128", s);
    const cudaError_t e = launch_g<G>(tq, tw, twr, dim3(nsplit, 64 / HG, a.batch),
                                      cluster ? nsplit : 1, a, sh, K, sm_log2, rsplit, cpr, nsplit,
                                      cluster, HG, WR, s);
    trace_after(s);
    if (e != cudaSuccess) return -1;
    return cluster ? 1 : nsplit;
}

// Launches the chunks of every sequence; returns the number of partial
// results the caller still has to merge (1 when the kernel wrote the final
// output itself), or a negative value on a launch error.
int launch_attention_t128(const kvc_config& c, const Shape& sh, const AttnArgs& a,
                          cudaStream_t s) {
    switch (sh.G) {
        case 8: return launch_t128_g<8>(c, a, sh, s);
        case 16: return launch_t128_g<16>(c, a, sh, s);
        case 32: return launch_t128_g<32>(c, a, sh, s);
        case 64: return launch_t128_g<64>(c, a, sh, s);
        default: return launch_t128_g<128>(c, a, sh, s);
    }
}

}  // namespace kvc
