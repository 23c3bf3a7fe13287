// attn_tc05.cu -- sparse decode attention on the 5th-generation tensor cores
// (tcgen05 MMA, accumulators in tensor memory) for the MLA shape: 64 query
// heads sharing 576-channel entries (512 latent + 64 RoPE), values = latent.
//
// Method: "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
// 压缩到 890 B的？" (acejoy.com) part 3 breakthrough 2 (heads share one latent
// entry, absorbed up-projections), breakthrough 4 (top-512 entries + 128-token
// window), part 4 "P4 main KV" (FP4 is dequantised before attention).  One
// softmax runs jointly over the selected entries and the window keys.
//
// One CTA (256 threads) owns one to a few chunks of 96 keys of one sequence;
// the operands are f16 (exact for every dequantised entry and for bf16
// queries and window rows in the f16 range):
//  1. Q (64 x 576) is converted from bf16 once into a 128B-swizzled K-major
//     tile.  Per chunk, cp.async gathers the selected records (16-byte
//     rows) as one group and the window rows as a second group.
//  2. Records are dequantised by the hardware E2M1 -> f16x2 conversion times
//     the f16x2 group scale (exact: at most 6 significant bits) into the K
//     tile, 128B-swizzled K-major: 9 atoms of 64 channels x 96 keys, while the
//     window rows land; those are then converted to f16 in place.
//  3. One thread issues S = Q K^T: 36 tcgen05.mma (M=128, N=96, K=16) into
//     TMEM; rows 64..127 of the A operand read the next atom (don't-care rows).
//  4. Four warps read the head rows of S from TMEM, take max / exp2 / sum in
//     fp32 against a lazily moved reference and write P (f16) 128B-swizzled.
//  5. One thread issues O^T += V^T P^T: the K tile's latent atoms read as an
//     MN-major operand (no second copy), 4 x 6 tcgen05.mma (M=128 channels,
//     N=64 heads, K=16 keys) into TMEM.
//  6. The splits of a sequence (at most 8) form a thread-block cluster: each
//     stores its unnormalised O and (m, l) (they stay in L2), one cluster
//     barrier orders the stores, and CTA r combines heads [r*64/n,
//     (r+1)*64/n) from all of them.  With more splits the partials go to
//     attn_merge.
// Every wait on an mbarrier is bounded by a 2-second clock; on expiry the CTA
// sets KVC_DEV_TIMEOUT, frees its tensor memory and returns.
#include <algorithm>
#include <cuda_fp16.h>

#include "kvc_internal.cuh"

namespace kvc {
namespace tc05 {

constexpr int H = 64, D = 576, DV = 512, CK = 96, NT = 256;
constexpr int NATOM = D / 64;                   // 9 channel atoms of 64
constexpr int KGRP = CK / 8;                    // 12 groups of 8 keys
constexpr uint32_t Q_BYTES = NATOM * 8 * 1024;  // 64 rows: 8 row groups per atom
constexpr uint32_t K_ATOM = KGRP * 1024;        // one channel atom of the K tile
constexpr uint32_t K_BYTES = NATOM * K_ATOM;
constexpr uint32_t RAW_STRIDE = 368;            // record bytes reserved per key (G >= 8)
constexpr uint32_t RAW_BYTES = CK * RAW_STRIDE;
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + Q_BYTES;
constexpr uint32_t OFF_RAW = OFF_K + K_BYTES;   // P (16 KB) reuses this after dequant
constexpr uint32_t OFF_P = OFF_RAW;
constexpr uint32_t OFF_MISC = OFF_RAW + RAW_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 4096 + 1024;  // + misc + table + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0, O_COL = 128;

// instruction descriptors (kind::f16): D f32, A and B f16 (type code 0), M = 128
constexpr uint32_t kIdescQK = (1u << 4) | ((uint32_t)(CK >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 15) /* A MN-major */ |
                              ((uint32_t)(H >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// shared-memory matrix descriptor, 128-byte swizzle, sm100 version field
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
// every group but the most recent one complete
__device__ __forceinline__ void cp_async_wait_prior() {
    asm volatile("cp.async.wait_group 1;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;\n" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t addr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(addr), "r"(count));
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// bounded wait for phase `parity` of an mbarrier; false after ~2 s
__device__ __forceinline__ bool mbar_wait(uint32_t addr, uint32_t parity) {
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(addr), "r"(parity)
            : "memory");
        if (ok) return true;
        if ((i & 255) == 255 && global_ns() - t0 > 2000000000ull) return false;
    }
}
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mbar)
        : "memory");
}
// 32 lanes x 32 consecutive columns of 32 bits: thread i gets lane (base+i)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    const __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}
// two bf16 (low half first) -> two f16; exact for |x| in [2^-14, 65504]
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    return pack_f16(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// eight E2M1 codes (channel 2i in the low nibble of byte i) -> four f16x2
// words, each times the f16x2 scale s2 (a code times a UE4M3 scale has at
// most 6 significant bits and stays in the f16 range: the product is exact)
__device__ __forceinline__ void e2m1x8_to_f16(uint32_t codes, __half2 s2, uint32_t (&w)[4]) {
    uint32_t r[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "r"(codes));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&r[k]), s2);
        w[k] = *reinterpret_cast<const uint32_t*>(&v);
    }
}

// byte offset of 16-byte chunk `c16` of row `r` inside a 128B-swizzled block
// whose rows are 128 bytes and whose 8-row groups are 1024 bytes apart
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t c16) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((c16 ^ (r & 7u)) << 4);
}

// 32 lanes x 16 consecutive columns
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// The reference maximum of a head only moves when a chunk's maximum passes it
// by more than this (log2 units): probabilities stay <= 2^8 in bf16 and the
// accumulated O^T is rescaled in tensor memory only on such a jump.
constexpr float kRescaleSlack = 8.0f;

// The CTAs of one cluster (the splits of one sequence) meet here; every
// thread of every CTA of the cluster executes it the same number of times.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;\n" ::
                     : "memory");
}
__global__ void __launch_bounds__(NT, 1)
attn_tc05_kernel(AttnArgs a, Shape sh, int K, float scale_log2, int nsplit, int cps, int ue4m3,
                 int cluster) {
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled tiles
    const uint32_t raw_base = smem_u32(smem_raw);
    const uint32_t base = (raw_base + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (base - raw_base);
    const uint32_t sQ = base + OFF_Q, sK = base + OFF_K, sP = base + OFF_P;
    unsigned char* raw = smem + OFF_RAW;
    int* kind = reinterpret_cast<int*>(smem + OFF_MISC);                 // [CK]
    float* mref = reinterpret_cast<float*>(smem + OFF_MISC + 512);       // [H] reference max
    float* lrun = mref + H;                                              // [H] running sum
    float* fac = lrun + H;                                               // [H] rescale factor
    float* part = fac + H;                                               // [2][H] half max/sum
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_MISC + 2048);  // S done, O done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC + 2112);
    int* flags = reinterpret_cast<int*>(smem + OFF_MISC + 2176);

    const int b = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total = K + a.window_len;
    const int rb = sh.rb;
    const int c0 = split * cps, c1 = min(c0 + cps, (total + CK - 1) / CK);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    if (tid == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (tid < H) {
        mref[tid] = -INFINITY;
        lrun[tid] = 0.f;
    }
    // Q (64 x 576) once, converted to f16, 128B-swizzled K-major: before the
    // wait when no kernel launched since the caller wrote q writes it
    auto load_q = [&]() {
        const uint4* qg = reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(a.q) +
                                                         (size_t)b * H * D * 2);
#pragma unroll 6
        for (int p = tid; p < H * (D / 8); p += NT) {
            const int h = p / (D / 8), c = p - h * (D / 8);
            const uint4 v = __ldg(qg + p);
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(
                             sQ + (c >> 3) * 8192u + swz(h, c & 7)),
                         "r"(bf16x2_to_f16x2(v.x)), "r"(bf16x2_to_f16x2(v.y)),
                         "r"(bf16x2_to_f16x2(v.z)), "r"(bf16x2_to_f16x2(v.w)));
        }
        fence_async_smem();
    };
    if (a.q_ready) load_q();
    pdl_wait();  // everything above was local set-up or reads of inputs
    const int n = a.n_entries[b];
    const bool len_ok = n >= 0 && n <= a.capacity;
    if (!a.q_ready) load_q();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    for (int c = c0; c < c1 && ok; ++c) {
        const int it = c - c0;
        // ---- slot kinds of this chunk
        if (tid < CK) {
            const int j = c * CK + tid;
            if (a.topk_copy && j < K)  // a Reuse layer's own copy of its head's top-K
                a.topk_copy[(size_t)b * K + j] = a.topk_idx[(size_t)b * K + j];
            int k = -1;
            if (j < total && len_ok) {
                if (j < K) {
                    const int idx = a.topk_idx[(size_t)b * K + j];
                    if (idx >= 0 && idx < n)
                        k = idx;
                    else if (idx != -1)
                        set_status(a.status, KVC_DEV_BAD_INDEX);
                } else {
                    k = -2 - (j - K);  // window row
                }
            }
            kind[tid] = k;
        }
        // any window or empty slot in this chunk?
        const int other_rows = __syncthreads_or(tid < CK && kind[tid < CK ? tid : 0] < 0);
        // ---- 1. gathers: records (raw rows) as one group of copies, then window
        // rows (swizzled) and zero rows, which only the QK product needs
        {
            const int pieces = rb >> 4;
            for (int p = tid; p < CK * pieces; p += NT) {
                const int s = p / pieces, pc = p - s * pieces;
                const int k = kind[s];
                if (k >= 0)
                    cp_async16(smem_u32(raw + s * RAW_STRIDE + pc * 16),
                               a.records + ((size_t)b * a.capacity + k) * rb + pc * 16);
            }
            cp_async_commit();
            for (int p = tid; other_rows && p < CK * (D / 8); p += NT) {
                const int s = p / (D / 8), cc = p - s * (D / 8);
                const int k = kind[s];
                const uint32_t dst = sK + (cc >> 3) * K_ATOM + swz(s, cc & 7);
                if (k <= -2) {
                    if (a.win_fp8) continue;  // FP8 rows are decoded after the dequantisation
                    const int t = -2 - k;
                    cp_async16(dst, static_cast<const unsigned char*>(a.window) +
                                        ((size_t)b * a.window_stride + t) * D * 2 + cc * 16);
                } else if (k == -1) {
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(dst), "r"(0u),
                                 "r"(0u), "r"(0u), "r"(0u));
                }
            }
            cp_async_commit();
            cp_async_wait_prior();  // this thread's record copies have landed
        }
        __syncthreads();
        // ---- 2. dequantise records into the swizzled K tile.  UE4M3 scales: 32
        // channels per item, a byte of two codes -> bf16x2 table entry times
        // the bf16x2 scale of its group (the products have at most 6
        // significant bits, so the bf16 multiply is exact).  Groups of >= 32
        // share one scale per item; groups of 8 or 16 take one per 8 channels.
        {
            // 32 channels per item: one 16-byte load of codes, a scale per group
            // (per 8 channels for groups of 8 or 16), hardware E2M1 -> f16x2
            // conversion times the f16x2 scale, four 16-byte stores
            const int lpg = sh.lpg;
            constexpr int NI = CK * (D / 32);
#pragma unroll 2
            for (int p = tid; p < NI; p += NT) {
                const int sk = p / (D / 32), ik = p - sk * (D / 32);
                if (kind[sk] < 0) continue;
                const unsigned char* rec = raw + sk * RAW_STRIDE;
                const uint4 codes = *reinterpret_cast<const uint4*>(rec + ik * 16);
                const uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
                const uint32_t row = sK + (ik >> 1) * K_ATOM;
                const float s0 = e4m3_to_f32(rec[sh.code_bytes + (4 * ik) / lpg]);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float su =
                        lpg >= 4 ? s0 : e4m3_to_f32(rec[sh.code_bytes + (4 * ik + u) / lpg]);
                    uint32_t w[4];
                    e2m1x8_to_f16(cw[u], __floats2half2_rn(su, su), w);
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(
                                     row + swz(sk, 4 * (ik & 1) + u)),
                                 "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]));
                }
            }
        }
        cp_async_wait_all();  // the window rows too
        if (other_rows && a.win_fp8) {
            // FP8 window rows: 16 codes per load, E4M3 -> f16x2 in hardware,
            // times the row's scale in fp32, two 16-byte pieces of the K tile
            for (int p = tid; p < CK * (D / 16); p += NT) {
                const int s = p / (D / 16), c16 = p - s * (D / 16);
                const int k = kind[s];
                if (k > -2) continue;
                const size_t row = (size_t)b * a.window_stride + (-2 - k);
                const uint4 cw = __ldg(reinterpret_cast<const uint4*>(a.win_fp8 + row * D) + c16);
                const float sc = __ldg(a.win_scale + row);
                const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
                uint32_t o[8];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    uint32_t h0, h1;
                    asm("{\n\t.reg .b16 lo, hi;\n\t"
                        "mov.b32 {lo, hi}, %2;\n\t"
                        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
                        "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
                        : "=r"(h0), "=r"(h1)
                        : "r"(words[u]));
                    const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
                    const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
                    o[2 * u] = pack_f16(f0.x * sc, f0.y * sc);
                    o[2 * u + 1] = pack_f16(f1.x * sc, f1.y * sc);
                }
#pragma unroll
                for (int hpc = 0; hpc < 2; ++hpc) {
                    const int cc = 2 * c16 + hpc;
                    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(
                                     sK + (cc >> 3) * K_ATOM + swz(s, cc & 7)),
                                 "r"(o[4 * hpc]), "r"(o[4 * hpc + 1]), "r"(o[4 * hpc + 2]),
                                 "r"(o[4 * hpc + 3]));
                }
            }
        } else if (other_rows) {
            __syncthreads();  // every thread's window copies have landed
            // window rows arrived as bf16: convert them in place to f16
            for (int p = tid; p < CK * (D / 8); p += NT) {
                const int s = p / (D / 8), cc = p - s * (D / 8);
                if (kind[s] > -2) continue;
                const uint32_t addr = sK + (cc >> 3) * K_ATOM + swz(s, cc & 7);
                uint32_t v0, v1, v2, v3;
                asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                             : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3)
                             : "r"(addr));
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr),
                             "r"(bf16x2_to_f16x2(v0)), "r"(bf16x2_to_f16x2(v1)),
                             "r"(bf16x2_to_f16x2(v2)), "r"(bf16x2_to_f16x2(v3)));
            }
        }
        fence_async_smem();
        __syncthreads();

        // ---- 3. S = Q K^T (one thread issues)
        if (tid == 0) {
            tc_fence_after();
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t at = ks >> 2, koff = (ks & 3) * 32;
                mma_bf16(tmem + S_COL, sdesc(sQ + at * 8192u + koff, 16, 1024),
                         sdesc(sK + at * K_ATOM + koff, 16, 1024), kIdescQK, ks > 0);
            }
            mma_commit(smem_u32(&bars[0]));
        }
        // warp 0 polls the barrier; the other warps wait in the block barrier
        bool got = warp == 0 ? mbar_wait(smem_u32(&bars[0]), it & 1) : true;
        ok = __syncthreads_and(got) != 0;
        tc_fence_after();
        if (!ok) break;

        // ---- 4. softmax: warps 0,1 take columns [0, 48) and warps 4,5 columns
        // [48, 96) of the head rows (TMEM lanes 0..63)
        const bool sm_warp = (warp & 3) < 2;
        const int h = (warp & 3) * 32 + lane, half = warp >> 2;
        float sv[CK / 2];
        if (sm_warp) {
            const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16) + S_COL + half * (CK / 2);
            uint32_t r32[32];
            uint32_t r16[16];
            tmem_ld32(ta, r32);
            tmem_ld16(ta + 32, r16);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[i] = __uint_as_float(r32[i]);
#pragma unroll
            for (int i = 0; i < 16; ++i) sv[32 + i] = __uint_as_float(r16[i]);
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < CK / 2; ++j) {
                const float x = kind[half * (CK / 2) + j] == -1 ? -INFINITY : sv[j] * scale_log2;
                sv[j] = x;
                m4[j & 3] = fmaxf(m4[j & 3], x);
            }
            part[half * H + h] = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        __syncthreads();
        if (sm_warp) {
            const float mc = fmaxf(part[h], part[H + h]);
            const float mo = mref[h];
            // move the reference only on a large jump (or the first keys)
            const float mn = (mo == -INFINITY || mc > mo + kRescaleSlack) ? mc : mo;
            float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int cj = 0; cj < CK / 16; ++cj) {
                float pv[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    pv[u] = mn == -INFINITY ? 0.f : exp2f(sv[cj * 8 + u] - mn);
                    l4[u & 3] += pv[u];
                }
                const int kc = half * (CK / 16) + cj;  // 8-key chunk index in the P row
                const uint32_t dst = sP + (kc >> 3) * 8192u + swz(h, kc & 7);
                asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(dst),
                             "r"(pack_f16(pv[0], pv[1])), "r"(pack_f16(pv[2], pv[3])),
                             "r"(pack_f16(pv[4], pv[5])), "r"(pack_f16(pv[6], pv[7])));
            }
            __syncwarp();
            sv[0] = (l4[0] + l4[1]) + (l4[2] + l4[3]);
            if (half == 0) fac[h] = mn;  // the new reference, published below
        }
        __syncthreads();
        if (sm_warp) part[half * H + h] = sv[0];
        if (tid == 0) flags[0] = 0;
        __syncthreads();
        if (tid < H) {
            const float mo = mref[tid], mn = fac[tid];
            const float f = mo == -INFINITY ? 0.f : exp2f(mo - mn);  // 1 when unchanged
            lrun[tid] = lrun[tid] * f + part[tid] + part[H + tid];
            mref[tid] = mn;
            fac[tid] = f;
            if (it > 0 && f != 1.f) flags[0] = 1;
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- rare: a head's reference moved after O^T holds earlier chunks
        if (flags[0]) {
            tc_fence_after();
            const int g = warp & 3;
            for (int t = 0; t < 2; ++t) {
                const int mt = (warp >> 2) * 2 + t;
                for (int h0 = 0; h0 < H; h0 += 32) {
                    const uint32_t ta = tmem + ((uint32_t)(g * 32) << 16) + O_COL + 64 * mt + h0;
                    uint32_t r[32];
                    tmem_ld32(ta, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[i] = __float_as_uint(__uint_as_float(r[i]) * fac[h0 + i]);
                    tmem_st32(ta, r);
                }
            }
            tc_fence_before();
            __syncthreads();
        }
        // ---- 5. O^T += V^T P^T (one thread issues); V^T = latent atoms of the K tile
        if (tid == 0) {
            tc_fence_after();
            for (int mt = 0; mt < DV / 128; ++mt)
                for (int kk = 0; kk < CK / 16; ++kk)
                    mma_bf16(tmem + O_COL + 64 * mt,
                             sdesc(sK + (2 * mt) * K_ATOM + kk * 2048u, K_ATOM, 1024),
                             sdesc(sP + (kk >> 2) * 8192u + (kk & 3) * 32u, 16, 1024), kIdescPV,
                             (it > 0 || kk > 0) ? 1u : 0u);
            mma_commit(smem_u32(&bars[1]));
        }
        got = warp == 0 ? mbar_wait(smem_u32(&bars[1]), it & 1) : true;
        ok = __syncthreads_and(got) != 0;  // the K tile and P are free again
        tc_fence_after();
    }

    pdl_trigger();  // only the epilogue is left: let the next kernel be scheduled

    if (cluster) {
        // ---- 6'. the nsplit CTAs of this sequence form one cluster.  Each
        // stores its unnormalised O and (m, l) to the partial buffers (they
        // stay in L2), the cluster barrier orders those stores before every
        // CTA's loads, then CTA r combines heads [r*hpc, (r+1)*hpc) from all
        // splits and writes the final rows: no separate merge launch.
        const bool mine = ok && c0 < c1;
        const size_t prow0 = (size_t)b * H * kMaxSplit;  // row (b, h, split) = prow0 + h*kMaxSplit + split
        if (mine) {
            const int g = warp & 3;
            for (int t = 0; t < 2; ++t) {
                const int mt = (warp >> 2) * 2 + t;
                const int d = mt * 128 + g * 32 + lane;
                for (int h0 = 0; h0 < H; h0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(tmem + ((uint32_t)(g * 32) << 16) + O_COL + 64 * mt + h0, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        __stcg(a.part_o + (prow0 + (size_t)(h0 + i) * kMaxSplit + split) * DV + d,
                               __uint_as_float(r[i]));
                }
            }
        }
        if (tid < H) {  // nothing (or nothing valid) from this split: weight 0
            const size_t row = prow0 + (size_t)tid * kMaxSplit + split;
            __stcg(a.part_ml + row * 2, mine ? mref[tid] : -INFINITY);
            __stcg(a.part_ml + row * 2 + 1, mine ? lrun[tid] : 0.f);
        }
        cluster_sync();  // every split's partial is stored
        const int hpc = (H + nsplit - 1) / nsplit;
        const int h_lo = split * hpc, h_hi = min(H, h_lo + hpc), nh = h_hi - h_lo;
        float* wts = part;  // [nh][nsplit] weights; fac[] = 1 / L
        if (tid < nh) {
            const int h = h_lo + tid;
            const size_t row = prow0 + (size_t)h * kMaxSplit;
            float m[8], l[8];
            float M = -INFINITY;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
                m[s2] = s2 < nsplit ? __ldcg(a.part_ml + (row + s2) * 2) : -INFINITY;
                l[s2] = s2 < nsplit ? __ldcg(a.part_ml + (row + s2) * 2 + 1) : 0.f;
                M = fmaxf(M, m[s2]);
            }
            float L = 0.f;
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
                if (s2 >= nsplit) break;
                const float w = (M == -INFINITY || m[s2] == -INFINITY) ? 0.f : exp2f(m[s2] - M);
                wts[tid * nsplit + s2] = w;
                L += w * l[s2];
            }
            fac[tid] = L > 0.f ? 1.f / L : 0.f;
            if (a.lse)
                a.lse[(size_t)b * H + h] = L > 0.f ? (M + __log2f(L)) * 0.6931471805599453f
                                                   : -INFINITY;
        }
        __syncthreads();
        // four items per pass: up to 4 x nsplit 16-byte L2 loads in flight
        constexpr int UNR = 4;
        for (int base = tid; base < nh * (DV / 4); base += UNR * NT) {
            float4 v[UNR][8];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int it2 = base + u * NT;
                if (it2 >= nh * (DV / 4)) continue;
                const int hh = it2 / (DV / 4), d4 = it2 - hh * (DV / 4);
                const float4* src = reinterpret_cast<const float4*>(
                    a.part_o + (prow0 + (size_t)(h_lo + hh) * kMaxSplit) * DV + 4 * d4);
#pragma unroll
                for (int s2 = 0; s2 < 8; ++s2)
                    if (s2 < nsplit && wts[hh * nsplit + s2] != 0.f)
                        v[u][s2] = __ldcg(src + (size_t)s2 * (DV / 4));
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int it2 = base + u * NT;
                if (it2 >= nh * (DV / 4)) continue;
                const int hh = it2 / (DV / 4), d4 = it2 - hh * (DV / 4);
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int s2 = 0; s2 < 8; ++s2) {
                    if (s2 >= nsplit) break;
                    const float w = wts[hh * nsplit + s2];
                    if (w == 0.f) continue;
                    acc.x = fmaf(w, v[u][s2].x, acc.x);
                    acc.y = fmaf(w, v[u][s2].y, acc.y);
                    acc.z = fmaf(w, v[u][s2].z, acc.z);
                    acc.w = fmaf(w, v[u][s2].w, acc.w);
                }
                const float inv = fac[hh];
                *reinterpret_cast<float4*>(a.out + ((size_t)b * H + h_lo + hh) * DV + 4 * d4) =
                    make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
            }
        }
        if (!ok && tid == 0) {
            set_status(a.status, KVC_DEV_TIMEOUT);
            mbar_wait(smem_u32(&bars[0]), 0);
            mbar_wait(smem_u32(&bars[1]), 0);
        }
    } else if (ok && c0 < c1) {
        // ---- 6. epilogue: thread = one latent channel, 64 heads from TMEM
        const int g = warp & 3;  // TMEM lanes 32g .. 32g+31
        for (int t = 0; t < 2; ++t) {
            const int mt = (warp >> 2) * 2 + t;
            const int d = mt * 128 + g * 32 + lane;
            for (int h0 = 0; h0 < H; h0 += 32) {
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(g * 32) << 16) + O_COL + 64 * mt + h0, r);
                if (nsplit == 1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float l = lrun[h0 + i];
                        a.out[((size_t)b * H + h0 + i) * DV + d] =
                            l > 0.f ? __uint_as_float(r[i]) / l : 0.f;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        a.part_o[(((size_t)b * H + h0 + i) * kMaxSplit + split) * DV + d] =
                            __uint_as_float(r[i]);
                }
            }
        }
        if (tid < H) {
            const float m = mref[tid], l = lrun[tid];
            if (nsplit == 1) {
                if (a.lse)
                    a.lse[(size_t)b * H + tid] =
                        l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
            } else {
                const size_t row = ((size_t)b * H + tid) * kMaxSplit + split;
                a.part_ml[row * 2] = m;
                a.part_ml[row * 2 + 1] = l;
            }
        }
    } else if (!ok && tid == 0) {
        // a bounded wait gave up: flag it, give the issued MMAs one more bounded
        // wait each, then free the tensor memory
        set_status(a.status, KVC_DEV_TIMEOUT);
        mbar_wait(smem_u32(&bars[0]), 0);
        mbar_wait(smem_u32(&bars[1]), 0);
    }
    cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                     "r"(TMEM_COLS));
    }
}

}  // namespace tc05

bool tc05_supported(const kvc_config& c, const Shape& sh) {
    return c.act_dtype == KVC_BF16 && c.scale_fmt == KVC_SCALE_UE4M3 && c.n_heads == tc05::H &&
           sh.D == tc05::D && sh.Dv == tc05::DV && sh.rb <= (int)tc05::RAW_STRIDE;
}

// Launches the chunks of every sequence; returns the number of partial
// results the caller still has to merge (1 when the kernel wrote the final
// output itself), or a negative value on a launch error.
int launch_attention_tc05(const kvc_config& c, const Shape& sh, const AttnArgs& a,
                          cudaStream_t s) {
    const int total = c.topk + a.window_len;
    const int nchunks = (total + tc05::CK - 1) / tc05::CK;
    static bool attr_set[64] = {};
    static int sm_count[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = 148;
    if (dev >= 0 && dev < 64) {
        if (!sm_count[dev]) cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
        sms = sm_count[dev];
    }
    // chunks per CTA: as few as keep every (sequence, split) CTA in one wave
    // (one CTA per SM), and at most kMaxSplit splits
    int cps = (int)(((long long)a.batch * nchunks + sms - 1) / sms);
    cps = std::max(cps, (nchunks + kMaxSplit - 1) / kMaxSplit);
    cps = std::max(cps, 1);
    const int nsplit = nchunks == 0 ? 1 : (nchunks + cps - 1) / cps;
    if (nsplit > kMaxSplit) return -1;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if (cudaFuncSetAttribute(tc05::attn_tc05_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)tc05::SMEM_BYTES) != cudaSuccess)
            return -1;
        attr_set[dev] = true;
    }
    // the splits of one sequence merge inside a cluster when they fit one
    const int cluster = (nsplit > 1 && nsplit <= 8) ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nsplit, a.batch);
    cfg.blockDim = dim3(tc05::NT);
    cfg.dynamicSmemBytes = tc05::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster ? nsplit : 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    trace_before("attn_tc05", s);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, tc05::attn_tc05_kernel, a, sh, c.topk,
                                             c.sm_scale * 1.4426950408889634f, nsplit, cps,
                                             (int)(c.scale_fmt == KVC_SCALE_UE4M3), cluster);
    trace_after(s);
    if (e != cudaSuccess) return -1;
    return cluster ? 1 : nsplit;  // a merged cluster needs no merge kernel
}

}  // namespace kvc
