// pack.cu -- 2:1 gated token compression + FP4 E2M1 group quantisation +
// indexer-key append (the write side of the compressed cache).
//
// Method: "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
// 压缩到 890 B的？" (acejoy.com) part 3 breakthrough 4 (CSA: every 2 tokens'
// KV become 1 entry) and part 4 "P4 main KV" (E2M1, groups of channels share
// one 8-bit scale); "DeepSeek V4.1 Flash KV Cache压缩实战" (gtnt.cn) 3.1 (each
// group gets a scale, elements stored relative to it) and 3.2 (a learned key
// compressor maps several tokens to one entry).
//
// Design (B200): a pure HBM stream.  A team of 8 lanes owns one entry (4
// entries per warp, 32 per CTA); lane l of a team owns the 8-channel chunks
// c = l, l+8, ..., so for the 576-channel MLA entry every lane holds 9 chunks
// and no lane idles.  Each chunk of each token is one 16-byte load and the 8
// lanes of a team read 128 contiguous bytes; a chunk's eight codes leave as one
// 4-byte store (a team writes 32 contiguous bytes per chunk step).  Appends of
// more than 4,096 entries with groups of at most 64 channels take the
// streaming kernel (pack_stream_kernel: the chunks read twice, L1-resident
// between the passes, arithmetic on fp32 pairs, no division); groups of 128
// channels the register-held kernel (pack_kernel: the raw chunks kept packed in
// registers between the passes, group maxima through shared memory); decode
// appends a warp per entry (pack_small_kernel) and 4:1 appends likewise
// (pack_group4_kernel).
//
// Bit-exactness: the gate logit difference is accumulated in fp32 in a fixed
// order -- lane l sums its chunks in increasing order, one fmaf per channel
// after an fp32 subtraction, then a xor tree over offsets 4, 2, 1 -- and the
// pair weight w0 = 1 / (1 + exp(-delta)) uses the exp below (Cody-Waite
// reduction with a 16-bit head of ln 2, degree-7 Taylor polynomial in Horner
// form, exact power-of-two scaling), so every implementation of this order
// produces the same fp32 entry and therefore the same codes.
#include "kvc_internal.cuh"
#include "tc05_common.cuh"

namespace kvc {
namespace {

constexpr float kLn2HiF = 0x1.62e4p-1f;
constexpr float kLn2LoF = 0x1.7f7d1cp-20f;
constexpr float kInvLn2F = 0x1.715476p+0f;

__device__ __forceinline__ float exp_cody_waite(float x) {
    if (x != x) return x;
    if (x > 88.0f) return __int_as_float(0x7f800000);
    if (x < -87.0f) return 0.0f;
    const float n = rintf(__fmul_rn(x, kInvLn2F));
    float r = __fmaf_rn(-n, kLn2HiF, x);
    r = __fmaf_rn(-n, kLn2LoF, r);
    // 1/k! for k = 7 .. 0
    float p = 0x1.a01a02p-13f;
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
    p = __fmaf_rn(p, r, 0x1.111112p-7f);
    p = __fmaf_rn(p, r, 0x1.555556p-5f);
    p = __fmaf_rn(p, r, 0x1.555556p-3f);
    p = __fmaf_rn(p, r, 0x1.0p-1f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    return __fmul_rn(p, __int_as_float(((int)n + 127) << 23));
}

// Raw token chunk (8 channels) kept in registers between the passes.
template <typename T>
struct Chunk;
template <>
struct Chunk<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) {
        v = __ldcs(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ void load_cached(const __nv_bfloat16* p) {
        v = __ldg(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ void zero() { v = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void load_shared(const __nv_bfloat16* p) {
        v = *reinterpret_cast<const uint4*>(p);
    }
    // first read of a chunk (kept in L1 for the second pass) / its last read
    __device__ __forceinline__ void load_keep(const __nv_bfloat16* p) {
        asm volatile("ld.global.nc.L1::evict_last.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "l"(p));
    }
    __device__ __forceinline__ void load_last(const __nv_bfloat16* p) {
        asm volatile("ld.global.nc.L1::evict_first.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "l"(p));
    }
    __device__ __forceinline__ void store_shared(__nv_bfloat16* p) const {
        *reinterpret_cast<uint4*>(p) = v;
    }
    __device__ __forceinline__ float get(int t) const {
        const uint32_t w = t < 2 ? v.x : t < 4 ? v.y : t < 6 ? v.z : v.w;
        return (t & 1) ? __uint_as_float(w & 0xFFFF0000u) : __uint_as_float(w << 16);
    }
    // channels 2k, 2k + 1 as an fp32 pair (f2_* below)
    __device__ __forceinline__ uint64_t pair(int k) const;
};
template <>
struct Chunk<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const float* p) {
        a = __ldcs(reinterpret_cast<const float4*>(p));
        b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void load_cached(const float* p) {
        a = __ldg(reinterpret_cast<const float4*>(p));
        b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void load_shared(const float* p) {
        a = reinterpret_cast<const float4*>(p)[0];
        b = reinterpret_cast<const float4*>(p)[1];
    }
    __device__ __forceinline__ void load_keep(const float* p) {
        asm volatile("ld.global.nc.L1::evict_last.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(a.x), "=f"(a.y), "=f"(a.z), "=f"(a.w)
                     : "l"(p));
        asm volatile("ld.global.nc.L1::evict_last.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(b.x), "=f"(b.y), "=f"(b.z), "=f"(b.w)
                     : "l"(p + 4));
    }
    __device__ __forceinline__ void load_last(const float* p) {
        asm volatile("ld.global.nc.L1::evict_first.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(a.x), "=f"(a.y), "=f"(a.z), "=f"(a.w)
                     : "l"(p));
        asm volatile("ld.global.nc.L1::evict_first.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(b.x), "=f"(b.y), "=f"(b.z), "=f"(b.w)
                     : "l"(p + 4));
    }
    __device__ __forceinline__ void store_shared(float* p) const {
        reinterpret_cast<float4*>(p)[0] = a;
        reinterpret_cast<float4*>(p)[1] = b;
    }
    __device__ __forceinline__ float get(int t) const {
        const float4& q = t < 4 ? a : b;
        const int u = t & 3;
        return u == 0 ? q.x : u == 1 ? q.y : u == 2 ? q.z : q.w;
    }
    __device__ __forceinline__ uint64_t pair(int k) const;
};

__device__ __forceinline__ void load8_gate(const float* p, float v[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Eight E2M1 codes of fl(x[t] / s) (s > 0, x finite) without a division per
// element.  With r = 1/s rounded, x * r(1 - 2^-20) and x * r(1 + 2^-20)
// (each product rounded) bracket the correctly rounded quotient: the few
// roundings move them by a handful of 2^-24 relative units, far less than
// the 2^-20 offset.  Rounding to the E2M1 grid is monotone, so when both
// brackets give the same codes the quotient gives them too; otherwise (a
// quotient within 2^-20 of a rounding midpoint, or r not finite) the eight
// quotients are divided out exactly.
__device__ __forceinline__ uint32_t e2m1x8_quotient(const float x[8], float s) {
    const float r = __frcp_rn(s);
    if (r < 3.0e38f) {
        const float rl = __fmul_rn(r, 1.0f - 0x1p-20f), rh = __fmul_rn(r, 1.0f + 0x1p-20f);
        float lo[8], hi[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            lo[t] = __fmul_rn(x[t], rl);
            hi[t] = __fmul_rn(x[t], rh);
        }
        const uint32_t cl = e2m1x8_from_f32(lo);
        if (cl == e2m1x8_from_f32(hi)) return cl;
    }
    float v[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) v[t] = fminf(fmaxf(__fdiv_rn(x[t], s), -6.f), 6.f);
    return e2m1x8_from_f32(v);
}

// ---- fp32 pairs: Blackwell's f32x2 instructions perform two IEEE
// single-precision operations at once, each rounded exactly as its scalar
// form, so pair arithmetic gives the bits of the scalar order it replaces.
__device__ __forceinline__ uint64_t f2_make(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float f2_lo(uint64_t p) { return __uint_as_float((uint32_t)p); }
__device__ __forceinline__ float f2_hi(uint64_t p) { return __uint_as_float((uint32_t)(p >> 32)); }
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t Chunk<__nv_bfloat16>::pair(int k) const {
    const uint32_t w = k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
    return f2_make(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
__device__ __forceinline__ uint64_t Chunk<float>::pair(int k) const {
    return k == 0 ? f2_make(a.x, a.y) : k == 1 ? f2_make(a.z, a.w) : k == 2 ? f2_make(b.x, b.y)
                                                                             : f2_make(b.z, b.w);
}
// max(|a|, |b|) in magnitude (the sign is that of neither), NaN if either is
__device__ __forceinline__ float absmax_nan(float a, float b) {
    float r;
    asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// m / 6 correctly rounded (m >= 0 finite) without a division: the product by
// c = RN(1/6) corrected once (q0 = m c; r = m - 6 q0, exact by one fma;
// q = q0 + r c by a second), Markstein's correction step as used for division
// by a constant known in advance (Brisebarre, Muller and Raina, 2004).  For
// the divisor 6 it is correctly rounded for every m >= 2^-122 (all fp32
// values checked); smaller m (subnormal quotients) are divided.
__device__ __forceinline__ float div6_rn(float m) {
    if (m < 0x1p-122f) return __fdiv_rn(m, 6.0f);
    constexpr float c = 0x1.555556p-3f;
    const float q0 = __fmul_rn(m, c);
    const float r = __fmaf_rn(-q0, 6.0f, m);
    return __fmaf_rn(r, c, q0);
}

// Eight E2M1 codes (raw: a zero keeps its sign) of four fp32 pairs in [-6, 6]
// or saturating, element 2k + h (h = 0 low, 1 high half of pair k) in the
// nibble of value 2k + h.
__device__ __forceinline__ uint32_t e2m1x8_raw_f2(uint64_t p0, uint64_t p1, uint64_t p2,
                                                  uint64_t p3) {
    uint32_t w;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .f32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
        "mov.b64 {l0, h0}, %1;\n\tmov.b64 {l1, h1}, %2;\n\t"
        "mov.b64 {l2, h2}, %3;\n\tmov.b64 {l3, h3}, %4;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, h0, l0;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, h1, l1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, h2, l2;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, h3, l3;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(w)
        : "l"(p0), "l"(p1), "l"(p2), "l"(p3));
    return w;
}
__device__ __forceinline__ uint32_t e2m1_clear_negzero(uint32_t w) {
    const uint32_t mag = w & 0x77777777u;
    const uint32_t nonzero = (mag + 0x77777777u) & 0x88888888u;
    return w & (0x77777777u | nonzero);
}

// e2m1x8_quotient for values held as four fp32 pairs, with the reciprocal and
// its two brackets given (rl = RN(r (1 - 2^-20)), rh = RN(r (1 + 2^-20)),
// r = RN(1 / s), s > 0 an E4M3 scale so r is finite): the same products,
// two to an instruction, and the same exact fallback.
__device__ __forceinline__ uint32_t e2m1x8_quotient_f2(const uint64_t v[4], float s, float rl,
                                                       float rh) {
    const uint64_t RL = f2_make(rl, rl), RH = f2_make(rh, rh);
    const uint32_t cl =
        e2m1x8_raw_f2(f2_mul(v[0], RL), f2_mul(v[1], RL), f2_mul(v[2], RL), f2_mul(v[3], RL));
    const uint32_t ch =
        e2m1x8_raw_f2(f2_mul(v[0], RH), f2_mul(v[1], RH), f2_mul(v[2], RH), f2_mul(v[3], RH));
    if (cl == ch) return e2m1_clear_negzero(cl);
    float q[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        q[2 * k] = fminf(fmaxf(__fdiv_rn(f2_lo(v[k]), s), -6.f), 6.f);
        q[2 * k + 1] = fminf(fmaxf(__fdiv_rn(f2_hi(v[k]), s), -6.f), 6.f);
    }
    return e2m1x8_from_f32(q);
}

constexpr int kThreads = 256;
constexpr int kTeams = kThreads / 8;  // entries per CTA
constexpr int kTailBytes = 528;       // >= 128 groups x 4 bytes, padded
constexpr int kMaxChunks = 128;       // D <= 1024

// MAXJ: chunks per lane (D <= 64 * MAXJ).
template <typename T, int MAXJ>
__global__ void __launch_bounds__(kThreads, (MAXJ <= 4 || (sizeof(T) == 2 && MAXJ <= 9)) ? 2 : 1)
pack_kernel(PackArgs a, Shape sh, int ue4m3, int di) {
    pdl_wait();
    __shared__ __align__(16) uint8_t tail_smem[kTeams][kTailBytes];
    __shared__ float cmax_smem[kTeams][kMaxChunks];  // only for groups wider than a team pass
    const int lane = threadIdx.x & 31;
    const int team = threadIdx.x >> 3, l = threadIdx.x & 7;
    const long long e = (long long)blockIdx.x * kTeams + team;
    const int half = a.n_new >> 1;
    const bool in_range = e < (long long)a.batch * half;
    int b = 0, i = 0, base = 0;
    bool valid = false;
    if (in_range) {
        b = (int)(e / half);
        i = (int)(e % half);
        base = a.n_entries[b];
        valid = base >= 0 && base + half <= a.capacity;
        if (!valid && i == 0 && l == 0) set_status(a.status, KVC_DEV_CAPACITY);
    }
    const int D = sh.D, nchunk = D >> 3;
    const long long pos = (long long)base + i;
    const T* k0p = static_cast<const T*>(a.tokens) + ((long long)b * a.n_new + 2 * i) * D;
    const T* k1p = k0p + D;

    Chunk<T> k0[MAXJ], k1[MAXJ];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = l + 8 * j;
        if (valid && c < nchunk) {
            k0[j].load(k0p + 8 * c);
            k1[j].load(k1p + 8 * c);
        } else {
            k0[j].zero();
            k1[j].zero();
        }
    }

    // gate logit difference, fixed order (all lanes take part in the shuffles)
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = l + 8 * j;
        if (valid && c < nchunk) {
            float g[8];
            load8_gate(a.gate + 8 * c, g);
#pragma unroll
            for (int t = 0; t < 8; ++t)
                acc = __fmaf_rn(g[t], __fsub_rn(k0[j].get(t), k1[j].get(t)), acc);
        }
    }
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 4));
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 2));
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 1));
    const float w0 = __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_cody_waite(-acc)));
    const float w1 = __fsub_rn(1.0f, w0);

    uint8_t* rec = a.records + ((long long)b * a.capacity + pos) * sh.rb;
    uint8_t* tail = tail_smem[team];
    const int tail_len = sh.rb - sh.code_bytes;  // multiple of 4
    for (int t = l * 4; t < tail_len; t += 32) *reinterpret_cast<uint32_t*>(tail + t) = 0u;

    // entry values (replacing the token chunks in registers) and lane-local
    // chunk maxima; non-finite values are flagged and coded as 0
    bool bad = false;
    float cmax[MAXJ];
    float x[MAXJ][8];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = l + 8 * j;
        const bool active = valid && c < nchunk;
        float m = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float v = __fmaf_rn(w0, k0[j].get(t), __fmul_rn(w1, k1[j].get(t)));
            if (!isfinite(v)) {
                if (active) bad = true;
                v = 0.f;
            }
            x[j][t] = v;
            m = fmaxf(m, fabsf(v));
        }
        cmax[j] = m;
    }
    // group maxima
    const int lpg = sh.lpg;
    if (lpg <= 8) {
#pragma unroll
        for (int j = 0; j < MAXJ; ++j)
            for (int o = 1; o < lpg; o <<= 1)
                cmax[j] = fmaxf(cmax[j], __shfl_xor_sync(0xffffffffu, cmax[j], o));
    } else {
#pragma unroll
        for (int j = 0; j < MAXJ; ++j)
            if (l + 8 * j < kMaxChunks) cmax_smem[team][l + 8 * j] = cmax[j];
        __syncwarp();
#pragma unroll
        for (int j = 0; j < MAXJ; ++j) {
            const int c = l + 8 * j;
            if (c < nchunk) {
                const int g0 = c / lpg * lpg;
                float m = 0.f;
                for (int u = g0; u < min(g0 + lpg, nchunk); ++u) m = fmaxf(m, cmax_smem[team][u]);
                cmax[j] = m;
            }
        }
    }
    __syncwarp();

    // scales and codes
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = l + 8 * j;
        if (!(valid && c < nchunk)) continue;
        float s = __fdiv_rn(cmax[j], 6.0f);
        uint32_t sbyte = 0;
        if (ue4m3) {
            sbyte = e4m3_from_f32(s);
            s = e4m3_to_f32(sbyte);
        }
        *reinterpret_cast<uint32_t*>(rec + 4 * c) = s > 0.f ? e2m1x8_quotient(x[j], s) : 0u;
        if (c % lpg == 0) {
            const int gi = c / lpg;
            if (ue4m3)
                tail[gi] = (uint8_t)sbyte;
            else
                *reinterpret_cast<float*>(tail + 4 * gi) = s;
        }
    }
    __syncwarp();
    if (valid) {
        for (int t = l * 4; t < tail_len; t += 32)
            *reinterpret_cast<uint32_t*>(rec + sh.code_bytes + t) =
                *reinterpret_cast<const uint32_t*>(tail + t);
        // indexer key append: Di bytes as 16-byte pieces
        const uint4* src =
            reinterpret_cast<const uint4*>(a.idx_k_new + ((long long)b * half + i) * di);
        uint4* dst = reinterpret_cast<uint4*>(a.idx_k + ((long long)b * a.capacity + pos) * di);
        for (int p = l; p < (di >> 4); p += 8) dst[p] = __ldcs(src + p);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, KVC_DEV_NONFINITE);
}

// One chunk of the gate logit difference, in the fixed order: for channels
// 2k, 2k + 1 of the chunk, d = k0 - k1 (an fp32 pair subtraction), then one
// fmaf per channel into the lane's running sum.
template <typename T>
__device__ __forceinline__ float gate_chunk(float acc, const Chunk<T>& x0, const Chunk<T>& x1,
                                            const float (&g)[8]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint64_t d = f2_sub(x0.pair(k), x1.pair(k));
        acc = __fmaf_rn(g[2 * k], f2_lo(d), acc);
        acc = __fmaf_rn(g[2 * k + 1], f2_hi(d), acc);
    }
    return acc;
}
// bf16 tokens: k0's halves enter the subtraction as bf16 operands (the
// mixed-precision sub widens them exactly, then rounds k0 - k1 once in fp32,
// as the pair subtraction does), so only k1 is unpacked.
__device__ __forceinline__ float bf16_minus_f32(uint32_t w, bool hi, float c) {
    float r;
    if (hi)
        asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tsub.rn.f32.bf16 %0, h, %2;\n\t}"
            : "=f"(r)
            : "r"(w), "f"(c));
    else
        asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tsub.rn.f32.bf16 %0, l, %2;\n\t}"
            : "=f"(r)
            : "r"(w), "f"(c));
    return r;
}
template <>
__device__ __forceinline__ float gate_chunk(float acc, const Chunk<__nv_bfloat16>& x0,
                                            const Chunk<__nv_bfloat16>& x1,
                                            const float (&g)[8]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t w0 = k == 0 ? x0.v.x : k == 1 ? x0.v.y : k == 2 ? x0.v.z : x0.v.w;
        const uint32_t w1 = k == 0 ? x1.v.x : k == 1 ? x1.v.y : k == 2 ? x1.v.z : x1.v.w;
        const float dlo = bf16_minus_f32(w0, false, __uint_as_float(w1 << 16));
        const float dhi = bf16_minus_f32(w0, true, __uint_as_float(w1 & 0xFFFF0000u));
        acc = __fmaf_rn(g[2 * k], dlo, acc);
        acc = __fmaf_rn(g[2 * k + 1], dhi, acc);
    }
    return acc;
}

// The pair weights from the team's eight running sums (xor tree over 4, 2, 1).
__device__ __forceinline__ void gate_weights(float acc, uint64_t& W0, uint64_t& W1) {
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 4));
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 2));
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 1));
    const float w0 = __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_cody_waite(-acc)));
    const float w1 = __fsub_rn(1.0f, w0);
    W0 = f2_make(w0, w0);
    W1 = f2_make(w1, w1);
}

// Pass 2 of one chunk step (chunk c of the lane's entry): the entry values
// v = w0 k0 + w1 k1, the group maximum across the LPG lanes holding the
// group's chunks, the scale and the eight codes.  Every lane of the warp
// calls it (the maximum is a warp shuffle); only `active` lanes store: the
// code word into the record, the scale (the group's first lane) into the
// team's tail.  Inactive lanes must pass zero chunks.
template <typename T, int LPG>
__device__ __forceinline__ void quantise_chunk(const Chunk<T>& x0, const Chunk<T>& x1,
                                               uint64_t W0, uint64_t W1, bool active, int c,
                                               int ue4m3, const float4* tab, uint8_t* rec,
                                               uint8_t* tail, bool& bad) {
    uint64_t v[4];  // v = w0 k0 + w1 k1, rounded as fmaf(w0, k0, w1 * k1)
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = f2_fma(W0, x0.pair(k), f2_mul(W1, x1.pair(k)));
    // the chunk's largest magnitude (a tree of pairwise maxima), then the group's
    float m = absmax_nan(absmax_nan(absmax_nan(f2_lo(v[0]), f2_hi(v[0])),
                                    absmax_nan(f2_lo(v[1]), f2_hi(v[1]))),
                         absmax_nan(absmax_nan(f2_lo(v[2]), f2_hi(v[2])),
                                    absmax_nan(f2_lo(v[3]), f2_hi(v[3]))));
#pragma unroll
    for (int o = 1; o < LPG; o <<= 1) m = absmax_nan(m, __shfl_xor_sync(0xffffffffu, m, o));
    m = fabsf(m);
    if (__any_sync(0xffffffffu, !(m <= 3.0e38f))) {
        // a NaN or inf somewhere in the warp: value by value, non-finite
        // values coded as 0 (and reported)
        m = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float lo = f2_lo(v[k]), hi = f2_hi(v[k]);
            if (!isfinite(lo)) {
                if (active) bad = true;
                lo = 0.f;
            }
            if (!isfinite(hi)) {
                if (active) bad = true;
                hi = 0.f;
            }
            v[k] = f2_make(lo, hi);
            m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
        }
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    if (!active) return;
    const float sc = div6_rn(m);
    uint32_t code, sbyte = 0;
    if (ue4m3) {
        sbyte = e4m3_from_f32(sc);
        const float4 t = tab[sbyte];  // the scale, its reciprocal brackets
        code = t.x > 0.f ? e2m1x8_quotient_f2(v, t.x, t.y, t.z) : 0u;
    } else {
        float x[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            x[2 * k] = f2_lo(v[k]);
            x[2 * k + 1] = f2_hi(v[k]);
        }
        code = sc > 0.f ? e2m1x8_quotient(x, sc) : 0u;
    }
    *reinterpret_cast<uint32_t*>(rec + 4 * c) = code;
    if ((c & (LPG - 1)) == 0) {
        const int gi = c / LPG;
        if (ue4m3)
            tail[gi] = (uint8_t)sbyte;
        else
            *reinterpret_cast<float*>(tail + 4 * gi) = sc;
    }
}

// Reciprocal brackets of the 128 UE4M3 scale values (entry i: scale byte i).
__device__ __forceinline__ void fill_scale_tables(float4* tab, int i) {
    const float sv = e4m3_to_f32(i);
    const float r = __frcp_rn(sv);
    tab[i] = make_float4(sv, __fmul_rn(r, 1.0f - 0x1p-20f), __fmul_rn(r, 1.0f + 0x1p-20f), 0.f);
}

// Streaming form of pack_kernel for groups of at most 64 channels (LPG <= 8
// chunks per group, so a group's chunks sit in the team's lanes at the same
// chunk step): the same arithmetic in the same order, but no token chunk is
// held across the whole entry.  Pass 1 streams the chunks for the gate (first
// reads, kept in L1 by an evict-last hint); pass 2 reads each chunk again
// (L1/L2, evict-first: its last use), forms the entry values, takes the group
// maximum across the team and quantises it right away.  The small register
// footprint keeps 40 warps per SM, which is what hides the two reads'
// latency.  CTA (x, b) packs entries [32 x, 32 x + 32) of sequence b's
// append, a team of 8 lanes per entry.
//
// Instruction count matters as much: the arithmetic runs on fp32 pairs
// (f2_*), the group maximum propagates NaN so that one test per chunk replaces
// a finiteness test per value (a warp that meets a non-finite value redoes
// that chunk value by value), the scale m / 6 needs no division (div6_rn),
// with E4M3 scales the reciprocal and its brackets come from a 128-entry table
// (one per scale byte), and the group width LPG is a compile-time constant.
template <typename T, int MAXJ, int LPG>
__global__ void __launch_bounds__(kThreads, 5)
pack_stream_kernel(PackArgs a, Shape sh, int ue4m3, int di, int tail_stride) {
    extern __shared__ __align__(16) uint8_t dsm[];  // per-entry tails
    __shared__ float4 tab[128];  // per E4M3 scale byte: scale, reciprocal brackets
    const int tid = threadIdx.x, lane = tid & 31, team = tid >> 3, l = tid & 7;
    const int b = blockIdx.y, half = a.n_new >> 1;
    const int e0 = blockIdx.x * kTeams, ne = min(kTeams, half - e0);
    const int i = e0 + team;  // this team's entry within the append
    const int D = sh.D, nchunk = D >> 3;
    uint8_t* tail = dsm + team * tail_stride;
    const int tail_len = sh.rb - sh.code_bytes;  // multiple of 4
    if (ue4m3 && tid < 128) fill_scale_tables(tab, tid);
    for (int t = l * 4; t < tail_len; t += 32) *reinterpret_cast<uint32_t*>(tail + t) = 0u;
    __syncthreads();
    pdl_wait();
    const int base = a.n_entries[b];
    if (!(base >= 0 && base + half <= a.capacity)) {  // the same for the whole CTA
        if (blockIdx.x == 0 && tid == 0) set_status(a.status, KVC_DEV_CAPACITY);
        return;
    }
    const bool valid = team < ne;
    const long long pos = (long long)base + i;
    const T* k0p = static_cast<const T*>(a.tokens) + ((long long)b * a.n_new + 2 * i) * D;
    const T* k1p = k0p + D;
    const int jn = valid ? (nchunk - l + 7) / 8 : 0;  // chunks of this lane

    // pass 1: gate logit difference, fixed order (lane l: chunks l, l+8, ...)
    float acc = 0.f;
#pragma unroll 3
    for (int j = 0; j < MAXJ; ++j) {
        const int c = l + 8 * j;
        if (j < jn) {
            Chunk<T> x0, x1;
            x0.load_keep(k0p + 8 * c);
            x1.load_keep(k1p + 8 * c);
            float g[8];
            load8_gate(a.gate + 8 * c, g);
            acc = gate_chunk(acc, x0, x1, g);
        }
    }
    uint64_t W0, W1;
    gate_weights(acc, W0, W1);
    uint8_t* rec = a.records + ((long long)b * a.capacity + pos) * sh.rb;

    // pass 2: entry values, group maxima (xor over the group's lanes), codes
    bool bad = false;
#pragma unroll 2
    for (int j = 0; j < MAXJ; ++j) {
        const int c = l + 8 * j;
        const bool active = j < jn;
        Chunk<T> x0, x1;
        if (active) {
            x0.load_last(k0p + 8 * c);
            x1.load_last(k1p + 8 * c);
        } else {
            x0.zero();
            x1.zero();
        }
        quantise_chunk<T, LPG>(x0, x1, W0, W1, active, c, ue4m3, tab, rec,
                               tail, bad);
    }
    __syncwarp();
    if (valid) {
        for (int t = l * 4; t < tail_len; t += 32)
            *reinterpret_cast<uint32_t*>(rec + sh.code_bytes + t) =
                *reinterpret_cast<const uint32_t*>(tail + t);
        const uint4* src =
            reinterpret_cast<const uint4*>(a.idx_k_new + ((long long)b * half + i) * di);
        uint4* dst = reinterpret_cast<uint4*>(a.idx_k + ((long long)b * a.capacity + pos) * di);
        for (int p = l; p < (di >> 4); p += 8) dst[p] = __ldcs(src + p);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, KVC_DEV_NONFINITE);
}

// Ring form of the streaming kernel for long appends of bf16 tokens (groups
// of at most 64 channels): the same arithmetic in the same order, fed from
// shared memory instead of L1/L2.  One persistent CTA per SM walks units of
// kRingE consecutive entries of one sequence (unit u of the grid-stride
// sequence u = blockIdx.x + k gridDim.x); a unit's token pairs are contiguous
// in the token array, so one producer thread moves each unit with a single
// bulk copy into a ring of shared-memory stages.  kRingGroups groups of
// kRingE / 4 consumer warps take the units in turn (group k mod kRingGroups,
// stage k mod stages), read every chunk twice from the stage -- the gate
// pass and the quantisation pass -- and hand the stage back on its `empty`
// barrier.  The second read of each chunk no longer goes out to L1/L2 (the
// streaming kernel's latency).  The kernel is bound by instruction issue, so
// the shared memory goes to the warps: at 576 channels the 12 stages of
// 18 KB hold 11 groups' units (22 consumer warps) and one unit in flight;
// measured on 32 x 4096 new tokens, 16 entries per unit in 4 groups (two
// units in flight) took 56 us, 8 in 10 groups 54 us, 8 in 11 groups 51.6 us
// (the streaming kernel 61.6 us).  Waits are bounded: a consumer or the
// producer that gives up sets KVC_DEV_TIMEOUT and stops; the producer always
// waits (up to 2 s) for its copies in flight before the CTA exits.
constexpr int kRingE = 8;        // entries per unit (and per stage): 2 warps of 4 teams
constexpr int kRingGroups = 11;  // consumer groups of kRingE / 4 warps (22 warps)
constexpr int kRingConsumerWarps = kRingGroups * kRingE / 4;
constexpr int kRingThreads = (kRingConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kRingMaxStages = 32;
constexpr unsigned long long kRingDrainNs = 2000000000ull;

__device__ __forceinline__ void ring_bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                               uint32_t bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
        "[%1], %2, [%3], %4;\n" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void ring_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}

template <int MAXJ, int LPG>
__global__ void __launch_bounds__(kRingThreads, 1)
pack_ring_kernel(PackArgs a, Shape sh, int ue4m3, int di, int tail_stride, int stages,
                 uint32_t stage_bytes, long long n_units, unsigned long long wait_ns) {
    using T = __nv_bfloat16;
    extern __shared__ __align__(128) uint8_t rsm[];  // stages | gate | team tails
    __shared__ float4 tab[128];
    // full[f]: unit k's copy has landed, f = k % nfull (nfull = stages +
    // kRingGroups); empty[k % stages]: unit k's stage has been read.  A stage
    // carries the units of every group in turn, so a full barrier per stage
    // could be tested by a group that never saw the stage's previous phase
    // complete (mbarrier waits tell phases apart by parity only).  With one
    // full barrier per unit index modulo stages + kRingGroups, the previous
    // use of unit k's barrier is unit k - stages - kRingGroups, which was read
    // before unit k - kRingGroups (the group's own previous unit) could be
    // copied into its stage: every parity wait tests the phase it means.
    __shared__ __align__(8) uint64_t full[kRingMaxStages + kRingGroups], empty[kRingMaxStages];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int D = sh.D, nchunk = D >> 3, half = a.n_new >> 1;
    const int units_per_seq = (half + kRingE - 1) / kRingE;
    const uint32_t ring = tc::smem_u32(rsm);
    float* gate_s = reinterpret_cast<float*>(rsm + (size_t)stages * stage_bytes);
    uint8_t* tails = rsm + (size_t)stages * stage_bytes + (size_t)D * 4;
    const int tail_len = sh.rb - sh.code_bytes;  // multiple of 4

    if (ue4m3 && tid < 128) fill_scale_tables(tab, tid);
    const int nfull = stages + kRingGroups;
    if (tid == 0) {
        for (int f = 0; f < nfull; ++f) tc::mbar_init(tc::smem_u32(&full[f]), 1);
        for (int st = 0; st < stages; ++st) tc::mbar_init(tc::smem_u32(&empty[st]), kRingE / 4);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    for (int t = tid * 4; t < kRingConsumerWarps * 4 * tail_stride; t += kRingThreads * 4)
        *reinterpret_cast<uint32_t*>(tails + t) = 0u;
    pdl_wait();
    for (int t = tid; t < D / 4; t += kRingThreads)
        reinterpret_cast<float4*>(gate_s)[t] = __ldg(reinterpret_cast<const float4*>(a.gate) + t);
    __syncthreads();

    if (warp == kRingConsumerWarps) {  // the producer
        if (lane != 0) return;
        const T* tokens = static_cast<const T*>(a.tokens);
        long long k = 0;
        int f = 0;
        for (;; ++k) {
            const long long u = blockIdx.x + k * gridDim.x;
            if (u >= n_units) break;
            const int st = (int)(k % stages);
            if (k >= stages &&
                !tc::mbar_wait(tc::smem_u32(&empty[st]), (uint32_t)((k / stages - 1) & 1),
                               wait_ns)) {
                set_status(a.status, KVC_DEV_TIMEOUT);
                break;
            }
            const unsigned ub = (unsigned)u / (unsigned)units_per_seq;
            const int b = (int)ub, e0 = (int)((unsigned)u - ub * (unsigned)units_per_seq) * kRingE;
            const int ne = min(kRingE, half - e0);
            ring_bulk_load(ring + (uint32_t)st * stage_bytes,
                           tokens + ((long long)b * a.n_new + 2 * e0) * D,
                           (uint32_t)(ne * 2 * D * (int)sizeof(T)), tc::smem_u32(&full[f]));
            if (++f == nfull) f = 0;
        }
        // copies still in flight must land before the CTA exits
        for (long long j = k > stages ? k - stages : 0; j < k; ++j)
            tc::mbar_wait(tc::smem_u32(&full[(int)(j % nfull)]), (uint32_t)((j / nfull) & 1),
                          kRingDrainNs);
        return;
    }

    // consumers: warp wi of group grp; team `team` of the warp takes entry
    // 4 wi + team of each of the group's units
    const int grp = warp / (kRingE / 4), wi = warp % (kRingE / 4);
    const int team = lane >> 3, l = lane & 7;
    uint8_t* tail = tails + (warp * 4 + team) * tail_stride;
    const int ei = wi * 4 + team;  // entry within the unit
    bool bad = false;
    int f = grp, rf = 0;
    for (long long k = grp;; k += kRingGroups) {
        const long long u = blockIdx.x + k * gridDim.x;
        if (u >= n_units) break;
        const int st = (int)(k % stages);
        const bool got = __all_sync(
            0xffffffffu,
            tc::mbar_wait(tc::smem_u32(&full[f]), (uint32_t)(rf & 1), wait_ns));
        if (!got) {
            if (lane == 0) set_status(a.status, KVC_DEV_TIMEOUT);
            break;
        }
        const unsigned ub = (unsigned)u / (unsigned)units_per_seq;
        const int b = (int)ub, e0 = (int)((unsigned)u - ub * (unsigned)units_per_seq) * kRingE;
        const int ne = min(kRingE, half - e0);
        const bool here = ei < ne;  // this team has an entry in the unit
        const int i = e0 + ei;
        // the sequence's length is first needed for the stores of pass 2: its
        // load and the indexer key's are in flight during pass 1
        const int base = a.n_entries[b];
        uint4 ik[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        const uint4* isrc =
            reinterpret_cast<const uint4*>(a.idx_k_new + ((long long)b * half + i) * di);
        if (here) {
#pragma unroll
            for (int r = 0; r < 2; ++r)
                if (l + 8 * r < (di >> 4)) ik[r] = __ldcs(isrc + l + 8 * r);
        }
        const T* k0s = reinterpret_cast<const T*>(rsm + (size_t)st * stage_bytes) +
                       (size_t)ei * 2 * D;
        const T* k1s = k0s + D;
        const int jn = here ? (nchunk - l + 7) / 8 : 0;  // chunks of this lane

        // pass 1: gate logit difference, fixed order (lane l: chunks l, l+8, ...)
        float acc = 0.f;
#pragma unroll 3
        for (int j = 0; j < MAXJ; ++j) {
            const int c = l + 8 * j;
            if (j < jn) {
                Chunk<T> x0, x1;
                x0.load_shared(k0s + 8 * c);
                x1.load_shared(k1s + 8 * c);
                float g[8];
                const float4 ga = reinterpret_cast<const float4*>(gate_s + 8 * c)[0];
                const float4 gb = reinterpret_cast<const float4*>(gate_s + 8 * c)[1];
                g[0] = ga.x; g[1] = ga.y; g[2] = ga.z; g[3] = ga.w;
                g[4] = gb.x; g[5] = gb.y; g[6] = gb.z; g[7] = gb.w;
                acc = gate_chunk(acc, x0, x1, g);
            }
        }
        uint64_t W0, W1;
        gate_weights(acc, W0, W1);
        const bool seq_ok = base >= 0 && base + half <= a.capacity;
        if (!seq_ok && e0 == 0 && wi == 0 && lane == 0) set_status(a.status, KVC_DEV_CAPACITY);
        const bool valid = seq_ok && here;
        const long long pos = (long long)base + i;
        uint8_t* rec = a.records + ((long long)b * a.capacity + pos) * sh.rb;

        // pass 2: entry values, group maxima, codes (stored by valid teams)
#pragma unroll 2
        for (int j = 0; j < MAXJ; ++j) {
            const int c = l + 8 * j;
            const bool active = valid && j < jn;
            Chunk<T> x0, x1;
            if (j < jn) {
                x0.load_shared(k0s + 8 * c);
                x1.load_shared(k1s + 8 * c);
            } else {
                x0.zero();
                x1.zero();
            }
            quantise_chunk<T, LPG>(x0, x1, W0, W1, active, c, ue4m3, tab, rec,
                                   tail, bad);
        }
        __syncwarp();
        if (lane == 0) ring_arrive(tc::smem_u32(&empty[st]));  // the stage is read
        if (valid) {
            for (int t = l * 4; t < tail_len; t += 32)
                *reinterpret_cast<uint32_t*>(rec + sh.code_bytes + t) =
                    *reinterpret_cast<const uint32_t*>(tail + t);
            uint4* dst =
                reinterpret_cast<uint4*>(a.idx_k + ((long long)b * a.capacity + pos) * di);
#pragma unroll
            for (int r = 0; r < 2; ++r)
                if (l + 8 * r < (di >> 4)) dst[l + 8 * r] = ik[r];
        }
        __syncwarp();  // the tail is read before the next unit writes it
        f += kRingGroups;
        if (f >= nfull) f -= nfull, ++rf;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, KVC_DEV_NONFINITE);
}

// Small appends (decode: one pair per sequence): one warp per entry so the
// work of a few dozen entries spreads over many SMs.  The whole warp first
// stages the token pair and the gate in shared memory (one round trip to
// HBM); lanes 0-7 then form the gate team in exactly the order above (lane l
// sums chunks l, l+8, ... then the xor tree over 4, 2, 1 inside the team), and
// all 32 lanes quantise from registers, lane l owning chunks l, l+32, l+64.
// Same arithmetic, same bits as pack_kernel.  With one pair per sequence the
// warp also commits the sequence's new length (no other warp touches it).
constexpr int kSmallWarps = 4;

template <typename T>
__host__ __device__ constexpr size_t small_stage_bytes(int D) {
    return (size_t)D * (2 * sizeof(T) + sizeof(float));  // k0, k1, gate
}

template <typename T, int MAXJ>
__global__ void __launch_bounds__(kSmallWarps * 32)
pack_small_kernel(PackArgs a, Shape sh, int ue4m3, int di) {
    extern __shared__ __align__(16) unsigned char stage_smem[];
    __shared__ __align__(16) uint8_t tail_smem[kSmallWarps][kTailBytes];
    pdl_trigger();  // a short kernel: the next one may be scheduled at once
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long e = (long long)blockIdx.x * kSmallWarps + wid;
    const int half = a.n_new >> 1;
    if (e >= (long long)a.batch * half) return;  // whole warp
    const int b = (int)(e / half), i = (int)(e % half);
    const int D = sh.D, nchunk = D >> 3;
    const T* k0p = static_cast<const T*>(a.tokens) + ((long long)b * a.n_new + 2 * i) * D;
    const T* k1p = k0p + D;
    T* s0 = reinterpret_cast<T*>(stage_smem + wid * small_stage_bytes<T>(D));
    T* s1 = s0 + D;
    float* sg = reinterpret_cast<float*>(s1 + D);

    // The entry is formed before waiting for the previous kernel: the token
    // pair, gate and indexer row are inputs no library kernel writes; only
    // the sequence's length and the cache stores wait.  Every load in flight
    // at once.
    uint4 ik = make_uint4(0, 0, 0, 0);
    if (lane < (di >> 4))
        ik = __ldcs(reinterpret_cast<const uint4*>(a.idx_k_new + ((long long)b * half + i) * di) +
                    lane);
    Chunk<T> x0[MAXJ], x1[MAXJ];
    float4 g0[MAXJ], g1[MAXJ];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) {
            x0[j].load(k0p + 8 * c);
            x1[j].load(k1p + 8 * c);
            g0[j] = __ldg(reinterpret_cast<const float4*>(a.gate + 8 * c));
            g1[j] = __ldg(reinterpret_cast<const float4*>(a.gate + 8 * c) + 1);
        } else {
            x0[j].zero();
            x1[j].zero();
        }
    }
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) {
            x0[j].store_shared(s0 + 8 * c);
            x1[j].store_shared(s1 + 8 * c);
            reinterpret_cast<float4*>(sg + 8 * c)[0] = g0[j];
            reinterpret_cast<float4*>(sg + 8 * c)[1] = g1[j];
        }
    }
    __syncwarp();

    float acc = 0.f;
    if (lane < 8) {
        for (int c = lane; c < nchunk; c += 8) {
            Chunk<T> y0, y1;
            y0.load_shared(s0 + 8 * c);
            y1.load_shared(s1 + 8 * c);
#pragma unroll
            for (int t = 0; t < 8; ++t)
                acc = __fmaf_rn(sg[8 * c + t], __fsub_rn(y0.get(t), y1.get(t)), acc);
        }
    }
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 4));
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 2));
    acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, 1));
    const float delta = __shfl_sync(0xffffffffu, acc, 0);
    const float w0 = __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_cody_waite(-delta)));
    const float w1 = __fsub_rn(1.0f, w0);

    uint8_t* tail = tail_smem[wid];
    const int tail_len = sh.rb - sh.code_bytes;
    for (int t = lane * 4; t < tail_len; t += 128) *reinterpret_cast<uint32_t*>(tail + t) = 0u;
    __syncwarp();

    bool bad = false;
    const int lpg = sh.lpg;
    uint32_t code[MAXJ];  // the 8 codes of chunk lane + 32 j
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        const bool active = c < nchunk;
        float x[8];
        float m = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float v = __fmaf_rn(w0, x0[j].get(t), __fmul_rn(w1, x1[j].get(t)));
            if (!isfinite(v)) {
                if (active) bad = true;
                v = 0.f;
            }
            x[t] = v;
            m = fmaxf(m, fabsf(v));
        }
        for (int o = 1; o < lpg; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        code[j] = 0u;
        if (!active) continue;
        float s = __fdiv_rn(m, 6.0f);
        uint32_t sbyte = 0;
        if (ue4m3) {
            sbyte = e4m3_from_f32(s);
            s = e4m3_to_f32(sbyte);
        }
        code[j] = s > 0.f ? e2m1x8_quotient(x, s) : 0u;
        if (c % lpg == 0) {
            const int gi = c / lpg;
            if (ue4m3)
                tail[gi] = (uint8_t)sbyte;
            else
                *reinterpret_cast<float*>(tail + 4 * gi) = s;
        }
    }
    __syncwarp();

    pdl_wait();  // the previous kernel is done: the length and the cache
    const int base = a.n_entries[b];
    if (base < 0 || base + half > a.capacity) {
        if (i == 0 && lane == 0) set_status(a.status, KVC_DEV_CAPACITY);
        return;
    }
    const long long pos = (long long)base + i;
    uint8_t* rec = a.records + ((long long)b * a.capacity + pos) * sh.rb;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) *reinterpret_cast<uint32_t*>(rec + 4 * c) = code[j];
    }
    for (int t = lane * 4; t < tail_len; t += 128)
        *reinterpret_cast<uint32_t*>(rec + sh.code_bytes + t) =
            *reinterpret_cast<const uint32_t*>(tail + t);
    if (lane < (di >> 4))
        *(reinterpret_cast<uint4*>(a.idx_k + ((long long)b * a.capacity + pos) * di) + lane) = ik;
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, KVC_DEV_NONFINITE);
    if (half == 1 && lane == 0) a.n_entries[b] = base + 1;
}

// 4:1 compression (the ratio 4 of [B] 4.3): four consecutive tokens form one
// entry, weighted by the softmax of their four gate logits.  One warp per
// entry, as for the decode append: the warp stages the four tokens and the
// gate in shared memory (one round trip), lanes 0-7 form the four logits
// each in the order of the pair's gate (lane l sums chunks l, l+8, ... then
// the xor tree over 4, 2, 1), every lane takes the weights
// (w_t = exp(logit_t - max) / S, S summed left to right) and quantises its
// chunks from registers: entry = fma(w0, k0, fma(w1, k1, fma(w2, k2, w3 k3))).
// The entry is formed before the wait for the previous kernel, as in the
// decode append; one entry per sequence also commits the new length.
template <typename T>
__host__ __device__ constexpr size_t group4_stage_bytes(int D) {
    return (size_t)D * (4 * sizeof(T) + sizeof(float));  // k0..k3, gate
}

template <typename T, int MAXJ>
__global__ void __launch_bounds__(kSmallWarps * 32)
pack_group4_kernel(PackArgs a, Shape sh, int ue4m3, int di) {
    extern __shared__ __align__(16) unsigned char stage_smem[];
    __shared__ __align__(16) uint8_t tail_smem[kSmallWarps][kTailBytes];
    pdl_trigger();  // a short kernel: the next one may be scheduled at once
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long e = (long long)blockIdx.x * kSmallWarps + wid;
    const int per = a.n_new >> 2;
    if (e >= (long long)a.batch * per) return;  // whole warp
    const int b = (int)(e / per), i = (int)(e % per);
    const int D = sh.D, nchunk = D >> 3;
    const T* kp = static_cast<const T*>(a.tokens) + ((long long)b * a.n_new + 4 * i) * D;
    T* st = reinterpret_cast<T*>(stage_smem + wid * group4_stage_bytes<T>(D));  // [4][D]
    float* sg = reinterpret_cast<float*>(st + 4 * D);

    uint4 ik = make_uint4(0, 0, 0, 0);
    if (lane < (di >> 4))
        ik = __ldcs(reinterpret_cast<const uint4*>(a.idx_k_new + ((long long)b * per + i) * di) +
                    lane);
    Chunk<T> x[4][MAXJ];
    float4 g0[MAXJ], g1[MAXJ];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) {
#pragma unroll
            for (int t = 0; t < 4; ++t) x[t][j].load(kp + (long long)t * D + 8 * c);
            g0[j] = __ldg(reinterpret_cast<const float4*>(a.gate + 8 * c));
            g1[j] = __ldg(reinterpret_cast<const float4*>(a.gate + 8 * c) + 1);
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) x[t][j].zero();
        }
    }
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) {
#pragma unroll
            for (int t = 0; t < 4; ++t) x[t][j].store_shared(st + t * D + 8 * c);
            reinterpret_cast<float4*>(sg + 8 * c)[0] = g0[j];
            reinterpret_cast<float4*>(sg + 8 * c)[1] = g1[j];
        }
    }
    __syncwarp();

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (lane < 8) {
        for (int c = lane; c < nchunk; c += 8) {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                Chunk<T> y;
                y.load_shared(st + t * D + 8 * c);
#pragma unroll
                for (int u = 0; u < 8; ++u) acc[t] = __fmaf_rn(sg[8 * c + u], y.get(u), acc[t]);
            }
        }
    }
    float lg[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float v = acc[t];
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 4));
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 2));
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 1));
        lg[t] = __shfl_sync(0xffffffffu, v, 0);
    }
    const float mx = fmaxf(fmaxf(lg[0], lg[1]), fmaxf(lg[2], lg[3]));
    float ex[4], w[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) ex[t] = exp_cody_waite(__fsub_rn(lg[t], mx));
    const float sum = __fadd_rn(__fadd_rn(__fadd_rn(ex[0], ex[1]), ex[2]), ex[3]);
#pragma unroll
    for (int t = 0; t < 4; ++t) w[t] = __fdiv_rn(ex[t], sum);

    uint8_t* tail = tail_smem[wid];
    const int tail_len = sh.rb - sh.code_bytes;
    for (int t = lane * 4; t < tail_len; t += 128) *reinterpret_cast<uint32_t*>(tail + t) = 0u;
    __syncwarp();

    bool bad = false;
    const int lpg = sh.lpg;
    uint32_t code[MAXJ];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        const bool active = c < nchunk;
        float xv[8];
        float m = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float v = __fmaf_rn(w[0], x[0][j].get(u),
                                __fmaf_rn(w[1], x[1][j].get(u),
                                          __fmaf_rn(w[2], x[2][j].get(u),
                                                    __fmul_rn(w[3], x[3][j].get(u)))));
            if (!isfinite(v)) {
                if (active) bad = true;
                v = 0.f;
            }
            xv[u] = v;
            m = fmaxf(m, fabsf(v));
        }
        for (int o = 1; o < lpg; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        code[j] = 0u;
        if (!active) continue;
        float sc = __fdiv_rn(m, 6.0f);
        uint32_t sbyte = 0;
        if (ue4m3) {
            sbyte = e4m3_from_f32(sc);
            sc = e4m3_to_f32(sbyte);
        }
        code[j] = sc > 0.f ? e2m1x8_quotient(xv, sc) : 0u;
        if (c % lpg == 0) {
            const int gi = c / lpg;
            if (ue4m3)
                tail[gi] = (uint8_t)sbyte;
            else
                *reinterpret_cast<float*>(tail + 4 * gi) = sc;
        }
    }
    __syncwarp();

    pdl_wait();  // the previous kernel is done: the length and the cache
    const int base = a.n_entries[b];
    if (base < 0 || base + per > a.capacity) {
        if (i == 0 && lane == 0) set_status(a.status, KVC_DEV_CAPACITY);
        return;
    }
    const long long pos = (long long)base + i;
    uint8_t* rec = a.records + ((long long)b * a.capacity + pos) * sh.rb;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) *reinterpret_cast<uint32_t*>(rec + 4 * c) = code[j];
    }
    for (int t = lane * 4; t < tail_len; t += 128)
        *reinterpret_cast<uint32_t*>(rec + sh.code_bytes + t) =
            *reinterpret_cast<const uint32_t*>(tail + t);
    if (lane < (di >> 4))
        *(reinterpret_cast<uint4*>(a.idx_k + ((long long)b * a.capacity + pos) * di) + lane) = ik;
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, KVC_DEV_NONFINITE);
    if (per == 1 && lane == 0) a.n_entries[b] = base + 1;
}

__global__ void pack_commit_kernel(int32_t* n_entries, int batch, int half, int capacity) {
    pdl_wait();
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
        const int n = n_entries[b];
        if (n >= 0 && n + half <= capacity) n_entries[b] = n + half;
    }
}

template <typename T, int MAXJ>
cudaError_t launch_small(unsigned grid, size_t smem, cudaStream_t s, const PackArgs& a,
                         const Shape& sh, int ue4m3, int di) {
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            pack_small_kernel<T, MAXJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(pack_small_kernel<T, MAXJ>, grid, kSmallWarps * 32, smem, s, a, sh, ue4m3,
                      di);
}

template <typename T, int MAXJ>
cudaError_t launch_group4(unsigned grid, size_t smem, cudaStream_t s, const PackArgs& a,
                          const Shape& sh, int ue4m3, int di) {
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            pack_group4_kernel<T, MAXJ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(pack_group4_kernel<T, MAXJ>, grid, kSmallWarps * 32, smem, s, a, sh, ue4m3,
                      di);
}

template <typename T, int MAXJ, int LPG>
cudaError_t launch_stream(dim3 grid, cudaStream_t s, const PackArgs& a, const Shape& sh,
                          int ue4m3, int di) {
    const int tail_stride = ((sh.rb - sh.code_bytes) + 15) / 16 * 16;
    return launch_pdl(pack_stream_kernel<T, MAXJ, LPG>, grid, kThreads,
                      (size_t)kTeams * tail_stride, s, a, sh, ue4m3, di, tail_stride);
}
template <typename T, int MAXJ>
cudaError_t launch_stream_j(dim3 grid, cudaStream_t s, const PackArgs& a, const Shape& sh,
                            int ue4m3, int di) {
    switch (sh.lpg) {
        case 1: return launch_stream<T, MAXJ, 1>(grid, s, a, sh, ue4m3, di);
        case 2: return launch_stream<T, MAXJ, 2>(grid, s, a, sh, ue4m3, di);
        case 4: return launch_stream<T, MAXJ, 4>(grid, s, a, sh, ue4m3, di);
        default: return launch_stream<T, MAXJ, 8>(grid, s, a, sh, ue4m3, di);
    }
}

// The ring kernel: one CTA per SM (fewer for short appends), as many stages
// as fit beside the gate and the team tails (at least one more than the
// consumer groups, else the streaming kernel runs).
template <int MAXJ, int LPG>
cudaError_t launch_ring(cudaStream_t s, const PackArgs& a, const Shape& sh, int ue4m3, int di,
                        int stages, uint32_t stage_bytes, long long n_units, int sms,
                        size_t smem) {
    const cudaError_t e = cudaFuncSetAttribute(
        pack_ring_kernel<MAXJ, LPG>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int tail_stride = ((sh.rb - sh.code_bytes) + 15) / 16 * 16;
    const unsigned grid = (unsigned)(n_units < sms ? n_units : sms);
    return launch_pdl(pack_ring_kernel<MAXJ, LPG>, grid, kRingThreads, smem, s, a, sh, ue4m3, di,
                      tail_stride, stages, stage_bytes, n_units, device_wait_limit_ns());
}

// Ring plan for a bf16 append: stage count and dynamic shared memory, or
// stages = 0 when the ring does not apply.
struct RingPlan {
    int stages = 0, sms = 0;
    uint32_t stage_bytes = 0;
    size_t smem = 0;
};
inline RingPlan ring_plan(const Shape& sh, const PackArgs& a, int di) {
    RingPlan p;
    const int D = sh.D;
    if (D % 8 != 0 || D > 576 || D <= 128 || sh.lpg > 8 || di > 256 || di % 16 != 0) return p;
    if (reinterpret_cast<uintptr_t>(a.tokens) % 16 != 0) return p;
    int dev = 0, optin = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return p;
    const int tail_stride = ((sh.rb - sh.code_bytes) + 15) / 16 * 16;
    const size_t fixed = (size_t)D * 4 + (size_t)kRingConsumerWarps * 4 * tail_stride;
    const uint32_t sb = (uint32_t)(kRingE * 2 * D * 2);
    const long long room = (long long)optin - 4096 - (long long)fixed;  // static smem margin
    int st = room > 0 ? (int)(room / sb) : 0;
    if (st > kRingMaxStages) st = kRingMaxStages;
    if (st < kRingGroups + 1) return p;
    p.stages = st;
    p.sms = sms;
    p.stage_bytes = sb;
    p.smem = fixed + (size_t)st * sb;
    return p;
}

template <int MAXJ>
cudaError_t launch_ring_j(cudaStream_t s, const PackArgs& a, const Shape& sh, int ue4m3, int di,
                          const RingPlan& p, long long n_units) {
    switch (sh.lpg) {
        case 1: return launch_ring<MAXJ, 1>(s, a, sh, ue4m3, di, p.stages, p.stage_bytes, n_units,
                                            p.sms, p.smem);
        case 2: return launch_ring<MAXJ, 2>(s, a, sh, ue4m3, di, p.stages, p.stage_bytes, n_units,
                                            p.sms, p.smem);
        case 4: return launch_ring<MAXJ, 4>(s, a, sh, ue4m3, di, p.stages, p.stage_bytes, n_units,
                                            p.sms, p.smem);
        default: return launch_ring<MAXJ, 8>(s, a, sh, ue4m3, di, p.stages, p.stage_bytes,
                                             n_units, p.sms, p.smem);
    }
}

// 4:1 appends: a warp per entry at every size
template <typename T>
cudaError_t launch_pack4_t(const Shape& sh, const PackArgs& a, int ue4m3, int di,
                           cudaStream_t s) {
    const long long entries = (long long)a.batch * (a.n_new / 4);
    const unsigned grid = (unsigned)((entries + kSmallWarps - 1) / kSmallWarps);
    const int maxj = (sh.D / 8 + 31) / 32;
    const size_t smem = kSmallWarps * group4_stage_bytes<T>(sh.D);
    trace_before("pack", s);
    cudaError_t err;
    if (maxj <= 1)
        err = launch_group4<T, 1>(grid, smem, s, a, sh, ue4m3, di);
    else if (maxj <= 2)
        err = launch_group4<T, 2>(grid, smem, s, a, sh, ue4m3, di);
    else if (maxj <= 3)
        err = launch_group4<T, 3>(grid, smem, s, a, sh, ue4m3, di);
    else
        err = launch_group4<T, 4>(grid, smem, s, a, sh, ue4m3, di);
    trace_after(s);
    return err;
}

template <typename T>
cudaError_t launch_pack_t(const Shape& sh, const PackArgs& a, int ue4m3, int di,
                          cudaStream_t s) {
    const long long entries = (long long)a.batch * (a.n_new / 2);
    cudaError_t err;
    if (entries <= 4096) {  // latency-bound append: a warp per entry
        const unsigned grid = (unsigned)((entries + kSmallWarps - 1) / kSmallWarps);
        const int maxj = (sh.D / 8 + 31) / 32;
        const size_t smem = kSmallWarps * small_stage_bytes<T>(sh.D);
        trace_before("pack", s);
        if (maxj <= 1)
            err = launch_small<T, 1>(grid, smem, s, a, sh, ue4m3, di);
        else if (maxj <= 2)
            err = launch_small<T, 2>(grid, smem, s, a, sh, ue4m3, di);
        else if (maxj <= 3)
            err = launch_small<T, 3>(grid, smem, s, a, sh, ue4m3, di);
        else
            err = launch_small<T, 4>(grid, smem, s, a, sh, ue4m3, di);
        trace_after(s);
        return err;
    }
    const unsigned grid = (unsigned)((entries + kTeams - 1) / kTeams);
    const int maxj = (sh.D / 8 + 7) / 8;
    trace_before("pack", s);
    if (sh.lpg <= 8 && sizeof(T) == 2) {  // bf16 tokens: the ring kernel where it fits
        const RingPlan p = ring_plan(sh, a, di);
        const int half = a.n_new / 2;
        const long long n_units = (long long)a.batch * ((half + kRingE - 1) / kRingE);
        if (p.stages > 0 && n_units < (1ll << 31) - p.sms) {  // unit indices fit 32 bits
            err = maxj <= 4 ? launch_ring_j<4>(s, a, sh, ue4m3, di, p, n_units)
                            : launch_ring_j<9>(s, a, sh, ue4m3, di, p, n_units);
            trace_after(s);
            return err;
        }
    }
    if (sh.lpg <= 8) {  // groups within one chunk step: the streaming kernel
        const int half = a.n_new / 2;
        const dim3 g2((unsigned)((half + kTeams - 1) / kTeams), (unsigned)a.batch);
        if (maxj <= 2)
            err = launch_stream_j<T, 2>(g2, s, a, sh, ue4m3, di);
        else if (maxj <= 4)
            err = launch_stream_j<T, 4>(g2, s, a, sh, ue4m3, di);
        else if (maxj <= 9)
            err = launch_stream_j<T, 9>(g2, s, a, sh, ue4m3, di);
        else
            err = launch_stream_j<T, 16>(g2, s, a, sh, ue4m3, di);
        trace_after(s);
        return err;
    }
    if (maxj <= 2)
        err = launch_pdl(pack_kernel<T, 2>, grid, kThreads, 0, s, a, sh, ue4m3, di);
    else if (maxj <= 4)
        err = launch_pdl(pack_kernel<T, 4>, grid, kThreads, 0, s, a, sh, ue4m3, di);
    else if (maxj <= 9)
        err = launch_pdl(pack_kernel<T, 9>, grid, kThreads, 0, s, a, sh, ue4m3, di);
    else
        err = launch_pdl(pack_kernel<T, 16>, grid, kThreads, 0, s, a, sh, ue4m3, di);
    trace_after(s);
    return err;
}

// ---- FP8 window rows: a warp per row.  s = absmax / 448 over the finite
// elements; codes = E4M3 of x / s, by the same bracket of two reciprocal
// products as the E2M1 codes (rounding to E4M3 is monotone too), with an
// exact division where the brackets disagree.
constexpr int kWinWarps = 4;
template <typename T, int MAXC>
__global__ void __launch_bounds__(kWinWarps * 32)
window_fp8_kernel(const T* __restrict__ rows, long long n, int D, uint8_t* __restrict__ codes,
                  float* __restrict__ scales, uint32_t* status) {
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * kWinWarps + (threadIdx.x >> 5);
    if (r >= n) return;
    const int nchunk = D >> 3;
    const T* src = rows + r * D;
    float x[MAXC][8];
    float amax = 0.f;
    bool bad = false;
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
        const int c = lane + 32 * j;
        Chunk<T> v;
        if (c < nchunk) v.load_cached(src + 8 * c); else v.zero();
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float e = v.get(t);
            if (!isfinite(e)) {
                if (c < nchunk) bad = true;
                e = 0.f;
            }
            x[j][t] = e;
            amax = fmaxf(amax, fabsf(e));
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = __fdiv_rn(amax, 448.0f);
    const float rc = __frcp_rn(sc);
    const bool fast = sc > 0.f && rc < 3.0e38f;
    const float rl = __fmul_rn(rc, 1.0f - 0x1p-20f), rh = __fmul_rn(rc, 1.0f + 0x1p-20f);
#pragma unroll
    for (int j = 0; j < MAXC; ++j) {
        const int c = lane + 32 * j;
        if (c >= nchunk) continue;
        uint32_t w[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float* e = x[j] + 4 * h;
            uint32_t code = 0;
            if (sc > 0.f) {
                bool done = false;
                if (fast) {
                    const uint32_t cl = e4m3x4_from_f32(__fmul_rn(e[0], rl), __fmul_rn(e[1], rl),
                                                        __fmul_rn(e[2], rl), __fmul_rn(e[3], rl));
                    const uint32_t ch = e4m3x4_from_f32(__fmul_rn(e[0], rh), __fmul_rn(e[1], rh),
                                                        __fmul_rn(e[2], rh), __fmul_rn(e[3], rh));
                    if (cl == ch) {
                        code = cl;
                        done = true;
                    }
                }
                if (!done)
                    code = e4m3x4_from_f32(__fdiv_rn(e[0], sc), __fdiv_rn(e[1], sc),
                                           __fdiv_rn(e[2], sc), __fdiv_rn(e[3], sc));
            }
            w[h] = code;
        }
        *reinterpret_cast<uint2*>(codes + r * D + 8 * c) = make_uint2(w[0], w[1]);
    }
    if (lane == 0) scales[r] = sc;
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(status, KVC_DEV_NONFINITE);
}

template <typename T>
cudaError_t launch_window_t(const void* rows, long long n, int D, uint8_t* codes, float* scales,
                            uint32_t* status, cudaStream_t s) {
    const unsigned grid = (unsigned)((n + kWinWarps - 1) / kWinWarps);
    const int maxc = (D / 8 + 31) / 32;
    const T* r = static_cast<const T*>(rows);
    trace_before("window_fp8", s);
    cudaError_t err;
    if (maxc <= 1)
        err = launch_pdl(window_fp8_kernel<T, 1>, grid, kWinWarps * 32, 0, s, r, n, D, codes, scales, status);
    else if (maxc <= 2)
        err = launch_pdl(window_fp8_kernel<T, 2>, grid, kWinWarps * 32, 0, s, r, n, D, codes, scales, status);
    else if (maxc <= 3)
        err = launch_pdl(window_fp8_kernel<T, 3>, grid, kWinWarps * 32, 0, s, r, n, D, codes, scales, status);
    else
        err = launch_pdl(window_fp8_kernel<T, 4>, grid, kWinWarps * 32, 0, s, r, n, D, codes, scales, status);
    trace_after(s);
    return err;
}

__device__ __forceinline__ float key_f32(float v) { return v; }
__device__ __forceinline__ float key_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// FP4 indexer keys (idx_fmt = 1): the new entries' keys quantised like a
// record of idx_dim channels with groups of 16 and UE4M3 scales (absmax / 6,
// round to nearest even; the same scale and quotient steps as the records).
// A thread per group of 16 channels; the rows are written at the entries'
// positions before the pack kernel that follows on the stream advances the
// lengths.  Row: idx_dim/2 code bytes (channel 2c in the low nibble of byte
// c), then idx_dim/16 scale bytes.
template <typename T>
__global__ void __launch_bounds__(256)
idx_fp4_pack_kernel(const T* __restrict__ keys, int per, int batch, int di, int capacity,
                    const int32_t* __restrict__ n_entries, uint8_t* __restrict__ rows,
                    uint32_t* status) {
    pdl_trigger();  // a short kernel: the next one may be scheduled at once
    pdl_wait();
    const int ng = di / 16;
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= (long long)batch * per * ng) return;
    const int g = (int)(t % ng);
    const long long e = t / ng;
    const int b = (int)(e / per), i = (int)(e % per);
    const int base = n_entries[b];
    if (base < 0 || base + per > capacity) return;  // the pack kernel flags it
    const T* k = keys + ((long long)b * per + i) * di + 16 * g;
    float x[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) x[u] = key_f32(k[u]);
    bool bad = false;
    float m = 0.f;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
        if (!isfinite(x[u])) {
            bad = true;
            x[u] = 0.f;
        }
        m = fmaxf(m, fabsf(x[u]));
    }
    float sc = __fdiv_rn(m, 6.0f);
    const uint32_t sbyte = e4m3_from_f32(sc);
    sc = e4m3_to_f32(sbyte);
    const uint32_t c0 = sc > 0.f ? e2m1x8_quotient(x, sc) : 0u;
    const uint32_t c1 = sc > 0.f ? e2m1x8_quotient(x + 8, sc) : 0u;
    uint8_t* row = rows + ((long long)b * capacity + base + i) * (di / 2 + di / 16);
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // byte stores: a row need not be 4-byte aligned
        row[8 * g + u] = (uint8_t)(c0 >> (8 * u));
        row[8 * g + 4 + u] = (uint8_t)(c1 >> (8 * u));
    }
    row[di / 2 + g] = (uint8_t)sbyte;
    if (bad) set_status(status, KVC_DEV_NONFINITE);
}

}  // namespace

cudaError_t launch_pack(const kvc_config& c, const Shape& sh, const PackArgs& a,
                        cudaStream_t s) {
    const bool four = c.ratio == 4;
    const int half = a.n_new / (four ? 4 : 2);  // entries per sequence
    if (half == 0 || a.batch == 0) return cudaSuccess;
    const int ue = c.scale_fmt == KVC_SCALE_UE4M3;
    cudaError_t err;
    int di_copy = c.idx_dim;  // int8 keys are copied by the pack kernel itself
    if (c.idx_fmt == 1) {     // FP4 keys: quantised first, at the entries' positions
        di_copy = 0;
        const long long groups = (long long)a.batch * half * (c.idx_dim / 16);
        const unsigned grid = (unsigned)((groups + 255) / 256);
        trace_before("pack_idx", s);
        err = c.act_dtype == KVC_BF16
                  ? launch_pdl(idx_fp4_pack_kernel<__nv_bfloat16>, grid, 256, 0, s,
                               reinterpret_cast<const __nv_bfloat16*>(a.idx_k_new), half, a.batch,
                               c.idx_dim, a.capacity, a.n_entries,
                               reinterpret_cast<uint8_t*>(a.idx_k), a.status)
                  : launch_pdl(idx_fp4_pack_kernel<float>, grid, 256, 0, s,
                               reinterpret_cast<const float*>(a.idx_k_new), half, a.batch,
                               c.idx_dim, a.capacity, a.n_entries,
                               reinterpret_cast<uint8_t*>(a.idx_k), a.status);
        trace_after(s);
        if (err != cudaSuccess) return err;
    }
    if (four)
        err = c.act_dtype == KVC_BF16 ? launch_pack4_t<__nv_bfloat16>(sh, a, ue, di_copy, s)
                                      : launch_pack4_t<float>(sh, a, ue, di_copy, s);
    else
        err = c.act_dtype == KVC_BF16 ? launch_pack_t<__nv_bfloat16>(sh, a, ue, di_copy, s)
                                      : launch_pack_t<float>(sh, a, ue, di_copy, s);
    if (err != cudaSuccess) return err;
    // one entry per sequence: committed by the append kernel
    if (half == 1 && (four || a.batch <= 4096)) return cudaSuccess;
    trace_before("pack_commit", s);
    err = launch_pdl(pack_commit_kernel, (a.batch + 255) / 256, 256, 0, s, a.n_entries, a.batch,
                     half, a.capacity);
    trace_after(s);
    return err;
}

cudaError_t launch_window_fp8(const kvc_config& c, const Shape& sh, const void* rows, long long n,
                              uint8_t* codes, float* scales, uint32_t* status, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    return c.act_dtype == KVC_BF16
               ? launch_window_t<__nv_bfloat16>(rows, n, sh.D, codes, scales, status, s)
               : launch_window_t<float>(rows, n, sh.D, codes, scales, status, s);
}

}  // namespace kvc
