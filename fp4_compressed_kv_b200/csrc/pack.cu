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
// Design (B200): one warp per entry, a pure HBM stream.  Lane l owns the
// 8-channel chunks c = l, l+32, ...; each chunk of each token is one 16-byte
// (bf16) or two 16-byte (fp32) coalesced loads, and each chunk's eight codes
// leave as one 4-byte store, so a warp writes 128 contiguous bytes per step.
// The group maximum is a xor-shuffle over the G/8 lanes of a group.
//
// Bit-exactness: the gate logit difference is accumulated in fp64 in a fixed
// order -- lane l sums its chunks in increasing order with one fma per
// channel, then a xor butterfly over offsets 16..1 -- and the pair weight
// w0 = 1 / (1 + exp(-delta)) uses the exp below (Cody-Waite reduction with a
// 32-bit head of ln 2, degree-13 Taylor polynomial in Horner form, exact
// power-of-two scaling), so every implementation of this order produces the
// same fp32 entry and therefore the same codes.
#include "kvc_internal.cuh"

namespace kvc {
namespace {

constexpr double kLn2Hi = 0x1.62e42feep-1;
constexpr double kLn2Lo = 0x1.a39ef35793c76p-33;
constexpr double kInvLn2 = 0x1.71547652b82fep+0;

__device__ __forceinline__ double exp_cody_waite(double x) {
    if (x != x) return x;
    if (x > 709.0) return __longlong_as_double(0x7ff0000000000000LL);
    if (x < -708.0) return 0.0;
    const double n = rint(__dmul_rn(x, kInvLn2));
    double r = __fma_rn(-n, kLn2Hi, x);
    r = __fma_rn(-n, kLn2Lo, r);
    // 1/k! for k = 13 .. 0
    double p = 0x1.6124613a86d09p-33;
    p = __fma_rn(p, r, 0x1.1eed8eff8d898p-29);
    p = __fma_rn(p, r, 0x1.ae64567f544e4p-26);
    p = __fma_rn(p, r, 0x1.27e4fb7789f5cp-22);
    p = __fma_rn(p, r, 0x1.71de3a556c734p-19);
    p = __fma_rn(p, r, 0x1.a01a01a01a01ap-16);
    p = __fma_rn(p, r, 0x1.a01a01a01a01ap-13);
    p = __fma_rn(p, r, 0x1.6c16c16c16c17p-10);
    p = __fma_rn(p, r, 0x1.1111111111111p-7);
    p = __fma_rn(p, r, 0x1.5555555555555p-5);
    p = __fma_rn(p, r, 0x1.5555555555555p-3);
    p = __fma_rn(p, r, 0x1.0p-1);
    p = __fma_rn(p, r, 1.0);
    p = __fma_rn(p, r, 1.0);
    const long long bits = ((long long)n + 1023) << 52;
    return __dmul_rn(p, __longlong_as_double(bits));
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float v[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

__device__ __forceinline__ void load8(const float* p, float v[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8_gate(const float* p, float v[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

constexpr int kWarps = 8;
constexpr int kTailBytes = 528;  // >= 1024/8 groups x 4 bytes + padding

// MAXJ: chunks per lane (D <= 256 * MAXJ).
template <typename T, int MAXJ>
__global__ void __launch_bounds__(kWarps * 32)
pack_kernel(PackArgs a, Shape sh, int ue4m3, int di) {
    __shared__ __align__(16) uint8_t tail_smem[kWarps][kTailBytes];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long e = (long long)blockIdx.x * kWarps + wid;
    const int half = a.n_new >> 1;
    if (e >= (long long)a.batch * half) return;
    const int b = (int)(e / half), i = (int)(e % half);
    const int base = a.n_entries[b];
    if (base < 0 || base + half > a.capacity) {
        if (lane == 0 && i == 0) set_status(a.status, KVC_DEV_CAPACITY);
        return;
    }
    const long long pos = (long long)base + i;
    const int D = sh.D, nchunk = D >> 3;
    const T* k0p = static_cast<const T*>(a.tokens) + ((long long)b * a.n_new + 2 * i) * D;
    const T* k1p = k0p + D;

    float k0[MAXJ][8], k1[MAXJ][8];
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) {
            load8(k0p + 8 * c, k0[j]);
            load8(k1p + 8 * c, k1[j]);
        } else {
#pragma unroll
            for (int t = 0; t < 8; ++t) k0[j][t] = k1[j][t] = 0.f;
        }
    }

    // gate logit difference, fixed order
    double acc = 0.0;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        if (c < nchunk) {
            float g[8];
            load8_gate(a.gate + 8 * c, g);
#pragma unroll
            for (int t = 0; t < 8; ++t)
                acc = __fma_rn((double)g[t], __dsub_rn((double)k0[j][t], (double)k1[j][t]), acc);
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        acc = __dadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
    const double w0 = __ddiv_rn(1.0, __dadd_rn(1.0, exp_cody_waite(-acc)));
    const double w1 = __dsub_rn(1.0, w0);

    uint8_t* rec = a.records + ((long long)b * a.capacity + pos) * sh.rb;
    uint8_t* tail = tail_smem[wid];
    const int tail_len = sh.rb - sh.code_bytes;  // multiple of 4
    for (int t = lane * 4; t < tail_len; t += 128) *reinterpret_cast<uint32_t*>(tail + t) = 0u;
    __syncwarp();

    bool bad = false;
#pragma unroll
    for (int j = 0; j < MAXJ; ++j) {
        const int c = lane + 32 * j;
        const bool active = c < nchunk;
        float x[8];
        float amax = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            float v = __double2float_rn(
                __fma_rn(w0, (double)k0[j][t], __dmul_rn(w1, (double)k1[j][t])));
            if (!isfinite(v)) {
                if (active) bad = true;
                v = 0.f;
            }
            x[t] = v;
            amax = fmaxf(amax, fabsf(v));
        }
        for (int o = 1; o < sh.lpg; o <<= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        float s = __fdiv_rn(amax, 6.0f);
        uint32_t sbyte = 0;
        if (ue4m3) {
            sbyte = e4m3_from_f32(s);
            s = e4m3_to_f32(sbyte);
        }
        if (active) {
            float v[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const float q = s > 0.f ? __fdiv_rn(x[t], s) : 0.f;
                v[t] = fminf(fmaxf(q, -6.f), 6.f);
            }
            *reinterpret_cast<uint32_t*>(rec + 4 * c) = e2m1x8_from_f32(v);
            if (c % sh.lpg == 0) {
                const int gi = c / sh.lpg;
                if (ue4m3)
                    tail[gi] = (uint8_t)sbyte;
                else
                    *reinterpret_cast<float*>(tail + 4 * gi) = s;
            }
        }
    }
    __syncwarp();
    for (int t = lane * 4; t < tail_len; t += 128)
        *reinterpret_cast<uint32_t*>(rec + sh.code_bytes + t) =
            *reinterpret_cast<const uint32_t*>(tail + t);

    // indexer key append: Di bytes as 16-byte pieces, one per lane
    if (lane < (di >> 4)) {
        const uint4 v = __ldcs(
            reinterpret_cast<const uint4*>(a.idx_k_new + ((long long)b * half + i) * di) + lane);
        *(reinterpret_cast<uint4*>(a.idx_k + ((long long)b * a.capacity + pos) * di) + lane) = v;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_status(a.status, KVC_DEV_NONFINITE);
}

__global__ void pack_commit_kernel(int32_t* n_entries, int batch, int half, int capacity) {
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
        const int n = n_entries[b];
        if (n >= 0 && n + half <= capacity) n_entries[b] = n + half;
    }
}

template <typename T>
cudaError_t launch_pack_t(const Shape& sh, const PackArgs& a, int ue4m3, int di,
                          cudaStream_t s) {
    const long long entries = (long long)a.batch * (a.n_new / 2);
    const unsigned grid = (unsigned)((entries + kWarps - 1) / kWarps);
    const int maxj = (sh.D / 8 + 31) / 32;
    trace_before("pack", s);
    switch (maxj) {
        case 1: pack_kernel<T, 1><<<grid, kWarps * 32, 0, s>>>(a, sh, ue4m3, di); break;
        case 2: pack_kernel<T, 2><<<grid, kWarps * 32, 0, s>>>(a, sh, ue4m3, di); break;
        case 3: pack_kernel<T, 3><<<grid, kWarps * 32, 0, s>>>(a, sh, ue4m3, di); break;
        default: pack_kernel<T, 4><<<grid, kWarps * 32, 0, s>>>(a, sh, ue4m3, di); break;
    }
    trace_after(s);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack(const kvc_config& c, const Shape& sh, const PackArgs& a,
                        cudaStream_t s) {
    const int half = a.n_new / 2;
    if (half == 0 || a.batch == 0) return cudaSuccess;
    const int ue = c.scale_fmt == KVC_SCALE_UE4M3;
    cudaError_t err = c.act_dtype == KVC_BF16
                          ? launch_pack_t<__nv_bfloat16>(sh, a, ue, c.idx_dim, s)
                          : launch_pack_t<float>(sh, a, ue, c.idx_dim, s);
    if (err != cudaSuccess) return err;
    trace_before("pack_commit", s);
    pack_commit_kernel<<<(a.batch + 255) / 256, 256, 0, s>>>(a.n_entries, a.batch, half,
                                                             a.capacity);
    trace_after(s);
    return cudaGetLastError();
}

}  // namespace kvc
