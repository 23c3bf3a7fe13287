// attention.cu -- sparse decode attention over the gathered top-K entries and
// the sliding window, with a split-K log-sum-exp merge.
//
// Method: "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
// 压缩到 890 B的？" (acejoy.com) part 3 breakthrough 2 (all heads share one
// 512 latent + 64 RoPE entry; up-projections are absorbed into q and the
// output, so the values are the latent channels), breakthrough 4 (sliding
// window of 128 plus the indexer's top 512 global entries), part 4 "P4 main
// KV" (FP4 is storage only: entries are dequantised before attention).  One
// softmax runs jointly over the selected entries and the window keys.
//
// Kernels
//  attn_t128  (attn_t128.cu) tensor-core path for 64 heads x 576 (512 latent)
//             bf16 entries.
//  attn_simt  generic fp32 / bf16 path for other shapes (one warp per head).
//  attn_merge combines the per-split (max, sum, O) partials by log-sum-exp.
#include "kvc_internal.cuh"

namespace kvc {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float e2m1_value(uint32_t c) {
    const uint32_t m = c & 7u;  // magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6
    const float mag = m < 4u ? 0.5f * (float)m : (float)(1u << (m >> 1)) * (1.0f + 0.5f * (m & 1u)) * 0.5f;
    return (c & 8u) ? -mag : mag;
}

// Slot kinds: >= 0 record index; -1 empty; <= -2 window row (-2 - t).
__device__ __forceinline__ int slot_kind(const AttnArgs& a, int b, int j, int K, int n) {
    if (j < K) {
        const int idx = a.topk_idx[(size_t)b * K + j];
        if (idx == -1) return -1;
        if (idx < 0 || idx >= n) {
            set_status(a.status, KVC_DEV_BAD_INDEX);
            return -1;
        }
        return idx;
    }
    const int t = j - K;
    if (t < a.window_len) return -2 - t;
    return -1;
}

__device__ __forceinline__ void write_result(const AttnArgs& a, int b, int h, int H, int Dv,
                                             int nsplit, int split, float m, float l,
                                             int dv, float o, bool write_ml) {
    if (nsplit == 1) {
        const float inv = l > 0.f ? 1.f / l : 0.f;
        a.out[((size_t)b * H + h) * Dv + dv] = o * inv;
        if (write_ml && a.lse)
            a.lse[(size_t)b * H + h] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
    } else {
        const size_t row = ((size_t)b * H + h) * kMaxSplit + split;
        a.part_o[row * Dv + dv] = o;
        if (write_ml) {
            a.part_ml[row * 2] = m;
            a.part_ml[row * 2 + 1] = l;
        }
    }
}

// ----------------------------------------------------------------------------
// generic SIMT path: grid (nsplit, ceil(H/8), B); warp w of block y is head 8y+w
constexpr int kSimtChunk = 32;

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

template <typename T>
__global__ void __launch_bounds__(256)
attn_simt_kernel(AttnArgs a, Shape sh, int H, int K, float scale_log2, int chunks_per_split,
                 int nsplit, int ue4m3) {
    extern __shared__ __align__(16) float keys[];  // [kSimtChunk][D]
    __shared__ int kind[kSimtChunk];
    pdl_wait();
    const int b = blockIdx.z, split = blockIdx.x;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int h = blockIdx.y * 8 + w;
    const int D = sh.D, Dv = sh.Dv;
    const int n = a.n_entries[b];
    const bool len_ok = n >= 0 && n <= a.capacity;
    const int total = K + a.window_len;
    const int c0 = split * chunks_per_split;
    const int c1 = min(c0 + chunks_per_split, (total + kSimtChunk - 1) / kSimtChunk);

    float q[32], o[32];
    float m = -INFINITY, l = 0.f;
    const T* qp = static_cast<const T*>(a.q) + ((size_t)b * H + (h < H ? h : 0)) * D;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int d = lane + 32 * i;
        q[i] = (d < D) ? to_f32(qp[d]) : 0.f;
        o[i] = 0.f;
    }
    for (int c = c0; c < c1; ++c) {
        if (threadIdx.x < kSimtChunk) {
            const int j = c * kSimtChunk + threadIdx.x;
            kind[threadIdx.x] = (j < total && len_ok) ? slot_kind(a, b, j, K, n) : -1;
        }
        __syncthreads();
        for (int p = threadIdx.x; p < kSimtChunk * D; p += blockDim.x) {
            const int s = p / D, d = p - s * D;
            const int k = kind[s];
            float v = 0.f;
            if (k >= 0) {
                const uint8_t* rec = a.records + ((size_t)b * a.capacity + k) * sh.rb;
                const uint32_t code = (rec[d >> 1] >> ((d & 1) * 4)) & 15u;
                const int g = (d >> 3) / sh.lpg;
                const float sc =
                    ue4m3 ? e4m3_to_f32(rec[sh.code_bytes + g])
                          : reinterpret_cast<const float*>(rec + sh.code_bytes)[g];
                v = e2m1_value(code) * sc;
            } else if (k <= -2) {
                const size_t row = (size_t)b * a.window_stride + (-2 - k);
                v = a.win_fp8 ? e4m3s_to_f32(a.win_fp8[row * D + d]) * a.win_scale[row]
                              : to_f32(static_cast<const T*>(a.window)[row * D + d]);
            }
            keys[p] = v;
        }
        __syncthreads();
        if (h < H) {
            for (int s = 0; s < kSimtChunk; ++s) {
                if (kind[s] == -1) continue;
                const float* kr = keys + s * D;
                float part = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int d = lane + 32 * i;
                    if (d < D) part = fmaf(q[i], kr[d], part);
                }
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                const float x = part * scale_log2;
                const float mn = fmaxf(m, x);
                const float alpha = exp2f(m - mn);  // m = -inf -> 0
                const float p = exp2f(x - mn);
                l = l * alpha + p;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int d = lane + 32 * i;
                    if (d < Dv) o[i] = fmaf(p, kr[d], o[i] * alpha);
                }
                m = mn;
            }
        }
        __syncthreads();
    }
    if (h >= H) return;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const int d = lane + 32 * i;
        if (d < Dv) write_result(a, b, h, H, Dv, nsplit, split, m, l, d, o[i], i == 0 && lane == 0);
    }
}

// ----------------------------------------------------------------------------
// merge of split partials: grid (H, B), 128 threads; all split loads of a
// thread are issued together
__global__ void __launch_bounds__(128)
attn_merge_kernel(AttnArgs a, int H, int Dv, int nsplit) {
    __shared__ float s_w[kMaxSplit];
    __shared__ float s_inv, s_lse;
    pdl_wait();
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const size_t row0 = ((size_t)b * H + h) * kMaxSplit;
    if (tid < 32) {
        const float m = tid < nsplit ? __ldcg(a.part_ml + (row0 + tid) * 2) : -INFINITY;
        const float l = tid < nsplit ? __ldcg(a.part_ml + (row0 + tid) * 2 + 1) : 0.f;
        float M = m;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float w = (M == -INFINITY || tid >= nsplit) ? 0.f : exp2f(m - M);
        float L = w * l;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (tid < kMaxSplit) s_w[tid] = w;
        if (tid == 0) {
            s_inv = L > 0.f ? 1.f / L : 0.f;
            s_lse = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
        }
    }
    __syncthreads();
    const float inv = s_inv;
    for (int d = tid * 4; d < Dv; d += 128 * 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int s = 0; s < nsplit; ++s) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part_o + (row0 + s) * Dv + d));
            const float w = s_w[s];
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
        }
        *reinterpret_cast<float4*>(a.out + ((size_t)b * H + h) * Dv + d) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (tid == 0 && a.lse) a.lse[(size_t)b * H + h] = s_lse;
}

// A Reuse layer's copy of its head's top-K (the tensor-core kernel writes it
// itself while it reads the indices).
__global__ void copy_topk_kernel(const int32_t* __restrict__ src, int32_t* __restrict__ dst,
                                 int n) {
    pdl_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
        dst[i] = src[i];
}

}  // namespace

bool t128_supported(const kvc_config& c, const Shape& sh);
int launch_attention_t128(const kvc_config& c, const Shape& sh, const AttnArgs& a, cudaStream_t s);

cudaError_t launch_attention(const kvc_config& c, const Shape& sh, const AttnArgs& a,
                             cudaStream_t s) {
    if (a.batch == 0) return cudaSuccess;
    const int K = c.topk;
    const int total = K + a.window_len;
    const float scale_log2 = c.sm_scale * kLog2e;
    const int ue4m3 = c.scale_fmt == KVC_SCALE_UE4M3;
    int dev = 0;
    cudaGetDevice(&dev);
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaError_t err = cudaSuccess;
    int nsplit;
    if (t128_supported(c, sh)) {
        nsplit = launch_attention_t128(c, sh, a, s);
        if (nsplit < 0) return cudaErrorLaunchFailure;
    } else {
        const int nchunks = (total + kSimtChunk - 1) / kSimtChunk;
        const int hblocks = (c.n_heads + 7) / 8;
        int want = (2 * sms) / (a.batch * hblocks);
        if (want < 1) want = 1;
        if (want > kMaxSplit) want = kMaxSplit;
        if (want > nchunks) want = nchunks;
        const int cps = nchunks == 0 ? 1 : (nchunks + want - 1) / want;
        nsplit = nchunks == 0 ? 1 : (nchunks + cps - 1) / cps;
        const size_t smem = (size_t)kSimtChunk * sh.D * sizeof(float);
        static bool attr_set2[64][2] = {};
        const int ti = c.act_dtype == KVC_BF16;
        if (dev >= 0 && dev < 64 && !attr_set2[dev][ti]) {
            err = ti ? cudaFuncSetAttribute(attn_simt_kernel<__nv_bfloat16>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kSimtChunk * 1024 * 4)
                     : cudaFuncSetAttribute(attn_simt_kernel<float>,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            kSimtChunk * 1024 * 4);
            if (err != cudaSuccess) return err;
            attr_set2[dev][ti] = true;
        }
        dim3 grid(nsplit, hblocks, a.batch);
        trace_before("attn_simt", s);
        if (ti)
            err = launch_pdl(attn_simt_kernel<__nv_bfloat16>, grid, 256, smem, s, a, sh, c.n_heads,
                             K, scale_log2, cps, nsplit, ue4m3);
        else
            err = launch_pdl(attn_simt_kernel<float>, grid, 256, smem, s, a, sh, c.n_heads, K,
                             scale_log2, cps, nsplit, ue4m3);
        trace_after(s);
        if (err != cudaSuccess) return err;
        if (a.topk_copy) {
            const int cnt = a.batch * K;
            trace_before("copy_topk", s);
            err = launch_pdl(copy_topk_kernel, (cnt + 1023) / 1024, 256, 0, s, a.topk_idx,
                             a.topk_copy, cnt);
            trace_after(s);
            if (err != cudaSuccess) return err;
        }
    }
    if (nsplit > 1) {
        trace_before("attn_merge", s);
        err = launch_pdl(attn_merge_kernel, dim3(c.n_heads, a.batch), 128, 0, s, a, c.n_heads, sh.Dv,
                         nsplit);
        trace_after(s);
    }
    return err;
}

}  // namespace kvc
