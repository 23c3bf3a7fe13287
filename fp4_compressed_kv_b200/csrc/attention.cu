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
//  attn_mma   bf16 path for 64 heads x 576 (512 latent) entries.  A CTA owns a
//             contiguous range of 64-key chunks of one sequence.  Per chunk the
//             selected records (16-byte aligned rows) and window rows are
//             gathered into shared memory with cp.async, records are
//             dequantised in registers to bf16 (exact for UE4M3 scales), then
//             S = Q K^T and O += P V run on the tensor cores with fp32
//             accumulation and an online softmax in the log2 domain.
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
                const int t = -2 - k;
                v = to_f32(static_cast<const T*>(a.window)[((size_t)b * a.window_stride + t) * D + d]);
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
        float4 v[kMaxSplit];
#pragma unroll
        for (int s = 0; s < kMaxSplit; ++s)
            if (s < nsplit)
                v[s] = __ldcg(reinterpret_cast<const float4*>(a.part_o + (row0 + s) * Dv + d));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int s = 0; s < kMaxSplit; ++s)
            if (s < nsplit) {
                const float w = s_w[s];
                acc.x = fmaf(w, v[s].x, acc.x);
                acc.y = fmaf(w, v[s].y, acc.y);
                acc.z = fmaf(w, v[s].z, acc.z);
                acc.w = fmaf(w, v[s].w, acc.w);
            }
        *reinterpret_cast<float4*>(a.out + ((size_t)b * H + h) * Dv + d) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    if (tid == 0 && a.lse) a.lse[(size_t)b * H + h] = s_lse;
}

// ----------------------------------------------------------------------------
// tensor-core path (bf16, 64 heads, 576-channel entries, 512-channel values)
namespace tc {
constexpr int H = 64, D = 576, DV = 512, CK = kChunk;
constexpr int QS = D + 8;    // shared row stride in elements (1168 B: ldmatrix conflict-free)
constexpr int PS = CK + 8;   // 144 B
constexpr int RAW = 384;     // bytes reserved per gathered record
constexpr int kThreadsTC = 256;
constexpr size_t kOffQ = 0;
constexpr size_t kOffK = kOffQ + (size_t)H * QS * 2;
constexpr size_t kOffP = kOffK + (size_t)CK * QS * 2;
constexpr size_t kOffRaw = kOffP + (size_t)H * PS * 2;
constexpr size_t kOffKind = kOffRaw + (size_t)CK * RAW;
constexpr size_t kOffMax = kOffKind + CK * 4;
constexpr size_t kOffSum = kOffMax + 2 * H * 4;
constexpr size_t kSmem = kOffSum + 2 * H * 4;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;\n" ::: "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreadsTC, 1)
attn_mma_kernel(AttnArgs a, Shape sh, int K, float scale_log2, int chunks_per_split,
                int nsplit, int ue4m3) {
    extern __shared__ __align__(128) unsigned char smem[];
    __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + kOffQ);
    __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem + kOffK);
    __nv_bfloat16* sP = reinterpret_cast<__nv_bfloat16*>(smem + kOffP);
    unsigned char* sRaw = smem + kOffRaw;
    int* sKind = reinterpret_cast<int*>(smem + kOffKind);
    float* sMax = reinterpret_cast<float*>(smem + kOffMax);
    float* sSum = reinterpret_cast<float*>(smem + kOffSum);

    const int b = blockIdx.y, split = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hg = warp & 3, kh = warp >> 2;  // head group (16 rows); key half / value half
    const int n = a.n_entries[b];
    const bool len_ok = n >= 0 && n <= a.capacity;
    const int total = K + a.window_len;
    const int c0 = split * chunks_per_split;
    const int c1 = min(c0 + chunks_per_split, (total + CK - 1) / CK);
    const int rb = sh.rb, pieces = rb >> 4;

    // Q: 64 rows x 72 16-byte pieces
    {
        const unsigned char* qg =
            static_cast<const unsigned char*>(a.q) + (size_t)b * H * D * 2;
        for (int p = tid; p < H * (D / 8); p += kThreadsTC) {
            const int r = p / (D / 8), c = p - r * (D / 8);
            cp_async16(smem_u32(sQ + r * QS + c * 8), qg + (size_t)r * D * 2 + c * 16);
        }
    }

    float o[32][4];
#pragma unroll
    for (int i = 0; i < 32; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const int r0 = hg * 16 + (lane >> 2);  // rows r0 and r0 + 8

    const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), p_base = smem_u32(sP);

    for (int c = c0; c < c1; ++c) {
        if (tid < CK) {
            const int j = c * CK + tid;
            sKind[tid] = (j < total && len_ok) ? slot_kind(a, b, j, K, n) : -1;
        }
        __syncthreads();
        // gather records into sRaw, window rows straight into sK, zero empty rows
        for (int p = tid; p < CK * pieces; p += kThreadsTC) {
            const int s = p / pieces, pc = p - s * pieces;
            const int k = sKind[s];
            if (k >= 0)
                cp_async16(smem_u32(sRaw + s * RAW + pc * 16),
                           a.records + ((size_t)b * a.capacity + k) * rb + pc * 16);
        }
        for (int p = tid; p < CK * (D / 8); p += kThreadsTC) {
            const int s = p / (D / 8), pc = p - s * (D / 8);
            const int k = sKind[s];
            if (k <= -2) {
                const int t = -2 - k;
                cp_async16(smem_u32(sK + s * QS + pc * 8),
                           static_cast<const unsigned char*>(a.window) +
                               (((size_t)b * a.window_stride + t) * D) * 2 + pc * 16);
            } else if (k == -1) {
                *reinterpret_cast<uint4*>(sK + s * QS + pc * 8) = make_uint4(0, 0, 0, 0);
            }
        }
        cp_async_wait_all();
        __syncthreads();
        // dequantise records: (slot, 8-channel chunk) per item
        for (int p = tid; p < CK * (D / 8); p += kThreadsTC) {
            const int s = p / (D / 8), pc = p - s * (D / 8);
            if (sKind[s] < 0) continue;
            const unsigned char* rec = sRaw + s * RAW;
            const uint32_t codes = *reinterpret_cast<const uint32_t*>(rec + pc * 4);
            const int g = pc / sh.lpg;
            const float sc = ue4m3 ? e4m3_to_f32(rec[sh.code_bytes + g])
                                   : reinterpret_cast<const float*>(rec + sh.code_bytes)[g];
            uint4 v;
            v.x = pack_bf16(e2m1_value(codes & 15u) * sc, e2m1_value((codes >> 4) & 15u) * sc);
            v.y = pack_bf16(e2m1_value((codes >> 8) & 15u) * sc, e2m1_value((codes >> 12) & 15u) * sc);
            v.z = pack_bf16(e2m1_value((codes >> 16) & 15u) * sc, e2m1_value((codes >> 20) & 15u) * sc);
            v.w = pack_bf16(e2m1_value((codes >> 24) & 15u) * sc, e2m1_value(codes >> 28) * sc);
            *reinterpret_cast<uint4*>(sK + s * QS + pc * 8) = v;
        }
        __syncthreads();

        // S[16 rows of group hg][32 keys of half kh] = Q K^T
        float sacc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll 4
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t af[4];
            ldsm_x4(af, q_base + ((hg * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * QS + ks * 16 +
                                  (lane >> 4) * 8) * 2);
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                uint32_t bf[4];
                const int key0 = kh * 32 + pr * 16;
                ldsm_x4(bf, k_base + ((key0 + (lane & 7) + (lane >> 4) * 8) * QS + ks * 16 +
                                      ((lane >> 3) & 1) * 8) * 2);
                mma16816(sacc[2 * pr], af, bf[0], bf[1]);
                mma16816(sacc[2 * pr + 1], af, bf[2], bf[3]);
            }
        }
        // scale, mask, chunk row max
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = kh * 32 + nt * 8 + 2 * (lane & 3) + (e & 1);
                float x = sacc[nt][e] * scale_log2;
                if (sKind[key] == -1) x = -INFINITY;
                sacc[nt][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
            mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
        }
        if ((lane & 3) == 0) {
            sMax[kh * H + r0] = mx[0];
            sMax[kh * H + r0 + 8] = mx[1];
        }
        __syncthreads();
        float alpha[2], mnew[2], rs[2] = {0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = r0 + 8 * i;
            const float mc = fmaxf(sMax[r], sMax[H + r]);
            mnew[i] = fmaxf(m_run[i], mc);
            alpha[i] = mnew[i] == -INFINITY ? 1.f : exp2f(m_run[i] - mnew[i]);
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            float p[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float mm = mnew[e >> 1];
                p[e] = mm == -INFINITY ? 0.f : exp2f(sacc[nt][e] - mm);
                rs[e >> 1] += p[e];
            }
            const int col = kh * 32 + nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<uint32_t*>(sP + r0 * PS + col) = pack_bf16(p[0], p[1]);
            *reinterpret_cast<uint32_t*>(sP + (r0 + 8) * PS + col) = pack_bf16(p[2], p[3]);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 1);
            rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 2);
        }
        if ((lane & 3) == 0) {
            sSum[kh * H + r0] = rs[0];
            sSum[kh * H + r0 + 8] = rs[1];
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int r = r0 + 8 * i;
            l_run[i] = l_run[i] * alpha[i] + sSum[r] + sSum[H + r];
            m_run[i] = mnew[i];
        }
        // O[16 rows][256 values of half kh] = O * alpha + P V
#pragma unroll
        for (int nt = 0; nt < 32; ++nt) {
            o[nt][0] *= alpha[0];
            o[nt][1] *= alpha[0];
            o[nt][2] *= alpha[1];
            o[nt][3] *= alpha[1];
        }
#pragma unroll
        for (int kk = 0; kk < CK / 16; ++kk) {
            uint32_t af[4];
            ldsm_x4(af, p_base + ((hg * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * PS + kk * 16 +
                                  (lane >> 4) * 8) * 2);
#pragma unroll
            for (int np = 0; np < 16; ++np) {
                uint32_t bf[4];
                const int col0 = kh * 256 + np * 16;
                ldsm_x4_t(bf, k_base + ((kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * QS + col0 +
                                        (lane >> 4) * 8) * 2);
                mma16816(o[2 * np], af, bf[0], bf[1]);
                mma16816(o[2 * np + 1], af, bf[2], bf[3]);
            }
        }
        __syncthreads();
    }
    cp_async_wait_all();  // a split without chunks still drains the Q copies

    // epilogue
    const int h0 = r0, h1 = r0 + 8;
    if (nsplit == 1) {
        const float inv0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
        const float inv1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
        for (int nt = 0; nt < 32; ++nt) {
            const int col = kh * 256 + nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(a.out + ((size_t)b * H + h0) * DV + col) =
                make_float2(o[nt][0] * inv0, o[nt][1] * inv0);
            *reinterpret_cast<float2*>(a.out + ((size_t)b * H + h1) * DV + col) =
                make_float2(o[nt][2] * inv1, o[nt][3] * inv1);
        }
        if (kh == 0 && (lane & 3) == 0 && a.lse) {
            a.lse[(size_t)b * H + h0] = l_run[0] > 0.f ? (m_run[0] + __log2f(l_run[0])) * kLn2 : -INFINITY;
            a.lse[(size_t)b * H + h1] = l_run[1] > 0.f ? (m_run[1] + __log2f(l_run[1])) * kLn2 : -INFINITY;
        }
    } else {
        const size_t row0 = ((size_t)b * H + h0) * kMaxSplit + split;
        const size_t row1 = ((size_t)b * H + h1) * kMaxSplit + split;
#pragma unroll
        for (int nt = 0; nt < 32; ++nt) {
            const int col = kh * 256 + nt * 8 + 2 * (lane & 3);
            *reinterpret_cast<float2*>(a.part_o + row0 * DV + col) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2*>(a.part_o + row1 * DV + col) = make_float2(o[nt][2], o[nt][3]);
        }
        if (kh == 0 && (lane & 3) == 0) {
            a.part_ml[row0 * 2] = m_run[0];
            a.part_ml[row0 * 2 + 1] = l_run[0];
            a.part_ml[row1 * 2] = m_run[1];
            a.part_ml[row1 * 2 + 1] = l_run[1];
        }
    }
}
}  // namespace tc

bool tc_supported(const kvc_config& c, const Shape& sh) {
    return c.act_dtype == KVC_BF16 && c.n_heads == tc::H && sh.D == tc::D && sh.Dv == tc::DV &&
           sh.rb <= tc::RAW;
}

}  // namespace

bool tc05_supported(const kvc_config& c, const Shape& sh);
int launch_attention_tc05(const kvc_config& c, const Shape& sh, const AttnArgs& a, cudaStream_t s);

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
    cudaError_t err;
    int nsplit;
    if (tc05_supported(c, sh)) {
        nsplit = launch_attention_tc05(c, sh, a, s);
        if (nsplit < 0) return cudaErrorLaunchFailure;
    } else if (tc_supported(c, sh)) {
        const int nchunks = (total + tc::CK - 1) / tc::CK;
        int want = sms / a.batch;
        if (want < 1) want = 1;
        if (want > kMaxSplit) want = kMaxSplit;
        if (want > nchunks) want = nchunks;
        const int cps = nchunks == 0 ? 1 : (nchunks + want - 1) / want;
        nsplit = nchunks == 0 ? 1 : (nchunks + cps - 1) / cps;
        static bool attr_set[64] = {};
        if (dev >= 0 && dev < 64 && !attr_set[dev]) {
            err = cudaFuncSetAttribute(tc::attn_mma_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kSmem);
            if (err != cudaSuccess) return err;
            attr_set[dev] = true;
        }
        trace_before("attn_mma", s);
        tc::attn_mma_kernel<<<dim3(nsplit, a.batch), tc::kThreadsTC, tc::kSmem, s>>>(
            a, sh, K, scale_log2, cps, nsplit, ue4m3);
        trace_after(s);
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
            attn_simt_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(a, sh, c.n_heads, K, scale_log2,
                                                                    cps, nsplit, ue4m3);
        else
            attn_simt_kernel<float><<<grid, 256, smem, s>>>(a, sh, c.n_heads, K, scale_log2, cps,
                                                            nsplit, ue4m3);
        trace_after(s);
    }
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (nsplit > 1) {
        trace_before("attn_merge", s);
        attn_merge_kernel<<<dim3(c.n_heads, a.batch), 128, 0, s>>>(a, c.n_heads, sh.Dv, nsplit);
        trace_after(s);
        err = cudaGetLastError();
    }
    return err;
}

}  // namespace kvc
