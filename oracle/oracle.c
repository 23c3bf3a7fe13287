/*
 * oracle.c -- plain, slow CPU oracle for compressed-KV sparse decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant
 * generator with the CUDA library; every step is written out here from the
 * pages' statement of the method.
 *
 * Sources (pages, by title and section):
 *  [P1] "DeepSeek V4.1 Flash KV Cache压缩实战：FP4+CSA2+CED将显存降至1/4"
 *       (gtnt.cn): 3.1 FP4 group quantisation, 3.2 CSA2 compression,
 *       4.1 KV-size estimate, 4.3 parameter table.
 *  [P2] "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B
 *       压缩到 890 B的？" (acejoy.com): part 1 "KV Cache 到底有多大";
 *       part 3 breakthrough 2 (MLA 512+64), breakthrough 4 (SWA-128,
 *       indexer top-512, CSA 2:1); part 4 "CSA2：三种模式", "P4 main KV",
 *       "890 字节是怎么算出来的".
 *
 * Readings where the pages leave a step open (each is documented with the
 * function that takes it):
 *  R1 gate: one D-vector g gives one logit per token; the pair's weights are
 *     the softmax of the two logits.  The pages fix no precision for this
 *     step; the quantised codes downstream depend on the exact fp32 entry, so
 *     the specification fixes one: fp32, the channels dealt round-robin in
 *     chunks of 8 to 8 running sums (chunk c to sum c mod 8), the 8 sums
 *     combined pairwise at distances 4, 2, 1.
 *  R2 exp: written here in fp32 from the Cody-Waite argument reduction and a
 *     degree-7 Taylor polynomial (Horner form), so that the gate weight is the
 *     same bits on every implementation of this specification.
 *  R3 grouping: latent and RoPE segments are grouped separately; a segment's
 *     last group may be short.
 *  R4 scale: s = absmax / 6 in fp32, stored as fp32 or rounded (RNE,
 *     saturating) to an unsigned E4M3 byte; elements are divided by the
 *     decoded scale and rounded to nearest-even onto the E2M1 grid.
 *  R5 attention: one joint softmax over the selected entries and the window
 *     tokens; values are the first Dv (latent) channels of each key.
 *  R18 FP4 indexer keys: quantised like a main-KV entry (no RoPE, groups of
 *     16, UE4M3), scored exactly against the int8 query (see
 *     orc_idx_fp4_score).
 *  R17 4:1 compression ([P1] 4.3 lists a CSA2 compression ratio of 2x or 4x):
 *     four consecutive tokens form one entry, weighted by the softmax of their
 *     four gate logits, each logit summed in the order of R1; see
 *     orc_compress_group4.
 *
 * Pins: every function is checked by the not-gpu tests against what the
 * pages or the mathematics fix (printed values, closed forms, brute force,
 * library routines).  orc_compress_pair and orc_compress_group4 are pinned by
 * invariants (identical tokens, zero gate, a dominant token, convexity) and
 * by an fp64 evaluation of the compression that shares none of this order:
 * every entry lies within a derived error bound of the exact softmax-weighted
 * sum, and the packed records equal those of the fp64 entry rounded once to
 * fp32 except for codes or scales whose quotient straddles a rounding
 * midpoint within that bound (about 5e-7 of the codes).  Only the choice of
 * the fp32 order itself (R1, R17) is a reading; the GPU follows the same one
 * so that its records match the oracle's bit for bit.
 *
 * Compile with -ffp-contract=off: every fused multiply-add below is an
 * explicit fma() call and nothing else may be contracted.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_INVALID 1
#define ORC_ERR_CAPACITY 2

#define ORC_SCALE_F32 0
#define ORC_SCALE_UE4M3 1

#define ORC_MODE_FULL 0
#define ORC_MODE_REINDEX 1
#define ORC_MODE_REUSE 2

/* status bits reported by the pack / attention oracles */
#define ORC_ST_NONFINITE 1u
#define ORC_ST_BAD_INDEX 2u

typedef struct {
    int latent_dim;  /* Dv: latent channels, also the value width        */
    int rope_dim;    /* RoPE channels appended to the key                 */
    int group;       /* FP4 group size G                                  */
    int scale_fmt;   /* ORC_SCALE_F32 or ORC_SCALE_UE4M3                  */
    int idx_dim;     /* indexer key width Di                              */
    int topk;        /* K                                                 */
    int window;      /* W                                                 */
    int n_heads;     /* H                                                 */
    double sm_scale; /* softmax scale applied to q.k                      */
    int ratio;       /* raw tokens per entry: 2 (0 also means 2) or 4     */
} orc_cfg;

/* ------------------------------------------------------------------ */
/* KV-size formula: [P2] part 1 "KV Cache 到底有多大" and [P1] 4.1.
 * bytes per token = 2 (K and V) x layers x heads x head_dim x bytes.    */
uint64_t orc_kv_bytes_per_token(int64_t layers, int64_t heads, int64_t dim,
                                int64_t bytes_per_elem) {
    return (uint64_t)(2 * layers * heads * dim * bytes_per_elem);
}

/* ------------------------------------------------------------------ */
/* R2: exp(x) in fp32.  Cody-Waite: x = n*ln2 + r with ln2 split into a
 * 16-significant-bit head (so n*LN2_HI is exact for |n| < 2^8) and the
 * rounded remainder; e^r from the Taylor series to degree 7 (truncation
 * below 6e-9 for |r| <= ln2/2, under half an fp32 ulp of e^r); the result is
 * scaled by an exactly built power of two.  Inputs above 88 give +inf;
 * inputs below -87 give 0 (there exp(x) < 2^-125 and 1 + exp(x) == 1 in the
 * gate).                                                                */
static const float ORC_LN2_HI_F = 0x1.62e4p-1f;
static const float ORC_LN2_LO_F = 0x1.7f7d1cp-20f;
static const float ORC_INV_LN2_F = 0x1.715476p+0f;
static const float ORC_INV_FACT_F[8] = {
    0x1.0p+0f, 0x1.0p+0f, 0x1.0p-1f, 0x1.555556p-3f,
    0x1.555556p-5f, 0x1.111112p-7f, 0x1.6c16c2p-10f, 0x1.a01a02p-13f};

float orc_expf(float x) {
    if (x != x) return x;
    if (x > 88.0f) return INFINITY;
    if (x < -87.0f) return 0.0f;
    float n = nearbyintf(x * ORC_INV_LN2_F); /* round-half-even, default mode */
    float r = fmaf(-n, ORC_LN2_HI_F, x);
    r = fmaf(-n, ORC_LN2_LO_F, r);
    float p = ORC_INV_FACT_F[7];
    for (int k = 6; k >= 0; --k) p = fmaf(p, r, ORC_INV_FACT_F[k]);
    int32_t bits = ((int32_t)n + 127) << 23;
    float two_n;
    memcpy(&two_n, &bits, sizeof two_n);
    return p * two_n;
}

/* ------------------------------------------------------------------ */
/* E2M1 ([P1] 3.1; [P2] "P4 main KV"): 1 sign, 2 exponent, 1 mantissa bit.
 * Magnitude codes 0..7 are {0, 0.5, 1, 1.5, 2, 3, 4, 6}; bit 3 is the sign. */
static const float ORC_E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f,
                                      2.0f, 3.0f, 4.0f, 6.0f};

float orc_e2m1_value(int code) {
    float m = ORC_E2M1_MAG[code & 7];
    return (code & 8) ? -m : m;
}

/* Round to the nearest grid magnitude; a tie goes to the even code (code
 * bit 0 clear); magnitudes past 6 saturate to 6.  A result of magnitude 0
 * is stored as +0 (code 0).  Non-finite input is the caller's business.   */
int orc_e2m1_encode(float v) {
    double m = fabs((double)v);
    int best = 0;
    double best_d = m; /* distance to magnitude 0 */
    for (int c = 1; c < 8; ++c) {
        double d = fabs(m - (double)ORC_E2M1_MAG[c]);
        if (d < best_d || (d == best_d && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_d = d;
        }
    }
    if (m > 6.0) best = 7;
    if (best == 0) return 0;
    return (v < 0.0f) ? (best | 8) : best;
}

/* E4M3 (OCP "fn": bias 7, no infinities, 0x7F/0xFF are NaN, max 448). */
float orc_e4m3_value(int b) {
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    float v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexpf((float)m, -9);
    else
        v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -v : v;
}

/* Unsigned E4M3 encode for v >= 0: nearest of the 127 finite non-negative
 * values by exhaustive search, ties to the even code, saturating at 448.  */
int orc_e4m3_encode(float v) {
    if (!(v > 0.0f)) return 0;
    if (v >= 448.0f) return 0x7E;
    double x = (double)v;
    int best = 0;
    double best_d = x;
    for (int b = 1; b <= 0x7E; ++b) {
        double d = fabs(x - (double)orc_e4m3_value(b));
        if (d < best_d || (d == best_d && (b & 1) == 0 && (best & 1) == 1)) {
            best = b;
            best_d = d;
        }
    }
    return best;
}

/* ------------------------------------------------------------------ */
/* FP8 window rows ([P2] part 4 "P4 main KV": the SWA KV stays FP8; the
 * pages give no scale layout).  Reading: one fp32 scale per row,
 * s = absmax / 448 over the row's finite values (IEEE RN), each element
 * coded as signed E4M3 of x / s rounded to nearest even and saturating at
 * 448; a magnitude of zero is stored as +0; non-finite elements are coded 0
 * and reported.  Returns 1 if the row held a non-finite value.            */
int orc_window_fp8(const float* row, int D, uint8_t* codes, float* scale) {
    float amax = 0.0f;
    int bad = 0;
    for (int d = 0; d < D; ++d) {
        if (!isfinite(row[d])) {
            bad = 1;
            continue;
        }
        float a = fabsf(row[d]);
        if (a > amax) amax = a;
    }
    float s = amax / 448.0f;
    *scale = s;
    for (int d = 0; d < D; ++d) {
        float x = row[d];
        int c = 0;
        if (isfinite(x) && s > 0.0f) {
            float v = x / s;
            int mag = orc_e4m3_encode(fabsf(v));
            c = mag == 0 ? 0 : ((v < 0.0f ? 0x80 : 0) | mag);
        }
        codes[d] = (uint8_t)c;
    }
    return bad;
}

/* Decoded FP8 window row: E4M3(code) x scale, in fp32.                 */
void orc_window_fp8_dequant(const uint8_t* codes, float scale, int D, float* out) {
    for (int d = 0; d < D; ++d) out[d] = orc_e4m3_value(codes[d]) * scale;
}

/* ------------------------------------------------------------------ */
/* R3 grouping and the record layout.                                 */
int orc_n_groups(int latent, int rope, int group) {
    return (latent + group - 1) / group + (rope + group - 1) / group;
}

/* Record = [codes: one byte per channel pair, even channel in the low
 * nibble][scales in group order][zero padding to a 16-byte multiple].
 * The padded size is the stride of the record array.                   */
int orc_record_bytes(const orc_cfg* c, int padded) {
    int d = c->latent_dim + c->rope_dim;
    int sb = (c->scale_fmt == ORC_SCALE_F32) ? 4 : 1;
    int n = d / 2 + orc_n_groups(c->latent_dim, c->rope_dim, c->group) * sb;
    return padded ? (n + 15) / 16 * 16 : n;
}

/* group boundaries: fills start[] / len[] with the channel range of each
 * group; returns the number of groups                                   */
static int orc_groups(const orc_cfg* c, int* start, int* len) {
    int g = 0;
    for (int s = 0; s < c->latent_dim; s += c->group, ++g) {
        start[g] = s;
        len[g] = (c->latent_dim - s < c->group) ? c->latent_dim - s : c->group;
    }
    for (int s = 0; s < c->rope_dim; s += c->group, ++g) {
        start[g] = c->latent_dim + s;
        len[g] = (c->rope_dim - s < c->group) ? c->rope_dim - s : c->group;
    }
    return g;
}

/* ------------------------------------------------------------------ */
/* R1: the 2:1 compression of a token pair ([P2] breakthrough 4: a trained
 * compressor turns every two tokens into one entry; [P1] 3.2: the key
 * compressor of CSA2).
 * logit_t = g . k_t; (w0, w1) = softmax(logit_0, logit_1);
 * entry = w0 k_0 + w1 k_1, everything in fp32.
 * Fixed evaluation order: delta = logit_0 - logit_1 = sum_d g_d (k0_d - k1_d)
 * accumulated by 8 partial sums; channel chunk c = [8c, 8c+8) goes to
 * partial c mod 8, chunks in increasing order and channels in increasing
 * order inside a chunk, each term added with one fmaf after an fp32
 * subtraction.  The partials are combined by a xor tree over offsets 4, 2, 1.
 * w0 = 1 / (1 + exp(-delta)), w1 = 1 - w0, entry_d = fmaf(w0, k0_d, w1 * k1_d). */
float orc_gate_delta(const float* k0, const float* k1, const float* g, int D) {
    float acc[8];
    for (int l = 0; l < 8; ++l) acc[l] = 0.0f;
    for (int c = 0; c * 8 < D; ++c) {
        int l = c % 8;
        for (int t = 0; t < 8 && 8 * c + t < D; ++t) {
            int d = 8 * c + t;
            float diff = k0[d] - k1[d];
            acc[l] = fmaf(g[d], diff, acc[l]);
        }
    }
    for (int off = 4; off >= 1; off >>= 1) {
        float nxt[8];
        for (int l = 0; l < 8; ++l) nxt[l] = acc[l] + acc[l ^ off];
        memcpy(acc, nxt, sizeof acc);
    }
    return acc[0];
}

void orc_compress_pair(const float* k0, const float* k1, const float* g, int D,
                       float* e) {
    float delta = orc_gate_delta(k0, k1, g, D);
    float w0 = 1.0f / (1.0f + orc_expf(-delta));
    float w1 = 1.0f - w0;
    for (int d = 0; d < D; ++d) e[d] = fmaf(w0, k0[d], w1 * k1[d]);
}

/* R17: the 4:1 compression of four consecutive tokens (the ratio 4 of [P1]
 * 4.3; the pages give the 2:1 rule only, this is its plainest extension).
 * logit_t = g . k_t, each summed like delta in R1: 8 partial sums over the
 * 8-channel chunks (chunk c to partial c mod 8, chunks and channels in
 * increasing order, one fmaf per term), combined by a xor tree over 4, 2, 1.
 * M = max_t logit_t; e_t = exp(logit_t - M) (R2, fp32 subtraction first);
 * S = ((e_0 + e_1) + e_2) + e_3; w_t = e_t / S;
 * entry_d = fmaf(w0, k0_d, fmaf(w1, k1_d, fmaf(w2, k2_d, w3 * k3_d))). */
float orc_gate_logit(const float* k, const float* g, int D) {
    float acc[8];
    for (int l = 0; l < 8; ++l) acc[l] = 0.0f;
    for (int c = 0; c * 8 < D; ++c) {
        int l = c % 8;
        for (int t = 0; t < 8 && 8 * c + t < D; ++t) {
            int d = 8 * c + t;
            acc[l] = fmaf(g[d], k[d], acc[l]);
        }
    }
    for (int off = 4; off >= 1; off >>= 1) {
        float nxt[8];
        for (int l = 0; l < 8; ++l) nxt[l] = acc[l] + acc[l ^ off];
        memcpy(acc, nxt, sizeof acc);
    }
    return acc[0];
}

void orc_compress_group4(const float* k0, const float* k1, const float* k2, const float* k3,
                         const float* g, int D, float* e) {
    const float* k[4] = {k0, k1, k2, k3};
    float lg[4], ex[4], w[4];
    float m = -INFINITY;
    for (int t = 0; t < 4; ++t) {
        lg[t] = orc_gate_logit(k[t], g, D);
        if (lg[t] > m) m = lg[t];
    }
    for (int t = 0; t < 4; ++t) ex[t] = orc_expf(lg[t] - m);
    float sum = ((ex[0] + ex[1]) + ex[2]) + ex[3];
    for (int t = 0; t < 4; ++t) w[t] = ex[t] / sum;
    for (int d = 0; d < D; ++d)
        e[d] = fmaf(w[0], k0[d], fmaf(w[1], k1[d], fmaf(w[2], k2[d], w[3] * k3[d])));
}

/* ------------------------------------------------------------------ */
/* R4: FP4 group quantisation of one entry into one record ([P1] 3.1;
 * [P2] "P4 main KV").  Returns the number of non-finite inputs, which are
 * treated as 0 for both the group maximum and their code.               */
int orc_quantize_entry(const orc_cfg* c, const float* e, uint8_t* rec) {
    int D = c->latent_dim + c->rope_dim;
    int start[1024], len[1024];
    int ng = orc_groups(c, start, len);
    int nonfinite = 0;
    memset(rec, 0, (size_t)orc_record_bytes(c, 1));
    for (int gi = 0; gi < ng; ++gi) {
        float a = 0.0f;
        for (int d = start[gi]; d < start[gi] + len[gi]; ++d) {
            float x = e[d];
            if (!isfinite(x)) continue;
            if (fabsf(x) > a) a = fabsf(x);
        }
        float s = a / 6.0f;
        if (c->scale_fmt == ORC_SCALE_UE4M3) {
            int sb = orc_e4m3_encode(s);
            rec[D / 2 + gi] = (uint8_t)sb;
            s = orc_e4m3_value(sb);
        } else {
            memcpy(rec + D / 2 + 4 * gi, &s, 4);
        }
        for (int d = start[gi]; d < start[gi] + len[gi]; ++d) {
            float x = e[d];
            int code = 0;
            if (!isfinite(x))
                ++nonfinite;
            else if (s > 0.0f)
                code = orc_e2m1_encode(x / s);
            rec[d / 2] |= (uint8_t)((d & 1) ? (code << 4) : code);
        }
    }
    return nonfinite;
}

/* Dequantisation before attention ([P2] "P4 main KV": FP4 is storage
 * only): x = E2M1(code) * scale, in fp32.                               */
void orc_dequantize_entry(const orc_cfg* c, const uint8_t* rec, float* x) {
    int D = c->latent_dim + c->rope_dim;
    int start[1024], len[1024];
    int ng = orc_groups(c, start, len);
    for (int gi = 0; gi < ng; ++gi) {
        float s;
        if (c->scale_fmt == ORC_SCALE_UE4M3)
            s = orc_e4m3_value(rec[D / 2 + gi]);
        else
            memcpy(&s, rec + D / 2 + 4 * gi, 4);
        for (int d = start[gi]; d < start[gi] + len[gi]; ++d) {
            int code = (d & 1) ? (rec[d / 2] >> 4) : (rec[d / 2] & 15);
            x[d] = orc_e2m1_value(code) * s;
        }
    }
}

/* ------------------------------------------------------------------ */
/* Pack: append n_new/r compressed entries per sequence (r = the ratio, 2
 * or 4), with their indexer keys, at position n_entries[b]; then advance
 * n_entries[b].  tokens [B][n_new][D] fp32 (bf16 inputs widened exactly by
 * the caller), idxk_new [B][n_new/r][Di], records [B][cap][record_bytes
 * (padded)], idx_cache [B][cap][Di].                                     */
int orc_pack(const orc_cfg* c, int B, int n_new, const float* tokens,
             const float* g, const int8_t* idxk_new, int cap, uint8_t* records,
             int8_t* idx_cache, int32_t* n_entries, uint32_t* status) {
    int D = c->latent_dim + c->rope_dim;
    int rb = orc_record_bytes(c, 1);
    int r = c->ratio == 0 ? 2 : c->ratio;
    if (r != 2 && r != 4) return ORC_ERR_INVALID;
    if (n_new < 0 || n_new % r) return ORC_ERR_INVALID;
    int per = n_new / r;
    for (int b = 0; b < B; ++b)
        if (n_entries[b] < 0 || n_entries[b] + per > cap) return ORC_ERR_CAPACITY;
    float* e = (float*)malloc(sizeof(float) * (size_t)D);
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < per; ++i) {
            const float* k0 = tokens + ((size_t)b * n_new + (size_t)r * i) * D;
            int64_t pos = n_entries[b] + i;
            if (r == 2)
                orc_compress_pair(k0, k0 + D, g, D, e);
            else
                orc_compress_group4(k0, k0 + D, k0 + 2 * D, k0 + 3 * D, g, D, e);
            if (orc_quantize_entry(c, e, records + ((size_t)b * cap + pos) * rb))
                *status |= ORC_ST_NONFINITE;
            memcpy(idx_cache + ((size_t)b * cap + pos) * c->idx_dim,
                   idxk_new + ((size_t)b * per + i) * c->idx_dim,
                   (size_t)c->idx_dim);
        }
        n_entries[b] += per;
    }
    free(e);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Lightweight indexer ([P2] breakthrough 4: a small indexer scores every
 * stored entry): score_j = sum_d q_d k_{j,d}, int8 x int8 -> int32.      */
void orc_index_scores(const int8_t* q, const int8_t* keys, int n, int di,
                      int32_t* scores) {
    for (int j = 0; j < n; ++j) {
        int32_t s = 0;
        for (int d = 0; d < di; ++d) s += (int32_t)q[d] * (int32_t)keys[(size_t)j * di + d];
        scores[j] = s;
    }
}

typedef struct {
    int32_t score;
    int32_t idx;
} orc_scored;

static int orc_by_score_desc_idx_asc(const void* pa, const void* pb) {
    const orc_scored* a = (const orc_scored*)pa;
    const orc_scored* b = (const orc_scored*)pb;
    if (a->score != b->score) return (a->score > b->score) ? -1 : 1;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static int orc_int_asc(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* Top-K ([P2] breakthrough 4: only the 512 best-scored entries are kept): order all n
 * entries by (score descending, index ascending), keep the first
 * min(k, n), write them sorted by index ascending and pad with -1.
 * Returns the number kept.                                              */
int orc_topk(const int32_t* scores, int n, int k, int32_t* out) {
    orc_scored* v = (orc_scored*)malloc(sizeof(orc_scored) * (size_t)(n > 0 ? n : 1));
    for (int j = 0; j < n; ++j) {
        v[j].score = scores[j];
        v[j].idx = j;
    }
    qsort(v, (size_t)n, sizeof(orc_scored), orc_by_score_desc_idx_asc);
    int kept = n < k ? n : k;
    for (int i = 0; i < kept; ++i) out[i] = v[i].idx;
    qsort(out, (size_t)kept, sizeof(int32_t), orc_int_asc);
    for (int i = kept; i < k; ++i) out[i] = -1;
    free(v);
    return kept;
}

/* index + top-K for a batch; scores (optional) [B][cap] receives the
 * visible scores (entries past n_entries[b] are left untouched).        */
int orc_index_topk(const orc_cfg* c, int B, const int8_t* idx_q,
                   const int8_t* idx_cache, int cap, const int32_t* n_entries,
                   int32_t* topk, int32_t* scores_out) {
    int32_t* s = (int32_t*)malloc(sizeof(int32_t) * (size_t)(cap > 0 ? cap : 1));
    for (int b = 0; b < B; ++b) {
        int n = n_entries[b];
        if (n < 0 || n > cap) {
            free(s);
            return ORC_ERR_CAPACITY;
        }
        orc_index_scores(idx_q + (size_t)b * c->idx_dim,
                         idx_cache + (size_t)b * cap * c->idx_dim, n, c->idx_dim, s);
        if (scores_out) memcpy(scores_out + (size_t)b * cap, s, sizeof(int32_t) * (size_t)n);
        orc_topk(s, n, c->topk, topk + (size_t)b * c->topk);
    }
    free(s);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* R18: FP4 indexer keys ([P2] "890 字节是怎么算出来的": an FP4 indexer K is
 * 128 dims x 0.5 B plus 8 scales = 72 B).  A key row is quantised exactly
 * like a main-KV entry of Di latent channels, no RoPE channels, groups of 16
 * and UE4M3 scales (orc_quantize_entry with that configuration): Di/2 code
 * bytes, then Di/16 scale bytes.  Its score against the int8 query is the
 * exact value of q . dequant(k): per group, the integer sum of q_d times
 * twice the E2M1 value (an integer in -12..12), times the scale times 2^9
 * (an integer: every UE4M3 value is a multiple of 2^-9), summed over the
 * groups -- the score times 2^10, exact in int64 (|.| < 2^36 for Di = 128),
 * so the top-K over these scores is as exact as over int8 keys.          */
int64_t orc_idx_fp4_score(const int8_t* q, const uint8_t* rec, int di) {
    int64_t total = 0;
    for (int g = 0; g < di / 16; ++g) {
        int64_t part = 0;
        for (int d = 16 * g; d < 16 * g + 16; ++d) {
            int code = (d & 1) ? (rec[d / 2] >> 4) : (rec[d / 2] & 15);
            int twice = (int)lrint(2.0 * (double)orc_e2m1_value(code));  /* exact */
            part += (int64_t)q[d] * twice;
        }
        int64_t s9 = (int64_t)llrint((double)orc_e4m3_value(rec[di / 2 + g]) * 512.0);
        total += part * s9;
    }
    return total;
}

/* Top-K over int64 scores, (score descending, index ascending); the same
 * output form as orc_topk.                                               */
typedef struct {
    int64_t score;
    int32_t idx;
} orc_scored64;

static int orc_by_score64_desc_idx_asc(const void* pa, const void* pb) {
    const orc_scored64* a = (const orc_scored64*)pa;
    const orc_scored64* b = (const orc_scored64*)pb;
    if (a->score != b->score) return (a->score > b->score) ? -1 : 1;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

int orc_topk64(const int64_t* scores, int n, int k, int32_t* out) {
    orc_scored64* v = (orc_scored64*)malloc(sizeof(orc_scored64) * (size_t)(n > 0 ? n : 1));
    for (int j = 0; j < n; ++j) {
        v[j].score = scores[j];
        v[j].idx = j;
    }
    qsort(v, (size_t)n, sizeof(orc_scored64), orc_by_score64_desc_idx_asc);
    int kept = n < k ? n : k;
    for (int i = 0; i < kept; ++i) out[i] = v[i].idx;
    qsort(out, (size_t)kept, sizeof(int32_t), orc_int_asc);
    for (int i = kept; i < k; ++i) out[i] = -1;
    free(v);
    return kept;
}

/* Indexer top-K over FP4 keys: idx_q [B][Di] int8, keys [B][cap][Di/2 +
 * Di/16] (R18 rows), scores_out [B][cap] int64 (times 2^10) or NULL.     */
int orc_index_topk_fp4(const orc_cfg* c, int B, const int8_t* idx_q, const uint8_t* keys,
                       int cap, const int32_t* n_entries, int32_t* topk, int64_t* scores_out) {
    int di = c->idx_dim, row = di / 2 + di / 16;
    if (di % 16) return ORC_ERR_INVALID;
    int64_t* s = (int64_t*)malloc(sizeof(int64_t) * (size_t)(cap > 0 ? cap : 1));
    for (int b = 0; b < B; ++b) {
        int n = n_entries[b];
        if (n < 0 || n > cap) {
            free(s);
            return ORC_ERR_CAPACITY;
        }
        for (int j = 0; j < n; ++j)
            s[j] = orc_idx_fp4_score(idx_q + (size_t)b * di,
                                     keys + ((size_t)b * cap + j) * row, di);
        if (scores_out) memcpy(scores_out + (size_t)b * cap, s, sizeof(int64_t) * (size_t)n);
        orc_topk64(s, n, c->topk, topk + (size_t)b * c->topk);
    }
    free(s);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* Hierarchical sparse indexer ([P2] part 4 "层级稀疏索引器：后面的层只在候选池
 * 里找"): after the first Full layer has scored every entry, the entries are
 * cut into blocks of `block` consecutive entries, each block scored by the
 * highest score inside it; the best `keep` blocks (2048 of 8 on the page)
 * form the candidate pool (16,384 entries) that later Reindex layers score
 * instead of the whole context.
 * Readings: the last block may be short (its visible entries only); blocks
 * are ranked like entries, (block score descending, block index ascending);
 * fewer than `keep` blocks means all of them.
 * blocks_out [keep]: chosen block indices ascending, -1 padded;
 * pool_out [keep * block]: their entries, ascending.  Returns the pool size. */
int orc_block_pool(const int32_t* scores, int n, int block, int keep,
                   int32_t* blocks_out, int32_t* pool_out) {
    int nb = (n + block - 1) / block;
    int32_t* bs = (int32_t*)malloc(sizeof(int32_t) * (size_t)(nb > 0 ? nb : 1));
    for (int i = 0; i < nb; ++i) {
        int32_t m = scores[(size_t)i * block];
        for (int j = i * block + 1; j < n && j < (i + 1) * block; ++j)
            if (scores[j] > m) m = scores[j];
        bs[i] = m;
    }
    int kept = orc_topk(bs, nb, keep, blocks_out);
    int pn = 0;
    for (int i = 0; i < kept; ++i)
        for (int j = blocks_out[i] * block; j < n && j < (blocks_out[i] + 1) * block; ++j)
            pool_out[pn++] = j;
    free(bs);
    return pn;
}

/* A Reindex layer over the pool: its own indexer query scores only the
 * pool's entries; top-K among them by (score descending, entry index
 * ascending), written ascending, -1 padded.  Returns the number kept.     */
int orc_pool_topk(const int8_t* q, const int8_t* keys, int di, const int32_t* pool,
                  int pool_n, int k, int32_t* out) {
    orc_scored* v = (orc_scored*)malloc(sizeof(orc_scored) * (size_t)(pool_n > 0 ? pool_n : 1));
    for (int p = 0; p < pool_n; ++p) {
        int32_t s = 0;
        for (int d = 0; d < di; ++d)
            s += (int32_t)q[d] * (int32_t)keys[(size_t)pool[p] * di + d];
        v[p].score = s;
        v[p].idx = pool[p];
    }
    qsort(v, (size_t)pool_n, sizeof(orc_scored), orc_by_score_desc_idx_asc);
    int kept = pool_n < k ? pool_n : k;
    for (int i = 0; i < kept; ++i) out[i] = v[i].idx;
    qsort(out, (size_t)kept, sizeof(int32_t), orc_int_asc);
    for (int i = kept; i < k; ++i) out[i] = -1;
    free(v);
    return kept;
}

/* ------------------------------------------------------------------ */
/* R5: decode attention for one query token, all heads, in fp64 ([P2]
 * breakthrough 2: heads share one 512+64 latent entry, values are the
 * latent; breakthrough 4: window + top-512 global branch).
 * q [H][D], keys [nk][D]; out [H][Dv]; lse [H] (natural log).
 * nk == 0 gives out = 0 and lse = -inf.                                 */
void orc_attention(const float* q, int H, int D, int Dv, const float* keys,
                   int nk, double sm_scale, double* out, double* lse) {
    double* s = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
    for (int h = 0; h < H; ++h) {
        double* o = out + (size_t)h * Dv;
        for (int d = 0; d < Dv; ++d) o[d] = 0.0;
        if (nk == 0) {
            lse[h] = -INFINITY;
            continue;
        }
        double m = -INFINITY;
        for (int j = 0; j < nk; ++j) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d)
                acc += (double)q[(size_t)h * D + d] * (double)keys[(size_t)j * D + d];
            s[j] = sm_scale * acc;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int j = 0; j < nk; ++j) {
            s[j] = exp(s[j] - m);
            l += s[j];
        }
        for (int j = 0; j < nk; ++j) {
            double p = s[j] / l;
            for (int d = 0; d < Dv; ++d) o[d] += p * (double)keys[(size_t)j * D + d];
        }
        lse[h] = m + log(l);
    }
    free(s);
}

/* Sparse decode attention for a batch: keys = dequantised records of the
 * selected entries (index -1 is padding and skipped) followed by the
 * window's window_len raw tokens.  Indices outside [0, n_entries[b]) are
 * skipped and reported through *status.
 * q [B][H][D]; records [B][cap][rb]; topk [B][K]; window [B][W][D];
 * out [B][H][Dv]; lse [B][H].                                           */
int orc_sparse_decode(const orc_cfg* c, int B, const float* q,
                      const uint8_t* records, int cap, const int32_t* n_entries,
                      const int32_t* topk, const float* window, int window_len,
                      double* out, double* lse, uint32_t* status) {
    int D = c->latent_dim + c->rope_dim, Dv = c->latent_dim, H = c->n_heads;
    int rb = orc_record_bytes(c, 1);
    if (window_len < 0 || window_len > c->window) return ORC_ERR_INVALID;
    float* keys = (float*)malloc(sizeof(float) * (size_t)(c->topk + c->window + 1) * D);
    for (int b = 0; b < B; ++b) {
        int nk = 0;
        for (int i = 0; i < c->topk; ++i) {
            int32_t j = topk[(size_t)b * c->topk + i];
            if (j == -1) continue;
            if (j < 0 || j >= n_entries[b]) {
                *status |= ORC_ST_BAD_INDEX;
                continue;
            }
            orc_dequantize_entry(c, records + ((size_t)b * cap + j) * rb, keys + (size_t)nk * D);
            ++nk;
        }
        for (int t = 0; t < window_len; ++t, ++nk)
            memcpy(keys + (size_t)nk * D, window + ((size_t)b * c->window + t) * D,
                   sizeof(float) * (size_t)D);
        orc_attention(q + (size_t)b * H * D, H, D, Dv, keys, nk, c->sm_scale,
                      out + (size_t)b * H * Dv, lse + (size_t)b * H);
    }
    free(keys);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* CSA2 layer group ([P2] part 4 "CSA2：三种模式，40 层只存 4 份"):
 *  Full    -- scores the stored cache with its own indexer q, own top-K;
 *  Reindex -- borrows the Full layer's stored main KV and indexer K and
 *             rescores with its own indexer q;
 *  Reuse   -- borrows the latest Full/Reindex layer's top-K indices.
 * Every layer has its own q and its own window.  All layers of the call
 * read the one stored cache (the Full layer's).  Arrays are layer-major:
 * q [L][B][H][D], idx_q [L][B][Di], windows [L][B][W][D],
 * out [L][B][H][Dv], lse [L][B][H], topk [L][B][K].                     */
/* hier_keep > 0 turns on the hierarchical indexer: every Full layer also
 * builds the block pool from its scores, and every Reindex layer after a
 * Full layer of the same call scores only that pool.                      */
int orc_group_step_hier(const orc_cfg* c, int n_layers, const int* modes, int B,
                        const float* q, const int8_t* idx_q, const float* windows,
                        int window_len, const uint8_t* records,
                        const int8_t* idx_cache, int cap, const int32_t* n_entries,
                        int hier_keep, int hier_block,
                        double* out, double* lse, int32_t* topk, uint32_t* status) {
    int D = c->latent_dim + c->rope_dim, Dv = c->latent_dim, H = c->n_heads;
    int K = c->topk, Di = c->idx_dim;
    if (n_layers < 1 || modes[0] == ORC_MODE_REUSE) return ORC_ERR_INVALID;
    if (hier_keep < 0 || (hier_keep > 0 && hier_block < 1)) return ORC_ERR_INVALID;
    size_t pool_cap = (size_t)(hier_keep > 0 ? hier_keep : 1) * (size_t)(hier_block > 0 ? hier_block : 1);
    int32_t* pool = (int32_t*)malloc(sizeof(int32_t) * (size_t)B * pool_cap);
    int32_t* pool_n = (int32_t*)calloc((size_t)B, sizeof(int32_t));
    int32_t* blocks = (int32_t*)malloc(sizeof(int32_t) * (size_t)(hier_keep > 0 ? hier_keep : 1));
    int32_t* sc = (int32_t*)malloc(sizeof(int32_t) * (size_t)(cap > 0 ? cap : 1));
    int have_pool = 0, rc = ORC_OK;
    int head = -1;
    for (int l = 0; l < n_layers && rc == ORC_OK; ++l) {
        int32_t* tk = topk + (size_t)l * B * K;
        const int8_t* ql = idx_q + (size_t)l * B * Di;
        if (modes[l] == ORC_MODE_FULL || (modes[l] == ORC_MODE_REINDEX && !have_pool)) {
            for (int b = 0; b < B && rc == ORC_OK; ++b) {
                int n = n_entries[b];
                if (n < 0 || n > cap) {
                    rc = ORC_ERR_CAPACITY;
                    break;
                }
                orc_index_scores(ql + (size_t)b * Di, idx_cache + (size_t)b * cap * Di, n, Di, sc);
                orc_topk(sc, n, K, tk + (size_t)b * K);
                if (hier_keep > 0 && modes[l] == ORC_MODE_FULL)
                    pool_n[b] = orc_block_pool(sc, n, hier_block, hier_keep, blocks,
                                               pool + (size_t)b * pool_cap);
            }
            if (hier_keep > 0 && modes[l] == ORC_MODE_FULL) have_pool = 1;
            head = l;
        } else if (modes[l] == ORC_MODE_REINDEX) {
            for (int b = 0; b < B; ++b)
                orc_pool_topk(ql + (size_t)b * Di, idx_cache + (size_t)b * cap * Di, Di,
                              pool + (size_t)b * pool_cap, pool_n[b], K, tk + (size_t)b * K);
            head = l;
        } else if (modes[l] == ORC_MODE_REUSE) {
            memcpy(tk, topk + (size_t)head * B * K, sizeof(int32_t) * (size_t)B * K);
        } else {
            rc = ORC_ERR_INVALID;
            break;
        }
        if (rc == ORC_OK)
            rc = orc_sparse_decode(c, B, q + (size_t)l * B * H * D, records, cap, n_entries, tk,
                                   windows + (size_t)l * B * c->window * D, window_len,
                                   out + (size_t)l * B * H * Dv, lse + (size_t)l * B * H, status);
    }
    free(pool);
    free(pool_n);
    free(blocks);
    free(sc);
    return rc;
}

int orc_group_step(const orc_cfg* c, int n_layers, const int* modes, int B,
                   const float* q, const int8_t* idx_q, const float* windows,
                   int window_len, const uint8_t* records,
                   const int8_t* idx_cache, int cap, const int32_t* n_entries,
                   double* out, double* lse, int32_t* topk, uint32_t* status) {
    return orc_group_step_hier(c, n_layers, modes, B, q, idx_q, windows, window_len, records,
                               idx_cache, cap, n_entries, 0, 0, out, lse, topk, status);
}

/* ------------------------------------------------------------------ */
/* Bytes resident for one sequence ([P2] "890 字节是怎么算出来的": count
 * the FP4 main entry with its scales plus the indexer key): stored
 * records (padded to the record stride, or not) + int8 indexer rows +
 * every layer's own window of raw keys.                                 */
uint64_t orc_bytes_resident(const orc_cfg* c, int64_t entries, int n_layers,
                            int window_elem_bytes, int padded) {
    int64_t D = c->latent_dim + c->rope_dim;
    return (uint64_t)(entries * orc_record_bytes(c, padded) + entries * c->idx_dim +
                      (int64_t)n_layers * c->window * D * window_elem_bytes);
}
