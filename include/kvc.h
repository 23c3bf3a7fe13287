/*
 * kvc.h -- C ABI of the compressed-KV sparse decode library (libkvc.so).
 *
 * The library implements, on one B200 GPU (sm_100a), the decode hot path of
 * attention over a KV cache whose entries are compressed 2:1 across tokens
 * and stored as FP4 E2M1 with per-group scales, as described on two pages:
 *
 *  [A] "DeepSeek V1 到 V4.1-Flash，单 token 的 global KV 如何从 389,000 B 压缩到
 *      890 B的？" (acejoy.com) -- part 3 breakthrough 2 (MLA entry: 512 latent
 *      + 64 RoPE channels shared by all heads), breakthrough 4 (128-token
 *      sliding window; a lightweight indexer scores all history and keeps the
 *      top 512; CSA compresses every 2 tokens into 1 entry), part 4 "CSA2：三种
 *      模式" (Full / Reindex / Reuse layers), "P4 main KV" (E2M1 with shared
 *      scales, dequantised before attention), "890 字节是怎么算出来的".
 *  [B] "DeepSeek V4.1 Flash KV Cache压缩实战：FP4+CSA2+CED将显存降至1/4"
 *      (gtnt.cn) -- 3.1 (FP4 group quantisation), 3.2 (2:1 key compressor),
 *      4.3 (group size 32/64/128, ratio 2x).
 *
 * Conventions shared by every call
 *  - Every pointer argument except `cfg`, `cache` and host arrays named as
 *    such is a DEVICE pointer on the current CUDA device.  The caller owns all
 *    memory; the library never allocates device memory, never frees, and never
 *    synchronises.  Work is enqueued on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and the call returns before it runs.
 *  - Host-detectable errors (bad configuration, null or misaligned pointers,
 *    sizes out of range, workspace too small) return a kvc_status before
 *    anything is enqueued.  A failed launch returns KVC_ERR_CUDA.
 *  - Anomalies only the device can see are OR-ed into `*dev_status` (a device
 *    uint32; may be NULL) as KVC_DEV_* bits; read it after the stream
 *    synchronises.  Kernels never trap, and every wait inside a kernel is
 *    bounded: when a bound is hit the kernel sets KVC_DEV_TIMEOUT and returns.
 *  - Records and token/query/window rows must start on 16-byte boundaries.
 *  - Kernels are launched as programmatic dependents of the kernel before
 *    them on the stream and wait for it to complete (griddepcontrol.wait)
 *    before reading anything a kernel may have written.  One exception:
 *    kvc_pack reads its tokens, gate and idx_k_new before that wait, while
 *    the previous kernel may still be finishing.  Ordinary kernels (which
 *    never execute griddepcontrol.launch_dependents) have completed before
 *    it starts, so this needs nothing; a caller's kernel that does signal
 *    launch_dependents must do so after its last write of those inputs.
 */
#ifndef KVC_H
#define KVC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KVC_OK = 0,
    KVC_ERR_INVALID = 1,     /* bad argument or configuration                */
    KVC_ERR_CAPACITY = 2,    /* a size exceeds what the buffers or kernel hold */
    KVC_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed          */
    KVC_ERR_UNSUPPORTED = 4, /* valid but not implemented for this shape      */
    KVC_ERR_TIMEOUT = 5,
    KVC_ERR_DEVICE = 6,      /* no sm_100 device current                      */
    KVC_ERR_WORKSPACE = 7    /* workspace pointer null, misaligned or too small */
} kvc_status;

typedef enum { KVC_SCALE_F32 = 0, KVC_SCALE_UE4M3 = 1 } kvc_scale_fmt;
typedef enum { KVC_FULL = 0, KVC_REINDEX = 1, KVC_REUSE = 2 } kvc_mode;
typedef enum { KVC_F32 = 0, KVC_BF16 = 1 } kvc_dtype;

/* device status bits */
#define KVC_DEV_NONFINITE 0x1u  /* a NaN/Inf input: a pack channel (coded as 0)
                                   or an attention query row                   */
#define KVC_DEV_BAD_INDEX 0x2u  /* a top-K index outside [-1, n_entries)       */
#define KVC_DEV_CAPACITY 0x4u   /* pack would pass the cache capacity          */
#define KVC_DEV_TIMEOUT 0x8u    /* a bounded in-kernel wait gave up            */
#define KVC_DEV_BAD_LENGTH 0x10u /* n_entries outside [0, capacity]            */

/* Shape and format of one compressed cache and its decode attention.
 *  latent_dim  Dv, latent channels; also the value width ([A] breakthrough 2: 512)
 *  rope_dim    RoPE channels appended to every key ([A]: 64); D = latent + rope
 *  group       FP4 group size G ([B] 4.3: 32/64/128); latent and RoPE are grouped
 *              separately and the last RoPE group may be short
 *  scale_fmt   per-group scale: fp32, or unsigned E4M3 (one byte)
 *  idx_dim     int8 indexer key width Di ([A] "890 字节": 128)
 *  topk        K entries kept by the indexer ([A] breakthrough 4: 512)
 *  window      W, sliding-window length ([A] breakthrough 4: 128)
 *  n_heads     H query heads sharing each entry
 *  sm_scale    softmax scale applied to q.k
 *  act_dtype   dtype of raw tokens, queries and window keys (fp32 or bf16)   */
typedef struct {
    int32_t latent_dim, rope_dim, group, scale_fmt;
    int32_t idx_dim, topk, window, n_heads;
    float sm_scale;
    int32_t act_dtype;
    int32_t ratio;   /* raw tokens per entry: 2 (0 also means 2) or 4 */
    int32_t idx_fmt; /* indexer keys: 0 = int8 rows of idx_dim bytes; 1 = FP4 rows of
                        idx_dim/2 E2M1 code bytes (channel 2c in the low nibble of
                        byte c) then idx_dim/16 UE4M3 scales, one per 16 channels
                        -- the 72-byte indexer K of [A] "890 字节是怎么算出来的" at
                        128 channels */
} kvc_config;

/* One stored cache (the Full layer's).  Caller-owned device buffers:
 *  records    [batch][capacity][kvc_record_bytes(cfg)] bytes, 16-byte aligned.
 *             Record = [D/2 bytes of E2M1 codes, channel 2c in the low nibble of
 *             byte c][one scale per group, in group order: 1 byte UE4M3 or 4
 *             bytes fp32][zero padding to a multiple of 16 bytes]
 *  idx_k      [batch][capacity][kvc_idx_row_bytes(cfg)] indexer keys (int8
 *             values, or FP4 rows when cfg->idx_fmt = 1)
 *  n_entries  [batch] int32, entries stored per sequence (visible to the
 *             indexer: entries 0 .. n_entries-1)                            */
typedef struct {
    void* records;
    int8_t* idx_k;
    int32_t* n_entries;
    int32_t batch, capacity;
} kvc_cache;

/* Bytes of one record (with padding) = the record stride. 0 if cfg invalid. */
size_t kvc_record_bytes(const kvc_config* cfg);

/* Bytes of one indexer row in the cache: idx_dim (int8 keys) or idx_dim/2 +
 * idx_dim/16 (FP4 keys, idx_fmt = 1).  0 if cfg invalid. */
size_t kvc_idx_row_bytes(const kvc_config* cfg);

/* Bytes resident per sequence for `entries` stored entries and `n_layers`
 * layers each holding its own window of W raw keys (record bytes with or
 * without padding + indexer rows + windows) -- the per-token accounting of
 * [A] "890 字节是怎么算出来的" applied to this cache. 0 if cfg invalid.      */
size_t kvc_bytes_resident(const kvc_config* cfg, int64_t entries, int n_layers,
                          int padded);

/* Device workspace needed by kvc_index_topk, kvc_sparse_decode_attn and
 * kvc_layer_group_step for `batch` sequences of up to `capacity` entries.
 * Every workspace (this one, the hierarchical and the batched ones) must be
 * zero-filled before its first use (for example with cudaMemset): the top-K
 * counters in it start at zero, and every call leaves them at zero again, so
 * no call spends a launch clearing them.  After a call that set
 * KVC_DEV_TIMEOUT in the status word, zero the workspace again.  Nothing
 * else in it needs initialisation.                                         */
size_t kvc_workspace_bytes(const kvc_config* cfg, int batch, int capacity);

/* Append n_new raw tokens per sequence (A1-A3 of the hot path).
 * tokens    [batch][n_new][D] act_dtype; n_new a multiple of r = cfg->ratio:
 *           tokens r i .. r i + r - 1 are compressed into entry i ([A]
 *           breakthrough 4: the trained compressor merges every two tokens
 *           into one cache entry; [B] 3.2; the
 *           ratio 4 of [B] 4.3).  The tokens' weights are the softmax of their
 *           gate logits g.k; the weighted sum is quantised per group to E2M1
 *           with scale absmax/6 ([B] 3.1; [A] "P4 main KV").
 * gate      [D] fp32 gate vector g.
 * idx_k_new [batch][n_new/r][idx_dim] indexer keys of the new entries: int8
 *           (idx_fmt = 0), or act_dtype values (idx_fmt = 1) quantised to FP4
 *           rows like a record of idx_dim channels with groups of 16 and UE4M3
 *           scales (absmax/6, round to nearest even).
 * Entries are written at positions n_entries[b] .. n_entries[b]+n_new/r-1 and
 * n_entries[b] then advances by n_new/r.  If that would pass the capacity the
 * sequence is left unchanged and KVC_DEV_CAPACITY is set.  NaN/Inf channels are
 * coded 0, left out of the group maximum, and set KVC_DEV_NONFINITE.  Long
 * bf16 appends stream the tokens through shared memory with bounded waits; if
 * one gives up (KVC_DEV_TIMEOUT) n_entries still advances but some of the new
 * entries may be unwritten: set n_entries back and append them again.        */
kvc_status kvc_pack(const kvc_config* cfg, const void* tokens, int n_new,
                    const float* gate, const int8_t* idx_k_new,
                    const kvc_cache* cache, uint32_t* dev_status, void* stream);

/* Indexer scoring and exact top-K (A4-A5; [A] breakthrough 4: a light indexer
 * scores every stored entry and the 512 best are attended; part 4 "CSA2").
 * idx_q     [batch][idx_dim] int8 indexer queries.
 * score_j = sum_d idx_q[d] * idx_k[j][d] in int32 over the visible entries.
 * topk_idx  [batch][topk] int32 out: the topk highest scores, ties to the lower
 *           index, written in ascending index order; -1 pads when fewer than
 *           topk entries are visible.
 * scores    [batch][capacity] int32 out, or NULL; when given it receives every
 *           visible score (positions past n_entries are not written).
 * ws        device workspace of at least kvc_workspace_bytes(cfg, batch,
 *           capacity) bytes, 256-byte aligned, zero-filled before its first
 *           use (see kvc_workspace_bytes).
 * capacity must not exceed 8,388,608 entries (KVC_ERR_CAPACITY).
 * FP4 indexer keys (idx_fmt = 1): the score of an entry is the exact value of
 * idx_q . dequant(k) (an integer multiple of 2^-10, held in 64 bits), the
 * selection as above; `scores` must be NULL (KVC_ERR_UNSUPPORTED).  The
 * hierarchical, batched and fixed-scratch variants take int8 keys only.         */
kvc_status kvc_index_topk(const kvc_config* cfg, const int8_t* idx_q,
                          const kvc_cache* cache, int32_t* topk_idx,
                          int32_t* scores, void* ws, size_t ws_bytes,
                          uint32_t* dev_status, void* stream);

/* kvc_index_topk without a workspace argument, for callers that cannot
 * allocate device memory: a plugin whose host framework owns every device
 * allocation and passes it only its inputs and outputs, or a latency-critical
 * path where cudaMalloc's implicit device synchronisation is not allowed.  The
 * pages have no counterpart of this call; it computes exactly what
 * kvc_index_topk computes (same kernels, same results).
 * Its scratch (scores, histograms, counters, candidate lists) is a fixed
 * array inside the library, about 10.5 MiB, held on every GPU that loads the
 * library until the process exits.  Limits: batch <= 64 and
 * batch * capacity <= 524,288 entries; larger problems return
 * KVC_ERR_CAPACITY before anything is enqueued.  The call allocates nothing.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call shares the one array: its counters start at zero
 * (a static array) and every call leaves them at zero, but calls whose work
 * overlaps on the GPU (different streams, or different host threads on one
 * device) race on it, and after a call that set KVC_DEV_TIMEOUT the array
 * stays unusable until the process exits.  The looked-up address is kept for
 * the life of the process: after anything that destroys the device's primary
 * context (cudaDeviceReset, a framework tearing the context down) it no
 * longer points at the array, and this entry point must not be called on
 * that device again.                                                     */
kvc_status kvc_index_topk_noalloc(const kvc_config* cfg, const int8_t* idx_q,
                                  const kvc_cache* cache, int32_t* topk_idx,
                                  int32_t* scores, uint32_t* dev_status,
                                  void* stream);

/* Several indexer queries per sequence scored in one pass over the cache
 * (the lightweight indexer of [A] breakthrough 4 for all the Full and
 * Reindex layers of a CSA2 stack at once, part 4 "CSA2：三种模式").  Valid
 * only where every query is known before the pass (a verification or prefill
 * schedule, or a stack whose indexer queries do not depend on earlier
 * layers); it computes exactly what nq calls of kvc_index_topk compute.  The
 * scores are one tensor-core product per 128-row tile (int8 x int8 -> int32,
 * tcgen05 kind::i8 with the queries as the N = 16 side), read once from HBM.
 * idx_q     [nq][batch][idx_dim] int8, 1 <= nq <= 8; idx_dim must be 128
 *           (else KVC_ERR_UNSUPPORTED).
 * topk_idx  [nq][batch][topk] int32, as kvc_index_topk's output per query.
 * ws        kvc_workspace_bytes_batched(cfg, nq, batch, capacity) bytes,
 *           256-byte aligned, zero-filled before its first use.           */
size_t kvc_workspace_bytes_batched(const kvc_config* cfg, int nq, int batch,
                                   int capacity);
kvc_status kvc_index_topk_batched(const kvc_config* cfg, int nq,
                                  const int8_t* idx_q, const kvc_cache* cache,
                                  int32_t* topk_idx, void* ws, size_t ws_bytes,
                                  uint32_t* dev_status, void* stream);

/* Sparse decode attention (A6-A10; [A] breakthrough 2 and 4, "P4 main KV").
 * q         [batch][n_heads][D] act_dtype queries (already in latent space).
 * topk_idx  [batch][topk] int32 selected entries; -1 entries are skipped, any
 *           other index outside [0, n_entries[b]) is skipped and sets
 *           KVC_DEV_BAD_INDEX.
 * window    [batch][window][D] act_dtype raw keys of the sliding window; the
 *           first window_len (0 <= window_len <= cfg->window) rows are used.
 * One softmax runs jointly over the dequantised selected entries and the
 * window keys; values are the first latent_dim channels of each key.
 * out       [batch][n_heads][latent_dim] fp32; lse [batch][n_heads] fp32
 *           natural-log sum of exp of the scaled logits, or NULL.  With no key
 *           at all the output row is 0 and lse is -inf.                   */
kvc_status kvc_sparse_decode_attn(const kvc_config* cfg, const void* q,
                                  const kvc_cache* cache, const int32_t* topk_idx,
                                  const void* window, int window_len, float* out,
                                  float* lse, void* ws, size_t ws_bytes,
                                  uint32_t* dev_status, void* stream);

/* FP8 window rows ([A] part 4 "P4 main KV": the sliding-window KV stays in
 * FP8; the pages give no scale layout, so this build keeps one fp32 scale
 * per row).  rows [n_rows][D] act_dtype -> codes [n_rows][D] signed E4M3
 * bytes and scales [n_rows] fp32 = absmax / 448 over the row's finite
 * elements; each code is x / scale rounded to nearest even, saturating at
 * 448, a magnitude of zero stored as +0; non-finite elements are coded 0 and
 * set KVC_DEV_NONFINITE.  rows 16-byte, codes 8-byte aligned.             */
kvc_status kvc_pack_window_fp8(const kvc_config* cfg, const void* rows,
                               int64_t n_rows, uint8_t* codes, float* scales,
                               uint32_t* dev_status, void* stream);

/* kvc_sparse_decode_attn with the window in FP8: win_codes [batch][window][D]
 * signed E4M3 (16-byte aligned), win_scales [batch][window] fp32, as written
 * by kvc_pack_window_fp8; each window key is E4M3(code) x scale.  D must be
 * a multiple of 16.  Everything else as kvc_sparse_decode_attn.           */
kvc_status kvc_sparse_decode_attn_fp8win(const kvc_config* cfg, const void* q,
                                         const kvc_cache* cache,
                                         const int32_t* topk_idx,
                                         const uint8_t* win_codes,
                                         const float* win_scales, int window_len,
                                         float* out, float* lse, void* ws,
                                         size_t ws_bytes, uint32_t* dev_status,
                                         void* stream);

/* One decode step through a CSA2 layer group (A11; [A] part 4 "CSA2：三种模式，
 * 40 层只存 4 份"): layers run in order on `stream`.
 *  Full    -- indexer top-K with its own idx_q over `cache`, then attention;
 *  Reindex -- same over the Full layer's stored cache and keys, own idx_q;
 *  Reuse   -- attention with the top-K of the latest Full/Reindex layer.
 * Every layer uses its own q and window.  modes is a HOST array of n_layers
 * kvc_mode values; modes[0] must be Full or Reindex.  Device arrays are
 * layer-major: q [L][batch][H][D], idx_q [L][batch][Di], windows
 * [L][batch][W][D], out [L][batch][H][Dv], lse [L][batch][H] (or NULL),
 * topk [L][batch][K] (receives every layer's indices; Reuse layers get a copy
 * of their head's).                                                       */
kvc_status kvc_layer_group_step(const kvc_config* cfg, int n_layers,
                                const int32_t* modes, const void* q,
                                const int8_t* idx_q, const void* windows,
                                int window_len, const kvc_cache* cache,
                                float* out, float* lse, int32_t* topk, void* ws,
                                size_t ws_bytes, uint32_t* dev_status,
                                void* stream);

/* The layer group step with the hierarchical sparse indexer ([A] part 4
 * "层级稀疏索引器：后面的层只在候选池里找"): every Full layer, after its own
 * top-K, cuts its scored entries into blocks of `hier_block` consecutive
 * entries (8 on the page), scores each block by its best entry and keeps the
 * best `hier_blocks` blocks (2048 on the page; ties to the lower block,
 * written ascending); every later Reindex layer of the call scores only that
 * pool (16,384 entries on the page) with its own indexer query and keeps its
 * top-K among them (ties to the lower entry index).  A Reindex layer before
 * any Full layer scores the whole cache.  The last block of a sequence may be
 * short.  hier_blocks = 0 is kvc_layer_group_step; otherwise
 * 1 <= hier_blocks <= 65536 and 1 <= hier_block <= 256 (else
 * KVC_ERR_INVALID).  ws must hold kvc_workspace_bytes_hier(cfg, batch,
 * capacity, hier_blocks, hier_block) bytes; all other arguments as in
 * kvc_layer_group_step.                                                     */
size_t kvc_workspace_bytes_hier(const kvc_config* cfg, int batch, int capacity,
                                int hier_blocks, int hier_block);
kvc_status kvc_layer_group_step_hier(const kvc_config* cfg, int hier_blocks,
                                     int hier_block, int n_layers,
                                     const int32_t* modes, const void* q,
                                     const int8_t* idx_q, const void* windows,
                                     int window_len, const kvc_cache* cache,
                                     float* out, float* lse, int32_t* topk,
                                     void* ws, size_t ws_bytes,
                                     uint32_t* dev_status, void* stream);

/* E2M1 / E4M3 codecs as the pack kernel applies them (format utilities).
 * kvc_e2m1_encode: x [n] fp32 -> codes [n] uint8 (0..15), round to nearest
 * even on the grid {0, 0.5, 1, 1.5, 2, 3, 4, 6}, saturating, -0 stored as 0.
 * kvc_e4m3_encode: x [n] fp32 >= 0 -> bytes [n], round to nearest even,
 * saturating at 448.                                                       */
kvc_status kvc_e2m1_encode(const float* x, int64_t n, uint8_t* codes, void* stream);
kvc_status kvc_e4m3_encode(const float* x, int64_t n, uint8_t* bytes, void* stream);

/* Tracing.  Between kvc_trace_begin and kvc_trace_end every kernel the
 * library enqueues is bracketed by a pair of CUDA events (at most
 * max_launches launches are recorded).  kvc_trace_kernel, called after the
 * traced work has completed, returns the number of recorded launches of the
 * kernel named `name` and their summed device time in milliseconds.  Names:
 * "pack", "pack_idx", "pack_commit", "window_fp8", "index_scan",
 * "index_scan_tc", "index_scan_fp4", "topk_select", "topk_select_fp4",
 * "block_max", "copy_topk", "attn_t128", "attn_simt", "attn_merge",
 * "fp4_codec".  Every enqueuing entry point also opens an NVTX range named
 * after itself for the duration of the call (a no-op without a profiler).  */
kvc_status kvc_trace_begin(int max_launches);
kvc_status kvc_trace_end(void);
kvc_status kvc_trace_kernel(const char* name, int* launches, double* total_ms);

/* TEST HOOK, not for production use.  Sets the bound on each in-kernel wait
 * (mbarrier phases of the bulk-copy ring and of the tensor-core products) of
 * every kernel enqueued after this call, in nanoseconds of %globaltimer; the
 * library starts with 2,000,000,000 (2 s).  0 makes every such wait a single
 * non-blocking poll, so a kernel reaches its timeout path at once: it sets
 * KVC_DEV_TIMEOUT, waits (with the normal 2 s bound) for the copies and
 * products it already issued, frees its tensor memory and returns normally.
 * After such a call the top-K counters in the workspace are left dirty and
 * the outputs are undefined: zero the workspace before the next call.  The
 * value is read when a kernel is enqueued (a captured graph keeps the value
 * it was captured with).  Not thread-safe with concurrent enqueues.        */
kvc_status kvc_debug_set_wait_limit_ns(uint64_t ns);

/* Number of kernels the library has enqueued since it was loaded. */
uint64_t kvc_launch_count(void);

const char* kvc_status_string(kvc_status s);
const char* kvc_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KVC_H */
