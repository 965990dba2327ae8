/*
 * kvq.h -- C ABI of libkvq: quantised KV cache and single-token decode
 * attention on NVIDIA B200 (sm_100a).
 *
 * Scope.  The library implements the hot path the source pages describe:
 *   - quantize-on-append of keys and values (or of the hidden state h in
 *     h-mode) into a fixed-capacity cache with INT8 or nibble-packed INT4
 *     codes and fp16 scales, independent key/value bit-widths;
 *   - split-KV decode attention that dequantises in registers inside
 *     q.K^T -> online softmax -> P.V and merges the partials;
 *   - in h-mode, the K/V reconstruction GEMM K = W_k h, V = W_v h on tensor
 *     cores, followed by the same decode attention over 16-bit K/V.
 *
 * Sources (web pages; cited by title and section):
 *   [TL]  TinyLoop docs, "KV Cache 模式": the five cache modes table, the
 *         memory-formula table "記憶體公式", and "運作原理" (how h-mode works).
 *   [KS]  KVSplit (vi.news.hada.io topic 20969): independent key/value
 *         precision K8V8/K8V4/K4V8/K4V4 ("Tính năng chính", flags --kvq-key,
 *         --kvq-val) and the 8K-token memory table.
 *   [MNI] "kv-cache-int8-35x-speedup-rust-cuda" (mni-ml/framework): KV cache
 *         keeps past K/V and computes one new K/V per step; INT8 KV.
 *   [OD]  gyaansetu.com on-device LLM page: INT4 keys with INT8 values; a
 *         sliding window of recent tokens plus anchor tokens.
 *
 * Conventions for every call:
 *   Ownership.  The caller allocates every buffer (cache, inputs, outputs,
 *     workspace, h-mode scratch) in device memory.  The library never
 *     allocates or frees memory and keeps no state between calls.
 *   Alignment.  Every device pointer must be 16-byte aligned.
 *   Asynchrony.  Calls that take a stream only enqueue work on it and return;
 *     a device fault shows up at the caller's next synchronisation.
 *   Errors.  Every call returns KVQ_OK (0) or a negative KVQ_ERR_* status,
 *     checks its arguments on the host before launching anything, and never
 *     aborts or throws.  Non-finite input values give unspecified codes.
 *   Layout.  "Row" below means one token of one KV head: head_dim elements.
 *     bits 8: head_dim bytes of int8 codes (two's complement).
 *     bits 4: head_dim/2 bytes; element 2j in the low nibble and 2j+1 in the
 *             high nibble of byte j, 4-bit two's complement.
 *     bits 16: head_dim fp16 values, no scales.
 *     Scales: head_dim/group fp16 values per row.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream).  NULL is the legacy default stream. */
typedef struct CUstream_st *kvq_stream_t;

enum kvq_status {
    KVQ_OK = 0,
    KVQ_ERR_INVALID_ARG = -1,  /* null pointer, bad size, bad dtype          */
    KVQ_ERR_UNSUPPORTED = -2,  /* bit-width / group / head-shape combination */
    KVQ_ERR_CAPACITY = -3,     /* position or length beyond the capacity     */
    KVQ_ERR_ALIGN = -4,        /* a pointer is not 16-byte aligned           */
    KVQ_ERR_WORKSPACE = -5,    /* workspace or scratch too small             */
    KVQ_ERR_LAUNCH = -6,       /* the CUDA launch itself failed              */
    KVQ_ERR_DEVICE = -7,       /* no usable sm_100 device / attribute query  */
    KVQ_ERR_TIMEOUT = -8       /* a kernel gave up a bounded wait (see
                                  kvq_workspace_status)                       */
};

enum kvq_mode {
    KVQ_MODE_KV = 0,  /* the cache stores quantised K and V                  */
    KVQ_MODE_H = 1    /* the cache stores quantised h = LN(residual) [TL]    */
};

enum kvq_format {
    KVQ_FMT_INT = 0,    /* signed integer codes (INT8 / INT4), symmetric scales     */
    KVQ_FMT_E4M3 = 1,   /* FP8 e4m3 codes, 8 bits                                   */
    KVQ_FMT_ASYM = 2,   /* asymmetric INT8: uint8 codes, scale + zero-point         */
    KVQ_FMT_TENSOR = 3  /* per-tensor INT8: one caller-set scale per K / V tensor   */
};

enum kvq_dtype {
    KVQ_F16 = 0,
    KVQ_F32 = 1,
    KVQ_BF16 = 2
};

/* Shape and format of a cache.  [TL] "記憶體公式": a cache has a capacity
 * max_seq_len fixed at creation and n_layers cached-attention layers; the
 * mode is chosen before use.  [KS]: key and value bit-widths are independent. */
typedef struct kvq_config {
    int32_t mode;        /* KVQ_MODE_KV or KVQ_MODE_H                             */
    int32_t batch;       /* sequences B                                           */
    int32_t capacity;    /* tokens per sequence; a multiple of 16                 */
    int32_t n_layers;    /* used by kvq_cache_bytes only                          */
    int32_t n_q_heads;   /* Hq                                                    */
    int32_t n_kv_heads;  /* Hkv; Hq is a multiple of Hkv, G = Hq/Hkv              */
    int32_t head_dim;    /* Dh: 64 or 128                                         */
    int32_t k_bits;      /* KV mode: 4, 8 or 16                                   */
    int32_t v_bits;      /* KV mode: 4, 8 or 16                                   */
    int32_t k_group;     /* elements per key scale: 32, 64 or 128, dividing Dh;
                            == Dh means one scale per (token, head)               */
    int32_t v_group;     /* same for values                                       */
    int32_t d_model;     /* h-mode: D = n_kv_heads * head_dim                     */
    int32_t h_bits;      /* h-mode: 4, 8 or 16                                    */
    int32_t h_groups;    /* h-mode: fp16 scales per token (the "per-head" scales
                            of [TL]); D / h_groups must be 32, 64 or 128          */
    int32_t window;      /* KV mode, 0 or a sliding window ([OD] "1536 recent + 64
                            anchors"): the cache keeps the first n_anchor tokens
                            and a ring of the most recent `window` tokens, and
                            capacity must equal n_anchor + window.  Token t (0-
                            based, counted over the whole sequence) lives in slot
                            t while t < n_anchor, else in slot n_anchor +
                            (t - n_anchor) mod window.  0: no window, slot t.     */
    int32_t n_anchor;    /* KV mode with a window: anchor tokens kept for good    */
    int32_t page_tokens; /* KV mode: 0 (each sequence owns `capacity` contiguous
                            slots) or 128: paged cache.  The layer's buffers are a
                            pool of n_pages pages of 128 tokens, [n_pages][Hkv]
                            [128][...], and kvq_layer.block_table maps logical page
                            j of sequence b (tokens 128j .. 128j+127) to a pool
                            page; capacity (a multiple of 128) is then the
                            logical tokens per sequence.  No sliding window.      */
    int32_t n_pages;     /* paged cache: pages in each layer's pool               */
    int32_t kv_format;   /* KV mode, k_bits = v_bits = 8 for every format but INT:
                            KVQ_FMT_INT: symmetric integer codes (above).
                            KVQ_FMT_E4M3: FP8 e4m3 codes, scale s = fp16(absmax /
                            448) per group, code = e4m3_rne(x / s) saturating at
                            448, value = e4m3(code) * s ([MNI] "Comparison với
                            production stack": FP8 KV caches of vLLM and
                            TensorRT-LLM).
                            KVQ_FMT_ASYM: per group lo = min(0, min x), hi =
                            max(0, max x), s = fp16((hi - lo) / 255), zero-point
                            z = clamp(rne(-lo / s), 0, 255), code = clamp(rne(x /
                            s) + z, 0, 255) stored as uint8, value = (code - z) *
                            s; each group keeps the fp16 pair (s, z) ([MNI] "Tại
                            sao INT8 mà không mất tốc": scale/zero-point metadata).
                            KVQ_FMT_TENSOR: one fp16 scale s per K tensor and one
                            per V tensor of a layer, set by the caller in
                            k_scales[0] / v_scales[0] before the first append
                            (e.g. from calibration) and never written by the
                            library; code = clamp(rne(x / s), -127, 127), value =
                            code * s ([MNI] "Limitations": symmetric per-tensor
                            INT8); k_group = v_group = head_dim.                 */
} kvq_config;

/* One layer's cache buffers (device pointers, caller-owned).
 * KV mode:  k_codes  [B][Hkv][capacity][Dh*k_bits/8] bytes
 *           k_scales [B][Hkv][capacity][Dh/k_group] fp16   (NULL at 16 bits)
 *           v_codes / v_scales likewise with v_bits, v_group.
 *           KVQ_FMT_ASYM: k_scales [B][Hkv][capacity][Dh/k_group][2] fp16
 *           (scale, zero-point) pairs.  KVQ_FMT_TENSOR: k_scales and v_scales
 *           each hold one fp16 scale (caller-set, 16-byte aligned).
 *           Paged (page_tokens 128): [n_pages][Hkv][128][...] for each of them,
 *           logical token t of sequence b at slot t % 128 of pool page
 *           block_table[b][t / 128].
 * h-mode:   k_codes  [B][capacity][D*h_bits/8] bytes  (the h codes)
 *           k_scales [B][capacity][h_groups] fp16      (NULL at 16 bits)
 *           v_codes = v_scales = NULL. */
typedef struct kvq_layer {
    void *k_codes;
    void *k_scales;
    void *v_codes;
    void *v_scales;
    const int32_t *block_table;  /* paged cache: device int32 [B][capacity/128], the
                                    pool page of each logical page (entries in
                                    [0, n_pages)); NULL otherwise.  The same table
                                    usually serves every layer. */
} kvq_layer;

/* Cache size.  [TL] "記憶體公式": bytes per token per layer are, at
 * D = 2048 and 16 heads, 8192 (FP16 KV), 4160 (INT8 KV), 4096 (FP16 h),
 * 2080 (INT8 h), 1056 (INT4 h); the whole cache costs that times
 * n_layers * max_seq_len.  Generalised here to separate K/V widths and
 * scale groups ([KS] 8K-token table):
 *   KV mode: sum over K and V of Hkv*Dh*bits/8 + Hkv*(Dh/group)*2 (no scale
 *            term at 16 bits; *4 with a zero-point (KVQ_FMT_ASYM); per-tensor
 *            scales are no per-token term, 4 bytes per layer);
 *   h-mode: D*h_bits/8 + h_groups*2 (none at 16).
 * Outputs (any may be NULL): bytes per token per layer, per layer
 * (x batch x capacity, or x n_pages x 128 for a paged cache) and total
 * (x n_layers).  Pure host function: no GPU needed.  Errors:
 * KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED for a bad config. */
KVQ_API int kvq_cache_bytes(const kvq_config *cfg, uint64_t *per_token_layer, uint64_t *per_layer,
                    uint64_t *total);

/* Sizes of the four buffers of one layer in bytes (any output may be NULL;
 * an unused buffer reports 0).  Pure host function. */
KVQ_API int kvq_layer_buffer_bytes(const kvq_config *cfg, uint64_t *k_codes, uint64_t *k_scales,
                           uint64_t *v_codes, uint64_t *v_scales);

/* Quantize-on-append.  [MNI] "Cách KV cache tạo ra tốc độ": each step computes
 * only the new tokens' K and V and keeps the old ones; [TL] mode table: INT8
 * codes with one fp16 scale per head, INT4 nibble-packed ("255" vs "15"
 * symmetric levels); [KS]/[OD]: keys and values at their own widths.
 *
 * For every sequence b, new token j < n_new and KV head, each group of
 * `group` elements x is quantised as
 *   s = fp16_rne(max|x| / qmax)   (IEEE fp32 division; qmax 127 or 7;
 *                                  +inf saturates to 65504)
 *   code = clamp(rne(x / s), -qmax, qmax)   (IEEE fp32 division; 0 if s == 0)
 * and stored at position d_pos[b] + j.  At 16 bits the value is stored as
 * fp16 (round to nearest even).
 *   k, v     device, [B][n_new][Hkv][Dh] in in_dtype (h-mode: k = h,
 *            [B][n_new][D], and v must be NULL)
 *   in_dtype KVQ_F16, KVQ_F32 or KVQ_BF16
 *   d_pos    device int32 [B]: first position written for each sequence
 *   max_pos_host  host-side upper bound of d_pos[]: the call fails with
 *            KVQ_ERR_CAPACITY if max_pos_host + n_new > capacity.  Rows whose
 *            device position still falls outside [0, capacity) are skipped.
 *   n_new    tokens per sequence (0 is a no-op).
 * Errors: INVALID_ARG, UNSUPPORTED, CAPACITY, ALIGN, LAUNCH. */
KVQ_API int kvq_append(const kvq_config *cfg, const kvq_layer *layer, const void *k, const void *v,
               int32_t in_dtype, const int32_t *d_pos, int32_t max_pos_host, int32_t n_new,
               kvq_stream_t stream);

/* Workspace bytes kvq_decode_attn needs for this config (KV mode, or the
 * attention half of h-mode) when launched with `num_ctas` persistent CTAs
 * (0 = the library's choice for the current device, which needs a CUDA
 * device; pass an explicit count to size it without one). */
KVQ_API int kvq_workspace_bytes(const kvq_config *cfg, int32_t num_ctas, uint64_t *bytes);

/* The decode-attention launch kvq_decode_attn / kvq_append_decode_attn /
 * kvq_decode_partials make for this config with `num_ctas` CTAs (0 = the
 * library's choice for the current device, which needs a CUDA device).
 *   engine     KVQ_ENGINE_WARP_MMA: the warp-level MMA kernel (the default for
 *              every format); KVQ_ENGINE_TCGEN05: the tcgen05/TMEM kernel (its
 *              P.V product is an exact integer MMA of the value codes with P in
 *              fixed point of 2^-24), chosen only when the environment
 *              variable KVQ_DECODE_TC is "1" at the call and the format is one
 *              it supports (head_dim 128, INT8/INT4 codes, value scales per
 *              (token, head), G <= 8).  The variable is read at every call, so
 *              size the workspace under the same setting as the call.
 *   num_ctas   persistent CTAs of the launch (the work split over them)
 *   ctas_per_sm_planned  CTAs per SM its shared memory and registers are sized for
 *   stages, stage_bytes  depth and bytes of the TMA ring (one 128-token K/V tile
 *              with its scales per stage); smem_bytes  dynamic shared memory
 *   threads    threads per CTA
 *   packed_columns  1 when the warp-MMA kernel packs the score MMA's columns (G <= 4 at
 *              head_dim 128 with INT4 / INT8 keys): the hi and lo query parts share one
 *              MMA, and each lane's softmax work covers live columns only
 * Errors: INVALID_ARG, UNSUPPORTED, DEVICE. */
#define KVQ_ENGINE_WARP_MMA 0
#define KVQ_ENGINE_TCGEN05 1
typedef struct kvq_decode_plan {
    int32_t engine, num_ctas, ctas_per_sm_planned, stages;
    int32_t stage_bytes, smem_bytes, threads, packed_columns;
} kvq_decode_plan;
KVQ_API int kvq_decode_plan_info(const kvq_config *cfg, int32_t num_ctas, kvq_decode_plan *info);

/* h-mode scratch bytes for kvq_decode_attn: the reconstructed fp16 K and V for
 * up to max_len tokens of every sequence ([2][B][Hkv][round_up(max_len,64)][Dh]),
 * followed by the bf16 GEMM operand (kvq_h_operand_bytes). */
KVQ_API int kvq_h_scratch_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes);

/* Bytes of the bf16 operand buffer kvq_h_reconstruct needs: the dequantised
 * h^ of every sequence, [B][round_up(max_len,128)][D] bf16. */
KVQ_API int kvq_h_operand_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes);

/* Decode attention for one query token per sequence (split-KV, dequantised in
 * registers).  [MNI]: the new token's query attends over every cached K/V;
 * [KS] "…tích hợp trực tiếp vào kiến trúc FlashAttention": dequantise inside
 * the attention kernel.  Computes, for query head h (KV head h / G):
 *   s_t = softmax_scale * q . k^_t,  p = softmax(s) over t < d_len[b],
 *   out = sum_t p_t v^_t,   k^ = code * scale (exact), v^ likewise,
 * with fp32 accumulation, then rounds to out_dtype.  A sequence with length
 * 0 gets zeros.  The token just appended is included (no mask).
 *   q        device [B][Hq][Dh], q_dtype KVQ_F16, KVQ_F32 or KVQ_BF16; G <= 8
 *            (with 16-bit keys, f32/bf16 queries need G <= 4).  With 4- or
 *            8-bit keys the query enters the int8 tensor-core product as two
 *            int8 parts per head, q ~ (max|q|/127)(hi + lo/254), i.e. with a
 *            relative error below 2^-15 of the head's largest element.
 *   d_len    device int32 [B]: tokens attended per sequence (clamped to
 *            [0, capacity] on the device)
 *   max_len_host  host bound of d_len[] (<= capacity; used for h-mode scratch)
 *   softmax_scale  0 selects 1/sqrt(Dh)
 *   out      device [B][Hq][Dh], out_dtype KVQ_F16 or KVQ_F32
 *   workspace/workspace_bytes  device scratch for split partials and the
 *            merge's arrival counters, at least kvq_workspace_bytes(cfg,
 *            num_ctas).  Zero-fill it once before its first use; every call
 *            leaves it ready for the next one, except one that reported
 *            KVQ_ERR_TIMEOUT (zero-fill it again then).  Calls that overlap
 *            on the GPU need separate workspaces.
 *   num_ctas persistent CTAs (0 = library's choice)
 *   h-mode only: w_kv device bf16 [2*Hkv*Dh][D] (rows of W_k then W_v;
 *            [TL] "運作原理": rebuild K = W_k h, V = W_v h at every attention
 *            call, skipping the Q slice), kv_scratch/kv_scratch_bytes at least
 *            kvq_h_scratch_bytes(cfg, max_len_host).  KV mode: pass NULL / 0.
 * Errors: INVALID_ARG, UNSUPPORTED, CAPACITY, ALIGN, WORKSPACE, LAUNCH, DEVICE. */
KVQ_API int kvq_decode_attn(const kvq_config *cfg, const kvq_layer *layer, const void *q, int32_t q_dtype,
                    const int32_t *d_len, int32_t max_len_host, float softmax_scale, void *out,
                    int32_t out_dtype, void *workspace, uint64_t workspace_bytes, int32_t num_ctas,
                    const void *w_kv, void *kv_scratch, uint64_t kv_scratch_bytes,
                    kvq_stream_t stream);

/* One decode step of a layer in one launch (KV mode): quantize-on-append of
 * each sequence's newest token, then decode attention over the cache that
 * includes it.  For every sequence b with L = d_len[b] >= 1 (clamped to the
 * capacity), k_new[b] and v_new[b] ([B][Hkv][Dh], in_dtype) are quantised
 * into position L - 1 exactly as kvq_append(d_pos = L - 1, n_new = 1) would
 * ([TL] "KV Cache 模式": codes at append time), and the query then attends
 * over positions [0, L) as in kvq_decode_attn.  Sequences with L = 0 append
 * nothing and get zeros.  Other arguments and errors as kvq_decode_attn;
 * h-mode configs return KVQ_ERR_INVALID_ARG. */
KVQ_API int kvq_append_decode_attn(const kvq_config *cfg, const kvq_layer *layer,
                                   const void *k_new, const void *v_new, int32_t in_dtype,
                                   const void *q, int32_t q_dtype, const int32_t *d_len,
                                   int32_t max_len_host, float softmax_scale, void *out,
                                   int32_t out_dtype, void *workspace, uint64_t workspace_bytes,
                                   int32_t num_ctas, kvq_stream_t stream);

/* The two halves of kvq_decode_attn in KV mode, for callers that schedule
 * them separately (e.g. to time the attention kernel alone, or to gather the
 * partials of several devices before merging).
 * kvq_decode_partials: the split-KV attention kernel alone; writes one
 *   (m, l, o) partial per (consumer warp, CTA, sequence, KV head) segment into
 *   `workspace` (arguments as kvq_decode_attn; the counters are not used).  The partials are unnormalised: o = sum_t p_t v^_t
 *   and l = sum_t p_t with p_t = 2^(s_t log2(e) - m).
 * kvq_merge_partials: combines the partials with log-sum-exp weights,
 *   out = sum_k o_k 2^(m_k - M) / sum_k l_k 2^(m_k - M), and rounds to
 *   out_dtype.  cfg, d_len, workspace and num_ctas must be those of the
 *   kvq_decode_partials call it follows on the same stream.
 * Errors as kvq_decode_attn; KVQ_ERR_INVALID_ARG in h-mode. */
KVQ_API int kvq_decode_partials(const kvq_config *cfg, const kvq_layer *layer, const void *q,
                                int32_t q_dtype, const int32_t *d_len, int32_t max_len_host,
                                float softmax_scale, void *workspace, uint64_t workspace_bytes,
                                int32_t num_ctas, kvq_stream_t stream);
KVQ_API int kvq_merge_partials(const kvq_config *cfg, const int32_t *d_len, void *out,
                               int32_t out_dtype, void *workspace, uint64_t workspace_bytes,
                               int32_t num_ctas, kvq_stream_t stream);

/* h-mode K/V reconstruction on its own ([TL] "運作原理"; the page's tensor-core
 * path replaces the scalar one): for every sequence b and token t < len,
 *   [K_t | V_t] = W_kv . bf16(h^_t)   (fp32 accumulation, rounded to fp16)
 * written to k_out / v_out, each [B][Hkv][out_capacity][Dh] fp16, with
 * len = max_len_host for every sequence (rows t >= len are not written).
 * out_capacity is a multiple of 64 and >= max_len_host.  `operand` is device
 * scratch of at least kvq_h_operand_bytes(cfg, max_len_host) bytes that
 * receives bf16(h^) first (contents on entry do not matter).
 * Errors as kvq_decode_attn. */
KVQ_API int kvq_h_reconstruct(const kvq_config *cfg, const kvq_layer *layer, const void *w_kv,
                              int32_t max_len_host, void *k_out, void *v_out,
                              int32_t out_capacity, void *operand, uint64_t operand_bytes,
                              kvq_stream_t stream);

/* h-mode decode attention with the reconstruction fused into it ([TL]
 * "運作原理": K = W_k h^, V = W_v h^ rebuilt at every call; here never written to
 * memory): the tcgen05 GEMM computes, per 128-token tile and KV head j, the tile's
 * K_j and V_j (bf16(h^) operands, fp32 accumulators in tensor memory), and the
 * epilogue warps attend over them (per 32 tokens: s_t = softmax_scale * q . K_t,
 * max, sum, o = sum 2^(s - max) V_t); a merge launch combines the partials:
 *   out = sum_t p_t V_t,  p = softmax(s) over t < d_len[b].
 * Same arithmetic as kvq_decode_attn's h-mode path except that K and V stay fp32
 * (no fp16 rounding).  Dh = 128, Hq / Hkv <= 8, h_bits 4, 8 or 16.
 *   w_kv, q, q_dtype, d_len, max_len_host, softmax_scale, out, out_dtype: as
 *            kvq_decode_attn
 *   scratch  device, at least kvq_h_fused_scratch_bytes(cfg, max_len_host) bytes:
 *            a 256-byte header whose first int32 is a status word like a
 *            workspace's (zero it once before the first call; read and clear it
 *            with kvq_workspace_status), then the bf16(h^) operand and the partials
 * Three launches (operand pre-pass, fused GEMM + attention, merge).  Errors as
 * kvq_h_decode_absorbed. */
KVQ_API int kvq_h_fused_scratch_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes);
KVQ_API int kvq_h_decode_fused(const kvq_config *cfg, const kvq_layer *layer, const void *w_kv,
                               const void *q, int32_t q_dtype, const int32_t *d_len,
                               int32_t max_len_host, float softmax_scale, void *out,
                               int32_t out_dtype, void *scratch, uint64_t scratch_bytes,
                               kvq_stream_t stream);

/* h-mode decode attention by query absorption: the attention of
 * kvq_decode_attn (h-mode) regrouped by the linearity of the reconstruction
 * ([TL] "運作原理": K = W_k h^, V = W_v h^), without rebuilding K and V:
 * for sequence b and query head h of KV head j = h / G,
 *   qa = W_k,j^T q            (W_k,j: rows j*Dh .. j*Dh+Dh-1 of w_kv)
 *   s_t = softmax_scale * qa . h^_t,  p = softmax(s) over t < d_len[b]
 *   out = W_v,j (sum_t p_t h^_t)   (W_v,j: rows Hkv*Dh + j*Dh .. of w_kv)
 * Equal in exact arithmetic to the reconstruction path; it reads the h codes
 * and W once per step instead of D x 2*Hkv*Dh MACs per cached token.  Here
 * qa is split per (head, scale group) into two int8 parts for the int8
 * tensor-core scores (relative error below 2^-15 of the group's largest
 * element) and p * scale enters the p . h^ product in fp16; everything else
 * accumulates in fp32.  The token splits of sum_t p_t h^_t are added in L2
 * (fp32 reductions), so the last bits of a result may differ between calls.
 * An empty sequence gets zeros.
 *   h_bits 4 or 8; Hkv*Dh = D, D a multiple of 256 and at most 3584, Dh 64 or
 *   128; Hq <= 32 (smaller limits where the score tile's shared memory runs out).
 *   w_kv     device bf16 [2*Hkv*Dh][D] (as kvq_decode_attn)
 *   q, q_dtype, d_len, max_len_host, softmax_scale, out, out_dtype: as
 *            kvq_decode_attn (max_len_host bounds d_len[] and sizes the scratch)
 *   scratch  device, at least kvq_h_absorbed_scratch_bytes(cfg, max_len_host)
 *            bytes (contents on entry do not matter; calls that overlap on
 *            the GPU need separate scratch)
 * Four kernel launches on `stream`, each a programmatic dependent of the
 * previous one.  Errors: INVALID_ARG (KV mode, null or
 * bad arguments), UNSUPPORTED (shape), CAPACITY, ALIGN (16 bytes), WORKSPACE,
 * LAUNCH. */
KVQ_API int kvq_h_absorbed_scratch_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes);
KVQ_API int kvq_h_decode_absorbed(const kvq_config *cfg, const kvq_layer *layer, const void *w_kv,
                                  const void *q, int32_t q_dtype, const int32_t *d_len,
                                  int32_t max_len_host, float softmax_scale, void *out,
                                  int32_t out_dtype, void *scratch, uint64_t scratch_bytes,
                                  kvq_stream_t stream);

/* Read and clear the device status word a decode launch leaves in its
 * workspace: KVQ_OK, or KVQ_ERR_TIMEOUT if a kernel gave up a bounded wait
 * (its outputs are then invalid).  Synchronises `stream`. */
KVQ_API int kvq_workspace_status(void *workspace, int32_t *status, kvq_stream_t stream);

/* Self-test of failure detection.  Every wait inside the library's kernels is
 * bounded: after its limit it gives up, the kernel stores KVQ_ERR_TIMEOUT in the
 * workspace status word, drains and returns, and the context stays usable.  This
 * call runs that wait on a barrier that nothing completes, for timeout_ns
 * (1 ns .. 2 s), so that the give-up path can be checked on a GPU without a fault
 * or a hang: afterwards kvq_workspace_status(workspace) reports KVQ_ERR_TIMEOUT.
 * Only the first 4 bytes of `workspace` (16-byte aligned device memory) are used.
 * Errors: INVALID_ARG, ALIGN, LAUNCH. */
KVQ_API int kvq_selftest_bounded_wait(void *workspace, uint64_t timeout_ns, kvq_stream_t stream);

/* The same for the decode kernel itself: kvq_decode_attn (KV mode, contiguous
 * cache) with a wait limit of timeout_ns (1 ns .. 2 s) and a producer warp that
 * copies nothing, so every consumer's wait for its first tile runs out: the
 * kernel records KVQ_ERR_TIMEOUT in the workspace status word, its other warps
 * see the abort flag and return, and `out` is left unwritten.  The workspace must
 * then be zero-filled again before its next use (as after any timeout).
 * Arguments as kvq_decode_attn.  Errors as kvq_decode_attn. */
KVQ_API int kvq_selftest_decode_timeout(const kvq_config *cfg, const kvq_layer *layer,
                                        const void *q, int32_t q_dtype, const int32_t *d_len,
                                        void *out, int32_t out_dtype, void *workspace,
                                        uint64_t workspace_bytes, uint64_t timeout_ns,
                                        kvq_stream_t stream);

/* Bytes of the device array behind kvq_decode_attn_noalloc (8 MiB). */
#define KVQ_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

/* kvq_decode_attn (KV mode) for callers that cannot allocate device memory.
 * The source pages have no counterpart: this is a deployment convenience.
 * Some callers may not call cudaMalloc at all: code that runs under a host
 * framework which owns every device allocation, real-time loops that forbid
 * allocation after start-up because cudaMalloc can stall the device for an
 * unbounded time, or library code that must not change the process's memory
 * footprint at run time.  Instead of a caller-provided workspace, this entry
 * point uses one array of KVQ_NOALLOC_SCRATCH_BYTES in device memory that is
 * part of libkvq itself; every GPU that loads the library holds it until the
 * process exits.  The caller still passes the cache, q, d_len and out.
 *   Set-up: the first call on each device (with that device current) looks up
 *     the array's device address; make that first call before any stream
 *     capture.
 *   Limit: configurations whose kvq_workspace_bytes(cfg, num_ctas) exceeds
 *     KVQ_NOALLOC_SCRATCH_BYTES are rejected with KVQ_ERR_WORKSPACE before
 *     anything is launched (for example B=16, Hkv=8, G=4, Dh=128 on 296 CTAs
 *     needs 3.5 MB).
 *   Sharing: all calls in the process share the one array and it keeps the
 *     last call's contents; calls that overlap on the GPU (different streams,
 *     or several host threads) race on it and give wrong results.  Each call
 *     clears the status word and the merge counters it needs zeroed.
 *   Status: a bounded wait that gives up inside this call records
 *     KVQ_ERR_TIMEOUT in the array's status word, not in a caller buffer; read
 *     it with kvq_noalloc_status after the call and before the next one (the
 *     next call clears it).
 *   Device reset: the array's device address is kept per device for the life
 *     of the process; after cudaDeviceReset (or anything else that destroys
 *     the primary context) the address may be stale, so neither noalloc entry
 *     point may be called again in that process.
 * Nothing here allocates or frees memory.  Other arguments and errors as
 * kvq_decode_attn; h-mode configs return KVQ_ERR_INVALID_ARG. */
KVQ_API int kvq_decode_attn_noalloc(const kvq_config *cfg, const kvq_layer *layer, const void *q,
                                    int32_t q_dtype, const int32_t *d_len, int32_t max_len_host,
                                    float softmax_scale, void *out, int32_t out_dtype,
                                    int32_t num_ctas, kvq_stream_t stream);

/* Read and clear the status word of the device array behind
 * kvq_decode_attn_noalloc on the current device, like kvq_workspace_status:
 * enqueues a 4-byte copy and a 4-byte clear on `stream` and synchronises it.
 * *status = KVQ_OK, or KVQ_ERR_TIMEOUT when a bounded wait of the last noalloc
 * call gave up (its `out` is then not valid).  Allocates nothing.  The source
 * pages have no counterpart: it only completes kvq_decode_attn_noalloc. */
KVQ_API int kvq_noalloc_status(int32_t *status, kvq_stream_t stream);

/* Self-test of the failure path of kvq_decode_attn_noalloc: the same clearing
 * of the library's array, then the decode kernel of kvq_selftest_decode_timeout
 * (its producer copies nothing, every consumer wait gives up after timeout_ns)
 * with that array as the workspace.  Afterwards kvq_noalloc_status reports
 * KVQ_ERR_TIMEOUT.  No fault, trap or hang is involved.  Arguments and limits
 * as kvq_selftest_decode_timeout; allocates nothing.  No counterpart on the
 * source pages. */
KVQ_API int kvq_selftest_noalloc_timeout(const kvq_config *cfg, const kvq_layer *layer,
                                         const void *q, int32_t q_dtype, const int32_t *d_len,
                                         void *out, int32_t out_dtype, uint64_t timeout_ns,
                                         kvq_stream_t stream);

/* Which step of the last call on this thread that returned KVQ_ERR_LAUNCH
 * failed, and the CUDA error name ("decode launch: cudaErrorX").  Valid until
 * the next failing call on the same thread; "" if none. */
KVQ_API const char *kvq_last_error_detail(void);

/* Static description of a status code. */
KVQ_API const char *kvq_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
