// kvq_internal.h -- declarations shared by the libkvq translation units.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "../../include/kvq.h"

namespace kvq {

// ------------------------------------------------------------------ append
struct AppendParams {
    const void *x;          // [B][n_new][rows_per_tok][dim] input
    const int32_t *d_pos;   // [B]
    uint8_t *codes;         // [B][rows_per_tok][cap][row_bytes]
    __half *scales;         // [B][rows_per_tok][cap][dim/group] (unused at 16 bits; pairs
                            // (scale, zero-point) when asymmetric; one scale when per-tensor)
    int32_t in_dtype;       // KVQ_F16 / KVQ_F32 / KVQ_BF16
    int32_t batch, n_new, rows_per_tok, dim, cap;
    int32_t bits, group;
    int32_t window, n_anchor;   // sliding window (0: slot = position)
    int32_t fmt;                // KVQ_FMT_*: integer, e4m3, asymmetric or per-tensor codes
    const int32_t *block_table; // paged cache: [batch][max_pages] pool page of each logical page
    int32_t max_pages, n_pages; // (rows_per_tok is the KV heads; pages hold kPageTokens rows)
};

constexpr int kPageTokens = 128;   // tokens per page of a paged cache (one decode tile)

// Cache slot of token position t: the first n_anchor tokens stay put, the rest
// share a ring of `window` slots (window 0: no ring, slot t).
__host__ __device__ inline int cache_slot(int t, int window, int n_anchor)
{
    if (window <= 0 || t < n_anchor) return t;
    return n_anchor + (t - n_anchor) % window;
}

cudaError_t launch_append(const AppendParams &k, const AppendParams *v, cudaStream_t stream);

// ------------------------------------------------------------------ decode
constexpr int kDecodeConsumerWarps = 4;
constexpr int kDecodeTileTokens = 32 * kDecodeConsumerWarps;   // tokens per stage (32 per warp)
// consumer warps, one producer warp, one combiner warp
constexpr int kDecodeThreads = 32 * (kDecodeConsumerWarps + 2);
// CTAs per SM the decode kernel is compiled for (168 registers per thread) and its
// shared-memory ring is planned for
constexpr int kDecodeCtasPerSm = 2;
constexpr int kWorkspaceHeaderFloats = 64;                      // status word + padding
// The new token's K/V for the append step fused into the decode kernel.
struct FusedAppend {
    const void *k_new, *v_new;    // [B][Hkv][Dh] in dtype; null: no append
    uint8_t *k_codes, *v_codes;   // the layer's cache (same memory the TMA maps read)
    __half *k_scales, *v_scales;
    int32_t dtype;                // KVQ_F16 / KVQ_F32 / KVQ_BF16
    int32_t k_group, v_group;     // elements per scale (32 at 16 bits)
};

// fp16 values per scale group in the scale arrays of a code format
__host__ __device__ constexpr int scale_vals(int fmt) { return fmt == KVQ_FMT_ASYM ? 2 : 1; }

// Shared-memory regions of the tensor-core decode kernel (kvq_decode_tc.cu) after its
// stage ring: widened INT4 keys and values, P digit tiles, int8 query rows, and the
// control area (barriers are at off_bar as for the warp-MMA kernel).
struct TcOffsets {
    uint32_t off_kx, off_vx, off_pb, off_qb, off_aux;
};
constexpr uint32_t kTcBarsBytes = 256;    // the kernel's extra mbarriers
constexpr uint32_t kTcAuxBytes = 1024;    // factors, max exchange, sums, TMEM address

struct DecodeParams {
    const int32_t *d_len;     // [B]
    const void *q;            // [B][Hq][Dh]
    const __half *k_scales;   // [B][Hkv][cap][ngs_k]   (null at 16 bits)
    const __half *v_scales;
    float *ws;                // per-warp partial slots
    int *status;              // workspace status word
    int *counters;            // [B*Hkv] warp arrivals; null: leave the partials for a merge launch
    void *out;                // [B][Hq][Dh] (fused merge only)
    int32_t out_f32;
    int32_t q_dtype;
    int32_t batch, n_q_heads, n_kv_heads, group_size_g, cap;
    int32_t ngs_k, ngs_v;     // scales per row
    int32_t kshift, vshift;   // scale index of 32-element block = blk >> shift
    int32_t num_ctas;         // persistent CTAs (work split over them)
    int32_t stages;
    uint32_t stage_bytes, off_v, off_sk, off_sv, off_meta, off_bar, off_merge;
    // packed-column int8 instances: where the consumer warps share a segment's query
    // quantisation: hi and lo bytes ([4 heads][Dh] each) and 4 factors + 2 mbarriers
    // (32 bytes); off_qmisc 0 for none
    uint32_t off_qhi, off_qlo, off_qmisc;
    float tau_log2e;
    uint64_t timeout_ns;
    FusedAppend app;
    int32_t window, n_anchor;  // sliding window: slot of the newest token (fused append)
    const int32_t *block_table;  // paged cache (null: contiguous per sequence)
    int32_t max_pages, n_pages;
    int32_t stall;            // self-test only: the producer issues no copy, so every
                              // consumer wait runs out (kvq_selftest_decode_timeout)
    TcOffsets tc;             // tensor-core kernel only
};

struct MergeParams {
    const int32_t *d_len;
    const float *ws;
    void *out;
    int32_t out_f32;
    int32_t batch, n_q_heads, n_kv_heads, group_size_g, cap, head_dim, num_ctas;
};

// Host helpers implemented in kvq_decode.cu.
// h-mode decode by query absorption (kvq_absorb.cu)
struct AbsorbParams {
    const uint8_t *h_codes;       // [B][cap][D*bits/8]
    const __half *h_scales;       // [B][cap][ng]
    const __nv_bfloat16 *w;       // [2*Hkv*Dh][D]: W_k rows, then W_v rows
    const void *q;                // [B][Hq][Dh]
    const int32_t *d_len;         // [B]
    void *out;                    // [B][Hq][Dh]
    int32_t q_dtype, out_f32;
    int32_t B, Hq, Hkv, Dh, D, cap, bits, group, ng;
    float tau_log2e;
    // scratch
    uint4 *qfrag;                 // [B][D/32][NT][32] int8 hi/lo B fragments of W_k^T q
    float *qfac;                  // [B][ng][NT*8] score factor per (group, head)
    float *p;                     // [B][Hq][capP] scores (log2 units)
    float2 *stats;                // [B][Hq][ntile] (max, sum 2^(s - max)) per score tile
    float *obp;                   // [splits][B][Hq][D] partial sum_t p_t h^_t
    int32_t capP, NT, T2, ntile, split;
};
int absorb_nt(int Hq);            // n-tiles of 8 query heads in the score MMA: 1, 2 or 4
bool absorb_fits(int D, int bits, int Hq, int ng);   // shared memory suffices for the shape
int absorb_t2(int D, int bits, int Hq, int ng);   // tokens per score tile
int absorb_split(int max_len);    // tokens per split of the p . h^ kernel
// scratch bytes; off[0..4] = qfrag, qfac, scores, stats, partial ob (256-byte aligned)
uint64_t absorb_scratch_layout(int B, int Hq, int D, int ng, int bits, int max_len, uint64_t off[6]);
cudaError_t launch_absorbed(const AbsorbParams &p, int max_len, cudaStream_t stream);

// self-test of the bounded wait (kvq_selftest.cu): a wait nothing completes gives up
cudaError_t launch_bounded_wait_selftest(int *status, uint64_t limit_ns, cudaStream_t stream);

struct DecodeLaunch {
    int dh, kb, vb;
    bool kg, vg;              // grouped key / value scales
    int fmt;                  // KVQ_FMT_* of the 8-bit codes
    bool tc;                  // the tensor-core kernel (kvq_decode_tc.cu)
    bool pk;                  // warp-MMA kernel with packed score columns (G <= 4)
    int G;                    // query heads per KV head (tensor-core kernel instance)
    int per_sm;               // CTAs per SM the plan's shared memory is sized for
    size_t smem_bytes;
    int stages;
    uint32_t stage_bytes, off_v, off_sk, off_sv, off_meta, off_bar, off_merge;
    uint32_t off_qhi, off_qlo, off_qmisc;   // shared query quantisation (off_qmisc 0: none)
    TcOffsets tco;
};

// Decode kernel instances (kvq_decode_k4/k8/k16.cu), by key width: the kernel
// for (head_dim, value width, grouped key scales, grouped value scales), or
// null if there is none.
void *decode_fn_kb4(int dh, int vb, bool kg, bool vg);
void *decode_fn_kb8(int dh, int vb, bool kg, bool vg);
void *decode_fn_kb16(int dh, int vb, bool kg, bool vg);
// e4m3, asymmetric and per-tensor 8-bit keys and values (kvq_decode_fmt.cu)
void *decode_fn_fmt(int dh, int fmt, bool kg, bool vg);
// packed score columns, G <= 4 at head_dim 128 (kvq_decode_pk4/pk8.cu): INT4 / INT8
// keys and values (fmt KVQ_FMT_INT), or per-tensor INT8
void *decode_fn_pk_kb4(int vb, bool kg, bool vg, int fmt);
void *decode_fn_pk_kb8(int vb, bool kg, bool vg, int fmt);
// the tensor-core kernel (head_dim 128; value scales per (token, head), key scales
// per (token, head) or per 32/64-element group; or per-tensor INT8): INT8 / INT4 keys
// and values with G query heads per KV head, or null (kvq_decode_tc.cu); and the
// bytes of one of its P digit tiles
void *decode_tc_fn(int kb, int vb, bool kg, int G, int fmt);
uint32_t decode_tc_pb_bytes(int G);

// Fill in the shared-memory plan; returns false if the shape is unsupported.
bool plan_decode(int dh, int kb, int vb, int ngs_k, int ngs_v, int G, int max_smem,
                 DecodeLaunch *plan, int fmt = 0);
cudaError_t decode_occupancy(const DecodeLaunch &plan, int *ctas_per_sm);
cudaError_t launch_decode(const DecodeLaunch &plan, const DecodeParams &p, const CUtensorMap &tm_k,
                          const CUtensorMap &tm_v, cudaStream_t stream);
cudaError_t launch_merge(const MergeParams &p, cudaStream_t stream);

// Workspace: [header][counters][partial slots].  A partial slot holds, for the
// G query heads of one KV head, a record of Dh + 4 floats each: o[Dh], m, l and
// two floats of padding that keep every record 16-byte aligned.  A CTA writes
// one slot for each (sequence, KV head) segment it works on.
__host__ __device__ constexpr int slot_col_floats(int dh) { return dh + 4; }
inline uint64_t slot_floats(int G, int dh) { return (uint64_t)G * (uint64_t)slot_col_floats(dh); }
inline uint64_t slot_count(int num_ctas, int batch, int n_kv_heads)
{
    return (uint64_t)num_ctas + (uint64_t)batch * (uint64_t)n_kv_heads;
}
inline uint64_t counter_ints(int batch, int n_kv_heads)
{
    return ((uint64_t)batch * (uint64_t)n_kv_heads + 63) / 64 * 64;
}

// ------------------------------------------------------------------ h-mode GEMM
struct HGemmParams {
    const uint8_t *h_codes;   // [B][cap][D*h_bits/8]
    const __half *h_scales;   // [B][cap][h_groups]
    const void *w;            // bf16 [N][D]
    __half *k_out, *v_out;    // [B][Hkv][out_cap][Dh]
    void *operand;            // bf16 [B][round_up(len, 128)][D] scratch for h^
    int *status;              // set to KVQ_ERR_TIMEOUT if a wait gives up (may be null)
    int32_t batch, cap, d_model, h_bits, h_groups, n_kv_heads, head_dim, len, out_cap;
    // fused reconstruction + attention (part != null): no K/V written; the GEMM epilogue
    // attends over each tile and fused_merge_kernel writes `out`
    const void *q;            // [B][Hq][Dh]
    const int32_t *d_len;     // [B]
    float *part;              // [B][Hq][m_tiles * 4][Dh + 2]
    void *out;                // [B][Hq][Dh]
    int32_t q_dtype, n_q_heads, out_f32;
    float tau_log2e;
};
cudaError_t launch_h_reconstruct(const HGemmParams &p, cudaStream_t stream);
constexpr int kHTileTokens = 128;   // token rows of one reconstruction tile

}  // namespace kvq
