// kvq_decode_common.cuh -- pieces shared by the decode attention kernels
// (kvq_decode_kernel.cuh: warp-level MMA consumers; kvq_decode_tc.cu: tcgen05
// consumers): the stage metadata and the 128-byte swizzle of the TMA tiles, the
// stream-K split of the work over persistent CTAs, the TMA producer warp with the
// fused append of each sequence's newest token, and the merge of the CTA partials.
#pragma once
#include <cfloat>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "kvq_quant.cuh"
#include "../../include/kvq.h"

namespace kvq {
namespace {

constexpr int T = kDecodeTileTokens;
constexpr unsigned FULL = 0xffffffffu;

struct __align__(16) StageMeta {
    int32_t bh;      // sequence * Hkv + kv_head
    int32_t t0;      // first token of the tile
    int32_t len;     // tokens attended by this sequence
    int32_t flags;   // bit0 first tile of a segment, bit1 last tile of a segment
    int32_t slot;    // partial slot of this CTA's segment: cta + bh
    int32_t ncta;    // CTAs holding a segment of this (sequence, KV head)
    int32_t cmin;    // the first of them
    int32_t pad;
};

// Byte offset of element byte `o` of token `t` inside a stage tile that TMA
// wrote with 128-byte swizzle.  Rows of R <= 128 bytes are packed 128/R tokens
// per 128-byte line; R = 256 is stored as two 128-byte-wide boxes.
template <int R>
__host__ __device__ constexpr uint32_t sw_off(int t, int o)
{
    if constexpr (R <= 128) {
        constexpr int TPL = 128 / R;
        const int line = t / TPL;
        const int col = (t % TPL) * R + o;
        return (uint32_t)(line * 128 + ((((col >> 4) ^ line) & 7) << 4) + (col & 15));
    } else {
        const int sub = o >> 7, col = o & 127;
        return (uint32_t)(sub * (T * 128) + t * 128 + ((((col >> 4) ^ t) & 7) << 4) + (col & 15));
    }
}

__device__ __forceinline__ float load_qf(const void *q, int dtype, int64_t idx)
{
    if (dtype == KVQ_F16) return __half2float(static_cast<const __half *>(q)[idx]);
    if (dtype == KVQ_F32) return static_cast<const float *>(q)[idx];
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[idx]);
}

// Eight consecutive query elements idx .. idx+7 as float: one 16-byte load (two for
// fp32).  Every entry point refuses a query base that is not 16-byte aligned, and
// idx is a multiple of 8.  The dtype test is uniform across the warp.
__device__ __forceinline__ void load_q8(const void *q, int dtype, int64_t idx, float (&x)[8])
{
    if (dtype == KVQ_F32) {
        const float4 *s = reinterpret_cast<const float4 *>(static_cast<const float *>(q) + idx);
        const float4 a = __ldg(s), b = __ldg(s + 1);
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
        x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
    } else {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(q) + idx));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; i++) {
            if (dtype == KVQ_F16) {
                x[2 * i] = __half2float(__ushort_as_half((unsigned short)(ws[i] & 0xFFFFu)));
                x[2 * i + 1] = __half2float(__ushort_as_half((unsigned short)(ws[i] >> 16)));
            } else {
                // bfloat16 -> float: the 16 bits become the high half of the word
                x[2 * i] = __uint_as_float(ws[i] << 16);
                x[2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u);
            }
        }
    }
}

__device__ __forceinline__ int clamp_len(int len, int cap)
{
    return len < 0 ? 0 : (len > cap ? cap : len);
}

__device__ __forceinline__ int tiles_of(int len, int cap) { return (clamp_len(len, cap) + T - 1) / T; }

// 2^x with the hardware approximation (relative error ~2^-22); results below
// 2^-126 flush to zero, which only drops probabilities that are zero anyway.
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Loads from the stage ring.  `b` is the 32-bit shared-window address of the
// 1024-aligned ring base and `o` a byte offset from it; explicit ld.shared keeps the
// address arithmetic 32-bit.  volatile keeps every load after the mbarrier wait
// that guards its stage (the wait is a volatile asm with a memory clobber).
__device__ __forceinline__ uint32_t lds_u16(uint32_t b, uint32_t o)
{
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(b + o));
    return v;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t b, uint32_t o)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(b + o));
    return v;
}
__device__ __forceinline__ uint2 lds_u64(uint32_t b, uint32_t o)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(b + o));
    return v;
}
__device__ __forceinline__ uint4 lds_u128(uint32_t b, uint32_t o)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(b + o));
    return v;
}

// The same loads at the shared address a + IMM, IMM a compile-time byte offset
// that the load instruction carries itself.
template <int IMM>
__device__ __forceinline__ uint32_t ldsi_u16(uint32_t a)
{
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1+%2];" : "=h"(v) : "r"(a), "n"(IMM));
    return v;
}
template <int IMM>
__device__ __forceinline__ uint32_t ldsi_u32(uint32_t a)
{
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(a), "n"(IMM));
    return v;
}
template <int IMM>
__device__ __forceinline__ uint2 ldsi_u64(uint32_t a)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(IMM));
    return v;
}
template <int IMM>
__device__ __forceinline__ uint4 ldsi_u128(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(a), "n"(IMM));
    return v;
}

// Merge the np CTA partials of one (sequence, KV head), all G query heads at once:
// slots slot0 .. slot0 + np - 1, each G records of DH + 4 floats holding per
// query head o[DH], m, l.  out[obase0 + col * DH + d] receives
//   sum_j o_j[d] 2^(m_j - M) / sum_j l_j 2^(m_j - M),  M = max_j m_j.
// LPC lanes share one query head (column) and split its DH outputs; the
// partials are read through L2 (ld.global.cg) because other SMs wrote them in
// this launch.  One warp.
template <int DH, int LPC>
__device__ void merge_segment_lpc(const float *ws, int64_t slot0, int np, int G, void *out,
                                  int out_f32, int64_t obase0, int lane)
{
    constexpr int PER = DH / LPC;       // floats of one partial per lane
    constexpr int CS = slot_col_floats(DH);
    const int col = lane / LPC, part = lane % LPC;
    const bool active = col < G;
    const int64_t stride = (int64_t)G * CS;
    const float *base = ws + slot0 * stride + (int64_t)(active ? col : 0) * CS;
    float M = -INFINITY;
    if (active)
        for (int j = part; j < np; j += LPC) M = fmaxf(M, __ldcg(base + j * stride + DH));
#pragma unroll
    for (int off = 1; off < LPC; off <<= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
    float L = 0.f;
    float o[PER];
#pragma unroll
    for (int i = 0; i < PER; i++) o[i] = 0.f;
    if (active && M != -INFINITY) {
#pragma unroll 4
        for (int j = 0; j < np; j++) {
            const float *src = base + (int64_t)j * stride;
            const float2 ml = __ldcg(reinterpret_cast<const float2 *>(src + DH));
            float4 x[PER / 4];
#pragma unroll
            for (int i = 0; i < PER / 4; i++)
                x[i] = __ldcg(reinterpret_cast<const float4 *>(src + part * PER) + i);
            const float e = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
            L = fmaf(e, ml.y, L);
#pragma unroll
            for (int i = 0; i < PER / 4; i++) {
                o[4 * i] = fmaf(e, x[i].x, o[4 * i]);
                o[4 * i + 1] = fmaf(e, x[i].y, o[4 * i + 1]);
                o[4 * i + 2] = fmaf(e, x[i].z, o[4 * i + 2]);
                o[4 * i + 3] = fmaf(e, x[i].w, o[4 * i + 3]);
            }
        }
    }
    if (!active) return;
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    const int64_t ob = obase0 + (int64_t)col * DH + part * PER;
#pragma unroll
    for (int i = 0; i < PER; i += 2) {
        if (out_f32)
            *reinterpret_cast<float2 *>(static_cast<float *>(out) + ob + i) =
                make_float2(o[i] * inv, o[i + 1] * inv);
        else
            *reinterpret_cast<__half2 *>(static_cast<__half *>(out) + ob + i) =
                __floats2half2_rn(o[i] * inv, o[i + 1] * inv);
    }
}

template <int DH>
__device__ __forceinline__ void merge_segment(const float *ws, int64_t slot0, int np, int G,
                                              void *out, int out_f32, int64_t obase0, int lane)
{
    if (G <= 4)
        merge_segment_lpc<DH, 8>(ws, slot0, np, G, out, out_f32, obase0, lane);
    else
        merge_segment_lpc<DH, 4>(ws, slot0, np, G, out, out_f32, obase0, lane);
}

// The work units are the 128-token tiles of every (sequence, KV head), in
// sequence-major, then KV-head, then token order; they are split stream-K style
// over the P' = min(P, units) CTAs that get work: CTA c takes units
// [c N / P', (c + 1) N / P').  One warp finds this CTA's range; lane 0 writes it.
// First unit of CTA c's range, c N / P', and the CTA whose range holds unit u,
// ((u + 1) P' + N - 1) / N - 1: 32-bit divisions when the products fit (a 64-bit
// division is several times longer, and these sit on the path to a segment's first
// copy), else 64-bit.
__device__ __forceinline__ long long range_begin(long long c, long long N, long long Pe)
{
    if (N * Pe < (1LL << 32)) return (long long)((uint32_t)(c * N) / (uint32_t)Pe);
    return c * N / Pe;
}
__device__ __forceinline__ long long range_cta(long long u, long long N, long long Pe)
{
    if (N * (Pe + 1) < (1LL << 32)) return (long long)((uint32_t)((u + 1) * Pe + N - 1) / (uint32_t)N) - 1;
    return ((u + 1) * Pe + N - 1) / N - 1;
}

struct WorkRange {
    long long u_begin;   // first unit of the range
    long long n;         // units in all
    long long pe;        // CTAs with work
    long long pre;       // units before sequence b
    int b;               // first sequence of the range (-1: none)
    int bh0;             // first (sequence, KV head) of the range
    int n_units;         // units of the range
    int tiles_b;         // tiles of each (sequence b, KV head)
};

__device__ void decode_work_range(const DecodeParams &p, int lane, WorkRange &wr)
{
    const int cap = p.cap;
    const int Hkv = p.n_kv_heads;
    long long total = 0;
    for (int b = lane; b < p.batch; b += 32) total += tiles_of(p.d_len[b], cap);
    for (int off = 16; off; off >>= 1) total += __shfl_xor_sync(FULL, total, off);
    const long long N = total * Hkv;
    const long long Pe = N < (long long)p.num_ctas ? N : (long long)p.num_ctas;
    long long ub = 0, ue = 0;
    if ((long long)blockIdx.x < Pe) {
        ub = range_begin(blockIdx.x, N, Pe);
        ue = range_begin((long long)blockIdx.x + 1, N, Pe);
    }
    // locate the sequence holding unit ub
    long long acc = 0;
    int fb = -1;
    long long fpre = 0, funits = 0;
    for (int base = 0; base < p.batch && fb < 0 && ue > ub; base += 32) {
        const int b = base + lane;
        const long long units = (b < p.batch) ? (long long)tiles_of(p.d_len[b], cap) * Hkv : 0;
        long long incl = units;
        for (int off = 1; off < 32; off <<= 1) {
            const long long v = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += v;
        }
        const long long excl = acc + incl - units;
        const bool hit = units > 0 && excl <= ub && ub < excl + units;
        const unsigned m = __ballot_sync(FULL, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            fb = __shfl_sync(FULL, b, src);
            fpre = __shfl_sync(FULL, excl, src);
            funits = __shfl_sync(FULL, units, src);
        }
        acc += __shfl_sync(FULL, incl, 31);
    }
    if (lane == 0) {
        wr.u_begin = ub;
        wr.n = N;
        wr.pe = Pe;
        wr.pre = fpre;
        wr.b = fb;
        wr.bh0 = fb >= 0 ? fb * Hkv + (int)((ub - fpre) / (funits / Hkv)) : 0;
        wr.n_units = (int)(ue > ub && fb >= 0 ? ue - ub : 0);
        wr.tiles_b = (int)(funits / Hkv);
    }
}

// The same range from lengths already in registers: lane l holds the lengths of
// sequences l + 32 k, k < 8 (batch <= kSpecBatch), zero past the batch.  The decode
// kernel computes it before its wait for the preceding launch, from lengths read
// through L2 (so that no early copy stays in L1), and reads them again after the
// wait: when a length changed in between, it computes the range anew.
constexpr int kSpecBatch = 256;

__device__ __forceinline__ void read_lens(const DecodeParams &p, int lane, int (&dl)[8])
{
#pragma unroll
    for (int k = 0; k < 8; k++) {
        const int b = lane + 32 * k;
        dl[k] = b < p.batch ? __ldcg(p.d_len + b) : 0;
    }
}

__device__ void work_range_from(const DecodeParams &p, int lane, WorkRange &wr, const int (&dl)[8])
{
    const int cap = p.cap;
    const int Hkv = p.n_kv_heads;
    long long total = 0;
#pragma unroll
    for (int k = 0; k < 8; k++) total += tiles_of(dl[k], cap);
    for (int off = 16; off; off >>= 1) total += __shfl_xor_sync(FULL, total, off);
    const long long N = total * Hkv;
    const long long Pe = N < (long long)p.num_ctas ? N : (long long)p.num_ctas;
    long long ub = 0, ue = 0;
    if ((long long)blockIdx.x < Pe) {
        ub = range_begin(blockIdx.x, N, Pe);
        ue = range_begin((long long)blockIdx.x + 1, N, Pe);
    }
    long long acc = 0;
    int fb = -1;
    long long fpre = 0, funits = 0;
#pragma unroll
    for (int k = 0; k < 8; k++) {
        if (fb >= 0 || ue <= ub) break;
        const int b = 32 * k + lane;
        const long long units = (long long)tiles_of(dl[k], cap) * Hkv;
        long long incl = units;
        for (int off = 1; off < 32; off <<= 1) {
            const long long v = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += v;
        }
        const long long excl = acc + incl - units;
        const bool hit = units > 0 && excl <= ub && ub < excl + units;
        const unsigned m = __ballot_sync(FULL, hit);
        if (m) {
            const int src = __ffs(m) - 1;
            fb = __shfl_sync(FULL, b, src);
            fpre = __shfl_sync(FULL, excl, src);
            funits = __shfl_sync(FULL, units, src);
        }
        acc += __shfl_sync(FULL, incl, 31);
    }
    if (lane == 0) {
        wr.u_begin = ub;
        wr.n = N;
        wr.pe = Pe;
        wr.pre = fpre;
        wr.b = fb;
        wr.bh0 = fb >= 0 ? fb * Hkv + (int)((ub - fpre) / (funits / Hkv)) : 0;
        wr.n_units = (int)(ue > ub && fb >= 0 ? ue - ub : 0);
        wr.tiles_b = (int)(funits / Hkv);
    }
}

// The producer warp: for each unit of the CTA's range, one TMA tile of key codes
// and one of value codes (3-D tiled maps, 128-byte swizzle; rows shorter than
// 128 bytes packed 128/R tokens per line), the tile's fp16 scales by 1-D bulk
// copies, and the stage's metadata, into the ring of p.stages stages guarded by
// full/empty mbarriers (`empty` must complete once per use of a stage).  With a
// fused append (p.app.k_new), the newest token of each (sequence, KV head) in
// the range is quantised into the cache before the tile holding it is loaded.
// Every wait is bounded; a give-up sets *abort_flag and the status word.  Before
// it returns, the warp waits (bounded by time only) for its copies in flight.
template <int DH, int KB, int VB, int FMT>
__device__ void decode_producer(const DecodeParams &p, const CUtensorMap *tm_k,
                                const CUtensorMap *tm_v, uint8_t *smem, uint64_t *full,
                                uint64_t *empty, StageMeta *meta, volatile int *abort_flag,
                                const WorkRange &wr, int lane)
{
    constexpr bool PT = FMT == KVQ_FMT_TENSOR;
    constexpr int RK = DH * KB / 8;
    constexpr int RV = DH * VB / 8;
    const int S = p.stages;
    const int cap = p.cap;
    const int Hkv = p.n_kv_heads;
    const int n_units = wr.n_units;
    if (p.stall) return;   // self-test: nothing is copied, the consumers' waits run out
    // codes and scales are read once: let them leave L2 first, so that the
    // partials and the queries stay cached
    const uint64_t pol = l2_evict_first_policy();
    const long long N = wr.n, Pe = wr.pe;
    int b = wr.b;
    long long pre = wr.pre;   // units before sequence b
    int len_b = (b >= 0) ? clamp_len(p.d_len[b], cap) : 0;
    int tiles_b = (len_b + T - 1) / T;
    const int off = (int)(wr.u_begin - pre);   // unit offset inside sequence b
    int kvh = tiles_b ? off / tiles_b : 0;
    int tile = tiles_b ? off % tiles_b : 0;
    int s = 0;
    uint32_t ph = 0;                            // phase parity of this use of stage s
    int issued = 0;
    int seg_ncta = 0, seg_cmin = 0;

    // Fused append.  The (sequence, KV head) pairs whose newest token lies in
    // a tile of this CTA are visited in unit order by a second walker; the
    // quantisation of the next one is done at the latest right before its
    // tile is loaded, and earlier whenever the ring is full and the warp
    // would only wait.  `app_rel` is the pending pair's tile index relative
    // to this CTA's first unit (n_units when none is left).
    const bool fuse_app = p.app.k_new != nullptr;
    int ab = b, akvh = kvh, alen = len_b, atiles = tiles_b;
    long long apre = pre;
    int app_rel = n_units;
    // cache slot of sequence ab's newest token (position d_len - 1; with a
    // sliding window its ring slot, anywhere among the cached tokens)
    auto newest_slot = [&]() {
        return p.window > 0 ? cache_slot(p.d_len[ab] - 1, p.window, p.n_anchor) : alen - 1;
    };
    int aslot = (ab >= 0 && ab < p.batch && alen > 0) ? newest_slot() : 0;
    auto find_app = [&]() {
        app_rel = n_units;
        while (ab < p.batch) {
            const long long ulast = apre + (long long)akvh * atiles + aslot / T;
            const long long rel = ulast - wr.u_begin;
            if (rel >= n_units) return;            // beyond this CTA's range
            if (atiles > 0 && rel >= 0) {
                app_rel = (int)rel;
                return;
            }
            // next (sequence, KV head)
            if (++akvh == Hkv) {
                akvh = 0;
                apre += (long long)atiles * Hkv;
                ++ab;
                alen = (ab < p.batch) ? clamp_len(p.d_len[ab], cap) : 0;
                atiles = (alen + T - 1) / T;
                aslot = alen > 0 ? newest_slot() : 0;
            }
        }
    };
    auto do_app = [&]() {
        const int bh = ab * Hkv + akvh;
        int64_t crow = (int64_t)bh * cap + aslot;
        if (p.block_table != nullptr) {
            // paged: the pool page of the newest token's logical page
            int page = p.block_table[(int64_t)ab * p.max_pages + aslot / T];
            page = min(max(page, 0), p.n_pages - 1);
            crow = ((int64_t)page * Hkv + akvh) * T + aslot % T;
        }
        constexpr int SCV = scale_vals(FMT);
        quantize_row(p.app.k_new, (int64_t)bh * DH, p.app.dtype, DH, KB, p.app.k_group,
                     p.app.k_codes + crow * RK,
                     KB == 16 ? nullptr
                     : PT     ? p.app.k_scales
                              : p.app.k_scales + crow * (DH / p.app.k_group) * SCV, lane, FMT);
        quantize_row(p.app.v_new, (int64_t)bh * DH, p.app.dtype, DH, VB, p.app.v_group,
                     p.app.v_codes + crow * RV,
                     VB == 16 ? nullptr
                     : PT     ? p.app.v_scales
                              : p.app.v_scales + crow * (DH / p.app.v_group) * SCV, lane, FMT);
        // order the writes before the copy engine reads the tile
        fence_proxy_async_global();
        __syncwarp();
        // move on to the next pair
        if (++akvh == Hkv) {
            akvh = 0;
            apre += (long long)atiles * Hkv;
            ++ab;
            alen = (ab < p.batch) ? clamp_len(p.d_len[ab], cap) : 0;
            atiles = (alen + T - 1) / T;
            aslot = alen > 0 ? newest_slot() : 0;
        }
        find_app();
    };
    if (fuse_app && n_units > 0) find_app();

    for (int i = 0; i < n_units; i++) {
        const int bh = b * Hkv + kvh;
        const int t0 = tile * T;
        if (i == 0 || tile == 0) {
            // CTAs whose unit ranges meet this (sequence, KV head)
            const long long u0 = pre + (long long)kvh * tiles_b, u1 = u0 + tiles_b;
            const long long cmin = range_cta(u0, N, Pe);
            const long long cmax = range_cta(u1 - 1, N, Pe);
            seg_cmin = (int)cmin;
            seg_ncta = (int)(cmax - cmin + 1);
        }
        // the newest token of a (sequence, KV head) must be in the cache
        // before the tile that holds its slot is loaded
        if (fuse_app && app_rel == i) do_app();
        int ok = 1;
        if (lane == 0 && i >= S) ok = mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, p.timeout_ns);
        ok = __shfl_sync(FULL, ok, 0);
        if (!ok) {
            if (lane == 0) {
                *abort_flag = 1;
                atomicExch(p.status, KVQ_ERR_TIMEOUT);
            }
            break;
        }
        if (lane == 0) {
            int flags = 0;
            if (i == 0 || tile == 0) flags |= 1;
            if (i == n_units - 1 || tile == tiles_b - 1) flags |= 2;
            StageMeta m;
            m.bh = bh; m.t0 = t0; m.len = len_b; m.flags = flags;
            m.slot = (int)blockIdx.x + bh;
            m.ncta = seg_ncta; m.cmin = seg_cmin; m.pad = 0;
            meta[s] = m;

            // physical tile: (bh, t0) of the contiguous layout, or the pool
            // page the block table names (whole page, row 0) in a paged one
            int z = bh, y0 = t0, zcap = cap;
            if (p.block_table != nullptr) {
                int page = p.block_table[(int64_t)b * p.max_pages + tile];
                page = min(max(page, 0), p.n_pages - 1);   // stay inside the pool
                z = page * Hkv + kvh;
                y0 = 0;
                zcap = T;
            }
            uint8_t *st = smem + (size_t)s * p.stage_bytes;
            const int n_s = min(T, zcap - y0);
            uint32_t bytes = (uint32_t)(T * RK + T * RV);
            if (KB != 16 && !PT) bytes += (uint32_t)(n_s * p.ngs_k * 2);
            if (VB != 16 && !PT) bytes += (uint32_t)(n_s * p.ngs_v * 2);
            mbar_arrive_expect_tx(&full[s], bytes);
            if constexpr (RK <= 128) {
                tma_load_3d_hint(st, tm_k, &full[s], 0, y0 / (128 / RK), z, pol);
            } else {
                tma_load_3d_hint(st, tm_k, &full[s], 0, y0, z, pol);
                tma_load_3d_hint(st + T * 128, tm_k, &full[s], 128, y0, z, pol);
            }
            if constexpr (RV <= 128) {
                tma_load_3d_hint(st + p.off_v, tm_v, &full[s], 0, y0 / (128 / RV), z, pol);
            } else {
                tma_load_3d_hint(st + p.off_v, tm_v, &full[s], 0, y0, z, pol);
                tma_load_3d_hint(st + p.off_v + T * 128, tm_v, &full[s], 128, y0, z, pol);
            }
            if (KB != 16 && !PT)
                bulk_load_hint(st + p.off_sk, p.k_scales + ((int64_t)z * zcap + y0) * p.ngs_k,
                               (uint32_t)(n_s * p.ngs_k * 2), &full[s], pol);
            if (VB != 16 && !PT)
                bulk_load_hint(st + p.off_sv, p.v_scales + ((int64_t)z * zcap + y0) * p.ngs_v,
                               (uint32_t)(n_s * p.ngs_v * 2), &full[s], pol);
        }
        issued = i + 1;
        if (++s == S) {
            s = 0;
            ph ^= 1u;
        }
        // ring full: quantise a pending newest token instead of only waiting
        if (fuse_app && i >= S - 1 && app_rel < n_units) do_app();
        // advance to the next unit (the length is re-read only when b changes)
        if (++tile == tiles_b) {
            tile = 0;
            if (++kvh == Hkv) {
                kvh = 0;
                do {
                    pre += (long long)tiles_b * Hkv;
                    ++b;
                    len_b = (b < p.batch) ? clamp_len(p.d_len[b], cap) : T;
                    tiles_b = (len_b + T - 1) / T;
                } while (tiles_b == 0);
            }
        }
    }
    // never leave with copies in flight: wait for the last issued phases, also
    // after another warp gave up (the copies still target this CTA's memory)
    if (lane == 0) {
        int ss = s;
        uint32_t pp = ph;
        for (int j = 0; j < min(S, issued); j++) {
            if (ss == 0) {
                ss = S;
                pp ^= 1u;
            }
            --ss;
            (void)mbar_wait_drain(&full[ss], pp, p.timeout_ns);
        }
    }
}

}  // namespace
}  // namespace kvq
