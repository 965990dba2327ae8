// kvq_decode.cu -- split-KV decode attention over a quantised KV cache.
//
// What it computes (the pages' problem statement): one query token per
// sequence attends over every cached token of its KV head (mni-ml page: keep
// past K/V, compute only the new token's); K and V are dequantised inside the
// attention kernel (KVSplit discussion: integrate the formats into the
// FlashAttention kernel), with INT8 / nibble-packed INT4 codes and fp16
// scales per (token, head) or per group (TinyLoop mode table; KVSplit 8K
// table).  Output = softmax(tau q.K^T) V, fp32 accumulation.
//
// Design for sm_100a (not taken from any page):
//   * Persistent CTAs, work split stream-K style: the units are 64-token tiles
//     of every (sequence, KV head); CTA c takes units [cN/P, (c+1)N/P).  Every
//     CTA therefore streams the same number of bytes whatever B, Hkv and the
//     lengths are.  A CTA's run of tiles inside one (sequence, KV head) is a
//     "segment"; each segment leaves one partial (m, l, o) in the workspace at
//     slot (cta + sequence*Hkv + kv_head), which is unique, and a small merge
//     kernel combines the partials with their log-sum-exp weights.
//   * One producer warp streams tiles with TMA: codes through 3-D tiled tensor
//     maps with 128-byte swizzle (bank-conflict-free fragment reads), scales
//     with 1-D bulk copies, into a multi-stage shared-memory ring guarded by
//     mbarriers.  Every wait is bounded (about a second) and a give-up sets
//     the workspace status word instead of hanging.
//   * Four consumer warps each take 16 tokens of a 64-token stage.  Codes are
//     turned into fp16 in registers with the exponent-bias trick (a code byte
//     u placed in the mantissa of 0x6400 reads 1024 + u), so no convert
//     instruction and no scale multiply touches an element: key scales scale
//     the 16x8 score tile, value scales are folded into the probabilities.
//     q.K^T and P.V run on warp-level tensor-core MMA (m16n8k16, f16 in, f32
//     accumulate) with tokens / head_dim as the M dimension and the G query
//     heads of the KV group as N.  The constant bias (1024+128 or 1024+8) is
//     removed in fp32 afterwards using sum(q) and sum(p).
//   * The online softmax tracks max(s + log2 s_V) so that p * s_V <= 1 fits
//     fp16 without underflow whatever the value scales are.
#include <cfloat>
#include <mutex>
#include <vector>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "../../include/kvq.h"

namespace kvq {
namespace {

constexpr int NW = kDecodeConsumerWarps;
constexpr int T = kDecodeTileTokens;
constexpr int NTHR = kDecodeThreads;

struct __align__(16) StageMeta {
    int32_t bh;      // sequence * Hkv + kv_head
    int32_t t0;      // first token of the tile
    int32_t len;     // tokens attended by this sequence
    int32_t flags;   // bit0 first tile of a segment, bit1 last tile, bits 8.. slot
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

// fp16 pair helpers: code bytes / nibbles -> half2 of (bias + code).
__device__ __forceinline__ uint32_t i8_lo_pair(uint32_t xw) { return prmt(xw, 0x64646464u, 0x4140u); }
__device__ __forceinline__ uint32_t i8_hi_pair(uint32_t xw) { return prmt(xw, 0x64646464u, 0x4342u); }
__device__ __forceinline__ uint32_t i4_pair(uint32_t w, int k)
{
    return and_xor(w >> (4 * k), 0x000F000Fu, 0x64086408u);
}

// Element offset (0..7 inside a lane's 8-element run of a 32-block) feeding
// k-slot j (0: 2tig, 1: 2tig+1, 2: 2tig+8, 3: 2tig+9) of k-step half hs.
template <int KB>
__device__ __forceinline__ int k_elem(int hs, int j)
{
    if constexpr (KB == 4) {
        return 2 * hs + ((j & 1) ? 4 : 0) + (j >> 1);
    } else {
        return 4 * hs + j;
    }
}

template <typename TQ>
__device__ __forceinline__ float ld_q(const void *q, int64_t idx)
{
    return static_cast<float>(static_cast<const TQ *>(q)[idx]);
}

__device__ __forceinline__ float load_qf(const void *q, int dtype, int64_t idx)
{
    if (dtype == KVQ_F16) return __half2float(static_cast<const __half *>(q)[idx]);
    if (dtype == KVQ_F32) return static_cast<const float *>(q)[idx];
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[idx]);
}

__device__ __forceinline__ int tiles_of(int len, int cap)
{
    len = len < 0 ? 0 : (len > cap ? cap : len);
    return (len + T - 1) / T;
}

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

// Address of block `blk` of a row whose block-0 address (stage base + per-lane
// swizzled offset) is `a0`, for a tile of R-byte rows whose 32-element blocks are
// STR bytes long: the swizzle is linear in the block index, so block blk sits at
// a0 ^ sw_off<R>(0, blk*STR).  Rows of 256 bytes keep their second half in a
// second box T*128 bytes further, which is added rather than XORed because the
// stage base is only 1024-byte aligned.
template <int R, int STR>
__device__ __forceinline__ uint32_t blk_addr(uint32_t a0, int blk)
{
    if constexpr (R <= 128) {
        return a0 ^ sw_off<R>(0, blk * STR);
    } else {
        const uint32_t x = sw_off<R>(0, blk * STR);
        return (a0 ^ (x & (T * 128 - 1))) + (x & ~(uint32_t)(T * 128 - 1));
    }
}

template <int DH, int KB, int VB>
__global__ void __launch_bounds__(NTHR, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const DecodeParams p)
{
    constexpr int NG = DH / 32;                // 32-element blocks along head_dim
    constexpr int RK = DH * KB / 8;            // bytes per key row
    constexpr int RV = DH * VB / 8;
    constexpr int SK = 32 * KB / 8;            // bytes per 32-element block of a key row
    constexpr int SV = 32 * VB / 8;
    constexpr float BIAS_K = KB == 8 ? 1152.f : (KB == 4 ? 1032.f : 0.f);
    constexpr float BIAS_V = VB == 8 ? 1152.f : (VB == 4 ? 1032.f : 0.f);
    // The running max is only raised when a tile beats it by more than 2^LAZY;
    // weights p * s_V then stay below 2^LAZY, well inside fp16.
    constexpr float LAZY = 8.f;
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // align to 1024 B (128-byte swizzle atoms) by pointer arithmetic on the shared
    // array itself, so every access below stays a shared-memory access
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);             // 32-bit shared address of the ring
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + p.off_meta);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *empty = full + p.stages;
    uint64_t *segbar = empty + p.stages;               // two: [0] partials written, [1] merged
    int *ctl = reinterpret_cast<int *>(segbar + 2);    // [0] abort, [1] units, [2..3] prefix
    float *mbuf = reinterpret_cast<float *>(smem + p.off_merge);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int S = p.stages;
    const int G = p.group_size_g;
    const int cap = p.cap;
    volatile int *abort_flag = ctl;

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NW);
        }
        mbar_init(&segbar[0], NW);
        mbar_init(&segbar[1], NW);
        ctl[0] = 0;
        fence_mbar_init();
    }

    // ---- work range of this CTA (computed by the producer warp) -------------
    __shared__ long long sh_u_begin;
    __shared__ int sh_b;
    if (warp == NW) {
        long long total = 0;
        for (int b = lane; b < p.batch; b += 32) total += tiles_of(p.d_len[b], cap);
        for (int off = 16; off; off >>= 1) total += __shfl_xor_sync(FULL, total, off);
        const long long N = total * p.n_kv_heads;
        const long long P = p.num_ctas;
        const long long ub = (long long)blockIdx.x * N / P;
        const long long ue = ((long long)blockIdx.x + 1) * N / P;
        // locate the sequence holding unit ub
        long long acc = 0;
        int fb = -1;
        long long fpre = 0;
        for (int base = 0; base < p.batch && fb < 0; base += 32) {
            const int b = base + lane;
            const long long units =
                (b < p.batch) ? (long long)tiles_of(p.d_len[b], cap) * p.n_kv_heads : 0;
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
            }
            acc += __shfl_sync(FULL, incl, 31);
        }
        if (lane == 0) {
            sh_u_begin = ub;
            sh_b = fb;
            ctl[1] = (int)(ue > ub && fb >= 0 ? ue - ub : 0);
            reinterpret_cast<long long *>(ctl + 2)[0] = fpre;
        }
    }
    __syncthreads();
    const int n_units = ctl[1];

    if (warp == NW) {
        // ====================== producer ======================
        if (lane != 0) return;
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        int b = sh_b;
        const long long pre = reinterpret_cast<long long *>(ctl + 2)[0];
        int len_b = (b >= 0) ? min(max(p.d_len[b], 0), cap) : 0;
        int tiles_b = (len_b + T - 1) / T;
        const int off = (int)(sh_u_begin - pre);   // unit offset inside sequence b
        int kvh = tiles_b ? off / tiles_b : 0;
        int tile = tiles_b ? off % tiles_b : 0;
        int s = 0;
        uint32_t ph = 0;                            // phase parity of this use of stage s
        int issued = 0;
        for (int i = 0; i < n_units; i++) {
            if (i >= S) {
                if (!mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, p.timeout_ns)) {
                    ctl[0] = 1;
                    atomicExch(p.status, KVQ_ERR_TIMEOUT);
                    break;
                }
            }
            const int bh = b * p.n_kv_heads + kvh;
            const int t0 = tile * T;
            int flags = 0;
            if (i == 0 || tile == 0) flags |= 1;
            if (i == n_units - 1 || tile == tiles_b - 1) flags |= 2;
            flags |= ((int)blockIdx.x + bh) << 8;
            StageMeta m;
            m.bh = bh; m.t0 = t0; m.len = len_b; m.flags = flags;
            meta[s] = m;

            uint8_t *st = smem + (size_t)s * p.stage_bytes;
            const int n_s = min(T, cap - t0);
            uint32_t bytes = (uint32_t)(T * RK + T * RV);
            if (KB != 16) bytes += (uint32_t)(n_s * p.ngs_k * 2);
            if (VB != 16) bytes += (uint32_t)(n_s * p.ngs_v * 2);
            mbar_arrive_expect_tx(&full[s], bytes);
            if constexpr (RK <= 128) {
                tma_load_3d(st, &tm_k, &full[s], 0, t0 / (128 / RK), bh);
            } else {
                tma_load_3d(st, &tm_k, &full[s], 0, t0, bh);
                tma_load_3d(st + T * 128, &tm_k, &full[s], 128, t0, bh);
            }
            if constexpr (RV <= 128) {
                tma_load_3d(st + p.off_v, &tm_v, &full[s], 0, t0 / (128 / RV), bh);
            } else {
                tma_load_3d(st + p.off_v, &tm_v, &full[s], 0, t0, bh);
                tma_load_3d(st + p.off_v + T * 128, &tm_v, &full[s], 128, t0, bh);
            }
            if (KB != 16)
                bulk_load(st + p.off_sk, p.k_scales + ((int64_t)bh * cap + t0) * p.ngs_k,
                          (uint32_t)(n_s * p.ngs_k * 2), &full[s]);
            if (VB != 16)
                bulk_load(st + p.off_sv, p.v_scales + ((int64_t)bh * cap + t0) * p.ngs_v,
                          (uint32_t)(n_s * p.ngs_v * 2), &full[s]);
            issued = i + 1;
            if (++s == S) {
                s = 0;
                ph ^= 1u;
            }
            // advance to the next unit (the length is re-read only when b changes)
            if (++tile == tiles_b) {
                tile = 0;
                if (++kvh == p.n_kv_heads) {
                    kvh = 0;
                    do {
                        ++b;
                        len_b = (b < p.batch) ? min(max(p.d_len[b], 0), cap) : T;
                        tiles_b = (len_b + T - 1) / T;
                    } while (tiles_b == 0);
                }
            }
        }
        // never leave with copies in flight: wait for the last issued phases
        int ss = s;
        uint32_t pp = ph;
        for (int j = 0; j < min(S, issued); j++) {
            if (ss == 0) {
                ss = S;
                pp ^= 1u;
            }
            --ss;
            (void)mbar_wait_bounded(&full[ss], pp, abort_flag, p.timeout_ns);
        }
        return;
    }

    // ====================== consumers ======================
    const int gid = lane >> 2;
    const int tig = lane & 3;
    const bool qsplit = p.q_dtype != KVQ_F16;
    const bool kgrp = p.ngs_k > 1;
    const bool vgrp = p.ngs_v > 1;
    const int colmax = qsplit ? 4 : 8;
    const bool col_ok0 = (2 * tig) < G && (2 * tig) < colmax;
    const bool col_ok1 = (2 * tig + 1) < G && (2 * tig + 1) < colmax;

    // per-lane swizzled offsets of block 0 of the rows this lane reads (relative
    // to a stage tile), for the two 16-token sub-tiles of the warp
    uint32_t kofs[2][2], vofs[2][4];
#pragma unroll
    for (int u = 0; u < 2; u++) {
        const int tw = warp * 32 + u * 16;
        kofs[u][0] = sw_off<RK>(tw + 2 * gid, tig * (SK / 4));
        kofs[u][1] = sw_off<RK>(tw + 2 * gid + 1, tig * (SK / 4));
        const int tv = tw + 2 * tig;
        vofs[u][0] = p.off_v + sw_off<RV>(tv, gid * (SV / 8));
        vofs[u][1] = p.off_v + sw_off<RV>(tv + 1, gid * (SV / 8));
        vofs[u][2] = p.off_v + sw_off<RV>(tv + 8, gid * (SV / 8));
        vofs[u][3] = p.off_v + sw_off<RV>(tv + 9, gid * (SV / 8));
    }
    // source lanes of the P transposition (score layout -> B-fragment layout)
    const int src0 = tig * 4 + (gid >> 1);
    const int src1 = (tig + 4) * 4 + (gid >> 1);
    const bool odd = gid & 1;

    uint32_t qb[NG][2][2];              // q B-fragments per (block, k-half)
    float qbias[NG][2];                 // BIAS_K * sum(q) per block, score cols 2tig, 2tig+1
    float m_run[2], l_run[2];
    float psum[NG][2];                  // sum of fp16 p*s_V per value block (or [0])
    float o_acc[2 * NG][4];             // O^T fragments, m-tile = 2*blk + u
    uint32_t seg_parity = 0;

    auto load_q = [&](int bh) {
        const int b = bh / p.n_kv_heads;
        const int kvh = bh % p.n_kv_heads;
        // B-fragment column n = gid: non-split: head n; split: hi (n<4) / lo (n>=4) of head n&3
        const int head = qsplit ? (gid & 3) : gid;
        const bool lo_part = qsplit && gid >= 4;
        const bool valid = head < G;
        const int64_t qbase = ((int64_t)b * p.n_q_heads + (int64_t)kvh * G + head) * DH;
#pragma unroll
        for (int blk = 0; blk < NG; blk++) {
            float colsum = 0.f;
#pragma unroll
            for (int hs = 0; hs < 2; hs++) {
                __half hv[4];
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const int d = 32 * blk + 8 * tig + k_elem<KB>(hs, j);
                    const float x = valid ? load_qf(p.q, p.q_dtype, qbase + d) : 0.f;
                    __half h = __float2half_rn(x);
                    if (lo_part) h = __float2half_rn(x - __half2float(h));
                    hv[j] = h;
                    colsum += __half2float(h);
                }
                __half2 b0 = __halves2half2(hv[0], hv[1]);
                __half2 b1 = __halves2half2(hv[2], hv[3]);
                qb[blk][hs][0] = *reinterpret_cast<uint32_t *>(&b0);
                qb[blk][hs][1] = *reinterpret_cast<uint32_t *>(&b1);
            }
            colsum += __shfl_xor_sync(FULL, colsum, 1);
            colsum += __shfl_xor_sync(FULL, colsum, 2);
            // score cols of this lane are 2tig and 2tig+1; column n lives on lanes with gid = n
            qbias[blk][0] = BIAS_K * __shfl_sync(FULL, colsum, (2 * tig) * 4);
            qbias[blk][1] = BIAS_K * __shfl_sync(FULL, colsum, (2 * tig + 1) * 4);
        }
        if (!kgrp) {
#pragma unroll
            for (int c = 0; c < 2; c++) {
                float t = 0.f;
#pragma unroll
                for (int blk = 0; blk < NG; blk++) t += qbias[blk][c];
                qbias[0][c] = t;
            }
        }
#pragma unroll
        for (int c = 0; c < 2; c++) {
            m_run[c] = -INFINITY;
            l_run[c] = 0.f;
        }
#pragma unroll
        for (int g = 0; g < NG; g++) psum[g][0] = psum[g][1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < 2 * NG; mt++)
#pragma unroll
            for (int i = 0; i < 4; i++) o_acc[mt][i] = 0.f;
    };

    // A fragments of block blk, k-half hs, for key rows at a[0] (row gid) and a[1] (row gid+8)
    auto key_frags = [&](uint32_t ra, uint32_t rb, int blk, uint32_t (&fa)[2][4]) {
        if constexpr (KB == 8) {
            const uint2 r0 = lds_u64(sbase, blk_addr<RK, SK>(ra, blk));
            const uint2 r1 = lds_u64(sbase, blk_addr<RK, SK>(rb, blk));
            const uint32_t x00 = r0.x ^ 0x80808080u, x01 = r0.y ^ 0x80808080u;
            const uint32_t x10 = r1.x ^ 0x80808080u, x11 = r1.y ^ 0x80808080u;
            fa[0][0] = i8_lo_pair(x00); fa[0][2] = i8_hi_pair(x00);
            fa[0][1] = i8_lo_pair(x10); fa[0][3] = i8_hi_pair(x10);
            fa[1][0] = i8_lo_pair(x01); fa[1][2] = i8_hi_pair(x01);
            fa[1][1] = i8_lo_pair(x11); fa[1][3] = i8_hi_pair(x11);
        } else if constexpr (KB == 4) {
            const uint32_t r0 = lds_u32(sbase, blk_addr<RK, SK>(ra, blk));
            const uint32_t r1 = lds_u32(sbase, blk_addr<RK, SK>(rb, blk));
            fa[0][0] = i4_pair(r0, 0); fa[0][2] = i4_pair(r0, 1);
            fa[0][1] = i4_pair(r1, 0); fa[0][3] = i4_pair(r1, 1);
            fa[1][0] = i4_pair(r0, 2); fa[1][2] = i4_pair(r0, 3);
            fa[1][1] = i4_pair(r1, 2); fa[1][3] = i4_pair(r1, 3);
        } else {
            const uint4 r0 = lds_u128(sbase, blk_addr<RK, SK>(ra, blk));
            const uint4 r1 = lds_u128(sbase, blk_addr<RK, SK>(rb, blk));
            fa[0][0] = r0.x; fa[0][2] = r0.y; fa[0][1] = r1.x; fa[0][3] = r1.y;
            fa[1][0] = r0.z; fa[1][2] = r0.w; fa[1][1] = r1.z; fa[1][3] = r1.w;
        }
    };

    const uint64_t limit = p.timeout_ns;
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < n_units; i++) {
        if (!mbar_wait_bounded(&full[s], ph, abort_flag, limit)) {
            ctl[0] = 1;
            atomicExch(p.status, KVQ_ERR_TIMEOUT);
            break;
        }
        StageMeta m;
        {
            const uint4 mm = *reinterpret_cast<const uint4 *>(&meta[s]);
            m.bh = (int)mm.x; m.t0 = (int)mm.y; m.len = (int)mm.z; m.flags = (int)mm.w;
        }
        if (m.flags & 1) load_q(m.bh);
        const uint32_t st = (uint32_t)s * p.stage_bytes;   // stage offset from smem
        const uint32_t ssk = st + p.off_sk;   // fp16 key scales of the stage
        const uint32_t ssv = st + p.off_sv;   // fp16 value scales

        // Work of this warp on the stage: two 16-token sub-tiles u = 0, 1, processed
        // phase by phase so that the two sub-tiles give the scheduler independent
        // instruction streams at every step.
        int tAu[2];
        bool vt[2][2];
#pragma unroll
        for (int u = 0; u < 2; u++) {
            tAu[u] = warp * 32 + u * 16 + 2 * gid;               // score rows: tAu, tAu + 1
            vt[u][0] = m.t0 + tAu[u] < m.len;
            vt[u][1] = m.t0 + tAu[u] + 1 < m.len;
        }

        // ---------------- phase 1: scores S^T = K q^T for both sub-tiles ----------
        float s2[2][4];
        if (!kgrp) {
            // two partial accumulators per sub-tile (even / odd blocks) halve the
            // dependent MMA chain
            float acc[2][2][4];
#pragma unroll
            for (int u = 0; u < 2; u++)
#pragma unroll
                for (int h = 0; h < 2; h++) acc[u][h][0] = acc[u][h][1] = acc[u][h][2] = acc[u][h][3] = 0.f;
#pragma unroll
            for (int blk = 0; blk < NG; blk++) {
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    uint32_t fa[2][4];
                    key_frags(st + kofs[u][0], st + kofs[u][1], blk, fa);
#pragma unroll
                    for (int hs = 0; hs < 2; hs++)
                        mma_16816(acc[u][blk & 1], fa[hs][0], fa[hs][1], fa[hs][2], fa[hs][3],
                                  qb[blk][hs][0], qb[blk][hs][1]);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; u++) {
                float ks0 = p.tau_log2e, ks1 = p.tau_log2e;
                if (KB != 16) {
                    const float2 kk = unpack_half2(lds_u32(sbase, ssk + 2 * tAu[u]));
                    ks0 *= kk.x;
                    ks1 *= kk.y;
                }
                s2[u][0] = (acc[u][0][0] + acc[u][1][0] - qbias[0][0]) * ks0;
                s2[u][1] = (acc[u][0][1] + acc[u][1][1] - qbias[0][1]) * ks0;
                s2[u][2] = (acc[u][0][2] + acc[u][1][2] - qbias[0][0]) * ks1;
                s2[u][3] = (acc[u][0][3] + acc[u][1][3] - qbias[0][1]) * ks1;
            }
        } else {
#pragma unroll
            for (int u = 0; u < 2; u++) {
                float acc[NG][4];
#pragma unroll
                for (int blk = 0; blk < NG; blk++) {
                    acc[blk][0] = acc[blk][1] = acc[blk][2] = acc[blk][3] = 0.f;
                    uint32_t fa[2][4];
                    key_frags(st + kofs[u][0], st + kofs[u][1], blk, fa);
#pragma unroll
                    for (int hs = 0; hs < 2; hs++)
                        mma_16816(acc[blk], fa[hs][0], fa[hs][1], fa[hs][2], fa[hs][3],
                                  qb[blk][hs][0], qb[blk][hs][1]);
                }
                float v[4] = {0.f, 0.f, 0.f, 0.f};
                const int tA = tAu[u];
#pragma unroll
                for (int blk = 0; blk < NG; blk++) {
                    const float k0 = __half2float(__ushort_as_half(
                        (unsigned short)lds_u16(sbase, ssk + 2 * (tA * p.ngs_k + (blk >> p.kshift)))));
                    const float k1 = __half2float(__ushort_as_half(
                        (unsigned short)lds_u16(sbase, ssk + 2 * ((tA + 1) * p.ngs_k + (blk >> p.kshift)))));
                    v[0] = fmaf(k0, acc[blk][0] - qbias[blk][0], v[0]);
                    v[1] = fmaf(k0, acc[blk][1] - qbias[blk][1], v[1]);
                    v[2] = fmaf(k1, acc[blk][2] - qbias[blk][0], v[2]);
                    v[3] = fmaf(k1, acc[blk][3] - qbias[blk][1], v[3]);
                }
#pragma unroll
                for (int e = 0; e < 4; e++) s2[u][e] = v[e] * p.tau_log2e;
            }
        }
#pragma unroll
        for (int u = 0; u < 2; u++) {
            if (qsplit) {
#pragma unroll
                for (int e = 0; e < 4; e++) s2[u][e] += __shfl_xor_sync(FULL, s2[u][e], 2);
            }
            // Padding columns (heads >= G, or the hi/lo halves of a split query)
            // carry finite scores from zero query columns; their outputs are never
            // written, so only tokens past the length are masked.
            s2[u][0] = vt[u][0] ? s2[u][0] : -INFINITY;
            s2[u][1] = vt[u][0] ? s2[u][1] : -INFINITY;
            s2[u][2] = vt[u][1] ? s2[u][2] : -INFINITY;
            s2[u][3] = vt[u][1] ? s2[u][3] : -INFINITY;
        }

        // ---------------- phase 2: value scales of the score rows -----------------
        float sv[2][2][NG];   // [sub-tile][row][value block]
        float lsv[2][2];
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const int tA = tAu[u];
            if (VB == 16) {
#pragma unroll
                for (int g = 0; g < NG; g++) sv[u][0][g] = sv[u][1][g] = 1.f;
            } else if (!vgrp) {
                const float2 vv = unpack_half2(lds_u32(sbase, ssv + 2 * tA));
#pragma unroll
                for (int g = 0; g < NG; g++) {
                    sv[u][0][g] = vv.x;
                    sv[u][1][g] = vv.y;
                }
            } else {
#pragma unroll
                for (int g = 0; g < NG; g++) {
                    sv[u][0][g] = __half2float(__ushort_as_half(
                        (unsigned short)lds_u16(sbase, ssv + 2 * (tA * p.ngs_v + (g >> p.vshift)))));
                    sv[u][1][g] = __half2float(__ushort_as_half(
                        (unsigned short)lds_u16(sbase, ssv + 2 * ((tA + 1) * p.ngs_v + (g >> p.vshift)))));
                }
            }
            // scales past the length may be stale shared memory: never use them
#pragma unroll
            for (int r = 0; r < 2; r++) {
                float mx = 0.f;
#pragma unroll
                for (int g = 0; g < NG; g++) {
                    sv[u][r][g] = vt[u][r] ? sv[u][r][g] : 0.f;
                    mx = fmaxf(mx, sv[u][r][g]);
                }
                lsv[u][r] = mx > 0.f ? fmaxf(__log2f(mx), -32.f) : -32.f;
            }
        }

        // ---------------- phase 3: online softmax, one lazy check for 32 tokens ---
        {
            float loc0 = -INFINITY, loc1 = -INFINITY;
#pragma unroll
            for (int u = 0; u < 2; u++) {
                loc0 = fmaxf(loc0, fmaxf(s2[u][0] + lsv[u][0], s2[u][2] + lsv[u][1]));
                loc1 = fmaxf(loc1, fmaxf(s2[u][1] + lsv[u][0], s2[u][3] + lsv[u][1]));
            }
            const bool need = (loc0 > m_run[0] + LAZY) || (loc1 > m_run[1] + LAZY);
            if (__any_sync(FULL, need)) {
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    loc0 = fmaxf(loc0, __shfl_xor_sync(FULL, loc0, off));
                    loc1 = fmaxf(loc1, __shfl_xor_sync(FULL, loc1, off));
                }
                const float mn0 = fmaxf(m_run[0], loc0), mn1 = fmaxf(m_run[1], loc1);
                const float a0 = (mn0 == -INFINITY) ? 1.f : fast_exp2(m_run[0] - mn0);
                const float a1 = (mn1 == -INFINITY) ? 1.f : fast_exp2(m_run[1] - mn1);
                m_run[0] = mn0;
                m_run[1] = mn1;
                l_run[0] *= a0;
                l_run[1] *= a1;
#pragma unroll
                for (int g = 0; g < NG; g++) {
                    psum[g][0] *= a0;
                    psum[g][1] *= a1;
                }
#pragma unroll
                for (int mt = 0; mt < 2 * NG; mt++) {
                    o_acc[mt][0] *= a0;
                    o_acc[mt][1] *= a1;
                    o_acc[mt][2] *= a0;
                    o_acc[mt][3] *= a1;
                }
            }
        }

        // ---------------- phase 4: P (fp16, value scale folded) -> B fragments ----
        uint32_t pb[2][NG][2];
        const int nvb = vgrp ? NG : 1;
#pragma unroll
        for (int u = 0; u < 2; u++) {
            float pr[4];
#pragma unroll
            for (int e = 0; e < 4; e++)
                pr[e] = (s2[u][e] == -INFINITY) ? 0.f : fast_exp2(s2[u][e] - m_run[e & 1]);
            l_run[0] += pr[0] + pr[2];
            l_run[1] += pr[1] + pr[3];
#pragma unroll
            for (int g = 0; g < NG; g++) {
                if (g < nvb) {
                    const uint32_t ha = pack_half2(pr[0] * sv[u][0][g], pr[2] * sv[u][1][g]);  // col 2tig
                    const uint32_t hb = pack_half2(pr[1] * sv[u][0][g], pr[3] * sv[u][1][g]);  // col 2tig+1
                    const float2 fa = unpack_half2(ha), fb = unpack_half2(hb);
                    psum[g][0] += fa.x + fa.y;
                    psum[g][1] += fb.x + fb.y;
                    const uint32_t x0 = __shfl_sync(FULL, ha, src0);
                    const uint32_t y0 = __shfl_sync(FULL, hb, src0);
                    const uint32_t x1 = __shfl_sync(FULL, ha, src1);
                    const uint32_t y1 = __shfl_sync(FULL, hb, src1);
                    pb[u][g][0] = odd ? y0 : x0;
                    pb[u][g][1] = odd ? y1 : x1;
                } else {
                    pb[u][g][0] = pb[u][0][0];
                    pb[u][g][1] = pb[u][0][1];
                }
            }
        }

        // ---------------- phase 5: O^T += V^T P for both sub-tiles ----------------
#pragma unroll
        for (int blk = 0; blk < NG; blk++) {
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const uint32_t va = st + vofs[u][0], vb = st + vofs[u][1];
                const uint32_t vc = st + vofs[u][2], ve = st + vofs[u][3];
                const uint32_t b0 = pb[u][blk][0], b1 = pb[u][blk][1];
                if constexpr (VB == 8) {
                    const uint32_t wA = lds_u32(sbase, blk_addr<RV, SV>(va, blk));
                    const uint32_t wB = lds_u32(sbase, blk_addr<RV, SV>(vb, blk));
                    const uint32_t wC = lds_u32(sbase, blk_addr<RV, SV>(vc, blk));
                    const uint32_t wE = lds_u32(sbase, blk_addr<RV, SV>(ve, blk));
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const uint32_t sel = h ? 0x7632u : 0x5410u;
                        const uint32_t yAB = prmt(wA, wB, sel), yCE = prmt(wC, wE, sel);
                        const uint32_t a0 = and_xor(yAB, 0x00FF00FFu, 0x64806480u);
                        const uint32_t a1 = and_xor(yAB >> 8, 0x00FF00FFu, 0x64806480u);
                        const uint32_t a2 = and_xor(yCE, 0x00FF00FFu, 0x64806480u);
                        const uint32_t a3 = and_xor(yCE >> 8, 0x00FF00FFu, 0x64806480u);
                        mma_16816(o_acc[2 * blk + h], a0, a1, a2, a3, b0, b1);
                    }
                } else if constexpr (VB == 4) {
                    const uint32_t hA = lds_u16(sbase, blk_addr<RV, SV>(va, blk));
                    const uint32_t hB = lds_u16(sbase, blk_addr<RV, SV>(vb, blk));
                    const uint32_t hC = lds_u16(sbase, blk_addr<RV, SV>(vc, blk));
                    const uint32_t hE = lds_u16(sbase, blk_addr<RV, SV>(ve, blk));
                    const uint32_t yAB = prmt(hA, hB, 0x5410u), yCE = prmt(hC, hE, 0x5410u);
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const uint32_t a0 = i4_pair(yAB, 2 * h);
                        const uint32_t a1 = i4_pair(yAB, 2 * h + 1);
                        const uint32_t a2 = i4_pair(yCE, 2 * h);
                        const uint32_t a3 = i4_pair(yCE, 2 * h + 1);
                        mma_16816(o_acc[2 * blk + h], a0, a1, a2, a3, b0, b1);
                    }
                } else {
                    // fp16 values past the length may be anything (NaN included): zero them
                    const int tg = m.t0 + warp * 32 + u * 16 + 2 * tig;
                    const uint2 z = make_uint2(0u, 0u);
                    const uint2 wA = tg < m.len ? lds_u64(sbase, blk_addr<RV, SV>(va, blk)) : z;
                    const uint2 wB = tg + 1 < m.len ? lds_u64(sbase, blk_addr<RV, SV>(vb, blk)) : z;
                    const uint2 wC = tg + 8 < m.len ? lds_u64(sbase, blk_addr<RV, SV>(vc, blk)) : z;
                    const uint2 wE = tg + 9 < m.len ? lds_u64(sbase, blk_addr<RV, SV>(ve, blk)) : z;
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const uint32_t A = h ? wA.y : wA.x, Bw = h ? wB.y : wB.x;
                        const uint32_t C = h ? wC.y : wC.x, E = h ? wE.y : wE.x;
                        const uint32_t a0 = prmt(A, Bw, 0x5410u), a1 = prmt(A, Bw, 0x7632u);
                        const uint32_t a2 = prmt(C, E, 0x5410u), a3 = prmt(C, E, 0x7632u);
                        mma_16816(o_acc[2 * blk + h], a0, a1, a2, a3, b0, b1);
                    }
                }
            }
        }

        // release the stage to the producer
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        if (++s == S) {
            s = 0;
            ph ^= 1u;
        }

        // ---------------- segment end: merge the warps, write the partial ---
        if (m.flags & 2) {
            float lt[2], ps[NG][2];
#pragma unroll
            for (int c = 0; c < 2; c++) {
                float v = l_run[c];
                v += __shfl_xor_sync(FULL, v, 4);
                v += __shfl_xor_sync(FULL, v, 8);
                v += __shfl_xor_sync(FULL, v, 16);
                lt[c] = v;
#pragma unroll
                for (int g = 0; g < NG; g++) {
                    float w = psum[g][c];
                    w += __shfl_xor_sync(FULL, w, 4);
                    w += __shfl_xor_sync(FULL, w, 8);
                    w += __shfl_xor_sync(FULL, w, 16);
                    ps[g][c] = w;
                }
            }
            // merge buffer: [NW][G][DH + 2] floats: o then (m, l)
            float *mine = mbuf + (size_t)warp * G * (DH + 2);
#pragma unroll
            for (int c = 0; c < 2; c++) {
                const int col = 2 * tig + c;
                if (c == 0 ? col_ok0 : col_ok1) {
                    float *oc = mine + (size_t)col * (DH + 2);
#pragma unroll
                    for (int blk = 0; blk < NG; blk++) {
                        const float corr = BIAS_V * ps[vgrp ? blk : 0][c];
#pragma unroll
                        for (int h = 0; h < 2; h++) {
                            const int d = 32 * blk + 4 * gid + 2 * h;
                            oc[d] = o_acc[2 * blk + h][c] - corr;
                            oc[d + 1] = o_acc[2 * blk + h][2 + c] - corr;
                        }
                    }
                    if (gid == 0) {
                        oc[DH] = m_run[c];
                        oc[DH + 1] = lt[c];
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&segbar[0]);
            if (!mbar_wait_bounded(&segbar[0], seg_parity, abort_flag, limit)) {
                ctl[0] = 1;
                atomicExch(p.status, KVQ_ERR_TIMEOUT);
                break;
            }
            // combine the NW warps deterministically and write the slot
            const int slot = m.flags >> 8;
            float *dst = p.ws + (size_t)slot * G * (DH + 2);
            for (int idx = tid; idx < G * DH; idx += 32 * NW) {
                const int col = idx / DH, d = idx % DH;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NW; w++) M = fmaxf(M, mbuf[((size_t)w * G + col) * (DH + 2) + DH]);
                float O = 0.f;
#pragma unroll
                for (int w = 0; w < NW; w++) {
                    const float *src = mbuf + ((size_t)w * G + col) * (DH + 2);
                    const float mw = src[DH];
                    const float e = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
                    O += e * src[d];
                }
                dst[(size_t)col * (DH + 2) + d] = O;
            }
            if (tid < G) {
                const int col = tid;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NW; w++) M = fmaxf(M, mbuf[((size_t)w * G + col) * (DH + 2) + DH]);
                float L = 0.f;
#pragma unroll
                for (int w = 0; w < NW; w++) {
                    const float *src = mbuf + ((size_t)w * G + col) * (DH + 2);
                    const float mw = src[DH];
                    L += (mw == -INFINITY) ? 0.f : exp2f(mw - M) * src[DH + 1];
                }
                dst[(size_t)col * (DH + 2) + DH] = M;
                dst[(size_t)col * (DH + 2) + DH + 1] = L;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&segbar[1]);
            if (!mbar_wait_bounded(&segbar[1], seg_parity, abort_flag, limit)) {
                ctl[0] = 1;
                atomicExch(p.status, KVQ_ERR_TIMEOUT);
                break;
            }
            seg_parity ^= 1u;
        }
    }
}

// ---------------------------------------------------------------------------
// merge: one warp per (sequence, query head)
// ---------------------------------------------------------------------------
template <int DH>
__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= (int64_t)p.batch * p.n_q_heads) return;
    const int b = (int)(gw / p.n_q_heads);
    const int h = (int)(gw % p.n_q_heads);
    const int G = p.group_size_g;
    const int kvh = h / G, col = h % G;
    const int cap = p.cap;

    // units before sequence b, and in total
    long long before = 0, total = 0;
    for (int bb = lane; bb < p.batch; bb += 32) {
        const long long t = tiles_of(p.d_len[bb], cap);
        total += t;
        if (bb < b) before += t;
    }
    for (int off = 16; off; off >>= 1) {
        total += __shfl_xor_sync(0xffffffffu, total, off);
        before += __shfl_xor_sync(0xffffffffu, before, off);
    }
    const int tiles_b = tiles_of(p.d_len[b], cap);
    const long long N = total * p.n_kv_heads;
    const long long P = p.num_ctas;
    const long long u0 = before * p.n_kv_heads + (long long)kvh * tiles_b;
    const long long u1 = u0 + tiles_b;
    const int bh = b * p.n_kv_heads + kvh;

    constexpr int PER = DH / 32;
    float o[PER];
#pragma unroll
    for (int i = 0; i < PER; i++) o[i] = 0.f;
    float M = -INFINITY, L = 0.f;
    if (tiles_b > 0) {
        const long long c_min = ((u0 + 1) * P + N - 1) / N - 1;
        const long long c_max = (u1 * P + N - 1) / N - 1;
        for (int pass = 0; pass < 2; pass++) {
            for (long long c = c_min; c <= c_max; c++) {
                const long long cs = c * N / P, ce = (c + 1) * N / P;
                if (!(max(cs, u0) < min(ce, u1))) continue;
                const float *slot = p.ws + (size_t)(c + bh) * G * (DH + 2) + (size_t)col * (DH + 2);
                const float mk = slot[DH];
                if (pass == 0) {
                    M = fmaxf(M, mk);
                } else if (mk != -INFINITY) {
                    const float e = exp2f(mk - M);
                    L += e * slot[DH + 1];
#pragma unroll
                    for (int i = 0; i < PER; i++) o[i] += e * slot[lane + 32 * i];
                }
            }
        }
    }
    const float inv = (L > 0.f) ? 1.f / L : 0.f;
    const int64_t obase = ((int64_t)b * p.n_q_heads + h) * DH;
#pragma unroll
    for (int i = 0; i < PER; i++) {
        const float v = o[i] * inv;
        if (p.out_f32)
            static_cast<float *>(p.out)[obase + lane + 32 * i] = v;
        else
            static_cast<__half *>(p.out)[obase + lane + 32 * i] = __float2half_rn(v);
    }
}

template <int DH, int KB, int VB>
void *decode_fn()
{
    return reinterpret_cast<void *>(&decode_kernel<DH, KB, VB>);
}

void *pick_decode(int dh, int kb, int vb)
{
#define KVQ_CASE(D, K, V) \
    if (dh == D && kb == K && vb == V) return decode_fn<D, K, V>();
#define KVQ_CASES_D(D)                                                                  \
    KVQ_CASE(D, 8, 8) KVQ_CASE(D, 8, 4) KVQ_CASE(D, 4, 8) KVQ_CASE(D, 4, 4)             \
    KVQ_CASE(D, 16, 16) KVQ_CASE(D, 8, 16) KVQ_CASE(D, 16, 8) KVQ_CASE(D, 4, 16)        \
    KVQ_CASE(D, 16, 4)
    KVQ_CASES_D(128)
    KVQ_CASES_D(64)
#undef KVQ_CASES_D
#undef KVQ_CASE
    return nullptr;
}

inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

}  // namespace

bool plan_decode(int dh, int kb, int vb, int ngs_k, int ngs_v, int G, int max_smem,
                 DecodeLaunch *plan)
{
    if (!pick_decode(dh, kb, vb)) return false;
    const uint32_t rk = dh * kb / 8, rv = dh * vb / 8;
    DecodeLaunch L{};
    L.dh = dh; L.kb = kb; L.vb = vb;
    L.off_v = align_up(T * rk, 1024);
    L.off_sk = L.off_v + align_up(T * rv, 1024);
    L.off_sv = L.off_sk + align_up(T * (kb == 16 ? 0 : ngs_k) * 2, 16);
    L.stage_bytes = align_up(L.off_sv + T * (vb == 16 ? 0 : ngs_v) * 2, 1024);
    const uint32_t merge_bytes = (uint32_t)NW * G * (dh + 2) * 4;
    // tail: meta[S] (16 B each), barriers (2S + 2) * 8, ctl 32 B, merge buffer
    for (int S = 8; S >= 2; S--) {
        const uint32_t off_meta = S * L.stage_bytes;
        const uint32_t off_bar = off_meta + S * 16;
        const uint32_t off_merge = align_up(off_bar + (2 * S + 2) * 8 + 32, 16);
        const uint32_t total = off_merge + merge_bytes + 1024;  // + alignment slack
        // keep two CTAs per SM when possible
        if (total <= (uint32_t)max_smem / 2 - 1024 || (S == 2 && total <= (uint32_t)max_smem)) {
            L.stages = S;
            L.off_meta = off_meta;
            L.off_bar = off_bar;
            L.off_merge = off_merge;
            L.smem_bytes = total;
            *plan = L;
            return true;
        }
    }
    return false;
}

// Per-device memos: the dynamic-shared-memory limit of a kernel instance is
// raised once to the device's opt-in maximum (the attribute is one value per
// function, so it must never be lowered by a later, smaller plan), and the
// occupancy of (instance, smem size) is remembered.  Neither changes a result;
// they only save microseconds of host time per call.
namespace {
struct AttrMemo {
    int dev;
    void *fn;
};
struct OccMemo {
    int dev;
    void *fn;
    size_t smem;
    int occupancy;
};
std::mutex g_memo_mu;
std::vector<AttrMemo> g_attr;
std::vector<OccMemo> g_occ;

cudaError_t prepare_fn(void *fn, size_t smem, int *occupancy)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(g_memo_mu);
    bool have_attr = false;
    for (const AttrMemo &m : g_attr)
        if (m.dev == dev && m.fn == fn) have_attr = true;
    if (!have_attr) {
        int max_optin = 0;
        e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, fn);
        if (e != cudaSuccess) return e;
        // the opt-in limit covers static + dynamic shared memory
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 max_optin - (int)fa.sharedSizeBytes);
        if (e != cudaSuccess) return e;
        g_attr.push_back(AttrMemo{dev, fn});
    }
    if (!occupancy) return cudaSuccess;
    for (const OccMemo &m : g_occ)
        if (m.dev == dev && m.fn == fn && m.smem == smem) {
            *occupancy = m.occupancy;
            return cudaSuccess;
        }
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, NTHR, smem);
    if (e != cudaSuccess) return e;
    g_occ.push_back(OccMemo{dev, fn, smem, occ});
    *occupancy = occ;
    return cudaSuccess;
}
}  // namespace

cudaError_t decode_occupancy(const DecodeLaunch &plan, int *ctas_per_sm)
{
    return prepare_fn(pick_decode(plan.dh, plan.kb, plan.vb), plan.smem_bytes, ctas_per_sm);
}

cudaError_t launch_decode(const DecodeLaunch &plan, const DecodeParams &p, const CUtensorMap &tm_k,
                          const CUtensorMap &tm_v, cudaStream_t stream)
{
    void *fn = pick_decode(plan.dh, plan.kb, plan.vb);
    cudaError_t e = prepare_fn(fn, plan.smem_bytes, nullptr);
    if (e != cudaSuccess) return e;
    void *args[] = {const_cast<CUtensorMap *>(&tm_k), const_cast<CUtensorMap *>(&tm_v),
                    const_cast<DecodeParams *>(&p)};
    return cudaLaunchKernel(fn, dim3(p.num_ctas), dim3(NTHR), args, plan.smem_bytes, stream);
}

cudaError_t launch_merge(const MergeParams &p, cudaStream_t stream)
{
    const int64_t warps = (int64_t)p.batch * p.n_q_heads;
    if (warps == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((warps + 7) / 8);
    (void)cudaGetLastError();  // drop a stale, already-reported error of an earlier call
    if (p.head_dim == 128)
        merge_kernel<128><<<blocks, 256, 0, stream>>>(p);
    else
        merge_kernel<64><<<blocks, 256, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace kvq
