// kvq_hgemm.cu -- h-mode K/V reconstruction GEMM on 5th-generation tensor cores.
//
// TinyLoop docs, "KV Cache 模式", section "運作原理": in h-mode the cache holds
// h = LN(residual) and every attention call rebuilds K = W_k h and V = W_v h for
// all cached positions, skipping the Q slice of attn_qkv; the page moves this GEMM
// from a scalar path to tensor cores.  Here, for every sequence b and token t:
//     [K_t | V_t] = W_kv . bf16(h^_t),   h^ = code * scale (dequantised in the
//     operand prologue), fp32 accumulation, rounded to fp16,
// written to K/V [B][Hkv][out_cap][Dh], the layout the 16-bit decode kernel reads.
//
// Two kernels:
//   dequant_h_kernel   h^ = code * scale rounded to bf16 (the GEMM operand), once per
//                      call, into a [B][len_pad][D] bf16 buffer (rows past the length
//                      are zero); memory-bound.
//   hgemm_kernel       persistent, one CTA per SM, 128 (tokens) x 256 (output
//                      features) tiles taken round-robin:
//     warp 0      TMA producer: A (bf16 h^) and W tiles of each 64-wide K stage,
//                 both with 128-byte swizzle, into a 4-stage shared-memory ring;
//     warp 1      allocates 2 x 256 TMEM columns (two accumulators) and, from one
//                 lane, issues tcgen05.mma (M=128, N=256, K=16, bf16 x bf16 ->
//                 fp32) four times per stage, committing each stage to its
//                 "empty" mbarrier and each finished tile to its buffer's
//                 "acc_full" mbarrier;
//     warps 2..5  drain the other accumulator while the next tile's MMAs run
//                 (tcgen05.ld, one 32-lane quarter each), store fp16 K/V rows and
//                 hand the buffer back through "acc_empty".
// Dequantising once instead of inside every (M, N) tile keeps the 16 N-tiles of a
// row block from redoing the same conversion.  Every wait is bounded; a give-up
// sets *status and the CTA drains and frees its TMEM before returning.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "../../include/kvq.h"

namespace kvq {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int NTHREADS = 192;                    // 6 warps
constexpr uint32_t A_BYTES = BM * BK * 2;        // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;        // 32 KB
constexpr uint32_t TMEM_COLS = 256;

struct GemmArgs {
    __half *k_out, *v_out;    // [B][Hkv][out_cap][Dh]
    int *status;              // may be null
    int32_t d_model, n_kv_heads, head_dim, len, out_cap, m_tiles, n_tiles, batch;
    uint32_t stage_bytes, stages;
    uint64_t timeout_ns;
    // fused attention (N tile = K_h | V_h of one KV head h)
    const void *q;            // [B][Hq][Dh]
    const int32_t *d_len;     // [B]
    float *part;              // [B][Hq][m_tiles * 4][Dh + 2]: o, m, l per (tile, warp)
    int32_t q_dtype, n_q_heads;
    float tau_log2e;
};

struct DequantArgs {
    const uint8_t *h_codes;   // [B][cap][D*bits/8]
    const __half *h_scales;   // [B][cap][h_groups]
    __nv_bfloat16 *out;       // [B][len_pad][D]
    int32_t cap, d_model, h_bits, h_groups, len, len_pad;
};

// Instruction descriptor: D f32, A/B bf16, both K-major, M = 128, N = 256.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint32_t bf2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// One block per (sequence, token) row, one thread per 8 elements (16 output bytes).
__global__ void __launch_bounds__(256) dequant_h_kernel(const DequantArgs a)
{
    // the GEMM that follows may be scheduled now; it waits for this grid to finish
    grid_launch_dependents();
    const int row = blockIdx.x;                      // b * len_pad + t
    const int b = row / a.len_pad, t = row % a.len_pad;
    const int nchunk = a.d_model / 8;
    const int gsz = a.d_model / a.h_groups;
    const bool live = t < a.len;
    const int64_t src_row = (int64_t)b * a.cap + t;
    for (int j = threadIdx.x; j < nchunk; j += blockDim.x) {
        uint4 o = make_uint4(0u, 0u, 0u, 0u);
        if (live) {
            uint32_t *ow = reinterpret_cast<uint32_t *>(&o);
            if (a.h_bits == 16) {
                const uint4 x = *reinterpret_cast<const uint4 *>(a.h_codes + (src_row * a.d_model + 8 * j) * 2);
                const __half2 *hx = reinterpret_cast<const __half2 *>(&x);
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const float2 f = __half22float2(hx[i]);
                    ow[i] = bf2(f.x, f.y);
                }
            } else {
                const float sv = __half2float(a.h_scales[src_row * a.h_groups + (8 * j) / gsz]);
                if (a.h_bits == 8) {
                    const uint2 x = *reinterpret_cast<const uint2 *>(a.h_codes + src_row * a.d_model + 8 * j);
                    const uint32_t w[2] = {x.x, x.y};
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const uint32_t ww = w[i >> 1];
                        const int sh = (i & 1) * 16;
                        ow[i] = bf2((float)(int8_t)((ww >> sh) & 0xff) * sv,
                                    (float)(int8_t)((ww >> (sh + 8)) & 0xff) * sv);
                    }
                } else {
                    // element 2i in the low nibble of byte i, 2i+1 in the high nibble
                    const uint32_t x = *reinterpret_cast<const uint32_t *>(a.h_codes + src_row * (a.d_model / 2) + 4 * j);
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        const int lo = (int)((x >> (8 * i)) & 0xf), hi = (int)((x >> (8 * i + 4)) & 0xf);
                        ow[i] = bf2((float)(lo >= 8 ? lo - 16 : lo) * sv, (float)(hi >= 8 ? hi - 16 : hi) * sv);
                    }
                }
            }
        }
        *reinterpret_cast<uint4 *>(a.out + ((int64_t)row * a.d_model + 8 * j)) = o;
    }
}

// Fused path, one epilogue warp over its 32 rows (tokens t0 + 32q + lane) of the
// tile [K_h | V_h] in TMEM (taddr: the warp's lane quarter, column 0).  For each query
// head of KV head h: s_t = tau log2(e) q . K_t (rows past the length masked), the
// warp's m = max s, l = sum 2^(s - m) and o = sum_t 2^(s_t - m) V_t, written as one
// partial (the column sums of o by a transposing butterfly: 31 shuffles per 32 columns).
__device__ __forceinline__ void fused_epilogue(const GemmArgs &g, uint32_t taddr, int b, int t0,
                                               int h, int q, int lane, float *qs)
{
    constexpr unsigned FULL = 0xffffffffu;
    const int G = g.n_q_heads / g.n_kv_heads;
    for (int k = lane; k < G * 128; k += 32) {
        const int64_t qi = ((int64_t)b * g.n_q_heads + h * G + (k >> 7)) * 128 + (k & 127);
        float v;
        if (g.q_dtype == KVQ_F32)
            v = static_cast<const float *>(g.q)[qi];
        else if (g.q_dtype == KVQ_F16)
            v = __half2float(static_cast<const __half *>(g.q)[qi]);
        else
            v = __bfloat162float(static_cast<const __nv_bfloat16 *>(g.q)[qi]);
        qs[k] = v;
    }
    __syncwarp();
    const int len_b = min(max(g.d_len[b], 0), g.len);
    const bool valid = t0 + 32 * q + lane < len_b;
    float sc[8];
#pragma unroll
    for (int gg = 0; gg < 8; gg++) sc[gg] = 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + (uint32_t)c0, v);
#pragma unroll
        for (int gg = 0; gg < 8; gg++) {
            if (gg >= G) break;
            float a = sc[gg];
#pragma unroll
            for (int j = 0; j < 32; j++) a = fmaf(__uint_as_float(v[j]), qs[gg * 128 + c0 + j], a);
            sc[gg] = a;
        }
    }
    float mw[8], lw[8], pw[8];
#pragma unroll
    for (int gg = 0; gg < 8; gg++) {
        if (gg >= G) break;
        const float sv = valid ? sc[gg] * g.tau_log2e : -INFINITY;
        float m = sv;
        for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
        const float pv = (m == -INFINITY || !valid) ? 0.f : exp2f(sv - m);
        float l = pv;
        for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(FULL, l, off);
        mw[gg] = m;
        lw[gg] = l;
        pw[gg] = pv;
    }
    const int P = g.m_tiles * 4;
    const int slot = (t0 / BM) * 4 + q;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + 128u + (uint32_t)c0, v);
#pragma unroll
        for (int gg = 0; gg < 8; gg++) {
            if (gg >= G) break;
            float x[32];
#pragma unroll
            // rows past the length may hold anything (stale scales): zero, not 0 * v
            for (int j = 0; j < 32; j++) x[j] = valid ? pw[gg] * __uint_as_float(v[j]) : 0.f;
#pragma unroll
            for (int w = 16; w >= 1; w >>= 1) {
                const bool upper = (lane & w) != 0;
#pragma unroll
                for (int i = 0; i < w; i++) {
                    const float send = upper ? x[i] : x[i + w];
                    const float keep = upper ? x[i + w] : x[i];
                    x[i] = keep + __shfl_xor_sync(FULL, send, w);
                }
            }
            float *dst = g.part + (((int64_t)b * g.n_q_heads + h * G + gg) * P + slot) * 130;
            dst[c0 + lane] = x[0];
            if (c0 == 0 && lane == 0) {
                dst[128] = mw[gg];
                dst[129] = lw[gg];
            }
        }
    }
}

// FUSED: the N tile of KV head h is [K_h | V_h] (W rows h*Dh.. and Hkv*Dh + h*Dh.., two
// 128-row boxes, Dh = 128) and the epilogue attends over the tile instead of storing it.
template <bool FUSED>
__global__ void __launch_bounds__(NTHREADS, 1)
    hgemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
                 const GemmArgs g)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t S = g.stages;
    // stage s: [A 16 KB][B 32 KB]; barriers after the ring
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * g.stage_bytes);
    uint64_t *full = bars;               // A + W tiles of a stage landed (TMA tx)
    uint64_t *empty = bars + S;          // MMAs of a stage finished (tcgen05.commit)
    uint64_t *acc_full = bars + 2 * S;   // [2] accumulator buffer complete (tcgen05.commit)
    uint64_t *acc_empty = bars + 2 * S + 2;   // [2] accumulator buffer drained (4 warps)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 4);
    int *abort_flag_p = reinterpret_cast<int *>(tmem_slot + 1);
    volatile int *abort_flag = abort_flag_p;
    // fused: per epilogue warp, the G <= 8 queries of the tile's KV head (fp32)
    float *qsm = reinterpret_cast<float *>(tmem_slot + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k_stages = g.d_model / BK;
    const int total = g.n_tiles * g.m_tiles * g.batch;
    const uint64_t limit = g.timeout_ns;

    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&acc_full[0], 1);
        mbar_init(&acc_full[1], 1);
        mbar_init(&acc_empty[0], 4);
        mbar_init(&acc_empty[1], 4);
        *abort_flag_p = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 2 * TMEM_COLS);   // two 256-column accumulators
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto give_up = [&]() {
        *abort_flag_p = 1;
        if (g.status) atomicExch(g.status, KVQ_ERR_TIMEOUT);
    };
    // tile index -> (n0, b, t0); N tiles vary fastest
    auto tile_coords = [&](int tile, int &n0, int &b, int &t0) {
        n0 = (tile % g.n_tiles) * BN;
        const int mt = tile / g.n_tiles;
        b = mt / g.m_tiles;
        t0 = (mt % g.m_tiles) * BM;
    };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (all tiles)
        if (lane == 0) {
            prefetch_tensormap(&tm_w);
            prefetch_tensormap(&tm_a);
            grid_dependency_wait();          // the operand pre-pass has finished
            uint32_t s = 0, ph = 0;
            int issued = 0;      // stage uses issued so far
            bool stop = false;
            for (int tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
                int n0, b, t0;
                tile_coords(tile, n0, b, t0);
                for (int k = 0; k < k_stages; k++) {
                    if (issued >= (int)S && !mbar_wait_bounded(&empty[s], ph ^ 1u, abort_flag, limit)) {
                        give_up();
                        stop = true;
                        break;
                    }
                    uint8_t *st = smem + s * g.stage_bytes;
                    mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
                    tma_load_3d(st, &tm_a, &full[s], k * BK, t0, b);
                    if constexpr (FUSED) {
                        // n0 / BN = KV head h: K_h rows, then V_h rows (128-row boxes)
                        const int h = n0 / BN;
                        tma_load_2d(st + A_BYTES, &tm_w, &full[s], k * BK, h * g.head_dim);
                        tma_load_2d(st + A_BYTES + B_BYTES / 2, &tm_w, &full[s], k * BK,
                                    (g.n_kv_heads + h) * g.head_dim);
                    } else {
                        tma_load_2d(st + A_BYTES, &tm_w, &full[s], k * BK, n0);
                    }
                    ++issued;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // drain: every issued copy must land before the CTA can exit
            uint32_t ss = s, pp = ph;
            for (int j = 0; j < min((int)S, issued); j++) {
                if (ss == 0) {
                    ss = S;
                    pp ^= 1u;
                }
                --ss;
                (void)mbar_wait_drain(&full[ss], pp, limit);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t s = 0, ph = 0;
            int done = 0;        // stage uses consumed
            int local = 0;       // tiles of this CTA
            bool stop = false;
            for (int tile = blockIdx.x; tile < total && !stop; tile += gridDim.x, ++local) {
                const int buf = local & 1;
                // the epilogue must have drained this buffer (its use two tiles ago)
                if (local >= 2 &&
                    !mbar_wait_bounded(&acc_empty[buf], ((local >> 1) - 1) & 1u, abort_flag, limit)) {
                    give_up();
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)buf * TMEM_COLS;
                for (int k = 0; k < k_stages; k++) {
                    if (!mbar_wait_bounded(&full[s], ph, abort_flag, limit)) {
                        give_up();
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(smem + s * g.stage_bytes);
                    const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; kk++) {
                        // K = 16 bf16 = 32 bytes further inside the 128-byte swizzle atom
                        umma_f16(d_tmem, sw128_desc(a_base + kk * 32), sw128_desc(b_base + kk * 32),
                                 kIdesc, (k > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                    ++done;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!stop) umma_commit(&acc_full[buf]);
            }
            if (*abort_flag && done > 0) {
                // aborted: wait (bounded) for the MMAs already issued to retire
                uint32_t ss = s, pp = ph;
                if (ss == 0) {
                    ss = S;
                    pp ^= 1u;
                }
                --ss;
                (void)mbar_wait_drain(&empty[ss], pp, limit);
            }
        }
    } else {
        // ------------------------------------------------ epilogue: TMEM -> fp16 K/V rows
        const int q = warp & 3;                       // TMEM lane quarter of this warp
        const int row = 32 * q + lane;                // accumulator row = tile row
        const int hd = g.n_kv_heads * g.head_dim;     // features of K (then of V)
        int local = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
            const int buf = local & 1;
            if (!mbar_wait_bounded(&acc_full[buf], (local >> 1) & 1u, abort_flag, limit)) {
                give_up();
                break;
            }
            tc_fence_after();
            int n0, b, t0;
            tile_coords(tile, n0, b, t0);
            const int tt = t0 + row;
            if constexpr (FUSED) {
                fused_epilogue(g, tmem + (uint32_t)buf * TMEM_COLS + ((uint32_t)(32 * q) << 16), b, t0,
                               n0 / BN, q, lane, qsm + (size_t)warp * 8 * 128);
            } else {
#pragma unroll 1
            for (int c0 = 0; c0 < BN; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + (uint32_t)buf * TMEM_COLS + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
                if (tt < g.len) {
                    const int n = n0 + c0;
                    __half *dst = n < hd ? g.k_out : g.v_out;
                    const int nn = n < hd ? n : n - hd;
                    const int head = nn / g.head_dim, d = nn % g.head_dim;
                    __half *p = dst + (((int64_t)b * g.n_kv_heads + head) * g.out_cap + tt) * g.head_dim + d;
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 o;
                        o.x = pack_half2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
                        o.y = pack_half2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
                        o.z = pack_half2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5]));
                        o.w = pack_half2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7]));
                        *reinterpret_cast<uint4 *>(p + j) = o;
                    }
                }
            }
            }
            // all TMEM reads of this buffer are done: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }

    // every role reaches this point; free TMEM after all tcgen05 work is done
    grid_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 2 * TMEM_COLS);
}

// Merge of the fused path's partials: one warp per (sequence, query head) over its
// m_tiles * 4 warp partials, out = sum_k o_k 2^(m_k - M) / sum_k l_k 2^(m_k - M).
__global__ void __launch_bounds__(128) fused_merge_kernel(const float *part, int P, int rows,
                                                          void *out, int out_f32)
{
    grid_dependency_wait();                          // the GEMM's partials are complete
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const float *pr = part + (int64_t)row * P * 130;
    float M = -INFINITY;
    for (int k = 0; k < P; k++) M = fmaxf(M, pr[(int64_t)k * 130 + 128]);
    float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
        for (int k = 0; k < P; k++) {
            const float m = pr[(int64_t)k * 130 + 128];
            if (m == -INFINITY) continue;
            const float e = exp2f(m - M);
            L = fmaf(e, pr[(int64_t)k * 130 + 129], L);
#pragma unroll
            for (int i = 0; i < 4; i++) o[i] = fmaf(e, pr[(int64_t)k * 130 + lane + 32 * i], o[i]);
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int64_t idx = (int64_t)row * 128 + lane + 32 * i;
        if (out_f32)
            static_cast<float *>(out)[idx] = o[i] * inv;
        else
            static_cast<__half *>(out)[idx] = __float2half_rn(o[i] * inv);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

}  // namespace

cudaError_t launch_h_reconstruct(const HGemmParams &p, cudaStream_t stream)
{
    const bool fused = p.part != nullptr;
    const int N = 2 * p.n_kv_heads * p.head_dim;
    if (p.head_dim % 32 != 0 || N % BN != 0 || p.d_model % BK != 0) return cudaErrorNotSupported;
    if (fused && (p.head_dim != BN / 2 || p.n_q_heads % p.n_kv_heads != 0 ||
                  p.n_q_heads / p.n_kv_heads > 8))
        return cudaErrorNotSupported;
    if (p.h_bits != 16 && (p.d_model / p.h_groups) % 8 != 0) return cudaErrorNotSupported;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    const int m_tiles = (p.len + BM - 1) / BM;
    const int len_pad = m_tiles * BM;

    // 1. h^ -> bf16 operand, once per call
    DequantArgs da{};
    da.h_codes = p.h_codes;
    da.h_scales = p.h_scales;
    da.out = reinterpret_cast<__nv_bfloat16 *>(p.operand);
    da.cap = p.cap;
    da.d_model = p.d_model;
    da.h_bits = p.h_bits;
    da.h_groups = p.h_groups;
    da.len = p.len;
    da.len_pad = len_pad;
    (void)cudaGetLastError();
    dequant_h_kernel<<<(unsigned)(p.batch * len_pad), 256, 0, stream>>>(da);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // 2. tensor maps: W bf16 [N][D] and the operand bf16 [B][len_pad][D], boxes of
    //    64 (K) x 256 (N) and 64 (K) x 128 (tokens), both with 128-byte swizzle
    CUtensorMap tm_w, tm_a;
    {
        cuuint64_t dims[2] = {(cuuint64_t)p.d_model, (cuuint64_t)N};
        cuuint64_t strides[1] = {(cuuint64_t)p.d_model * 2};
        // fused: two 128-row boxes per stage (K_h, then V_h)
        cuuint32_t box[2] = {BK, fused ? (cuuint32_t)(BN / 2) : (cuuint32_t)BN}, es[2] = {1, 1};
        if (fn(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(p.w), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        cuuint64_t dims[3] = {(cuuint64_t)p.d_model, (cuuint64_t)len_pad, (cuuint64_t)p.batch};
        cuuint64_t strides[2] = {(cuuint64_t)p.d_model * 2, (cuuint64_t)p.d_model * 2 * len_pad};
        cuuint32_t box[3] = {BK, BM, 1}, es[3] = {1, 1, 1};
        if (fn(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.operand, dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    GemmArgs g{};
    g.k_out = p.k_out;
    g.v_out = p.v_out;
    g.status = p.status;
    g.d_model = p.d_model;
    g.n_kv_heads = p.n_kv_heads;
    g.head_dim = p.head_dim;
    g.len = p.len;
    g.out_cap = p.out_cap;
    g.m_tiles = m_tiles;
    g.stage_bytes = A_BYTES + B_BYTES;
    g.stages = 4;
    g.timeout_ns = 1000000000ull;
    g.q = p.q;
    g.d_len = p.d_len;
    g.part = p.part;
    g.q_dtype = p.q_dtype;
    g.n_q_heads = p.n_q_heads;
    g.tau_log2e = p.tau_log2e;
    // + fused: 6 warps x 8 queries x 128 fp32 of query staging
    const size_t smem = (size_t)g.stages * g.stage_bytes + 1024 + 8 * (2 * g.stages + 4) + 16 +
                        (fused ? (size_t)NTHREADS / 32 * 8 * 128 * 4 : 0);
    void *kfn = fused ? reinterpret_cast<void *>(&hgemm_kernel<true>) : reinterpret_cast<void *>(&hgemm_kernel<false>);
    e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    g.n_tiles = fused ? p.n_kv_heads : N / BN;
    g.batch = p.batch;
    // persistent: one CTA per SM (the 197 KB ring allows no more), tiles round-robin
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        (void)cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = g.n_tiles * m_tiles * p.batch;
    const dim3 grid((unsigned)(tiles < sms ? tiles : sms), 1);
    void *args[] = {&tm_w, &tm_a, &g};
    // programmatic dependent launches: each kernel may be scheduled while the previous
    // one drains and waits (griddepcontrol.wait) before touching its outputs
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = dim3(NTHREADS);
    lc.dynamicSmemBytes = smem;
    lc.stream = stream;
    lc.attrs = attr;
    lc.numAttrs = 1;
    e = cudaLaunchKernelExC(&lc, kfn, args);
    if (e != cudaSuccess || !fused) return e;
    const int rows = p.batch * p.n_q_heads;
    const int P = m_tiles * 4;
    cudaLaunchConfig_t lm = {};
    lm.gridDim = dim3((rows + 3) / 4);
    lm.blockDim = dim3(128);
    lm.stream = stream;
    lm.attrs = attr;
    lm.numAttrs = 1;
    return cudaLaunchKernelEx(&lm, fused_merge_kernel, (const float *)p.part, P, rows, p.out, (int)p.out_f32);
}

}  // namespace kvq
