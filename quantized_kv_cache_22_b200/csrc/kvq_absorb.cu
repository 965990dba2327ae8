// kvq_absorb.cu -- h-mode decode attention by query absorption.
//
// TinyLoop docs, "運作原理": an h cache rebuilds K = W_k h^ and V = W_v h^ at
// every attention call.  Both maps are linear in h^, so for query head h of KV
// head j the same attention regroups as
//   qa = W_k,j^T q                  (one D-vector per query head)
//   s_t = tau * qa . h^_t,  p = softmax(s)
//   ob = sum_t p_t h^_t             (one D-vector per query head)
//   out = W_v,j ob
// which streams the h codes once and multiplies by W once per step instead of
// reconstructing every cached token (D x 2 Hkv Dh MACs per token).  Five
// launches on the caller's stream:
//   absorb_q_kernel       qa, split per (head, scale group) into int8 hi/lo parts
//                         laid out as the B fragments of the score MMA
//   absorb_scores_kernel  int8 tensor-core scores over a tile of h codes
//   absorb_softmax_kernel one warp per (sequence, head): p = softmax(s) in place
//   absorb_pv_kernel      ob per (sequence, scale group) on f16 tensor cores
//   absorb_out_kernel     out = W_v,j ob (CUDA cores, W_v read once)
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "../../include/kvq.h"

namespace kvq {

namespace {

constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ float load_qf(const void *q, int dtype, int64_t i)
{
    if (dtype == KVQ_F32) return static_cast<const float *>(q)[i];
    if (dtype == KVQ_F16) return __half2float(static_cast<const __half *>(q)[i]);
    return __bfloat162float(static_cast<const __nv_bfloat16 *>(q)[i]);
}

// Tokens attended by sequence b: d_len clamped to the capacity and to the
// scratch's score rows (capP >= max_len_host, which bounds d_len).
__device__ __forceinline__ int seq_len(const AbsorbParams &p, int b)
{
    return min(max(p.d_len[b], 0), min(p.cap, p.capP));
}

// ---------------------------------------------------------------- qa
// Grid (Hkv, ng, query chunks of 16): block `group` threads, thread d owns
// element g*group + d of qa for the chunk's queries (b, head j*G + g').  Per
// query and scale group, qa ~ (amax/127)(hi + lo/254) with hi, lo in
// [-127, 127]; the bytes land where the score MMA's B fragment wants them and
// the factor amax/(127*254) * tau*log2(e) (/16 for 4-bit codes, which enter the
// MMA as 16 * code) goes to qfac[b][g][head].
__global__ void __launch_bounds__(128) absorb_q_kernel(AbsorbParams p)
{
    const int j = blockIdx.x, g = blockIdx.y;
    const int d = threadIdx.x;              // < group
    const int G = p.Hq / p.Hkv;
    const int nq = p.B * G;
    const int q0 = blockIdx.z * 16;
    const int nqc = min(16, nq - q0);
    __shared__ float qs[16][128];           // the chunk's queries, Dh <= 128
    __shared__ float red[16][4];            // per-warp amax partials
    for (int k = d; k < nqc * p.Dh; k += blockDim.x) {
        const int c = k / p.Dh, i = k % p.Dh;
        const int qi = q0 + c, b = qi / G, h = j * G + qi % G;
        qs[c][i] = load_qf(p.q, p.q_dtype, ((int64_t)b * p.Hq + h) * p.Dh + i);
    }
    __syncthreads();
    float acc[16];
#pragma unroll
    for (int c = 0; c < 16; c++) acc[c] = 0.f;
    const int col = g * p.group + d;
    const __nv_bfloat16 *wc = p.w + (int64_t)j * p.Dh * p.D + col;
    for (int i = 0; i < p.Dh; i++) {
        const float w = __bfloat162float(wc[(int64_t)i * p.D]);
#pragma unroll
        for (int c = 0; c < 16; c++) acc[c] = fmaf(qs[c][i], w, acc[c]);
    }
    // amax per query over the group's threads
    const int warp = d >> 5, lane = d & 31, nw = blockDim.x >> 5;
#pragma unroll
    for (int c = 0; c < 16; c++) {
        float a = fabsf(acc[c]);
        for (int off = 16; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(FULL, a, off));
        if (lane == 0) red[c][warp] = a;
    }
    __syncthreads();
    const int KS = p.D / 32;
    const int ks = col / 32, e = col % 32;
    const int tig = e / 8;
    int reg, byte;
    if (p.bits == 8) {
        reg = (e % 8) / 4;     // k-slot 4tig+i <-> element 8tig+i, 16+4tig+i <-> 8tig+4+i
        byte = e % 4;
    } else {
        reg = (e % 8) % 2;     // k-slot 4tig+i <-> element 8tig+2i, 16+4tig+i <-> 8tig+2i+1
        byte = (e % 8) / 2;
    }
    uint8_t *qb = reinterpret_cast<uint8_t *>(p.qfrag);
#pragma unroll
    for (int c = 0; c < 16; c++) {
        if (c >= nqc) break;
        float amax = red[c][0];
        for (int w = 1; w < nw; w++) amax = fmaxf(amax, red[c][w]);
        const int qi = q0 + c, b = qi / G, h = j * G + qi % G;
        const float inv = amax > 0.f ? 127.f / amax : 0.f;
        const float y = acc[c] * inv;
        const float r = rintf(y);
        const int hi = (int)r;
        const int lo = __float2int_rn((y - r) * 254.f);
        const int nt = h / 8, ln = (h % 8) * 4 + tig;
        const int64_t base = ((((int64_t)b * KS + ks) * p.NT + nt) * 32 + ln) * 16;
        qb[base + reg * 4 + byte] = (uint8_t)(int8_t)hi;
        qb[base + 8 + reg * 4 + byte] = (uint8_t)(int8_t)lo;
        if (d == 0)
            p.qfac[((int64_t)b * p.ng + g) * (p.NT * 8) + h] =
                amax * (1.f / (127.f * 254.f)) * p.tau_log2e * (p.bits == 4 ? 0.0625f : 1.f);
    }
}

// ---------------------------------------------------------------- scores
// Grid (token tiles of T, B); T / 16 warps, each 16 tokens x all heads.
// Scores in log2 units, s[b][h][t] = sum_g s_h(t, g) * qfac[g][h] * (254 acc_hi + acc_lo),
// written for t < len only.
template <int BITS, int NT>
__global__ void __launch_bounds__(128) absorb_scores_kernel(AbsorbParams p, int T)
{
    extern __shared__ __align__(16) uint8_t sm[];
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * T;
    const int len = seq_len(p, b);
    if (t0 >= len) return;
    const int rowb = p.D * BITS / 8;
    const int rs = rowb + 16;                       // padded row stride: conflict-free rows
    const int KS = p.D / 32;
    uint8_t *tile = sm;                             // [T][rs]
    uint4 *qf = reinterpret_cast<uint4 *>(sm + (size_t)T * rs);          // [KS][NT][32]
    __half *sk = reinterpret_cast<__half *>(qf + (size_t)KS * NT * 32);  // [T][ng]
    float *fac = reinterpret_cast<float *>(sk + (((size_t)T * p.ng + 7) & ~(size_t)7));  // [ng][NT*8]
    const int tid = threadIdx.x;
    const int nrow = min(T, len - t0);
    // stage the tile's codes, scales and this sequence's query fragments
    const int chunks = rowb / 16;
    const uint4 *src = reinterpret_cast<const uint4 *>(p.h_codes + ((int64_t)b * p.cap + t0) * rowb);
    for (int k = tid; k < nrow * chunks; k += blockDim.x) {
        const int r = k / chunks, c = k % chunks;
        *reinterpret_cast<uint4 *>(tile + (size_t)r * rs + 16 * c) = __ldg(src + (size_t)r * chunks + c);
    }
    const uint4 *qsrc = p.qfrag + (size_t)b * KS * NT * 32;
    for (int k = tid; k < KS * NT * 32; k += blockDim.x) qf[k] = __ldg(qsrc + k);
    for (int k = tid; k < nrow * p.ng; k += blockDim.x)
        sk[k] = p.h_scales[((int64_t)b * p.cap + t0) * p.ng + k];
    for (int k = tid; k < p.ng * NT * 8; k += blockDim.x)
        fac[k] = p.qfac[(int64_t)b * p.ng * NT * 8 + k];
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    const int r0 = warp * 16 + gid, r1 = r0 + 8;
    if (warp * 16 >= nrow) return;
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; nt++) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    const int ksg = p.group / 32;                   // k-steps per scale group
    const uint32_t tbase = smem_u32(tile);
    for (int g = 0; g < p.ng; g++) {
        int ah[NT][4], al[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int e = 0; e < 4; e++) ah[nt][e] = al[nt][e] = 0;
        for (int kk = 0; kk < ksg; kk++) {
            const int ks = g * ksg + kk;
            uint32_t fa[4];
            if constexpr (BITS == 8) {
                uint2 x0, x1;
                asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x0.x), "=r"(x0.y)
                             : "r"(tbase + r0 * rs + 32 * ks + 8 * tig));
                asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x1.x), "=r"(x1.y)
                             : "r"(tbase + r1 * rs + 32 * ks + 8 * tig));
                fa[0] = x0.x; fa[1] = x1.x; fa[2] = x0.y; fa[3] = x1.y;
            } else {
                uint32_t x0, x1;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x0) : "r"(tbase + r0 * rs + 16 * ks + 4 * tig));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x1) : "r"(tbase + r1 * rs + 16 * ks + 4 * tig));
                fa[0] = (x0 << 4) & 0xF0F0F0F0u; fa[1] = (x1 << 4) & 0xF0F0F0F0u;
                fa[2] = x0 & 0xF0F0F0F0u;        fa[3] = x1 & 0xF0F0F0F0u;
            }
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                const uint4 bq = qf[((size_t)ks * NT + nt) * 32 + lane];
                imma_16832(ah[nt], fa[0], fa[1], fa[2], fa[3], bq.x, bq.y);
                imma_16832(al[nt], fa[0], fa[1], fa[2], fa[3], bq.z, bq.w);
            }
        }
        const float k0 = __half2float(sk[r0 * p.ng + g]);
        const float k1 = __half2float(sk[r1 * p.ng + g]);
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
            const float f0 = fac[g * NT * 8 + nt * 8 + 2 * tig];
            const float f1 = fac[g * NT * 8 + nt * 8 + 2 * tig + 1];
            s[nt][0] = fmaf((float)(ah[nt][0] * 254 + al[nt][0]), f0 * k0, s[nt][0]);
            s[nt][1] = fmaf((float)(ah[nt][1] * 254 + al[nt][1]), f1 * k0, s[nt][1]);
            s[nt][2] = fmaf((float)(ah[nt][2] * 254 + al[nt][2]), f0 * k1, s[nt][2]);
            s[nt][3] = fmaf((float)(ah[nt][3] * 254 + al[nt][3]), f1 * k1, s[nt][3]);
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int h = nt * 8 + 2 * tig + (e & 1);
            const int r = (e < 2) ? r0 : r1;
            if (h < p.Hq && r < nrow) p.p[((int64_t)b * p.Hq + h) * p.capP + t0 + r] = s[nt][e];
        }
}

// ---------------------------------------------------------------- softmax
// One warp per (sequence, head): p_t = 2^(s_t - m) / sum, in place.
__global__ void __launch_bounds__(128) absorb_softmax_kernel(AbsorbParams p)
{
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= p.B * p.Hq) return;
    const int b = row / p.Hq;
    const int len = seq_len(p, b);
    float *s = p.p + (int64_t)row * p.capP;
    float m = -INFINITY;
    for (int t = lane; t < len; t += 32) m = fmaxf(m, s[t]);
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
    float l = 0.f;
    for (int t = lane; t < len; t += 32) l += exp2f(s[t] - m);
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(FULL, l, off);
    const float inv = l > 0.f ? 1.f / l : 0.f;
    for (int t = lane; t < len; t += 32) s[t] = exp2f(s[t] - m) * inv;
}

// ---------------------------------------------------------------- p . h^
// Grid (D / group, B): block 128 (4 warps), one scale group's columns of ob for
// every head.  Per chunk of 64 tokens: P~[head][t] = fp16(p * s_h(t, g)) and
// the codes as exact fp16 integers in [t][d]; then O[head][d] += P~ . H on
// f16 tensor cores (M = heads, N = d, K = tokens; the H fragments by
// ldmatrix.trans), warp w owning a quarter of the group's columns.
template <int BITS, int MT>
__global__ void __launch_bounds__(128) absorb_pv_kernel(AbsorbParams p)
{
    constexpr int TC = 64, TS = TC + 8;            // tokens per chunk, padded row (halves)
    __shared__ __align__(16) __half pt[MT * 16][TS];
    constexpr int VS = 128 + 8;                    // padded row of vt (halves)
    __shared__ __align__(16) __half vt[TC][VS];
    const int g = blockIdx.x, b = blockIdx.y;
    const int GS = p.group;
    const int len = seq_len(p, b);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    const int ntw = GS / 32;                       // n-tiles of 8 columns per warp (1, 2 or 4)
    float acc[MT][4][4];
#pragma unroll
    for (int mt = 0; mt < MT; mt++)
#pragma unroll
        for (int n = 0; n < 4; n++) acc[mt][n][0] = acc[mt][n][1] = acc[mt][n][2] = acc[mt][n][3] = 0.f;
    const int rowb = p.D * BITS / 8;
    for (int c0 = 0; c0 < len; c0 += TC) {
        // P~ for MT*16 head rows x 64 tokens (zero past the length or the heads)
        for (int k = tid; k < MT * 16 * TC; k += blockDim.x) {
            const int h = k / TC, t = k % TC, tt = c0 + t;
            float v = 0.f;
            if (h < p.Hq && tt < len)
                v = p.p[((int64_t)b * p.Hq + h) * p.capP + tt] *
                    __half2float(p.h_scales[((int64_t)b * p.cap + tt) * p.ng + g]);
            pt[h][t] = __float2half_rn(v);
        }
        // codes of the group's columns, 8 per thread-item, as fp16 integers in [d][t]
        for (int k = tid; k < TC * (GS / 8); k += blockDim.x) {
            const int t = k / (GS / 8), d8 = 8 * (k % (GS / 8)), tt = c0 + t;
            int c[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (tt < len) {
                const uint8_t *row = p.h_codes + ((int64_t)b * p.cap + tt) * rowb;
                if constexpr (BITS == 8) {
                    const uint2 w = *reinterpret_cast<const uint2 *>(row + g * GS + d8);
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        c[i] = (int)(int8_t)(w.x >> (8 * i));
                        c[4 + i] = (int)(int8_t)(w.y >> (8 * i));
                    }
                } else {
                    const uint32_t w = *reinterpret_cast<const uint32_t *>(row + (g * GS + d8) / 2);
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const int nib = (int)((w >> (4 * i)) & 0xFu);
                        c[i] = nib >= 8 ? nib - 16 : nib;
                    }
                }
            }
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
                const __half2 h2 = __halves2half2(__int2half_rn(c[2 * i]), __int2half_rn(c[2 * i + 1]));
                pk[i] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            *reinterpret_cast<uint4 *>(&vt[t][d8]) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        __syncthreads();
        const uint32_t pb = smem_u32(&pt[0][0]), vb = smem_u32(&vt[0][0]);
#pragma unroll
        for (int kk = 0; kk < TC / 16; kk++) {
            uint32_t a[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; mt++) {
                const uint32_t r0 = pb + ((mt * 16 + gid) * TS + 16 * kk + 2 * tig) * 2;
                const uint32_t r1 = r0 + 8 * TS * 2;
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[mt][0]) : "r"(r0));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[mt][1]) : "r"(r1));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[mt][2]) : "r"(r0 + 16));
                asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[mt][3]) : "r"(r1 + 16));
            }
#pragma unroll
            for (int n = 0; n < 4; n++) {
                if (n >= ntw) break;
                const int d0 = (warp * ntw + n) * 8;
                // lanes 0-7: rows (tokens) 16kk .. +7, lanes 8-15: the next 8, at column d0
                const int lr = lane & 15;
                const uint32_t bb = vb + ((16 * kk + (lr & 7) + 8 * (lr >> 3)) * VS + d0) * 2;
                uint32_t b0, b1;
                asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                             : "=r"(b0), "=r"(b1) : "r"(bb));
#pragma unroll
                for (int mt = 0; mt < MT; mt++)
                    mma_16816(acc[mt][n], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int n = 0; n < 4; n++) {
        if (n >= ntw) break;
        const int d = g * GS + (warp * ntw + n) * 8 + 2 * tig;
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
            const int h0 = mt * 16 + gid, h1 = h0 + 8;
            if (h0 < p.Hq)
                *reinterpret_cast<float2 *>(p.ob + ((int64_t)b * p.Hq + h0) * p.D + d) =
                    make_float2(acc[mt][n][0], acc[mt][n][1]);
            if (h1 < p.Hq)
                *reinterpret_cast<float2 *>(p.ob + ((int64_t)b * p.Hq + h1) * p.D + d) =
                    make_float2(acc[mt][n][2], acc[mt][n][3]);
        }
    }
}

// ---------------------------------------------------------------- W_v . ob
// Grid (Hkv, Dh / 32): 8 warps x 4 rows of W_v,j; the chunk's queries' ob in
// shared memory, each W_v row read once into registers (64 bf16 per lane).
__global__ void __launch_bounds__(256) absorb_out_kernel(AbsorbParams p)
{
    extern __shared__ __align__(16) float obs[];    // [8][D]
    const int j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.Hq / p.Hkv;
    const int nq = p.B * G;
    const int per = p.D / 256;                      // uint4 (8 bf16) per lane per row
    for (int q0 = 0; q0 < nq; q0 += 8) {
        const int nqc = min(8, nq - q0);
        __syncthreads();
        for (int k = threadIdx.x; k < nqc * p.D / 4; k += blockDim.x) {
            const int c = k / (p.D / 4), d4 = k % (p.D / 4);
            const int qi = q0 + c, b = qi / G, h = j * G + qi % G;
            reinterpret_cast<float4 *>(obs)[(size_t)c * (p.D / 4) + d4] =
                reinterpret_cast<const float4 *>(p.ob + ((int64_t)b * p.Hq + h) * p.D)[d4];
        }
        __syncthreads();
        for (int rr = 0; rr < 4; rr++) {
            const int i = blockIdx.y * 32 + warp * 4 + rr;
            const uint4 *wr = reinterpret_cast<const uint4 *>(
                p.w + ((int64_t)p.Hkv * p.Dh + (int64_t)j * p.Dh + i) * p.D);
            float acc[8];
#pragma unroll
            for (int c = 0; c < 8; c++) acc[c] = 0.f;
            for (int k = 0; k < per; k++) {
                const int d0 = 8 * (lane + 32 * k);
                const uint4 w = __ldg(wr + lane + 32 * k);
                float wf[8];
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    wf[2 * e] = __uint_as_float(ws[e] << 16);
                    wf[2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
                }
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    if (c < nqc) {
                        const float4 o0 = *reinterpret_cast<const float4 *>(obs + (size_t)c * p.D + d0);
                        const float4 o1 = *reinterpret_cast<const float4 *>(obs + (size_t)c * p.D + d0 + 4);
                        acc[c] = fmaf(wf[0], o0.x, acc[c]);
                        acc[c] = fmaf(wf[1], o0.y, acc[c]);
                        acc[c] = fmaf(wf[2], o0.z, acc[c]);
                        acc[c] = fmaf(wf[3], o0.w, acc[c]);
                        acc[c] = fmaf(wf[4], o1.x, acc[c]);
                        acc[c] = fmaf(wf[5], o1.y, acc[c]);
                        acc[c] = fmaf(wf[6], o1.z, acc[c]);
                        acc[c] = fmaf(wf[7], o1.w, acc[c]);
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < 8; c++) {
                float v = acc[c];
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(FULL, v, off);
                if (lane == 0 && c < nqc) {
                    const int qi = q0 + c, b = qi / G, h = j * G + qi % G;
                    const int64_t o = ((int64_t)b * p.Hq + h) * p.Dh + i;
                    if (p.out_f32)
                        static_cast<float *>(p.out)[o] = v;
                    else
                        static_cast<__half *>(p.out)[o] = __float2half_rn(v);
                }
            }
        }
    }
}

}  // namespace

int absorb_nt(int Hq) { return Hq <= 8 ? 1 : (Hq <= 16 ? 2 : 4); }

uint64_t absorb_scratch_layout(int B, int Hq, int D, int ng, int max_len, uint64_t off[4])
{
    const int NT = absorb_nt(Hq);
    const uint64_t capP = (uint64_t)((max_len + 63) / 64 * 64);
    const uint64_t sz[4] = {(uint64_t)B * (D / 32) * NT * 32 * 16, (uint64_t)B * ng * NT * 8 * 4,
                            (uint64_t)B * Hq * capP * 4, (uint64_t)B * Hq * D * 4};
    uint64_t o = 0;
    for (int i = 0; i < 4; i++) {
        off[i] = o;
        o += (sz[i] + 255) / 256 * 256;
    }
    return o;
}

namespace {

template <int BITS, int NT>
cudaError_t launch_scores(const AbsorbParams &p, int max_len, cudaStream_t stream)
{
    const int rowb = p.D * BITS / 8;
    const int KS = p.D / 32;
    // tokens per CTA: 64 (4 warps), or 32 when the tile and fragments outgrow shared memory
    for (int T = 64; T >= 16; T /= 2) {
        const size_t smem = (size_t)T * (rowb + 16) + (size_t)KS * NT * 512 +
                            (((size_t)T * p.ng + 7) & ~(size_t)7) * 2 + (size_t)p.ng * NT * 8 * 4;
        if (smem > 227 * 1024) continue;
        cudaError_t e = cudaFuncSetAttribute(absorb_scores_kernel<BITS, NT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        dim3 grid((max_len + T - 1) / T, p.B);
        absorb_scores_kernel<BITS, NT><<<grid, 128, smem, stream>>>(p, T);
        return cudaGetLastError();
    }
    return cudaErrorInvalidValue;
}

template <int BITS>
cudaError_t launch_scores_nt(const AbsorbParams &p, int max_len, cudaStream_t stream)
{
    switch (p.NT) {
    case 1: return launch_scores<BITS, 1>(p, max_len, stream);
    case 2: return launch_scores<BITS, 2>(p, max_len, stream);
    case 4: return launch_scores<BITS, 4>(p, max_len, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_absorbed(const AbsorbParams &p, int max_len, cudaStream_t stream)
{
    (void)cudaGetLastError();   // drop a stale, already-reported error of an earlier call
    const int G = p.Hq / p.Hkv;
    if (p.NT * 8 != p.Hq) {
        // padding heads of the last n-tile must hold zero fragments
        cudaError_t e = cudaMemsetAsync(p.qfrag, 0, (size_t)p.B * (p.D / 32) * p.NT * 512, stream);
        if (e != cudaSuccess) return e;
    }
    absorb_q_kernel<<<dim3(p.Hkv, p.ng, (p.B * G + 15) / 16), p.group, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (max_len > 0) {
        e = p.bits == 8 ? launch_scores_nt<8>(p, max_len, stream) : launch_scores_nt<4>(p, max_len, stream);
        if (e != cudaSuccess) return e;
        absorb_softmax_kernel<<<(p.B * p.Hq + 3) / 4, 128, 0, stream>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    const dim3 pv(p.D / p.group, p.B);
    const bool two = p.Hq > 16;
    if (p.bits == 8)
        two ? absorb_pv_kernel<8, 2><<<pv, 128, 0, stream>>>(p) : absorb_pv_kernel<8, 1><<<pv, 128, 0, stream>>>(p);
    else
        two ? absorb_pv_kernel<4, 2><<<pv, 128, 0, stream>>>(p) : absorb_pv_kernel<4, 1><<<pv, 128, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t osm = (size_t)8 * p.D * 4;
    e = cudaFuncSetAttribute(absorb_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)osm);
    if (e != cudaSuccess) return e;
    absorb_out_kernel<<<dim3(p.Hkv, p.Dh / 32), 256, osm, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace kvq
