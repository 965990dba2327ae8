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
// reconstructing every cached token (D x 2 Hkv Dh MACs per token).  Four
// launches on the caller's stream, each a programmatic dependent of the one
// before (it waits for that one's completion before touching its outputs):
//   absorb_q_kernel       qa, split per (head, scale group) into int8 hi/lo parts
//                         laid out as the B fragments of the score MMA
//   absorb_scores_kernel  int8 tensor-core scores over a tile of h codes, plus the
//                         tile's softmax statistics (max, sum of 2^(s - max))
//   absorb_pv_kernel      per (scale group, sequence, token split): p from the
//                         scores and the merged statistics, p . h^ on f16 tensor
//                         cores, added into ob (fp32 reductions in L2)
//   absorb_out_kernel     out = W_v,j ob (CUDA cores)
// The first launch also asks the copy engine to bring the h codes, their scales and
// W_v into L2 while it works on W_k, so that the later launches read them from L2:
// the call's DRAM reads overlap instead of following one another.
// Global data is staged into shared memory with cp.async, all copies of a stage
// in flight at once.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "../../include/kvq.h"

namespace kvq {

namespace {

constexpr unsigned FULL = 0xffffffffu;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Tokens attended by sequence b: d_len clamped to the capacity and to the
// scratch's score rows (capP >= max_len_host, which bounds d_len).
__device__ __forceinline__ int seq_len(const AbsorbParams &p, int b)
{
    return min(max(p.d_len[b], 0), min(p.cap, p.capP));
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d)
{
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

// bf16 hi and lo parts of the pair (a, b): a ~ hi + lo to 16 significant bits
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t &hi, uint32_t &lo)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

// ---------------------------------------------------------------- qa
// Grid (Hkv, D / 128, query chunks of 8), 128 threads: the CTA's 128 columns of
// W_k,j^T q for the chunk's queries on tensor cores (see below), then thread
// (q, cg) quantises 8 columns of query q.  Per query and scale group, qa ~ (amax/127)(hi + lo/254), hi, lo in [-127, 127]; a thread's 8
// columns are exactly one lane's slot of the score MMA's B fragment (k-slot order
// of 8-bit or 4-bit codes), written as one 16-byte store {hi0, hi1, lo0, lo1}.
// The factor amax/(127*254) * tau*log2(e) (/16 for 4-bit codes, which enter the
// MMA as 16 * code) goes to qfac[b][g][head].
template <int DH>
__global__ void __launch_bounds__(128) absorb_q_kernel(AbsorbParams p)
{
    constexpr int WS = 128 + 8;   // padded row stride of the W tile (conflict-free ldmatrix)
    __shared__ __align__(16) float qs[8][DH + 8];
    __shared__ __align__(16) __nv_bfloat16 wt[DH * WS];   // W_k,j [DH][the tile's 128 columns]
    __shared__ __align__(16) float part[8][128 + 4];      // qa of the chunk [query][column]
    const int j = blockIdx.x, tile = blockIdx.y;
    const int tid = threadIdx.x;
    const int G = p.Hq / p.Hkv;
    const int nq = p.B * G;
    const int q0 = blockIdx.z * 8;
    const int nqc = min(8, nq - q0);
    // L2 prefetch of the later launches' inputs (this CTA's share of 32 KB pieces):
    // the h codes and scales of every sequence up to the scratch's rows, and W_v.
    // L2 is where global writes land, so lines brought in before an earlier
    // launch's writes to them cannot be stale.
    {
        const int cid = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
        const int ncta = gridDim.x * gridDim.y * gridDim.z;
        constexpr uint32_t PIECE = 32768;
        const int rows = min(p.cap, p.capP);
        const uint64_t code_b = (uint64_t)rows * (p.D * p.bits / 8);      // per sequence
        const uint64_t scale_b = (uint64_t)rows * p.ng * 2 / 16 * 16;
        const uint64_t wv_b = (uint64_t)p.Hkv * p.Dh * p.D * 2;
        const uint64_t nc = (code_b + PIECE - 1) / PIECE, ns = (scale_b + PIECE - 1) / PIECE;
        const uint64_t nw = (wv_b + PIECE - 1) / PIECE;
        const uint64_t total = (uint64_t)p.B * (nc + ns) + nw;
        for (uint64_t k = cid + (uint64_t)ncta * tid; k < total; k += (uint64_t)ncta * blockDim.x) {
            const uint8_t *base;
            uint64_t off, len;
            if (k < (uint64_t)p.B * nc) {
                const uint64_t b = k / nc;
                base = p.h_codes + b * p.cap * (p.D * p.bits / 8);
                off = (k % nc) * PIECE;
                len = code_b;
            } else if (k < (uint64_t)p.B * (nc + ns)) {
                const uint64_t kk = k - (uint64_t)p.B * nc, b = kk / ns;
                base = reinterpret_cast<const uint8_t *>(p.h_scales + b * p.cap * p.ng);
                off = (kk % ns) * PIECE;
                len = scale_b;
            } else {
                base = reinterpret_cast<const uint8_t *>(p.w + (int64_t)p.Hkv * p.Dh * p.D);
                off = (k - (uint64_t)p.B * (nc + ns)) * PIECE;
                len = wv_b;
            }
            const uint32_t n = (uint32_t)(len - off < PIECE ? len - off : PIECE);
            if (n >= 16 && (reinterpret_cast<uintptr_t>(base + off) & 15u) == 0)
                bulk_prefetch_l2(base + off, n / 16 * 16);
        }
    }
    // W_k does not depend on earlier launches: its copies start before the wait
    {
        const uint32_t wb = smem_u32(wt);
        const __nv_bfloat16 *src = p.w + (int64_t)j * DH * p.D + tile * 128;
#pragma unroll
        for (int r = 0; r < DH * 16 / 128; r++) {
            const int k = tid + 128 * r, row = k / 16, c = k % 16;
            cp_async16(wb + row * (2 * WS) + 16 * c, src + (int64_t)row * p.D + 8 * c);
        }
    }
    // element offset of each query row of the chunk in q (no run-time division per load)
    __shared__ int64_t qoff[8];
    if (tid < 8) {
        const int qi = q0 + min(tid, nqc - 1);
        qoff[tid] = ((int64_t)(qi / G) * p.Hq + j * G + qi % G) * DH;
    }
    __syncthreads();
    grid_dependency_wait();
    // ob, which the p . h^ launch accumulates into, starts at zero
    {
        const int cid = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
        const int ncta = gridDim.x * gridDim.y * gridDim.z;
        const int64_t n4 = (int64_t)p.B * p.Hq * p.D / 4;
        for (int64_t k = cid + (int64_t)ncta * tid; k < n4; k += (int64_t)ncta * blockDim.x)
            reinterpret_cast<float4 *>(p.obp)[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    {
        // all loads in flight before the stores (one dtype branch for the lot)
        constexpr int R = 8 * DH / 128;
        float v[R];
        int64_t idx[R];
#pragma unroll
        for (int r = 0; r < R; r++) {
            const int k = tid + 128 * r;
            idx[r] = qoff[k / DH] + k % DH;
        }
        if (p.q_dtype == KVQ_F32) {
#pragma unroll
            for (int r = 0; r < R; r++) v[r] = __ldg(static_cast<const float *>(p.q) + idx[r]);
        } else if (p.q_dtype == KVQ_F16) {
#pragma unroll
            for (int r = 0; r < R; r++) v[r] = __half2float(static_cast<const __half *>(p.q)[idx[r]]);
        } else {
#pragma unroll
            for (int r = 0; r < R; r++) v[r] = __bfloat162float(static_cast<const __nv_bfloat16 *>(p.q)[idx[r]]);
        }
#pragma unroll
        for (int r = 0; r < R; r++)
            if ((tid + 128 * r) / DH >= nqc) v[r] = 0.f;
#pragma unroll
        for (int r = 0; r < 8 * DH / 128; r++) {
            const int k = tid + 128 * r;
            qs[k / DH][k % DH] = v[r];
        }
    }
    __syncthreads();
    // qa^T (the tile's 128 columns x 8 queries) = W^T (columns x DH) q^T (DH x 8 queries) on
    // bf16 tensor cores, warp w taking columns 32w .. 32w + 31: A fragments by transposed
    // ldmatrix from the W tile, B fragments from the queries split into bf16 hi and lo
    // parts (q = hi + lo to 16 significant bits; W_k is bf16 itself), fp32 accumulation.
    const int warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    uint32_t bhi[DH / 16][2], blo[DH / 16][2];
#pragma unroll
    for (int ks = 0; ks < DH / 16; ks++)
#pragma unroll
        for (int h = 0; h < 2; h++) {
            const float2 v = *reinterpret_cast<const float2 *>(&qs[gid][16 * ks + 8 * h + 2 * tig]);
            split_bf16x2(v.x, v.y, bhi[ks][h], blo[ks][h]);
        }
    float acc[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; mt++) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    cp_async_wait_all();
    __syncthreads();
    {
        // matrices (k 0-7, m 0-7), (k 0-7, m 8-15), (k 8-15, m 0-7), (k 8-15, m 8-15) of the
        // tile stored [k][m]: lane l gives row (l & 7) + 8 (l >> 4), column 8 ((l >> 3) & 1)
        const uint32_t a0 = smem_u32(wt) +
                            2 * (((lane & 7) + 8 * (lane >> 4)) * WS + 32 * warp + 8 * ((lane >> 3) & 1));
#pragma unroll
        for (int ks = 0; ks < DH / 16; ks++)
#pragma unroll
            for (int mt = 0; mt < 2; mt++) {
                uint32_t a[4];
                ldsm_x4_trans<0>(a0 + 2 * (16 * ks * WS + 16 * mt), a);
                mma_bf16_16816(acc[mt], a[0], a[1], a[2], a[3], bhi[ks][0], bhi[ks][1]);
                mma_bf16_16816(acc[mt], a[0], a[1], a[2], a[3], blo[ks][0], blo[ks][1]);
            }
    }
    // accumulator rows are columns of the tile, its columns queries
#pragma unroll
    for (int mt = 0; mt < 2; mt++) {
        const int c = 32 * warp + 16 * mt + gid;
        part[2 * tig][c] = acc[mt][0];
        part[2 * tig + 1][c] = acc[mt][1];
        part[2 * tig][c + 8] = acc[mt][2];
        part[2 * tig + 1][c + 8] = acc[mt][3];
    }
    __syncthreads();
    // thread (q = tid / 16, cg): 8 columns of query q
    const int q = tid >> 4, cg = tid & 15;
    const int c0 = tile * 128 + cg * 8;
    float x[8];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < 8; e++) {
        x[e] = part[q][cg * 8 + e];
        amax = fmaxf(amax, fabsf(x[e]));
    }
    // amax over the scale group's threads (consecutive lanes of a half-warp)
    for (int off = 1; off < p.group / 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
    grid_launch_dependents();
    if (q >= nqc) return;
    const float inv = amax > 0.f ? 127.f / amax : 0.f;
    int hi[8], lo[8];
#pragma unroll
    for (int e = 0; e < 8; e++) {
        const float y = x[e] * inv;
        const float r = rintf(y);
        hi[e] = (int)r;
        lo[e] = __float2int_rn((y - r) * 254.f);
    }
    uint4 frag;
    if (p.bits == 8) {   // k-slot 4tig+i <-> element 8tig+i, 16+4tig+i <-> 8tig+4+i
        frag = make_uint4(pack4(hi[0], hi[1], hi[2], hi[3]), pack4(hi[4], hi[5], hi[6], hi[7]),
                          pack4(lo[0], lo[1], lo[2], lo[3]), pack4(lo[4], lo[5], lo[6], lo[7]));
    } else {             // k-slot 4tig+i <-> element 8tig+2i, 16+4tig+i <-> 8tig+2i+1
        frag = make_uint4(pack4(hi[0], hi[2], hi[4], hi[6]), pack4(hi[1], hi[3], hi[5], hi[7]),
                          pack4(lo[0], lo[2], lo[4], lo[6]), pack4(lo[1], lo[3], lo[5], lo[7]));
    }
    const int qi = q0 + q, b = qi / G, h = j * G + qi % G;
    // the score MMA's B-fragment slot of these 8 columns: k-step, n-tile, lane
    const int fks = c0 / 32, ftig = (c0 % 32) / 8;
    const int nt = h / 8, flane = (h % 8) * 4 + ftig;
    p.qfrag[(((int64_t)b * (p.D / 32) + fks) * p.NT + nt) * 32 + flane] = frag;
    if (c0 % p.group == 0)
        p.qfac[((int64_t)b * p.ng + c0 / p.group) * (p.NT * 8) + h] =
            amax * (1.f / (127.f * 254.f)) * p.tau_log2e * (p.bits == 4 ? 0.0625f : 1.f);
}

// ---------------------------------------------------------------- scores
// Grid (token tiles of T <= 64, B), 8 warps: warp w takes 16 tokens (w mod 4) x all
// heads over half of the scale groups (w / 4), the halves summed in shared memory.  The tile's
// codes (rows padded by 16 bytes: conflict-free fragment loads), this sequence's
// query fragments, the tile's scales and the factors are staged by cp.async.
// Scores in log2 units, s[b][h][t] = sum_g s_h(t, g) * qfac[g][h] * (254 acc_hi +
// acc_lo), written for t < len; the tile's (max, sum 2^(s - max)) per head go to
// stats[b][h][tile].
template <int BITS, int NT>
__global__ void __launch_bounds__(256) absorb_scores_kernel(AbsorbParams p)
{
    extern __shared__ __align__(16) uint8_t sm[];
    __shared__ float red[4][NT * 8];
    __shared__ float half2s[4][NT * 4][32];    // second group half's partial scores
    __shared__ float tmax[NT * 8];
    const int T = p.T2;
    const int b = blockIdx.y;
    const int t0 = blockIdx.x * T;
    const int tid = threadIdx.x;
    const int rowb = p.D * BITS / 8;
    const int rs = rowb + 16;
    const int KS = p.D / 32;
    uint8_t *tile = sm;                                                   // [T][rs]
    uint4 *qf = reinterpret_cast<uint4 *>(sm + (size_t)T * rs);          // [KS][NT][32]
    __half *sk = reinterpret_cast<__half *>(qf + (size_t)KS * NT * 32);  // [T][ng]
    float *fac = reinterpret_cast<float *>(sk + (((size_t)T * p.ng + 7) & ~(size_t)7));  // [ng][NT*8]
    grid_dependency_wait();
    const int len = seq_len(p, b);
    if (t0 >= len) return;
    const int nrow = min(T, len - t0);
    const int chunks = rowb / 16;
    const uint8_t *src = p.h_codes + ((int64_t)b * p.cap + t0) * rowb;
    const uint32_t tb = smem_u32(tile);
    {
        // (row, piece) walk with one division per thread
        int r = tid / chunks, c = tid % chunks;
        while (r < nrow) {
            cp_async16(tb + r * rs + 16 * c, src + (size_t)r * rowb + 16 * c);
            c += blockDim.x;
            while (c >= chunks) {
                c -= chunks;
                ++r;
            }
        }
    }
    const uint4 *qsrc = p.qfrag + (size_t)b * KS * NT * 32;
    const uint32_t qb = smem_u32(qf);
    for (int k = tid; k < KS * NT * 32; k += blockDim.x) cp_async16(qb + 16 * k, qsrc + k);
    // the tile's scales (whole 16-byte pieces by cp.async, a ragged end by plain
    // loads: nothing past the tile is read) and the factors
    const __half *ssrc = p.h_scales + ((int64_t)b * p.cap + t0) * p.ng;
    const uint32_t skb = smem_u32(sk);
    const int nsk = nrow * p.ng;                        // halves
    for (int k = tid; k < nsk / 8; k += blockDim.x) cp_async16(skb + 16 * k, ssrc + 8 * k);
    if (tid < nsk % 8) sk[nsk / 8 * 8 + tid] = ssrc[nsk / 8 * 8 + tid];
    const uint8_t *fsrc = reinterpret_cast<const uint8_t *>(p.qfac + (int64_t)b * p.ng * NT * 8);
    const uint32_t fb = smem_u32(fac);
    for (int k = tid; k < p.ng * NT * 8 * 4 / 16; k += blockDim.x) cp_async16(fb + 16 * k, fsrc + 16 * k);
    cp_async_wait_all();
    __syncthreads();
    grid_launch_dependents();

    const int wq = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    const int warp = wq & 3, gh = wq >> 2;    // token block, group half
    const int r0 = warp * 16 + gid, r1 = r0 + 8;
    const bool active = warp * 16 < nrow;     // inactive warps still join the reductions
    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; nt++) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    if (active) {
        const int ksg = p.group / 32;                   // k-steps per scale group
        const int ghn = p.ng / 2;                       // groups per half (ng is even)
        for (int g = gh * ghn; g < (gh + 1) * ghn; g++) {
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
                                 : "r"(tb + r0 * rs + 32 * ks + 8 * tig));
                    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x1.x), "=r"(x1.y)
                                 : "r"(tb + r1 * rs + 32 * ks + 8 * tig));
                    fa[0] = x0.x; fa[1] = x1.x; fa[2] = x0.y; fa[3] = x1.y;
                } else {
                    uint32_t x0, x1;
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x0) : "r"(tb + r0 * rs + 16 * ks + 4 * tig));
                    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x1) : "r"(tb + r1 * rs + 16 * ks + 4 * tig));
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
    }
    // the second half's partial scores join the first half's
    if (gh == 1)
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int e = 0; e < 4; e++) half2s[warp][nt * 4 + e][lane] = s[nt][e];
    __syncthreads();
    if (gh == 0)
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int e = 0; e < 4; e++) s[nt][e] += half2s[warp][nt * 4 + e][lane];
    // rows past the length (or of an inactive warp, or the second half) take no part
    const bool v0 = gh == 0 && active && r0 < nrow, v1 = gh == 0 && active && r1 < nrow;
#pragma unroll
    for (int nt = 0; nt < NT; nt++) {
        s[nt][0] = v0 ? s[nt][0] : -INFINITY;
        s[nt][1] = v0 ? s[nt][1] : -INFINITY;
        s[nt][2] = v1 ? s[nt][2] : -INFINITY;
        s[nt][3] = v1 ? s[nt][3] : -INFINITY;
    }
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int e = 0; e < 4; e++) {
            const int h = nt * 8 + 2 * tig + (e & 1);
            const int r = (e < 2) ? r0 : r1;
            if (h < p.Hq && s[nt][e] != -INFINITY)
                p.p[((int64_t)b * p.Hq + h) * p.capP + t0 + r] = s[nt][e];
        }
    // tile statistics per head: max over the tile's rows, then sum of 2^(s - max)
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int c = 0; c < 2; c++) {
            float m = fmaxf(s[nt][c], s[nt][2 + c]);
            for (int off = 4; off < 32; off <<= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
            if (gid == 0 && gh == 0) red[warp][nt * 8 + 2 * tig + c] = m;
        }
    __syncthreads();
    if (tid < NT * 8) {
        float m = red[0][tid];
        for (int w = 1; w < 4; w++) m = fmaxf(m, red[w][tid]);
        tmax[tid] = m;
    }
    __syncthreads();
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int c = 0; c < 2; c++) {
            const float m = tmax[nt * 8 + 2 * tig + c];
            float l = (s[nt][c] == -INFINITY ? 0.f : exp2f(s[nt][c] - m)) +
                      (s[nt][2 + c] == -INFINITY ? 0.f : exp2f(s[nt][2 + c] - m));
            for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(FULL, l, off);
            if (gid == 0 && gh == 0) red[warp][nt * 8 + 2 * tig + c] = l;
        }
    __syncthreads();
    if (tid < p.Hq) {
        float l = 0.f;
        for (int w = 0; w < 4; w++) l += red[w][tid];
        p.stats[((int64_t)b * p.Hq + tid) * p.ntile + blockIdx.x] = make_float2(tmax[tid], l);
    }
}

// ---------------------------------------------------------------- p . h^
// Grid (D / group, B, token splits of p.split tokens), 128 threads.  The merged
// softmax statistics of the sequence give p_t = 2^(s_t - M) / L per head; per
// block of 256 tokens the raw scores and the group's codes are staged by
// cp.async, then per 64 tokens P~[head][t] = fp16(p_t * s_h(t, g)) and the codes
// as exact fp16 integers [t][d] feed f16 MMAs (M = heads, N = the group's
// columns, K = tokens; the h fragments by ldmatrix.trans), warp w owning a
// quarter of the columns.  The split's partial ob goes to obp[split][b][h][d].
template <int BITS, int MT, int GS>
__global__ void __launch_bounds__(128) absorb_pv_kernel(AbsorbParams p)
{
    constexpr int TB = 256, TC = 64, TS = TC + 8, VS = 128 + 8;
    extern __shared__ __align__(16) uint8_t sm[];
    float *ss = reinterpret_cast<float *>(sm);                                  // [MT*16][TB]
    uint8_t *sc = sm + (size_t)MT * 16 * TB * 4;                                // [TB][group*BITS/8]
    __half *pt = reinterpret_cast<__half *>(sc + (size_t)TB * 128 * BITS / 8);  // [MT*16][TS]
    __half *vt = pt + MT * 16 * TS;                                             // [TC][VS]
    __shared__ float hm[MT * 16], hinv[MT * 16];
    __shared__ float sv[TB];
    const int g = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
    constexpr int cb = GS * BITS / 8;              // code bytes of the group per token
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    grid_dependency_wait();
    const int len = seq_len(p, b);
    const int t_begin = split * p.split;
    if (t_begin >= len) return;
    const int t_end = min(len, t_begin + p.split);
    // merged statistics: M = max_k m_k, L = sum_k l_k 2^(m_k - M) over the score tiles
    {
        // merged statistics, TPH consecutive threads per head, each over every TPH-th
        // tile, combined by shuffles
        constexpr int TPH = 128 / (MT * 16);
        const int h = tid / TPH, part = tid % TPH;
        const int nt = (len + p.T2 - 1) / p.T2;
        float M = -INFINITY, L = 0.f;
        const float2 *st = p.stats + ((int64_t)b * p.Hq + min(h, p.Hq - 1)) * p.ntile;
        if (h < p.Hq)
            for (int k = part; k < nt; k += TPH) M = fmaxf(M, st[k].x);
#pragma unroll
        for (int off = 1; off < TPH; off <<= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
        if (h < p.Hq)
            for (int k = part; k < nt; k += TPH) L += st[k].y * exp2f(st[k].x - M);
#pragma unroll
        for (int off = 1; off < TPH; off <<= 1) L += __shfl_xor_sync(FULL, L, off);
        if (part == 0) {
            hm[h] = M;
            hinv[h] = L > 0.f ? 1.f / L : 0.f;
        }
    }
    grid_launch_dependents();
    constexpr int ntw = GS / 32;                   // n-tiles of 8 columns per warp (1, 2 or 4)
    float acc[MT][4][4];
#pragma unroll
    for (int mt = 0; mt < MT; mt++)
#pragma unroll
        for (int n = 0; n < 4; n++) acc[mt][n][0] = acc[mt][n][1] = acc[mt][n][2] = acc[mt][n][3] = 0.f;
    const int rowb = p.D * BITS / 8;
    const uint32_t ssb = smem_u32(ss), scb = smem_u32(sc);
    for (int tb0 = t_begin; tb0 < t_end; tb0 += TB) {
        const int nb = min(TB, t_end - tb0);       // tokens of this block (a multiple of 16 but the last)
        __syncthreads();                           // the previous block's data is consumed
        // raw scores [h][t] (16-byte pieces: 4 tokens) and the group's codes [t][cb]
#pragma unroll
        for (int r = 0; r < MT * 16 * (TB / 4) / 128; r++) {
            const int k = tid + 128 * r, h = k / (TB / 4), t4 = 4 * (k % (TB / 4));
            if (h < p.Hq && t4 < nb)
                cp_async16(ssb + (h * TB + t4) * 4, p.p + ((int64_t)b * p.Hq + h) * p.capP + tb0 + t4);
        }
        constexpr int c16 = cb / 16;
#pragma unroll
        for (int r = 0; r < TB * c16 / 128; r++) {
            const int k = tid + 128 * r, t = k / c16, c = k % c16;
            if (t < nb)
                cp_async16(scb + t * cb + 16 * c, p.h_codes + ((int64_t)b * p.cap + tb0 + t) * rowb + g * cb + 16 * c);
        }
#pragma unroll
        for (int r = 0; r < TB / 128; r++) {
            const int t = tid + 128 * r;
            if (t < nb) sv[t] = __half2float(p.h_scales[((int64_t)b * p.cap + tb0 + t) * p.ng + g]);
        }
        cp_async_wait_all();
        __syncthreads();
        for (int c0 = 0; c0 < nb; c0 += TC) {
            const int nc = min(TC, nb - c0);
            if (c0 > 0) __syncthreads();           // pt / vt of the previous chunk are consumed
            for (int k = tid; k < MT * 16 * TC; k += blockDim.x) {
                const int h = k / TC, t = k % TC;
                float v = 0.f;
                if (h < p.Hq && t < nc)
                    v = exp2f(ss[h * TB + c0 + t] - hm[h]) * hinv[h] * sv[c0 + t];
                pt[h * TS + t] = __float2half_rn(v);
            }
            // Each 8-element run of codes becomes 4 half2 in a permuted element order
            // (VPERM below), with the exponent-bias conversion: a code sits in the
            // mantissa of 1024 (sign-flipped: 1152 + c for bytes, 1032 + c for
            // nibbles) and one half2 subtraction leaves the exact code.
            for (int k = tid; k < TC * (GS / 8); k += blockDim.x) {
                const int t = k / (GS / 8), d8 = 8 * (k % (GS / 8));
                uint32_t pk[4] = {0u, 0u, 0u, 0u};
                if (t < nc) {
                    const uint8_t *row = sc + (size_t)(c0 + t) * cb;
                    if constexpr (BITS == 8) {
                        // halves (e0, e2), (e1, e3), (e4, e6), (e5, e7)
                        const uint2 w = *reinterpret_cast<const uint2 *>(row + d8);
                        const uint32_t B = 0x64806480u, SUB = 0x64806480u;   // 1152
                        pk[0] = hsub2_u32(and_xor(w.x, 0x00FF00FFu, B), SUB);
                        pk[1] = hsub2_u32(and_xor(w.x >> 8, 0x00FF00FFu, B), SUB);
                        pk[2] = hsub2_u32(and_xor(w.y, 0x00FF00FFu, B), SUB);
                        pk[3] = hsub2_u32(and_xor(w.y >> 8, 0x00FF00FFu, B), SUB);
                    } else {
                        // halves (e0, e4), (e1, e5), (e2, e6), (e3, e7)
                        const uint32_t w = *reinterpret_cast<const uint32_t *>(row + d8 / 2) ^ 0x88888888u;
                        const uint32_t SUB = 0x64086408u;                   // 1032
#pragma unroll
                        for (int i = 0; i < 4; i++)
                            pk[i] = hsub2_u32(((w >> (4 * i)) & 0x000F000Fu) | 0x64006400u, SUB);
                    }
                }
                *reinterpret_cast<uint4 *>(vt + t * VS + d8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            __syncthreads();
            const uint32_t pb = smem_u32(pt), vb = smem_u32(vt);
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
        }
    }
    float *ob = p.obp + (int64_t)b * p.Hq * p.D;   // the splits add into one ob
    // accumulator columns 2tig, 2tig + 1 hold elements VPERM of the n-tile's 8 columns
    const int e0 = BITS == 8 ? ((tig & 1) + 4 * (tig >> 1)) : tig;
    const int e1 = BITS == 8 ? e0 + 2 : tig + 4;
#pragma unroll
    for (int n = 0; n < 4; n++) {
        if (n >= ntw) break;
        const int d = g * GS + (warp * ntw + n) * 8;
#pragma unroll
        for (int mt = 0; mt < MT; mt++) {
            const int h0 = mt * 16 + gid, h1 = h0 + 8;
            if (h0 < p.Hq) {
                atomicAdd(&ob[(int64_t)h0 * p.D + d + e0], acc[mt][n][0]);
                atomicAdd(&ob[(int64_t)h0 * p.D + d + e1], acc[mt][n][1]);
            }
            if (h1 < p.Hq) {
                atomicAdd(&ob[(int64_t)h1 * p.D + d + e0], acc[mt][n][2]);
                atomicAdd(&ob[(int64_t)h1 * p.D + d + e1], acc[mt][n][3]);
            }
        }
    }
}


// ---------------------------------------------------------------- p . h^, group 128
// The same product for 128-element scale groups, without the shared-memory pass of
// converted codes and without a CTA barrier per chunk: each warp owns 32 columns of
// the group and walks the block's tokens on its own.  P~[head][t] = 2^(s_t - M) / L *
// s_h(t, g) is computed once per staged block of 256 tokens into shared memory (fp16),
// whence the warps read their A fragments; their B fragments come from
// ldmatrix.trans of the raw codes (token rows
// padded by 16 bytes, so that the 8 rows of a matrix fall in 8 different bank
// groups) and become exact fp16 integers in registers: per 16-bit word of a token
// pair, a 4-bit code in the mantissa of 1024 (sign flipped: 1032 + c) minus 1032,
// an 8-bit code as 1152 + c minus 1152.
template <int BITS, int MT>
__global__ void __launch_bounds__(128) absorb_pv128_kernel(AbsorbParams p)
{
    constexpr int TB = 256;                        // tokens staged per block
    constexpr int cb = 128 * BITS / 8;             // code bytes of the group per token
    constexpr int RS = cb + 16;                    // padded row stride of the staged codes
    constexpr int PS = TB + 8;                     // padded row stride of P~ (halves)
    extern __shared__ __align__(16) uint8_t sm[];
    float *ss = reinterpret_cast<float *>(sm);                       // [MT*16][TB]
    uint8_t *sc = sm + (size_t)MT * 16 * TB * 4;                     // [TB][RS]
    __half *pt = reinterpret_cast<__half *>(sc + (size_t)TB * RS);   // [MT*16][PS]
    __shared__ float hm[MT * 16], hinv[MT * 16];
    __shared__ float sv[TB];
    const int g = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
    grid_dependency_wait();
    const int len = seq_len(p, b);
    const int t_begin = split * p.split;
    if (t_begin >= len) return;
    const int t_end = min(len, t_begin + p.split);
    {
        // merged statistics, TPH consecutive threads per head, each over every TPH-th
        // tile, combined by shuffles
        constexpr int TPH = 128 / (MT * 16);
        const int h = tid / TPH, part = tid % TPH;
        const int nt = (len + p.T2 - 1) / p.T2;
        float M = -INFINITY, L = 0.f;
        const float2 *st = p.stats + ((int64_t)b * p.Hq + min(h, p.Hq - 1)) * p.ntile;
        if (h < p.Hq)
            for (int k = part; k < nt; k += TPH) M = fmaxf(M, st[k].x);
#pragma unroll
        for (int off = 1; off < TPH; off <<= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
        if (h < p.Hq)
            for (int k = part; k < nt; k += TPH) L += st[k].y * exp2f(st[k].x - M);
#pragma unroll
        for (int off = 1; off < TPH; off <<= 1) L += __shfl_xor_sync(FULL, L, off);
        if (part == 0) {
            hm[h] = M;
            hinv[h] = L > 0.f ? 1.f / L : 0.f;
        }
    }
    grid_launch_dependents();
    float acc[MT][4][4];
#pragma unroll
    for (int mt = 0; mt < MT; mt++)
#pragma unroll
        for (int n = 0; n < 4; n++) acc[mt][n][0] = acc[mt][n][1] = acc[mt][n][2] = acc[mt][n][3] = 0.f;
    const int rowb = p.D * BITS / 8;
    const uint32_t ssb = smem_u32(ss), scb = smem_u32(sc);
    // ldmatrix rows of this lane: matrix l / 8 = (k16 step l / 16, token half (l / 8) % 2)
    const int lrow = 16 * (lane >> 4) + 8 * ((lane >> 3) & 1) + (lane & 7);
    for (int tb0 = t_begin; tb0 < t_end; tb0 += TB) {
        const int nb = min(TB, t_end - tb0);
        __syncthreads();                           // the previous block is consumed
#pragma unroll
        for (int r = 0; r < MT * 16 * (TB / 4) / 128; r++) {
            const int k = tid + 128 * r, h = k / (TB / 4), t4 = 4 * (k % (TB / 4));
            if (h < p.Hq && t4 < nb)
                cp_async16(ssb + (h * TB + t4) * 4, p.p + ((int64_t)b * p.Hq + h) * p.capP + tb0 + t4);
        }
        constexpr int c16 = cb / 16;
#pragma unroll
        for (int r = 0; r < TB * c16 / 128; r++) {
            const int k = tid + 128 * r, t = k / c16, c = k % c16;
            if (t < nb)
                cp_async16(scb + t * RS + 16 * c, p.h_codes + ((int64_t)b * p.cap + tb0 + t) * rowb + g * cb + 16 * c);
        }
#pragma unroll
        for (int r = 0; r < TB / 128; r++) {
            const int t = tid + 128 * r;
            sv[t] = t < nb ? __half2float(p.h_scales[((int64_t)b * p.cap + tb0 + t) * p.ng + g]) : 0.f;
        }
        cp_async_wait_all();
        __syncthreads();
        for (int k = tid; k < MT * 16 * TB / 2; k += 128) {
            const int h = k / (TB / 2), t = 2 * (k % (TB / 2));
            float v0 = 0.f, v1 = 0.f;
            if (h < p.Hq) {
                const float f = hinv[h], m = hm[h];
                if (t < nb) v0 = exp2f(ss[h * TB + t] - m) * f * sv[t];
                if (t + 1 < nb) v1 = exp2f(ss[h * TB + t + 1] - m) * f * sv[t + 1];
            }
            *reinterpret_cast<uint32_t *>(pt + h * PS + t) = pack_half2(v0, v1);
        }
        __syncthreads();
        const uint32_t ptb = smem_u32(pt);
        for (int c0 = 0; c0 < nb; c0 += 32) {
            // B: y[m] = token pair (2tig, 2tig+1) of matrix m, 16-bit word gid of its 16 bytes
            uint32_t y[BITS == 4 ? 1 : 2][4];
#pragma unroll
            for (int sg = 0; sg < (BITS == 4 ? 1 : 2); sg++)
                ldsm_x4_trans<0>(scb + (c0 + lrow) * RS + (BITS == 4 ? 16 * warp : 32 * warp + 16 * sg), y[sg]);
#pragma unroll
            for (int ks = 0; ks < 2; ks++) {
                // A: P~ of heads 16mt + gid (+8), tokens c0 + 16ks + 2tig (+1), (+8)
                uint32_t a[MT][4];
#pragma unroll
                for (int mt = 0; mt < MT; mt++)
#pragma unroll
                    for (int q = 0; q < 4; q++) {
                        const int h = 16 * mt + gid + 8 * (q & 1);
                        const int t = c0 + 16 * ks + 2 * tig + 8 * (q >> 1);
                        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[mt][q]) : "r"(ptb + (h * PS + t) * 2));
                    }
#pragma unroll
                for (int n = 0; n < 4; n++) {
                    uint32_t b0, b1;
                    if constexpr (BITS == 4) {
                        // n-tile n: nibble n of each word (columns 4 gid + n)
                        const uint32_t w0 = (y[0][2 * ks] ^ 0x88888888u) >> (4 * n);
                        const uint32_t w1 = (y[0][2 * ks + 1] ^ 0x88888888u) >> (4 * n);
                        b0 = hsub2_u32((w0 & 0x000F000Fu) | 0x64006400u, 0x64086408u);
                        b1 = hsub2_u32((w1 & 0x000F000Fu) | 0x64006400u, 0x64086408u);
                    } else {
                        // n-tile n: piece n / 2, byte n % 2 of each word (columns 2 gid + n % 2)
                        const uint32_t w0 = (y[n >> 1][2 * ks] ^ 0x80808080u) >> (8 * (n & 1));
                        const uint32_t w1 = (y[n >> 1][2 * ks + 1] ^ 0x80808080u) >> (8 * (n & 1));
                        b0 = hsub2_u32((w0 & 0x00FF00FFu) | 0x64006400u, 0x64806480u);
                        b1 = hsub2_u32((w1 & 0x00FF00FFu) | 0x64006400u, 0x64806480u);
                    }
#pragma unroll
                    for (int mt = 0; mt < MT; mt++)
                        mma_16816(acc[mt][n], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
                }
            }
        }
    }
    // accumulator column 2tig + e of n-tile n: 4-bit, column 4 (2tig + e) + n of the warp's
    // 32; 8-bit, column 16 (n / 2) + 2 (2tig + e) + n % 2
    float *ob = p.obp + (int64_t)b * p.Hq * p.D + g * 128 + 32 * warp;
#pragma unroll
    for (int mt = 0; mt < MT; mt++)
#pragma unroll
        for (int n = 0; n < 4; n++)
#pragma unroll
            for (int e = 0; e < 4; e++) {
                const int h = 16 * mt + gid + 8 * (e >> 1), col = 2 * tig + (e & 1);
                const int d = BITS == 4 ? 4 * col + n : 16 * (n >> 1) + 2 * col + (n & 1);
                if (h < p.Hq) atomicAdd(&ob[(int64_t)h * p.D + d], acc[mt][n][e]);
            }
}

// ---------------------------------------------------------------- W_v . ob
// Grid (Hkv, Dh / 16), 8 warps: the CTA's 16 rows of W_v,j against the ob of every
// query of KV head j (B * G of them, 8 at a time) on bf16 tensor cores, out^T (16 rows
// x 8 queries) = W (16 x D) ob^T (D x 8): ob enters as bf16 hi and lo parts (16
// significant bits; W_v is bf16 itself), warp w takes the k-steps (16 columns of D) w,
// w + 8, ..., and the 8 warps' fp32 partial sums are added in shared memory.  The W_v
// rows are copied to shared memory (cp.async) before the wait for the previous launch,
// so that they stream in while it finishes; ob is staged after it, every piece of a
// chunk of queries in flight at once.  Rows are padded by 16 (W) and 32 (ob) bytes:
// conflict-free ldmatrix and fragment loads.
__global__ void __launch_bounds__(256) absorb_out_kernel(AbsorbParams p)
{
    // [8][D + 8] fp32 ob, [16][D + 8] bf16 W_v rows, [8 warps][16 rows][8 queries] fp32
    extern __shared__ __align__(16) float obs[];
    const int OS = p.D + 8;
    const int j = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const int rbase = blockIdx.y * 16;
    const int G = p.Hq / p.Hkv;
    const int nq = p.B * G;
    const int D4 = p.D / 4;
    __nv_bfloat16 *ws = reinterpret_cast<__nv_bfloat16 *>(obs + (size_t)8 * OS);
    float *red = reinterpret_cast<float *>(ws + (size_t)16 * OS);
    {
        const uint32_t wb = smem_u32(ws);
        const __nv_bfloat16 *src = p.w + ((int64_t)p.Hkv * p.Dh + (int64_t)j * p.Dh + rbase) * p.D;
        const int per_row = p.D / 8;                // 16-byte pieces of a row
        for (int r = 0; r < 16; r++)
            for (int c = threadIdx.x; c < per_row; c += blockDim.x)
                cp_async16(wb + 2 * r * OS + 16 * c, src + (int64_t)r * p.D + 8 * c);
    }
    grid_dependency_wait();
    // ldmatrix row addresses of the matrices (rows 0-7, k 0-7), (rows 8-15, k 0-7),
    // (rows 0-7, k 8-15), (rows 8-15, k 8-15): lane l gives row (l & 7) + 8 ((l >> 3) & 1),
    // column 8 (l >> 4)
    const uint32_t arow = smem_u32(ws) + 2 * (((lane & 7) + 8 * ((lane >> 3) & 1)) * OS + 8 * (lane >> 4));
    const int nks = p.D / 16;
    for (int q0 = 0; q0 < nq; q0 += 8) {
        const int nqc = min(8, nq - q0);
        __syncthreads();                            // the previous chunk's ob and sums are consumed
        {
            // per query, its D / 4 pieces (no division by run-time sizes per piece)
            const uint32_t ob_s = smem_u32(obs);
            for (int c = 0; c < nqc; c++) {
                const int qi = q0 + c, b = qi / G, h = j * G + qi % G;
                const float *src = p.obp + ((int64_t)b * p.Hq + h) * p.D;
                for (int d4 = threadIdx.x; d4 < D4; d4 += blockDim.x)
                    cp_async16(ob_s + 4 * (c * OS + 4 * d4), src + 4 * d4);
            }
        }
        cp_async_wait_all();
        __syncthreads();
        // B columns of queries past nqc hold the previous chunk's ob or garbage: they
        // only reach accumulator columns that are never written
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const float *ob_row = obs + (size_t)gid * OS + 2 * tig;
#pragma unroll 4
        for (int ks = warp; ks < nks; ks += 8) {
            uint32_t a[4];
            ldsm_x4(arow + 32 * ks, a);
            const float2 v0 = *reinterpret_cast<const float2 *>(ob_row + 16 * ks);
            const float2 v1 = *reinterpret_cast<const float2 *>(ob_row + 16 * ks + 8);
            uint32_t h0, l0, h1, l1;
            split_bf16x2(v0.x, v0.y, h0, l0);
            split_bf16x2(v1.x, v1.y, h1, l1);
            mma_bf16_16816(acc, a[0], a[1], a[2], a[3], h0, h1);
            mma_bf16_16816(acc, a[0], a[1], a[2], a[3], l0, l1);
        }
        // accumulator rows are W_v rows, its columns queries
        float *rw = red + warp * 128;
        *reinterpret_cast<float2 *>(rw + gid * 8 + 2 * tig) = make_float2(acc[0], acc[1]);
        *reinterpret_cast<float2 *>(rw + (gid + 8) * 8 + 2 * tig) = make_float2(acc[2], acc[3]);
        __syncthreads();
        if (threadIdx.x < 128) {
            const int r = threadIdx.x >> 3, c = threadIdx.x & 7;
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < 8; w++) v += red[w * 128 + r * 8 + c];
            if (c < nqc) {
                const int qi = q0 + c, b = qi / G, h = j * G + qi % G;
                const int64_t o = ((int64_t)b * p.Hq + h) * p.Dh + rbase + r;
                if (p.out_f32)
                    static_cast<float *>(p.out)[o] = v;
                else
                    static_cast<__half *>(p.out)[o] = __float2half_rn(v);
            }
        }
    }
}

// shared-memory bytes of absorb_out_kernel: ob chunk, W_v rows, partial sums
size_t out_smem(int D) { return (size_t)(D + 8) * (8 * 4 + 16 * 2) + (size_t)8 * 128 * 4; }

// shared-memory bytes of the kernels that size it at run time
size_t scores_smem(int D, int bits, int NT, int ng, int T)
{
    return (size_t)T * (D * bits / 8 + 16) + (size_t)(D / 32) * NT * 512 +
           (((size_t)T * ng + 7) & ~(size_t)7) * 2 + (size_t)ng * NT * 8 * 4;
}

size_t pv_smem(int bits, int MT)
{
    return (size_t)MT * 16 * 256 * 4 + (size_t)256 * 128 * bits / 8 + (size_t)MT * 16 * 72 * 2 +
           (size_t)64 * 136 * 2;
}

template <typename... Args>
cudaError_t launch_pdl(void (*fn)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args)
{
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    return cudaLaunchKernelEx(&lc, fn, args...);
}

template <typename K>
cudaError_t set_smem(K fn, size_t bytes)
{
    return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int BITS, int NT>
cudaError_t launch_scores(const AbsorbParams &p, int max_len, cudaStream_t st)
{
    const size_t smem = scores_smem(p.D, BITS, NT, p.ng, p.T2);
    cudaError_t e = set_smem(absorb_scores_kernel<BITS, NT>, smem);
    if (e != cudaSuccess) return e;
    (void)max_len;
    return launch_pdl(absorb_scores_kernel<BITS, NT>, dim3(p.ntile, p.B), dim3(256), smem, st, p);
}

template <int BITS, int MT, int GS>
cudaError_t launch_pv_gs(const AbsorbParams &p, int max_len, cudaStream_t st)
{
    const size_t smem = pv_smem(BITS, MT);
    cudaError_t e = set_smem(absorb_pv_kernel<BITS, MT, GS>, smem);
    if (e != cudaSuccess) return e;
    const int ns = max(1, (max_len + p.split - 1) / p.split);
    return launch_pdl(absorb_pv_kernel<BITS, MT, GS>, dim3(p.D / GS, p.B, ns), dim3(128), smem, st, p);
}

template <int BITS, int MT>
cudaError_t launch_pv(const AbsorbParams &p, int max_len, cudaStream_t st)
{
    if (p.group == 128) {
        const size_t smem = (size_t)MT * 16 * 256 * 4 + (size_t)256 * (128 * BITS / 8 + 16) +
                            (size_t)MT * 16 * (256 + 8) * 2;
        cudaError_t e = set_smem(absorb_pv128_kernel<BITS, MT>, smem);
        if (e != cudaSuccess) return e;
        const int ns = max(1, (max_len + p.split - 1) / p.split);
        return launch_pdl(absorb_pv128_kernel<BITS, MT>, dim3(p.D / 128, p.B, ns), dim3(128), smem,
                          st, p);
    }
    switch (p.group) {
    case 32: return launch_pv_gs<BITS, MT, 32>(p, max_len, st);
    case 64: return launch_pv_gs<BITS, MT, 64>(p, max_len, st);
    case 128: return launch_pv_gs<BITS, MT, 128>(p, max_len, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int absorb_nt(int Hq) { return Hq <= 8 ? 1 : (Hq <= 16 ? 2 : 4); }

// The shape fits the kernels' shared memory: a 16-token score tile with the query
// fragments, and an 8-query ob chunk with 16 W_v rows.
bool absorb_fits(int D, int bits, int Hq, int ng)
{
    return scores_smem(D, bits, absorb_nt(Hq), ng, 16) <= 227 * 1024 && out_smem(D) <= 227 * 1024;
}

// Tokens per score tile: 64 (4 warps), fewer when the tile and the fragments
// outgrow shared memory.
int absorb_t2(int D, int bits, int Hq, int ng)
{
    for (int T = 64; T > 16; T /= 2)
        if (scores_smem(D, bits, absorb_nt(Hq), ng, T) <= 227 * 1024) return T;
    return 16;
}

// Token split of the p . h^ kernel: at least 256 tokens, at most 16 splits.
int absorb_split(int max_len)
{
    const int per = (max_len + 15) / 16;
    return max(256, (per + 255) / 256 * 256);
}

uint64_t absorb_scratch_layout(int B, int Hq, int D, int ng, int bits, int max_len, uint64_t off[6])
{
    const int NT = absorb_nt(Hq);
    const uint64_t capP = (uint64_t)((max_len + 63) / 64 * 64);
    const uint64_t ntile = capP / absorb_t2(D, bits, Hq, ng);   // tiles up to capP (T2 divides 64)
    const uint64_t sz[5] = {(uint64_t)B * (D / 32) * NT * 32 * 16, (uint64_t)B * ng * NT * 8 * 4,
                            (uint64_t)B * Hq * capP * 4, (uint64_t)B * Hq * (ntile ? ntile : 1) * 8,
                            (uint64_t)B * Hq * D * 4};
    uint64_t o = 0;
    for (int i = 0; i < 5; i++) {
        off[i] = o;
        o += (sz[i] + 255) / 256 * 256;
    }
    off[5] = o;
    return o;
}

cudaError_t launch_absorbed(const AbsorbParams &p, int max_len, cudaStream_t stream)
{
    (void)cudaGetLastError();   // drop a stale, already-reported error of an earlier call
    const int G = p.Hq / p.Hkv;
    cudaError_t e;
    if (p.NT * 8 != p.Hq) {
        // padding heads of the last n-tile must hold zero fragments
        e = cudaMemsetAsync(p.qfrag, 0, (size_t)p.B * (p.D / 32) * p.NT * 512, stream);
        if (e != cudaSuccess) return e;
    }
    const dim3 qgrid(p.Hkv, p.D / 128, (p.B * G + 7) / 8);
    e = p.Dh == 128 ? launch_pdl(absorb_q_kernel<128>, qgrid, dim3(128), 0, stream, p)
                    : launch_pdl(absorb_q_kernel<64>, qgrid, dim3(128), 0, stream, p);
    if (e != cudaSuccess) return e;
    if (max_len > 0) {
        switch (p.NT) {
        case 1: e = p.bits == 8 ? launch_scores<8, 1>(p, max_len, stream) : launch_scores<4, 1>(p, max_len, stream); break;
        case 2: e = p.bits == 8 ? launch_scores<8, 2>(p, max_len, stream) : launch_scores<4, 2>(p, max_len, stream); break;
        default: e = p.bits == 8 ? launch_scores<8, 4>(p, max_len, stream) : launch_scores<4, 4>(p, max_len, stream); break;
        }
        if (e != cudaSuccess) return e;
        const bool two = p.Hq > 16;
        e = p.bits == 8 ? (two ? launch_pv<8, 2>(p, max_len, stream) : launch_pv<8, 1>(p, max_len, stream))
                        : (two ? launch_pv<4, 2>(p, max_len, stream) : launch_pv<4, 1>(p, max_len, stream));
        if (e != cudaSuccess) return e;
    }
    // 16 W_v rows per CTA
    const size_t osm = out_smem(p.D);
    if ((e = set_smem(absorb_out_kernel, osm)) != cudaSuccess) return e;
    return launch_pdl(absorb_out_kernel, dim3(p.Hkv, p.Dh / 16), dim3(256), osm, stream, p);
}

}  // namespace kvq
