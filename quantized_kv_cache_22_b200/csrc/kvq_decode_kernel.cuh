// kvq_decode_kernel.cuh -- the split-KV decode attention kernel over a quantised
// KV cache (instantiated in kvq_decode_k4/k8/k16.cu; host side in kvq_decode.cu).
//
// What it computes (the pages' problem statement): one query token per
// sequence attends over every cached token of its KV head (mni-ml page: keep
// past K/V, compute only the new token's); K and V are dequantised inside the
// attention kernel (KVSplit discussion: integrate the formats into the
// FlashAttention kernel), with INT8 / nibble-packed INT4 codes and fp16
// scales per (token, head) or per group (TinyLoop mode table; KVSplit 8K
// table).  Output = softmax(tau q.K^T) V, fp32 accumulation.  Optionally the
// new token's K/V are quantised into the cache by the same launch first
// (quantize-on-append, TinyLoop "KV Cache 模式").
//
// Design for sm_100a (not taken from any page):
//   * Persistent CTAs, work split stream-K style: the units are 128-token
//     tiles of every (sequence, KV head); CTA c of the P' = min(P, units) CTAs
//     that get work takes units [cN/P', (c+1)N/P').  Every CTA streams the same
//     number of bytes whatever B, Hkv and the lengths are.  A CTA's run of
//     tiles inside one (sequence, KV head) is a "segment"; at its end the
//     consumer warps combine their partials (m, l, o) in shared memory and
//     write one per segment to the workspace, at slot (cta + sequence*Hkv +
//     kv_head), which is unique.  The warp that completes the last of the
//     partials of a (sequence, KV head) -- an arrival counter tells it --
//     merges them with their log-sum-exp weights and writes the output, so one
//     launch does the whole layer.
//   * One producer warp streams tiles with TMA: codes through 3-D tiled tensor
//     maps with 128-byte swizzle (bank-conflict-free fragment reads), scales
//     with 1-D bulk copies, into a multi-stage shared-memory ring guarded by
//     mbarriers.  Every wait is bounded (about a second) and a give-up sets
//     the workspace status word instead of hanging.  Before it loads the tile
//     that holds a sequence's newest token, the producer warp quantises that
//     token into the cache (the fused append) and fences the writes against
//     the copy engine.
//   * Four consumer warps each take 32 tokens of a stage as two 16-token
//     sub-tiles.  q.K^T runs on int8 tensor-core MMA (m16n8k32): the key codes
//     feed the MMA as they are stored (4-bit codes after one mask, as 16x the
//     code), and the query is split per head into two int8 parts, q ~ s (hi +
//     lo/254), so the products keep ~16 bits of the query.  P.V runs on f16
//     MMA (m16n8k16, f32 accumulate) with head_dim as M and the G query heads
//     of the KV group as N: value codes become fp16 in registers with the
//     exponent-bias trick (a code byte u in the mantissa of 0x6400 reads 1024
//     + u), value scales are folded into the probabilities, and the constant
//     bias is removed at the end with the probability sums, which one extra
//     MMA against a matrix of ones accumulates.  The score tile is turned into
//     the P operand by two 8x8 transposes (movmatrix).
//   * The online softmax tracks max(s + log2 s_V) so that p * s_V <= 2^8 fits
//     fp16 without underflow whatever the value scales are.
//   * In a chain of launches the next layer's CTAs start while this one's last
//     CTAs finish: each finds its work range and asks its first tiles and its
//     queries into L2 before the wait for the previous launch, and checks the
//     lengths it used after it.
#pragma once
#include <cfloat>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_decode_common.cuh"

namespace kvq {
namespace {

constexpr int NW = kDecodeConsumerWarps;
constexpr int NTHR = kDecodeThreads;

// Token of row g (g < 8) of a 16-token sub-tile's score tile; row g + 8 holds
// the next token.  The permutation pi keeps the key-row reads of the score MMA
// and the value-row reads of the P.V MMA (whose k order follows the score rows
// through the transpose) free of shared-memory bank conflicts under the 128-byte
// swizzle (checked against a model of the banks for every head_dim-128
// format): pi(g) = g ^ (g >> 2) when keys are read 4 or 8 bytes per row and
// block, and pi = (0, 6, 2, 4, 5, 3, 7, 1) when they are read 16 bytes per row
// (KW), which also needs the two rows of each quarter-warp in different halves
// of the bank space.
template <bool KW>
__host__ __device__ constexpr int row_token(int g)
{
    if constexpr (KW)
        return 2 * (int)((0x17354260u >> (4 * g)) & 7u);
    else
        return 2 * (g ^ (g >> 2));
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

__device__ __forceinline__ uint32_t pack_bytes(int a, int b, int c, int d)
{
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

// KG / VG: keys / values carry one scale per 32/64-element group (else one per
// (token, head)); compile-time so the per-head case keeps no per-group state.
// FMT: the code format of 8-bit keys and values (KVQ_FMT_*; KB = VB = 8 unless
// KVQ_FMT_INT): symmetric integer, FP8 e4m3, asymmetric (uint8 codes with a
// zero-point) or per-tensor (one fixed scale per tensor).
// PK ("packed columns", G <= 4 with int8 keys): the score MMA's eight columns carry
// the hi parts of the four heads and their lo parts, against sub-tile 0's keys with
// [hi | lo] and sub-tile 1's with [lo | hi]; one shuffle joins hi and lo, after which
// lanes tig < 2 own sub-tile 0's scores of their heads and lanes tig >= 2 sub-tile
// 1's.  Half the score MMAs, and no softmax work on padding columns: every lane
// carries 4 live scores instead of 8 (4 of them padding).  Both sub-tiles' P then
// share one transposed fragment, masked per sub-tile for the P.V MMAs, whose output
// columns 0-3 accumulate sub-tile 0 and 4-7 sub-tile 1 (joined at the segment end).
template <int DH, int KB, int VB, bool KG, bool VG, int FMT, bool PK = false>
__global__ void __launch_bounds__(NTHR, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ DecodeParams p)
{
    constexpr bool F8 = FMT == KVQ_FMT_E4M3;   // e4m3 codes
    constexpr bool ZP = FMT == KVQ_FMT_ASYM;   // uint8 codes, (scale, zero-point) per group
    constexpr bool PT = FMT == KVQ_FMT_TENSOR; // one scale per tensor, no per-token scales
    constexpr int NG = DH / 32;                // 32-element blocks along head_dim
    constexpr int RK = DH * KB / 8;            // bytes per key row
    constexpr int RV = DH * VB / 8;
    constexpr int SK = 32 * KB / 8;            // bytes per 32-element block of a key row
    constexpr int SV = 32 * VB / 8;
    constexpr int NVG = VG ? NG : 1;           // value-scale groups tracked per token
    // Value fragments: with one value scale per (token, head) a lane reads 8
    // consecutive head_dim elements of a row per 64-element half ("wide": one
    // load feeds four m-tiles); grouped value scales need one P per 32-element
    // block, so a lane then reads 4 elements per block.  Rows of 32 bytes (Dh 64
    // at 4 bits) keep the block mapping, which stays free of bank conflicts.
    constexpr bool VWIDE = !VG && RV >= 64 && !F8;
    // 4-bit values, wide: one ldmatrix.trans per sub-tile and 64-element half gives
    // each lane the (k-slot pair, 4 dims) words of four 8-token x 32-dim matrices
    constexpr bool VLDSM = VWIDE && VB == 4;
    constexpr int VL = VWIDE ? 2 * SV / 8 : SV / 8;   // value bytes per lane per row and load
    // Key fragments: with one key scale per (token, head), int8 keys are read 16
    // bytes per lane and row ("wide": 2 blocks of 32 elements per load at 8
    // bits, 4 at 4 bits); an int8 MMA block must share one key scale, so
    // grouped key scales keep one load per block.
    constexpr bool KWIDE = !KG && KB != 16 && RK >= 64 && !F8;
    constexpr int KLW = KWIDE ? 16 : SK / 4;          // key bytes per lane per row and load
    constexpr int KPL = KWIDE ? 16 * 8 / KB / 8 : 1;  // 32-element blocks per load
    // value codes enter the P.V MMA as (bias + code): 1152 + code at 8 bits (1024
    // + code for uint8 codes), per row at 4 bits (see the segment end); fp16 and
    // e4m3 values convert exactly, no bias.  psum = sum of P (times the bias),
    // from an MMA of P against a constant matrix (ones; 1024 + zero-point for
    // uint8 codes, so that the zero-point comes off with the bias).
    constexpr float BIAS_V = (VB == 8 && !F8) ? (ZP ? 1.f : 1152.f) : 0.f;
    constexpr bool VBIAS = VB == 4 || (VB == 8 && !F8);
    constexpr uint32_t VX = ZP ? 0x64006400u : 0x64806480u;   // byte -> fp16 1024 + byte (^0x80)
    // The running max is only raised when a tile beats it by more than 2^LAZY;
    // weights p * s_V then stay below 2^LAZY, well inside fp16.
    constexpr float LAZY = 8.f;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // align to 1024 B (128-byte swizzle atoms) by pointer arithmetic on the shared
    // array itself, so every access below stays a shared-memory access
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);             // 32-bit shared address of the ring
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + p.off_meta);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *empty = full + p.stages;
    uint64_t *segbar = empty + p.stages;                // [0] partials in mbuf, [1] mbuf read
    // [0] abort, [4..8] segment handed to the combiner: bh, slot, ncta, cmin, end
    int *ctl = reinterpret_cast<int *>(segbar + 2);
    float *mbuf = reinterpret_cast<float *>(smem + p.off_merge);   // [NW][G][DH + 4]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int S = p.stages;
    const int G = p.group_size_g;
    const int cap = p.cap;
    const int Hkv = p.n_kv_heads;
    volatile int *abort_flag = ctl;

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NW);
        }
        mbar_init(&segbar[0], NW);   // consumers: partials of a segment in mbuf
        mbar_init(&segbar[1], 1);    // combiner: mbuf read
        if (PK && KB != 16 && !F8 && FMT != KVQ_FMT_ASYM && p.off_qmisc != 0) {
            // shared query quantisation: [0] every head written, [1] every warp has read
            uint64_t *qbar = reinterpret_cast<uint64_t *>(smem + p.off_qmisc + 16);
            mbar_init(&qbar[0], NW);
            mbar_init(&qbar[1], NW);
        }
        ctl[0] = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    // The queries are read right after the work range: ask for this CTA's share of
    // them to be brought into L2 now, while a preceding launch may still run (a
    // prefetch only fills L2, which the preceding launch's writes update, and
    // nothing waits for it).
    if (tid == 32 * (NW + 1)) {
        const uint64_t qbytes = (uint64_t)p.batch * p.n_q_heads * DH * (p.q_dtype == KVQ_F32 ? 4 : 2);
        const uint64_t per = ((qbytes + gridDim.x - 1) / gridDim.x + 15) & ~(uint64_t)15;
        const uint64_t off = (uint64_t)blockIdx.x * per;
        if (off < qbytes) {
            const uint64_t n = qbytes - off < per ? qbytes - off : per;
            bulk_prefetch_l2(static_cast<const uint8_t *>(p.q) + off, (uint32_t)n);
        }
    }
    // Launched as a programmatic dependent: until grid_dependency_wait() below the
    // preceding grid (whatever it is) may still be writing global memory.  Before
    // the wait the kernel touches only its shared memory and the launch parameters,
    // asks for L2 prefetches, and reads the sequence lengths (through L2) to find its
    // work range speculatively; after the wait it reads the lengths again and finds
    // the range anew if any changed, so nothing read early is used unchecked.  The
    // next launch may be scheduled once this one has passed the wait.
    // ---- work range of this CTA (computed by the producer warp) -------------
    // With more than kSpecBatch sequences it is found after the wait only.
    __shared__ WorkRange wr;
    const bool spec = p.batch <= kSpecBatch;
    int dl[8];
    if (warp == NW && spec) {
        read_lens(p, lane, dl);
        work_range_from(p, lane, wr, dl);
        __syncwarp();
        if (lane == 0 && wr.n_units > 0 && p.block_table == nullptr && !p.stall) {
            const int kvh = wr.bh0 % Hkv;
            const int tile0 = (int)(wr.u_begin - wr.pre) - kvh * wr.tiles_b;
            for (int t = tile0; t < tile0 + 2 && t - tile0 < wr.n_units && t < wr.tiles_b; t++) {
                const int y0 = t * T, z = wr.bh0;
                constexpr int RK = DH * KB / 8, RV = DH * VB / 8;
                if constexpr (RK <= 128) {
                    tma_prefetch_3d(&tm_k, 0, y0 / (128 / RK), z);
                } else {
                    tma_prefetch_3d(&tm_k, 0, y0, z);
                    tma_prefetch_3d(&tm_k, 128, y0, z);
                }
                if constexpr (RV <= 128) {
                    tma_prefetch_3d(&tm_v, 0, y0 / (128 / RV), z);
                } else {
                    tma_prefetch_3d(&tm_v, 0, y0, z);
                    tma_prefetch_3d(&tm_v, 128, y0, z);
                }
                const int n_s = min(T, cap - y0);
                if (KB != 16 && !PT)
                    bulk_prefetch_l2(p.k_scales + ((int64_t)z * cap + y0) * p.ngs_k, (uint32_t)(n_s * p.ngs_k * 2));
                if (VB != 16 && !PT)
                    bulk_prefetch_l2(p.v_scales + ((int64_t)z * cap + y0) * p.ngs_v, (uint32_t)(n_s * p.ngs_v * 2));
            }
        }
    }
    grid_dependency_wait();
    grid_launch_dependents();
    if (warp == NW) {
        if (spec) {
            int now[8];
            read_lens(p, lane, now);
            bool same = true;
#pragma unroll
            for (int k = 0; k < 8; k++) same = same && now[k] == dl[k];
            if (!__all_sync(FULL, same)) work_range_from(p, lane, wr, now);
        } else {
            decode_work_range(p, lane, wr);
        }
    }
    __syncthreads();
    const int n_units = wr.n_units;

    if (warp == NW) {
        decode_producer<DH, KB, VB, FMT>(p, &tm_k, &tm_v, smem, full, empty, meta, abort_flag, wr,
                                         lane);
        return;
    }

    if (warp == NW + 1) {
        // ====================== combiner ======================
        // Per segment end: combine the consumer warps' partials from mbuf into
        // this CTA's slot, hand mbuf back, publish, and merge when this CTA's
        // partial is the last one of its (sequence, KV head).
        constexpr int CS = slot_col_floats(DH);
        const int ncol = ((KB == 16 || F8) && p.q_dtype != KVQ_F16) ? min(G, 4) : G;
        for (uint32_t k = 0;; k++) {
            if (!mbar_wait_bounded(&segbar[0], k & 1u, abort_flag, p.timeout_ns)) {
                if (lane == 0 && *abort_flag == 0) {
                    ctl[0] = 1;
                    atomicExch(p.status, KVQ_ERR_TIMEOUT);
                }
                return;
            }
            const volatile int *seg = ctl + 4;
            const int bh = seg[0], slot = seg[1], ncta = seg[2], cmin = seg[3], end = seg[4];
            if (end) return;
            float *dst = p.ws + (size_t)slot * G * CS;
            for (int c = lane; c < ncol * (DH / 4); c += 32) {
                const int col = c / (DH / 4), d = 4 * (c % (DH / 4));
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < NW; w++) M = fmaxf(M, mbuf[((size_t)w * G + col) * CS + DH]);
                float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
                float L = 0.f;
#pragma unroll
                for (int w = 0; w < NW; w++) {
                    const float *src = mbuf + ((size_t)w * G + col) * CS;
                    const float mw = src[DH];
                    const float e = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
                    const float4 x = *reinterpret_cast<const float4 *>(src + d);
                    O.x = fmaf(e, x.x, O.x);
                    O.y = fmaf(e, x.y, O.y);
                    O.z = fmaf(e, x.z, O.z);
                    O.w = fmaf(e, x.w, O.w);
                    L = fmaf(e, src[DH + 1], L);
                }
                *reinterpret_cast<float4 *>(dst + (size_t)col * CS + d) = O;
                if (d == 0) *reinterpret_cast<float2 *>(dst + (size_t)col * CS + DH) = make_float2(M, L);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&segbar[1]);   // the consumers may refill mbuf
            if (p.counters != nullptr) {
                // publish the warp's writes (warp barrier, then one acq_rel fence
                // and the arrival count); the CTA whose arrival completes the
                // count acquires the others' partials the same way and merges
                __syncwarp();
                int last = 0;
                if (lane == 0) {
                    fence_acq_rel_gpu();
                    last = atomicAdd(&p.counters[bh], 1) == ncta - 1;
                    if (last) fence_acq_rel_gpu();
                }
                last = __shfl_sync(FULL, last, 0);
                __syncwarp();
                if (last) {
                    const int b = bh / Hkv, kvh = bh % Hkv;
                    merge_segment<DH>(p.ws, (int64_t)cmin + bh, ncta, G, p.out, p.out_f32,
                                      ((int64_t)b * p.n_q_heads + (int64_t)kvh * G) * DH, lane);
                    if (lane == 0) p.counters[bh] = 0;   // ready for the next launch
                }
            }
        }
    }

    // ====================== consumers ======================
    constexpr bool IMMA_K = KB != 16 && !F8;   // else f16 MMA (fp16 keys, or e4m3 converted)
    // packed columns: int8 keys without zero-points, or e4m3 keys with one scale per
    // (token, head), whose f16 score MMA then always takes the fp16 query and its
    // residual (zero for fp16 queries) as the hi / lo parts
    static_assert(!PK || (IMMA_K && (!ZP || !KG)) || (F8 && !KG), "no packed columns for this format");
    constexpr int NU = PK ? 1 : 2;             // score sub-tiles a lane carries
    const int gid = lane >> 2;
    const int tig = lane & 3;
    // fp16 keys keep an f16 MMA; f32 / bf16 queries then use columns 4..7 for
    // the fp16 residual of the query (G <= 4)
    const bool qsplit = !IMMA_K && p.q_dtype != KVQ_F16;
    constexpr bool kgrp = KG;
    constexpr bool vgrp = VG;
    const int colmax = qsplit ? 4 : 8;
    // PK: lane tig holds sub-tile tig >> 1's heads 2 (tig & 1) + c; lanes tig < 2 write
    const bool col_ok0 = PK ? (tig < 2 && 2 * tig < G) : ((2 * tig) < G && (2 * tig) < colmax);
    const bool col_ok1 = PK ? (tig < 2 && 2 * tig + 1 < G)
                            : ((2 * tig + 1) < G && (2 * tig + 1) < colmax);
    const int ul = tig >> 1;                   // PK: the lane's score sub-tile

    // sequences with nothing cached get zeros (fused merge only; the merge
    // launch writes them otherwise)
    if (p.counters != nullptr) {
        const int64_t n_out = (int64_t)p.n_q_heads * DH;
        for (int b = blockIdx.x; b < p.batch; b += gridDim.x) {
            if (tiles_of(p.d_len[b], cap) != 0) continue;
            for (int64_t i = tid; i < n_out; i += 32 * NW) {
                if (p.out_f32)
                    static_cast<float *>(p.out)[(int64_t)b * n_out + i] = 0.f;
                else
                    static_cast<__half *>(p.out)[(int64_t)b * n_out + i] = __float2half_rn(0.f);
            }
        }
    }

    // Rows of the score tile: row gid is token tw + rt, row gid + 8 token tw + rt + 1.
    // The P.V MMA takes k-slots 2tig, 2tig+1, 2tig+8, 2tig+9 = tokens
    // tw + vA, tw + vB, tw + vA + 1, tw + vB + 1 (the transpose of the score rows).
    const int rt = row_token<KWIDE>(gid);
    const int vA = row_token<KWIDE>(2 * tig), vB = row_token<KWIDE>(2 * tig + 1);
    uint32_t kofs[2][2], vofs[2][4];
#pragma unroll
    for (int u = 0; u < 2; u++) {
        const int tw = warp * 32 + u * 16;
        kofs[u][0] = sw_off<RK>(tw + rt, tig * KLW);
        kofs[u][1] = sw_off<RK>(tw + rt + 1, tig * KLW);
        // ldmatrix rows: lane l gives row l % 8 of matrix l / 8 = (token half, 32-dim
        // window): k-slot l % 8 (+ 8 for the second token half) of the P.V MMA
        vofs[u][0] = VLDSM
                         ? p.off_v + sw_off<RV>(tw + row_token<KWIDE>(lane & 7) + ((lane >> 3) & 1),
                                                16 * (lane >> 4))
                         : p.off_v + sw_off<RV>(tw + vA, gid * VL);
        vofs[u][1] = p.off_v + sw_off<RV>(tw + vB, gid * VL);
        vofs[u][2] = p.off_v + sw_off<RV>(tw + vA + 1, gid * VL);
        vofs[u][3] = p.off_v + sw_off<RV>(tw + vB + 1, gid * VL);
    }
    // Sub-tile 1 lies 16 tokens after sub-tile 0.  For rows of >= 64 bytes the
    // swizzle phase repeats every 16 tokens, so its addresses are those of
    // sub-tile 0 plus KU / VU, which the loads carry as immediate offsets;
    // shorter rows (Dh 64 at 4 bits) keep their own offsets.
    constexpr bool KREP = RK >= 64, VREP = RV >= 64;
    constexpr int KU = RK <= 128 ? 16 * RK : 16 * 128;
    constexpr int VU = RV <= 128 ? 16 * RV : 16 * 128;

    uint32_t qh[NG][2], ql[NG][2];      // int8 query B-fragments (hi / lo parts) per block
    float sqc[2];                       // score factor of columns 2tig, 2tig+1
    // uint8 keys with a zero-point z: q.(c - z) = q.c - z * sum(q), with sum(q) in
    // the hi/lo units of the MMA (254 sum(hi) + sum(lo)), per head (columns 2tig,
    // 2tig+1) and per 32-element block when the key scales are grouped
    int zq[KG ? NG : 1][2];
    uint32_t qb[NG][2][2];              // fp16 query B-fragments (fp16 keys)
    uint32_t qb2[PK && F8 ? NG : 1][2][2];   // PK e4m3: the [lo | hi] fragments of sub-tile 1
    float m_run[2], l_run[2];
    float psum[NVG][4];                 // sum of fp16 p*s_V per value group (cols in [0], [1])
    float o_acc[2 * NG][4];             // O^T fragments, m-tile = 2*blk + h

    auto load_q = [&](int bh) {
        const int b = bh / Hkv;
        const int kvh = bh % Hkv;
        if constexpr (IMMA_K) {
            // q ~ (amax / 127) * (hi + lo / 254) per head, hi, lo in [-127, 127];
            // lane (gid, tig) holds head gid and, for block blk, the 8 elements its
            // key fragments hold: from (blk / KPL) 32 KPL + 8 KPL tig + 8 (blk % KPL)
            // PK: columns gid and gid + 4 carry the hi / lo parts of head gid & 3
            const int qhd = PK ? (gid & 3) : gid;
            const bool valid = qhd < G;
            const int64_t qbase = ((int64_t)b * p.n_q_heads + (int64_t)kvh * G + qhd) * DH;
            float x[NG][8];
            float amax = 0.f;
#pragma unroll
            for (int blk = 0; blk < NG; blk++) {
                // the lane's 8 elements of the block are contiguous
                if (valid)
                    load_q8(p.q, p.q_dtype,
                            qbase + (blk / KPL) * 32 * KPL + 8 * KPL * tig + 8 * (blk % KPL), x[blk]);
                else
#pragma unroll
                    for (int j = 0; j < 8; j++) x[blk][j] = 0.f;
#pragma unroll
                for (int j = 0; j < 8; j++) amax = fmaxf(amax, fabsf(x[blk][j]));
            }
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 1));
            amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, 2));
            const float inv = amax > 0.f ? 127.f / amax : 0.f;
            int qs_all = 0;
#pragma unroll
            for (int blk = 0; blk < NG; blk++) {
                int hi[8], lo[8];
                int qs_blk = 0;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    const float y = x[blk][j] * inv;
                    const float r = rintf(y);
                    hi[j] = (int)r;
                    lo[j] = __float2int_rn((y - r) * 254.f);
                    qs_blk += 254 * hi[j] + lo[j];
                }
                if constexpr (ZP) {
                    if constexpr (KG) {
                        // the block's 32 elements sit in the 4 lanes of the head
                        qs_blk += __shfl_xor_sync(FULL, qs_blk, 1);
                        qs_blk += __shfl_xor_sync(FULL, qs_blk, 2);
                        zq[blk][0] = __shfl_sync(FULL, qs_blk, (2 * tig) * 4);
                        zq[blk][1] = __shfl_sync(FULL, qs_blk, (2 * tig + 1) * 4);
                    } else {
                        qs_all += qs_blk;
                    }
                }
                if constexpr (KB == 8) {
                    // k-slot 4tig+i <-> element 8tig+i, 16+4tig+i <-> 8tig+4+i
                    qh[blk][0] = pack_bytes(hi[0], hi[1], hi[2], hi[3]);
                    qh[blk][1] = pack_bytes(hi[4], hi[5], hi[6], hi[7]);
                    ql[blk][0] = pack_bytes(lo[0], lo[1], lo[2], lo[3]);
                    ql[blk][1] = pack_bytes(lo[4], lo[5], lo[6], lo[7]);
                } else {
                    // k-slot 4tig+i <-> element 8tig+2i (low nibbles), 16+4tig+i <-> 8tig+2i+1
                    qh[blk][0] = pack_bytes(hi[0], hi[2], hi[4], hi[6]);
                    qh[blk][1] = pack_bytes(hi[1], hi[3], hi[5], hi[7]);
                    ql[blk][0] = pack_bytes(lo[0], lo[2], lo[4], lo[6]);
                    ql[blk][1] = pack_bytes(lo[1], lo[3], lo[5], lo[7]);
                }
                if constexpr (PK) {
                    // qh = [hi | lo] (sub-tile 0's B operand), ql = [lo | hi] (sub-tile 1's)
                    if (gid >= 4) {
                        const uint32_t t0 = qh[blk][0], t1 = qh[blk][1];
                        qh[blk][0] = ql[blk][0];
                        qh[blk][1] = ql[blk][1];
                        ql[blk][0] = t0;
                        ql[blk][1] = t1;
                    }
                }
            }
            if constexpr (ZP && !KG) {
                qs_all += __shfl_xor_sync(FULL, qs_all, 1);
                qs_all += __shfl_xor_sync(FULL, qs_all, 2);
                const int zc = PK ? 2 * (tig & 1) : 2 * tig;   // the lane's first head column
                zq[0][0] = __shfl_sync(FULL, qs_all, zc * 4);
                zq[0][1] = __shfl_sync(FULL, qs_all, (zc + 1) * 4);
            }
            // 4-bit key codes enter the MMA as 16 * code
            const float f = amax * (1.f / (127.f * 254.f)) * p.tau_log2e * (KB == 4 ? 0.0625f : 1.f);
            const int hc = PK ? 2 * (tig & 1) : 2 * tig;   // the lane's first head column
            sqc[0] = __shfl_sync(FULL, f, hc * 4);
            sqc[1] = __shfl_sync(FULL, f, (hc + 1) * 4);
        } else {
            // B-fragment column n = gid: non-split: head n; split (and PK): hi (n<4) / lo
            // (n>=4) of head n&3; PK's second set qb2 swaps hi and lo
            const int head = (qsplit || PK) ? (gid & 3) : gid;
            const bool lo_part = (qsplit || PK) && gid >= 4;
            const bool valid = head < G;
            const int64_t qbase = ((int64_t)b * p.n_q_heads + (int64_t)kvh * G + head) * DH;
#pragma unroll
            for (int blk = 0; blk < NG; blk++)
#pragma unroll
                for (int hs = 0; hs < 2; hs++) {
                    __half hv[4];
                    __half hw[4];   // the other part (PK e4m3)
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        // k-slots 2tig, 2tig+1, 2tig+8, 2tig+9 <-> elements 8tig + 4hs + j
                        const int d = 32 * blk + 8 * tig + 4 * hs + j;
                        const float xq = valid ? load_qf(p.q, p.q_dtype, qbase + d) : 0.f;
                        const __half hh = __float2half_rn(xq);
                        const __half hl = __float2half_rn(xq - __half2float(hh));
                        hv[j] = lo_part ? hl : hh;
                        hw[j] = lo_part ? hh : hl;
                    }
                    __half2 b0 = __halves2half2(hv[0], hv[1]);
                    __half2 b1 = __halves2half2(hv[2], hv[3]);
                    qb[blk][hs][0] = *reinterpret_cast<uint32_t *>(&b0);
                    qb[blk][hs][1] = *reinterpret_cast<uint32_t *>(&b1);
                    if constexpr (PK && F8) {
                        __half2 c0 = __halves2half2(hw[0], hw[1]);
                        __half2 c1 = __halves2half2(hw[2], hw[3]);
                        qb2[blk][hs][0] = *reinterpret_cast<uint32_t *>(&c0);
                        qb2[blk][hs][1] = *reinterpret_cast<uint32_t *>(&c1);
                    }
                }
        }
#pragma unroll
        for (int c = 0; c < 2; c++) {
            m_run[c] = -INFINITY;
            l_run[c] = 0.f;
        }
#pragma unroll
        for (int g = 0; g < NVG; g++) psum[g][0] = psum[g][1] = psum[g][2] = psum[g][3] = 0.f;
#pragma unroll
        for (int mt = 0; mt < 2 * NG; mt++)
#pragma unroll
            for (int i = 0; i < 4; i++) o_acc[mt][i] = 0.f;
    };

    // The same fragments with the quantisation shared (packed-column int8 keys without
    // zero-points): consumer warp w quantises head w of the segment (lane l: elements
    // 4l .. 4l+3) into shared memory, and after every warp has written (qbar[0]) each
    // lane reads its fragments back.  k counts the shared segment starts of this CTA;
    // a warp writes only after every warp has read the previous segment's (qbar[1]).
    // The arithmetic is that of load_q, so the fragments are the same bits; like
    // load_q it starts the segment's softmax state and accumulators afresh.
    constexpr bool QSHARE = PK && IMMA_K && !ZP;
    auto share_q = [&](int bh, uint32_t k) -> bool {
        uint8_t *qhi = smem + p.off_qhi;                                 // [4][DH] bytes
        uint8_t *qlo = smem + p.off_qlo;                                 // [4][DH] bytes
        float *qfac = reinterpret_cast<float *>(smem + p.off_qmisc);
        uint64_t *qbar = reinterpret_cast<uint64_t *>(smem + p.off_qmisc + 16);
        if (k > 0 && !mbar_wait_bounded(&qbar[1], (k - 1) & 1u, abort_flag, p.timeout_ns)) return false;
        if (warp < G) {
            const int b = bh / Hkv, kvh = bh % Hkv;
            const int64_t base = ((int64_t)b * p.n_q_heads + (int64_t)kvh * G + warp) * DH + 4 * lane;
            float x[4];
            if (p.q_dtype == KVQ_F32) {
                const float4 v = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(p.q) + base));
                x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
            } else {
                const uint2 w = __ldg(reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(p.q) + base));
                const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
                for (int i2 = 0; i2 < 2; i2++) {
                    if (p.q_dtype == KVQ_F16) {
                        x[2 * i2] = __half2float(__ushort_as_half((unsigned short)(ws[i2] & 0xFFFFu)));
                        x[2 * i2 + 1] = __half2float(__ushort_as_half((unsigned short)(ws[i2] >> 16)));
                    } else {
                        x[2 * i2] = __uint_as_float(ws[i2] << 16);
                        x[2 * i2 + 1] = __uint_as_float(ws[i2] & 0xFFFF0000u);
                    }
                }
            }
            float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
            const float inv = amax > 0.f ? 127.f / amax : 0.f;
            int hi[4], lo[4];
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const float y = x[j] * inv;
                const float r = rintf(y);
                hi[j] = (int)r;
                lo[j] = __float2int_rn((y - r) * 254.f);
            }
            *reinterpret_cast<uint32_t *>(qhi + warp * DH + 4 * lane) = pack_bytes(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint32_t *>(qlo + warp * DH + 4 * lane) = pack_bytes(lo[0], lo[1], lo[2], lo[3]);
            if (lane == 0)
                qfac[warp] = amax * (1.f / (127.f * 254.f)) * p.tau_log2e * (KB == 4 ? 0.0625f : 1.f);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&qbar[0]);
        if (!mbar_wait_bounded(&qbar[0], k & 1u, abort_flag, p.timeout_ns)) return false;
        const int qhd = gid & 3;
        const bool valid = qhd < G;
#pragma unroll
        for (int blk = 0; blk < NG; blk++) {
            const int e0 = (blk / KPL) * 32 * KPL + 8 * KPL * tig + 8 * (blk % KPL);
            uint2 h8 = make_uint2(0u, 0u), l8 = make_uint2(0u, 0u);
            if (valid) {
                h8 = lds_u64(smem_u32(qhi), qhd * DH + e0);
                l8 = lds_u64(smem_u32(qlo), qhd * DH + e0);
            }
            if constexpr (KB == 8) {
                // k-slot 4tig+i <-> element 8tig+i, 16+4tig+i <-> 8tig+4+i
                qh[blk][0] = h8.x; qh[blk][1] = h8.y;
                ql[blk][0] = l8.x; ql[blk][1] = l8.y;
            } else {
                // k-slot 4tig+i <-> element 8tig+2i (low nibbles), 16+4tig+i <-> 8tig+2i+1
                qh[blk][0] = prmt(h8.x, h8.y, 0x6420u); qh[blk][1] = prmt(h8.x, h8.y, 0x7531u);
                ql[blk][0] = prmt(l8.x, l8.y, 0x6420u); ql[blk][1] = prmt(l8.x, l8.y, 0x7531u);
            }
            // qh = [hi | lo] (sub-tile 0's B operand), ql = [lo | hi] (sub-tile 1's)
            if (gid >= 4) {
                const uint32_t t0 = qh[blk][0], t1 = qh[blk][1];
                qh[blk][0] = ql[blk][0];
                qh[blk][1] = ql[blk][1];
                ql[blk][0] = t0;
                ql[blk][1] = t1;
            }
        }
        const int hc = 2 * (tig & 1);   // the lane's first head column
        sqc[0] = hc < G ? qfac[hc] : 0.f;
        sqc[1] = hc + 1 < G ? qfac[hc + 1] : 0.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(&qbar[1]);
        // a fresh softmax state and accumulators for the segment
#pragma unroll
        for (int c = 0; c < 2; c++) {
            m_run[c] = -INFINITY;
            l_run[c] = 0.f;
        }
#pragma unroll
        for (int g = 0; g < NVG; g++) psum[g][0] = psum[g][1] = psum[g][2] = psum[g][3] = 0.f;
#pragma unroll
        for (int mt = 0; mt < 2 * NG; mt++)
#pragma unroll
            for (int i2 = 0; i2 < 4; i2++) o_acc[mt][i2] = 0.f;
        return true;
    };

    // int8 A fragments of one 32-element key block for the rows at shared
    // addresses ra (row gid) and rb (row gid + 8), plus IMM bytes
    auto key_frags = [&](auto imm, uint32_t ra, uint32_t rb, uint32_t (&fa)[4]) {
        constexpr int IMM = decltype(imm)::value;
        if constexpr (KB == 8) {
            const uint2 r0 = ldsi_u64<IMM>(ra);
            const uint2 r1 = ldsi_u64<IMM>(rb);
            fa[0] = r0.x; fa[1] = r1.x; fa[2] = r0.y; fa[3] = r1.y;
        } else {
            const uint32_t r0 = ldsi_u32<IMM>(ra);
            const uint32_t r1 = ldsi_u32<IMM>(rb);
            fa[0] = (r0 << 4) & 0xF0F0F0F0u; fa[1] = (r1 << 4) & 0xF0F0F0F0u;
            fa[2] = r0 & 0xF0F0F0F0u;        fa[3] = r1 & 0xF0F0F0F0u;
        }
    };
    // key-row addresses of block blk for sub-tile u: {address, immediate}
    using Imm0 = std::integral_constant<int, 0>;
    using ImmK = std::integral_constant<int, KREP ? KU : 0>;
    using ImmV = std::integral_constant<int, VREP ? VU : 0>;

    const uint64_t limit = p.timeout_ns;
    const uint32_t ONE2 = 0x3C003C00u;   // half2(1, 1)
    // per-tensor scales (caller-set, read once)
    const float k_tensor = PT ? __half2float(p.k_scales[0]) : 0.f;
    const float v_tensor = PT ? __half2float(p.v_scales[0]) : 0.f;
    int s = 0;
    uint32_t ph = 0;
    uint32_t nseg = 0;           // segment ends handed to the combiner
    uint32_t nqs = 0;            // segment starts with the query quantisation shared
    bool aborted = false;
    // the first segment's query is loaded while its first tile is in flight
    if (n_units > 0) load_q(wr.bh0);
    for (int i = 0; i < n_units; i++) {
        if (!mbar_wait_bounded(&full[s], ph, abort_flag, limit)) {
            ctl[0] = 1;
            atomicExch(p.status, KVQ_ERR_TIMEOUT);
            aborted = true;
            break;
        }
        StageMeta m;
        {
            const uint4 m0 = *reinterpret_cast<const uint4 *>(&meta[s]);
            const uint4 m1 = *(reinterpret_cast<const uint4 *>(&meta[s]) + 1);
            m.bh = (int)m0.x; m.t0 = (int)m0.y; m.len = (int)m0.z; m.flags = (int)m0.w;
            m.slot = (int)m1.x; m.ncta = (int)m1.y; m.cmin = (int)m1.z;
        }
        if ((m.flags & 1) && i > 0) {
            if (QSHARE && p.off_qmisc != 0) {
                if (!share_q(m.bh, nqs++)) {
                    ctl[0] = 1;
                    atomicExch(p.status, KVQ_ERR_TIMEOUT);
                    aborted = true;
                    break;
                }
            } else {
                load_q(m.bh);
            }
        }
        const uint32_t st = (uint32_t)s * p.stage_bytes;   // stage offset from smem
        const uint32_t sst = sbase + st;                    // shared address of the stage
        const uint32_t ssk = st + p.off_sk;   // fp16 key scales of the stage
        const uint32_t ssv = st + p.off_sv;   // fp16 value scales

        // Work of this warp on the stage: two 16-token sub-tiles u = 0, 1, processed
        // phase by phase so that the two sub-tiles give the scheduler independent
        // instruction streams at every step.
        int tAu[2];
        bool vt[2][2];
#pragma unroll
        for (int u = 0; u < 2; u++) {
            tAu[u] = warp * 32 + u * 16 + rt;               // score rows: tAu, tAu + 1
            vt[u][0] = m.t0 + tAu[u] < m.len;
            vt[u][1] = m.t0 + tAu[u] + 1 < m.len;
        }

        // ---------------- phase 1: scores S^T = K q^T for both sub-tiles ----------
        float s2[2][4];
        if constexpr (IMMA_K) {
            if constexpr (!kgrp) {
                // hi and lo chains are independent; combined once per tile
                int ah[2][4], al[2][4];
#pragma unroll
                for (int u = 0; u < 2; u++)
#pragma unroll
                    for (int e = 0; e < 4; e++) ah[u][e] = al[u][e] = 0;
                if constexpr (KWIDE) {
                    // one 16-byte load per row and sub-tile holds KPL blocks
#pragma unroll
                    for (int lp = 0; lp < NG / KPL; lp++) {
                        const uint32_t ra = sst + blk_addr<RK, 4 * KLW>(kofs[0][0], lp);
                        const uint32_t rb = sst + blk_addr<RK, 4 * KLW>(kofs[0][1], lp);
                        uint4 r[2][2];
                        r[0][0] = ldsi_u128<0>(ra);
                        r[0][1] = ldsi_u128<0>(rb);
                        r[1][0] = ldsi_u128<ImmK::value>(KREP ? ra : sst + blk_addr<RK, 4 * KLW>(kofs[1][0], lp));
                        r[1][1] = ldsi_u128<ImmK::value>(KREP ? rb : sst + blk_addr<RK, 4 * KLW>(kofs[1][1], lp));
#pragma unroll
                        for (int bi = 0; bi < KPL; bi++) {
                            const int blk = lp * KPL + bi;
#pragma unroll
                            for (int u = 0; u < 2; u++) {
                                const uint4 r0 = r[u][0], r1 = r[u][1];
                                uint32_t fa[4];
                                if constexpr (KB == 8) {
                                    // block bi: bytes 8bi .. 8bi+7 of the lane's 16
                                    fa[0] = bi ? r0.z : r0.x; fa[2] = bi ? r0.w : r0.y;
                                    fa[1] = bi ? r1.z : r1.x; fa[3] = bi ? r1.w : r1.y;
                                } else {
                                    // block bi: word bi (8 nibbles) of the lane's 16 bytes
                                    const uint32_t w0 = bi == 0 ? r0.x : (bi == 1 ? r0.y : (bi == 2 ? r0.z : r0.w));
                                    const uint32_t w1 = bi == 0 ? r1.x : (bi == 1 ? r1.y : (bi == 2 ? r1.z : r1.w));
                                    fa[0] = (w0 << 4) & 0xF0F0F0F0u; fa[1] = (w1 << 4) & 0xF0F0F0F0u;
                                    fa[2] = w0 & 0xF0F0F0F0u;        fa[3] = w1 & 0xF0F0F0F0u;
                                }
                                if constexpr (PK) {
                                    imma_16832<ZP>(ah[u], fa[0], fa[1], fa[2], fa[3], u ? ql[blk][0] : qh[blk][0],
                                                   u ? ql[blk][1] : qh[blk][1]);
                                } else {
                                    imma_16832<ZP>(ah[u], fa[0], fa[1], fa[2], fa[3], qh[blk][0], qh[blk][1]);
                                    imma_16832<ZP>(al[u], fa[0], fa[1], fa[2], fa[3], ql[blk][0], ql[blk][1]);
                                }
                            }
                        }
                    }
                } else {
#pragma unroll
                for (int blk = 0; blk < NG; blk++) {
                    const uint32_t ra = sst + blk_addr<RK, SK>(kofs[0][0], blk);
                    const uint32_t rb = sst + blk_addr<RK, SK>(kofs[0][1], blk);
                    uint32_t fa[2][4];
                    key_frags(Imm0{}, ra, rb, fa[0]);
                    if constexpr (KREP)
                        key_frags(ImmK{}, ra, rb, fa[1]);
                    else
                        key_frags(Imm0{}, sst + blk_addr<RK, SK>(kofs[1][0], blk),
                                  sst + blk_addr<RK, SK>(kofs[1][1], blk), fa[1]);
#pragma unroll
                    for (int u = 0; u < 2; u++) {
                        if constexpr (PK) {
                            imma_16832<ZP>(ah[u], fa[u][0], fa[u][1], fa[u][2], fa[u][3], u ? ql[blk][0] : qh[blk][0],
                                           u ? ql[blk][1] : qh[blk][1]);
                        } else {
                            imma_16832<ZP>(ah[u], fa[u][0], fa[u][1], fa[u][2], fa[u][3], qh[blk][0], qh[blk][1]);
                            imma_16832<ZP>(al[u], fa[u][0], fa[u][1], fa[u][2], fa[u][3], ql[blk][0], ql[blk][1]);
                        }
                    }
                }
                }
                if constexpr (PK) {
                    // lanes tig < 2: own hi of sub-tile 0 (ah[0]), partner's lo (its ah[0]);
                    // lanes tig >= 2: own hi of sub-tile 1 (ah[1]), partner's lo (its ah[1])
                    const int tl = ul ? tAu[1] : tAu[0];
                    float2 kk;
                    int z0 = 0, z1 = 0;   // zero-points of the lane's two score rows
                    if constexpr (PT) {
                        kk = make_float2(k_tensor, k_tensor);
                    } else if constexpr (ZP) {
                        const uint2 w = lds_u64(sbase, ssk + 4 * tl);
                        kk = make_float2(__half2float(__ushort_as_half((unsigned short)(w.x & 0xFFFFu))),
                                         __half2float(__ushort_as_half((unsigned short)(w.y & 0xFFFFu))));
                        z0 = __half2int_rn(__ushort_as_half((unsigned short)(w.x >> 16)));
                        z1 = __half2int_rn(__ushort_as_half((unsigned short)(w.y >> 16)));
                    } else {
                        kk = unpack_half2(lds_u32(sbase, ssk + 2 * tl));
                    }
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const int mine = ul ? ah[1][e] : ah[0][e];
                        const int send = ul ? ah[0][e] : ah[1][e];
                        int a = mine * 254 + __shfl_xor_sync(FULL, send, 2);
                        if constexpr (ZP) a -= ((e < 2) ? z0 : z1) * zq[0][e & 1];
                        s2[0][e] = (float)a * (((e < 2) ? kk.x : kk.y) * sqc[e & 1]);
                    }
                } else {
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    float2 kk;
                    int z0 = 0, z1 = 0;   // zero-points of the two score rows
                    if constexpr (PT) {
                        kk = make_float2(k_tensor, k_tensor);
                    } else if constexpr (ZP) {
                        // (scale, zero-point) of tokens tA, tA + 1
                        const uint2 w = lds_u64(sbase, ssk + 4 * tAu[u]);
                        kk = make_float2(__half2float(__ushort_as_half((unsigned short)(w.x & 0xFFFFu))),
                                         __half2float(__ushort_as_half((unsigned short)(w.y & 0xFFFFu))));
                        z0 = __half2int_rn(__ushort_as_half((unsigned short)(w.x >> 16)));
                        z1 = __half2int_rn(__ushort_as_half((unsigned short)(w.y >> 16)));
                    } else {
                        kk = unpack_half2(lds_u32(sbase, ssk + 2 * tAu[u]));
                    }
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const float ks = (e < 2) ? kk.x : kk.y;
                        int a = ah[u][e] * 254 + al[u][e];
                        if constexpr (ZP) a -= ((e < 2) ? z0 : z1) * zq[0][e & 1];
                        s2[u][e] = (float)a * (ks * sqc[e & 1]);
                    }
                }
                }
            } else {
                float fk[2][4];   // PK: each sub-tile's single (hi | lo) chain, scaled per block
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    float v[4] = {0.f, 0.f, 0.f, 0.f};
                    const int tA = tAu[u];
                    constexpr int SCV = scale_vals(FMT);
                    // key scales of rows tA, tA + 1 per block: with 32-element groups
                    // (no zero-points) a row's NG scales are contiguous, one load per row
                    float kr0[NG], kr1[NG];
                    if (!ZP && p.kshift == 0) {
                        if constexpr (NG == 4) {
                            const uint2 a = lds_u64(sbase, ssk + 8 * tA), b = lds_u64(sbase, ssk + 8 * (tA + 1));
                            const float2 a0 = unpack_half2(a.x), a1 = unpack_half2(a.y);
                            const float2 b0 = unpack_half2(b.x), b1 = unpack_half2(b.y);
                            kr0[0] = a0.x; kr0[1] = a0.y; kr0[2] = a1.x; kr0[3] = a1.y;
                            kr1[0] = b0.x; kr1[1] = b0.y; kr1[2] = b1.x; kr1[3] = b1.y;
                        } else {
                            const float2 a = unpack_half2(lds_u32(sbase, ssk + 4 * tA));
                            const float2 b = unpack_half2(lds_u32(sbase, ssk + 4 * (tA + 1)));
                            kr0[0] = a.x; kr0[1] = a.y;
                            kr1[0] = b.x; kr1[1] = b.y;
                        }
                    } else {
#pragma unroll
                        for (int blk = 0; blk < NG; blk++) {
                            const uint32_t o0 = ssk + 2 * (tA * p.ngs_k + SCV * (blk >> p.kshift));
                            const uint32_t o1 = ssk + 2 * ((tA + 1) * p.ngs_k + SCV * (blk >> p.kshift));
                            kr0[blk] = __half2float(__ushort_as_half((unsigned short)lds_u16(sbase, o0)));
                            kr1[blk] = __half2float(__ushort_as_half((unsigned short)lds_u16(sbase, o1)));
                        }
                    }
#pragma unroll
                    for (int blk = 0; blk < NG; blk++) {
                        int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
                        uint32_t fa[4];
                        key_frags(Imm0{}, sst + blk_addr<RK, SK>(kofs[u][0], blk),
                                  sst + blk_addr<RK, SK>(kofs[u][1], blk), fa);
                        const float k0 = kr0[blk], k1 = kr1[blk];
                        if constexpr (PK) {
                            imma_16832<ZP>(ah, fa[0], fa[1], fa[2], fa[3], u ? ql[blk][0] : qh[blk][0],
                                           u ? ql[blk][1] : qh[blk][1]);
                            v[0] = fmaf(k0, (float)ah[0], v[0]);
                            v[1] = fmaf(k0, (float)ah[1], v[1]);
                            v[2] = fmaf(k1, (float)ah[2], v[2]);
                            v[3] = fmaf(k1, (float)ah[3], v[3]);
                            continue;
                        }
                        imma_16832<ZP>(ah, fa[0], fa[1], fa[2], fa[3], qh[blk][0], qh[blk][1]);
                        imma_16832<ZP>(al, fa[0], fa[1], fa[2], fa[3], ql[blk][0], ql[blk][1]);
                        if constexpr (ZP) {
                            // minus zero-point x the block's query sum
                            const uint32_t o0 = ssk + 2 * (tA * p.ngs_k + SCV * (blk >> p.kshift));
                            const uint32_t o1 = ssk + 2 * ((tA + 1) * p.ngs_k + SCV * (blk >> p.kshift));
                            const int z0 = __half2int_rn(__ushort_as_half((unsigned short)lds_u16(sbase, o0 + 2)));
                            const int z1 = __half2int_rn(__ushort_as_half((unsigned short)lds_u16(sbase, o1 + 2)));
                            ah[0] = ah[0] * 254 + al[0] - z0 * zq[blk][0];
                            ah[1] = ah[1] * 254 + al[1] - z0 * zq[blk][1];
                            ah[2] = ah[2] * 254 + al[2] - z1 * zq[blk][0];
                            ah[3] = ah[3] * 254 + al[3] - z1 * zq[blk][1];
                        } else {
#pragma unroll
                            for (int e = 0; e < 4; e++) ah[e] = ah[e] * 254 + al[e];
                        }
                        v[0] = fmaf(k0, (float)ah[0], v[0]);
                        v[1] = fmaf(k0, (float)ah[1], v[1]);
                        v[2] = fmaf(k1, (float)ah[2], v[2]);
                        v[3] = fmaf(k1, (float)ah[3], v[3]);
                    }
                    if constexpr (PK) {
#pragma unroll
                        for (int e = 0; e < 4; e++) fk[u][e] = v[e];
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; e++) s2[u][e] = v[e] * sqc[e & 1];
                    }
                }
                if constexpr (PK) {
                    // join hi (own chain) and lo (partner's) as for per-head key scales
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const float mine = ul ? fk[1][e] : fk[0][e];
                        const float send = ul ? fk[0][e] : fk[1][e];
                        s2[0][e] = fmaf(254.f, mine, __shfl_xor_sync(FULL, send, 2)) * sqc[e & 1];
                    }
                }
            }
        } else if constexpr (F8) {
            // e4m3 keys: each code pair converts exactly to a half2 in registers;
            // lane tig's 8 bytes of a block are elements 8tig .. 8tig+7, the k-slot
            // order of the fp16 query fragments
            auto f8_frags = [&](uint2 r0, uint2 r1, int hs, uint32_t (&fa)[4]) {
                const uint32_t w0 = hs ? r0.y : r0.x, w1 = hs ? r1.y : r1.x;
                fa[0] = e4m3x2_to_half2(w0 & 0xFFFFu); fa[1] = e4m3x2_to_half2(w1 & 0xFFFFu);
                fa[2] = e4m3x2_to_half2(w0 >> 16);     fa[3] = e4m3x2_to_half2(w1 >> 16);
            };
            if constexpr (!kgrp) {
                float acc[2][2][4];
#pragma unroll
                for (int u = 0; u < 2; u++)
#pragma unroll
                    for (int h = 0; h < 2; h++) acc[u][h][0] = acc[u][h][1] = acc[u][h][2] = acc[u][h][3] = 0.f;
#pragma unroll
                for (int blk = 0; blk < NG; blk++) {
                    const uint32_t ra = sst + blk_addr<RK, SK>(kofs[0][0], blk);
                    const uint32_t rb = sst + blk_addr<RK, SK>(kofs[0][1], blk);
                    uint2 r[2][2];
                    r[0][0] = ldsi_u64<0>(ra);
                    r[0][1] = ldsi_u64<0>(rb);
                    r[1][0] = ldsi_u64<ImmK::value>(KREP ? ra : sst + blk_addr<RK, SK>(kofs[1][0], blk));
                    r[1][1] = ldsi_u64<ImmK::value>(KREP ? rb : sst + blk_addr<RK, SK>(kofs[1][1], blk));
#pragma unroll
                    for (int u = 0; u < 2; u++)
#pragma unroll
                        for (int hs = 0; hs < 2; hs++) {
                            uint32_t fa[4];
                            f8_frags(r[u][0], r[u][1], hs, fa);
                            if constexpr (PK)
                                mma_16816(acc[u][hs], fa[0], fa[1], fa[2], fa[3],
                                          u ? qb2[PK && F8 ? blk : 0][hs][0] : qb[blk][hs][0],
                                          u ? qb2[PK && F8 ? blk : 0][hs][1] : qb[blk][hs][1]);
                            else
                                mma_16816(acc[u][hs], fa[0], fa[1], fa[2], fa[3], qb[blk][hs][0], qb[blk][hs][1]);
                        }
                }
                if constexpr (PK) {
                    // as for int8 keys: the lane's own chain holds its heads' hi part, the
                    // partner's (lane ^ 2) the lo part of the same heads
                    const float2 kk = unpack_half2(lds_u32(sbase, ssk + 2 * (ul ? tAu[1] : tAu[0])));
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        const float v0 = acc[0][0][e] + acc[0][1][e], v1 = acc[1][0][e] + acc[1][1][e];
                        const float mine = ul ? v1 : v0, send = ul ? v0 : v1;
                        s2[0][e] = (mine + __shfl_xor_sync(FULL, send, 2)) *
                                   (((e < 2) ? kk.x : kk.y) * p.tau_log2e);
                    }
                } else {
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    const float2 kk = unpack_half2(lds_u32(sbase, ssk + 2 * tAu[u]));
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        float v = (acc[u][0][e] + acc[u][1][e]) * (((e < 2) ? kk.x : kk.y) * p.tau_log2e);
                        if (qsplit) v += __shfl_xor_sync(FULL, v, 2);
                        s2[u][e] = v;
                    }
                }
                }
            } else {
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    float v[4] = {0.f, 0.f, 0.f, 0.f};
                    const int tA = tAu[u];
#pragma unroll
                    for (int blk = 0; blk < NG; blk++) {
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
                        const uint2 r0 = ldsi_u64<0>(sst + blk_addr<RK, SK>(kofs[u][0], blk));
                        const uint2 r1 = ldsi_u64<0>(sst + blk_addr<RK, SK>(kofs[u][1], blk));
#pragma unroll
                        for (int hs = 0; hs < 2; hs++) {
                            uint32_t fa[4];
                            f8_frags(r0, r1, hs, fa);
                            mma_16816(acc, fa[0], fa[1], fa[2], fa[3], qb[blk][hs][0], qb[blk][hs][1]);
                        }
                        const float k0 = __half2float(__ushort_as_half(
                            (unsigned short)lds_u16(sbase, ssk + 2 * (tA * p.ngs_k + (blk >> p.kshift)))));
                        const float k1 = __half2float(__ushort_as_half(
                            (unsigned short)lds_u16(sbase, ssk + 2 * ((tA + 1) * p.ngs_k + (blk >> p.kshift)))));
                        v[0] = fmaf(k0, acc[0], v[0]);
                        v[1] = fmaf(k0, acc[1], v[1]);
                        v[2] = fmaf(k1, acc[2], v[2]);
                        v[3] = fmaf(k1, acc[3], v[3]);
                    }
#pragma unroll
                    for (int e = 0; e < 4; e++) {
                        float x = v[e] * p.tau_log2e;
                        if (qsplit) x += __shfl_xor_sync(FULL, x, 2);
                        s2[u][e] = x;
                    }
                }
            }
        } else {
            // fp16 keys: two partial accumulators per sub-tile halve the MMA chain
            float acc[2][2][4];
#pragma unroll
            for (int u = 0; u < 2; u++)
#pragma unroll
                for (int h = 0; h < 2; h++) acc[u][h][0] = acc[u][h][1] = acc[u][h][2] = acc[u][h][3] = 0.f;
#pragma unroll
            for (int blk = 0; blk < NG; blk++) {
                const uint32_t ra = sst + blk_addr<RK, SK>(kofs[0][0], blk);
                const uint32_t rb = sst + blk_addr<RK, SK>(kofs[0][1], blk);
                uint4 r[2][2];
                r[0][0] = ldsi_u128<0>(ra);
                r[0][1] = ldsi_u128<0>(rb);
                r[1][0] = ldsi_u128<ImmK::value>(KREP ? ra : sst + blk_addr<RK, SK>(kofs[1][0], blk));
                r[1][1] = ldsi_u128<ImmK::value>(KREP ? rb : sst + blk_addr<RK, SK>(kofs[1][1], blk));
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    const uint4 r0 = r[u][0], r1 = r[u][1];
                    mma_16816(acc[u][blk & 1], r0.x, r1.x, r0.y, r1.y, qb[blk][0][0], qb[blk][0][1]);
                    mma_16816(acc[u][blk & 1], r0.z, r1.z, r0.w, r1.w, qb[blk][1][0], qb[blk][1][1]);
                }
            }
#pragma unroll
            for (int u = 0; u < 2; u++)
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    float v = (acc[u][0][e] + acc[u][1][e]) * p.tau_log2e;
                    if (qsplit) v += __shfl_xor_sync(FULL, v, 2);
                    s2[u][e] = v;
                }
        }
        if constexpr (PK) {
            // from here on a lane's score rows are those of its own sub-tile
            tAu[0] = ul ? tAu[1] : tAu[0];
            vt[0][0] = ul ? vt[1][0] : vt[0][0];
            vt[0][1] = ul ? vt[1][1] : vt[0][1];
        }
#pragma unroll
        for (int u = 0; u < NU; u++) {
            // Padding columns (heads >= G, or the residual columns of a split
            // query) carry finite scores from zero query columns; their outputs
            // are never written, so only tokens past the length are masked.
            s2[u][0] = vt[u][0] ? s2[u][0] : -INFINITY;
            s2[u][1] = vt[u][0] ? s2[u][1] : -INFINITY;
            s2[u][2] = vt[u][1] ? s2[u][2] : -INFINITY;
            s2[u][3] = vt[u][1] ? s2[u][3] : -INFINITY;
        }

        // ---------------- phase 2: value scales of the score rows -----------------
        float sv[2][2][NVG];   // [sub-tile][row][value group]
        float lsv[2][2];
        // uint8 values: A fragments half2(1024 + z) of the P.V k-slot tokens (tw + vA,
        // tw + vB; tw + vA + 1, tw + vB + 1), zero past the length (stale scales), set
        // after the scale loop below
        uint32_t za[2][NVG][2];
#pragma unroll
        for (int u = 0; u < NU; u++) {
            const int tA = tAu[u];
            constexpr int SCV = scale_vals(FMT);
            if constexpr (VB == 16) {
                sv[u][0][0] = sv[u][1][0] = 1.f;
            } else if constexpr (PT) {
                sv[u][0][0] = sv[u][1][0] = v_tensor;
            } else if constexpr (!vgrp) {
                if constexpr (ZP) {
                    const uint2 w = lds_u64(sbase, ssv + 4 * tA);
                    sv[u][0][0] = __half2float(__ushort_as_half((unsigned short)(w.x & 0xFFFFu)));
                    sv[u][1][0] = __half2float(__ushort_as_half((unsigned short)(w.y & 0xFFFFu)));
                } else {
                    const float2 vv = unpack_half2(lds_u32(sbase, ssv + 2 * tA));
                    sv[u][0][0] = vv.x;
                    sv[u][1][0] = vv.y;
                }
            } else {
#pragma unroll
                for (int g = 0; g < NG; g++) {
                    sv[u][0][g] = __half2float(__ushort_as_half(
                        (unsigned short)lds_u16(sbase, ssv + 2 * (tA * p.ngs_v + SCV * (g >> p.vshift)))));
                    sv[u][1][g] = __half2float(__ushort_as_half(
                        (unsigned short)lds_u16(sbase, ssv + 2 * ((tA + 1) * p.ngs_v + SCV * (g >> p.vshift)))));
                }
            }
            // scales past the length may be stale shared memory: never use them
#pragma unroll
            for (int r = 0; r < 2; r++) {
                float mx = 0.f;
#pragma unroll
                for (int g = 0; g < NVG; g++) {
                    sv[u][r][g] = vt[u][r] ? sv[u][r][g] : 0.f;
                    mx = fmaxf(mx, sv[u][r][g]);
                }
                lsv[u][r] = mx > 0.f ? fmaxf(__log2f(mx), -32.f) : -32.f;
            }
        }

        // uint8 values: the za fragments of both sub-tiles (with packed columns too, each
        // sub-tile's P.V MMA takes its own)
        if constexpr (ZP) {
            constexpr int SCV = scale_vals(FMT);
            const uint32_t B1024 = 0x64006400u;   // half2(1024, 1024)
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int tw = warp * 32 + u * 16;
                const int rem = m.len - m.t0 - tw;   // valid tokens of the sub-tile
                const uint32_t mlo = (vA < rem ? 0x0000FFFFu : 0u) | (vB < rem ? 0xFFFF0000u : 0u);
                const uint32_t mhi = (vA + 1 < rem ? 0x0000FFFFu : 0u) | (vB + 1 < rem ? 0xFFFF0000u : 0u);
                if constexpr (!vgrp) {
                    const uint2 wA = lds_u64(sbase, ssv + 4 * (tw + vA));   // (s, z) of tw+vA, tw+vA+1
                    const uint2 wB = lds_u64(sbase, ssv + 4 * (tw + vB));
                    za[u][0][0] = hadd2_u32(prmt(wA.x, wB.x, 0x7632u) & mlo, B1024);
                    za[u][0][1] = hadd2_u32(prmt(wA.y, wB.y, 0x7632u) & mhi, B1024);
                } else {
#pragma unroll
                    for (int g = 0; g < NG; g++) {
                        const uint32_t zo = 2 * (SCV * (g >> p.vshift) + 1);
                        const uint32_t a0 = lds_u16(sbase, ssv + 2 * (tw + vA) * p.ngs_v + zo);
                        const uint32_t b0 = lds_u16(sbase, ssv + 2 * (tw + vB) * p.ngs_v + zo);
                        const uint32_t a1 = lds_u16(sbase, ssv + 2 * (tw + vA + 1) * p.ngs_v + zo);
                        const uint32_t b1 = lds_u16(sbase, ssv + 2 * (tw + vB + 1) * p.ngs_v + zo);
                        za[u][g][0] = hadd2_u32((a0 | (b0 << 16)) & mlo, B1024);
                        za[u][g][1] = hadd2_u32((a1 | (b1 << 16)) & mhi, B1024);
                    }
                }
            }
        }

        // ---------------- phase 3: online softmax, one lazy check for 32 tokens ---
        {
            float loc0 = -INFINITY, loc1 = -INFINITY;
#pragma unroll
            for (int u = 0; u < NU; u++) {
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
                for (int g = 0; g < NVG; g++) {
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
        // x0 = rows 0..7 of the score tile (tokens tw + row_token(r)), x1 = rows
        // 8..15; their 8x8 transposes are the B fragments of the P.V MMA.
        uint32_t pb[2][NVG][2];
        if constexpr (PK) {
            // one transposed fragment holds both sub-tiles' P: columns (= gid after the
            // transpose) 0-3 sub-tile 0's heads, 4-7 sub-tile 1's; each sub-tile's P.V
            // MMA gets it with the other's columns zeroed
            float pr[4];
#pragma unroll
            for (int e = 0; e < 4; e++)
                pr[e] = (s2[0][e] == -INFINITY) ? 0.f : fast_exp2(s2[0][e] - m_run[e & 1]);
            l_run[0] += pr[0] + pr[2];
            l_run[1] += pr[1] + pr[3];
            const uint32_t keep0 = gid < 4 ? 0xFFFFFFFFu : 0u;
#pragma unroll
            for (int g = 0; g < NVG; g++) {
                const uint32_t t0 = movmatrix_trans(pack_half2(pr[0] * sv[0][0][g], pr[1] * sv[0][0][g]));
                const uint32_t t1 = movmatrix_trans(pack_half2(pr[2] * sv[0][1][g], pr[3] * sv[0][1][g]));
                pb[0][g][0] = t0 & keep0;
                pb[0][g][1] = t1 & keep0;
                pb[1][g][0] = t0 & ~keep0;
                pb[1][g][1] = t1 & ~keep0;
                if constexpr (ZP) {
                    // each sub-tile's zero-points against its own columns
#pragma unroll
                    for (int u = 0; u < 2; u++)
                        mma_16816(psum[g], za[u][g][0], za[u][g][0], za[u][g][1], za[u][g][1], pb[u][g][0],
                                  pb[u][g][1]);
                } else if constexpr (VBIAS) {
                    mma_16816(psum[g], ONE2, ONE2, ONE2, ONE2, t0, t1);
                }
            }
        } else {
#pragma unroll
        for (int u = 0; u < 2; u++) {
            float pr[4];
#pragma unroll
            for (int e = 0; e < 4; e++)
                pr[e] = (s2[u][e] == -INFINITY) ? 0.f : fast_exp2(s2[u][e] - m_run[e & 1]);
            l_run[0] += pr[0] + pr[2];
            l_run[1] += pr[1] + pr[3];
#pragma unroll
            for (int g = 0; g < NVG; g++) {
                const uint32_t x0 = pack_half2(pr[0] * sv[u][0][g], pr[1] * sv[u][0][g]);
                const uint32_t x1 = pack_half2(pr[2] * sv[u][1][g], pr[3] * sv[u][1][g]);
                pb[u][g][0] = movmatrix_trans(x0);
                pb[u][g][1] = movmatrix_trans(x1);
                // column sums of the fp16 weights, for the code bias
                if constexpr (ZP)
                    mma_16816(psum[g], za[u][g][0], za[u][g][0], za[u][g][1], za[u][g][1], pb[u][g][0],
                              pb[u][g][1]);
                else if constexpr (VBIAS)
                    mma_16816(psum[g], ONE2, ONE2, ONE2, ONE2, pb[u][g][0], pb[u][g][1]);
            }
        }
        }

        // ---------------- phase 5: O^T += V^T P for both sub-tiles ----------------
        if constexpr (VWIDE) {
            // m-tile 4sb + j: row gid <-> d = 64sb + 8gid + 2j, row gid + 8 <-> d + 1
#pragma unroll
            for (int sb = 0; sb < NG / 2; sb++) {
                uint32_t va[2][4];
#pragma unroll
                for (int r = 0; r < 4; r++) {
                    va[0][r] = sst + blk_addr<RV, 2 * SV>(vofs[0][r], sb);
                    va[1][r] = VREP ? va[0][r] : sst + blk_addr<RV, 2 * SV>(vofs[1][r], sb);
                }
#pragma unroll
                for (int u = 0; u < 2; u++) {
                    const uint32_t b0 = pb[u][0][0], b1 = pb[u][0][1];
                    if constexpr (F8) {
                        // e4m3 values past the length may be stale (a NaN code): zero them
                        const int tg = m.t0 + warp * 32 + u * 16;
                        uint2 w[4];
#pragma unroll
                        for (int r = 0; r < 4; r++) {
                            const int tok = tg + ((r & 1) ? vB : vA) + (r >> 1);
                            w[r] = make_uint2(0u, 0u);
                            if (tok < m.len) w[r] = u == 0 ? ldsi_u64<0>(va[0][r]) : ldsi_u64<ImmV::value>(va[1][r]);
                        }
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            // bytes 2j', 2j'+1 (j' = j mod 2) of tokens A, B interleaved:
                            // low half (A, B) element 2j', high half the next element
                            const uint32_t sel = (j & 1) ? 0x7362u : 0x5140u;
                            const uint32_t A = j < 2 ? w[0].x : w[0].y, Bw = j < 2 ? w[1].x : w[1].y;
                            const uint32_t C = j < 2 ? w[2].x : w[2].y, E = j < 2 ? w[3].x : w[3].y;
                            const uint32_t yAB = prmt(A, Bw, sel), yCE = prmt(C, E, sel);
                            mma_16816(o_acc[4 * sb + j], e4m3x2_to_half2(yAB & 0xFFFFu), e4m3x2_to_half2(yAB >> 16),
                                      e4m3x2_to_half2(yCE & 0xFFFFu), e4m3x2_to_half2(yCE >> 16), b0, b1);
                        }
                    } else if constexpr (VB == 8) {
                        uint2 w[4];
#pragma unroll
                        for (int r = 0; r < 4; r++)
                            w[r] = u == 0 ? ldsi_u64<0>(va[0][r]) : ldsi_u64<ImmV::value>(va[1][r]);
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
                            const uint32_t A = j < 2 ? w[0].x : w[0].y, Bw = j < 2 ? w[1].x : w[1].y;
                            const uint32_t C = j < 2 ? w[2].x : w[2].y, E = j < 2 ? w[3].x : w[3].y;
                            const uint32_t yAB = prmt(A, Bw, sel), yCE = prmt(C, E, sel);
                            const uint32_t a0 = and_xor(yAB, 0x00FF00FFu, VX);
                            const uint32_t a1 = and_xor(yAB >> 8, 0x00FF00FFu, VX);
                            const uint32_t a2 = and_xor(yCE, 0x00FF00FFu, VX);
                            const uint32_t a3 = and_xor(yCE >> 8, 0x00FF00FFu, VX);
                            mma_16816(o_acc[4 * sb + j], a0, a1, a2, a3, b0, b1);
                        }
                    } else if constexpr (VLDSM) {
                        // y[2wi + h]: token half h, 32-dim window wi; per lane the 4 dims
                        // 64sb + 32wi + 4gid .. + 3 of its k-slot pair.  m-tile 4sb + 2wi + q
                        // takes dims 4gid + 2q (rows gid: 1032 + code) and 4gid + 2q + 1
                        // (rows gid + 8: 1152 + 16 code)
                        uint32_t y[4];
                        if (u == 0)
                            ldsm_x4_trans<0>(va[0][0], y);
                        else
                            ldsm_x4_trans<ImmV::value>(va[1][0], y);
#pragma unroll
                        for (int wi = 0; wi < 2; wi++)
#pragma unroll
                            for (int q = 0; q < 2; q++) {
                                const uint32_t x0 = q ? y[2 * wi] >> 8 : y[2 * wi];
                                const uint32_t x1 = q ? y[2 * wi + 1] >> 8 : y[2 * wi + 1];
                                const uint32_t a0 = and_xor(x0, 0x000F000Fu, 0x64086408u);
                                const uint32_t a1 = and_xor(x0, 0x00F000F0u, 0x64806480u);
                                const uint32_t a2 = and_xor(x1, 0x000F000Fu, 0x64086408u);
                                const uint32_t a3 = and_xor(x1, 0x00F000F0u, 0x64806480u);
                                mma_16816(o_acc[4 * sb + 2 * wi + q], a0, a1, a2, a3, b0, b1);
                            }
                    } else if constexpr (VB == 4) {
                        uint32_t w[4];
#pragma unroll
                        for (int r = 0; r < 4; r++)
                            w[r] = u == 0 ? ldsi_u32<0>(va[0][r]) : ldsi_u32<ImmV::value>(va[1][r]);
#pragma unroll
                        for (int hb = 0; hb < 2; hb++) {
                            // bytes 2hb, 2hb+1 of tokens A, B (C, E): elements 4hb .. 4hb+3
                            const uint32_t sel = hb ? 0x7632u : 0x5410u;
                            const uint32_t yAB = prmt(w[0], w[1], sel), yCE = prmt(w[2], w[3], sel);
#pragma unroll
                            for (int h = 0; h < 2; h++) {
                                // rows gid take the even nibble (1032 + code), rows gid + 8
                                // the odd one in place (1152 + 16 code)
                                const uint32_t xAB = h ? yAB >> 8 : yAB, xCE = h ? yCE >> 8 : yCE;
                                const uint32_t a0 = and_xor(xAB, 0x000F000Fu, 0x64086408u);
                                const uint32_t a1 = and_xor(xAB, 0x00F000F0u, 0x64806480u);
                                const uint32_t a2 = and_xor(xCE, 0x000F000Fu, 0x64086408u);
                                const uint32_t a3 = and_xor(xCE, 0x00F000F0u, 0x64806480u);
                                mma_16816(o_acc[4 * sb + 2 * hb + h], a0, a1, a2, a3, b0, b1);
                            }
                        }
                    } else {
                        // fp16 values past the length may be anything (NaN included): zero them
                        const int tg = m.t0 + warp * 32 + u * 16;
                        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                        uint4 w[4];
#pragma unroll
                        for (int r = 0; r < 4; r++) {
                            const int tok = tg + ((r & 1) ? vB : vA) + (r >> 1);
                            w[r] = z;
                            if (tok < m.len)
                                w[r] = u == 0 ? ldsi_u128<0>(va[0][r]) : ldsi_u128<ImmV::value>(va[1][r]);
                        }
#pragma unroll
                        for (int j = 0; j < 4; j++) {
                            const uint32_t A = j == 0 ? w[0].x : (j == 1 ? w[0].y : (j == 2 ? w[0].z : w[0].w));
                            const uint32_t Bw = j == 0 ? w[1].x : (j == 1 ? w[1].y : (j == 2 ? w[1].z : w[1].w));
                            const uint32_t C = j == 0 ? w[2].x : (j == 1 ? w[2].y : (j == 2 ? w[2].z : w[2].w));
                            const uint32_t E = j == 0 ? w[3].x : (j == 1 ? w[3].y : (j == 2 ? w[3].z : w[3].w));
                            const uint32_t a0 = prmt(A, Bw, 0x5410u), a1 = prmt(A, Bw, 0x7632u);
                            const uint32_t a2 = prmt(C, E, 0x5410u), a3 = prmt(C, E, 0x7632u);
                            mma_16816(o_acc[4 * sb + j], a0, a1, a2, a3, b0, b1);
                        }
                    }
                }
            }
        } else {
#pragma unroll
        for (int blk = 0; blk < NG; blk++) {
            // value-row addresses of this block (sub-tile 0; sub-tile 1 adds VU)
            uint32_t va[2][4];
#pragma unroll
            for (int r = 0; r < 4; r++) {
                va[0][r] = sst + blk_addr<RV, SV>(vofs[0][r], blk);
                va[1][r] = VREP ? va[0][r] : sst + blk_addr<RV, SV>(vofs[1][r], blk);
            }
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const uint32_t b0 = pb[u][VG ? blk : 0][0], b1 = pb[u][VG ? blk : 0][1];
                if constexpr (F8) {
                    // e4m3 values past the length may be stale (a NaN code): zero them
                    const int tg = m.t0 + warp * 32 + u * 16;
                    uint32_t w[4];
#pragma unroll
                    for (int r = 0; r < 4; r++) {
                        const int tok = tg + ((r & 1) ? vB : vA) + (r >> 1);
                        w[r] = 0u;
                        if (tok < m.len) w[r] = u == 0 ? ldsi_u32<0>(va[0][r]) : ldsi_u32<ImmV::value>(va[1][r]);
                    }
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        // (A, B) byte pairs 2h and 2h+1: rows gid and gid + 8
                        const uint32_t sel = h ? 0x7362u : 0x5140u;
                        const uint32_t yAB = prmt(w[0], w[1], sel), yCE = prmt(w[2], w[3], sel);
                        mma_16816(o_acc[2 * blk + h], e4m3x2_to_half2(yAB & 0xFFFFu), e4m3x2_to_half2(yAB >> 16),
                                  e4m3x2_to_half2(yCE & 0xFFFFu), e4m3x2_to_half2(yCE >> 16), b0, b1);
                    }
                } else if constexpr (VB == 8) {
                    uint32_t wA, wB, wC, wE;
                    if (u == 0) {
                        wA = ldsi_u32<0>(va[0][0]); wB = ldsi_u32<0>(va[0][1]);
                        wC = ldsi_u32<0>(va[0][2]); wE = ldsi_u32<0>(va[0][3]);
                    } else {
                        wA = ldsi_u32<ImmV::value>(va[1][0]); wB = ldsi_u32<ImmV::value>(va[1][1]);
                        wC = ldsi_u32<ImmV::value>(va[1][2]); wE = ldsi_u32<ImmV::value>(va[1][3]);
                    }
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const uint32_t sel = h ? 0x7632u : 0x5410u;
                        const uint32_t yAB = prmt(wA, wB, sel), yCE = prmt(wC, wE, sel);
                        const uint32_t a0 = and_xor(yAB, 0x00FF00FFu, VX);
                        const uint32_t a1 = and_xor(yAB >> 8, 0x00FF00FFu, VX);
                        const uint32_t a2 = and_xor(yCE, 0x00FF00FFu, VX);
                        const uint32_t a3 = and_xor(yCE >> 8, 0x00FF00FFu, VX);
                        mma_16816(o_acc[2 * blk + h], a0, a1, a2, a3, b0, b1);
                    }
                } else if constexpr (VB == 4) {
                    uint32_t hA, hB, hC, hE;
                    if (u == 0) {
                        hA = ldsi_u16<0>(va[0][0]); hB = ldsi_u16<0>(va[0][1]);
                        hC = ldsi_u16<0>(va[0][2]); hE = ldsi_u16<0>(va[0][3]);
                    } else {
                        hA = ldsi_u16<ImmV::value>(va[1][0]); hB = ldsi_u16<ImmV::value>(va[1][1]);
                        hC = ldsi_u16<ImmV::value>(va[1][2]); hE = ldsi_u16<ImmV::value>(va[1][3]);
                    }
                    const uint32_t yAB = prmt(hA, hB, 0x5410u), yCE = prmt(hC, hE, 0x5410u);
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        // rows gid take the even nibble (1032 + code), rows gid + 8 the
                        // odd one in place (1152 + 16 code): no shift for it
                        const uint32_t xAB = h ? yAB >> 8 : yAB, xCE = h ? yCE >> 8 : yCE;
                        const uint32_t a0 = and_xor(xAB, 0x000F000Fu, 0x64086408u);
                        const uint32_t a1 = and_xor(xAB, 0x00F000F0u, 0x64806480u);
                        const uint32_t a2 = and_xor(xCE, 0x000F000Fu, 0x64086408u);
                        const uint32_t a3 = and_xor(xCE, 0x00F000F0u, 0x64806480u);
                        mma_16816(o_acc[2 * blk + h], a0, a1, a2, a3, b0, b1);
                    }
                } else {
                    // fp16 values past the length may be anything (NaN included): zero them
                    const int tg = m.t0 + warp * 32 + u * 16;
                    const uint2 z = make_uint2(0u, 0u);
                    uint2 w[4];
#pragma unroll
                    for (int r = 0; r < 4; r++) {
                        const int tok = tg + ((r & 1) ? vB : vA) + (r >> 1);
                        w[r] = z;
                        if (tok < m.len) w[r] = u == 0 ? ldsi_u64<0>(va[0][r]) : ldsi_u64<ImmV::value>(va[1][r]);
                    }
#pragma unroll
                    for (int h = 0; h < 2; h++) {
                        const uint32_t A = h ? w[0].y : w[0].x, Bw = h ? w[1].y : w[1].x;
                        const uint32_t C = h ? w[2].y : w[2].x, E = h ? w[3].y : w[3].x;
                        const uint32_t a0 = prmt(A, Bw, 0x5410u), a1 = prmt(A, Bw, 0x7632u);
                        const uint32_t a2 = prmt(C, E, 0x5410u), a3 = prmt(C, E, 0x7632u);
                        mma_16816(o_acc[2 * blk + h], a0, a1, a2, a3, b0, b1);
                    }
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

        // ---------------- segment end: hand this warp's partial to the combiner ---
        if (m.flags & 2) {
            constexpr int CS = slot_col_floats(DH);
            float lt[2];
#pragma unroll
            for (int c = 0; c < 2; c++) {
                float v = l_run[c];
                v += __shfl_xor_sync(FULL, v, 4);
                v += __shfl_xor_sync(FULL, v, 8);
                v += __shfl_xor_sync(FULL, v, 16);
                lt[c] = v;
            }
            // the combiner must have read the previous segment out of mbuf
            if (nseg > 0 && !mbar_wait_bounded(&segbar[1], (nseg - 1) & 1u, abort_flag, limit)) {
                ctl[0] = 1;
                atomicExch(p.status, KVQ_ERR_TIMEOUT);
                aborted = true;
                break;
            }
            float mw[2] = {m_run[0], m_run[1]};
            if constexpr (PK) {
                // join the two sub-tiles' partials of each head (lanes tig and tig ^ 2):
                // remove the code bias from each, then weight by 2^(m - max)
                float es[2], eo[2];
#pragma unroll
                for (int c = 0; c < 2; c++) {
                    const float mo = __shfl_xor_sync(FULL, m_run[c], 2);
                    const float lo_ = __shfl_xor_sync(FULL, lt[c], 2);
                    const float M = fmaxf(m_run[c], mo);
                    es[c] = (m_run[c] == -INFINITY) ? 0.f : exp2f(m_run[c] - M);
                    eo[c] = (mo == -INFINITY) ? 0.f : exp2f(mo - M);
                    lt[c] = lt[c] * es[c] + lo_ * eo[c];
                    mw[c] = M;
                }
#pragma unroll
                for (int mt = 0; mt < 2 * NG; mt++)
#pragma unroll
                    for (int c = 0; c < 2; c++) {
                        const float ps = psum[VG ? (mt >> 1) : 0][c];
                        float lo = o_acc[mt][c], hi = o_acc[mt][2 + c];
                        if constexpr (VB == 4) {
                            lo -= 1032.f * ps;
                            hi = (hi - 1152.f * ps) * 0.0625f;
                        } else {
                            lo -= BIAS_V * ps;
                            hi -= BIAS_V * ps;
                        }
                        o_acc[mt][c] = lo * es[c] + __shfl_xor_sync(FULL, lo, 2) * eo[c];
                        o_acc[mt][2 + c] = hi * es[c] + __shfl_xor_sync(FULL, hi, 2) * eo[c];
                    }
            }
            // this warp's partial into mbuf[warp]: [G][DH + 4] floats, o then (m, l)
            float *mine = mbuf + (size_t)warp * G * CS;
#pragma unroll
            for (int c = 0; c < 2; c++) {
                const int col = 2 * tig + c;
                if (c == 0 ? col_ok0 : col_ok1) {
                    float *oc = mine + (size_t)col * CS;
#pragma unroll
                    for (int blk = 0; blk < NG; blk++) {
                        const float ps = psum[VG ? blk : 0][c];
#pragma unroll
                        for (int h = 0; h < 2; h++) {
                            // 4-bit wide (ldmatrix): m-tile 4sb + 2wi + q, row gid <-> d =
                            // 64sb + 32wi + 4gid + 2q; wide: m-tile 4sb + j, row gid <-> d = 64sb + 8gid + 2j;
                            // block mapping: m-tile 2blk + h, row gid <-> d = 32blk + 4gid + 2h;
                            // row gid + 8 <-> d + 1
                            const int mt = 2 * blk + h;
                            const int d = VLDSM    ? 64 * (mt >> 2) + 32 * ((mt >> 1) & 1) + 4 * gid + 2 * (mt & 1)
                                        : VWIDE  ? 64 * (mt >> 2) + 8 * gid + 2 * (mt & 3)
                                                 : 32 * blk + 4 * gid + 2 * h;
                            float lo = o_acc[mt][c], hi = o_acc[mt][2 + c];
                            if constexpr (PK) {
                                // joined and unbiased above
                            } else if constexpr (VB == 4) {
                                lo -= 1032.f * ps;                // even nibble: 1032 + code
                                hi = (hi - 1152.f * ps) * 0.0625f;  // odd nibble: 1152 + 16 code
                            } else {
                                lo -= BIAS_V * ps;
                                hi -= BIAS_V * ps;
                            }
                            *reinterpret_cast<float2 *>(oc + d) = make_float2(lo, hi);
                        }
                    }
                    if (gid == 0) *reinterpret_cast<float2 *>(oc + DH) = make_float2(mw[c], lt[c]);
                }
            }
            if (warp == 0 && lane == 0) {
                volatile int *seg = ctl + 4;
                seg[0] = m.bh; seg[1] = m.slot; seg[2] = m.ncta; seg[3] = m.cmin; seg[4] = 0;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&segbar[0]);
            nseg++;
        }
    }
    if (!aborted) {
        // tell the combiner there is no further segment
        if (nseg > 0 && !mbar_wait_bounded(&segbar[1], (nseg - 1) & 1u, abort_flag, limit)) {
            ctl[0] = 1;
            atomicExch(p.status, KVQ_ERR_TIMEOUT);
            return;
        }
        if (warp == 0 && lane == 0) ctl[8] = 1;
        __syncwarp();
        if (lane == 0) mbar_arrive(&segbar[0]);
    }
}

}  // namespace
}  // namespace kvq
