// kvq_decode_tc.cu -- split-KV decode attention with both products on the
// 5th-generation tensor cores (tcgen05), for INT8 / nibble-packed INT4 keys and
// values with one fp16 scale per (token, head) or one per tensor, head_dim 128.
//
// What it computes is the same as the warp-MMA kernel (kvq_decode_kernel.cuh):
// for each sequence b and query head h of KV head j, softmax(tau q.K^T) V over
// the cached tokens, K and V dequantised from codes and scales (TinyLoop mode
// table; KVSplit 8K table), split over persistent CTAs and merged by
// log-sum-exp; optionally the newest token is quantised into the cache first.
//
// Design (sm_100a):
//   * Work split, TMA producer warp, fused append and the cross-CTA merge are
//     shared with the warp-MMA kernel (kvq_decode_common.cuh).
//   * q.K^T: one tcgen05.mma kind::i8 chain per 128-token tile, M = 128 tokens,
//     N = 16 (the int8 hi and lo parts of each of the G <= 8 query heads,
//     q ~ (max|q|/127)(hi + lo/254)), K = head_dim, s32 accumulator in TMEM.
//     INT8 key codes are read by the MMA straight from the TMA tile (K-major,
//     128-byte swizzle); INT4 codes are first widened to int8 (16 x code) by the
//     compute warps into a swizzled copy.
//   * Softmax: each compute thread owns one token row of the score tile
//     (tcgen05.ld), scales it by its key scale, and the four compute warps agree
//     on a per-head reference max through shared memory once per tile (raised
//     lazily, only when a token beats it by more than 2^8 in p * s_V).
//   * P.V: tcgen05.mma kind::f16, M = 128 (head_dim), N = 16 (heads), K = 16
//     tokens per instruction, fp32 accumulator O^T in TMEM for the whole
//     segment.  A = V^T: the compute warps turn the value codes into exact fp16
//     integers (exponent-bias trick, one LOP3 per pair of codes, then one f16x2
//     add or fma that removes the bias: the tensor core's accumulation keeps
//     about 15 bits relative to the accumulated value, so the bias must not reach
//     it) into an MN-major, 128-byte-swizzled tile; B = P, fp16 p * s_V written
//     by the token's thread.  When the reference max moves, O is rescaled in TMEM
//     by the warps (each its lane quarter) after the previous tile's MMAs complete.
//   * Warps: 0 = TMA producer, 1 = TMEM allocator and MMA issuer (one thread),
//     2..5 = compute (TMEM lane quarter = warp % 4).  Every wait is bounded.
#include "kvq_decode_common.cuh"

namespace kvq {
namespace {

constexpr int TC_THREADS = 192;
// TMEM: S[2] (16 columns per 32-element key block with grouped key scales, else 16),
// then O[2] (16 columns each)
template <bool KG>
struct TcCols {
    static constexpr uint32_t S = KG ? 64 : 16;      // columns of one score buffer
    static constexpr uint32_t O = 2 * S;             // first column of O[0]
    static constexpr uint32_t ALLOC = KG ? 256 : 64; // power of two >= 2 S + 32
};
constexpr float TC_LAZY = 8.f;
// half2 constants of the exact code conversion: -1152, -1032, 1/16, -72
constexpr uint32_t kNeg1152 = 0xE480E480u, kNeg1032 = 0xE408E408u;
constexpr uint32_t kSixteenth = 0x2C002C00u, kNeg72 = 0xD480D480u;

// Instruction descriptors.  q.K^T: D s32, A (keys) and B (queries) signed int8,
// both K-major, N = 16, M = 128.  P.V: D f32, A (values) and B (P) f16, A
// MN-major, B K-major, N = 16, M = 128.
constexpr uint32_t kIdescQK = (2u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) |
                              ((128u >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 15) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

// Shared-memory regions after the stage ring (offsets in DecodeParams.tc).
constexpr uint32_t TC_KX_BYTES = 128 * 128;        // widened INT4 keys of one tile
constexpr uint32_t TC_V16_BYTES = 128 * 128 * 2;   // fp16 values of one tile (2 panels)
constexpr uint32_t TC_PB_BYTES = 2 * 16 * 128;     // P of one tile (2 K-panels x 16 rows)
constexpr uint32_t TC_QB_BYTES = 16 * 128;         // int8 query rows of one segment

struct TcBars {
    uint64_t kx[2], qrdy[2], sfull[2], sfree[2], pvr[2], pvd[2], xbar[2], ofree[2];
    uint64_t sred, sdone, drain;
};
struct TcAux {
    float qf[2][8];            // score factor per head, by segment parity
    float xch[2][4][8];        // per-warp proposals of the reference max, by tile parity
    float red[2][4][8];        // per-warp sums of p, by segment parity
    uint32_t tmem;             // TMEM base column
    int abort;
};
static_assert(sizeof(TcBars) <= kTcBarsBytes, "mbarriers fit their area");
static_assert(sizeof(TcAux) <= kTcAuxBytes, "control words fit their area");

// Position p of a widened INT4 key row holds element e(p): within each group of 8,
// the low nibbles (even elements) come first, then the high nibbles.
__device__ __forceinline__ int k4_elem(int p)
{
    const int j = p & 7;
    return (p & ~7) + (j < 4 ? 2 * j : 2 * (j - 4) + 1);
}

// Head-dim element of row m of the fp16 value tile (and of the O^T accumulator).
// INT8 codes come out in pairs (0, 2), (1, 3) of each group of 4; INT4 codes as
// (0, 4), (1, 5), (2, 6), (3, 7) of each group of 8.
template <int VB>
__device__ __forceinline__ int v_elem(int m)
{
    if constexpr (VB == 8) {
        const int j = m & 3;
        return (m & ~3) + ((j & 1) << 1) + (j >> 1);
    } else {
        const int j = m & 7;
        return (m & ~7) + (j >> 1) + 4 * (j & 1);
    }
}

// KG: keys carry one scale per 32- or 64-element group (q.K^T then accumulates each
// 32-element block in its own TMEM columns and the scales apply per block).
template <int KB, int VB, bool KG, int FMT>
__global__ void __launch_bounds__(TC_THREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ DecodeParams p)
{
    constexpr int DH = 128;
    constexpr bool PT = FMT == KVQ_FMT_TENSOR;
    constexpr int RK = DH * KB / 8;
    constexpr int RV = DH * VB / 8;
    constexpr int CS = slot_col_floats(DH);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    StageMeta *meta = reinterpret_cast<StageMeta *>(smem + p.off_meta);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.off_bar);
    uint64_t *empty = full + p.stages;
    TcBars *bars = reinterpret_cast<TcBars *>(empty + p.stages);
    TcAux *aux = reinterpret_cast<TcAux *>(smem + p.tc.off_aux);
    volatile int *abort_flag = &aux->abort;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int S = p.stages;
    const int G = p.group_size_g;
    const int Hkv = p.n_kv_heads;
    const uint64_t limit = p.timeout_ns;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicExch(p.status, KVQ_ERR_TIMEOUT);
    };

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);           // tcgen05.commit after the tile's P.V
        }
        for (int j = 0; j < 2; j++) {
            mbar_init(&bars->kx[j], 4);
            mbar_init(&bars->qrdy[j], 4);
            mbar_init(&bars->sfull[j], 1);
            mbar_init(&bars->sfree[j], 4);
            mbar_init(&bars->pvr[j], 4);
            mbar_init(&bars->pvd[j], 1);
            mbar_init(&bars->xbar[j], 4);
            mbar_init(&bars->ofree[j], 4);
        }
        mbar_init(&bars->sred, 4);
        mbar_init(&bars->sdone, 4);
        mbar_init(&bars->drain, 1);
        aux->abort = 0;
        fence_mbar_init();
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(&aux->tmem, TcCols<KG>::ALLOC);
        tmem_relinquish();
    }
    if (warp >= 2) {
        // P rows of heads >= G are never written: zero both P buffers once
        const uint32_t pb = sbase + p.tc.off_pb;
        for (uint32_t o = (uint32_t)(tid - 64) * 16; o < 2 * TC_PB_BYTES; o += 128 * 16)
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(pb + o), "r"(0u) : "memory");
        fence_proxy_async_shared();
    }
    // global memory is touched from here on (programmatic dependent launch)
    grid_dependency_wait();
    grid_launch_dependents();

    __shared__ WorkRange wr;
    if (warp == 0) decode_work_range(p, lane, wr);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int n_units = wr.n_units;
    const uint32_t tmem = aux->tmem;

    if (warp == 0) {
        // ====================== producer ======================
        decode_producer<DH, KB, VB, FMT>(p, &tm_k, &tm_v, smem, full, empty, meta, abort_flag, wr,
                                         lane);
    } else if (warp == 1) {
        // ====================== MMA issuer ======================
        if (lane == 0 && n_units > 0) {
            int s = 0;
            uint32_t ph = 0;
            int kq = -1;                 // segment of the tile whose q.K^T was issued last
            int prev_s = 0, prev_flags = 0, prev_k = 0;
            bool issued = false;
            for (int i = 0; i <= n_units; i++) {
                int cur_s = 0, cur_flags = 0;
                if (i < n_units) {
                    // ---- q.K^T of tile i into S[i & 1]
                    const int j = i & 1;
                    const bool ok = KB == 4 ? mbar_wait_bounded(&bars->kx[j], (i >> 1) & 1, abort_flag, limit)
                                            : mbar_wait_bounded(&full[s], ph, abort_flag, limit);
                    if (!ok) { give_up(); break; }
                    cur_flags = meta[s].flags;
                    cur_s = s;
                    if (cur_flags & 1) {
                        ++kq;
                        if (!mbar_wait_bounded(&bars->qrdy[kq & 1], (kq >> 1) & 1, abort_flag, limit)) {
                            give_up();
                            break;
                        }
                    }
                    if (i >= 2 && !mbar_wait_bounded(&bars->sfree[j], ((i - 2) >> 1) & 1, abort_flag, limit)) {
                        give_up();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = KB == 4 ? sbase + p.tc.off_kx + (uint32_t)j * TC_KX_BYTES
                                                : sbase + (uint32_t)s * p.stage_bytes;
                    const uint32_t b0 = sbase + p.tc.off_qb + (uint32_t)(kq & 1) * TC_QB_BYTES;
#pragma unroll
                    for (int kk = 0; kk < DH / 32; kk++)
                        umma_i8(tmem + TcCols<KG>::S * (uint32_t)j + (KG ? 16u * kk : 0u),
                                sw128_desc(a0 + 32u * kk), sw128_desc(b0 + 32u * kk), kIdescQK,
                                (!KG && kk > 0) ? 1u : 0u);
                    umma_commit(&bars->sfull[j]);
                    issued = true;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (i >= 1) {
                    // ---- P.V of tile i - 1 into O[segment & 1]
                    const int i1 = i - 1, j = i1 & 1;
                    if (!mbar_wait_bounded(&bars->pvr[j], (i1 >> 1) & 1, abort_flag, limit)) {
                        give_up();
                        break;
                    }
                    const bool first = prev_flags & 1;
                    if (first && prev_k >= 2 &&
                        !mbar_wait_bounded(&bars->ofree[prev_k & 1], ((prev_k >> 1) - 1) & 1, abort_flag, limit)) {
                        give_up();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t v0 = sbase + p.tc.off_v16 + (uint32_t)j * TC_V16_BYTES;
                    const uint32_t p0 = sbase + p.tc.off_pb + (uint32_t)j * TC_PB_BYTES;
                    const uint32_t d = tmem + TcCols<KG>::O + 16u * (uint32_t)(prev_k & 1);
#pragma unroll
                    for (int kk = 0; kk < 128 / 16; kk++)
                        umma_f16(d, sw128_mn_desc(v0 + 2048u * kk, 128u * 128u, 1024u),
                                 sw128_desc(p0 + 2048u * (kk >> 2) + 32u * (kk & 3)), kIdescPV,
                                 (first && kk == 0) ? 0u : 1u);
                    umma_commit(&bars->pvd[j]);
                    umma_commit(&empty[prev_s]);
                }
                if (i < n_units) {
                    prev_s = cur_s;
                    prev_flags = cur_flags;
                    prev_k = kq;
                }
            }
            if (issued) {
                // every MMA issued must complete before the CTA frees TMEM and exits
                umma_commit(&bars->drain);
                (void)mbar_wait_drain(&bars->drain, 0, limit);
            }
        }
    } else {
        // ====================== compute warps ======================
        const int q4 = warp & 3;                 // TMEM lane quarter
        const int t = 32 * q4 + lane;            // token row of the tile, and d-row of O^T
        const int ctid = tid - 64;               // 0..127
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const int cw = warp - 2;
        const float k_tensor = PT ? __half2float(p.k_scales[0]) : 0.f;
        const float v_tensor = PT ? __half2float(p.v_scales[0]) : 0.f;

        // sequences with nothing cached get zeros (fused merge only)
        if (p.counters != nullptr) {
            const int64_t n_out = (int64_t)p.n_q_heads * DH;
            for (int b = blockIdx.x; b < p.batch; b += gridDim.x) {
                if (tiles_of(p.d_len[b], p.cap) != 0) continue;
                for (int64_t i = ctid; i < n_out; i += 128) {
                    if (p.out_f32)
                        static_cast<float *>(p.out)[(int64_t)b * n_out + i] = 0.f;
                    else
                        static_cast<__half *>(p.out)[(int64_t)b * n_out + i] = __float2half_rn(0.f);
                }
            }
        }

        int s_prep = 0, s_proc = 0;
        uint32_t ph_prep = 0;
        int k_prep = -1, k = -1;                 // segment counters (prep runs one tile ahead)
        float m_ref[8], l_acc[8], qf[8];
        bool ok = true;

        // ---- prep(i): the tile's data has landed; a segment start writes the int8
        // query rows; INT4 keys are widened to int8 for the MMA
        auto prep = [&](int i) -> bool {
            if (!mbar_wait_bounded(&full[s_prep], ph_prep, abort_flag, limit)) return false;
            const StageMeta m = meta[s_prep];
            if (m.flags & 1) {
                ++k_prep;
                const int b = m.bh / Hkv, kvh = m.bh % Hkv;
                const int h = ctid >> 4, pc = ctid & 15;   // head, 8 positions 8pc .. 8pc+7
                const bool valid = h < G;
                const int64_t qbase = ((int64_t)b * p.n_q_heads + (int64_t)kvh * G + (valid ? h : 0)) * DH;
                float x[8];
                float amax = 0.f;
#pragma unroll
                for (int jj = 0; jj < 8; jj++) {
                    const int pos = 8 * pc + jj;
                    const int e = KB == 4 ? k4_elem(pos) : pos;
                    x[jj] = valid ? load_qf(p.q, p.q_dtype, qbase + e) : 0.f;
                    amax = fmaxf(amax, fabsf(x[jj]));
                }
#pragma unroll
                for (int off = 1; off < 16; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, off));
                const float inv = amax > 0.f ? 127.f / amax : 0.f;
                uint32_t hw[2] = {0u, 0u}, lw[2] = {0u, 0u};
#pragma unroll
                for (int jj = 0; jj < 8; jj++) {
                    const float y = x[jj] * inv;
                    const float r = rintf(y);
                    const int hi = (int)r;
                    const int lo = __float2int_rn((y - r) * 254.f);
                    hw[jj >> 2] |= (uint32_t)(hi & 0xff) << (8 * (jj & 3));
                    lw[jj >> 2] |= (uint32_t)(lo & 0xff) << (8 * (jj & 3));
                }
                const uint32_t qb = sbase + p.tc.off_qb + (uint32_t)(k_prep & 1) * TC_QB_BYTES;
                // rows h (hi) and 8 + h (lo): 16-byte chunk pc / 2, swizzled by row % 8
                const uint32_t col = (uint32_t)((((pc >> 1) ^ (h & 7)) << 4) + ((pc & 1) << 3));
                asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(qb + (uint32_t)h * 128u + col),
                             "r"(hw[0]), "r"(hw[1]) : "memory");
                asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(qb + (uint32_t)(8 + h) * 128u + col),
                             "r"(lw[0]), "r"(lw[1]) : "memory");
                if (pc == 0)
                    aux->qf[k_prep & 1][h] = amax * (1.f / (127.f * 254.f)) * p.tau_log2e *
                                             (KB == 4 ? 0.0625f : 1.f);
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->qrdy[k_prep & 1]);
            }
            if constexpr (KB == 4) {
                // widen this thread's key row: 64 bytes of nibbles -> 128 int8 (16 x code)
                const uint32_t src = sbase + (uint32_t)s_prep * p.stage_bytes;
                const uint32_t dst = sbase + p.tc.off_kx + (uint32_t)(i & 1) * TC_KX_BYTES + (uint32_t)t * 128u;
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    const uint4 w = lds_u128(src, sw_off<RK>(t, 16 * c));
                    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int hp = 0; hp < 2; hp++) {
                        const uint32_t a = ww[2 * hp], bb = ww[2 * hp + 1];
                        const uint32_t cc = (uint32_t)(2 * c + hp);        // output chunk
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                                         dst + (((cc ^ (uint32_t)(t & 7)) & 7u) << 4)),
                                     "r"((a << 4) & 0xF0F0F0F0u), "r"(a & 0xF0F0F0F0u),
                                     "r"((bb << 4) & 0xF0F0F0F0u), "r"(bb & 0xF0F0F0F0u)
                                     : "memory");
                    }
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->kx[i & 1]);
            }
            if (++s_prep == S) {
                s_prep = 0;
                ph_prep ^= 1u;
            }
            return true;
        };

        if (n_units > 0) ok = prep(0);
        for (int i = 0; i < n_units && ok; i++) {
            if (i + 1 < n_units && !(ok = prep(i + 1))) break;
            const int j = i & 1;
            const StageMeta m = meta[s_proc];
            const uint32_t sst = sbase + (uint32_t)s_proc * p.stage_bytes;
            const bool first = m.flags & 1;
            if (first) {
                ++k;
                if (!(ok = mbar_wait_bounded(&bars->qrdy[k & 1], (k >> 1) & 1, abort_flag, limit))) break;
#pragma unroll
                for (int h = 0; h < 8; h++) {
                    m_ref[h] = -INFINITY;
                    l_acc[h] = 0.f;
                    qf[h] = aux->qf[k & 1][h];
                }
            }
            const bool valid = m.t0 + t < m.len;

            // ---- the fp16 value tile (A of P.V): buffers of tile i - 2 must be free
            if (i >= 2 && !(ok = mbar_wait_bounded(&bars->pvd[j], ((i - 2) >> 1) & 1, abort_flag, limit)))
                break;
            {
                const uint32_t v16 = sbase + p.tc.off_v16 + (uint32_t)j * TC_V16_BYTES + (uint32_t)t * 128u;
                const uint32_t sw = (uint32_t)(t & 7);
                if constexpr (VB == 8) {
#pragma unroll
                    for (int c = 0; c < 8; c++) {
                        const uint4 w = lds_u128(sst + p.off_v, sw_off<RV>(t, 16 * c));
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                        uint32_t o[8];
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            // bytes 0, 2 and 1, 3 as fp16 1152 + code, then the code exactly
                            o[2 * e] = hadd2_u32(and_xor(ww[e], 0x00FF00FFu, 0x64806480u), kNeg1152);
                            o[2 * e + 1] = hadd2_u32(and_xor(ww[e] >> 8, 0x00FF00FFu, 0x64806480u), kNeg1152);
                        }
                        // d 16c .. 16c+15 -> panel c / 4, chunks (2c) % 8 and (2c + 1) % 8
                        const uint32_t pan = v16 + (uint32_t)(c >> 2) * (128u * 128u);
                        const uint32_t c0 = (uint32_t)((2 * c) & 7), c1 = (uint32_t)((2 * c + 1) & 7);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pan + ((c0 ^ sw) << 4)),
                                     "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3]) : "memory");
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pan + ((c1 ^ sw) << 4)),
                                     "r"(o[4]), "r"(o[5]), "r"(o[6]), "r"(o[7]) : "memory");
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 4; c++) {
                        const uint4 w = lds_u128(sst + p.off_v, sw_off<RV>(t, 16 * c));
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; e++) {
                            // d 32c + 8e .. +7 -> chunk k = 4c + e (panel k / 8)
                            const uint32_t x0 = ww[e], x1 = ww[e] >> 8;
                            const int kc = 4 * c + e;
                            const uint32_t addr = v16 + (uint32_t)(kc >> 3) * (128u * 128u) +
                                                  ((((uint32_t)kc & 7u) ^ sw) << 4);
                            // low nibbles as fp16 1032 + code, high nibbles as 1152 + 16 code,
                            // then the codes exactly (x - 1032; x / 16 - 72)
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                                         "r"(hadd2_u32(and_xor(x0, 0x000F000Fu, 0x64086408u), kNeg1032)),
                                         "r"(hfma2_u32(and_xor(x0, 0x00F000F0u, 0x64806480u), kSixteenth, kNeg72)),
                                         "r"(hadd2_u32(and_xor(x1, 0x000F000Fu, 0x64086408u), kNeg1032)),
                                         "r"(hfma2_u32(and_xor(x1, 0x00F000F0u, 0x64806480u), kSixteenth, kNeg72))
                                         : "memory");
                        }
                    }
                }
            }

            // ---- scores of this thread's token
            if (!(ok = mbar_wait_bounded(&bars->sfull[j], (i >> 1) & 1, abort_flag, limit))) break;
            tc_fence_after();
            // integer scores hi * 254 + lo of each head, per 32-element key block when
            // the key scales are grouped, times the key scale
            float sc[8];
#pragma unroll
            for (int h = 0; h < 8; h++) sc[h] = 0.f;
            const uint32_t sbuf = tmem + TcCols<KG>::S * (uint32_t)j + lane_off;
#pragma unroll
            for (int blk = 0; blk < (KG ? DH / 32 : 1); blk++) {
                uint32_t sr[16];
                tmem_ld16(sbuf + 16u * (uint32_t)blk, sr);
                float ks;
                if constexpr (PT)
                    ks = k_tensor;
                else
                    ks = __half2float(__ushort_as_half((unsigned short)lds_u16(
                        sst, p.off_sk + 2 * (t * p.ngs_k + (KG ? (blk >> p.kshift) : 0)))));
#pragma unroll
                for (int h = 0; h < 8; h++) sc[h] = fmaf((float)((int)sr[h] * 254 + (int)sr[8 + h]), ks, sc[h]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sfree[j]);
            float sv = PT ? v_tensor : __half2float(__ushort_as_half((unsigned short)lds_u16(sst, p.off_sv + 2 * t)));
            sv = valid ? sv : 0.f;               // scales past the length may be stale
            const float lsv = sv > 0.f ? fmaxf(__log2f(sv), -32.f) : -32.f;
            bool need = false;
#pragma unroll
            for (int h = 0; h < 8; h++) {
                sc[h] = (valid && h < G) ? sc[h] * qf[h] : -INFINITY;
                need |= sc[h] + lsv > m_ref[h] + TC_LAZY;
            }

            // ---- the four warps agree on the reference max of this tile
            float prop[8];
#pragma unroll
            for (int h = 0; h < 8; h++) prop[h] = -INFINITY;
            if (__any_sync(FULL, need)) {
#pragma unroll
                for (int h = 0; h < 8; h++) {
                    float v = sc[h] + lsv;
#pragma unroll
                    for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, off));
                    prop[h] = v;
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int h = 0; h < 8; h++) aux->xch[j][cw][h] = prop[h];
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->xbar[j]);
            if (!(ok = mbar_wait_bounded(&bars->xbar[j], (i >> 1) & 1, abort_flag, limit))) break;
            float alpha[8];
            bool moved = false;
#pragma unroll
            for (int h = 0; h < 8; h++) {
                float mx = m_ref[h];
#pragma unroll
                for (int w = 0; w < 4; w++) mx = fmaxf(mx, aux->xch[j][w][h]);
                alpha[h] = (mx > m_ref[h] && m_ref[h] != -INFINITY) ? fast_exp2(m_ref[h] - mx) : 1.f;
                moved |= mx > m_ref[h] && m_ref[h] != -INFINITY;
                m_ref[h] = mx;
            }

            // ---- P (fp16 p * s_V) of this token for each head, the sums of p and P
            {
                const uint32_t pb = sbase + p.tc.off_pb + (uint32_t)j * TC_PB_BYTES +
                                    (uint32_t)(t >> 6) * 2048u;
                const uint32_t cc = (uint32_t)((t & 63) >> 3), byte = (uint32_t)(t & 7) * 2u;
#pragma unroll
                for (int h = 0; h < 8; h++) {
                    if (h >= G) break;
                    l_acc[h] *= alpha[h];
                    const float pr = sc[h] == -INFINITY ? 0.f : fast_exp2(sc[h] - m_ref[h]);
                    const __half ph16 = __float2half_rn(pr * sv);
                    l_acc[h] += pr;
                    const uint32_t addr = pb + (uint32_t)h * 128u + (((cc ^ (uint32_t)(h & 7)) & 7u) << 4) + byte;
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(__half_as_ushort(ph16)) : "memory");
                }
            }

            // ---- a moved reference rescales the accumulated O^T (its lane quarter)
            if (moved && !first) {
                if (!(ok = mbar_wait_bounded(&bars->pvd[j ^ 1], ((i - 1) >> 1) & 1, abort_flag, limit))) break;
                tc_fence_after();
                const uint32_t oaddr = tmem + TcCols<KG>::O + 16u * (uint32_t)(k & 1) + lane_off;
                uint32_t o[16];
                tmem_ld16(oaddr, o);
#pragma unroll
                for (int h = 0; h < 8; h++) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                tmem_st16(oaddr, o);
            }
            fence_proxy_async_shared();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->pvr[j]);

            // ---- segment end: partial (o, m, l) of this CTA into its workspace slot
            if (m.flags & 2) {
#pragma unroll
                for (int h = 0; h < 8; h++) {
#pragma unroll
                    for (int off = 16; off; off >>= 1) {
                        l_acc[h] += __shfl_xor_sync(FULL, l_acc[h], off);
                    }
                }
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < 8; h++) {
                        aux->red[k & 1][cw][h] = l_acc[h];
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->sred);
                if (!(ok = mbar_wait_bounded(&bars->sred, k & 1, abort_flag, limit))) break;
                float L[8];
#pragma unroll
                for (int h = 0; h < 8; h++) {
                    L[h] = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; w++) {
                        L[h] += aux->red[k & 1][w][h];
                    }
                }
                if (!(ok = mbar_wait_bounded(&bars->pvd[j], (i >> 1) & 1, abort_flag, limit))) break;
                tc_fence_after();
                uint32_t o[16];
                tmem_ld16(tmem + TcCols<KG>::O + 16u * (uint32_t)(k & 1) + lane_off, o);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->ofree[k & 1]);
                // row t of O^T is head-dim element v_elem(t)
                const int dlane = v_elem<VB>(t);
                float *dst = p.ws + (size_t)m.slot * G * CS;
#pragma unroll
                for (int h = 0; h < 8; h++) {
                    if (h >= G) break;
                    dst[(size_t)h * CS + dlane] = __uint_as_float(o[h]);
                }
                if (cw == 0 && lane < G) {
                    float mm = m_ref[0], ll = L[0];
#pragma unroll
                    for (int h = 1; h < 8; h++)
                        if (lane == h) {
                            mm = m_ref[h];
                            ll = L[h];
                        }
                    *reinterpret_cast<float2 *>(dst + (size_t)lane * CS + DH) = make_float2(mm, ll);
                }
                __syncwarp();
                if (lane == 0) {
                    fence_acq_rel_gpu();
                    mbar_arrive(&bars->sdone);
                }
                if (cw == 0) {
                    // all four warps wrote their part: publish, and merge when this
                    // CTA's partial is the last one of its (sequence, KV head)
                    if (!(ok = mbar_wait_bounded(&bars->sdone, k & 1, abort_flag, limit))) break;
                    if (p.counters != nullptr) {
                        int last = 0;
                        if (lane == 0) {
                            fence_acq_rel_gpu();
                            last = atomicAdd(&p.counters[m.bh], 1) == m.ncta - 1;
                            if (last) fence_acq_rel_gpu();
                        }
                        last = __shfl_sync(FULL, last, 0);
                        __syncwarp();
                        if (last) {
                            const int b = m.bh / Hkv, kvh = m.bh % Hkv;
                            merge_segment<DH>(p.ws, (int64_t)m.cmin + m.bh, m.ncta, G, p.out, p.out_f32,
                                              ((int64_t)b * p.n_q_heads + (int64_t)kvh * G) * DH, lane);
                            if (lane == 0) p.counters[m.bh] = 0;   // ready for the next launch
                        }
                    }
                }
            }
            if (++s_proc == S) s_proc = 0;
        }
        if (!ok) give_up();
    }

    // every role reaches this point; TMEM is freed after all tcgen05 work is done
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TcCols<KG>::ALLOC);
}

template <int KB, int VB, bool KG, int FMT>
void *tc_fn()
{
    return reinterpret_cast<void *>(&decode_tc_kernel<KB, VB, KG, FMT>);
}

template <bool KG>
void *tc_by_bits(int kb, int vb)
{
    if (kb == 8 && vb == 8) return tc_fn<8, 8, KG, KVQ_FMT_INT>();
    if (kb == 8 && vb == 4) return tc_fn<8, 4, KG, KVQ_FMT_INT>();
    if (kb == 4 && vb == 8) return tc_fn<4, 8, KG, KVQ_FMT_INT>();
    if (kb == 4 && vb == 4) return tc_fn<4, 4, KG, KVQ_FMT_INT>();
    return nullptr;
}

}  // namespace

void *decode_tc_fn(int kb, int vb, bool kg, int fmt)
{
    if (fmt == KVQ_FMT_TENSOR)
        return (kb == 8 && vb == 8 && !kg) ? tc_fn<8, 8, false, KVQ_FMT_TENSOR>() : nullptr;
    if (fmt != KVQ_FMT_INT) return nullptr;
    return kg ? tc_by_bits<true>(kb, vb) : tc_by_bits<false>(kb, vb);
}

}  // namespace kvq
