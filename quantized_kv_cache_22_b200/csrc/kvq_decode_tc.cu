// kvq_decode_tc.cu -- split-KV decode attention with both products on the
// 5th-generation tensor cores (tcgen05) in integer arithmetic, for INT8 /
// nibble-packed INT4 keys and values with fp16 value scales per (token, head),
// key scales per (token, head) or per 32/64-element group, or one scale per
// tensor; head_dim 128.
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
//   * q.K^T: tcgen05.mma kind::i8, M = 128 tokens, N = 16 (the int8 hi and lo
//     parts of each of the G <= 8 query heads, q ~ (max|q|/127)(hi + lo/254)),
//     K = head_dim, exact s32 accumulator in TMEM.  INT8 key codes are read by
//     the MMA straight from the TMA tile (K-major, 128-byte swizzle); INT4 codes
//     are first widened to int8 (16 x code).  Grouped key scales keep each
//     32-element block in its own TMEM columns.
//   * Softmax: each compute thread owns one token row of the score tile
//     (tcgen05.ld) and scales it by its key scale; the four compute warps agree
//     on a per-head reference m once per tile (raised lazily, only when a token's
//     p * s_V would exceed 2^8), so every P = 2^(s - m) * s_V lies in [0, 2^8].
//   * P.V: also kind::i8.  P becomes a 32-bit fixed-point number
//     x = rne(P * 2^24), whose four bytes are four unsigned 8-bit "digit"
//     columns of the B operand (one 16-byte row per token and 4 heads); A is
//     the value codes themselves -- INT8 codes straight from the TMA tile
//     (MN-major), INT4 codes widened to int8 (16 x code) -- so no value is
//     converted to floating point.  The s32 accumulators in TMEM, D_k =
//     sum_t digit_k(x_t) * code_t, are exact; sum_t P_t code_t =
//     2^-24 sum_k 256^k D_k.  The rounding of x is at most 2^-25 per token, so
//     a segment of n tokens is off by at most n 2^-25 max|V^| (about 1e-4 of
//     max|V^| at 3.5K tokens, far inside the 2e-3 bound).  An accumulation
//     "epoch" ends when the reference moves (or every 128 tiles, which keeps
//     the s32 sums in range) and at the segment end: the warps then read the
//     accumulator (each its TMEM lane quarter of head_dim), add it to fp32
//     registers and rescale those; the next epoch starts a fresh accumulator.
//   * Warps: 0 = TMA producer, 1 = TMEM allocator and MMA issuer (one thread),
//     2..5 = compute (TMEM lane quarter = warp % 4).  Every wait is bounded.
#include "kvq_decode_common.cuh"

namespace kvq {
namespace {

constexpr int TC_THREADS = 192;
constexpr float TC_LAZY = 8.f;
constexpr int TC_EPOCH_TILES = 128;   // tiles per accumulation epoch at most (s32 range)

// TMEM columns: S[2] (16 per 32-element key block with grouped key scales, else
// 16), then O[2] (4 digit columns per head: 4 NH).
template <bool KG, int NH>
struct TcCols {
    static constexpr uint32_t S = KG ? 64 : 16;
    static constexpr uint32_t O = 2 * S;
    static constexpr uint32_t ON = 4 * NH;                       // columns of one O buffer
    static constexpr uint32_t NEED = 2 * S + 2 * ON;
    static constexpr uint32_t ALLOC = NEED <= 64 ? 64 : (NEED <= 128 ? 128 : 256);
};

// Instruction descriptors.  q.K^T: D s32, A (keys) and B (queries) signed int8, both
// K-major, N = 16, M = 128.  P.V: D s32, A (value codes) signed int8 MN-major, B (P
// digits) unsigned int8 MN-major, N = 4 NH, M = 128.
constexpr uint32_t kIdescQK = (2u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) |
                              ((128u >> 4) << 24);
template <int NH>
constexpr uint32_t idesc_pv()
{
    return (2u << 4) | (1u << 7) | (0u << 10) | (1u << 15) | (1u << 16) |
           ((uint32_t)(4 * NH >> 3) << 17) | ((128u >> 4) << 24);
}

// Shared-memory regions after the stage ring (offsets in DecodeParams.tc).
constexpr uint32_t TC_X_BYTES = 128 * 128;         // a widened INT4 key or value tile
constexpr uint32_t TC_QB_BYTES = 16 * 128;         // int8 query rows of one segment
template <int NH>
constexpr uint32_t tc_pb_bytes() { return 4 * NH * 128; }   // P digits of one tile

// No-swizzle shared-memory matrix descriptor (8 rows of 16 bytes per core matrix):
// `lbo` between core matrices along K, `sbo` between 16-byte blocks along M/N.
__device__ __forceinline__ uint64_t interleave_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;                             // descriptor version (sm_100)
    return d;                                            // layout 0: no swizzle
}

__device__ __forceinline__ uint32_t f2u32_rne_sat(float x)
{
    uint32_t r;
    asm("cvt.rni.sat.u32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

struct TcBars {
    uint64_t kx[2], qrdy[2], sfull[2], sfree[2], pvr[2], pvd[2], xbar[2], ofree[2];
    uint64_t sred, sdone, drain;
};
struct TcAux {
    float qf[2][8];            // score factor per head, by segment parity
    float xch[2][4][8];        // per-warp proposals of the reference, by tile parity
    int xneed[2][4];           // whether warp w proposed (some token beat the reference)
    float red[2][4][8];        // per-warp sums of p, by segment parity
    int ep[2], fresh[2];       // epoch of a tile's P.V and whether it starts the epoch
    uint32_t tmem;             // TMEM base column
    int abort;
};
static_assert(sizeof(TcBars) <= kTcBarsBytes, "mbarriers fit their area");
static_assert(sizeof(TcAux) <= kTcAuxBytes, "control words fit their area");

// Position p of a widened INT4 row holds element e(p): within each group of 8,
// the low nibbles (even elements) come first, then the high nibbles.
__device__ __forceinline__ int k4_elem(int p)
{
    const int j = p & 7;
    return (p & ~7) + (j < 4 ? 2 * j : 2 * (j - 4) + 1);
}

// Widen one 64-byte row of nibble-packed INT4 codes (token t of a TMA tile at
// shared address `src`, two tokens per 128-byte line) to 128 int8 = 16 x code, in
// the 128-byte-swizzled row t of the tile at `dst`.
__device__ __forceinline__ void widen4_row(uint32_t src, uint32_t dst, int t)
{
    const uint32_t row = dst + (uint32_t)t * 128u;
    // all four loads first (the shared-memory accesses are volatile asm and keep
    // their program order), then the stores
    uint4 wv[4];
#pragma unroll
    for (int c = 0; c < 4; c++) wv[c] = lds_u128(src, sw_off<64>(t, 16 * c));
#pragma unroll
    for (int c = 0; c < 4; c++) {
        const uint32_t ww[4] = {wv[c].x, wv[c].y, wv[c].z, wv[c].w};
#pragma unroll
        for (int hp = 0; hp < 2; hp++) {
            const uint32_t a = ww[2 * hp], b = ww[2 * hp + 1];
            const uint32_t cc = (uint32_t)(2 * c + hp);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(
                             row + (((cc ^ (uint32_t)(t & 7)) & 7u) << 4)),
                         "r"((a << 4) & 0xF0F0F0F0u), "r"(a & 0xF0F0F0F0u),
                         "r"((b << 4) & 0xF0F0F0F0u), "r"(b & 0xF0F0F0F0u)
                         : "memory");
        }
    }
}

// KG: keys carry one scale per 32- or 64-element group.  NH: query heads per KV
// head handled (4 when G <= 4, else 8).
template <int KB, int VB, bool KG, int NH, int FMT>
__global__ void __launch_bounds__(TC_THREADS, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ DecodeParams p)
{
    constexpr int DH = 128;
    constexpr bool PT = FMT == KVQ_FMT_TENSOR;
    using Cols = TcCols<KG, NH>;
    constexpr uint32_t PB_BYTES = tc_pb_bytes<NH>();
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
        tmem_alloc(&aux->tmem, Cols::ALLOC);
        tmem_relinquish();
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
            int prev_s = 0;
            bool issued = false;
            for (int i = 0; i <= n_units; i++) {
                int cur_s = 0;
                if (i < n_units) {
                    // ---- q.K^T of tile i into S[i & 1]
                    const int j = i & 1;
                    const bool ok = KB == 4 ? mbar_wait_bounded(&bars->kx[0], i & 1, abort_flag, limit)
                                            : mbar_wait_bounded(&full[s], ph, abort_flag, limit);
                    if (!ok) { give_up(); break; }
                    cur_s = s;
                    if (meta[s].flags & 1) {
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
                    const uint32_t a0 = KB == 4 ? sbase + p.tc.off_kx : sbase + (uint32_t)s * p.stage_bytes;
                    const uint32_t b0 = sbase + p.tc.off_qb + (uint32_t)(kq & 1) * TC_QB_BYTES;
#pragma unroll
                    for (int kk = 0; kk < DH / 32; kk++)
                        umma_i8(tmem + Cols::S * (uint32_t)j + (KG ? 16u * kk : 0u),
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
                    // ---- P.V of tile i - 1 into O[epoch & 1]
                    const int i1 = i - 1, j = i1 & 1;
                    if (!mbar_wait_bounded(&bars->pvr[j], (i1 >> 1) & 1, abort_flag, limit)) {
                        give_up();
                        break;
                    }
                    const int ep = aux->ep[j];
                    const bool fresh = aux->fresh[j] != 0;
                    if (fresh && ep >= 2 &&
                        !mbar_wait_bounded(&bars->ofree[ep & 1], ((ep >> 1) - 1) & 1, abort_flag, limit)) {
                        give_up();
                        break;
                    }
                    tc_fence_after();
                    const uint32_t v0 = VB == 4 ? sbase + p.tc.off_vx + (uint32_t)j * TC_X_BYTES
                                                : sbase + (uint32_t)prev_s * p.stage_bytes + p.off_v;
                    const uint32_t p0 = sbase + p.tc.off_pb + (uint32_t)j * PB_BYTES;
                    const uint32_t d = tmem + Cols::O + Cols::ON * (uint32_t)(ep & 1);
#pragma unroll
                    for (int kk = 0; kk < 128 / 32; kk++)
                        umma_i8(d, sw128_mn_desc(v0 + 4096u * kk, 8192u, 1024u),
                                interleave_desc(p0 + 512u * kk, 128u, 2048u), idesc_pv<NH>(),
                                (fresh && kk == 0) ? 0u : 1u);
                    umma_commit(&bars->pvd[j]);
                    umma_commit(&empty[prev_s]);
                }
                if (i < n_units) prev_s = cur_s;
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
        // head-dim element and factor of row t of the P.V accumulator
        const int dlane = VB == 4 ? k4_elem(t) : t;
        constexpr double OFAC = (VB == 4 ? 1.0 / 16.0 : 1.0) / 16777216.0;   // 2^-24 (/16)

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
        int e = 0, ep_tiles = 0;                 // accumulation epoch and its tiles so far
        float m_ref[NH], l_acc[NH], qf[NH], o_acc[NH];
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
                    const int el = KB == 4 ? k4_elem(pos) : pos;
                    x[jj] = valid ? load_qf(p.q, p.q_dtype, qbase + el) : 0.f;
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
                // one widened-key buffer: q.K^T of tile i - 1 must have read it
                if (i >= 1 && !mbar_wait_bounded(&bars->sfull[(i - 1) & 1], ((i - 1) >> 1) & 1, abort_flag, limit))
                    return false;
                widen4_row(sbase + (uint32_t)s_prep * p.stage_bytes, sbase + p.tc.off_kx, t);
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->kx[0]);
            }
            if (++s_prep == S) {
                s_prep = 0;
                ph_prep ^= 1u;
            }
            return true;
        };

        // ---- end of an accumulation epoch: add the s32 digit sums of this lane's
        // head-dim row to the fp32 accumulators (the epoch's P.V must be complete)
        auto flush = [&]() {
            tc_fence_after();
            uint32_t dg[4 * NH];
            if constexpr (NH == 4) {
                tmem_ld16(tmem + Cols::O + Cols::ON * (uint32_t)(e & 1) + lane_off,
                          *reinterpret_cast<uint32_t(*)[16]>(dg));
            } else {
                tmem_ld32(tmem + Cols::O + Cols::ON * (uint32_t)(e & 1) + lane_off,
                          *reinterpret_cast<uint32_t(*)[32]>(dg));
            }
#pragma unroll
            for (int h = 0; h < NH; h++) {
                const double v = (((double)(int)dg[4 * h + 3] * 256.0 + (double)(int)dg[4 * h + 2]) * 256.0 +
                                  (double)(int)dg[4 * h + 1]) * 256.0 + (double)(int)dg[4 * h];
                o_acc[h] += (float)(v * OFAC);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->ofree[e & 1]);
            ++e;
            ep_tiles = 0;
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
                for (int h = 0; h < NH; h++) {
                    m_ref[h] = -INFINITY;
                    l_acc[h] = 0.f;
                    o_acc[h] = 0.f;
                    qf[h] = aux->qf[k & 1][h];
                }
            }
            const bool valid = m.t0 + t < m.len;

            // ---- P digits and widened values of tile i - 2 are consumed
            if (i >= 2 && !(ok = mbar_wait_bounded(&bars->pvd[j], ((i - 2) >> 1) & 1, abort_flag, limit)))
                break;
            if constexpr (VB == 4)
                widen4_row(sst + p.off_v, sbase + p.tc.off_vx + (uint32_t)j * TC_X_BYTES, t);

            // ---- scores of this thread's token: hi * 254 + lo of each head (per
            // 32-element key block when the key scales are grouped), times the key scale
            if (!(ok = mbar_wait_bounded(&bars->sfull[j], (i >> 1) & 1, abort_flag, limit))) break;
            tc_fence_after();
            float sc[NH];
#pragma unroll
            for (int h = 0; h < NH; h++) sc[h] = 0.f;
            const uint32_t sbuf = tmem + Cols::S * (uint32_t)j + lane_off;
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
                for (int h = 0; h < NH; h++) sc[h] = fmaf((float)((int)sr[h] * 254 + (int)sr[8 + h]), ks, sc[h]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sfree[j]);
            float sv = PT ? v_tensor : __half2float(__ushort_as_half((unsigned short)lds_u16(sst, p.off_sv + 2 * t)));
            sv = valid ? sv : 0.f;               // scales past the length may be stale
            const float lsv = sv > 0.f ? fmaxf(__log2f(sv), -32.f) : -32.f;
            bool need = false;
#pragma unroll
            for (int h = 0; h < NH; h++) {
                sc[h] = (valid && h < G) ? sc[h] * qf[h] : -INFINITY;
                need |= sc[h] + lsv > m_ref[h] + TC_LAZY;
            }

            // ---- the four warps agree on the reference of this tile
            const bool any_need = __any_sync(FULL, need);
            if (any_need) {
#pragma unroll
                for (int h = 0; h < NH; h++) {
                    float v = sc[h] + lsv;
#pragma unroll
                    for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, off));
                    if (lane == 0) aux->xch[j][cw][h] = v;
                }
            }
            if (lane == 0) aux->xneed[j][cw] = any_need;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->xbar[j]);
            if (!(ok = mbar_wait_bounded(&bars->xbar[j], (i >> 1) & 1, abort_flag, limit))) break;
            float alpha[NH];
            bool moved = false;
#pragma unroll
            for (int h = 0; h < NH; h++) alpha[h] = 1.f;
            const int4 nd = *reinterpret_cast<const int4 *>(aux->xneed[j]);
            if (nd.x | nd.y | nd.z | nd.w) {
                const int nw[4] = {nd.x, nd.y, nd.z, nd.w};
#pragma unroll
                for (int h = 0; h < NH; h++) {
                    float mx = m_ref[h];
#pragma unroll
                    for (int w = 0; w < 4; w++)
                        if (nw[w]) mx = fmaxf(mx, aux->xch[j][w][h]);
                    const bool up = mx > m_ref[h] && m_ref[h] != -INFINITY;
                    alpha[h] = up ? fast_exp2(m_ref[h] - mx) : 1.f;
                    moved |= up;
                    m_ref[h] = mx;
                }
            }

            // ---- a moved reference (or a full epoch) ends the epoch before this tile
            if ((moved || ep_tiles == TC_EPOCH_TILES) && ep_tiles > 0) {
                if (!(ok = mbar_wait_bounded(&bars->pvd[j ^ 1], ((i - 1) >> 1) & 1, abort_flag, limit))) break;
                flush();
            }
            if (moved) {
#pragma unroll
                for (int h = 0; h < NH; h++) {
                    o_acc[h] *= alpha[h];
                    l_acc[h] *= alpha[h];
                }
            }

            // ---- P of this token as 32-bit fixed point, one byte per digit column
            {
                uint32_t x[NH];
#pragma unroll
                for (int h = 0; h < NH; h++) {
                    const float pr = sc[h] == -INFINITY ? 0.f : fast_exp2(sc[h] - m_ref[h]);
                    l_acc[h] += pr;
                    x[h] = f2u32_rne_sat(pr * sv * 16777216.f);
                }
                const uint32_t pb = sbase + p.tc.off_pb + (uint32_t)j * PB_BYTES + (uint32_t)t * 16u;
#pragma unroll
                for (int b4 = 0; b4 < NH / 4; b4++)
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pb + 2048u * b4),
                                 "r"(x[4 * b4]), "r"(x[4 * b4 + 1]), "r"(x[4 * b4 + 2]), "r"(x[4 * b4 + 3])
                                 : "memory");
            }
            if (cw == 0 && lane == 0) {
                aux->ep[j] = e;
                aux->fresh[j] = ep_tiles == 0;
            }
            ++ep_tiles;
            fence_proxy_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->pvr[j]);

            // ---- segment end: partial (o, m, l) of this CTA into its workspace slot
            if (m.flags & 2) {
#pragma unroll
                for (int h = 0; h < NH; h++) {
#pragma unroll
                    for (int off = 16; off; off >>= 1) l_acc[h] += __shfl_xor_sync(FULL, l_acc[h], off);
                }
                if (lane == 0) {
#pragma unroll
                    for (int h = 0; h < NH; h++) aux->red[k & 1][cw][h] = l_acc[h];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->sred);
                if (!(ok = mbar_wait_bounded(&bars->pvd[j], (i >> 1) & 1, abort_flag, limit))) break;
                flush();
                if (!(ok = mbar_wait_bounded(&bars->sred, k & 1, abort_flag, limit))) break;
                float *dst = p.ws + (size_t)m.slot * G * CS;
#pragma unroll
                for (int h = 0; h < NH; h++) {
                    if (h >= G) break;
                    dst[(size_t)h * CS + dlane] = o_acc[h];
                }
                if (cw == 0 && lane < G) {
                    float mm = m_ref[0], ll = 0.f;
#pragma unroll
                    for (int h = 0; h < NH; h++)
                        if (lane == h) {
                            mm = m_ref[h];
                            ll = aux->red[k & 1][0][h] + aux->red[k & 1][1][h] + aux->red[k & 1][2][h] +
                                 aux->red[k & 1][3][h];
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
    if (warp == 1) tmem_dealloc(tmem, Cols::ALLOC);
}

template <int KB, int VB, bool KG, int NH, int FMT>
void *tc_fn()
{
    return reinterpret_cast<void *>(&decode_tc_kernel<KB, VB, KG, NH, FMT>);
}

template <bool KG, int NH>
void *tc_by_bits(int kb, int vb)
{
    if (kb == 8 && vb == 8) return tc_fn<8, 8, KG, NH, KVQ_FMT_INT>();
    if (kb == 8 && vb == 4) return tc_fn<8, 4, KG, NH, KVQ_FMT_INT>();
    if (kb == 4 && vb == 8) return tc_fn<4, 8, KG, NH, KVQ_FMT_INT>();
    if (kb == 4 && vb == 4) return tc_fn<4, 4, KG, NH, KVQ_FMT_INT>();
    return nullptr;
}

}  // namespace

void *decode_tc_fn(int kb, int vb, bool kg, int G, int fmt)
{
    const bool wide = G > 4;
    if (fmt == KVQ_FMT_TENSOR) {
        if (kb != 8 || vb != 8 || kg) return nullptr;
        return wide ? tc_fn<8, 8, false, 8, KVQ_FMT_TENSOR>() : tc_fn<8, 8, false, 4, KVQ_FMT_TENSOR>();
    }
    if (fmt != KVQ_FMT_INT) return nullptr;
    if (kg) return wide ? tc_by_bits<true, 8>(kb, vb) : tc_by_bits<true, 4>(kb, vb);
    return wide ? tc_by_bits<false, 8>(kb, vb) : tc_by_bits<false, 4>(kb, vb);
}

uint32_t decode_tc_pb_bytes(int G) { return G > 4 ? tc_pb_bytes<8>() : tc_pb_bytes<4>(); }

}  // namespace kvq
