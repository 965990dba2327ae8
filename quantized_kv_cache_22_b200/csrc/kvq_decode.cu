// kvq_decode.cu -- host side of the decode attention: shared-memory plan,
// kernel selection, launches, and the merge kernel for partials left by a
// decode launch without arrival counters.
#include <cstdlib>
#include <mutex>
#include <vector>

#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace {

// ---------------------------------------------------------------------------
// merge launch (partials left by a decode launch without counters): one warp
// per (sequence, KV head)
// ---------------------------------------------------------------------------
template <int DH>
__global__ void __launch_bounds__(256) merge_kernel(const MergeParams p)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (gw >= (int64_t)p.batch * p.n_kv_heads) return;
    const int b = (int)(gw / p.n_kv_heads);
    const int kvh = (int)(gw % p.n_kv_heads);
    const int G = p.group_size_g;
    const int cap = p.cap;
    const int64_t obase0 = ((int64_t)b * p.n_q_heads + (int64_t)kvh * G) * DH;

    // units before sequence b, and in total
    long long before = 0, total = 0;
    for (int bb = lane; bb < p.batch; bb += 32) {
        const long long t = tiles_of(p.d_len[bb], cap);
        total += t;
        if (bb < b) before += t;
    }
    for (int off = 16; off; off >>= 1) {
        total += __shfl_xor_sync(FULL, total, off);
        before += __shfl_xor_sync(FULL, before, off);
    }
    const int tiles_b = tiles_of(p.d_len[b], cap);
    if (tiles_b == 0) {
        for (int i = lane; i < G * DH; i += 32) {
            if (p.out_f32)
                static_cast<float *>(p.out)[obase0 + i] = 0.f;
            else
                static_cast<__half *>(p.out)[obase0 + i] = __float2half_rn(0.f);
        }
        return;
    }
    const long long N = total * p.n_kv_heads;
    const long long Pe = N < (long long)p.num_ctas ? N : (long long)p.num_ctas;
    const long long u0 = before * p.n_kv_heads + (long long)kvh * tiles_b;
    const long long u1 = u0 + tiles_b;
    const long long cmin = range_cta(u0, N, Pe);
    const long long cmax = range_cta(u1 - 1, N, Pe);
    const int bh = b * p.n_kv_heads + kvh;
    merge_segment<DH>(p.ws, cmin + bh, (int)(cmax - cmin + 1), G, p.out, p.out_f32, obase0, lane);
}

void *pick_decode(int dh, int kb, int vb, bool kg, bool vg, int fmt)
{
    if (kb == 16) kg = false;
    if (vb == 16) vg = false;
    if (fmt != KVQ_FMT_INT) return (kb == 8 && vb == 8) ? decode_fn_fmt(dh, fmt, kg, vg) : nullptr;
    switch (kb) {
    case 4: return decode_fn_kb4(dh, vb, kg, vg);
    case 8: return decode_fn_kb8(dh, vb, kg, vg);
    case 16: return decode_fn_kb16(dh, vb, kg, vg);
    default: return nullptr;
    }
}

// the packed-column instance for G <= 4, or null
void *pick_decode_pk(int dh, int kb, int vb, bool kg, bool vg, int fmt, int G)
{
    if (dh != 128 || G > 4) return nullptr;
    if (kb == 4) return decode_fn_pk_kb4(vb, kg, vg, fmt);
    if (kb == 8) return decode_fn_pk_kb8(vb, kg, vg, fmt);
    return nullptr;
}

inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// The warp-MMA kernel serves every format by default: on the 8K workload it is as
// fast as the tensor-core kernel for INT8 keys and values and faster for INT4
// ones.  KVQ_DECODE_TC=1 in the environment (read at each call) selects the
// tensor-core kernel for the formats it supports; its integer P.V is exact up to
// the 2^-25 rounding of P per token.
static bool tc_selected()
{
    const char *e = std::getenv("KVQ_DECODE_TC");
    return e && e[0] == '1' && e[1] == '\0';
}

}  // namespace

// The tensor-core kernel takes INT8 / INT4 codes with per-(token, head) value scales,
// key scales per (token, head) or per 32/64-element group (or per-tensor INT8),
// head_dim 128 and up to 8 query heads per KV head.  Two CTAs per SM when a ring of
// at least 3 stages fits next to the widened-code, P-digit and query tiles of each,
// else one CTA per SM with as many stages as fit (2 stages per CTA measured slower).
static bool plan_decode_tc(int dh, int kb, int vb, bool kg, bool vg, int ngs_k, int G,
                           int max_smem, DecodeLaunch *plan, int fmt)
{
    if (dh != 128 || vg || G > 8 || !decode_tc_fn(kb, vb, kg, G, fmt)) return false;
    DecodeLaunch L{};
    L.dh = dh; L.kb = kb; L.vb = vb; L.kg = kg; L.vg = false; L.fmt = fmt; L.tc = true; L.G = G;
    const bool pt = fmt == KVQ_FMT_TENSOR;
    const uint32_t rk = dh * kb / 8, rv = dh * vb / 8;
    L.off_v = align_up(T * rk, 1024);
    L.off_sk = L.off_v + align_up(T * rv, 1024);
    L.off_sv = L.off_sk + align_up(T * (pt ? 0 : ngs_k) * 2, 16);
    L.stage_bytes = align_up(L.off_sv + T * (pt ? 0 : 1) * 2, 1024);
    const uint32_t pb = decode_tc_pb_bytes(G);
    for (int per_sm = 2; per_sm >= 1; per_sm--) {
        const uint32_t budget = per_sm == 2 ? 233472u / 2 - 1024u - 128u : (uint32_t)max_smem;
        for (int S = 8; S >= (per_sm == 2 ? 3 : 2); S--) {
            TcOffsets o{};
            uint32_t off = S * L.stage_bytes;
            o.off_kx = off;
            off += kb == 4 ? 128u * 128u : 0u;
            o.off_vx = off;
            off += vb == 4 ? 2u * 128u * 128u : 0u;
            o.off_pb = off;
            off += 2u * pb;
            o.off_qb = off;
            off += 2u * 16u * 128u;
            const uint32_t off_meta = off;
            const uint32_t off_bar = align_up(off_meta + S * (uint32_t)sizeof(StageMeta), 16);
            o.off_aux = align_up(off_bar + 2u * S * 8u + kTcBarsBytes, 16);
            const uint32_t total = o.off_aux + kTcAuxBytes + 1024;   // + alignment slack
            if (total <= budget && total <= (uint32_t)max_smem) {
                L.stages = S;
                L.per_sm = per_sm;
                L.off_meta = off_meta;
                L.off_bar = off_bar;
                L.off_merge = 0;
                L.tco = o;
                L.smem_bytes = total;
                *plan = L;
                return true;
            }
        }
    }
    return false;
}

bool plan_decode(int dh, int kb, int vb, int ngs_k, int ngs_v, int G, int max_smem,
                 DecodeLaunch *plan, int fmt)
{
    // ngs_k / ngs_v: fp16 values per row in the scale arrays (a pair per group with
    // a zero-point; none for 16-bit or per-tensor codes)
    const int sv = scale_vals(fmt);
    const bool kg = kb != 16 && ngs_k / sv > 1, vg = vb != 16 && ngs_v / sv > 1;
    if (tc_selected() && plan_decode_tc(dh, kb, vb, kg, vg, ngs_k, G, max_smem, plan, fmt)) return true;
    if (!pick_decode(dh, kb, vb, kg, vg, fmt)) return false;
    const uint32_t rk = dh * kb / 8, rv = dh * vb / 8;
    DecodeLaunch L{};
    L.dh = dh; L.kb = kb; L.vb = vb; L.kg = kg; L.vg = vg; L.fmt = fmt; L.G = G;
    L.pk = pick_decode_pk(dh, kb, vb, kg, vg, fmt, G) != nullptr;
    L.off_v = align_up(T * rk, 1024);
    L.off_sk = L.off_v + align_up(T * rv, 1024);
    L.off_sv = L.off_sk + align_up(T * (kb == 16 ? 0 : ngs_k) * 2, 16);
    L.stage_bytes = align_up(L.off_sv + T * (vb == 16 ? 0 : ngs_v) * 2, 1024);
    const uint32_t merge_bytes = (uint32_t)NW * G * slot_col_floats(dh) * 4;
    // tail: meta[S] (32 B each), barriers (2S + 2) * 8 B, control words 64 B, merge buffer;
    // as many stages as fit next to the other CTAs of an SM (228 KB of shared memory,
    // 1 KB of it reserved per CTA, 1 KB for the kernel's static shared memory),
    // else two stages in one CTA per SM (16-bit K and V at 128-element heads, 64 KB a
    // stage: a third stage measured slower, 29.6-30.3 against 28.5 us for 8 x 1024 tokens
    // of 16 heads)
    // (with one CTA per SM the dynamic part may use the opt-in maximum less the kernel's
    // static shared memory, about 1 KB)
    max_smem -= 2048;
    // beside another CTA: 228 KB per SM, of which 1 KB is reserved per CTA and 1 KB is
    // the kernel's static part (the dynamic part starts 1024-byte aligned)
    const uint32_t per_cta = 233472u / (uint32_t)kDecodeCtasPerSm - 1024u - 1024u;
    // packed-column int8 keys without zero-points: the consumer warps may quantise a
    // segment's query rows one head each and share them (hi and lo bytes, [4][Dh]
    // each, then 4 factors and 2 mbarriers), where that costs neither a stage nor a
    // CTA: after the merge buffer, or else in the unused tails of the first three
    // stages (no copy writes past a stage's scales)
    const bool qshare = L.pk && kb != 16 && fmt != KVQ_FMT_E4M3 && fmt != KVQ_FMT_ASYM;
    const uint32_t qs_bytes = 8u * dh + 16u + 16u;
    const uint32_t used = align_up(L.off_sv + T * (vb == 16 ? 0 : ngs_v) * 2, 16);
    const uint32_t tail = L.stage_bytes - used;
    for (int S = 8; S >= 2; S--) {
        const uint32_t off_meta = S * L.stage_bytes;
        const uint32_t off_bar = off_meta + S * (uint32_t)sizeof(StageMeta);
        const uint32_t off_merge = align_up(off_bar + (2 * S + 2) * 8 + 64, 16);
        const uint32_t total = off_merge + merge_bytes + 1024;  // + alignment slack
        if ((total <= per_cta && total <= (uint32_t)max_smem) || (S == 2 && total <= (uint32_t)max_smem)) {
            L.stages = S;
            L.per_sm = total <= per_cta ? kDecodeCtasPerSm : 1;
            L.off_meta = off_meta;
            L.off_bar = off_bar;
            L.off_merge = off_merge;
            L.smem_bytes = total;
            const uint32_t off_qs = align_up(off_merge + merge_bytes, 16);
            const uint32_t with_qs = off_qs + qs_bytes + 1024;
            if (qshare && with_qs <= (uint32_t)max_smem && (with_qs <= per_cta || L.per_sm == 1)) {
                L.off_qhi = off_qs;
                L.off_qlo = off_qs + 4u * dh;
                L.off_qmisc = off_qs + 8u * dh;
                L.smem_bytes = with_qs;
            } else if (qshare && S >= 3 && tail >= 4u * dh) {
                L.off_qhi = used;
                L.off_qlo = L.stage_bytes + used;
                L.off_qmisc = 2u * L.stage_bytes + used;
            }
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

cudaError_t prepare_fn(void *fn, size_t smem, int *occupancy, int threads)
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
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, threads, smem);
    if (e != cudaSuccess) return e;
    g_occ.push_back(OccMemo{dev, fn, smem, occ});
    *occupancy = occ;
    return cudaSuccess;
}
}  // namespace

static void *plan_fn(const DecodeLaunch &plan)
{
    if (plan.tc) return decode_tc_fn(plan.kb, plan.vb, plan.kg, plan.G, plan.fmt);
    if (plan.pk) return pick_decode_pk(plan.dh, plan.kb, plan.vb, plan.kg, plan.vg, plan.fmt, plan.G);
    return pick_decode(plan.dh, plan.kb, plan.vb, plan.kg, plan.vg, plan.fmt);
}

cudaError_t decode_occupancy(const DecodeLaunch &plan, int *ctas_per_sm)
{
    return prepare_fn(plan_fn(plan), plan.smem_bytes, ctas_per_sm, plan.tc ? 192 : NTHR);
}

cudaError_t launch_decode(const DecodeLaunch &plan, const DecodeParams &p, const CUtensorMap &tm_k,
                          const CUtensorMap &tm_v, cudaStream_t stream)
{
    void *fn = plan_fn(plan);
    cudaError_t e = prepare_fn(fn, plan.smem_bytes, nullptr, 0);
    if (e != cudaSuccess) return e;
    void *args[] = {const_cast<CUtensorMap *>(&tm_k), const_cast<CUtensorMap *>(&tm_v),
                    const_cast<DecodeParams *>(&p)};
    // Programmatic dependent launch: the kernel may be scheduled while the
    // previous work on the stream drains; it waits for that work's completion
    // (griddepcontrol.wait) before its first global-memory access.
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(p.num_ctas);
    lc.blockDim = dim3(plan.tc ? 192 : NTHR);
    lc.dynamicSmemBytes = plan.smem_bytes;
    lc.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 1;
    (void)cudaGetLastError();  // drop a stale, already-reported error of an earlier call
    return cudaLaunchKernelExC(&lc, fn, args);
}

cudaError_t launch_merge(const MergeParams &p, cudaStream_t stream)
{
    const int64_t warps = (int64_t)p.batch * p.n_kv_heads;
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
