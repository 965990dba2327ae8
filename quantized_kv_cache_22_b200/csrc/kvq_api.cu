// kvq_api.cu -- the extern "C" boundary of libkvq: argument validation, TMA
// descriptor encoding and stream-ordered launches.  No allocation, no state
// that changes results (the only memos are the driver entry point address and
// per-device attribute / occupancy queries).
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kvq_internal.h"
#include "../../include/kvq.h"

using namespace kvq;

namespace {

constexpr uint64_t kTimeoutNs = 1000000000ull;  // bounded waits give up after ~1 s

thread_local char g_detail[160] = "";

// Record which step failed with which CUDA error (read by kvq_last_error_detail).
int fail(const char *where, cudaError_t e)
{
    snprintf(g_detail, sizeof(g_detail), "%s: %s", where, e == cudaSuccess ? "ok" : cudaGetErrorName(e));
    return KVQ_ERR_LAUNCH;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_group(int group, int dim)
{
    return (group == 32 || group == 64 || group == 128) && dim % group == 0;
}

bool valid_bits(int b) { return b == 4 || b == 8 || b == 16; }

int check_cfg(const kvq_config *c)
{
    if (!c) return KVQ_ERR_INVALID_ARG;
    if (c->mode != KVQ_MODE_KV && c->mode != KVQ_MODE_H) return KVQ_ERR_INVALID_ARG;
    if (c->batch < 1 || c->capacity < 16 || c->n_layers < 0) return KVQ_ERR_INVALID_ARG;
    if (c->capacity % 16 != 0) return KVQ_ERR_UNSUPPORTED;
    if (c->mode == KVQ_MODE_KV) {
        if (c->n_kv_heads < 1 || c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads != 0)
            return KVQ_ERR_INVALID_ARG;
        if (c->head_dim != 64 && c->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
        if (!valid_bits(c->k_bits) || !valid_bits(c->v_bits)) return KVQ_ERR_UNSUPPORTED;
        if (c->k_bits != 16 && !valid_group(c->k_group, c->head_dim)) return KVQ_ERR_UNSUPPORTED;
        if (c->v_bits != 16 && !valid_group(c->v_group, c->head_dim)) return KVQ_ERR_UNSUPPORTED;
        if (c->window < 0 || c->n_anchor < 0) return KVQ_ERR_INVALID_ARG;
        if (c->window == 0 && c->n_anchor != 0) return KVQ_ERR_INVALID_ARG;
        if (c->window > 0 && (int64_t)c->n_anchor + c->window != c->capacity)
            return KVQ_ERR_INVALID_ARG;
        if (c->kv_format < KVQ_FMT_INT || c->kv_format > KVQ_FMT_TENSOR) return KVQ_ERR_INVALID_ARG;
        if (c->kv_format != KVQ_FMT_INT && (c->k_bits != 8 || c->v_bits != 8))
            return KVQ_ERR_UNSUPPORTED;
        if (c->kv_format == KVQ_FMT_TENSOR && (c->k_group != c->head_dim || c->v_group != c->head_dim))
            return KVQ_ERR_UNSUPPORTED;
        if (c->page_tokens != 0) {
            if (c->page_tokens != kPageTokens) return KVQ_ERR_UNSUPPORTED;
            if (c->window != 0) return KVQ_ERR_UNSUPPORTED;
            if (c->n_pages < 1 || c->capacity % kPageTokens != 0) return KVQ_ERR_INVALID_ARG;
        } else if (c->n_pages != 0) {
            return KVQ_ERR_INVALID_ARG;
        }
    } else {
        if (c->window != 0 || c->n_anchor != 0 || c->page_tokens != 0 || c->n_pages != 0 ||
            c->kv_format != KVQ_FMT_INT)
            return KVQ_ERR_UNSUPPORTED;
        if (c->d_model < 128 || c->d_model % 128 != 0) return KVQ_ERR_UNSUPPORTED;
        if (!valid_bits(c->h_bits)) return KVQ_ERR_UNSUPPORTED;
        if (c->h_bits != 16) {
            if (c->h_groups < 1 || c->d_model % c->h_groups != 0) return KVQ_ERR_UNSUPPORTED;
            if (!valid_group(c->d_model / c->h_groups, c->d_model)) return KVQ_ERR_UNSUPPORTED;
        }
    }
    return KVQ_OK;
}

uint64_t tensor_row_bytes(int dim, int bits) { return (uint64_t)dim * bits / 8; }

int scale_groups(int dim, int bits, int group) { return bits == 16 ? 0 : dim / group; }

// fp16 values per (token, head) row in a KV-mode scale array
int scale_row_vals(const kvq_config *c, int bits, int group)
{
    if (bits == 16 || c->kv_format == KVQ_FMT_TENSOR) return 0;
    return scale_groups(c->head_dim, bits, group) * scale_vals(c->kv_format);
}

// ---------------------------------------------------------------- TMA encode
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

// Codes of one layer viewed as [bh][cap][R bytes]; a tile of T tokens is one
// 128-byte-swizzled box (R <= 128: 128/R tokens per 128-byte line) or two
// 128-byte-wide boxes (R = 256).
bool encode_codes_map_uncached(CUtensorMap *m, const void *codes, int bh, int cap, int R);

// The descriptor depends only on (address, bh, cap, R): the last few encodings
// of this thread are kept, so a decode loop over layers does not re-encode.
bool encode_codes_map(CUtensorMap *m, const void *codes, int bh, int cap, int R)
{
    struct Entry {
        const void *codes;
        int bh, cap, R;
        CUtensorMap map;
    };
    constexpr int kEntries = 256;
    thread_local Entry cache[kEntries];
    thread_local int used = 0, next = 0;
    for (int i = 0; i < used; i++) {
        const Entry &e = cache[i];
        if (e.codes == codes && e.bh == bh && e.cap == cap && e.R == R) {
            *m = e.map;
            return true;
        }
    }
    if (!encode_codes_map_uncached(m, codes, bh, cap, R)) return false;
    Entry &e = cache[next];
    e.codes = codes;
    e.bh = bh;
    e.cap = cap;
    e.R = R;
    e.map = *m;
    next = (next + 1) % kEntries;
    if (used < kEntries) used++;
    return true;
}

bool encode_codes_map_uncached(CUtensorMap *m, const void *codes, int bh, int cap, int R)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3], strides[2];
    cuuint32_t box[3], estr[3] = {1, 1, 1};
    if (R <= 128) {
        dims[0] = 128;
        dims[1] = (cuuint64_t)cap * R / 128;
        dims[2] = (cuuint64_t)bh;
        strides[0] = 128;
        strides[1] = (cuuint64_t)cap * R;
        box[0] = 128;
        box[1] = (cuuint32_t)(kDecodeTileTokens * R / 128);
        box[2] = 1;
    } else {
        dims[0] = (cuuint64_t)R;
        dims[1] = (cuuint64_t)cap;
        dims[2] = (cuuint64_t)bh;
        strides[0] = (cuuint64_t)R;
        strides[1] = (cuuint64_t)cap * R;
        box[0] = 128;
        box[1] = kDecodeTileTokens;
        box[2] = 1;
    }
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(codes), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int current_device_props(int *sms, int *max_smem)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_DEVICE;
    // memo of the three attributes per device (they never change)
    static std::mutex mu;
    static int memo[64][3];
    static bool have[64];
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lk(mu);
        if (have[dev]) {
            if (memo[dev][0] != 10) return KVQ_ERR_DEVICE;
            *sms = memo[dev][1];
            *max_smem = memo[dev][2];
            return KVQ_OK;
        }
    }
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return KVQ_ERR_DEVICE;
    if (major != 10) return KVQ_ERR_DEVICE;  // sm_100a kernels only
    if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return KVQ_ERR_DEVICE;
    if (cudaDeviceGetAttribute(max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
        return KVQ_ERR_DEVICE;
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lk(mu);
        memo[dev][0] = major;
        memo[dev][1] = *sms;
        memo[dev][2] = *max_smem;
        have[dev] = true;
    }
    return KVQ_OK;
}

// Shapes of the attention half (KV mode, or h-mode after reconstruction).
struct AttnShape {
    int hkv, hq, G, dh, kb, vb, kg, vg, ngs_k, ngs_v;
    int fmt;   // KVQ_FMT_* of the 8-bit codes
};

AttnShape attn_shape(const kvq_config *c)
{
    AttnShape s{};
    s.hkv = c->n_kv_heads;
    s.hq = c->n_q_heads;
    s.G = s.hq / s.hkv;
    s.dh = c->head_dim;
    if (c->mode == KVQ_MODE_KV) {
        s.kb = c->k_bits;
        s.vb = c->v_bits;
        s.kg = c->k_group;
        s.vg = c->v_group;
        s.fmt = c->kv_format;
    } else {
        s.kb = s.vb = 16;
        s.kg = s.vg = s.dh;
    }
    // fp16 values per (token, head) row of the scale arrays
    s.ngs_k = c->mode == KVQ_MODE_KV ? scale_row_vals(c, s.kb, s.kg) : scale_groups(s.dh, s.kb, s.kg);
    s.ngs_v = c->mode == KVQ_MODE_KV ? scale_row_vals(c, s.vb, s.vg) : scale_groups(s.dh, s.vb, s.vg);
    return s;
}

int resolve_plan(const kvq_config *cfg, int32_t num_ctas, DecodeLaunch *plan, int *ctas)
{
    const AttnShape a = attn_shape(cfg);
    if (a.G > 8) return KVQ_ERR_UNSUPPORTED;
    int sms = 148, max_smem = 232448;
    if (num_ctas <= 0) {
        int rc = current_device_props(&sms, &max_smem);
        if (rc) return rc;
    }
    if (!plan_decode(a.dh, a.kb, a.vb, a.ngs_k, a.ngs_v, a.G, max_smem, plan, a.fmt))
        return KVQ_ERR_UNSUPPORTED;
    if (num_ctas > 0) {
        *ctas = num_ctas;
        return KVQ_OK;
    }
    int per_sm = 0;
    if (decode_occupancy(*plan, &per_sm) != cudaSuccess || per_sm < 1) return KVQ_ERR_DEVICE;
    // the occupancy query reports one CTA per SM for the tensor-core kernel although
    // two of the size it is planned for run side by side (measured: 296 CTAs of the
    // 8K K8V8 launch take 54.9 us, 148 take 73.8 us), so its plan decides
    if (plan->tc) per_sm = plan->per_sm;
    *ctas = sms * per_sm;
    return KVQ_OK;
}

uint64_t workspace_need(const kvq_config *cfg, int ctas)
{
    const AttnShape a = attn_shape(cfg);
    return (uint64_t)kWorkspaceHeaderFloats * 4 + counter_ints(cfg->batch, a.hkv) * 4 +
           slot_count(ctas, cfg->batch, a.hkv) * slot_floats(a.G, a.dh) * 4;
}

}  // namespace

extern "C" {

const char *kvq_last_error_detail(void) { return g_detail; }

const char *kvq_status_string(int status)
{
    switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported bit-width, group or head shape";
    case KVQ_ERR_CAPACITY: return "position or length beyond the cache capacity";
    case KVQ_ERR_ALIGN: return "pointer not 16-byte aligned";
    case KVQ_ERR_WORKSPACE: return "workspace or scratch too small";
    case KVQ_ERR_LAUNCH: return "CUDA launch failed";
    case KVQ_ERR_DEVICE: return "no usable sm_100 CUDA device";
    case KVQ_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    default: return "unknown status";
    }
}

int kvq_cache_bytes(const kvq_config *cfg, uint64_t *per_token_layer, uint64_t *per_layer,
                    uint64_t *total)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    uint64_t b = 0;
    if (cfg->mode == KVQ_MODE_KV) {
        const int bits[2] = {cfg->k_bits, cfg->v_bits};
        const int grp[2] = {cfg->k_group, cfg->v_group};
        for (int i = 0; i < 2; i++) {
            b += (uint64_t)cfg->n_kv_heads * tensor_row_bytes(cfg->head_dim, bits[i]);
            b += (uint64_t)cfg->n_kv_heads * scale_row_vals(cfg, bits[i], grp[i]) * 2;
        }
    } else {
        b = tensor_row_bytes(cfg->d_model, cfg->h_bits);
        if (cfg->h_bits != 16) b += (uint64_t)cfg->h_groups * 2;
    }
    const uint64_t slots = cfg->page_tokens ? (uint64_t)cfg->n_pages * kPageTokens
                                            : (uint64_t)cfg->batch * (uint64_t)cfg->capacity;
    // per-tensor scales: one fp16 for K and one for V per layer
    const uint64_t layer = b * slots + (cfg->mode == KVQ_MODE_KV && cfg->kv_format == KVQ_FMT_TENSOR ? 4 : 0);
    if (per_token_layer) *per_token_layer = b;
    if (per_layer) *per_layer = layer;
    if (total) *total = layer * (uint64_t)cfg->n_layers;
    return KVQ_OK;
}

int kvq_layer_buffer_bytes(const kvq_config *cfg, uint64_t *k_codes, uint64_t *k_scales,
                           uint64_t *v_codes, uint64_t *v_scales)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    const uint64_t rows = cfg->page_tokens ? (uint64_t)cfg->n_pages * kPageTokens
                                           : (uint64_t)cfg->batch * cfg->capacity;
    uint64_t kc, ks, vc = 0, vs = 0;
    if (cfg->mode == KVQ_MODE_KV) {
        const uint64_t hr = rows * cfg->n_kv_heads;
        kc = hr * tensor_row_bytes(cfg->head_dim, cfg->k_bits);
        ks = hr * scale_row_vals(cfg, cfg->k_bits, cfg->k_group) * 2;
        vc = hr * tensor_row_bytes(cfg->head_dim, cfg->v_bits);
        vs = hr * scale_row_vals(cfg, cfg->v_bits, cfg->v_group) * 2;
        if (cfg->kv_format == KVQ_FMT_TENSOR) ks = vs = 2;   // one fp16 scale each
    } else {
        kc = rows * tensor_row_bytes(cfg->d_model, cfg->h_bits);
        ks = cfg->h_bits == 16 ? 0 : rows * (uint64_t)cfg->h_groups * 2;
    }
    if (k_codes) *k_codes = kc;
    if (k_scales) *k_scales = ks;
    if (v_codes) *v_codes = vc;
    if (v_scales) *v_scales = vs;
    return KVQ_OK;
}

int kvq_append(const kvq_config *cfg, const kvq_layer *layer, const void *k, const void *v,
               int32_t in_dtype, const int32_t *d_pos, int32_t max_pos_host, int32_t n_new,
               kvq_stream_t stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!layer || !d_pos || n_new < 0 || max_pos_host < 0) return KVQ_ERR_INVALID_ARG;
    if (in_dtype != KVQ_F16 && in_dtype != KVQ_F32 && in_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    // with a sliding window positions grow without bound (ring slots)
    if (cfg->window == 0 && (int64_t)max_pos_host + n_new > cfg->capacity) return KVQ_ERR_CAPACITY;
    if (n_new == 0) return KVQ_OK;
    AppendParams pk{};
    pk.window = cfg->window;
    pk.n_anchor = cfg->n_anchor;
    pk.fmt = cfg->mode == KVQ_MODE_KV ? cfg->kv_format : KVQ_FMT_INT;
    if (cfg->mode == KVQ_MODE_KV && cfg->page_tokens) {
        if (!layer->block_table) return KVQ_ERR_INVALID_ARG;
        pk.block_table = layer->block_table;
        pk.max_pages = cfg->capacity / kPageTokens;
        pk.n_pages = cfg->n_pages;
    }
    pk.in_dtype = in_dtype;
    pk.batch = cfg->batch;
    pk.n_new = n_new;
    pk.cap = cfg->capacity;
    pk.d_pos = d_pos;
    if (cfg->mode == KVQ_MODE_KV) {
        if (!k || !v || !layer->k_codes || !layer->v_codes) return KVQ_ERR_INVALID_ARG;
        if ((cfg->k_bits != 16 && !layer->k_scales) || (cfg->v_bits != 16 && !layer->v_scales))
            return KVQ_ERR_INVALID_ARG;
        if (!aligned16(k) || !aligned16(v) || !aligned16(layer->k_codes) ||
            !aligned16(layer->v_codes) || (layer->k_scales && !aligned16(layer->k_scales)) ||
            (layer->v_scales && !aligned16(layer->v_scales)))
            return KVQ_ERR_ALIGN;
        pk.rows_per_tok = cfg->n_kv_heads;
        pk.dim = cfg->head_dim;
        AppendParams pv = pk;
        pk.x = k;
        pk.codes = static_cast<uint8_t *>(layer->k_codes);
        pk.scales = static_cast<__half *>(layer->k_scales);
        pk.bits = cfg->k_bits;
        pk.group = cfg->k_bits == 16 ? 32 : cfg->k_group;
        pv.x = v;
        pv.codes = static_cast<uint8_t *>(layer->v_codes);
        pv.scales = static_cast<__half *>(layer->v_scales);
        pv.bits = cfg->v_bits;
        pv.group = cfg->v_bits == 16 ? 32 : cfg->v_group;
        cudaError_t e = launch_append(pk, &pv, reinterpret_cast<cudaStream_t>(stream));
        return e == cudaSuccess ? KVQ_OK : fail("append launch", e);
    }
    if (!k || v || !layer->k_codes) return KVQ_ERR_INVALID_ARG;
    if (cfg->h_bits != 16 && !layer->k_scales) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(layer->k_codes) ||
        (layer->k_scales && !aligned16(layer->k_scales)))
        return KVQ_ERR_ALIGN;
    pk.rows_per_tok = 1;
    pk.dim = cfg->d_model;
    pk.x = k;
    pk.codes = static_cast<uint8_t *>(layer->k_codes);
    pk.scales = static_cast<__half *>(layer->k_scales);
    pk.bits = cfg->h_bits;
    pk.group = cfg->h_bits == 16 ? 32 : cfg->d_model / cfg->h_groups;
    cudaError_t e = launch_append(pk, nullptr, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : fail("append launch", e);
}

int kvq_workspace_bytes(const kvq_config *cfg, int32_t num_ctas, uint64_t *bytes)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!bytes || num_ctas < 0) return KVQ_ERR_INVALID_ARG;
    if (cfg->mode == KVQ_MODE_H && cfg->n_kv_heads * cfg->head_dim != cfg->d_model)
        return KVQ_ERR_INVALID_ARG;
    DecodeLaunch plan;
    int ctas = 0;
    rc = resolve_plan(cfg, num_ctas, &plan, &ctas);
    if (rc) return rc;
    *bytes = workspace_need(cfg, ctas);
    return KVQ_OK;
}

int kvq_decode_plan_info(const kvq_config *cfg, int32_t num_ctas, kvq_decode_plan *info)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!info || num_ctas < 0) return KVQ_ERR_INVALID_ARG;
    if (cfg->mode == KVQ_MODE_H && cfg->n_kv_heads * cfg->head_dim != cfg->d_model)
        return KVQ_ERR_INVALID_ARG;
    DecodeLaunch plan;
    int ctas = 0;
    rc = resolve_plan(cfg, num_ctas, &plan, &ctas);
    if (rc) return rc;
    info->engine = plan.tc ? KVQ_ENGINE_TCGEN05 : KVQ_ENGINE_WARP_MMA;
    info->num_ctas = ctas;
    info->ctas_per_sm_planned = plan.per_sm;
    info->stages = plan.stages;
    info->stage_bytes = plan.stage_bytes;
    info->smem_bytes = (int32_t)plan.smem_bytes;
    info->threads = plan.tc ? 192 : kDecodeThreads;
    info->packed_columns = plan.pk ? 1 : 0;
    return KVQ_OK;
}

static uint64_t h_operand_need(const kvq_config *cfg, int32_t max_len)
{
    const uint64_t pad = ((uint64_t)max_len + kHTileTokens - 1) / kHTileTokens * kHTileTokens;
    return (uint64_t)cfg->batch * pad * (uint64_t)cfg->d_model * 2;
}

static uint64_t h_kv_need(const kvq_config *cfg, int32_t max_len)
{
    const uint64_t cap = ((uint64_t)max_len + 63) / 64 * 64;
    return 2ull * cfg->batch * cfg->n_kv_heads * cap * cfg->head_dim * 2;
}

int kvq_h_scratch_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_H || !bytes || max_len < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len > cfg->capacity) return KVQ_ERR_CAPACITY;
    *bytes = h_kv_need(cfg, max_len) + h_operand_need(cfg, max_len);
    return KVQ_OK;
}

int kvq_h_operand_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_H || !bytes || max_len < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len > cfg->capacity) return KVQ_ERR_CAPACITY;
    *bytes = h_operand_need(cfg, max_len);
    return KVQ_OK;
}

// Validated KV-layout attention.  do_partials && do_merge: one launch that
// also merges (arrival counters in the workspace); do_partials alone leaves
// the per-warp partials; do_merge alone launches the merge kernel over them.
// `app` (optional) fuses the append of each sequence's newest token.
static int decode_kv_layout(const kvq_config *cfg, const void *k_codes, const void *k_scales,
                            const void *v_codes, const void *v_scales, int cap, const void *q,
                            int32_t q_dtype, const int32_t *d_len, float softmax_scale, void *out,
                            int32_t out_dtype, void *workspace, uint64_t workspace_bytes,
                            int32_t num_ctas, cudaStream_t stream, bool do_partials, bool do_merge,
                            const FusedAppend *app = nullptr,
                            const int32_t *block_table = nullptr, uint64_t stall_ns = 0)
{
    const AttnShape a = attn_shape(cfg);
    // fp16 and e4m3 keys use an f16 MMA whose f32 / bf16 queries take two columns per head
    if ((a.kb == 16 || a.fmt == KVQ_FMT_E4M3) && q_dtype != KVQ_F16 && a.G > 4)
        return KVQ_ERR_UNSUPPORTED;
    DecodeLaunch plan;
    int ctas = 0;
    int rc = resolve_plan(cfg, num_ctas, &plan, &ctas);
    if (rc) return rc;
    if (workspace_bytes < workspace_need(cfg, ctas)) return KVQ_ERR_WORKSPACE;
    int *counters = reinterpret_cast<int *>(static_cast<float *>(workspace) + kWorkspaceHeaderFloats);
    float *ws = reinterpret_cast<float *>(counters + counter_ints(cfg->batch, a.hkv));

    if (do_partials) {
        CUtensorMap tm_k, tm_v;
        // contiguous: [B*Hkv][cap] rows; paged: the pool, [n_pages*Hkv][128] rows
        const int zdim = block_table ? cfg->n_pages * a.hkv : cfg->batch * a.hkv;
        const int ydim = block_table ? kPageTokens : cap;
        if (!encode_codes_map(&tm_k, k_codes, zdim, ydim, a.dh * a.kb / 8) ||
            !encode_codes_map(&tm_v, v_codes, zdim, ydim, a.dh * a.vb / 8))
            return fail("tensor map encode", cudaErrorInvalidValue);
        DecodeParams p{};
        p.d_len = d_len;
        p.q = q;
        p.k_scales = static_cast<const __half *>(k_scales);
        p.v_scales = static_cast<const __half *>(v_scales);
        p.status = static_cast<int *>(workspace);
        p.ws = ws;
        p.counters = do_merge ? counters : nullptr;
        p.out = do_merge ? out : nullptr;
        p.out_f32 = out_dtype == KVQ_F32;
        p.q_dtype = q_dtype;
        p.batch = cfg->batch;
        p.n_q_heads = a.hq;
        p.n_kv_heads = a.hkv;
        p.group_size_g = a.G;
        p.cap = cap;
        p.ngs_k = a.ngs_k;
        p.ngs_v = a.ngs_v;
        p.kshift = a.kb == 16 ? 0 : (a.kg == 32 ? 0 : (a.kg == 64 ? 1 : 2));
        p.vshift = a.vb == 16 ? 0 : (a.vg == 32 ? 0 : (a.vg == 64 ? 1 : 2));
        p.num_ctas = ctas;
        p.stages = plan.stages;
        p.stage_bytes = plan.stage_bytes;
        p.off_v = plan.off_v;
        p.off_sk = plan.off_sk;
        p.off_sv = plan.off_sv;
        p.off_meta = plan.off_meta;
        p.off_bar = plan.off_bar;
        p.off_merge = plan.off_merge;
        p.off_qhi = plan.off_qhi;
        p.off_qlo = plan.off_qlo;
        p.off_qmisc = plan.off_qmisc;
        p.tc = plan.tco;
        const float scale = softmax_scale != 0.f ? softmax_scale : 1.f / std::sqrt((float)a.dh);
        p.tau_log2e = scale * 1.4426950408889634f;
        p.timeout_ns = stall_ns ? stall_ns : kTimeoutNs;
        p.stall = stall_ns ? 1 : 0;
        if (app) p.app = *app;
        p.window = cfg->mode == KVQ_MODE_KV ? cfg->window : 0;
        p.n_anchor = cfg->mode == KVQ_MODE_KV ? cfg->n_anchor : 0;
        p.block_table = block_table;
        p.max_pages = block_table ? cap / kPageTokens : 0;
        p.n_pages = block_table ? cfg->n_pages : 0;
        cudaError_t e = launch_decode(plan, p, tm_k, tm_v, stream);
        if (e != cudaSuccess) return fail("decode launch", e);
        return KVQ_OK;
    }
    if (do_merge) {
        MergeParams mp{};
        mp.d_len = d_len;
        mp.ws = ws;
        mp.out = out;
        mp.out_f32 = out_dtype == KVQ_F32;
        mp.batch = cfg->batch;
        mp.n_q_heads = a.hq;
        mp.n_kv_heads = a.hkv;
        mp.group_size_g = a.G;
        mp.cap = cap;
        mp.head_dim = a.dh;
        mp.num_ctas = ctas;
        cudaError_t e = launch_merge(mp, stream);
        if (e != cudaSuccess) return fail("merge launch", e);
    }
    return KVQ_OK;
}

static int check_kv_layer(const kvq_config *cfg, const kvq_layer *layer)
{
    if (!layer->k_codes || !layer->v_codes) return KVQ_ERR_INVALID_ARG;
    if (cfg->page_tokens && !layer->block_table) return KVQ_ERR_INVALID_ARG;
    if ((cfg->k_bits != 16 && !layer->k_scales) || (cfg->v_bits != 16 && !layer->v_scales))
        return KVQ_ERR_INVALID_ARG;
    if (!aligned16(layer->k_codes) || !aligned16(layer->v_codes) ||
        (layer->k_scales && !aligned16(layer->k_scales)) ||
        (layer->v_scales && !aligned16(layer->v_scales)))
        return KVQ_ERR_ALIGN;
    return KVQ_OK;
}

int kvq_decode_partials(const kvq_config *cfg, const kvq_layer *layer, const void *q,
                        int32_t q_dtype, const int32_t *d_len, int32_t max_len_host,
                        float softmax_scale, void *workspace, uint64_t workspace_bytes,
                        int32_t num_ctas, kvq_stream_t stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_KV) return KVQ_ERR_INVALID_ARG;
    if (!layer || !q || !d_len || !workspace || num_ctas < 0) return KVQ_ERR_INVALID_ARG;
    if (q_dtype != KVQ_F16 && q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || max_len_host < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len_host > cfg->capacity && cfg->window == 0) return KVQ_ERR_CAPACITY;
    if (!aligned16(q) || !aligned16(workspace)) return KVQ_ERR_ALIGN;
    rc = check_kv_layer(cfg, layer);
    if (rc) return rc;
    return decode_kv_layout(cfg, layer->k_codes, layer->k_scales, layer->v_codes, layer->v_scales,
                            cfg->capacity, q, q_dtype, d_len, softmax_scale, nullptr, KVQ_F32,
                            workspace, workspace_bytes, num_ctas,
                            reinterpret_cast<cudaStream_t>(stream), true, false, nullptr,
                            cfg->page_tokens ? layer->block_table : nullptr);
}

int kvq_merge_partials(const kvq_config *cfg, const int32_t *d_len, void *out, int32_t out_dtype,
                       void *workspace, uint64_t workspace_bytes, int32_t num_ctas,
                       kvq_stream_t stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_KV) return KVQ_ERR_INVALID_ARG;
    if (!d_len || !out || !workspace || num_ctas < 0) return KVQ_ERR_INVALID_ARG;
    if (out_dtype != KVQ_F16 && out_dtype != KVQ_F32) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(workspace)) return KVQ_ERR_ALIGN;
    return decode_kv_layout(cfg, nullptr, nullptr, nullptr, nullptr, cfg->capacity, nullptr,
                            KVQ_F16, d_len, 0.f, out, out_dtype, workspace, workspace_bytes,
                            num_ctas, reinterpret_cast<cudaStream_t>(stream), false, true);
}

static int h_reconstruct_impl(const kvq_config *cfg, const kvq_layer *layer, const void *w_kv,
                              int32_t max_len_host, void *k_out, void *v_out,
                              int32_t out_capacity, void *operand, uint64_t operand_bytes,
                              int *status, kvq_stream_t stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_H || !layer || !layer->k_codes || !w_kv || !k_out || !v_out ||
        !operand)
        return KVQ_ERR_INVALID_ARG;
    if (cfg->n_kv_heads * cfg->head_dim != cfg->d_model) return KVQ_ERR_INVALID_ARG;
    if (cfg->h_bits != 16 && !layer->k_scales) return KVQ_ERR_INVALID_ARG;
    if (max_len_host < 0 || out_capacity < max_len_host || out_capacity % 64 != 0)
        return KVQ_ERR_INVALID_ARG;
    if (max_len_host > cfg->capacity && cfg->window == 0) return KVQ_ERR_CAPACITY;
    if (!aligned16(layer->k_codes) || !aligned16(w_kv) || !aligned16(k_out) ||
        !aligned16(v_out) || !aligned16(operand) ||
        (layer->k_scales && !aligned16(layer->k_scales)))
        return KVQ_ERR_ALIGN;
    if (cfg->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
    if (operand_bytes < h_operand_need(cfg, max_len_host)) return KVQ_ERR_WORKSPACE;
    if (max_len_host == 0) return KVQ_OK;
    HGemmParams p{};
    p.h_codes = static_cast<const uint8_t *>(layer->k_codes);
    p.h_scales = static_cast<const __half *>(layer->k_scales);
    p.w = w_kv;
    p.k_out = static_cast<__half *>(k_out);
    p.v_out = static_cast<__half *>(v_out);
    p.batch = cfg->batch;
    p.cap = cfg->capacity;
    p.d_model = cfg->d_model;
    p.h_bits = cfg->h_bits;
    p.h_groups = cfg->h_bits == 16 ? 1 : cfg->h_groups;
    p.n_kv_heads = cfg->n_kv_heads;
    p.head_dim = cfg->head_dim;
    p.len = max_len_host;
    p.out_cap = out_capacity;
    p.operand = operand;
    p.status = status;
    cudaError_t e = launch_h_reconstruct(p, reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return KVQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? KVQ_OK : fail("reconstruction launch", e);
}

int kvq_decode_attn(const kvq_config *cfg, const kvq_layer *layer, const void *q, int32_t q_dtype,
                    const int32_t *d_len, int32_t max_len_host, float softmax_scale, void *out,
                    int32_t out_dtype, void *workspace, uint64_t workspace_bytes, int32_t num_ctas,
                    const void *w_kv, void *kv_scratch, uint64_t kv_scratch_bytes,
                    kvq_stream_t stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!layer || !q || !d_len || !out || !workspace || num_ctas < 0) return KVQ_ERR_INVALID_ARG;
    if (q_dtype != KVQ_F16 && q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (out_dtype != KVQ_F16 && out_dtype != KVQ_F32) return KVQ_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale)) return KVQ_ERR_INVALID_ARG;
    if (max_len_host < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len_host > cfg->capacity && cfg->window == 0) return KVQ_ERR_CAPACITY;
    if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return KVQ_ERR_ALIGN;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    if (cfg->mode == KVQ_MODE_KV) {
        if (w_kv || kv_scratch || kv_scratch_bytes) return KVQ_ERR_INVALID_ARG;
        rc = check_kv_layer(cfg, layer);
        if (rc) return rc;
        return decode_kv_layout(cfg, layer->k_codes, layer->k_scales, layer->v_codes,
                                layer->v_scales, cfg->capacity, q, q_dtype, d_len, softmax_scale,
                                out, out_dtype, workspace, workspace_bytes, num_ctas, st, true,
                                true, nullptr, cfg->page_tokens ? layer->block_table : nullptr);
    }

    // h-mode: rebuild K, V into the scratch, then attend over 16-bit K/V.
    if (cfg->n_kv_heads * cfg->head_dim != cfg->d_model) return KVQ_ERR_INVALID_ARG;
    if (!w_kv || !kv_scratch || !layer->k_codes) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(w_kv) || !aligned16(kv_scratch)) return KVQ_ERR_ALIGN;
    if (cfg->head_dim != 128 || cfg->n_q_heads % cfg->n_kv_heads != 0) return KVQ_ERR_UNSUPPORTED;
    uint64_t need = 0;
    rc = kvq_h_scratch_bytes(cfg, max_len_host, &need);
    if (rc) return rc;
    if (kv_scratch_bytes < need) return KVQ_ERR_WORKSPACE;
    const int scap = (max_len_host + 63) / 64 * 64;
    if (scap == 0) {
        // nothing cached: every output is zero
        const size_t ob = (size_t)cfg->batch * cfg->n_q_heads * cfg->head_dim *
                          (out_dtype == KVQ_F32 ? 4 : 2);
        cudaError_t e = cudaMemsetAsync(out, 0, ob, st);
        return e == cudaSuccess ? KVQ_OK : fail("zero output", e);
    }
    __half *kout = static_cast<__half *>(kv_scratch);
    __half *vout = kout + (size_t)cfg->batch * cfg->n_kv_heads * scap * cfg->head_dim;
    uint8_t *operand = static_cast<uint8_t *>(kv_scratch) + h_kv_need(cfg, max_len_host);
    rc = h_reconstruct_impl(cfg, layer, w_kv, max_len_host, kout, vout, scap, operand,
                            h_operand_need(cfg, max_len_host), static_cast<int *>(workspace),
                            stream);
    if (rc) return rc;
    return decode_kv_layout(cfg, kout, nullptr, vout, nullptr, scap, q, q_dtype, d_len,
                            softmax_scale, out, out_dtype, workspace, workspace_bytes, num_ctas, st,
                            true, true);
}

int kvq_append_decode_attn(const kvq_config *cfg, const kvq_layer *layer, const void *k_new,
                           const void *v_new, int32_t in_dtype, const void *q, int32_t q_dtype,
                           const int32_t *d_len, int32_t max_len_host, float softmax_scale,
                           void *out, int32_t out_dtype, void *workspace, uint64_t workspace_bytes,
                           int32_t num_ctas, kvq_stream_t stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_KV) return KVQ_ERR_INVALID_ARG;
    if (!layer || !k_new || !v_new || !q || !d_len || !out || !workspace || num_ctas < 0)
        return KVQ_ERR_INVALID_ARG;
    if (in_dtype != KVQ_F16 && in_dtype != KVQ_F32 && in_dtype != KVQ_BF16)
        return KVQ_ERR_INVALID_ARG;
    if (q_dtype != KVQ_F16 && q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (out_dtype != KVQ_F16 && out_dtype != KVQ_F32) return KVQ_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || max_len_host < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len_host > cfg->capacity && cfg->window == 0) return KVQ_ERR_CAPACITY;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(q) || !aligned16(out) ||
        !aligned16(workspace))
        return KVQ_ERR_ALIGN;
    rc = check_kv_layer(cfg, layer);
    if (rc) return rc;
    FusedAppend app{};
    app.k_new = k_new;
    app.v_new = v_new;
    app.k_codes = static_cast<uint8_t *>(layer->k_codes);
    app.v_codes = static_cast<uint8_t *>(layer->v_codes);
    app.k_scales = static_cast<__half *>(layer->k_scales);
    app.v_scales = static_cast<__half *>(layer->v_scales);
    app.dtype = in_dtype;
    app.k_group = cfg->k_bits == 16 ? 32 : cfg->k_group;
    app.v_group = cfg->v_bits == 16 ? 32 : cfg->v_group;
    return decode_kv_layout(cfg, layer->k_codes, layer->k_scales, layer->v_codes, layer->v_scales,
                            cfg->capacity, q, q_dtype, d_len, softmax_scale, out, out_dtype,
                            workspace, workspace_bytes, num_ctas,
                            reinterpret_cast<cudaStream_t>(stream), true, true, &app,
                            cfg->page_tokens ? layer->block_table : nullptr);
}

int kvq_h_reconstruct(const kvq_config *cfg, const kvq_layer *layer, const void *w_kv,
                      int32_t max_len_host, void *k_out, void *v_out, int32_t out_capacity,
                      void *operand, uint64_t operand_bytes, kvq_stream_t stream)
{
    return h_reconstruct_impl(cfg, layer, w_kv, max_len_host, k_out, v_out, out_capacity, operand,
                              operand_bytes, nullptr, stream);
}

// ------------------------------------------------------------ fused reconstruction
static int fused_shape_check(const kvq_config *cfg)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_H) return KVQ_ERR_INVALID_ARG;
    if (cfg->n_kv_heads * cfg->head_dim != cfg->d_model) return KVQ_ERR_INVALID_ARG;
    if (cfg->head_dim != 128 || cfg->n_q_heads % cfg->n_kv_heads != 0 ||
        cfg->n_q_heads / cfg->n_kv_heads > 8)
        return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
}

static uint64_t fused_part_bytes(const kvq_config *cfg, int max_len)
{
    const uint64_t m_tiles = (uint64_t)((max_len + kHTileTokens - 1) / kHTileTokens);
    return (uint64_t)cfg->batch * cfg->n_q_heads * m_tiles * 4 * (cfg->head_dim + 2) * 4;
}

int kvq_h_fused_scratch_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes)
{
    int rc = fused_shape_check(cfg);
    if (rc) return rc;
    if (!bytes || max_len < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len > cfg->capacity) return KVQ_ERR_CAPACITY;
    *bytes = 256 + h_operand_need(cfg, max_len) + fused_part_bytes(cfg, max_len);
    return KVQ_OK;
}

int kvq_h_decode_fused(const kvq_config *cfg, const kvq_layer *layer, const void *w_kv,
                       const void *q, int32_t q_dtype, const int32_t *d_len, int32_t max_len_host,
                       float softmax_scale, void *out, int32_t out_dtype, void *scratch,
                       uint64_t scratch_bytes, kvq_stream_t stream)
{
    int rc = fused_shape_check(cfg);
    if (rc) return rc;
    if (!layer || !layer->k_codes || (cfg->h_bits != 16 && !layer->k_scales) || !w_kv || !q ||
        !d_len || !out || !scratch)
        return KVQ_ERR_INVALID_ARG;
    if (q_dtype != KVQ_F16 && q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (out_dtype != KVQ_F16 && out_dtype != KVQ_F32) return KVQ_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || max_len_host < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len_host > cfg->capacity) return KVQ_ERR_CAPACITY;
    if (!aligned16(layer->k_codes) || (layer->k_scales && !aligned16(layer->k_scales)) ||
        !aligned16(w_kv) || !aligned16(q) || !aligned16(out) || !aligned16(scratch))
        return KVQ_ERR_ALIGN;
    uint64_t need = 0;
    rc = kvq_h_fused_scratch_bytes(cfg, max_len_host, &need);
    if (rc) return rc;
    if (scratch_bytes < need) return KVQ_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (max_len_host == 0) {
        // nothing cached: every output is zero
        const size_t ob = (size_t)cfg->batch * cfg->n_q_heads * cfg->head_dim * (out_dtype == KVQ_F32 ? 4 : 2);
        cudaError_t e = cudaMemsetAsync(out, 0, ob, st);
        return e == cudaSuccess ? KVQ_OK : fail("zero output", e);
    }
    uint8_t *base = static_cast<uint8_t *>(scratch);
    HGemmParams p{};
    p.h_codes = static_cast<const uint8_t *>(layer->k_codes);
    p.h_scales = static_cast<const __half *>(layer->k_scales);
    p.w = w_kv;
    p.batch = cfg->batch;
    p.cap = cfg->capacity;
    p.d_model = cfg->d_model;
    p.h_bits = cfg->h_bits;
    p.h_groups = cfg->h_bits == 16 ? 1 : cfg->h_groups;
    p.n_kv_heads = cfg->n_kv_heads;
    p.head_dim = cfg->head_dim;
    p.len = max_len_host;
    p.out_cap = 0;
    p.operand = base + 256;
    p.status = reinterpret_cast<int *>(base);
    p.q = q;
    p.d_len = d_len;
    p.part = reinterpret_cast<float *>(base + 256 + h_operand_need(cfg, max_len_host));
    p.out = out;
    p.q_dtype = q_dtype;
    p.n_q_heads = cfg->n_q_heads;
    p.out_f32 = out_dtype == KVQ_F32;
    const float scale = softmax_scale != 0.f ? softmax_scale : 1.f / std::sqrt((float)cfg->head_dim);
    p.tau_log2e = scale * 1.4426950408889634f;
    cudaError_t e = launch_h_reconstruct(p, st);
    if (e == cudaErrorNotSupported) return KVQ_ERR_UNSUPPORTED;
    return e == cudaSuccess ? KVQ_OK : fail("fused reconstruction launch", e);
}

// ------------------------------------------------------------ query absorption
static int absorbed_shape_check(const kvq_config *cfg)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_H) return KVQ_ERR_INVALID_ARG;
    if (cfg->n_kv_heads * cfg->head_dim != cfg->d_model) return KVQ_ERR_INVALID_ARG;
    if (cfg->h_bits != 4 && cfg->h_bits != 8) return KVQ_ERR_UNSUPPORTED;
    if (cfg->head_dim % 32 != 0 || cfg->head_dim > 128 || cfg->d_model % 256 != 0)
        return KVQ_ERR_UNSUPPORTED;
    if (cfg->n_q_heads % cfg->n_kv_heads != 0 || cfg->n_q_heads > 32) return KVQ_ERR_UNSUPPORTED;
    if (!absorb_fits(cfg->d_model, cfg->h_bits, cfg->n_q_heads, cfg->h_groups)) return KVQ_ERR_UNSUPPORTED;
    return KVQ_OK;
}

int kvq_h_absorbed_scratch_bytes(const kvq_config *cfg, int32_t max_len, uint64_t *bytes)
{
    int rc = absorbed_shape_check(cfg);
    if (rc) return rc;
    if (!bytes || max_len < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len > cfg->capacity) return KVQ_ERR_CAPACITY;
    uint64_t off[6];
    *bytes = absorb_scratch_layout(cfg->batch, cfg->n_q_heads, cfg->d_model, cfg->h_groups,
                                   cfg->h_bits, max_len, off);
    return KVQ_OK;
}

int kvq_h_decode_absorbed(const kvq_config *cfg, const kvq_layer *layer, const void *w_kv,
                          const void *q, int32_t q_dtype, const int32_t *d_len,
                          int32_t max_len_host, float softmax_scale, void *out, int32_t out_dtype,
                          void *scratch, uint64_t scratch_bytes, kvq_stream_t stream)
{
    int rc = absorbed_shape_check(cfg);
    if (rc) return rc;
    if (!layer || !layer->k_codes || !layer->k_scales || !w_kv || !q || !d_len || !out || !scratch)
        return KVQ_ERR_INVALID_ARG;
    if (q_dtype != KVQ_F16 && q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (out_dtype != KVQ_F16 && out_dtype != KVQ_F32) return KVQ_ERR_INVALID_ARG;
    if (!std::isfinite(softmax_scale) || max_len_host < 0) return KVQ_ERR_INVALID_ARG;
    if (max_len_host > cfg->capacity) return KVQ_ERR_CAPACITY;
    if (!aligned16(layer->k_codes) || !aligned16(layer->k_scales) || !aligned16(w_kv) ||
        !aligned16(q) || !aligned16(out) || !aligned16(scratch))
        return KVQ_ERR_ALIGN;
    uint64_t off[6];
    const uint64_t need = absorb_scratch_layout(cfg->batch, cfg->n_q_heads, cfg->d_model,
                                                cfg->h_groups, cfg->h_bits, max_len_host, off);
    if (scratch_bytes < need) return KVQ_ERR_WORKSPACE;
    AbsorbParams p{};
    p.h_codes = static_cast<const uint8_t *>(layer->k_codes);
    p.h_scales = static_cast<const __half *>(layer->k_scales);
    p.w = static_cast<const __nv_bfloat16 *>(w_kv);
    p.q = q;
    p.d_len = d_len;
    p.out = out;
    p.q_dtype = q_dtype;
    p.out_f32 = out_dtype == KVQ_F32;
    p.B = cfg->batch;
    p.Hq = cfg->n_q_heads;
    p.Hkv = cfg->n_kv_heads;
    p.Dh = cfg->head_dim;
    p.D = cfg->d_model;
    p.cap = cfg->capacity;
    p.bits = cfg->h_bits;
    p.ng = cfg->h_groups;
    p.group = cfg->d_model / cfg->h_groups;
    const float scale = softmax_scale != 0.f ? softmax_scale : 1.f / std::sqrt((float)cfg->head_dim);
    p.tau_log2e = scale * 1.4426950408889634f;
    uint8_t *base = static_cast<uint8_t *>(scratch);
    p.qfrag = reinterpret_cast<uint4 *>(base + off[0]);
    p.qfac = reinterpret_cast<float *>(base + off[1]);
    p.p = reinterpret_cast<float *>(base + off[2]);
    p.stats = reinterpret_cast<float2 *>(base + off[3]);
    p.obp = reinterpret_cast<float *>(base + off[4]);
    p.capP = (max_len_host + 63) / 64 * 64;
    p.NT = absorb_nt(p.Hq);
    p.T2 = absorb_t2(p.D, p.bits, p.Hq, p.ng);
    p.ntile = p.capP / p.T2;
    p.split = absorb_split(max_len_host);
    cudaError_t e = launch_absorbed(p, max_len_host, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : fail("absorbed decode launch", e);
}

int kvq_selftest_decode_timeout(const kvq_config *cfg, const kvq_layer *layer, const void *q,
                                int32_t q_dtype, const int32_t *d_len, void *out,
                                int32_t out_dtype, void *workspace, uint64_t workspace_bytes,
                                uint64_t timeout_ns, kvq_stream_t stream)
{
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->mode != KVQ_MODE_KV || cfg->page_tokens) return KVQ_ERR_INVALID_ARG;
    if (!layer || !q || !d_len || !out || !workspace) return KVQ_ERR_INVALID_ARG;
    if (timeout_ns == 0 || timeout_ns > 2000000000ull) return KVQ_ERR_INVALID_ARG;
    if (q_dtype != KVQ_F16 && q_dtype != KVQ_F32 && q_dtype != KVQ_BF16) return KVQ_ERR_INVALID_ARG;
    if (out_dtype != KVQ_F16 && out_dtype != KVQ_F32) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return KVQ_ERR_ALIGN;
    rc = check_kv_layer(cfg, layer);
    if (rc) return rc;
    return decode_kv_layout(cfg, layer->k_codes, layer->k_scales, layer->v_codes, layer->v_scales,
                            cfg->capacity, q, q_dtype, d_len, 0.f, out, out_dtype, workspace,
                            workspace_bytes, 0, reinterpret_cast<cudaStream_t>(stream), true, true,
                            nullptr, nullptr, timeout_ns);
}

int kvq_selftest_bounded_wait(void *workspace, uint64_t timeout_ns, kvq_stream_t stream)
{
    if (!workspace || timeout_ns == 0 || timeout_ns > 2000000000ull) return KVQ_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return KVQ_ERR_ALIGN;
    cudaError_t e = launch_bounded_wait_selftest(static_cast<int *>(workspace), timeout_ns,
                                                 reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? KVQ_OK : fail("self-test launch", e);
}

int kvq_workspace_status(void *workspace, int32_t *status, kvq_stream_t stream)
{
    if (!workspace || !status) return KVQ_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return fail("status copy", e);
    e = cudaMemsetAsync(workspace, 0, 4, st);
    if (e != cudaSuccess) return fail("status clear", e);
    e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return fail("status sync", e);
    *status = v;
    return KVQ_OK;
}

}  // extern "C"
