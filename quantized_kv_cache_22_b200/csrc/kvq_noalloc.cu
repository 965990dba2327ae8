// kvq_noalloc.cu -- decode attention whose scratch lives in a device array that
// is part of the library, for callers that may not allocate device memory
// (see kvq_decode_attn_noalloc in include/kvq.h for who they are and why).
//
// The split-KV partials and the status word go into g_noalloc_scratch instead
// of a caller-provided workspace; everything else is the regular
// kvq_decode_attn path.  Host code cannot hand the array's name to a kernel:
// on the host it only names a stand-in object, so the device address is looked
// up once per device with cudaGetSymbolAddress and passed as the workspace.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "kvq_internal.h"
#include "../../include/kvq.h"

namespace {

constexpr uint64_t kScratchBytes = KVQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch: every call in the process shares it (see the race note in kvq.h).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per
// device and kept for the life of the process; a cudaDeviceReset reloads the
// module and can move the array, so the entry points must not be used after one).
int scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return KVQ_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
            return KVQ_ERR_DEVICE;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KVQ_OK;
}

}  // namespace

extern "C" int kvq_decode_attn_noalloc(const kvq_config *cfg, const kvq_layer *layer,
                                       const void *q, int32_t q_dtype, const int32_t *d_len,
                                       int32_t max_len_host, float softmax_scale, void *out,
                                       int32_t out_dtype, int32_t num_ctas, kvq_stream_t stream)
{
    if (!cfg || cfg->mode != KVQ_MODE_KV) return KVQ_ERR_INVALID_ARG;
    uint64_t need = 0;
    int rc = kvq_workspace_bytes(cfg, num_ctas, &need);
    if (rc) return rc;
    if (need > kScratchBytes) return KVQ_ERR_WORKSPACE;
    void *ws = nullptr;
    rc = scratch_address(&ws);
    if (rc) return rc;
    // the status word and the merge's arrival counters must start at zero (a
    // call that timed out can leave counters behind); the partial slots are
    // written before they are read, so nothing else needs clearing
    const uint64_t zero_bytes = (uint64_t)kvq::kWorkspaceHeaderFloats * 4 +
                                kvq::counter_ints(cfg->batch, cfg->n_kv_heads) * 4;
    if (cudaMemsetAsync(ws, 0, zero_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return KVQ_ERR_LAUNCH;
    return kvq_decode_attn(cfg, layer, q, q_dtype, d_len, max_len_host, softmax_scale, out,
                           out_dtype, ws, kScratchBytes, num_ctas, nullptr, nullptr, 0, stream);
}

extern "C" int kvq_noalloc_status(int32_t *status, kvq_stream_t stream)
{
    if (!status) return KVQ_ERR_INVALID_ARG;
    void *ws = nullptr;
    const int rc = scratch_address(&ws);
    if (rc) return rc;
    return kvq_workspace_status(ws, status, stream);
}

extern "C" int kvq_selftest_noalloc_timeout(const kvq_config *cfg, const kvq_layer *layer,
                                            const void *q, int32_t q_dtype, const int32_t *d_len,
                                            void *out, int32_t out_dtype, uint64_t timeout_ns,
                                            kvq_stream_t stream)
{
    if (!cfg || cfg->mode != KVQ_MODE_KV) return KVQ_ERR_INVALID_ARG;
    uint64_t need = 0;
    int rc = kvq_workspace_bytes(cfg, 0, &need);
    if (rc) return rc;
    if (need > kScratchBytes) return KVQ_ERR_WORKSPACE;
    void *ws = nullptr;
    rc = scratch_address(&ws);
    if (rc) return rc;
    // the same clearing as a regular call, then the decode kernel whose producer
    // copies nothing: every consumer wait runs out and the kernel records
    // KVQ_ERR_TIMEOUT in the array's status word
    const uint64_t zero_bytes = (uint64_t)kvq::kWorkspaceHeaderFloats * 4 +
                                kvq::counter_ints(cfg->batch, cfg->n_kv_heads) * 4;
    if (cudaMemsetAsync(ws, 0, zero_bytes, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return KVQ_ERR_LAUNCH;
    return kvq_selftest_decode_timeout(cfg, layer, q, q_dtype, d_len, out, out_dtype, ws,
                                       kScratchBytes, timeout_ns, stream);
}
