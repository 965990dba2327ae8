// kvq_append.cu -- quantize-on-append.
//
// One warp quantises one row (one token of one KV head, or one token's h
// vector) with the row quantiser of kvq_quant.cuh (TinyLoop docs "KV Cache
// 模式" modes table; KVSplit independent key/value widths and groups).  With a
// sliding window (on-device page, "Sliding Window Eviction": recent tokens
// plus anchors) a token goes to its ring slot; in a paged cache to its slot of
// the pool page the block table names.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"
#include "kvq_quant.cuh"
#include "../../include/kvq.h"

namespace kvq {
namespace {

struct AppendPair {
    AppendParams t[2];
};

__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ AppendPair pp, int ntensor)
{
    const int lane = threadIdx.x & 31;
    const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t rows = (int64_t)pp.t[0].batch * pp.t[0].n_new * pp.t[0].rows_per_tok;
    if (gw >= rows * ntensor) return;
    const AppendParams &p = pp.t[ntensor == 2 ? (int)(gw & 1) : 0];
    const int64_t row = (ntensor == 2) ? gw / 2 : gw;

    const int head = (int)(row % p.rows_per_tok);
    const int64_t bj = row / p.rows_per_tok;
    const int j = (int)(bj % p.n_new);
    const int b = (int)(bj / p.n_new);
    const int first = p.d_pos[b];
    const int pos = first + j;
    if (pos < 0) return;
    int slot = pos;
    if (p.window > 0) {
        // a token that a later token of this call overwrites in the ring is skipped
        if (pos >= p.n_anchor && pos + p.window <= first + p.n_new - 1) return;
        slot = cache_slot(pos, p.window, p.n_anchor);
    }
    if (slot >= p.cap) return;  // the kernel's own bounds checks

    const int dim = p.dim;
    int64_t cache_row;
    if (p.block_table != nullptr) {
        // paged: slot pos % 128 of the pool page holding logical page pos / 128
        const int page = p.block_table[(int64_t)b * p.max_pages + pos / kPageTokens];
        if (page < 0 || page >= p.n_pages) return;
        cache_row = ((int64_t)page * p.rows_per_tok + head) * kPageTokens + pos % kPageTokens;
    } else {
        cache_row = ((int64_t)b * p.rows_per_tok + head) * p.cap + slot;
    }
    uint8_t *codes_row = p.codes + cache_row * ((int64_t)dim * p.bits / 8);
    __half *scales_row = p.bits == 16            ? nullptr
                         : p.fmt == KVQ_FMT_TENSOR ? p.scales   // the tensor's one scale
                                                   : p.scales + cache_row * (dim / p.group) * scale_vals(p.fmt);
    quantize_row(p.x, row * (int64_t)dim, p.in_dtype, dim, p.bits, p.group, codes_row, scales_row,
                 lane, p.fmt);
}

}  // namespace

cudaError_t launch_append(const AppendParams &k, const AppendParams *v, cudaStream_t stream)
{
    const int ntensor = v ? 2 : 1;
    const int64_t warps = (int64_t)k.batch * k.n_new * k.rows_per_tok * ntensor;
    if (warps == 0) return cudaSuccess;
    const int64_t blocks = (warps + 7) / 8;
    if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
    AppendPair pp;
    pp.t[0] = k;
    pp.t[1] = v ? *v : k;
    (void)cudaGetLastError();  // drop a stale, already-reported error of an earlier call
    append_kernel<<<(unsigned)blocks, 256, 0, stream>>>(pp, ntensor);
    return cudaGetLastError();
}

}  // namespace kvq
