// kvq_append.cu -- quantize-on-append.
//
// TinyLoop docs "KV Cache 模式", modes table: INT8 codes with one fp16 scale
// per head, INT4 nibble-packed with 15 symmetric levels (INT8: 255).  KVSplit:
// keys and values at independent widths.  One warp quantises one row (one
// token of one KV head, or one token's h vector) in chunks of 128 elements,
// four per lane; a scale group spans group/4 lanes and its absmax is a
// butterfly shuffle reduction.  Divisions are IEEE (__fdiv_rn) and code
// rounding is round-to-nearest-even (__float2int_rn), so codes and scales
// match an IEEE reference bit for bit.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"
#include "../../include/kvq.h"

namespace kvq {
namespace {

__device__ __forceinline__ void load4(const void *base, int64_t idx, int dtype, float (&x)[4])
{
    if (dtype == KVQ_F32) {
        const float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(base) + idx);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else if (dtype == KVQ_F16) {
        const uint2 v = *reinterpret_cast<const uint2 *>(static_cast<const __half *>(base) + idx);
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
        const uint2 v =
            *reinterpret_cast<const uint2 *>(static_cast<const __nv_bfloat16 *>(base) + idx);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    }
}

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
    const int pos = p.d_pos[b] + j;
    if (pos < 0 || pos >= p.cap) return;  // the kernel's own bounds check

    const int dim = p.dim;
    const int64_t in_row = row * (int64_t)dim;
    const int64_t cache_row = ((int64_t)b * p.rows_per_tok + head) * p.cap + pos;
    const int lanes_per_group = p.group >> 2;

    for (int base = 0; base < dim; base += 128) {
        const int e0 = base + lane * 4;
        const bool active = e0 < dim;
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (active) load4(p.x, in_row + e0, p.in_dtype, x);

        if (p.bits == 16) {
            if (active) {
                __half2 lo = __floats2half2_rn(x[0], x[1]);
                __half2 hi = __floats2half2_rn(x[2], x[3]);
                uint2 v;
                v.x = *reinterpret_cast<uint32_t *>(&lo);
                v.y = *reinterpret_cast<uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(p.codes + (cache_row * dim + e0) * 2) = v;
            }
            continue;
        }

        const int qmax = (p.bits == 8) ? 127 : 7;
        float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
        for (int off = 1; off < lanes_per_group; off <<= 1)
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        const float s32 = __fdiv_rn(a, (float)qmax);
        __half s16 = __float2half_rn(s32);
        if (__half_as_ushort(s16) == 0x7c00u) s16 = __ushort_as_half(0x7bffu);
        const float s = __half2float(s16);

        int c[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            int v = 0;
            if (s != 0.0f) {
                v = __float2int_rn(__fdiv_rn(x[i], s));
                v = max(-qmax, min(qmax, v));
            }
            c[i] = v;
        }
        if (!active) continue;
        if (p.bits == 8) {
            const uint32_t w = (uint32_t)(c[0] & 0xff) | ((uint32_t)(c[1] & 0xff) << 8) |
                               ((uint32_t)(c[2] & 0xff) << 16) | ((uint32_t)(c[3] & 0xff) << 24);
            *reinterpret_cast<uint32_t *>(p.codes + cache_row * dim + e0) = w;
        } else {
            const uint32_t w = (uint32_t)(c[0] & 0xf) | ((uint32_t)(c[1] & 0xf) << 4) |
                               ((uint32_t)(c[2] & 0xf) << 8) | ((uint32_t)(c[3] & 0xf) << 12);
            *reinterpret_cast<uint16_t *>(p.codes + cache_row * (dim / 2) + e0 / 2) = (uint16_t)w;
        }
        if ((lane % lanes_per_group) == 0)
            p.scales[cache_row * (dim / p.group) + e0 / p.group] = s16;
    }
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
