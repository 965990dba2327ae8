// kvq_quant.cuh -- warp-collective quantisation of one cache row, shared by the
// append kernel and the append step fused into the decode kernel.
//
// TinyLoop docs "KV Cache 模式", modes table: INT8 codes with one fp16 scale
// per head, INT4 nibble-packed with 15 symmetric levels (INT8: 255).  KVSplit:
// keys and values at independent widths, scales per group of elements.  The
// warp walks the row in chunks of 128 elements, four per lane; a scale group
// spans group/4 lanes and its absmax is a butterfly shuffle reduction.
// Divisions are IEEE (__fdiv_rn) and code rounding is round-to-nearest-even
// (__float2int_rn), so codes and scales match an IEEE reference bit for bit.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "../../include/kvq.h"

namespace kvq {

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

// Quantise `dim` elements of x, starting at element `in_off` (dtype KVQ_F16 /
// F32 / BF16, 16-byte aligned rows), into one cache row: `codes_row` is the
// row's first byte (dim*bits/8 bytes; at 16 bits the row holds fp16 values)
// and `scales_row` its first fp16 scale (dim/group of them; unused at 16 bits).
// Scale s = fp16(absmax / qmax) with qmax 127 (8 bits) or 7 (4 bits), an
// overflow to +inf saturating to 65504; code = clamp(rne(x / s), -qmax, qmax),
// all codes 0 when s = 0.  4-bit element 2j sits in the low nibble of byte j.
// fmt (8 bits only, else KVQ_FMT_INT):
//   KVQ_FMT_E4M3: s = fp16(absmax / 448) and code = e4m3(x / s), rounded to
//     nearest even and saturating at 448.
//   KVQ_FMT_ASYM: lo = min(0, min x), hi = max(0, max x), s = fp16((hi - lo) / 255),
//     z = clamp(rne(-lo / s), 0, 255), code = clamp(rne(x / s) + z, 0, 255) as a
//     uint8; the group's scale pair is (s, fp16(z)) (scales_row holds 2 per group).
//   KVQ_FMT_TENSOR: s = scales_row[0], the tensor's fixed scale (read, never
//     written), code = clamp(rne(x / s), -127, 127).
// All 32 lanes of the warp must call it with the same arguments.
__device__ __forceinline__ void quantize_row(const void *x, int64_t in_off, int dtype, int dim,
                                             int bits, int group, uint8_t *codes_row,
                                             __half *scales_row, int lane, int fmt = KVQ_FMT_INT)
{
    const bool e4m3 = fmt == KVQ_FMT_E4M3;
    const int lanes_per_group = group >> 2;
    for (int base = 0; base < dim; base += 128) {
        const int e0 = base + lane * 4;
        const bool active = e0 < dim;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (active) load4(x, in_off + e0, dtype, v);

        if (bits == 16) {
            if (active) {
                __half2 lo = __floats2half2_rn(v[0], v[1]);
                __half2 hi = __floats2half2_rn(v[2], v[3]);
                uint2 w;
                w.x = *reinterpret_cast<uint32_t *>(&lo);
                w.y = *reinterpret_cast<uint32_t *>(&hi);
                *reinterpret_cast<uint2 *>(codes_row + (int64_t)e0 * 2) = w;
            }
            continue;
        }

        if (fmt == KVQ_FMT_ASYM) {
            float lo = fminf(fminf(fminf(v[0], v[1]), fminf(v[2], v[3])), 0.0f);
            float hi = fmaxf(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])), 0.0f);
            for (int off = 1; off < lanes_per_group; off <<= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
            }
            __half s16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 255.0f));
            if (__half_as_ushort(s16) == 0x7c00u) s16 = __ushort_as_half(0x7bffu);
            const float s = __half2float(s16);
            int z = 0;
            if (s != 0.0f) z = max(0, min(255, __float2int_rn(__fdiv_rn(-lo, s))));
            if (active) {
                uint32_t w = 0;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int q = s != 0.0f ? max(0, min(255, __float2int_rn(__fdiv_rn(v[i], s)) + z)) : 0;
                    w |= (uint32_t)q << (8 * i);
                }
                *reinterpret_cast<uint32_t *>(codes_row + e0) = w;
                if ((lane % lanes_per_group) == 0) {
                    scales_row[2 * (e0 / group)] = s16;
                    scales_row[2 * (e0 / group) + 1] = __int2half_rn(z);
                }
            }
            continue;
        }
        if (fmt == KVQ_FMT_TENSOR) {
            const float s = __half2float(scales_row[0]);
            if (active) {
                uint32_t w = 0;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int q = s != 0.0f ? max(-127, min(127, __float2int_rn(__fdiv_rn(v[i], s)))) : 0;
                    w |= (uint32_t)(q & 0xff) << (8 * i);
                }
                *reinterpret_cast<uint32_t *>(codes_row + e0) = w;
            }
            continue;
        }

        const int qmax = (bits == 8) ? 127 : 7;
        float a = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
        for (int off = 1; off < lanes_per_group; off <<= 1)
            a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
        const float s32 = __fdiv_rn(a, e4m3 ? 448.0f : (float)qmax);
        __half s16 = __float2half_rn(s32);
        if (__half_as_ushort(s16) == 0x7c00u) s16 = __ushort_as_half(0x7bffu);
        const float s = __half2float(s16);

        if (e4m3) {
            if (active) {
                uint32_t w = 0;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const uint32_t c = s != 0.0f
                        ? (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(v[i], s), __NV_SATFINITE, __NV_E4M3)
                        : 0u;
                    w |= c << (8 * i);
                }
                *reinterpret_cast<uint32_t *>(codes_row + e0) = w;
                if ((lane % lanes_per_group) == 0) scales_row[e0 / group] = s16;
            }
            continue;
        }

        int c[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            int q = 0;
            if (s != 0.0f) {
                q = __float2int_rn(__fdiv_rn(v[i], s));
                q = max(-qmax, min(qmax, q));
            }
            c[i] = q;
        }
        if (!active) continue;
        if (bits == 8) {
            const uint32_t w = (uint32_t)(c[0] & 0xff) | ((uint32_t)(c[1] & 0xff) << 8) |
                               ((uint32_t)(c[2] & 0xff) << 16) | ((uint32_t)(c[3] & 0xff) << 24);
            *reinterpret_cast<uint32_t *>(codes_row + e0) = w;
        } else {
            const uint32_t w = (uint32_t)(c[0] & 0xf) | ((uint32_t)(c[1] & 0xf) << 4) |
                               ((uint32_t)(c[2] & 0xf) << 8) | ((uint32_t)(c[3] & 0xf) << 12);
            *reinterpret_cast<uint16_t *>(codes_row + e0 / 2) = (uint16_t)w;
        }
        if ((lane % lanes_per_group) == 0) scales_row[e0 / group] = s16;
    }
}

}  // namespace kvq
