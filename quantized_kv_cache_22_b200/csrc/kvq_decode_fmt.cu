// kvq_decode_fmt.cu -- decode kernel instances for the 8-bit code formats other
// than symmetric integers: FP8 e4m3, asymmetric (uint8 + zero-point) and
// per-tensor INT8 keys and values.
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace {

template <int DH, int FMT, bool KG, bool VG>
void *fn()
{
    return reinterpret_cast<void *>(&decode_kernel<DH, 8, 8, KG, VG, FMT>);
}

template <int DH, int FMT>
void *by_kg(bool kg, bool vg)
{
    if constexpr (FMT == KVQ_FMT_TENSOR) {
        return (kg || vg) ? nullptr : fn<DH, FMT, false, false>();   // one scale per tensor
    } else {
        if (kg) return vg ? fn<DH, FMT, true, true>() : fn<DH, FMT, true, false>();
        return vg ? fn<DH, FMT, false, true>() : fn<DH, FMT, false, false>();
    }
}

template <int DH>
void *by_fmt(int fmt, bool kg, bool vg)
{
    switch (fmt) {
    case KVQ_FMT_E4M3: return by_kg<DH, KVQ_FMT_E4M3>(kg, vg);
    case KVQ_FMT_ASYM: return by_kg<DH, KVQ_FMT_ASYM>(kg, vg);
    case KVQ_FMT_TENSOR: return by_kg<DH, KVQ_FMT_TENSOR>(kg, vg);
    default: return nullptr;
    }
}

}  // namespace

void *decode_fn_fmt(int dh, int fmt, bool kg, bool vg)
{
    if (dh == 128) return by_fmt<128>(fmt, kg, vg);
    if (dh == 64) return by_fmt<64>(fmt, kg, vg);
    return nullptr;
}

}  // namespace kvq
