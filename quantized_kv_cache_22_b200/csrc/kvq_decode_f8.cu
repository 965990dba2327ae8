// kvq_decode_f8.cu -- decode kernel instances with FP8 e4m3 keys and values.
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace {

template <int DH, bool KG, bool VG>
void *fn()
{
    return reinterpret_cast<void *>(&decode_kernel<DH, 8, 8, KG, VG, true>);
}

template <int DH>
void *by_kg(bool kg, bool vg)
{
    if (kg) return vg ? fn<DH, true, true>() : fn<DH, true, false>();
    return vg ? fn<DH, false, true>() : fn<DH, false, false>();
}

}  // namespace

void *decode_fn_f8(int dh, bool kg, bool vg)
{
    if (dh == 128) return by_kg<128>(kg, vg);
    if (dh == 64) return by_kg<64>(kg, vg);
    return nullptr;
}

}  // namespace kvq
