// kvq_decode_k4.cu -- decode kernel instances with 4-bit keys.
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace {

template <int DH, int VB, bool KG, bool VG>
void *fn()
{
    return reinterpret_cast<void *>(&decode_kernel<DH, 4, VB, KG, VG, KVQ_FMT_INT>);
}

template <int DH, int VB, bool KG>
void *by_vg(bool vg)
{
    if constexpr (VB == 16) {
        return vg ? nullptr : fn<DH, VB, KG, false>();
    } else {
        return vg ? fn<DH, VB, KG, true>() : fn<DH, VB, KG, false>();
    }
}

template <int DH, int VB>
void *by_kg(bool kg, bool vg)
{
    return kg ? by_vg<DH, VB, true>(vg) : by_vg<DH, VB, false>(vg);
}

template <int DH>
void *by_vb(int vb, bool kg, bool vg)
{
    switch (vb) {
    case 4: return by_kg<DH, 4>(kg, vg);
    case 8: return by_kg<DH, 8>(kg, vg);
    case 16: return by_kg<DH, 16>(kg, vg);
    default: return nullptr;
    }
}

}  // namespace

void *decode_fn_kb4(int dh, int vb, bool kg, bool vg)
{
    if (dh == 128) return by_vb<128>(vb, kg, vg);
    if (dh == 64) return by_vb<64>(vb, kg, vg);
    return nullptr;
}

}  // namespace kvq
