// kvq_decode_pk8.cu -- decode kernel instances with packed score columns (G <= 4,
// head_dim 128) for 8-bit keys: symmetric INT4 / INT8 values, per-tensor INT8, and FP8
// e4m3 and asymmetric INT8 keys and values (key scales per (token, head))
#include "kvq_decode_kernel.cuh"

namespace kvq {
namespace {

template <int VB, bool KG, bool VG, int FMT>
void *fn()
{
    return reinterpret_cast<void *>(&decode_kernel<128, 8, VB, KG, VG, FMT, true>);
}

template <int VB>
void *by_kg(bool kg, bool vg)
{
    if (kg) return vg ? fn<VB, true, true, KVQ_FMT_INT>() : fn<VB, true, false, KVQ_FMT_INT>();
    return vg ? fn<VB, false, true, KVQ_FMT_INT>() : fn<VB, false, false, KVQ_FMT_INT>();
}

}  // namespace

void *decode_fn_pk_kb8(int vb, bool kg, bool vg, int fmt)
{
    if (fmt == KVQ_FMT_TENSOR)
        return (vb == 8 && !kg && !vg) ? fn<8, false, false, KVQ_FMT_TENSOR>() : nullptr;
    if (fmt == KVQ_FMT_ASYM) {
        if (vb != 8 || kg) return nullptr;
        return vg ? fn<8, false, true, KVQ_FMT_ASYM>() : fn<8, false, false, KVQ_FMT_ASYM>();
    }
    if (fmt == KVQ_FMT_E4M3) {
        if (vb != 8 || kg) return nullptr;
        return vg ? fn<8, false, true, KVQ_FMT_E4M3>() : fn<8, false, false, KVQ_FMT_E4M3>();
    }
    if (fmt != KVQ_FMT_INT) return nullptr;
    switch (vb) {
    case 4: return by_kg<4>(kg, vg);
    case 8: return by_kg<8>(kg, vg);
    default: return nullptr;
    }
}

}  // namespace kvq
