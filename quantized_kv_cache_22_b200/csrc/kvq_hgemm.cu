// kvq_hgemm.cu -- h-mode K/V reconstruction GEMM (tcgen05).  Not built yet:
// the launcher reports cudaErrorNotSupported, which the ABI maps to
// KVQ_ERR_UNSUPPORTED.
#include "kvq_internal.h"

namespace kvq {

cudaError_t launch_h_reconstruct(const HGemmParams &, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace kvq
