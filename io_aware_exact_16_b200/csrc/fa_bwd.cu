// fa_bwd.cu -- backward kernels (placeholder until the fused kernel lands).
#include "fa_internal.h"

namespace fa {
cudaError_t launch_bwd(int, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                       const CUtensorMap&, const CUtensorMap&, const BwdParams&, int, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace fa
