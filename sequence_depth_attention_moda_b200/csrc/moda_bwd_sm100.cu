// moda_bwd_sm100.cu -- backward launcher for the bf16 path.
#include "moda_internal.h"

namespace moda {

cudaError_t launch_bwd_sm100(const Problem& p, const void* Q, const void* K, const void* V,
                             const void* Kd, const void* Vd, const void* O, const float* LSE,
                             const void* dO, void* dQ, void* dK, void* dV, void* dKd, void* dVd,
                             float* Dws, cudaStream_t stream) {
    return launch_bwd_simt(p, Q, K, V, Kd, Vd, O, LSE, dO, dQ, dK, dV, dKd, dVd, Dws, stream);
}

}  // namespace moda
