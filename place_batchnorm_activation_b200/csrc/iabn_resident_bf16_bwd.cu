// iabn_resident_bf16_bwd.cu -- instantiations of the resident-plan backward
// kernels for bf16 storage (one file per storage type and direction, so they
// compile in parallel).
#include "iabn_resident.cuh"

namespace iabn {

cudaError_t launch_resident_bf16_bwd(const ResArgs& a, int layout, int cpt, int act, int mode,
                                 int smem_optin, cudaStream_t s) {
    if (mode == kModeBwdZ) return launch_resident_mode<kBF16, kModeBwdZ>(a, layout, cpt, act, smem_optin, s);
    if (mode == kModeBwdX) return launch_resident_mode<kBF16, kModeBwdX>(a, layout, cpt, act, smem_optin, s);
    if (mode == kModeBwdXhat)
        return launch_resident_mode<kBF16, kModeBwdXhat>(a, layout, cpt, act, smem_optin, s);
    return cudaErrorNotSupported;
}

}  // namespace iabn
