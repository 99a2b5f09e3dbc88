// iabn_resident_f32_fwd.cu -- instantiations of the resident-plan forward
// kernels for f32 storage (one file per storage type and direction, so they
// compile in parallel).
#include "iabn_resident.cuh"

namespace iabn {

cudaError_t launch_resident_f32_fwd(const ResArgs& a, int layout, int cpt, int act, int mode,
                                 int smem_optin, cudaStream_t s) {
    if (mode == kModeFwd) return launch_resident_mode<kF32, kModeFwd>(a, layout, cpt, act, smem_optin, s);
    if (mode == kModeFwdCkpt)
        return launch_resident_mode<kF32, kModeFwdCkpt>(a, layout, cpt, act, smem_optin, s);
    return cudaErrorNotSupported;
}

}  // namespace iabn
