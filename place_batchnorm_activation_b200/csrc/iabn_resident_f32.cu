// iabn_resident_f32.cu -- instantiations of the resident-plan kernels for
// f32 storage (one file per storage type so they compile in parallel).
#include "iabn_resident.cuh"

namespace iabn {

cudaError_t launch_resident_f32(const ResArgs& a, int layout, int cpt, int act, int dir,
                               int smem_optin, cudaStream_t s) {
    if (dir == 0) return launch_resident_dir<kF32, 0>(a, layout, cpt, act, smem_optin, s);
    return launch_resident_dir<kF32, 1>(a, layout, cpt, act, smem_optin, s);
}

}  // namespace iabn
