// iabn_resident_f16.cu -- instantiations of the resident-plan kernels for
// f16 storage (one file per storage type so they compile in parallel).
#include "iabn_resident.cuh"

namespace iabn {

cudaError_t launch_resident_f16(const ResArgs& a, int layout, int cpt, int act, int dir,
                               int smem_optin, cudaStream_t s) {
    if (dir == 0) return launch_resident_dir<kF16, 0>(a, layout, cpt, act, smem_optin, s);
    return launch_resident_dir<kF16, 1>(a, layout, cpt, act, smem_optin, s);
}

}  // namespace iabn
