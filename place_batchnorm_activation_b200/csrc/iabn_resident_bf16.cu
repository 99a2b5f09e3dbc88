// iabn_resident_bf16.cu -- instantiations of the resident-plan kernels for
// bf16 storage (one file per storage type so they compile in parallel).
#include "iabn_resident.cuh"

namespace iabn {

cudaError_t launch_resident_bf16(const ResArgs& a, int layout, int cpt, int act, int dir,
                               int smem_optin, cudaStream_t s) {
    if (dir == 0) return launch_resident_dir<kBF16, 0>(a, layout, cpt, act, smem_optin, s);
    return launch_resident_dir<kBF16, 1>(a, layout, cpt, act, smem_optin, s);
}

}  // namespace iabn
