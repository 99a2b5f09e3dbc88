// iabn_resident.cu -- resident plan (placeholder until the co-resident
// kernels land): reports every shape as unsupported so the two-phase plan runs.
#include "iabn_device.cuh"
#include "iabn_internal.h"

namespace iabn {

bool resident_supported(const Geom&) { return false; }

cudaError_t forward_resident(const Geom&, const FwdArgs&, const Workspace&, cudaStream_t) {
    return cudaErrorNotSupported;
}

cudaError_t backward_resident(const Geom&, const BwdArgs&, const Workspace&, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace iabn
