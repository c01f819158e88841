// chunk_fused.cu -- KF: the fused chunk-sweep kernel (tcgen05, sm_100a).
#include "ssd_device.cuh"
#include "ssd_kernels.h"

namespace ssd {

bool fused_path_available() { return false; }

cudaError_t launch_chunk_fused(const Shape&, const FwdArgs&, const void*, const float*,
                               const float*, int*, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace ssd
