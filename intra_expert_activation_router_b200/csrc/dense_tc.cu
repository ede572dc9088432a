// dense_tc.cu -- dense tensor-core (tcgen05) grouped-GEMM path.
#include "internal.h"

namespace moe {

bool dense_path_available() { return false; }

cudaError_t launch_dense(const Dims &, const DeviceWeights &, const Workspace &, const uint16_t *,
                         int, float, bool, uint16_t *, int, cudaStream_t)
{
    return cudaErrorNotSupported;
}

}  // namespace moe
