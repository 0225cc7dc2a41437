// tc_forward.cu -- tensor-core (tcgen05) path of the Mesa layer forward.
// Placeholder until the sm_100a kernels land: no shape is routed here yet.
#include "mesa_common.cuh"
#include "mesa_internal.h"

namespace mesa {

bool tc_supported(int, int, int, mesa_dtype) { return false; }
size_t tc_workspace_bytes(int, int, int) { return 0; }
cudaError_t forward_tc(const ForwardArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace mesa
