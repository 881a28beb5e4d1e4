// Tensor-core (tcgen05) chunked prefill -- placeholder until the kernel lands.
#include "gdn_common.cuh"
#include "gdn_internal.h"

namespace gdn {

bool prefill_tc_supported(int, int, int, int) { return false; }
size_t prefill_tc_workspace(int, int, int, int64_t, int, int) { return 0; }
cudaError_t launch_prefill_tc(const PrefillArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace gdn
