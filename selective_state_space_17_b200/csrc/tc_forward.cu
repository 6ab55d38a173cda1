// tc_forward.cu — tensor-core forward path (placeholder until the kernel lands).
#include "tc_forward.cuh"

namespace ssd {

bool tc_supported(const FwdArgs&) { return false; }
size_t tc_workspace_bytes(const FwdArgs&) { return 0; }
cudaError_t tc_forward(const FwdArgs&, void*, const LaunchCtx&) { return cudaErrorNotSupported; }
int tc_kernel_count(const FwdArgs&) { return 0; }

}  // namespace ssd
