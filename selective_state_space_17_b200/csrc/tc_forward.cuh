// tc_forward.cuh — launcher interface of the tensor-core (tcgen05) forward path.
#pragma once
#include "common.cuh"

namespace ssd {

// True when the bf16 tensor-core path handles these sizes.
bool tc_supported(const FwdArgs& a);
size_t tc_workspace_bytes(const FwdArgs& a);
cudaError_t tc_forward(const FwdArgs& a, void* workspace, const LaunchCtx& ctx);
int tc_kernel_count(const FwdArgs& a);
// True when the chains are cut into so many segments that the forward runs
// segment-parallel (local states, a scan, the outputs).
bool tc_segment_parallel(const FwdArgs& a);
// Test hook: when nonzero, tiles never publish their end state, so every
// look-back wait runs into its iteration limit.
void tc_set_skip_publish(int v);

}  // namespace ssd
