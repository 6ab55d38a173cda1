// grouped_forward.cuh — launcher interface of the head-group tensor-core
// forward (grouped_forward.cu).
#pragma once
#include "common.cuh"

namespace ssd {
namespace grouped {

// True when the kernel handles these sizes (bf16, P a multiple of 64, N <= 128).
bool supported(const FwdArgs& a);
// True when it is the faster of the tensor-core forms for these sizes on a
// GPU with `ctas` SMs.
bool preferred(const FwdArgs& a, int ctas);
size_t workspace_bytes(const FwdArgs& a, int ctas);
cudaError_t forward(const FwdArgs& a, void* workspace, const LaunchCtx& ctx);
// Test hook: when nonzero, segments never publish their end state.
void set_skip_publish(int v);

}  // namespace grouped
}  // namespace ssd
