// common.cuh — shared device helpers of the SSD library (I/O types, status word).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/ssd.h"

namespace ssd {

// Device status word: 0 = fine, otherwise the code of the first bounded wait
// that gave up (set with atomicCAS so the first cause is kept).
enum DeviceStatus : unsigned int {
    kDevOk = 0,
    kDevWaitTimeout = 1,
};

// The word lives in api.cu; kernels receive its device address as an argument
// (one translation unit per kernel family, no relocatable device code).
__device__ __forceinline__ void record_status(unsigned int* status, unsigned int code)
{
    if (status) atomicCAS(status, 0u, code);
}

// I/O element access: fp32 or bf16 storage, fp32 arithmetic.
template <typename T> struct io;
template <> struct io<float> {
    static __device__ __forceinline__ float load(const float* p) { return __ldg(p); }
    static __device__ __forceinline__ void store(float* p, float v) { *p = v; }
};
template <> struct io<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p)
    {
        return __bfloat162float(__ldg(p));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float v)
    {
        *p = __float2bfloat16_rn(v);
    }
};

// Per-call context every launcher receives from api.cu.
struct LaunchCtx {
    cudaStream_t stream;
    unsigned int* status;        // device status word
    unsigned long long wait_limit;  // iterations of a bounded device wait
    int num_sms;
    // Tag of this call, never 0. The control words a call keeps in its
    // workspace (look-back flags, ticket counter) are 64-bit values whose high
    // half is the tag of the call that wrote them, so whatever an earlier call
    // of any path or size left there reads as not yet written: a workspace
    // needs no clearing, before its first use or between calls.
    uint32_t epoch;
};

// Control word of this call: (epoch, count).
__host__ __device__ __forceinline__ unsigned long long tagged(uint32_t epoch, uint32_t count)
{
    return (static_cast<unsigned long long>(epoch) << 32) | count;
}

// Takes the next value of a per-call counter kept as a tagged word: the first
// taker of a call finds another call's tag (or garbage) and restarts the count
// at 0 for this call.
__device__ __forceinline__ unsigned int take_ticket(unsigned long long* ctr, uint32_t epoch)
{
    unsigned long long cur = atomicAdd(ctr, 0ull);
    for (;;) {
        const bool mine = static_cast<uint32_t>(cur >> 32) == epoch;
        const unsigned long long want = mine ? cur + 1ull : tagged(epoch, 1u);
        const unsigned long long prev = atomicCAS(ctr, cur, want);
        if (prev == cur) return mine ? static_cast<unsigned int>(cur) : 0u;
        cur = prev;
    }
}

}  // namespace ssd

namespace ssd {

// Arguments of one forward call as the launchers see them (pointers are device
// pointers; x, Bm, Cm, y are in the I/O dtype named by `bf16`).
struct FwdArgs {
    const void* x;
    const float* dt;
    const float* A;
    const void* Bm;
    const void* Cm;
    const float* D;         // may be null
    const float* init;      // may be null
    void* y;
    float* final_state;     // may be null
    int B, L, H, P, G, N, chunk;
    bool bf16;
};

struct StepArgs {
    const void* x;
    const float* dt;
    const float* A;
    const void* Bm;
    const void* Cm;
    const float* D;
    float* state;
    void* y;
    int B, H, P, G, N;
    bool bf16;
};

// SIMT path (simt_forward.cu): any valid size, fp32 arithmetic.
size_t simt_workspace_bytes(const FwdArgs& a);
cudaError_t simt_forward(const FwdArgs& a, void* workspace, const LaunchCtx& ctx);

// Device status word, stream and limits for a launch on the current device
// (api.cu).
ssd_status acquire_launch_ctx(cudaStream_t stream, LaunchCtx* ctx);

// Size checks of every entry point: SSD_OK or the status to return (api.cu).
ssd_status check_dims(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype);

// Decode step (step.cu).
cudaError_t step_forward(const StepArgs& a, const LaunchCtx& ctx);

}  // namespace ssd
