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

    // Tag of the i-th launch of this call (i < 8): each launch of a call that
    // runs several (two passes over the state columns) keeps its own tag, so
    // it never reads the flags an earlier launch of the same call set.
    __host__ __device__ uint32_t launch_tag(int i) const
    {
        const uint32_t t = epoch * 8u + static_cast<uint32_t>(i);
        return t ? t : 1u;
    }
};

// Control word of this call: (epoch, count).
__host__ __device__ __forceinline__ unsigned long long tagged(uint32_t epoch, uint32_t count)
{
    return (static_cast<unsigned long long>(epoch) << 32) | count;
}

// Takes the next value of a per-call counter. The word holds the count in
// its high half and the call's tag in its low half, so the common case is one
// atomicAdd (an add never carries into the tag). The first takers of a call
// find another call's tag (or garbage): one of them installs this call's tag
// with count 1 and keeps ticket 0, the others see the new tag and add again.
// Unlike a compare-and-swap loop, every call costs a bounded number of round
// trips to L2, however many CTAs take their ticket at the same moment.
__device__ __forceinline__ unsigned int take_ticket(unsigned long long* ctr, uint32_t epoch)
{
    constexpr unsigned long long kOne = 1ull << 32;
    unsigned long long old = atomicAdd(ctr, kOne);
    for (;;) {
        if (static_cast<uint32_t>(old) == epoch) return static_cast<unsigned int>(old >> 32);
        unsigned long long cur = old + kOne;  // the word after our add, if no one else added
        for (;;) {
            const unsigned long long prev = atomicCAS(ctr, cur, kOne | epoch);
            if (prev == cur) return 0u;
            if (static_cast<uint32_t>(prev) == epoch) break;  // installed by another taker
            cur = prev;
        }
        old = atomicAdd(ctr, kOne);
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
