// api.cu — the C ABI of libssd_b200.so: argument checks, workspace sizing,
// dispatch to the kernel families, the device status word and the host-buffer
// entry point. Declarations and contracts are in include/ssd.h.
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "tc_forward.cuh"

namespace ssd {

__device__ unsigned int g_device_status;

namespace {

constexpr unsigned long long kDefaultWaitLimit = 1ull << 23;  // ~seconds of polling
constexpr int kMaxDevices = 64;

unsigned long long g_wait_limit = kDefaultWaitLimit;
std::mutex g_mu;
unsigned int* g_status_ptr[kMaxDevices];
int g_num_sms[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ssd_status make_ctx(cudaStream_t stream, LaunchCtx* ctx)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSD_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return SSD_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SSD_ERR_CUDA;
        g_status_ptr[dev] = static_cast<unsigned int*>(p);
        g_num_sms[dev] = sms;
    }
    ctx->stream = stream;
    ctx->status = g_status_ptr[dev];
    ctx->wait_limit = g_wait_limit;
    ctx->num_sms = g_num_sms[dev];
    return SSD_OK;
}

ssd_status check_dims(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype)
{
    if (B < 0 || L < 0 || H < 1 || G < 1 || P < 1 || N < 1 || chunk < 1) return SSD_ERR_INVALID_ARG;
    if (H % G != 0) return SSD_ERR_INVALID_ARG;
    if (dtype != SSD_F32 && dtype != SSD_BF16) return SSD_ERR_INVALID_ARG;
    if (P > 256 || N > 256 || chunk > 256) return SSD_ERR_UNSUPPORTED;
    // index arithmetic is 64-bit; keep per-dimension products inside int
    if ((long long)B * L > (1ll << 31) - 1 || (long long)H * P > (1 << 20) ||
        (long long)G * N > (1 << 20))
        return SSD_ERR_UNSUPPORTED;
    return SSD_OK;
}

FwdArgs make_args(const void* x, const float* dt, const float* A, const void* Bm, const void* Cm,
                  const float* D, const float* init, void* y, float* fs, int B, int L, int H,
                  int P, int G, int N, int chunk, ssd_dtype dtype)
{
    FwdArgs a;
    a.x = x; a.dt = dt; a.A = A; a.Bm = Bm; a.Cm = Cm; a.D = D; a.init = init; a.y = y;
    a.final_state = fs;
    a.B = B; a.L = L; a.H = H; a.P = P; a.G = G; a.N = N; a.chunk = chunk;
    a.bf16 = dtype == SSD_BF16;
    return a;
}

size_t round_up(size_t v, size_t m) { return (v + m - 1) / m * m; }

size_t workspace_bytes(const FwdArgs& a)
{
    if (tc_supported(a)) return tc_workspace_bytes(a);
    return simt_workspace_bytes(a);
}

// B*L == 0: no tokens. final_state = initial_state (or zero).
ssd_status empty_forward(const FwdArgs& a, cudaStream_t stream)
{
    if (!a.final_state) return SSD_OK;
    const size_t bytes = (size_t)a.B * a.H * a.P * a.N * sizeof(float);
    if (bytes == 0) return SSD_OK;
    cudaError_t e = a.init ? cudaMemcpyAsync(a.final_state, a.init, bytes,
                                             cudaMemcpyDeviceToDevice, stream)
                           : cudaMemsetAsync(a.final_state, 0, bytes, stream);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

}  // namespace

ssd_status acquire_launch_ctx(cudaStream_t stream, LaunchCtx* ctx) { return make_ctx(stream, ctx); }

}  // namespace ssd

using namespace ssd;

extern "C" {

const char* ssd_status_string(ssd_status s)
{
    switch (s) {
    case SSD_OK: return "SSD_OK";
    case SSD_ERR_INVALID_ARG: return "SSD_ERR_INVALID_ARG: null pointer or invalid size";
    case SSD_ERR_UNSUPPORTED: return "SSD_ERR_UNSUPPORTED: size not handled by this build";
    case SSD_ERR_MISALIGNED: return "SSD_ERR_MISALIGNED: pointer not 16-byte aligned";
    case SSD_ERR_CUDA: return "SSD_ERR_CUDA: a CUDA call failed";
    case SSD_ERR_TIMEOUT: return "SSD_ERR_TIMEOUT: a bounded device-side wait gave up";
    case SSD_ERR_WORKSPACE: return "SSD_ERR_WORKSPACE: workspace missing or too small";
    }
    return "SSD_ERR_UNKNOWN";
}

size_t ssd_workspace_size(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype)
{
    if (check_dims(B, L, H, P, G, N, chunk, dtype) != SSD_OK) return 0;
    FwdArgs a = make_args(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                          nullptr, B, L, H, P, G, N, chunk, dtype);
    return round_up(workspace_bytes(a), 256) + 256;
}

ssd_status ssd_forward(const void* x, const float* dt, const float* A, const void* Bm,
                       const void* Cm, const float* D, const float* initial_state, void* y,
                       float* final_state, int B, int L, int H, int P, int G, int N, int chunk,
                       ssd_dtype dtype, void* workspace, size_t workspace_bytes_given,
                       ssd_stream_t stream)
{
    ssd_status st = check_dims(B, L, H, P, G, N, chunk, dtype);
    if (st != SSD_OK) return st;
    FwdArgs a = make_args(x, dt, A, Bm, Cm, D, initial_state, y, final_state, B, L, H, P, G, N,
                          chunk, dtype);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((long long)B * L == 0) {
        if (initial_state && !aligned16(initial_state)) return SSD_ERR_MISALIGNED;
        if (final_state && !aligned16(final_state)) return SSD_ERR_MISALIGNED;
        return empty_forward(a, s);
    }
    if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt, A, Bm, Cm, D, initial_state, y, final_state, workspace};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_MISALIGNED;
    const size_t need = ssd_workspace_size(B, L, H, P, G, N, chunk, dtype);
    if (!workspace || workspace_bytes_given < need) return SSD_ERR_WORKSPACE;
    LaunchCtx ctx;
    st = make_ctx(s, &ctx);
    if (st != SSD_OK) return st;
    cudaError_t e = tc_supported(a) ? tc_forward(a, workspace, ctx)
                                    : simt_forward(a, workspace, ctx);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

size_t ssd_forward_host_buffer_size(int B, int L, int H, int P, int G, int N, int chunk,
                                    ssd_dtype dtype)
{
    const size_t ws = ssd_workspace_size(B, L, H, P, G, N, chunk, dtype);
    if (ws == 0) return 0;
    const size_t es = dtype == SSD_BF16 ? 2 : 4;
    const size_t BL = (size_t)B * L;
    size_t total = ws;
    total += round_up(BL * H * P * es, 256) * 2;           // x, y
    total += round_up(BL * H * 4, 256);                    // dt
    total += round_up((size_t)H * 4, 256) * 2;             // A, D
    total += round_up(BL * G * N * es, 256) * 2;           // Bm, Cm
    total += round_up((size_t)B * H * P * N * 4, 256) * 2; // initial, final state
    return total;
}

ssd_status ssd_forward_host(const void* x_host, const float* dt_host, const float* A_host,
                            const void* Bm_host, const void* Cm_host, const float* D_host,
                            const float* initial_state_host, void* y_host,
                            float* final_state_host, int B, int L, int H, int P, int G, int N,
                            int chunk, ssd_dtype dtype, void* device_buffer,
                            size_t device_buffer_bytes, ssd_stream_t stream)
{
    ssd_status st = check_dims(B, L, H, P, G, N, chunk, dtype);
    if (st != SSD_OK) return st;
    const size_t need = ssd_forward_host_buffer_size(B, L, H, P, G, N, chunk, dtype);
    if (!device_buffer || device_buffer_bytes < need) return SSD_ERR_WORKSPACE;
    if (!aligned16(device_buffer)) return SSD_ERR_MISALIGNED;
    const size_t BL = (size_t)B * L;
    if (BL > 0 && (!x_host || !dt_host || !A_host || !Bm_host || !Cm_host || !y_host))
        return SSD_ERR_INVALID_ARG;
    const size_t es = dtype == SSD_BF16 ? 2 : 4;
    const size_t ws = ssd_workspace_size(B, L, H, P, G, N, chunk, dtype);
    char* p = static_cast<char*>(device_buffer);
    void* d_ws = p; p += ws;
    const size_t bx = BL * H * P * es, bdt = BL * H * 4, bbc = BL * G * N * es;
    const size_t bst = (size_t)B * H * P * N * 4;
    void* d_x = p; p += round_up(bx, 256);
    void* d_y = p; p += round_up(bx, 256);
    float* d_dt = reinterpret_cast<float*>(p); p += round_up(bdt, 256);
    float* d_A = reinterpret_cast<float*>(p); p += round_up((size_t)H * 4, 256);
    float* d_D = reinterpret_cast<float*>(p); p += round_up((size_t)H * 4, 256);
    void* d_B = p; p += round_up(bbc, 256);
    void* d_C = p; p += round_up(bbc, 256);
    float* d_init = reinterpret_cast<float*>(p); p += round_up(bst, 256);
    float* d_fs = reinterpret_cast<float*>(p);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto h2d = [&](void* dst, const void* src, size_t n) {
        return (n == 0 || !src) ? cudaSuccess
                                : cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s);
    };
    cudaError_t e = cudaSuccess;
    if (e == cudaSuccess) e = h2d(d_x, x_host, bx);
    if (e == cudaSuccess) e = h2d(d_dt, dt_host, bdt);
    if (e == cudaSuccess) e = h2d(d_A, A_host, (size_t)H * 4);
    if (e == cudaSuccess) e = h2d(d_D, D_host, (size_t)H * 4);
    if (e == cudaSuccess) e = h2d(d_B, Bm_host, bbc);
    if (e == cudaSuccess) e = h2d(d_C, Cm_host, bbc);
    if (e == cudaSuccess) e = h2d(d_init, initial_state_host, bst);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    st = ssd_forward(d_x, d_dt, d_A, d_B, d_C, D_host ? d_D : nullptr,
                     initial_state_host ? d_init : nullptr, d_y,
                     final_state_host ? d_fs : nullptr, B, L, H, P, G, N, chunk, dtype, d_ws, ws,
                     stream);
    if (st != SSD_OK) return st;
    if (BL > 0) e = cudaMemcpyAsync(y_host, d_y, bx, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess && final_state_host)
        e = cudaMemcpyAsync(final_state_host, d_fs, bst, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

ssd_status ssd_step(const void* x, const float* dt, const float* A, const void* Bm,
                    const void* Cm, const float* D, float* state, void* y, int B, int H, int P,
                    int G, int N, ssd_dtype dtype, ssd_stream_t stream)
{
    ssd_status st = check_dims(B, 1, H, P, G, N, 1, dtype);
    if (st != SSD_OK) return st;
    if (B == 0) return SSD_OK;
    if (!x || !dt || !A || !Bm || !Cm || !state || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt, A, Bm, Cm, D, state, y};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return SSD_ERR_MISALIGNED;
    LaunchCtx ctx;
    st = make_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx);
    if (st != SSD_OK) return st;
    StepArgs a;
    a.x = x; a.dt = dt; a.A = A; a.Bm = Bm; a.Cm = Cm; a.D = D; a.state = state; a.y = y;
    a.B = B; a.H = H; a.P = P; a.G = G; a.N = N; a.bf16 = dtype == SSD_BF16;
    return step_forward(a, ctx) == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

int ssd_forward_kernel_count(int B, int L, int H, int P, int G, int N, int chunk,
                             ssd_dtype dtype)
{
    if (check_dims(B, L, H, P, G, N, chunk, dtype) != SSD_OK) return 0;
    if ((long long)B * L == 0) return 0;
    FwdArgs a = make_args(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                          nullptr, B, L, H, P, G, N, chunk, dtype);
    return tc_supported(a) ? tc_kernel_count(a) : 3;
}

int ssd_forward_path(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype)
{
    if (check_dims(B, L, H, P, G, N, chunk, dtype) != SSD_OK) return 0;
    if ((long long)B * L == 0) return 0;
    FwdArgs a = make_args(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                          nullptr, B, L, H, P, G, N, chunk, dtype);
    if (!tc_supported(a)) return 1;
    return tc_segment_parallel(a) ? 3 : 2;
}

ssd_status ssd_poll_status(ssd_stream_t stream)
{
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return SSD_ERR_CUDA;
    LaunchCtx ctx;
    if (make_ctx(reinterpret_cast<cudaStream_t>(stream), &ctx) != SSD_OK) return SSD_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpy(&word, ctx.status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return SSD_ERR_CUDA;
    if (word != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpy(ctx.status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
            return SSD_ERR_CUDA;
        return SSD_ERR_TIMEOUT;
    }
    return SSD_OK;
}

void ssd_set_fault_injection(int skip_publish) { tc_set_skip_publish(skip_publish); }

void ssd_set_wait_limit(uint64_t iterations)
{
    std::lock_guard<std::mutex> lock(g_mu);
    g_wait_limit = iterations ? iterations : kDefaultWaitLimit;
}

}  // extern "C"
