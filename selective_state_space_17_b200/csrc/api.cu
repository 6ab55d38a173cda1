// api.cu — the C ABI of libssd_b200.so: argument checks, workspace sizing,
// dispatch to the kernel families, the device status word and the host-buffer
// entry point. Declarations and contracts are in include/ssd.h.
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "grouped_forward.cuh"
#include "tc_forward.cuh"

namespace ssd {

__device__ unsigned int g_device_status;

namespace {

constexpr unsigned long long kDefaultWaitLimit = 1ull << 23;  // ~seconds of polling
constexpr int kMaxDevices = 64;

unsigned long long g_wait_limit = kDefaultWaitLimit;
int g_variant = 0;  // test hook: 0 automatic, 1 per-head tensor-core kernel, 2 head-group kernel
std::atomic<uint32_t> g_epoch{0x5EED0001u};  // call tags (see LaunchCtx::epoch)
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
    uint32_t e = g_epoch.fetch_add(1u, std::memory_order_relaxed);
    if (e == 0) e = g_epoch.fetch_add(1u, std::memory_order_relaxed);
    ctx->epoch = e;
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

int device_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

// Which kernel family runs a call: 1 SIMT, 2 per-head tensor-core kernel, 3 the
// same in its segment-parallel form, 4 head-group tensor-core kernel.
int forward_path(const FwdArgs& a, int sms)
{
    const bool grp = grouped::supported(a), tc = tc_supported(a);
    if (grp && (g_variant == 2 || (g_variant == 0 && grouped::preferred(a, sms)))) return 4;
    if (tc) return tc_segment_parallel(a) ? 3 : 2;
    if (grp) return 4;
    return 1;
}

// Enough for whichever kernel family the call may take.
size_t workspace_bytes(const FwdArgs& a)
{
    size_t w = 0;
    if (grouped::supported(a)) w = grouped::workspace_bytes(a, device_sms());
    if (tc_supported(a)) w = std::max(w, tc_workspace_bytes(a));
    if (!grouped::supported(a) && !tc_supported(a)) w = simt_workspace_bytes(a);
    return w;
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

// Size checks shared by every forward and step entry point.
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
    const int path = forward_path(a, ctx.num_sms);
    cudaError_t e = path == 4   ? grouped::forward(a, workspace, ctx)
                    : path >= 2 ? tc_forward(a, workspace, ctx)
                                : simt_forward(a, workspace, ctx);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}

// ssd_forward_host runs the batch in slices of rows so that the copies of one
// slice overlap the forward pass and the copies of others: slices alternate
// between two internal streams of the device (created once), each with its
// own workspace. The copy engines move host-to-device and device-to-host
// traffic at the same time, so the call costs about the larger of the two
// directions instead of their sum.
namespace {

constexpr int kHostSlices = 4;  // batch slices of one ssd_forward_host call (at most)
constexpr int kHostStreams = 2;

struct HostStreams {
    cudaStream_t s[kHostStreams] = {nullptr, nullptr};
    cudaEvent_t start = nullptr, params = nullptr, done[kHostStreams] = {nullptr, nullptr};
    bool ok = false;
};
HostStreams g_host[kMaxDevices];

bool host_streams(int dev, HostStreams** out)
{
    std::lock_guard<std::mutex> lock(g_mu);
    HostStreams& h = g_host[dev];
    if (!h.ok) {
        for (int i = 0; i < kHostStreams; ++i) {
            if (cudaStreamCreateWithFlags(&h.s[i], cudaStreamNonBlocking) != cudaSuccess) return false;
            if (cudaEventCreateWithFlags(&h.done[i], cudaEventDisableTiming) != cudaSuccess) return false;
        }
        if (cudaEventCreateWithFlags(&h.start, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&h.params, cudaEventDisableTiming) != cudaSuccess)
            return false;
        h.ok = true;
    }
    *out = &h;
    return true;
}

int host_slices(int B) { return B < kHostSlices ? (B > 0 ? B : 1) : kHostSlices; }

// Rows of the largest slice.
int host_slice_rows(int B) { return (B + host_slices(B) - 1) / host_slices(B); }

// A workspace that serves every slice (the last one may hold fewer rows).
size_t host_slice_workspace(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype)
{
    const int rows = host_slice_rows(B);
    const int last = B - (host_slices(B) - 1) * rows;
    size_t ws = ssd_workspace_size(rows, L, H, P, G, N, chunk, dtype);
    if (last > 0 && last != rows) ws = std::max(ws, ssd_workspace_size(last, L, H, P, G, N, chunk, dtype));
    return round_up(ws, 256);
}

}  // namespace

size_t ssd_forward_host_buffer_size(int B, int L, int H, int P, int G, int N, int chunk,
                                    ssd_dtype dtype)
{
    if (check_dims(B, L, H, P, G, N, chunk, dtype) != SSD_OK) return 0;
    const size_t ws = host_slice_workspace(B, L, H, P, G, N, chunk, dtype);
    if (ws == 0) return 0;
    const size_t es = dtype == SSD_BF16 ? 2 : 4;
    const size_t BL = (size_t)B * L;
    size_t total = ws * kHostStreams;                       // one workspace per stream
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
    cudaStream_t us = reinterpret_cast<cudaStream_t>(stream);
    const size_t es = dtype == SSD_BF16 ? 2 : 4;
    const size_t ws = host_slice_workspace(B, L, H, P, G, N, chunk, dtype);
    char* p = static_cast<char*>(device_buffer);
    void* d_ws[kHostStreams];
    for (int i = 0; i < kHostStreams; ++i) { d_ws[i] = p; p += ws; }
    const size_t row_x = (size_t)L * H * P * es, row_dt = (size_t)L * H * 4;
    const size_t row_bc = (size_t)L * G * N * es, row_st = (size_t)H * P * N * 4;
    char* d_x = p; p += round_up(BL * H * P * es, 256);
    char* d_y = p; p += round_up(BL * H * P * es, 256);
    char* d_dt = p; p += round_up(BL * H * 4, 256);
    float* d_A = reinterpret_cast<float*>(p); p += round_up((size_t)H * 4, 256);
    float* d_D = reinterpret_cast<float*>(p); p += round_up((size_t)H * 4, 256);
    char* d_B = p; p += round_up(BL * G * N * es, 256);
    char* d_C = p; p += round_up(BL * G * N * es, 256);
    char* d_init = p; p += round_up((size_t)B * row_st, 256);
    char* d_fs = p;
    if (BL == 0) {  // nothing to slice: final_state = initial_state or 0
        cudaError_t e = cudaSuccess;
        if (initial_state_host) e = cudaMemcpyAsync(d_init, initial_state_host, B * row_st,
                                                    cudaMemcpyHostToDevice, us);
        if (e != cudaSuccess) return SSD_ERR_CUDA;
        st = ssd_forward(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                         initial_state_host ? reinterpret_cast<float*>(d_init) : nullptr, nullptr,
                         final_state_host ? reinterpret_cast<float*>(d_fs) : nullptr, B, L, H, P,
                         G, N, chunk, dtype, d_ws[0], ws, stream);
        if (st != SSD_OK) return st;
        if (final_state_host && B * row_st > 0)
            e = cudaMemcpyAsync(final_state_host, d_fs, B * row_st, cudaMemcpyDeviceToHost, us);
        if (e == cudaSuccess) e = cudaStreamSynchronize(us);
        return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSD_ERR_CUDA;
    HostStreams* hs = nullptr;
    if (!host_streams(dev, &hs)) return SSD_ERR_CUDA;
    auto h2d = [](void* dst, const void* src, size_t n, cudaStream_t s) {
        return (n == 0 || !src) ? cudaSuccess : cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s);
    };
    // the internal streams start after the work already queued on `stream`
    cudaError_t e = cudaEventRecord(hs->start, us);
    for (int i = 0; e == cudaSuccess && i < kHostStreams; ++i) e = cudaStreamWaitEvent(hs->s[i], hs->start, 0);
    if (e == cudaSuccess) e = h2d(d_A, A_host, (size_t)H * 4, hs->s[0]);
    if (e == cudaSuccess) e = h2d(d_D, D_host, (size_t)H * 4, hs->s[0]);
    if (e == cudaSuccess) e = cudaEventRecord(hs->params, hs->s[0]);
    for (int i = 1; e == cudaSuccess && i < kHostStreams; ++i) e = cudaStreamWaitEvent(hs->s[i], hs->params, 0);
    if (e != cudaSuccess) return SSD_ERR_CUDA;
    const int nsl = host_slices(B), rows = host_slice_rows(B);
    const char* xh = static_cast<const char*>(x_host);
    const char* dth = reinterpret_cast<const char*>(dt_host);
    const char* bh = static_cast<const char*>(Bm_host);
    const char* ch = static_cast<const char*>(Cm_host);
    const char* ih = reinterpret_cast<const char*>(initial_state_host);
    char* yh = static_cast<char*>(y_host);
    char* fh = reinterpret_cast<char*>(final_state_host);
    for (int j = 0; j < nsl; ++j) {
        const int b0 = j * rows, nb = std::min(rows, B - b0);
        if (nb <= 0) break;
        cudaStream_t s = hs->s[j % kHostStreams];
        e = h2d(d_x + b0 * row_x, xh + b0 * row_x, nb * row_x, s);
        if (e == cudaSuccess) e = h2d(d_dt + b0 * row_dt, dth + b0 * row_dt, nb * row_dt, s);
        if (e == cudaSuccess) e = h2d(d_B + b0 * row_bc, bh + b0 * row_bc, nb * row_bc, s);
        if (e == cudaSuccess) e = h2d(d_C + b0 * row_bc, ch + b0 * row_bc, nb * row_bc, s);
        if (e == cudaSuccess && ih) e = h2d(d_init + b0 * row_st, ih + b0 * row_st, nb * row_st, s);
        if (e != cudaSuccess) return SSD_ERR_CUDA;
        st = ssd_forward(d_x + b0 * row_x, reinterpret_cast<float*>(d_dt + b0 * row_dt), d_A,
                         d_B + b0 * row_bc, d_C + b0 * row_bc, D_host ? d_D : nullptr,
                         ih ? reinterpret_cast<float*>(d_init + b0 * row_st) : nullptr,
                         d_y + b0 * row_x, fh ? reinterpret_cast<float*>(d_fs + b0 * row_st) : nullptr,
                         nb, L, H, P, G, N, chunk, dtype, d_ws[j % kHostStreams], ws,
                         reinterpret_cast<ssd_stream_t>(s));
        if (st != SSD_OK) return st;
        e = cudaMemcpyAsync(yh + b0 * row_x, d_y + b0 * row_x, nb * row_x, cudaMemcpyDeviceToHost, s);
        if (e == cudaSuccess && fh)
            e = cudaMemcpyAsync(fh + b0 * row_st, d_fs + b0 * row_st, nb * row_st, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return SSD_ERR_CUDA;
    }
    for (int i = 0; e == cudaSuccess && i < kHostStreams; ++i) {
        e = cudaEventRecord(hs->done[i], hs->s[i]);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(us, hs->done[i], 0);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(us);
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
    const int path = forward_path(a, device_sms());
    return path == 4 ? 1 : path >= 2 ? tc_kernel_count(a) : 3;
}

int ssd_forward_path(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype)
{
    if (check_dims(B, L, H, P, G, N, chunk, dtype) != SSD_OK) return 0;
    if ((long long)B * L == 0) return 0;
    FwdArgs a = make_args(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                          nullptr, B, L, H, P, G, N, chunk, dtype);
    return forward_path(a, device_sms());
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

void ssd_set_fault_injection(int skip_publish)
{
    tc_set_skip_publish(skip_publish);
    grouped::set_skip_publish(skip_publish);
}

void ssd_set_forward_variant(int variant)
{
    std::lock_guard<std::mutex> lock(g_mu);
    g_variant = (variant >= 0 && variant <= 2) ? variant : 0;
}

void ssd_set_wait_limit(uint64_t iterations)
{
    std::lock_guard<std::mutex> lock(g_mu);
    g_wait_limit = iterations ? iterations : kDefaultWaitLimit;
}

}  // extern "C"
