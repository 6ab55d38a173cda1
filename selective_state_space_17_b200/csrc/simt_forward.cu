// simt_forward.cu — chunked SSD forward on CUDA cores, fp32 arithmetic.
//
// The general path: any valid size, fp32 or bf16 I/O. It takes the chunked
// algorithm's steps as three launches ("Mamba-2", docsaid.org, section "Half
// of each route": quadratic form inside a chunk, only chunk-end states carried
// across chunks):
//   1. simt_chunk_state: per (b, h, chunk) the chunk's own end state
//      s_c = sum_j exp(cs_end - cs_j) dt_j x_j B_j^T and its total decay
//      exp(cs_end), with cs the chunk-local cumulative sum of dt * A;
//   2. simt_state_pass: per (b, h) the recurrence across chunks,
//      h_c = exp(cs_end,c) h_{c-1} + s_c, replacing s_c by h_{c-1} in place
//      (the affine-map composition of "Selective SSM guide", auturnal.com,
//      eq. (3));
//   3. simt_chunk_output: per (b, h, chunk, 32-row tile)
//      y_i = sum_{j<=i} (C_i . B_j) exp(cs_i - cs_j) dt_j x_j
//            + exp(cs_i) C_i . h_{c-1} + D_h x_i.
// Workspace: states [B][H][nc][P][N] fp32, then decays [B][H][nc] fp32.
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kThreads = 256;
constexpr int kRowTile = 32;
constexpr int kMaxChunk = 256;

template <typename T>
__device__ __forceinline__ void chunk_cumsum(const FwdArgs& a, int b, int h, int c0, int Qc,
                                             float* s_cs, float* s_dt)
{
    if (threadIdx.x == 0) {
        const float Ah = a.A[h];
        float acc = 0.f;
        for (int j = 0; j < Qc; ++j) {
            const float d = a.dt[((size_t)b * a.L + c0 + j) * a.H + h];
            acc += d * Ah;
            s_cs[j] = acc;
            s_dt[j] = d;
        }
    }
    __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
simt_chunk_state(FwdArgs a, float* states, float* decay, int nc)
{
    const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int c0 = c * a.chunk;
    const int Qc = min(a.chunk, a.L - c0);
    const int g = h / (a.H / a.G);
    __shared__ float s_cs[kMaxChunk], s_dt[kMaxChunk], s_w[kMaxChunk];
    chunk_cumsum<T>(a, b, h, c0, Qc, s_cs, s_dt);
    const float cs_end = s_cs[Qc - 1];
    for (int j = threadIdx.x; j < Qc; j += blockDim.x) s_w[j] = expf(cs_end - s_cs[j]) * s_dt[j];
    if (threadIdx.x == 0) decay[((size_t)b * a.H + h) * nc + c] = expf(cs_end);
    __syncthreads();

    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.Bm);
    float* out = states + (((size_t)b * a.H + h) * nc + c) * a.P * a.N;
    for (int e = threadIdx.x; e < a.P * a.N; e += blockDim.x) {
        const int p = e / a.N, n = e % a.N;
        float acc = 0.f;
        for (int j = 0; j < Qc; ++j) {
            const size_t t = (size_t)b * a.L + c0 + j;
            acc += s_w[j] * io<T>::load(x + (t * a.H + h) * a.P + p) *
                   io<T>::load(Bm + (t * a.G + g) * a.N + n);
        }
        out[e] = acc;
    }
}

__global__ void __launch_bounds__(kThreads)
simt_state_pass(float* states, const float* decay, const float* init, float* final_state,
                int H, int PN, int nc)
{
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int h = blockIdx.y, b = blockIdx.z;
    if (e >= PN) return;
    const size_t bh = (size_t)b * H + h;
    float hc = init ? init[bh * PN + e] : 0.f;
    float* st = states + bh * nc * PN + e;
    const float* dc = decay + bh * nc;
    for (int c = 0; c < nc; ++c) {
        const float s = st[(size_t)c * PN];
        st[(size_t)c * PN] = hc;
        hc = dc[c] * hc + s;
    }
    if (final_state) final_state[bh * PN + e] = hc;
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
simt_chunk_output(FwdArgs a, const float* states, int nc, int tiles_per_chunk)
{
    const int c = blockIdx.x / tiles_per_chunk;
    const int i0 = (blockIdx.x % tiles_per_chunk) * kRowTile;
    const int h = blockIdx.y, b = blockIdx.z;
    const int c0 = c * a.chunk;
    const int Qc = min(a.chunk, a.L - c0);
    if (i0 >= Qc) return;
    const int g = h / (a.H / a.G);
    __shared__ float s_cs[kMaxChunk], s_dt[kMaxChunk];
    __shared__ float s_S[kRowTile][kMaxChunk + 1];
    chunk_cumsum<T>(a, b, h, c0, Qc, s_cs, s_dt);

    const T* x = static_cast<const T*>(a.x);
    const T* Bm = static_cast<const T*>(a.Bm);
    const T* Cm = static_cast<const T*>(a.Cm);
    T* y = static_cast<T*>(a.y);
    const int rows = min(kRowTile, Qc - i0);
    const int jmax = i0 + rows;  // columns j < jmax can be nonzero
    for (int e = threadIdx.x; e < rows * jmax; e += blockDim.x) {
        const int r = e / jmax, j = e % jmax, i = i0 + r;
        float v = 0.f;
        if (j <= i) {
            const T* Ci = Cm + (((size_t)b * a.L + c0 + i) * a.G + g) * a.N;
            const T* Bj = Bm + (((size_t)b * a.L + c0 + j) * a.G + g) * a.N;
            float dot = 0.f;
            for (int n = 0; n < a.N; ++n) dot += io<T>::load(Ci + n) * io<T>::load(Bj + n);
            v = dot * expf(s_cs[i] - s_cs[j]) * s_dt[j];
        }
        s_S[r][j] = v;
    }
    __syncthreads();

    const float* hprev = states + (((size_t)b * a.H + h) * nc + c) * a.P * a.N;
    const float Dh = a.D ? a.D[h] : 0.f;
    for (int e = threadIdx.x; e < rows * a.P; e += blockDim.x) {
        const int r = e / a.P, p = e % a.P, i = i0 + r;
        float acc = 0.f;
        for (int j = 0; j <= i; ++j)
            acc += s_S[r][j] * io<T>::load(x + (((size_t)b * a.L + c0 + j) * a.H + h) * a.P + p);
        const T* Ci = Cm + (((size_t)b * a.L + c0 + i) * a.G + g) * a.N;
        const float* hp = hprev + (size_t)p * a.N;
        float st = 0.f;
        for (int n = 0; n < a.N; ++n) st += io<T>::load(Ci + n) * hp[n];
        const size_t yi = (((size_t)b * a.L + c0 + i) * a.H + h) * a.P + p;
        acc += expf(s_cs[i]) * st + Dh * io<T>::load(x + yi);
        io<T>::store(y + yi, acc);
    }
}

template <typename T>
cudaError_t run(const FwdArgs& a, void* workspace, const LaunchCtx& ctx)
{
    const int nc = (a.L + a.chunk - 1) / a.chunk;
    float* states = static_cast<float*>(workspace);
    float* decay = states + (size_t)a.B * a.H * nc * a.P * a.N;
    dim3 g1(nc, a.H, a.B);
    simt_chunk_state<T><<<g1, kThreads, 0, ctx.stream>>>(a, states, decay, nc);
    const int PN = a.P * a.N;
    dim3 g2((PN + kThreads - 1) / kThreads, a.H, a.B);
    simt_state_pass<<<g2, kThreads, 0, ctx.stream>>>(states, decay, a.init, a.final_state, a.H,
                                                     PN, nc);
    const int tiles = (a.chunk + kRowTile - 1) / kRowTile;
    dim3 g3(nc * tiles, a.H, a.B);
    simt_chunk_output<T><<<g3, kThreads, 0, ctx.stream>>>(a, states, nc, tiles);
    return cudaGetLastError();
}

}  // namespace

size_t simt_workspace_bytes(const FwdArgs& a)
{
    const size_t nc = (size_t)(a.L + a.chunk - 1) / a.chunk;
    return ((size_t)a.B * a.H * nc * (size_t)(a.P * a.N + 1)) * sizeof(float);
}

cudaError_t simt_forward(const FwdArgs& a, void* workspace, const LaunchCtx& ctx)
{
    return a.bf16 ? run<__nv_bfloat16>(a, workspace, ctx) : run<float>(a, workspace, ctx);
}

}  // namespace ssd
