// step.cu — single-token decode step of the SSD layer.
//
// Per (b, h): a = exp(dt A_h); state <- a * state + dt * x B^T; y = state C + D x.
// This is the recurrent route the pages recommend for generation ("Mamba-2",
// docsaid.org, section "Computing with four tokens": the recurrent form keeps a
// constant-size state and suits generation), with the discretisation of
// "Mamba paper review" (youngju.dev), section 3.3.
//
// The step is bound by HBM: the fp32 state is read and written once (P*N*8
// bytes per head) and everything else is small. A warp owns whole state rows p
// and moves them with 128-bit accesses (lane l holds n = 4l .. 4l+3 of each
// 128-column stripe), eight rows at a time, and reduces y_p with shuffles.
// For N <= 128 persistent warps stream items of eight rows, each warp loading
// the next item (state rows and every small operand) before it updates and
// stores the current one; otherwise one CTA of 8 warps per (b, h).
#include "common.cuh"

namespace ssd {
namespace {

constexpr int kWarps = 8;
constexpr int kRowsInFlight = 8;

template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p)
{
    return __ldg(reinterpret_cast<const float4*>(p));
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p)
{
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    float4 f;
    f.x = __uint_as_float(u.x << 16);
    f.y = __uint_as_float(u.x & 0xffff0000u);
    f.z = __uint_as_float(u.y << 16);
    f.w = __uint_as_float(u.y & 0xffff0000u);
    return f;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Vector path: N % 4 == 0 (every row starts 16-byte aligned).
template <typename T>
__global__ void __launch_bounds__(kWarps * 32, 3)
step_vec(StepArgs a)
{
    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.G);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float d = a.dt[bh];
    const float decay = expf(d * a.A[h]);
    const float Dh = a.D ? a.D[h] : 0.f;
    const T* x = static_cast<const T*>(a.x) + (size_t)bh * a.P;
    const T* Bv = static_cast<const T*>(a.Bm) + ((size_t)b * a.G + g) * a.N;
    const T* Cv = static_cast<const T*>(a.Cm) + ((size_t)b * a.G + g) * a.N;
    T* y = static_cast<T*>(a.y) + (size_t)bh * a.P;
    float* st = a.state + (size_t)bh * a.P * a.N;

    for (int p0 = warp * kRowsInFlight; p0 < a.P; p0 += kWarps * kRowsInFlight) {
        float acc[kRowsInFlight];
        float u[kRowsInFlight];
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            acc[r] = 0.f;
            u[r] = (p0 + r < a.P) ? d * io<T>::load(x + p0 + r) : 0.f;
        }
        for (int n = lane * 4; n < a.N; n += 128) {
            const float4 bq = load4<T>(Bv + n);
            const float4 cq = load4<T>(Cv + n);
            float4 hv[kRowsInFlight];
#pragma unroll
            for (int r = 0; r < kRowsInFlight; ++r)
                if (p0 + r < a.P)
                    hv[r] = __ldcs(reinterpret_cast<const float4*>(st + (size_t)(p0 + r) * a.N + n));
#pragma unroll
            for (int r = 0; r < kRowsInFlight; ++r) {
                if (p0 + r >= a.P) continue;
                float4 v = hv[r];
                v.x = decay * v.x + u[r] * bq.x;
                v.y = decay * v.y + u[r] * bq.y;
                v.z = decay * v.z + u[r] * bq.z;
                v.w = decay * v.w + u[r] * bq.w;
                acc[r] += v.x * cq.x + v.y * cq.y + v.z * cq.z + v.w * cq.w;
                __stcs(reinterpret_cast<float4*>(st + (size_t)(p0 + r) * a.N + n), v);
            }
        }
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            const float s = warp_sum(acc[r]);
            if (lane == 0 && p0 + r < a.P)
                io<T>::store(y + p0 + r, s + Dh * io<T>::load(x + p0 + r));
        }
    }
}

// Streaming path: N <= 128, N % 4 == 0 (one 128-bit access per lane and state
// row). Persistent warps walk items of eight rows of one head's state (a warp
// owns whole rows, so y_p is a warp reduction); each warp loads the next
// item's rows before it updates and stores the current ones, so that the
// state stream has no gaps between items and no tail of partly filled waves.
constexpr int kStreamCtasPerSm = 2;

// Division by a divisor fixed for the launch: with s = ceil(log2 d) and
// m = ceil(2^(32 + s) / d) - 2^32, q = (hi32(n * m) + n) >> s, exact for
// 0 <= n < 2^31 (the round-up method of Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994).
struct FastDiv {
    uint32_t m, s;
    __host__ explicit FastDiv(uint32_t d) : m(0), s(0)
    {
        while ((1ull << s) < d) ++s;
        m = static_cast<uint32_t>(((1ull << (32 + s)) + d - 1) / d - (1ull << 32));
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const { return (__umulhi(n, m) + n) >> s; }
};

// One item's operands, loaded a whole item ahead of their use.
struct StreamItem {
    float4 h[kRowsInFlight];  // state rows p0 .. p0 + 7, columns 4 lane .. 4 lane + 3
    float4 bq, cq;            // B and C at those columns
    float xr[kRowsInFlight];  // x of the rows
    float dt, A, D;
};

template <typename T>
__global__ void __launch_bounds__(kWarps * 32, kStreamCtasPerSm)
step_stream(StepArgs a, int items, FastDiv by_rb, FastDiv by_h, FastDiv by_hpg)
{
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * kWarps;
    const int rb = (a.P + kRowsInFlight - 1) / kRowsInFlight;  // items per head
    const bool lane_live = lane * 4 < a.N;
    auto fetch = [&](int item, StreamItem& it) {
        const int bh = by_rb.div(item), p0 = (item - bh * rb) * kRowsInFlight;
        const int b = by_h.div(bh), h = bh - b * a.H, g = by_hpg.div(h);
        const float* st = a.state + ((size_t)bh * a.P + p0) * a.N + lane * 4;
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r)
            it.h[r] = (lane_live && p0 + r < a.P) ? __ldcs(reinterpret_cast<const float4*>(st + (size_t)r * a.N))
                                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        it.bq = it.cq = make_float4(0.f, 0.f, 0.f, 0.f);
        if (lane_live) {
            it.bq = load4<T>(static_cast<const T*>(a.Bm) + ((size_t)b * a.G + g) * a.N + lane * 4);
            it.cq = load4<T>(static_cast<const T*>(a.Cm) + ((size_t)b * a.G + g) * a.N + lane * 4);
        }
        const T* x = static_cast<const T*>(a.x) + (size_t)bh * a.P + p0;
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) it.xr[r] = p0 + r < a.P ? io<T>::load(x + r) : 0.f;
        it.dt = a.dt[bh];
        it.A = a.A[h];
        it.D = a.D ? a.D[h] : 0.f;
    };
    int item = blockIdx.x * kWarps + (threadIdx.x >> 5);
    StreamItem cur;
    if (item < items) fetch(item, cur);
    while (item < items) {
        const int next = item + nwarps;
        StreamItem nxt;
        if (next < items) fetch(next, nxt);
        const int bh = by_rb.div(item), p0 = (item - bh * rb) * kRowsInFlight;
        const float decay = expf(cur.dt * cur.A);
        T* y = static_cast<T*>(a.y) + (size_t)bh * a.P + p0;
        float* st = a.state + ((size_t)bh * a.P + p0) * a.N + lane * 4;
        float dot[kRowsInFlight];  // this lane's part of y_p for each row
#pragma unroll
        for (int r = 0; r < kRowsInFlight; ++r) {
            const float u = cur.dt * cur.xr[r];  // 0 for rows past P
            float4 v = cur.h[r];
            v.x = decay * v.x + u * cur.bq.x;
            v.y = decay * v.y + u * cur.bq.y;
            v.z = decay * v.z + u * cur.bq.z;
            v.w = decay * v.w + u * cur.bq.w;
            dot[r] = v.x * cur.cq.x + v.y * cur.cq.y + v.z * cur.cq.z + v.w * cur.cq.w;
            if (lane_live && p0 + r < a.P) __stcs(reinterpret_cast<float4*>(st + (size_t)r * a.N), v);
        }
        // the eight row sums in 9 shuffles instead of 40: at each step a lane
        // keeps half of its rows and adds the partner's part of them, so after
        // the 16-, 8- and 4-lane exchanges lane l holds row (l >> 2) & 7 (over
        // its quad), and the 2- and 1-lane exchanges finish the sum
        {
            const bool hi16 = lane & 16, hi8 = lane & 8, hi4 = lane & 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float give = hi16 ? dot[i] : dot[i + 4];
                const float keep = hi16 ? dot[i + 4] : dot[i];
                dot[i] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float give = hi8 ? dot[i] : dot[i + 2];
                const float keep = hi8 ? dot[i + 2] : dot[i];
                dot[i] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
            }
            {
                const float give = hi4 ? dot[0] : dot[1];
                const float keep = hi4 ? dot[1] : dot[0];
                dot[0] = keep + __shfl_xor_sync(0xffffffffu, give, 4);
            }
            dot[0] += __shfl_xor_sync(0xffffffffu, dot[0], 2);
            dot[0] += __shfl_xor_sync(0xffffffffu, dot[0], 1);
            const int r = (hi16 ? 4 : 0) + (hi8 ? 2 : 0) + (hi4 ? 1 : 0);
            float xr = cur.xr[0];
#pragma unroll
            for (int q = 1; q < kRowsInFlight; ++q)
                if (r == q) xr = cur.xr[q];
            if ((lane & 3) == 0 && p0 + r < a.P) io<T>::store(y + r, dot[0] + cur.D * xr);
        }
        cur = nxt;
        item = next;
    }
}

// Scalar path: any N.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
step_scalar(StepArgs a)
{
    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh % a.H, g = h / (a.H / a.G);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float d = a.dt[bh];
    const float decay = expf(d * a.A[h]);
    const float Dh = a.D ? a.D[h] : 0.f;
    const T* x = static_cast<const T*>(a.x) + (size_t)bh * a.P;
    const T* Bv = static_cast<const T*>(a.Bm) + ((size_t)b * a.G + g) * a.N;
    const T* Cv = static_cast<const T*>(a.Cm) + ((size_t)b * a.G + g) * a.N;
    T* y = static_cast<T*>(a.y) + (size_t)bh * a.P;
    float* st = a.state + (size_t)bh * a.P * a.N;
    for (int p = warp; p < a.P; p += kWarps) {
        const float u = d * io<T>::load(x + p);
        float acc = 0.f;
        for (int n = lane; n < a.N; n += 32) {
            float* hv = st + (size_t)p * a.N + n;
            const float v = decay * *hv + u * io<T>::load(Bv + n);
            *hv = v;
            acc += v * io<T>::load(Cv + n);
        }
        acc = warp_sum(acc);
        if (lane == 0) io<T>::store(y + p, acc + Dh * io<T>::load(x + p));
    }
}

template <typename T>
cudaError_t run(const StepArgs& a, const LaunchCtx& ctx)
{
    const int grid = a.B * a.H;
    const long long stream_items = static_cast<long long>(a.B) * a.H * ((a.P + kRowsInFlight - 1) / kRowsInFlight);
    if (a.N % 4 == 0 && a.N <= 128 && stream_items < (1ll << 30)) {  // item indices stay below 2^31
        const int items = static_cast<int>(stream_items);
        const int sms = ctx.num_sms > 0 ? ctx.num_sms : 1;
        const int ctas = min((items + kWarps - 1) / kWarps, sms * kStreamCtasPerSm);
        step_stream<T><<<ctas, kWarps * 32, 0, ctx.stream>>>(
            a, items, FastDiv((a.P + kRowsInFlight - 1) / kRowsInFlight), FastDiv(a.H), FastDiv(a.H / a.G));
    } else if (a.N % 4 == 0)
        step_vec<T><<<grid, kWarps * 32, 0, ctx.stream>>>(a);
    else
        step_scalar<T><<<grid, kWarps * 32, 0, ctx.stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t step_forward(const StepArgs& a, const LaunchCtx& ctx)
{
    return a.bf16 ? run<__nv_bfloat16>(a, ctx) : run<float>(a, ctx);
}

}  // namespace ssd
