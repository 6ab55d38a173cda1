// tc_forward.cu — tensor-core (tcgen05) forward path of the SSD layer.
//
// The chunked algorithm of "Mamba-2" (docsaid.org), section "Half of each
// route": inside a tile the quadratic ("attention") form runs on the tensor
// cores; across tiles only the end state is carried. Each CTA takes one work
// item = one head of one batch row over one 128-token tile (item order is
// tile-major, handed out by an atomic ticket so that an item's predecessor on
// the same head always started earlier). Per item, with cs the tile-local
// cumulative sum of dt * A (log2 units), everything on chip:
//
//   1. TMA loads C, B (128 x N) and X (128 x 64) tiles (128-byte swizzle).
//   2. MMA1:   S  = C B^T                  (128 x 128, K = N)       -> TMEM
//      states: s  = B^T (w o X), w_j = exp(cs_end - cs_j) dt_j
//                                          (N x 64, K = 128)        -> TMEM
//   3. mask:   S~_ij = S_ij exp(cs_i - cs_j) dt_j for j <= i, else 0 (bf16, smem)
//      MMA2:   Yd = S~ X                   (128 x 64, K = 128)      -> TMEM
//   4. look-back: wait until the head's previous tile published h_prev
//      (fp32, [P][N], in a two-slot ring of the workspace), then
//      h = exp(cs_end) h_prev + s is published for the next tile (or written
//      to final_state), and h_prev in bf16 feeds
//      MMA3:   Ys = C h_prev^T              (128 x 64, K = N)       -> TMEM
//   5. y_i = Yd_i + exp(cs_i) Ys_i + D x_i, stored as bf16.
//
// The masked product is the structured masked attention of "Mamba-2 SSD note"
// (0h-n0.github.io), section "SSD layer: equivalence under the scalar
// constraint" (C as queries, B as keys, X as values); the tile states are the
// low-rank representation of the blocks below the diagonal ("Mamba-2",
// section "Half of each route"); carrying h across tiles is the composition of
// affine maps of "Selective SSM guide" (auturnal.com), eq. (3).
//
// A chunk of 256 tokens is evaluated as two 128-token tiles: its quadratic
// form split into 2 x 2 blocks, the diagonal blocks computed directly and the
// block below the diagonal through its rank-N factorisation (the state of the
// first tile read out by C of the second). The result is the same up to
// rounding.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "sm100.cuh"
#include "tc_forward.cuh"

namespace ssd {
namespace {

using namespace sm100;

constexpr int kT = 128;        // tokens per tile
constexpr int kP = 64;         // head dim on this path
constexpr int kThreads = 128;  // 4 warps: thread i <-> tile row / TMEM lane i
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kMbarLimit = 1ull << 22;  // hardware-completion waits (~seconds)

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t kColS = 0;      // S: 128 columns
constexpr uint32_t kColState = 128;  // s: 64 columns per 128 rows of N
constexpr uint32_t kColYd = 256;   // Yd: 64
constexpr uint32_t kColYs = 320;   // Ys: 64
constexpr uint32_t kTmemCols = 512;

struct TcParams {
    const float* dt;
    const float* A;
    const float* D;
    const float* init;
    __nv_bfloat16* y;
    float* final_state;
    unsigned int* ctrl;   // [0] ticket, [1] CTAs done
    unsigned int* flags;  // per (b, h): number of tiles published
    float* ring;          // per (b, h): 2 x [P][N] fp32
    unsigned int* status;
    unsigned long long wait_limit;
    int B, L, H, G, N, ntiles, total, chains;
    int skip_publish;  // fault-injection hook: never publish states
};

template <int N>
struct Smem {
    static constexpr uint32_t kC = 0;
    static constexpr uint32_t kB = kC + N * 256;      // N/64 regions of 16 KB
    static constexpr uint32_t kX = kB + N * 256;
    static constexpr uint32_t kXt = kX + 16384;
    static constexpr uint32_t kSt = kXt + 16384;       // 2 regions of 16 KB
    static constexpr uint32_t kHs = kSt + 32768;       // N/64 regions of 8 KB
    static constexpr uint32_t kMisc = kHs + N * 128;
    static constexpr uint32_t kCs = kMisc;             // 128 floats
    static constexpr uint32_t kDt = kCs + 512;
    static constexpr uint32_t kW = kDt + 512;
    static constexpr uint32_t kRed = kW + 512;         // 8 floats
    static constexpr uint32_t kBars = kRed + 64;       // 4 mbarriers
    static constexpr uint32_t kTmemPtr = kBars + 32;
    static constexpr uint32_t kItem = kTmemPtr + 4;
    static constexpr uint32_t kFlag = kItem + 4;
    static constexpr uint32_t kEnd = kFlag + 8;
    static constexpr uint32_t kBytes = kEnd + 1024;    // + alignment slack
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u)
{
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

template <int N>
__global__ void __launch_bounds__(kThreads, 1)
tc_forward_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, TcParams p)
{
    using S = Smem<N>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    float* s_cs = reinterpret_cast<float*>(sm + S::kCs);
    float* s_dt = reinterpret_cast<float*>(sm + S::kDt);
    float* s_w = reinterpret_cast<float*>(sm + S::kW);
    float* s_red = reinterpret_cast<float*>(sm + S::kRed);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kBars);
    uint64_t* bar_tma = bars + 0;
    uint64_t* bar_mma1 = bars + 1;
    uint64_t* bar_mma2 = bars + 2;
    uint64_t* bar_mma3 = bars + 3;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + S::kTmemPtr);
    int* s_item = reinterpret_cast<int*>(sm + S::kItem);
    int* s_flag = reinterpret_cast<int*>(sm + S::kFlag);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;

    if (tid == 0) {
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmC);
        for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
        mbar_fence_init();
        *s_item = static_cast<int>(atomicAdd(p.ctrl, 1u));
        s_flag[0] = 0;  // set if a bounded wait gave up
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *s_tmem;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

    const int item = *s_item;
    const int tile = item / (p.B * p.H);
    const int chain = item - tile * (p.B * p.H);
    const int b = chain / p.H;
    const int h = chain - b * p.H;
    const int g = h / (p.H / p.G);
    const int t0 = tile * kT;
    const int rows = min(kT, p.L - t0);

    // ---- 1. TMA loads
    if (tid == 0) {
        mbar_arrive_expect_tx(bar_tma, 2 * N * 256 + 16384);
#pragma unroll
        for (int k = 0; k < N / 64; ++k) {
            tma_load_4d(sm + S::kC + k * 16384, &tmC, k * 64, g, t0, b, bar_tma);
            tma_load_4d(sm + S::kB + k * 16384, &tmB, k * 64, g, t0, b, bar_tma);
        }
        tma_load_4d(sm + S::kX, &tmX, 0, h, t0, b, bar_tma);
    }

    // ---- tile-local cumulative sum of dt * A (log2 units)
    const float Ah = p.A[h] * kLog2e;
    const float dti = tid < rows ? p.dt[(static_cast<size_t>(b) * p.L + t0 + tid) * p.H + h] : 0.f;
    float v = dti * Ah;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if ((tid & 31) >= o) v += u;
    }
    if ((tid & 31) == 31) s_red[warp] = v;
    __syncthreads();
    for (int w = 0; w < warp; ++w) v += s_red[w];
    s_cs[tid] = v;
    s_dt[tid] = dti;
    __syncthreads();
    const float cs_end = s_cs[kT - 1];
    const float cs_i = v;
    s_w[tid] = exp2f(cs_end - cs_i) * dti;
    __syncthreads();

    // ---- wait for the tiles
    if (!mbar_wait(bar_tma, 0, kMbarLimit)) {
        record_status(p.status, kDevWaitTimeout);
        s_flag[0] = 1;
    }

    // ---- X~ = w o X (row j of the swizzled tile is the 128 bytes at j * 128)
    {
        const uint4* src = reinterpret_cast<const uint4*>(sm + S::kX);
        uint4* dst = reinterpret_cast<uint4*>(sm + S::kXt);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int chunk = tid + k * kThreads;
            const float wj = s_w[chunk >> 3];
            uint4 q = src[chunk];
            uint32_t* u = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = unpack_bf16x2(u[e]);
                u[e] = pack_bf16x2(f.x * wj, f.y * wj);
            }
            dst[chunk] = q;
        }
    }
    fence_async_shared();
    tc_fence_before_sync();
    __syncthreads();

    // ---- 2. MMA1 (S = C B^T) and the tile states (s = B^T X~)
    if (tid == 0) {
        tc_fence_after_sync();
        const uint32_t c_base = smem_addr(sm + S::kC);
        const uint32_t b_base = smem_addr(sm + S::kB);
        const uint32_t xt_base = smem_addr(sm + S::kXt);
        constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
            const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;
            mma_bf16(tmem + kColS, sdesc_sw128(c_base + off, 16, 1024),
                     sdesc_sw128(b_base + off, 16, 1024), id_s, k > 0);
        }
        constexpr uint32_t id_st = idesc_bf16(128, kP, true, true);
#pragma unroll
        for (int m = 0; m < N / 128; ++m) {
#pragma unroll
            for (int k = 0; k < kT / 16; ++k) {
                mma_bf16(tmem + kColState + m * 64,
                         sdesc_sw128(b_base + m * 32768 + k * 2048, 16384, 1024),
                         sdesc_sw128(xt_base + k * 2048, 16384, 1024), id_st, k > 0);
            }
        }
        mma_commit(bar_mma1);
    }
    if (!mbar_wait(bar_mma1, 0, kMbarLimit)) {
        record_status(p.status, kDevWaitTimeout);
        s_flag[0] = 1;
    }
    tc_fence_after_sync();

    // ---- 3. mask S into S~ (bf16, K-major, two 64-column regions)
    {
        const int i = tid;
        uint8_t* st = sm + S::kSt;
#pragma unroll 1
        for (int jb = 0; jb < 4; ++jb) {
            float sv[32];
            tmem_ld32(tmem + lane_off + kColS + jb * 32, sv);
            tmem_wait_ld();
            uint32_t packed[16];
#pragma unroll
            for (int jj = 0; jj < 32; jj += 2) {
                const int j0 = jb * 32 + jj, j1 = j0 + 1;
                const float m0 = j0 <= i ? sv[jj] * exp2f(cs_i - s_cs[j0]) * s_dt[j0] : 0.f;
                const float m1 = j1 <= i ? sv[jj + 1] * exp2f(cs_i - s_cs[j1]) * s_dt[j1] : 0.f;
                packed[jj >> 1] = pack_bf16x2(m0, m1);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int col = jb * 32 + q * 8;
                uint8_t* dst = st + (col >> 6) * 16384 + sw128_offset(i, col & 63);
                *reinterpret_cast<uint4*>(dst) =
                    make_uint4(packed[q * 4], packed[q * 4 + 1], packed[q * 4 + 2], packed[q * 4 + 3]);
            }
        }
    }
    fence_async_shared();
    tc_fence_before_sync();
    __syncthreads();

    // ---- MMA2: Yd = S~ X
    if (tid == 0) {
        tc_fence_after_sync();
        const uint32_t st_base = smem_addr(sm + S::kSt);
        const uint32_t x_base = smem_addr(sm + S::kX);
        constexpr uint32_t id_y = idesc_bf16(128, kP, false, true);
#pragma unroll
        for (int k = 0; k < kT / 16; ++k) {
            mma_bf16(tmem + kColYd, sdesc_sw128(st_base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                     sdesc_sw128(x_base + k * 2048, 16384, 1024), id_y, k > 0);
        }
        mma_commit(bar_mma2);
    }

    // ---- 4. look-back: the previous tile of this head publishes h_prev
    const size_t PN = static_cast<size_t>(kP) * N;
    if (tid == 0 && tile > 0) {
        const unsigned int* f = p.flags + chain;
        bool ok = false;
        for (unsigned long long it = 0; it < p.wait_limit; ++it) {
            if (ld_acquire_gpu(f) >= static_cast<unsigned int>(tile)) { ok = true; break; }
            __nanosleep(64);
        }
        if (!ok) {
            record_status(p.status, kDevWaitTimeout);
            s_flag[0] = 1;
        }
    }
    __syncthreads();

    // thread n owns state rows n (and n + 128 for N = 256): 64 p values each
    const float dec_tile = exp2f(cs_end);
    const float* hsrc = nullptr;
    if (tile == 0) {
        hsrc = p.init ? p.init + static_cast<size_t>(chain) * PN : nullptr;
    } else if (!s_flag[0]) {
        hsrc = p.ring + (static_cast<size_t>(chain) * 2 + ((tile - 1) & 1)) * PN;
    }
    const bool last = tile == p.ntiles - 1;
    float* hdst = last ? (p.final_state ? p.final_state + static_cast<size_t>(chain) * PN : nullptr)
                       : p.ring + (static_cast<size_t>(chain) * 2 + (tile & 1)) * PN;
#pragma unroll 1
    for (int m = 0; m < N / 128; ++m) {
        const int n = tid + m * 128;
        float hp[kP];
#pragma unroll
        for (int q = 0; q < kP; ++q)
            hp[q] = hsrc ? __ldcg(hsrc + static_cast<size_t>(q) * N + n) : 0.f;
        // h_prev (bf16) as the K-major B operand of MMA3: row p, column n
        uint8_t* hs = sm + S::kHs + (n >> 6) * 8192;
#pragma unroll
        for (int q = 0; q < kP; ++q)
            *reinterpret_cast<__nv_bfloat16*>(hs + sw128_offset(q, n & 63)) = __float2bfloat16_rn(hp[q]);
        // h = exp(cs_end) h_prev + s
        float sv[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tmem_ld32(tmem + lane_off + kColState + m * 64 + half * 32, sv);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
                const int pq = half * 32 + q;
                const float hn = dec_tile * hp[pq] + sv[q];
                if (hdst) hdst[static_cast<size_t>(pq) * N + n] = hn;
            }
        }
    }
    __threadfence();
    fence_async_shared();
    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0 && !last && !p.skip_publish) st_release_gpu(p.flags + chain, tile + 1);

    // ---- MMA3: Ys = C h_prev^T
    if (tid == 0) {
        tc_fence_after_sync();
        const uint32_t c_base = smem_addr(sm + S::kC);
        const uint32_t hs_base = smem_addr(sm + S::kHs);
        constexpr uint32_t id_y = idesc_bf16(128, kP, false, false);
#pragma unroll
        for (int k = 0; k < N / 16; ++k) {
            mma_bf16(tmem + kColYs, sdesc_sw128(c_base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                     sdesc_sw128(hs_base + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024), id_y, k > 0);
        }
        mma_commit(bar_mma3);
    }
    bool ok2 = mbar_wait(bar_mma2, 0, kMbarLimit);
    bool ok3 = mbar_wait(bar_mma3, 0, kMbarLimit);
    if (!ok2 || !ok3) record_status(p.status, kDevWaitTimeout);
    tc_fence_after_sync();

    // ---- 5. epilogue: y_i = Yd_i + exp(cs_i) Ys_i + D x_i
    {
        const int i = tid;
        const float Dh = p.D ? p.D[h] : 0.f;
        const float ei = exp2f(cs_i);
        const uint8_t* xrow = sm + S::kX;
        __nv_bfloat16* yrow = p.y + ((static_cast<size_t>(b) * p.L + t0 + i) * p.H + h) * kP;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float yd[32], ys[32];
            tmem_ld32(tmem + lane_off + kColYd + half * 32, yd);
            tmem_ld32(tmem + lane_off + kColYs + half * 32, ys);
            tmem_wait_ld();
            uint32_t out[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int col = half * 32 + q * 8;
                const uint4 xq = *reinterpret_cast<const uint4*>(xrow + sw128_offset(i, col));
                const uint32_t* xu = reinterpret_cast<const uint32_t*>(&xq);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 xf = unpack_bf16x2(xu[e]);
                    const int c = q * 8 + e * 2;
                    out[q * 4 + e] = pack_bf16x2(yd[c] + ei * ys[c] + Dh * xf.x,
                                                 yd[c + 1] + ei * ys[c + 1] + Dh * xf.y);
                }
            }
            if (i < rows) {
                uint4* dst = reinterpret_cast<uint4*>(yrow + half * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    dst[q] = make_uint4(out[q * 4], out[q * 4 + 1], out[q * 4 + 2], out[q * 4 + 3]);
            }
        }
    }

    // ---- teardown
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    if (tid == 0) {
        __threadfence();
        const unsigned int done = atomicAdd(p.ctrl + 1, 1u);
        if (done == static_cast<unsigned int>(p.total) - 1u) {
            // every other CTA has finished: leave the control words zeroed
            for (int c = 0; c < p.chains; ++c) p.flags[c] = 0u;
            p.ctrl[0] = 0u;
            p.ctrl[1] = 0u;
            __threadfence();
        }
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 4-D bf16 map over a [d3][d2][d1][d0] tensor, box {64, 1, 128, 1}, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t d3)
{
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[4] = {d0, d1, d2, d3};
    cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

struct WsLayout {
    size_t ctrl, flags, ring, total;
};

WsLayout ws_layout(const FwdArgs& a)
{
    WsLayout w;
    const size_t chains = static_cast<size_t>(a.B) * a.H;
    w.ctrl = 0;
    w.flags = 256;
    w.ring = w.flags + ((chains * 4 + 255) / 256) * 256;
    w.total = w.ring + chains * 2 * kP * a.N * sizeof(float);
    return w;
}

int g_skip_publish = 0;

template <int N>
cudaError_t launch(const FwdArgs& a, void* workspace, const LaunchCtx& ctx)
{
    CUtensorMap tmX, tmB, tmC;
    if (!make_map(&tmX, a.x, kP, a.H, a.L, a.B) || !make_map(&tmB, a.Bm, N, a.G, a.L, a.B) ||
        !make_map(&tmC, a.Cm, N, a.G, a.L, a.B))
        return cudaErrorInvalidValue;
    const WsLayout w = ws_layout(a);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    TcParams p;
    p.dt = a.dt;
    p.A = a.A;
    p.D = a.D;
    p.init = a.init;
    p.y = static_cast<__nv_bfloat16*>(a.y);
    p.final_state = a.final_state;
    p.ctrl = reinterpret_cast<unsigned int*>(ws + w.ctrl);
    p.flags = reinterpret_cast<unsigned int*>(ws + w.flags);
    p.ring = reinterpret_cast<float*>(ws + w.ring);
    p.status = ctx.status;
    p.wait_limit = ctx.wait_limit;
    p.B = a.B;
    p.L = a.L;
    p.H = a.H;
    p.G = a.G;
    p.N = N;
    p.ntiles = (a.L + kT - 1) / kT;
    p.chains = a.B * a.H;
    p.total = p.ntiles * p.chains;
    p.skip_publish = g_skip_publish;
    const uint32_t smem = Smem<N>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(tc_forward_kernel<N>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    tc_forward_kernel<N><<<p.total, kThreads, smem, ctx.stream>>>(tmX, tmB, tmC, p);
    return cudaGetLastError();
}

}  // namespace

bool tc_supported(const FwdArgs& a)
{
    return a.bf16 && a.P == kP && a.N == 128 && (a.chunk == 128 || a.chunk == 256) &&
           static_cast<long long>(a.B) * a.L > 0 &&
           static_cast<long long>((a.L + kT - 1) / kT) * a.B * a.H < (1ll << 31);
}

size_t tc_workspace_bytes(const FwdArgs& a) { return ws_layout(a).total; }

int tc_kernel_count(const FwdArgs&) { return 1; }

void tc_set_skip_publish(int v) { g_skip_publish = v; }

cudaError_t tc_forward(const FwdArgs& a, void* workspace, const LaunchCtx& ctx)
{
    switch (a.N) {
    case 128: return launch<128>(a, workspace, ctx);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssd

// ---------------------------------------------------------------------------
// Allocation-free forward pass.
//
// Some callers cannot allocate device memory: code that runs where an
// allocation is not allowed or would be unsafe (for instance inside a
// framework callback that must not call cudaMalloc, on a memory pool that is
// already full, or in an embedded host that owns every byte of device memory)
// and callers that have no convenient place to keep a workspace alive between
// calls. For them, ssd_forward_noalloc runs the tensor-core forward with its
// scratch (look-back control words and the per-head state ring) in the fixed
// device array below instead of a caller-provided workspace. The caller still
// passes every input and output buffer.
//
// The array belongs to the library: each GPU that loads it holds the array
// until the process exits. Every call on a device shares it and leaves its
// contents behind, so calls that may overlap on the GPU (different streams,
// or host threads without ordering) race and must not be issued; calls on one
// stream are ordered and safe. Host code cannot use the array's name as a
// device address, so the first call on each device looks its address up with
// cudaGetSymbolAddress (make that first call before any stream capture).
namespace ssd {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(24) << 20;  // 24 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices];

bool noalloc_aligned(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

}  // namespace
}  // namespace ssd

extern "C" ssd_status ssd_forward_noalloc(const void* x, const float* dt, const float* A,
                                          const void* Bm, const void* Cm, const float* D,
                                          const float* initial_state, void* y,
                                          float* final_state, int B, int L, int H, int P, int G,
                                          int N, int chunk, ssd_dtype dtype, ssd_stream_t stream)
{
    using namespace ssd;
    if (B < 0 || L < 0 || H < 1 || G < 1 || P < 1 || N < 1 || chunk < 1 || H % G != 0 ||
        (dtype != SSD_F32 && dtype != SSD_BF16))
        return SSD_ERR_INVALID_ARG;
    if ((long long)B * L == 0) return SSD_ERR_UNSUPPORTED;  // nothing for the scratch to do
    if (!x || !dt || !A || !Bm || !Cm || !y) return SSD_ERR_INVALID_ARG;
    const void* ptrs[] = {x, dt, A, Bm, Cm, D, initial_state, y, final_state};
    for (const void* q : ptrs)
        if (q && !noalloc_aligned(q)) return SSD_ERR_MISALIGNED;
    FwdArgs a;
    a.x = x; a.dt = dt; a.A = A; a.Bm = Bm; a.Cm = Cm; a.D = D; a.init = initial_state;
    a.y = y; a.final_state = final_state;
    a.B = B; a.L = L; a.H = H; a.P = P; a.G = G; a.N = N; a.chunk = chunk;
    a.bf16 = dtype == SSD_BF16;
    if (!tc_supported(a)) return SSD_ERR_UNSUPPORTED;  // tensor-core sizes only
    const WsLayout w = ws_layout(a);
    if (w.total > kNoAllocScratchBytes) return SSD_ERR_WORKSPACE;  // scratch would not fit

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
        return SSD_ERR_CUDA;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mu);
        if (!g_noalloc_ptr[dev]) {
            void* addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr)
                return SSD_ERR_CUDA;
            g_noalloc_ptr[dev] = addr;
        }
        scratch = g_noalloc_ptr[dev];
    }
    LaunchCtx ctx;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const ssd_status st = acquire_launch_ctx(s, &ctx);
    if (st != SSD_OK) return st;
    // the ticket, done counter and look-back flags must start at zero
    if (cudaMemsetAsync(scratch, 0, w.ring, s) != cudaSuccess) return SSD_ERR_CUDA;
    const cudaError_t e = tc_forward(a, scratch, ctx);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
