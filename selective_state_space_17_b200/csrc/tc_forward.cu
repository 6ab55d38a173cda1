// tc_forward.cu — tensor-core (tcgen05) forward path of the SSD layer.
//
// The chunked algorithm of "Mamba-2" (docsaid.org), section "Half of each
// route": inside a 128-token tile the quadratic ("attention") form runs on the
// tensor cores; across tiles only the end state is carried. Per tile, with cs
// the tile-local cumulative sum of dt * A (log2 units):
//
//   MMA1    S  = C B^T                                  (128 x 128, K = N)  TMEM
//   states  s  = B^T (w o X),  w_j = exp(cs_end - cs_j) dt_j  (N x 64, K = 128) TMEM
//   mask    S~_ij = S_ij exp(cs_i - cs_j) dt_j (j <= i), plus D_h on the diagonal,
//           in registers, written back as bf16 pairs over S in TMEM (the A
//           operand of MMA2)
//   MMA2    Yd = S~ X                                   (128 x 64, K = 128) TMEM
//   MMA3    Ys = C h_prev^T                             (128 x 64, K = N)   TMEM
//   output  y_i = Yd_i + exp(cs_i) Ys_i (bf16, round to nearest even)
//   state   h = exp(cs_end) h_prev + s
//
// The masked product is the structured masked attention of "Mamba-2 SSD note"
// (0h-n0.github.io), section "SSD layer: equivalence under the scalar
// constraint" (C as queries, B as keys, X as values, D x folded in as the
// diagonal D_h I); the tile states are the low-rank representation of the
// blocks below the diagonal ("Mamba-2", section "Half of each route"); carrying
// h is the composition of affine maps of "Selective SSM guide"
// (auturnal.com), eq. (3). The mask's exponentials are factored per 32-column
// block: for a block wholly left of row i with last column a,
// exp(cs_i - cs_j) = exp(cs_i - cs_a) * exp(cs_a - cs_j), both factors <= 1,
// so only the block on the diagonal needs one exponential per element.
//
// Schedule. Each (batch row, head) is a chain of tiles (a head of P = 64m
// channels is m chains of 64 channels); chains are cut into segments of
// `seg_len` tiles. A work item is one segment of one chain, and
// items are numbered segment-major, so an item's predecessor (the previous
// segment of the same chain) is numbered `chains` earlier. One persistent CTA
// per SM takes items blockIdx.x, blockIdx.x + gridDim.x, ... and walks each
// item's tiles in order with the state h kept in registers; only at a segment
// boundary does h travel through the workspace (a two-slot fp32 ring per
// chain, published with a release flag and read after a bounded acquire poll).
// Few chains cut into many segments would wait on each other's states one
// after another; they run segment-parallel instead, in three launches: every
// segment's local end state and total decay (mode 1, the state path only), a
// scan over the segments (segment_scan_kernel), then every segment's outputs
// from its scanned entering state (mode 2). A state dim above 128 runs as two
// passes over the state columns, the second adding into y.
//
// Warp roles inside the CTA (416 threads), linked by full/empty mbarrier rings
// whose waits sleep rather than spin:
//   warp 0        TMA producer: C, B (2 stages) and X (2 stages) as two
//                 independent streams, L2 prefetch of the X tiles further
//                 ahead; TMEM allocation
//   warp 1        MMA stream A: MMA1 and states of each tile
//   warp 2        MMA stream B: MMA2 and MMA3 of each tile (S is double
//                 buffered in TMEM, so stream A runs a tile ahead of stream B)
// The producer and MMA warps run their loops warp-wide and issue from one
// elected lane, with the shared-memory descriptors built once per stage (a K
// step only moves the start address), which keeps the issue path short.
//   warps 3, 12   tile prologue: cumsum, column factors, w o X
//   warps 4-7     mask S -> S~, in place in TMEM
//   warps 8-11    h_prev -> bf16 operand, state update, epilogue through a
//                 TMA store (a TMA reduce-add in a second pass over the
//                 state columns), look-back and segment publication
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

constexpr int kT = 128;   // tokens per tile
constexpr int kP = 64;    // channels of a tile's head (a head of P = 64m runs as m of them)
constexpr int kN = 128;   // state dim of a pass; a smaller N is zero-padded, a larger one takes two passes
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint64_t kMbarLimit = 1ull << 22;  // polls; each wait is also capped at ~2 s

constexpr int kThreads = 416;
constexpr int kWarpProducer = 0;
constexpr int kWarpMmaA = 1;   // MMA1 and states
constexpr int kWarpMmaB = 2;   // MMA2 and MMA3
constexpr int kWarpPrepA = 3;  // prologue: warps 3 and 12
constexpr int kWarpPrepB = 12;
constexpr int kWarpAlloc = 0;
constexpr int kWgMask0 = 4;    // warps 4..7
constexpr int kWgOut0 = 8;     // warps 8..11
constexpr int kBarPrep = 1;    // named barrier ids
constexpr int kBarOut = 2;

constexpr int kCbStages = 2;
constexpr int kXStages = 2;
constexpr int kCsStages = 4;
constexpr int kPrefetchAhead = 2;

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t kColS = 0;     // 2 x 128: S, then S~ (bf16, cols 0-63) and Ys (cols 64-127)
constexpr uint32_t kColSt = 256;  // 2 x 64: tile states, lanes = n
constexpr uint32_t kColY = 384;   // 2 x 64: Yd
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kTileBytesCB = kT * kN * 2;  // one C or B tile: 32 KB
constexpr uint32_t kTileBytesX = kT * kP * 2;   // one X tile: 16 KB

struct TcParams {
    const float* dt;
    const float* A;
    const float* D;
    const float* init;
    __nv_bfloat16* y;
    float* final_state;
    unsigned long long* flags;  // per chain: (epoch, number of segments published)
    uint32_t epoch;             // tag of this call (see LaunchCtx)
    float* ring;          // per chain: 2 slots of [N][P] fp32
    // Segment-parallel form (chains with many segments): `mode` 1 computes each
    // segment's local end state from zero and its total log2 decay, running only
    // the state path (B and X loads, w o X, the tile states, h); mode 2 starts
    // each segment from the state that a scan over those wrote to seg_hin (no
    // look-back, no publication); mode 0 is the single pass with look-back.
    int mode;
    float* seg_state;     // [chain][seg][kN][kP]
    float* seg_decay;     // [chain][seg]
    const float* seg_hin; // [chain][seg][kN][kP]
    unsigned int* status;
    unsigned long long wait_limit;
    int B, L, G;
    // A head with P = sub * kP channels runs as `sub` heads of kP channels
    // (each row of the P x N state evolves on its own, and x, y [B][L][H][P]
    // and the states [B][H][P][N] read as [B][L][H sub][kP] and
    // [B][H sub][kP][N]); those share the head's dt, A and D.
    int H;        // heads of kP channels (H_model * sub)
    int Hr;       // heads of the model: dt [B][L][Hr], A and D [Hr]
    int sub;      // kP-channel heads per model head
    // A state dim above kN runs as two passes over the state columns
    // [n_off, n_off + N): the output is linear in the state columns (y sums
    // C_i,n h_n and the masked C_i,n B_j,n over n), so the second pass adds its
    // share into y (TMA reduce-add) and leaves out the D x term.
    int N;        // state columns of this pass (<= kN)
    int n_off;    // first state column of this pass
    int ldn;      // state dim of Bm, Cm, initial and final state
    int accumulate;  // 1: add into y instead of storing it
    int nkh;      // 64-wide halves of the pass's state columns that hold data (1 or 2)
    int ntiles;   // tiles per chain
    int chains;   // B * H
    int seg_len;  // tiles per segment
    int nseg;     // segments per chain
    int items;    // chains * nseg
    int skip_publish;
};

// Per-tile prologue record (one per cumsum stage).
struct TileRec {
    float cs[kT];    // cumulative dt * A, log2 units
    float dt[kT];
    float colf[kT];  // exp2(cs[j | 31] - cs[j]) * dt[j]
    float w[kT];     // exp2(cs[kT - 1] - cs[j]) * dt[j]
    float Dh;
    float pad[31];
};

// Shared memory (offsets from a 1024-aligned base).
struct Smem {
    static constexpr uint32_t kC = 0;                                   // 2 x 32 KB
    static constexpr uint32_t kB = kC + kCbStages * kTileBytesCB;       // 2 x 32 KB (B, then S~)
    static constexpr uint32_t kX = kB + kCbStages * kTileBytesCB;       // 3 x 16 KB
    static constexpr uint32_t kXt = kX + kXStages * kTileBytesX;        // 16 KB
    static constexpr uint32_t kHs = kXt + kTileBytesX;                  // N x 64 bf16
    static constexpr uint32_t kYs = kHs + kN * kP * 2;                  // y staging, 16 KB
    static constexpr uint32_t kRec = kYs + kT * kP * 2;                 // 4 x TileRec
    static constexpr uint32_t kRed = kRec + kCsStages * sizeof(TileRec);  // 8 floats
    static constexpr uint32_t kBars = kRed + 32;
    static constexpr int kNumBars = 40;
    static constexpr uint32_t kTmemPtr = kBars + kNumBars * 8;
    static constexpr uint32_t kAbort = kTmemPtr + 4;
    static constexpr uint32_t kEnd = kAbort + 4;
    static constexpr uint32_t kBytes = kEnd + 1024;  // alignment slack
};
static_assert(Smem::kBytes <= 227 * 1024, "shared memory budget");

// mbarrier indices
enum Bar : int {
    kFullCB = 0,      // 2
    kEmptyCB = 2,     // 2 (two arrivals: after states, after MMA3)
    kFullX = 4,       // 3
    kEmptyX = 7,      // 3 (two arrivals: stream B's products and the w o X pass; one in mode 1)
    kFullXt = 10,
    kEmptyXt = 11,
    kFullRec = 12,    // 4
    kEmptyRec = 16,   // 4 (five arrivals: the four mask warps and the output warpgroup)
    kFullS = 20,      // 2: MMA1 done (S readable)
    kFullSt = 22,     // 2: S~ written over S in TMEM (one arrival per mask warp)
    kFullStates = 24, // 2
    kEmptyStates = 26,// 2
    kFullHs = 28,     // h_prev operand written
    kEmptyHs = 29,
    kFullY = 30,      // 2
    kEmptyY = 32,     // 2
    kDrain = 34,
};

// Position in this CTA's sequence of tiles (identical in every role).
struct Seq {
    int item, tile, tile_end, seg, chain, b, h;
    bool valid;

    __device__ __noinline__ void setup(const TcParams& p)
    {
        valid = item < p.items;
        if (!valid) return;
        seg = item / p.chains;
        chain = item - seg * p.chains;
        b = chain / p.H;
        h = chain - b * p.H;
        tile = seg * p.seg_len;
        tile_end = min(tile + p.seg_len, p.ntiles);
    }
    __device__ void begin(const TcParams& p)
    {
        item = blockIdx.x;
        setup(p);
    }
    __device__ void next(const TcParams& p)
    {
        if (++tile >= tile_end) {
            item += gridDim.x;
            setup(p);
        }
    }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Bounded wait that turns a give-up into the CTA's abort mode: from then on
// waits return at once, every role runs to the end of its loop on whatever is
// in its buffers, and the device status word reports the timeout.
__device__ __noinline__ void wait_gave_up(volatile int* abort_flag, unsigned int* status)
{
    record_status(status, kDevWaitTimeout);
    *abort_flag = 1;
}

// Bounded wait (polls, each of which may sleep; the clock is read every 256
// polls). The give-up path is out of line: it runs at most once per CTA.
__device__ __forceinline__ void wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                        unsigned int* status)
{
    if (*abort_flag) return;
    if (mbar_try_wait(bar, parity)) return;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return;
        if ((it & 255u) == 0u && (it >= kMbarLimit || global_timer_ns() - t0 > 2000000000ull)) break;
    }
    wait_gave_up(abort_flag, status);
}

__global__ void __launch_bounds__(kThreads, 1)
tc_forward_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmY,
                  TcParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the swizzle atoms, by offsetting the shared array
    // itself so that every access below stays in the shared address space
    uint8_t* sm = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::kBars);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + Smem::kTmemPtr);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Smem::kAbort);
    TileRec* recs = reinterpret_cast<TileRec*>(sm + Smem::kRec);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    // mode 1 needs only the tile states: no C, no MMA1 / mask / MMA2 / MMA3, no y
    const bool states_only = p.mode == 1;

    if (tid == 0) {
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmC);
        prefetch_tensormap(&tmY);
        for (int i = 0; i < Smem::kNumBars; ++i)
            mbar_init(bars + i, (i >= kEmptyRec && i < kEmptyRec + kCsStages) ? (states_only ? 1u : 5u)
                                : (i >= kFullSt && i < kFullSt + 2)          ? 4u
                                : (i >= kEmptyCB && i < kEmptyCB + 2)        ? (states_only ? 1u : 2u)
                                : (i >= kEmptyX && i < kEmptyX + kXStages)   ? (states_only ? 1u : 2u)
                                                                             : 1u);
        mbar_fence_init();
        *abort_flag = 0;
    }
    if (warp == kWarpAlloc) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    if (p.nkh == 1) {
        // N <= 64: the second half of every C/B tile is never loaded; zero it
        // once so the states MMA (which spans the full 128 rows) reads zeros
        for (int cb = 0; cb < kCbStages; ++cb)
            for (int base = 0; base < 2; ++base) {
                uint4* z = reinterpret_cast<uint4*>(sm + (base ? Smem::kB : Smem::kC) +
                                                    cb * kTileBytesCB + 16384);
                for (int u = tid; u < 16384 / 16; u += kThreads) z[u] = make_uint4(0u, 0u, 0u, 0u);
            }
        fence_async_shared();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *s_tmem;

    if (warp == kWarpProducer) {
        // ------------------------------------------------------------- producer
        // Two independent load streams, C/B (2 stages) and X (2 stages), each in
        // tile order: the warp polls both stage rings and issues whichever is
        // free, so a late X stage never holds back the next C/B tile. One
        // elected lane issues; the whole warp polls.
        Seq s, sx, pf;
        s.begin(p);
        sx = s;
        pf = s;
        for (int d = 0; d < kPrefetchAhead && pf.valid; ++d) pf.next(p);
        int k = 0, kx = 0;
        uint64_t idle_since = 0;
        while (s.valid || sx.valid) {
            if (*abort_flag) break;
            bool issued = false;
            if (s.valid) {
                const int cb = k % kCbStages;
                const bool ready = __shfl_sync(0xffffffffu,
                    mbar_test_wait(bars + kEmptyCB + cb, ((k / kCbStages) & 1) ^ 1) ? 1 : 0, 0) != 0;
                if (ready) {
                    const int g = s.h / (p.H / p.G);
                    const int t0 = s.tile * kT;
                    if (elect_one_sync()) {
                        if (pf.valid) tma_prefetch_l2_4d(&tmX, 0, pf.h, pf.tile * kT, pf.b);
                        mbar_arrive_expect_tx(bars + kFullCB + cb,
                                              p.nkh * (states_only ? 1 : 2) * 16384);
#pragma unroll
                        for (int q = 0; q < kN / 64; ++q) {
                            if (q >= p.nkh) break;
                            if (!states_only)
                                tma_load_4d(sm + Smem::kC + cb * kTileBytesCB + q * 16384, &tmC, p.n_off + q * 64,
                                            g, t0, s.b, bars + kFullCB + cb);
                            tma_load_4d(sm + Smem::kB + cb * kTileBytesCB + q * 16384, &tmB, p.n_off + q * 64, g,
                                        t0, s.b, bars + kFullCB + cb);
                        }
                    }
                    __syncwarp();
                    ++k;
                    s.next(p);
                    if (pf.valid) pf.next(p);
                    issued = true;
                }
            }
            if (sx.valid) {
                const int xs = kx % kXStages;
                const bool ready = __shfl_sync(0xffffffffu,
                    mbar_test_wait(bars + kEmptyX + xs, ((kx / kXStages) & 1) ^ 1) ? 1 : 0, 0) != 0;
                if (ready) {
                    if (elect_one_sync()) {
                        mbar_arrive_expect_tx(bars + kFullX + xs, kTileBytesX);
                        tma_load_4d(sm + Smem::kX + xs * kTileBytesX, &tmX, 0, sx.h, sx.tile * kT,
                                    sx.b, bars + kFullX + xs);
                    }
                    __syncwarp();
                    ++kx;
                    sx.next(p);
                    issued = true;
                }
            }
            if (issued) {
                idle_since = 0;
            } else {
                // nothing free: back off, and give up after ~2 s without progress
                const uint64_t now = global_timer_ns();
                if (idle_since == 0) {
                    idle_since = now;
                } else if (now - idle_since > 2000000000ull) {
                    if (lane == 0) wait_gave_up(abort_flag, p.status);
                    __syncwarp();
                    break;
                }
                __nanosleep(64);
            }
        }
        // drain: every load issued has landed before the CTA can exit
        for (int j = max(0, k - kCbStages); j < k; ++j)
            mbar_wait(bars + kFullCB + j % kCbStages, (j / kCbStages) & 1, kMbarLimit);
        for (int j = max(0, kx - kXStages); j < kx; ++j)
            mbar_wait(bars + kFullX + j % kXStages, (j / kXStages) & 1, kMbarLimit);
    } else if (warp == kWarpMmaA) {
        // ---------------------------------------------- stream A: MMA1, states
        constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
        constexpr uint32_t id_st = idesc_bf16(128, kP, true, true);
        // descriptors of stage 0; a stage or K step only moves the start address
        const uint64_t dc0 = sdesc_sw128(smem_addr(sm + Smem::kC), 16, 1024);
        const uint64_t db0 = sdesc_sw128(smem_addr(sm + Smem::kB), 16, 1024);
        const uint64_t dbt0 = sdesc_sw128(smem_addr(sm + Smem::kB), 16384, 1024);  // B^T, MN-major
        const uint64_t dxt = sdesc_sw128(smem_addr(sm + Smem::kXt), 16384, 1024);
        Seq s;
        s.begin(p);
        for (int k = 0; s.valid; ++k, s.next(p)) {
            const int cb = k % kCbStages, sb = k & 1;
            const uint64_t dc = dc0 + cb * (kTileBytesCB >> 4);
            const uint64_t db = db0 + cb * (kTileBytesCB >> 4);
            const uint64_t dbt = dbt0 + cb * (kTileBytesCB >> 4);
            wait_bar(bars + kFullCB + cb, (k / kCbStages) & 1, abort_flag, p.status);
            // S[sb] held S~ and Ys of tile k-2 until its epilogue read them
            if (k >= 2 && !states_only)
                wait_bar(bars + kEmptyY + sb, ((k - 2) >> 1) & 1, abort_flag, p.status);
            tc_fence_after_sync();
            if (!states_only && elect_one_sync()) {
#pragma unroll
                for (int q = 0; q < kN / 16; ++q) {
                    if (q >= 4 * p.nkh) break;
                    const uint32_t off = ((q >> 2) * 16384 + (q & 3) * 32) >> 4;
                    mma_bf16(tmem + kColS + sb * 128, dc + off, db + off, id_s, q > 0);
                }
                mma_commit(bars + kFullS + sb);
            }
            __syncwarp();
            wait_bar(bars + kEmptyStates + sb, ((k >> 1) & 1) ^ 1, abort_flag, p.status);
            wait_bar(bars + kFullXt, k & 1, abort_flag, p.status);
            tc_fence_after_sync();
            if (elect_one_sync()) {
#pragma unroll
                for (int q = 0; q < kT / 16; ++q)
                    mma_bf16(tmem + kColSt + sb * 64, dbt + q * (2048 >> 4), dxt + q * (2048 >> 4), id_st,
                             q > 0);
                mma_commit(bars + kEmptyXt);
                mma_commit(bars + kFullStates + sb);
                mma_commit(bars + kEmptyCB + cb);
            }
            __syncwarp();
        }
        if (elect_one_sync()) mma_commit(bars + kDrain);
        __syncwarp();
        mbar_wait(bars + kDrain, 0, kMbarLimit);
    } else if (warp == kWarpMmaB && !states_only) {
        // ----------------------------------------------- stream B: MMA2, MMA3
        constexpr uint32_t id_y2 = idesc_bf16(128, kP, false, true);
        const uint64_t dc0 = sdesc_sw128(smem_addr(sm + Smem::kC), 16, 1024);
        const uint64_t dx0 = sdesc_sw128(smem_addr(sm + Smem::kX), 16384, 1024);
        const uint64_t dhs = sdesc_sw128(smem_addr(sm + Smem::kHs), 16384, 1024);
        Seq s;
        s.begin(p);
        for (int k = 0; s.valid; ++k, s.next(p)) {
            const int cb = k % kCbStages, xs = k % kXStages, sb = k & 1;
            const uint64_t dc = dc0 + cb * (kTileBytesCB >> 4);
            const uint64_t dx = dx0 + xs * (kTileBytesX >> 4);
            wait_bar(bars + kFullSt + sb, (k >> 1) & 1, abort_flag, p.status);
            wait_bar(bars + kEmptyY + sb, ((k >> 1) & 1) ^ 1, abort_flag, p.status);
            wait_bar(bars + kFullX + xs, (k / kXStages) & 1, abort_flag, p.status);
            tc_fence_after_sync();
            if (elect_one_sync()) {
#pragma unroll
                for (int q = 0; q < kT / 16; ++q)
                    mma_bf16_tmem_a(tmem + kColY + sb * 64, tmem + kColS + sb * 128 + q * 8,
                                    dx + q * (2048 >> 4), id_y2, q > 0);
            }
            __syncwarp();
            wait_bar(bars + kFullCB + cb, (k / kCbStages) & 1, abort_flag, p.status);
            wait_bar(bars + kFullHs, k & 1, abort_flag, p.status);
            tc_fence_after_sync();
            if (elect_one_sync()) {
#pragma unroll
                for (int q = 0; q < kN / 16; ++q) {
                    if (q >= 4 * p.nkh) break;
                    mma_bf16(tmem + kColS + sb * 128 + 64, dc + (((q >> 2) * 16384 + (q & 3) * 32) >> 4),
                             dhs + q * (2048 >> 4), id_y2, q > 0);
                }
                mma_commit(bars + kFullY + sb);
                mma_commit(bars + kEmptyHs);
                mma_commit(bars + kEmptyX + xs);
                mma_commit(bars + kEmptyCB + cb);
            }
            __syncwarp();
        }
        if (elect_one_sync()) mma_commit(bars + kDrain + 1);
        __syncwarp();
        mbar_wait(bars + kDrain + 1, 0, kMbarLimit);
    } else if (warp == kWarpPrepA || warp == kWarpPrepB) {
        // ------------------------------------- prologue: cumsum, factors, w o X
        const int wq = warp == kWarpPrepA ? 0 : 1;
        const int t = wq * 32 + lane;  // 0..63, tokens 2t and 2t + 1
        float* red = reinterpret_cast<float*>(sm + Smem::kRed);
        Seq s;
        s.begin(p);
        float2 dt_next = make_float2(0.f, 0.f);
        float A_next = 0.f, D_next = 0.f;
        auto fetch = [&](const Seq& q) {
            const int rows = min(kT, p.L - q.tile * kT);
            const int hr = p.sub == 1 ? q.h : q.h / p.sub;  // the model head
            const size_t base = (static_cast<size_t>(q.b) * p.L + q.tile * kT) * p.Hr + hr;
            dt_next.x = 2 * t < rows ? p.dt[base + static_cast<size_t>(2 * t) * p.Hr] : 0.f;
            dt_next.y = 2 * t + 1 < rows ? p.dt[base + static_cast<size_t>(2 * t + 1) * p.Hr] : 0.f;
            A_next = p.A[hr];
            D_next = p.D ? p.D[hr] : 0.f;
        };
        if (s.valid) fetch(s);
        for (int k = 0; s.valid; ++k) {
            const int c = k % kCsStages, xs = k % kXStages;
            TileRec& r = recs[c];
            const float2 dtv = dt_next;
            const float Ah = A_next * kLog2e;
            const float Dh = D_next;
            s.next(p);
            if (s.valid) fetch(s);

            wait_bar(bars + kEmptyRec + c, ((k / kCsStages) & 1) ^ 1, abort_flag, p.status);
            const float a0 = dtv.x * Ah;
            const float a1 = a0 + dtv.y * Ah;
            float v = a1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (lane == 31) red[wq] = v;
            named_bar_sync(kBarPrep, 64);
            const float excl = v - a1 + (wq == 1 ? red[0] : 0.f);
            r.cs[2 * t] = excl + a0;
            r.cs[2 * t + 1] = excl + a1;
            r.dt[2 * t] = dtv.x;
            r.dt[2 * t + 1] = dtv.y;
            if (t == 0) r.Dh = Dh;
            named_bar_sync(kBarPrep, 64);
            const float cs_end = r.cs[kT - 1];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int j = 2 * t + e;
                const float csj = r.cs[j];
                const float dj = e ? dtv.y : dtv.x;
                r.colf[j] = ex2_approx(r.cs[j | 31] - csj) * dj;
                r.w[j] = ex2_approx(cs_end - csj) * dj;
            }
            named_bar_sync(kBarPrep, 64);
            if (t == 0) mbar_arrive(bars + kFullRec + c);

            // X~ = w o X (row j of the swizzled tile is the 128 bytes at j * 128)
            wait_bar(bars + kFullX + xs, (k / kXStages) & 1, abort_flag, p.status);
            wait_bar(bars + kEmptyXt, (k & 1) ^ 1, abort_flag, p.status);
            {
                const uint4* src = reinterpret_cast<const uint4*>(sm + Smem::kX + xs * kTileBytesX);
                uint4* dst = reinterpret_cast<uint4*>(sm + Smem::kXt);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint4 v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) v[q] = src[t + (half * 8 + q) * 64];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const int chunk = t + (half * 8 + q) * 64;
                        const __nv_bfloat162 w2 = __float2bfloat162_rn(r.w[chunk >> 3]);
                        __nv_bfloat162* e = reinterpret_cast<__nv_bfloat162*>(&v[q]);
#pragma unroll
                        for (int u = 0; u < 4; ++u) e[u] = __hmul2(e[u], w2);
                        dst[chunk] = v[q];
                    }
                }
            }
            fence_async_shared();
            named_bar_sync(kBarPrep, 64);
            if (t == 0) {
                mbar_arrive(bars + kFullXt);
                // the X stage is free once w o X has read it as well: stream B's
                // products finishing first does not mean this read is done
                mbar_arrive(bars + kEmptyX + xs);
            }
        }
    } else if (warp >= kWgMask0 && warp < kWgMask0 + 4 && !states_only) {
        // ------------------------------------------- mask S -> S~ (in place, TMEM)
        // S~ (bf16 pairs) overwrites the first 64 columns of the tile's S: block
        // jb of S~ lands on columns 16 jb .. 16 jb + 15, which hold S values that
        // were read before (blocks <= jb), so reads always stay ahead of writes.
        const int wq = warp - kWgMask0;  // lane quadrant: rows 32 wq .. 32 wq + 31
        const int i = wq * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        Seq s;
        s.begin(p);
        for (int k = 0; s.valid; ++k, s.next(p)) {
            const int c = k % kCsStages, sb = k & 1;
            const TileRec& r = recs[c];
            wait_bar(bars + kFullRec + c, (k / kCsStages) & 1, abort_flag, p.status);
            wait_bar(bars + kFullS + sb, (k >> 1) & 1, abort_flag, p.status);
            tc_fence_after_sync();
            const float cs_i = r.cs[i];
            const float Dh = r.Dh;
            const uint32_t s_col = tmem + lane_off + kColS + sb * 128;
#pragma unroll 1
            for (int jb = 0; jb < 4; ++jb) {
                uint32_t packed[16];
                if (jb < wq) {
                    // block wholly left of the diagonal: row factor x column factor
                    float sv[32];
                    {
                        uint32_t raw[32];
                        tmem_ld32_sync(s_col + jb * 32, raw);
#pragma unroll
                        for (int q = 0; q < 32; ++q) sv[q] = __uint_as_float(raw[q]);
                    }
                    const float rf = ex2_approx(cs_i - r.cs[jb * 32 + 31]);
                    const float4* cf = reinterpret_cast<const float4*>(r.colf + jb * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 f = cf[q];
                        packed[q * 2] = pack_bf16x2(sv[q * 4] * f.x * rf, sv[q * 4 + 1] * f.y * rf);
                        packed[q * 2 + 1] =
                            pack_bf16x2(sv[q * 4 + 2] * f.z * rf, sv[q * 4 + 3] * f.w * rf);
                    }
                } else if (jb == wq) {
                    // block on the diagonal. Every lane evaluates every term and the
                    // position only selects values: rows diverge on j < i, and a
                    // per-element branch would serialise the warp.
                    float sv[32];
                    {
                        uint32_t raw[32];
                        tmem_ld32_sync(s_col + jb * 32, raw);
#pragma unroll
                        for (int q = 0; q < 32; ++q) sv[q] = __uint_as_float(raw[q]);
                    }
                    const float4* cs4 = reinterpret_cast<const float4*>(r.cs + jb * 32);
                    const float4* dt4 = reinterpret_cast<const float4*>(r.dt + jb * 32);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 c4 = cs4[q];
                        const float4 d4 = dt4[q];
                        const float csj[4] = {c4.x, c4.y, c4.z, c4.w};
                        const float dtj[4] = {d4.x, d4.y, d4.z, d4.w};
                        float m[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int jj = q * 4 + e;
                            const float below = sv[jj] * ex2_approx(fminf(cs_i - csj[e], 0.f)) * dtj[e];
                            const float diag = fmaf(sv[jj], dtj[e], Dh);
                            const float v = jj < lane ? below : 0.f;
                            m[e] = jj == lane ? diag : v;
                        }
                        packed[q * 2] = pack_bf16x2(m[0], m[1]);
                        packed[q * 2 + 1] = pack_bf16x2(m[2], m[3]);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) packed[q] = 0u;
                }
                tmem_st16(s_col + jb * 16, packed);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bars + kFullSt + sb);
                mbar_arrive(bars + kEmptyRec + c);
            }
        }
    } else if (warp >= kWgOut0 && warp < kWgOut0 + 4) {
        // ------------------ h_prev operand, state, epilogue, look-back, publish
        const int wq = warp - kWgOut0;
        const int n = wq * 32 + lane;  // state row / tile row / TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const size_t PN = static_cast<size_t>(kP) * p.ldn;
        const bool n_live = n < p.N;  // rows past the pass's columns are zero padding
        float h[kP];
        float lam = 0.f;  // log2 decay of the segment so far (mode 1)
        // the bf16 h_prev operand of MMA3 for tile kk (row n of [N][P],
        // MN-major), once MMA3 of tile kk - 1 has read the previous one
        auto write_hs = [&](int kk) {
            wait_bar(bars + kEmptyHs, (kk & 1) ^ 1, abort_flag, p.status);
            uint8_t* row = sm + Smem::kHs + n * 128;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint4 v = make_uint4(pack_bf16x2(h[q * 8 + 0], h[q * 8 + 1]),
                                           pack_bf16x2(h[q * 8 + 2], h[q * 8 + 3]),
                                           pack_bf16x2(h[q * 8 + 4], h[q * 8 + 5]),
                                           pack_bf16x2(h[q * 8 + 6], h[q * 8 + 7]));
                *reinterpret_cast<uint4*>(row + (((q ^ n) & 7) << 4)) = v;
            }
            fence_async_shared();
            named_bar_sync(kBarOut, 128);
            if (n == 0) mbar_arrive(bars + kFullHs);
        };
        Seq s;
        s.begin(p);
        for (int k = 0; s.valid; ++k, s.next(p)) {
            const bool first = s.tile == s.seg * p.seg_len;
            const bool last = s.tile == s.tile_end - 1;
            const int c = k % kCsStages, sb = k & 1;
            if (first) {
                // the state entering this segment: zero (a segment's local state,
                // mode 1), the initial state (first segment), or the state the
                // predecessor published (mode 0, after a bounded acquire poll) or
                // the scan wrote (mode 2)
                lam = 0.f;
                if (p.mode == 1 || (s.seg == 0 && !p.init)) {
#pragma unroll
                    for (int q = 0; q < kP; ++q) h[q] = 0.f;
                } else if (s.seg == 0) {
                    const float* src = p.init + static_cast<size_t>(s.chain) * PN + p.n_off + n;
#pragma unroll
                    for (int q = 0; q < kP; ++q) h[q] = n_live ? src[static_cast<size_t>(q) * p.ldn] : 0.f;
                } else {
                    if (p.mode == 0) {
                        if (n == 0 && !*abort_flag) {
                            const unsigned long long* f = p.flags + s.chain;
                            bool ok = false;
                            const uint64_t t0 = global_timer_ns();
                            for (unsigned long long it = 0; it < p.wait_limit; ++it) {
                                const uint64_t v = ld_acquire_gpu_u64(f);
                                if (static_cast<uint32_t>(v >> 32) == p.epoch &&
                                    static_cast<uint32_t>(v) >= static_cast<uint32_t>(s.seg)) {
                                    ok = true;
                                    break;
                                }
                                if ((it & 255) == 255 && global_timer_ns() - t0 > 4000000000ull) break;
                                __nanosleep(64);
                            }
                            if (!ok) {
                                record_status(p.status, kDevWaitTimeout);
                                *abort_flag = 1;
                            }
                        }
                        named_bar_sync(kBarOut, 128);
                    }
                    const size_t slot = p.mode == 2
                                            ? static_cast<size_t>(s.chain) * p.nseg + s.seg
                                            : static_cast<size_t>(s.chain) * 2 + ((s.seg - 1) & 1);
                    const float4* src = reinterpret_cast<const float4*>(
                        (p.mode == 2 ? p.seg_hin : p.ring) + (slot * kN + n) * kP);
#pragma unroll
                    for (int q = 0; q < kP / 4; ++q) {
                        const float4 v = __ldcg(src + q);
                        h[q * 4 + 0] = v.x;
                        h[q * 4 + 1] = v.y;
                        h[q * 4 + 2] = v.z;
                        h[q * 4 + 3] = v.w;
                    }
                }
            }
            const TileRec& r = recs[c];
            wait_bar(bars + kFullRec + c, (k / kCsStages) & 1, abort_flag, p.status);
            const float cs_n = r.cs[n];
            const float cs_end = r.cs[kT - 1];
            const float dec = ex2_approx(cs_end);
            if (!states_only) write_hs(k);

            // h = exp(cs_end) h_prev + s
            wait_bar(bars + kFullStates + sb, (k >> 1) & 1, abort_flag, p.status);
            tc_fence_after_sync();
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                float sv[32];
                {
                    uint32_t raw[32];
                    tmem_ld32_sync(tmem + lane_off + kColSt + sb * 64 + half * 32, raw);
#pragma unroll
                    for (int q = 0; q < 32; ++q) sv[q] = __uint_as_float(raw[q]);
                }
#pragma unroll
                for (int q = 0; q < 32; ++q) h[half * 32 + q] = dec * h[half * 32 + q] + sv[q];
            }
            tc_fence_before_sync();
            named_bar_sync(kBarOut, 128);
            if (n == 0) mbar_arrive(bars + kEmptyStates + sb);

            if (states_only) lam += cs_end;
            if (last) {
                if (s.tile == p.ntiles - 1) {
                    if (p.final_state && n_live) {
                        float* dst = p.final_state + static_cast<size_t>(s.chain) * PN + p.n_off + n;
#pragma unroll
                        for (int q = 0; q < kP; ++q) dst[static_cast<size_t>(q) * p.ldn] = h[q];
                    }
                } else if (p.mode != 2) {
                    // mode 0 publishes the segment's end state to the ring; mode 1
                    // stores the local end state and the segment's decay
                    const size_t slot = p.mode == 1 ? static_cast<size_t>(s.chain) * p.nseg + s.seg
                                                    : static_cast<size_t>(s.chain) * 2 + (s.seg & 1);
                    float4* dst = reinterpret_cast<float4*>((p.mode == 1 ? p.seg_state : p.ring) +
                                                            (slot * kN + n) * kP);
#pragma unroll
                    for (int q = 0; q < kP / 4; ++q)
                        dst[q] = make_float4(h[q * 4], h[q * 4 + 1], h[q * 4 + 2], h[q * 4 + 3]);
                    if (p.mode == 1) {
                        if (n == 0) p.seg_decay[slot] = lam;
                    } else {
                        __threadfence();
                        named_bar_sync(kBarOut, 128);
                        if (n == 0 && !p.skip_publish)
                            st_release_gpu_u64(p.flags + s.chain,
                                               tagged(p.epoch, static_cast<uint32_t>(s.seg + 1)));
                    }
                }
            }

            if (states_only) {
                // no outputs in this pass: the record is free once every output
                // warp has read it (the named barrier after the state update)
                if (n == 0) mbar_arrive(bars + kEmptyRec + c);
                continue;
            }

            // epilogue: y_n = Yd_n + exp(cs_n) Ys_n (bf16), staged in shared memory
            // (128-byte swizzle) and written by one TMA store, which also clips
            // the rows of a ragged last tile
            wait_bar(bars + kFullY + sb, (k >> 1) & 1, abort_flag, p.status);
            if (n == 0) tma_store_wait_read();  // previous tile's store has read the stage
            named_bar_sync(kBarOut, 128);
            tc_fence_after_sync();
            {
                const float en = ex2_approx(cs_n);
                uint8_t* yrow = sm + Smem::kYs + n * 128;
#pragma unroll
                for (int qd = 0; qd < 4; ++qd) {
                    float yd[16], ys[16];
                    {
                        uint32_t ra[16], rb[16];
                        tmem_ld16x2_sync(tmem + lane_off + kColY + sb * 64 + qd * 16, ra,
                                         tmem + lane_off + kColS + sb * 128 + 64 + qd * 16, rb);
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            yd[q] = __uint_as_float(ra[q]);
                            ys[q] = __uint_as_float(rb[q]);
                        }
                    }
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t o[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c2 = h2 * 8 + e * 2;
                            o[e] = pack_bf16x2(fmaf(en, ys[c2], yd[c2]), fmaf(en, ys[c2 + 1], yd[c2 + 1]));
                        }
                        const int chunk = qd * 2 + h2;
                        *reinterpret_cast<uint4*>(yrow + (((chunk ^ n) & 7) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
            fence_async_shared();
            tc_fence_before_sync();
            named_bar_sync(kBarOut, 128);
            if (n == 0) {
                if (p.accumulate)
                    tma_reduce_add_4d(&tmY, sm + Smem::kYs, 0, s.h, s.tile * kT, s.b);
                else
                    tma_store_4d(&tmY, sm + Smem::kYs, 0, s.h, s.tile * kT, s.b);
                tma_store_commit();
                mbar_arrive(bars + kEmptyY + sb);
                mbar_arrive(bars + kEmptyRec + c);
            }
        }
    }

    if (warp == kWgOut0 && lane == 0) tma_store_wait_all();

    // ---- teardown
    __syncwarp();
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpAlloc) tmem_dealloc(tmem, kTmemCols);
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

// Heads of kP channels: a model head of P = sub * kP channels is sub of them.
int tile_heads(const FwdArgs& a) { return a.H * (a.P / kP); }

// Segments per chain: enough items for about `per_cta` per CTA, at least one
// tile each.
void choose_segments(int ntiles, int chains, int ctas, int per_cta, int* seg_len, int* nseg)
{
    long long want = (static_cast<long long>(per_cta) * ctas + chains - 1) / chains;
    if (want < 1) want = 1;
    if (want > ntiles) want = ntiles;
    *seg_len = static_cast<int>((ntiles + want - 1) / want);
    *nseg = (ntiles + *seg_len - 1) / *seg_len;
}

// Segments are numbered segment-major and handed out round-robin, so a
// segment's predecessor is `chains` items earlier. With fewer chains than
// half the CTAs, several segments of one chain run in the same round and wait
// on each other's published states one after another; such chains, cut into
// this many segments or more, run segment-parallel (three launches) instead.
// (Measured: 32 chains of 512 tiles 1.60 ms single pass, 0.70 ms parallel;
// 128 chains of 64 tiles 0.26 ms single pass, 0.43 ms parallel.)
constexpr int kParallelSegments = 8;
// Items per CTA: the single pass takes about four (each segment boundary
// costs a state hand-off, and four rounds still balance: 4.3 items per CTA
// at 320 chains ran 4% faster than 8.6, and 12 or 16 ran slower); the
// segment-parallel form, whose segments do not wait on each other, about eight.
constexpr int kItemsPerCtaSingle = 4;
constexpr int kItemsPerCtaParallel = 8;

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    return n;
}

struct Segments {
    int ntiles, chains, seg_len, nseg;
    bool parallel;
};

Segments segments(const FwdArgs& a, int ctas)
{
    Segments g;
    g.ntiles = (a.L + kT - 1) / kT;
    g.chains = a.B * tile_heads(a);
    choose_segments(g.ntiles, g.chains, ctas, kItemsPerCtaSingle, &g.seg_len, &g.nseg);
    g.parallel = g.nseg >= kParallelSegments && 2 * g.chains < ctas;
    if (g.parallel) choose_segments(g.ntiles, g.chains, ctas, kItemsPerCtaParallel, &g.seg_len, &g.nseg);
    return g;
}

struct WsLayout {
    size_t ctrl, flags, ring, seg_state, seg_decay, seg_hin, total;
};

WsLayout ws_layout(const FwdArgs& a, const Segments& g)
{
    WsLayout w;
    const size_t chains = static_cast<size_t>(a.B) * tile_heads(a);
    const size_t slot = static_cast<size_t>(kP) * kN * sizeof(float);
    w.ctrl = 0;
    w.flags = 256;
    w.ring = w.flags + ((chains * 8 + 255) / 256) * 256;
    w.total = w.ring + chains * 2 * slot;
    w.seg_state = w.seg_decay = w.seg_hin = w.total;
    if (g.parallel) {
        const size_t units = chains * g.nseg;
        w.seg_state = w.total;
        w.seg_decay = w.seg_state + units * slot;
        w.seg_hin = w.seg_decay + ((units * 4 + 255) / 256) * 256;
        w.total = w.seg_hin + units * slot;
    }
    return w;
}

int g_skip_publish = 0;

// The state entering every segment of a chain, from the segments' local end
// states and decays: h_in(0) = initial state, h_in(s + 1) = 2^decay(s) h_in(s)
// + local(s) (the composition of affine maps of "Selective SSM guide", eq. (3),
// applied segment by segment). One thread per state element of a chain
// (blockIdx.y = chain); states are [kN][kP] with rows past N zero, and the
// initial state's columns [n_off, n_off + N) of its ldn feed this pass.
constexpr int kScanThreads = 256;
static_assert(kN * kP % kScanThreads == 0, "scan grid covers the state exactly");

__global__ void __launch_bounds__(kScanThreads)
segment_scan_kernel(const float* init, const float* seg_state, const float* seg_decay,
                    float* seg_hin, int P, int N, int n_off, int ldn, int nseg)
{
    const size_t chain = blockIdx.y;
    const int e = blockIdx.x * kScanThreads + threadIdx.x;  // < kN * kP by the grid
    const int n = e / kP, q = e - n * kP;
    float v = init && n < N ? init[(chain * P + q) * ldn + n_off + n] : 0.f;
    const size_t u0 = chain * nseg;
#pragma unroll 8
    for (int sg = 0; sg < nseg; ++sg) {
        seg_hin[(u0 + sg) * kN * kP + e] = v;
        if (sg + 1 < nseg)
            v = fmaf(exp2f(__ldg(seg_decay + u0 + sg)), v, __ldcg(seg_state + (u0 + sg) * kN * kP + e));
    }
}

cudaError_t launch(const FwdArgs& a, void* workspace, const LaunchCtx& ctx)
{
    CUtensorMap tmX, tmB, tmC, tmY;
    const int Ht = tile_heads(a);
    if (!make_map(&tmX, a.x, kP, Ht, a.L, a.B) || !make_map(&tmB, a.Bm, a.N, a.G, a.L, a.B) ||
        !make_map(&tmC, a.Cm, a.N, a.G, a.L, a.B) || !make_map(&tmY, a.y, kP, Ht, a.L, a.B))
        return cudaErrorInvalidValue;
    const int ctas_max = ctx.num_sms > 0 ? ctx.num_sms : 1;
    const Segments g = segments(a, ctas_max);
    const WsLayout w = ws_layout(a, g);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    TcParams p;
    p.dt = a.dt;
    p.A = a.A;
    p.D = a.D;
    p.init = a.init;
    p.y = static_cast<__nv_bfloat16*>(a.y);
    p.final_state = a.final_state;
    p.flags = reinterpret_cast<unsigned long long*>(ws + w.flags);
    p.ring = reinterpret_cast<float*>(ws + w.ring);
    p.seg_state = reinterpret_cast<float*>(ws + w.seg_state);
    p.seg_decay = reinterpret_cast<float*>(ws + w.seg_decay);
    p.seg_hin = reinterpret_cast<const float*>(ws + w.seg_hin);
    p.status = ctx.status;
    p.wait_limit = ctx.wait_limit;
    p.B = a.B;
    p.L = a.L;
    p.H = Ht;
    p.Hr = a.H;
    p.sub = a.P / kP;
    p.G = a.G;
    p.ldn = a.N;
    p.ntiles = g.ntiles;
    p.chains = g.chains;
    p.seg_len = g.seg_len;
    p.nseg = g.nseg;
    p.skip_publish = g_skip_publish;
    const uint32_t smem = Smem::kBytes;
    cudaError_t e = cudaFuncSetAttribute(tc_forward_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int nlaunch = 0;
    auto run = [&](int mode, int items) {
        p.mode = mode;
        p.items = items;
        p.epoch = ctx.launch_tag(nlaunch++);
        const int grid = items < ctas_max ? items : ctas_max;
        tc_forward_kernel<<<grid, kThreads, smem, ctx.stream>>>(tmX, tmB, tmC, tmY, p);
        return cudaGetLastError();
    };
    // one pass per kN state columns; every pass after the first adds into y
    for (int n_off = 0; n_off < a.N; n_off += kN) {
        p.n_off = n_off;
        p.N = a.N - n_off < kN ? a.N - n_off : kN;
        p.nkh = p.N <= 64 ? 1 : 2;
        p.accumulate = n_off > 0;
        p.D = n_off > 0 ? nullptr : a.D;
        if (!g.parallel) {
            if ((e = run(0, g.chains * g.nseg)) != cudaSuccess) return e;
            continue;
        }
        // segment-parallel: local states of every segment but each chain's last
        // (segment-major numbering puts those first), the scan, then the outputs
        if ((e = run(1, g.chains * (g.nseg - 1))) != cudaSuccess) return e;
        segment_scan_kernel<<<dim3(kN * kP / kScanThreads, g.chains), kScanThreads, 0, ctx.stream>>>(
            a.init, p.seg_state, p.seg_decay, reinterpret_cast<float*>(ws + w.seg_hin), kP, p.N,
            n_off, a.N, g.nseg);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = run(2, g.chains * g.nseg)) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

bool tc_supported(const FwdArgs& a)
{
    return a.bf16 && a.P % kP == 0 && a.P >= kP && a.N % 8 == 0 && a.N >= 8 && a.N <= 2 * kN &&
           (a.chunk == 64 || a.chunk == 128 || a.chunk == 256) &&
           static_cast<long long>(a.B) * a.L > 0 &&
           static_cast<long long>((a.L + kT - 1) / kT) * a.B * a.H * (a.P / kP) < (1ll << 31);
}

size_t tc_workspace_bytes(const FwdArgs& a) { return ws_layout(a, segments(a, sm_count())).total; }

int tc_passes(const FwdArgs& a) { return (a.N + kN - 1) / kN; }

int tc_kernel_count(const FwdArgs& a)
{
    return tc_passes(a) * (segments(a, sm_count()).parallel ? 3 : 1);
}

bool tc_segment_parallel(const FwdArgs& a) { return segments(a, sm_count()).parallel; }

void tc_set_skip_publish(int v) { g_skip_publish = v; }

cudaError_t tc_forward(const FwdArgs& a, void* workspace, const LaunchCtx& ctx)
{
    if (!tc_supported(a)) return cudaErrorInvalidValue;
    return launch(a, workspace, ctx);
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
    // the same size checks as ssd_forward
    const ssd_status dims = check_dims(B, L, H, P, G, N, chunk, dtype);
    if (dims != SSD_OK) return dims;
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
    const WsLayout w = ws_layout(a, segments(a, sm_count()));
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
    // nothing in the array needs clearing: the look-back flags carry the tag
    // of the call that wrote them (see LaunchCtx::epoch)
    const cudaError_t e = tc_forward(a, scratch, ctx);
    return e == cudaSuccess ? SSD_OK : SSD_ERR_CUDA;
}
