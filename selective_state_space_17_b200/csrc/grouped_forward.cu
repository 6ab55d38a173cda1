// grouped_forward.cu — tensor-core (tcgen05) forward of the SSD layer with the
// heads of one B/C group processed together.
//
// "Mamba-2" (docsaid.org), section "Mamba-2 block", item 2: B and C are shared
// by every head of a group, like keys and queries shared across the heads of
// an attention layer. So for a 128-token tile the matrix S = C B^T is the same
// for every head of the group, and only the decay mask and X differ per head.
// This kernel takes KH heads of one group (KH = 2, or 1 when a group has an
// odd number of heads) through each tile together.
//
// The decay of a tile. With cs the tile-local cumulative sum of dt * A in
// log2 units (non-increasing, since dt >= 0 and A <= 0) and any reference
// value c, the mask of the masked form factors into a row and a column term,
//     2^(cs_i - cs_j) dt_j = 2^(cs_i - c) * (2^(c - cs_j) dt_j),
// which turns the per-head masked product into one shared matrix tril(S)
// times a per-head row-scaled X ("Mamba-2 SSD note" (0h-n0.github.io),
// section "SSD layer: equivalence under the scalar constraint": the mask is a
// product of decays, L_ij = a_i ... a_{j+1}). With c = cs_end / 2 every
// factor lies in [2^(cs_end/2), 2^(-cs_end/2)], so while the tile's total
// decay -cs_end stays below kHardLog2 nothing overflows or underflows. Per tile
// ("scaled form"):
//
//   MMA1    S   = C B^T                              (128 x 128, K = N), TMEM
//   mask    tril(S) as bf16 pairs, in place in TMEM (shared by the heads)
//   X'      X'_h = diag(2^(c_h - cs_h,j) dt_h,j) X_h  (in place in shared memory)
//   H'      H'_h = 2^(c_h) h_prev,h (bf16 operand), h <- 2^(c_h) h_prev,h in TMEM
//   Z init  Z_h,i = D_h x_h,i 2^(c_h - cs_h,i)          (the skip term over e_i)
//   MMA3    Z  += C [H'_0 ... H'_KH-1]^T             (128 x 64 KH, K = N)
//   MMA2    Z  += tril(S) [X'_0 ... X'_KH-1]         (128 x 64 KH, K = 128; A from TMEM)
//   states  h  += B^T [X'_0 ... X'_KH-1]             (N x 64 KH, K = 128), so that
//           h_new = 2^(cs_end - c) h (kept as a pending scalar)
//   output  y_h,i = e_h,i Z_h,i, e_h,i = 2^(cs_h,i - c_h)   (bf16, round to nearest even)
//
// A tile whose decay exceeds the bound ("exact form") keeps every factor <= 1:
// X'_h = diag(2^(cs_end - cs_j) dt_j) X_h feeds the states only, H' = h_prev,
// Z starts from 0, MMA3 adds C h_prev^T, the output warps scale row i of Z by
// 2^(cs_h,i) in place, and each head adds its own masked product
// S~_h X_h with S~_h,ij = tril(S)_ij 2^(cs_h,i - cs_h,j) dt_h,j (built per head
// in TMEM, X_h reloaded raw); then y = Z + D x. Both forms compute the chunked
// algorithm of "Mamba-2", section "Half of each route": the quadratic form
// inside a tile, the state across tiles (the composition of affine maps of
// "Selective SSM guide" (auturnal.com), eq. (3)).
//
// Schedule. A chain is one batch row and one head group. The pieces a CTA runs
// (see Pieces) come from a global ticket counter: each piece that starts
// inside a chain waits only on a piece that a running CTA took before it, so
// the look-back cannot deadlock however many CTAs are resident. The state h
// of the group's heads stays in TMEM from tile to tile; between pieces it
// travels through a per-chain slot in the workspace (release flag, bounded
// acquire poll).
//
// Warp roles (512 threads), linked by full/empty mbarriers whose waits sleep
// and are bounded (no named barriers, so a role that gives up cannot leave
// another stuck):
//   warp 0        producer: pieces, TMA loads of C, B (2 stages) and X (KH
//                 heads, 2 stages); TMEM allocation
//   warp 1        MMA issue: MMA3, MMA2 (the exact form's per-head products,
//                 with the raw X reload), MMA1 of the next tile
//   warp 2        MMA issue: states
//   warp 3        prologue: cumulative decay of the tile's heads, tile record
//   warps 4-7     state and mask: h_prev -> H' and the scaled h, piece
//                 hand-off and final state; then S -> tril(S) (exact form:
//                 S~_h per head)
//   warps 8-11    output: y = e Z staged in the tile's C buffer and stored by
//                 TMA (exact form: the row scaling of Z first, and y = Z + D x)
// The exact-form parts of warps 1, 4-7 and 8-11 are out-of-line functions: it
// is rare, and the hot loops of all roles together already miss in the SM's
// instruction cache, so code in them that never runs still costs time.
//   warps 12-15   scale: X' in place and Z's initial value
#include <cuda.h>
#include <cuda_bf16.h>

#include "grouped_forward.cuh"
#include "sm100.cuh"
#include "tma_map.cuh"

namespace ssd {
namespace grouped {
namespace {

using namespace sm100;

constexpr int kT = 128;  // tokens per tile
constexpr int kP = 64;   // channels of one head (a head of P = 64m is m of them)
constexpr int kN = 128;  // largest state dim; a smaller N is zero-padded
constexpr float kLog2e = 1.4426950408889634f;
// Tiles whose decay (log2 units) exceeds this take the exact form: the scaled
// form's factors then stay within 2^-72 .. 2^72.
constexpr float kHardLog2 = 144.f;
constexpr uint64_t kWaitNs = 2000000000ull;  // a role's wait on another gives up after ~2 s
constexpr uint32_t kWaitPolls = 1u << 24;     // ... or after this many polls (each at most ~128 ns)
constexpr uint32_t kRolePolls = 1u << 22;     // a role's wait on another: this many polls (<= 1 us each)

constexpr int kThreads = 512;  // 16 warps of at most 128 registers: the whole register file
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;    // MMA3, MMA2, MMA1
constexpr int kWarpMmaS = 2;   // states
constexpr int kWarpPro = 3;    // prologue of the tile's heads
constexpr int kWgState = 4;    // warps 4..7
constexpr int kWgOut = 8;      // warps 8..11
constexpr int kWgScale = 12;   // warps 12..15
constexpr int kSchedSlots = 4;
constexpr int kSchedConsumers = 15;  // warps 1..15 read every piece

// TMEM columns (fp32, 128 lanes)
constexpr uint32_t kColS = 0;    // 128: S, then tril(S) (bf16, cols 0-63) and S~_h (64-127)
constexpr uint32_t kColH = 128;  // KH x 64: the states h, lane = state row n
constexpr uint32_t kColZ = 256;  // 2 x (KH x 64): Z of even and odd tiles, lane = token
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kHalf = 16384;  // one 128 x 64 bf16 block (a head's X, half of C or B)

struct Rec {
    float cs[2][kT];  // cumulative dt * A per head, log2 units
    float cref[2];    // reference value c of the scaled form
    float csend[2];   // cs of the tile's last token
    int hard;         // exact form for this tile
    int pad[11];
};
static_assert(sizeof(Rec) == 1088, "record layout");

struct Smem {
    static constexpr uint32_t kC = 0;                    // 2 stages x 32 KB
    static constexpr uint32_t kB = kC + 4 * kHalf;       // 2 stages x 32 KB
    static constexpr uint32_t kX = kB + 4 * kHalf;       // 2 stages x KH x 16 KB (X, then X')
    static constexpr uint32_t kHp = kX + 4 * kHalf;      // KH x 16 KB: H' (exact form: raw X)
    static constexpr uint32_t kRec = kHp + 2 * kHalf;    // 2 records
    static constexpr uint32_t kSched = kRec + 2 * sizeof(Rec);
    static constexpr uint32_t kBars = kSched + 16 * 4;  // kSchedSlots pieces of 16 bytes
    static constexpr int kNumBars = 48;
    static constexpr uint32_t kTmemPtr = kBars + kNumBars * 8;
    static constexpr uint32_t kAbort = kTmemPtr + 4;
    static constexpr uint32_t kBytes = kAbort + 4;
};
static_assert(Smem::kBytes <= 227 * 1024, "shared memory budget");

enum Bar : int {
    kFullCB = 0,      // 2 (tx)
    kEmptyCB = 2,     // 2 (the two MMA warps, the TMA store of y staged in C)
    kFullX = 4,       // 2 (tx)
    kEmptyX = 6,      // 2 (the two MMA warps)
    kXpFull = 8,      // 2 (four scale warps)
    kRecFull = 10,    // 2 (the prologue warp)
    kRecEmpty = 12,   // 2 (MMA B, four state, four output and four scale warps)
    kSFull = 14,      // MMA1 wrote S
    kSFree = 16,      // MMA2 (exact form: the per-head products) read tril(S)
    kTrilFull = 18,   // 2 (four state warps)
    kHReady = 20,
    kHpFull = 21,
    kHpEmpty = 22,
    kStatesDone = 23,
    kZFull = 24,      // 2 (per Z buffer)
    kM3Done = 26,     // exact form
    kZScaled = 27,
    kRawX = 28,
    kSlotFull = 29,   // four state warps
    kSlotFree = 30,
    kSchedFull = 31,  // 4
    kSchedEmpty = 35, // 4 (kSchedConsumers)
    kDrain = 39,
    kDrainS = 40,
    kPub = 42,        // four state warps wrote a segment's end state
    kYStaged = 43,    // four output warps wrote y into the tile's C buffer
    kZEmpty = 44,     // 2 (per Z buffer): four output warps read Z
    kZInit = 46,      // 2 (per Z buffer): four scale warps wrote Z's initial value
};

uint32_t bar_count(int i)
{
    if (i == kEmptyCB || i == kEmptyCB + 1) return 3;
    if (i == kEmptyX || i == kEmptyX + 1) return 2;
    if (i == kRecEmpty || i == kRecEmpty + 1) return 13;
    if (i == kTrilFull || i == kTrilFull + 1 || i == kZEmpty || i == kZEmpty + 1 || i == kSlotFull ||
        i == kHReady || i == kHpFull || i == kZScaled || i == kPub || i == kXpFull || i == kXpFull + 1 ||
        i == kZInit || i == kZInit + 1 ||
        i == kYStaged)
        return 4;
    if (i >= kSchedEmpty && i < kSchedEmpty + kSchedSlots) return kSchedConsumers;
    return 1;
}

struct GParams {
    const float* dt;
    const float* A;
    const float* D;
    const float* init;
    const __nv_bfloat16* x;
    __nv_bfloat16* y;
    float* final_state;
    unsigned long long* ctrl;   // [0] next ticket (tagged with the call's epoch)
    unsigned long long* flags;  // per chain: (epoch, segments published)
    uint32_t epoch;
    float* ring;          // per chain: KH x [kN][kP] fp32, the state leaving a segment
    unsigned int* status;
    unsigned long long wait_limit;
    uint32_t bar_counts[Smem::kNumBars];
    int B, L;
    int Ht;    // heads of kP channels (model heads x sub)
    int Hr;    // model heads: dt [B][L][Hr], A and D [Hr]
    int sub;   // kP-channel heads per model head
    int G;
    int N;     // state dim (<= kN)
    int nkh;   // 64-wide halves of the state dim that hold data (1 or 2)
    int gpr;   // head groups per batch row (Ht / KH)
    int hpg;   // kP-channel heads per B/C group (Ht / G)
    int ntiles, chains, seg_len, nseg, items;
    int wrap;     // 1: static ranges of the chain-major tile order (see Pieces)
    int grid;
    int skip_publish;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// a read-only load issued where it stands (not moved towards its first use)
__device__ __forceinline__ float ldg_f32_now(const float* ptr)
{
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(ptr));
    return v;
}

__device__ __forceinline__ void prefetch_l2(const void* ptr)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

// two fp32 products in one instruction, (a.x b.x, a.y b.y), each rounded to nearest
__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

__device__ __noinline__ void wait_gave_up(volatile int* abort_flag, unsigned int* status)
{
    record_status(status, kDevWaitTimeout);
    *abort_flag = 1;
}

// Bounded wait of one thread that ignores the abort mode: true once the phase
// completes, false after ~2 s (or kWaitPolls polls, whichever comes first).
__device__ __forceinline__ bool wait_bounded_1(uint64_t* bar, uint32_t parity)
{
    if (mbar_try_wait_short(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
#pragma unroll 1
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_short(bar, parity)) return true;
        if ((it & 63u) == 0u && (it >= kWaitPolls || global_timer_ns() - t0 > kWaitNs)) return false;
    }
}

// Bounded wait of one thread on an mbarrier phase: each poll suspends the
// thread until the phase completes or ~1 us passes; it gives up after
// kRolePolls polls (a fraction of a second to a few seconds). A give-up puts
// the CTA into abort mode: later waits return at once and every role runs out
// its loop; the status word reports it. (The bound is a poll count, so the
// loop inlined at every wait stays a few instructions long.)
__device__ __forceinline__ void wait_bar_1(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned int* status)
{
    if (*abort_flag) return;
#pragma unroll 1
    for (uint32_t it = 0; it < kRolePolls; ++it)
        if (mbar_try_wait_1us(bar, parity)) return;
    wait_gave_up(abort_flag, status);
}

// The same for a whole warp: lane 0 polls, and the warp leaves converged (the
// tcgen05.ld / st / mma issue that follow a wait are .sync.aligned warp
// instructions, which every lane must reach together; one poller also keeps
// the barrier words' shared-memory traffic low).
__device__ __forceinline__ void wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned int* status)
{
    if ((threadIdx.x & 31) == 0) wait_bar_1(bar, parity, abort_flag, status);
    __syncwarp();
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity)
{
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = wait_bounded_1(bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// A piece of one chain: its batch row, head group and tiles [tile_begin,
// tile_end). `seg` counts the pieces of the chain before this one: a piece
// with seg > 0 starts from the state its predecessor published.
struct Pos {
    int chain, seg, b, hs0, g, tile, tile_begin, tile_end;
    bool valid;

    __device__ void set(const GParams& p, int4 pc, int kh)
    {
        valid = pc.x >= 0;
        if (!valid) return;
        chain = pc.x;
        seg = pc.y;
        tile_begin = tile = pc.z;
        tile_end = pc.w;
        b = chain / p.gpr;
        hs0 = (chain - b * p.gpr) * kh;
        g = hs0 / p.hpg;
    }
};

// The pieces one CTA runs, in order.
//  Segment mode: ticket t is segment t / chains of chain t % chains (segments
//  of seg_len tiles, numbered segment-major, so a segment's predecessor was
//  taken by a CTA that was already running).
//  Wrap mode (at least as many chains as CTAs): one ticket per CTA gives its
//  rank c, which owns tiles [c U / grid, (c+1) U / grid) of the chain-major
//  order of all U tiles. That range is the tail of one chain, whole chains and
//  the head of another; the CTA runs the head first and the tail last. The
//  head's other part is the tail of rank c + 1, which runs it last, so it
//  waits on a piece that a running CTA does first, with a slack of
//  U / grid - ntiles tiles (the range is at least one chain long).
struct Pieces {
    long long u0 = 0, u1 = 0;
    int idx = 0;
    __device__ __noinline__ int4 next(const GParams& p, volatile int* abort_flag)
    {
        const int4 none = make_int4(-1, 0, 0, 0);
        if (*abort_flag) return none;
        if (!p.wrap) {
            const unsigned int t = take_ticket(p.ctrl, p.epoch);
            if (t >= static_cast<unsigned int>(p.items)) return none;
            const int seg = static_cast<int>(t) / p.chains;
            const int tb = seg * p.seg_len;
            return make_int4(static_cast<int>(t) - seg * p.chains, seg, tb, min(tb + p.seg_len, p.ntiles));
        }
        const long long U = static_cast<long long>(p.chains) * p.ntiles;
        if (idx == 0) {
            const unsigned int c = take_ticket(p.ctrl, p.epoch);
            if (c >= static_cast<unsigned int>(p.grid)) return none;
            u0 = c * U / p.grid;
            u1 = (c + 1ll) * U / p.grid;
        }
        const int nt = p.ntiles;
        const int ca = static_cast<int>(u0 / nt), oa = static_cast<int>(u0 % nt);
        const int cb = static_cast<int>(u1 / nt), ob = static_cast<int>(u1 % nt);
        const int first_full = oa > 0 ? ca + 1 : ca;
        int j = idx++;
        if (ob > 0) {
            if (j == 0) return make_int4(cb, 0, 0, ob);  // head of chain cb
            --j;
        }
        if (first_full + j < cb) return make_int4(first_full + j, 0, 0, nt);
        j -= cb - first_full;
        if (oa > 0 && j == 0) return make_int4(ca, 1, oa, nt);  // tail of chain ca
        return none;
    }
};

// Piece ring: the producer pushes pieces, warps 1..12 read each one.
struct SchedReader {
    uint32_t n = 0;
    // Every reader sees the same sequence (the producer never overwrites an
    // unread slot and pushes an end marker), so the warps of one role walk the
    // same tiles. A reader that waits in vain (the producer is gone) ends its
    // sequence after the bounded wait; in abort mode every reader ends at once
    // (the roles are linked by mbarriers only, so no role waits on a warp
    // that has left its loop for longer than a bounded wait).
    __device__ __noinline__ int4 pop(uint8_t* sm, uint64_t* bars, volatile int* abort_flag,
                                     unsigned int* status)
    {
        if (*abort_flag) return make_int4(-1, 0, 0, 0);  // aborted: every role just ends
        const uint32_t slot = n % kSchedSlots;
        const bool ok = wait_bounded(bars + kSchedFull + slot, (n / kSchedSlots) & 1);
        int4 pc = make_int4(-1, 0, 0, 0);
        if (ok) {
            const volatile int* v = reinterpret_cast<const volatile int*>(sm + Smem::kSched + slot * 16);
            pc = make_int4(v[0], v[1], v[2], v[3]);
        }
        if (!ok && (threadIdx.x & 31) == 0) wait_gave_up(abort_flag, status);
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(bars + kSchedEmpty + slot);
        ++n;
        return pc;
    }
};

template <int KH>
struct Walker {
    Pos s;
    SchedReader rd;
    __device__ void begin(const GParams& p, uint8_t* sm, uint64_t* bars, volatile int* ab)
    {
        s.set(p, rd.pop(sm, bars, ab, p.status), KH);
    }
    __device__ void next(const GParams& p, uint8_t* sm, uint64_t* bars, volatile int* ab)
    {
        if (++s.tile >= s.tile_end) s.set(p, rd.pop(sm, bars, ab, p.status), KH);
    }
};

// Exact-form tiles are rare; their parts of the role loops live out of line so
// that the hot loops stay compact in the instruction cache.

// MMA warp, exact form: once the raw X is in the H' buffer and the output
// warps have scaled Z, one masked product per head (Z_h += S~_h X_h, S~_h from
// TMEM as the state warps hand it over), then the tile's Z, S and H' buffers
// are released.
template <int KH>
__device__ __noinline__ void mma_exact_products(uint64_t* bars, volatile int* abort_flag, unsigned int* status,
                                                uint32_t zcol, uint32_t tmem, uint64_t dhp, uint32_t nh, int zb)
{
    constexpr uint32_t id_y1 = idesc_bf16(128, 64, false, true);
    wait_bar(bars + kRawX, nh & 1, abort_flag, status);
    wait_bar(bars + kZScaled, nh & 1, abort_flag, status);
#pragma unroll 1
    for (int hh = 0; hh < KH; ++hh) {
        const uint32_t u = nh * KH + hh;
        wait_bar(bars + kSlotFull, u & 1, abort_flag, status);
        tc_fence_after_sync();
        if (elect_one_sync()) {
#pragma unroll 1
            for (int q = 0; q < kT / 16; ++q)
                mma_bf16_tmem_a(zcol + hh * 64, tmem + kColS + 64 + q * 8, dhp + ((hh * kHalf) >> 4) + q * (2048 >> 4),
                                id_y1, true);
            mma_commit(bars + kSlotFree);
        }
        __syncwarp();
    }
    if (elect_one_sync()) {
        mma_commit(bars + kZFull + zb);
        mma_commit(bars + kSFree);
        mma_commit(bars + kHpEmpty);
    }
    __syncwarp();
}

// State warps: S~_h,ij = tril(S)_ij 2^(cs_i - cs_j) dt_j of each head into
// columns 64-127 of the S buffer, handed to the MMA warp one head at a time.
template <int KH>
__device__ __noinline__ void state_exact_stilde(const GParams& p, uint64_t* bars, volatile int* abort_flag,
                                                const Rec& rc, int b, int tile, int hs0, uint32_t s_col,
                                                uint32_t nh, int r, int lane)
{
    const int rows = min(kT, p.L - tile * kT);
#pragma unroll
    for (int hh = 0; hh < KH; ++hh) {
        const int hr = (hs0 + hh) / p.sub;
        const size_t base = (static_cast<size_t>(b) * p.L + tile * kT) * p.Hr + hr;
        float dtl[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = lane + 32 * u;
            dtl[u] = j < rows ? __ldg(p.dt + base + static_cast<size_t>(j) * p.Hr) : 0.f;
        }
        const float cs_i = rc.cs[hh][r];
        const uint32_t u_slot = nh * KH + hh;
        wait_bar(bars + kSlotFree, (u_slot & 1) ^ 1, abort_flag, p.status);
        tc_fence_after_sync();
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            uint32_t wv[32];
            tmem_ld32_sync(s_col + half * 32, wv);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int j0 = half * 64 + 2 * e;  // tokens j0, j0 + 1 (same 32-block)
                const float dsrc = half ? dtl[2 + (e >> 4)] : dtl[e >> 4];
                const float d0 = __shfl_sync(0xffffffffu, dsrc, j0 & 31);
                const float d1 = __shfl_sync(0xffffffffu, dsrc, (j0 + 1) & 31);
                const float m0 = ex2_approx(fminf(cs_i - rc.cs[hh][j0], 0.f)) * d0;
                const float m1 = ex2_approx(fminf(cs_i - rc.cs[hh][j0 + 1], 0.f)) * d1;
                wv[e] = pack_bf16x2(bf16_lo(wv[e]) * m0, bf16_hi(wv[e]) * m1);
            }
            tmem_st32(s_col + 64 + half * 32, wv);
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kSlotFull);
    }
}

// State warps, exact form: row r of each head's h in TMEM times rh.
template <int KH>
__device__ __noinline__ void state_exact_rescale(uint32_t hcol, float r0, float r1)
{
#pragma unroll 1
    for (int hh = 0; hh < KH; ++hh) {
        uint32_t v[64];
        tmem_ld64_sync(hcol + hh * 64, v);
        const float rh = hh ? r1 : r0;
#pragma unroll
        for (int q = 0; q < 64; ++q) v[q] = __float_as_uint(rh * __uint_as_float(v[q]));
        tmem_st64(hcol + hh * 64, v);
    }
}

// Output warps, exact form: Z_r *= 2^(cs_r) once MMA3 is done, before the
// per-head masked products add to it.
template <int KH>
__device__ __noinline__ void out_exact_scale(uint64_t* bars, volatile int* abort_flag, unsigned int* status,
                                             uint32_t zaddr, float zs0, float zs1, uint32_t nh, int lane)
{
    wait_bar(bars + kM3Done, nh & 1, abort_flag, status);
    tc_fence_after_sync();
#pragma unroll 1
    for (int hh = 0; hh < KH; ++hh) {
        uint32_t v[64];
        const uint32_t a = zaddr + hh * 64;
        tmem_ld64_sync(a, v);
        const float zsh = hh ? zs1 : zs0;
#pragma unroll
        for (int q = 0; q < 64; ++q) v[q] = __float_as_uint(__uint_as_float(v[q]) * zsh);
        tmem_st64(a, v);
    }
    tmem_wait_st();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + kZScaled);
}

// Output warps, exact form with a skip term: y = Z + D x, x from global memory.
template <int KH>
__device__ __noinline__ void out_exact_epilogue(uint64_t* bars, uint32_t zaddr, uint8_t* ys,
                                                const __nv_bfloat16* x, size_t row0, const float* D, int hs0,
                                                int sub, bool live, int r, int lane, int zb)
{
#pragma unroll 1
    for (int j = 0; j < 2 * KH; ++j) {
        const int hh = j >> 1, half = j & 1;
        uint32_t zv[32];
        tmem_ld32_sync(zaddr + hh * 64 + half * 32, zv);
        if (j == 2 * KH - 1) {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kZEmpty + zb);
        }
        const float dh = __ldg(D + (hs0 + hh) / sub);
        const uint4* xg = reinterpret_cast<const uint4*>(x + (row0 + hh) * kP + half * 32);
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            float xv[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) xv[u] = 0.f;
            if (live) {
                const uint4 xq = __ldg(xg + c4);
                const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    xv[2 * u] = dh * bf16_lo(xw[u]);
                    xv[2 * u + 1] = dh * bf16_hi(xw[u]);
                }
            }
            uint32_t o[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = 8 * c4 + 2 * u;
                o[u] = pack_bf16x2(__uint_as_float(zv[i]) + xv[2 * u], __uint_as_float(zv[i + 1]) + xv[2 * u + 1]);
            }
            const int c = 4 * half + c4;
            *reinterpret_cast<uint4*>(ys + hh * kHalf + (((c ^ r) & 7) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

template <int KH>
__global__ void __launch_bounds__(kThreads, 1)
grouped_forward_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmC,
                       const __grid_constant__ CUtensorMap tmY, const GParams p)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Smem::kBars);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + Smem::kTmemPtr);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Smem::kAbort);
    Rec* recs = reinterpret_cast<Rec*>(sm + Smem::kRec);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // the 128-byte swizzle needs 1024-byte aligned tiles; the layout above
    // assumes the dynamic shared memory itself starts on such a boundary
    if ((smem_addr(sm) & 1023u) != 0) {
        if (tid == 0) record_status(p.status, kDevWaitTimeout);
        return;
    }
    if (tid == 0) {
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmC);
        prefetch_tensormap(&tmY);
        for (int i = 0; i < Smem::kNumBars; ++i) mbar_init(bars + i, p.bar_counts[i]);
        mbar_fence_init();
        *abort_flag = 0;
    }
    if (warp == kWarpProducer) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    if (p.nkh == 1) {
        // N <= 64: the second halves of the C and B tiles are never loaded; zero
        // them once so the states MMA (which spans all 128 state rows) reads zeros
        for (int st = 0; st < 2; ++st)
            for (int base = 0; base < 2; ++base) {
                uint4* z = reinterpret_cast<uint4*>(sm + (base ? Smem::kB : Smem::kC) +
                                                    st * 2 * kHalf + kHalf);
                for (int u = tid; u < int(kHalf / 16); u += kThreads) z[u] = make_uint4(0u, 0u, 0u, 0u);
            }
        fence_async_shared();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *s_tmem;

    if (warp == kWarpProducer) {
        // ------------------------------------------------------------ producer
        uint32_t npush = 0;
        Pieces src;
        auto fetch = [&]() {
            int4 pc = make_int4(-1, 0, 0, 0);
            if (lane == 0) pc = src.next(p, abort_flag);
            pc.x = __shfl_sync(0xffffffffu, pc.x, 0);
            pc.y = __shfl_sync(0xffffffffu, pc.y, 0);
            pc.z = __shfl_sync(0xffffffffu, pc.z, 0);
            pc.w = __shfl_sync(0xffffffffu, pc.w, 0);
            return pc;
        };
        auto push = [&](int4 pc) {
            if (*abort_flag) return false;  // the readers end at once in abort mode
            const uint32_t slot = npush % kSchedSlots;
            // never overwrite a slot a reader has not taken yet, even when aborting
            if (!wait_bounded(bars + kSchedEmpty + slot, ((npush / kSchedSlots) & 1) ^ 1)) {
                if (lane == 0) wait_gave_up(abort_flag, p.status);
                __syncwarp();
                return false;
            }
            if (lane == 0) {
                volatile int* v = reinterpret_cast<volatile int*>(sm + Smem::kSched + slot * 16);
                v[0] = pc.x;
                v[1] = pc.y;
                v[2] = pc.z;
                v[3] = pc.w;
                mbar_arrive(bars + kSchedFull + slot);
            }
            __syncwarp();
            ++npush;
            return true;
        };
        Pos s;
        int4 pc = fetch();
        s.set(p, pc, KH);
        bool alive = push(pc);
        int k = 0;
        while (alive && s.valid && !*abort_flag) {
            const int st = k & 1;
            const uint32_t par = ((k >> 1) & 1) ^ 1;
            const int t0 = s.tile * kT;
            // X first: its stage frees when MMA2 and the states product have
            // read it, the C/B stage only once y, staged in C, is stored
            wait_bar(bars + kEmptyX + st, par, abort_flag, p.status);
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(bars + kFullX + st, KH * kHalf);
#pragma unroll
                for (int hh = 0; hh < KH; ++hh)
                    tma_load_4d(sm + Smem::kX + st * 2 * kHalf + hh * kHalf, &tmX, 0, s.hs0 + hh, t0, s.b,
                                bars + kFullX + st);
            }
            __syncwarp();
            wait_bar(bars + kEmptyCB + st, par, abort_flag, p.status);
            if (elect_one_sync()) {
                mbar_arrive_expect_tx(bars + kFullCB + st, p.nkh * 2 * kHalf);
                for (int q = 0; q < p.nkh; ++q) {
                    tma_load_4d(sm + Smem::kC + st * 2 * kHalf + q * kHalf, &tmC, q * 64, s.g, t0, s.b,
                                bars + kFullCB + st);
                    tma_load_4d(sm + Smem::kB + st * 2 * kHalf + q * kHalf, &tmB, q * 64, s.g, t0, s.b,
                                bars + kFullCB + st);
                }
            }
            __syncwarp();
            ++k;
            if (++s.tile >= s.tile_end) {
                pc = fetch();
                s.set(p, pc, KH);
                alive = push(pc);
            }
        }
        if (alive && s.valid) push(make_int4(-1, 0, 0, 0));  // aborted: tell every role to stop
        // every load issued has landed before the CTA can exit
        for (int j = max(0, k - 2); j < k; ++j) {
            wait_bounded(bars + kFullCB + (j & 1), (j >> 1) & 1);
            wait_bounded(bars + kFullX + (j & 1), (j >> 1) & 1);
        }
    } else if (warp == kWarpMma) {
        // ------------------------------------------------- MMA issue: Z and S.
        // Per tile k: MMA3(k), MMA2(k), then MMA1(k + 1), so S of the next tile
        // is ready when the state warps get to its mask. (An MMA issue blocks
        // while the tensor pipe is busy, so the states products, which carry
        // the recurrence from tile to tile, have their own issuing warp.)
        constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);
        constexpr uint32_t id_y = idesc_bf16(128, 64 * KH, false, true);
        const uint64_t dc0 = sdesc_sw128(smem_addr(sm + Smem::kC), 16, 1024);
        const uint64_t db0 = sdesc_sw128(smem_addr(sm + Smem::kB), 16, 1024);
        const uint64_t dx0 = sdesc_sw128(smem_addr(sm + Smem::kX), kHalf, 1024);   // X', MN-major
        const uint64_t dhp = sdesc_sw128(smem_addr(sm + Smem::kHp), kHalf, 1024);  // H', MN-major
        auto stage_of = [](int kk) { return static_cast<uint64_t>((kk & 1) * 2 * kHalf) >> 4; };
        // MMA1 of tile kk: S = C B^T into the S buffer of its stage
        auto mma1 = [&](int kk) {
            const int s1 = kk & 1;
            const uint32_t p1 = (kk >> 1) & 1;
            wait_bar(bars + kFullCB + s1, p1, abort_flag, p.status);
            if (kk > 0) wait_bar(bars + kSFree, (kk - 1) & 1, abort_flag, p.status);  // MMA2 of tile kk - 1
            tc_fence_after_sync();
            if (elect_one_sync()) {
                for (int q = 0; q < 4 * p.nkh; ++q) {
                    const uint32_t off = ((q >> 2) * kHalf + (q & 3) * 32) >> 4;
                    mma_bf16(tmem + kColS, dc0 + stage_of(kk) + off, db0 + stage_of(kk) + off, id_s, q > 0);
                }
                mma_commit(bars + kSFull);
            }
            __syncwarp();
        };
        Walker<KH> w;
        w.begin(p, sm, bars, abort_flag);
        uint32_t nh = 0;  // exact-form tiles so far
        // iteration k: the products of tile k (k >= 0), MMA1 of tile k + 1, the
        // states of tile k (one MMA1 call site keeps the loop small)
        for (int k = -1;; ++k) {
            if (k < 0) {
                if (!w.s.valid) break;
                mma1(0);
                continue;
            }
            const int st = k & 1;
            const uint32_t par = (k >> 1) & 1;
            const uint64_t stage = stage_of(k);
            wait_bar(bars + kRecFull + st, par, abort_flag, p.status);
            const bool hard = recs[st].hard != 0;
            const int tile_k = w.s.tile, hs0_k = w.s.hs0, b_k = w.s.b;
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kRecEmpty + st);
            // ---- MMA3: Z += C H'^T (Z holds D x / e, or 0)
            wait_bar(bars + kHpFull, k & 1, abort_flag, p.status);
            const int zb = k & 1;
            const uint32_t zpar = (k >> 1) & 1;
            const uint32_t zcol = tmem + kColZ + zb * 128;
            wait_bar(bars + kZInit + zb, zpar, abort_flag, p.status);
            tc_fence_after_sync();
            if (elect_one_sync()) {
                for (int q = 0; q < 4 * p.nkh; ++q)
                    mma_bf16(zcol, dc0 + stage + (((q >> 2) * kHalf + (q & 3) * 32) >> 4),
                             dhp + q * (2048 >> 4), id_y, true);
                if (!hard) mma_commit(bars + kHpEmpty);
            }
            __syncwarp();
            if (__builtin_expect(!hard, 1)) {
                // ---- MMA2: Z += tril(S) X'
                wait_bar(bars + kTrilFull + st, par, abort_flag, p.status);
                wait_bar(bars + kXpFull + st, par, abort_flag, p.status);
                tc_fence_after_sync();
                if (elect_one_sync()) {
#pragma unroll 1
                    for (int q = 0; q < kT / 16; ++q)
                        mma_bf16_tmem_a(zcol, tmem + kColS + q * 8, dx0 + stage + q * (2048 >> 4), id_y, true);
                    mma_commit(bars + kZFull + zb);
                    mma_commit(bars + kSFree);
                }
                __syncwarp();
            } else {
                // exact form: raw X into the H' buffer once MMA3 has read it,
                // Z scaled by the output warps, then one masked product per head
                if (elect_one_sync()) mma_commit(bars + kM3Done);
                __syncwarp();
                wait_bar(bars + kM3Done, nh & 1, abort_flag, p.status);
                if (elect_one_sync()) {
                    mbar_arrive_expect_tx(bars + kRawX, KH * kHalf);
#pragma unroll
                    for (int hh = 0; hh < KH; ++hh)
                        tma_load_4d(sm + Smem::kHp + hh * kHalf, &tmX, 0, hs0_k + hh, tile_k * kT, b_k,
                                    bars + kRawX);
                }
                __syncwarp();
                mma_exact_products<KH>(bars, abort_flag, p.status, zcol, tmem, dhp, nh, zb);
                ++nh;
            }
            if (elect_one_sync()) {
                mma_commit(bars + kEmptyCB + st);
                mma_commit(bars + kEmptyX + st);
            }
            __syncwarp();
            // ---- MMA1 of the next tile
            w.next(p, sm, bars, abort_flag);
            const bool more = w.s.valid;
            if (more) mma1(k + 1);
            if (!more) break;
        }
        if (elect_one_sync()) mma_commit(bars + kDrain);
        __syncwarp();
        wait_bounded(bars + kDrain, 0);
    } else if (warp == kWarpMmaS) {
        // --------------------------------------------- MMA issue: the states.
        // h += B^T [X'_0 ... X'_KH-1] as soon as X' is in and the state warps
        // have read and rescaled h.
        constexpr uint32_t id_st = idesc_bf16(128, 64 * KH, true, true);
        const uint64_t dbt0 = sdesc_sw128(smem_addr(sm + Smem::kB), kHalf, 1024);  // B^T, MN-major
        const uint64_t dx0 = sdesc_sw128(smem_addr(sm + Smem::kX), kHalf, 1024);   // X', MN-major
        Walker<KH> w;
        w.begin(p, sm, bars, abort_flag);
        for (int k = 0; w.s.valid; ++k, w.next(p, sm, bars, abort_flag)) {
            const int st = k & 1;
            const uint32_t par = (k >> 1) & 1;
            const uint64_t stage = static_cast<uint64_t>(st * 2 * kHalf) >> 4;
            // B of this tile has landed (the states product reads it; nothing
            // else that this warp waits for implies it: X' only needs X)
            wait_bar(bars + kFullCB + st, par, abort_flag, p.status);
            wait_bar(bars + kXpFull + st, par, abort_flag, p.status);
            wait_bar(bars + kHReady, k & 1, abort_flag, p.status);
            tc_fence_after_sync();
            if (elect_one_sync()) {
#pragma unroll 1
                for (int q = 0; q < kT / 16; ++q)
                    mma_bf16(tmem + kColH, dbt0 + stage + q * (2048 >> 4), dx0 + stage + q * (2048 >> 4), id_st,
                             true);
                mma_commit(bars + kStatesDone);
                mma_commit(bars + kEmptyCB + st);
                mma_commit(bars + kEmptyX + st);
            }
            __syncwarp();
        }
        if (elect_one_sync()) mma_commit(bars + kDrainS);
        __syncwarp();
        wait_bounded(bars + kDrainS, 0);
    } else if (warp == kWarpPro) {
        // ------------------------------ prologue: cumulative decay, tile record
        Walker<KH> w;
        w.begin(p, sm, bars, abort_flag);
        // lane l holds tokens 4 l .. 4 l + 3 of the tile
        float dtv[KH][4];
        float Aval[KH];
        auto fetch = [&](const Pos& q) {
            const int rows = min(kT, p.L - q.tile * kT);
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) {
                const int hr = (q.hs0 + hh) / p.sub;
                const size_t base = (static_cast<size_t>(q.b) * p.L + q.tile * kT) * p.Hr + hr;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = 4 * lane + u;
                    dtv[hh][u] = j < rows ? ldg_f32_now(p.dt + base + static_cast<size_t>(j) * p.Hr) : 0.f;
                }
                Aval[hh] = __ldg(p.A + hr);
            }
            // the dt lines of the tiles two and three ahead into L2
#pragma unroll
            for (int ahead = 2; ahead <= 3; ++ahead) {
                const int t = (q.tile + ahead) * kT;
                const int hr = q.hs0 / p.sub;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int j = t + lane + 32 * u;
                    if (j < p.L) prefetch_l2(p.dt + (static_cast<size_t>(q.b) * p.L + j) * p.Hr + hr);
                }
            }
        };
        if (w.s.valid) fetch(w.s);
        for (int k = 0; w.s.valid; ++k) {
            const int st = k & 1;
            const uint32_t par = (k >> 1) & 1;
            float dtc[KH][4], Ah[KH];
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) {
                Ah[hh] = Aval[hh] * kLog2e;
#pragma unroll
                for (int u = 0; u < 4; ++u) dtc[hh][u] = dtv[hh][u];
            }
            w.next(p, sm, bars, abort_flag);
            if (w.s.valid) fetch(w.s);  // next tile's dt, in flight during this one

            Rec& rc = recs[st];
            wait_bar(bars + kRecEmpty + st, par ^ 1, abort_flag, p.status);
            int hard = 0;
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) {
                // running sum over the lane's four tokens, then one scan over
                // the lanes' totals
                float a[4];
                a[0] = dtc[hh][0] * Ah[hh];
#pragma unroll
                for (int u = 1; u < 4; ++u) a[u] = fmaf(dtc[hh][u], Ah[hh], a[u - 1]);
                float incl = a[3];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                float excl = __shfl_up_sync(0xffffffffu, incl, 1);
                if (lane == 0) excl = 0.f;
                const float total = __shfl_sync(0xffffffffu, incl, 31);
                *reinterpret_cast<float4*>(&rc.cs[hh][4 * lane]) =
                    make_float4(excl + a[0], excl + a[1], excl + a[2], excl + a[3]);
                // total is the same in every lane: the tile's total decay
                hard |= -total > kHardLog2 ? 1 : 0;
                if (lane == 0) {
                    rc.cref[hh] = 0.5f * total;
                    rc.csend[hh] = total;
                }
            }
            if (lane == 0) rc.hard = hard;
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kRecFull + st);
        }
    } else if (warp >= kWgState && warp < kWgState + 4) {
        // ------------- state: H', the scaled h, segment hand-off; mask: tril(S)
        const int wq = warp - kWgState;
        const int r = wq * 32 + lane;  // state row n, token row i = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const size_t Nst = static_cast<size_t>(p.N);
        const bool n_live = r < p.N;  // state rows past N are zero padding
        Walker<KH> w;
        w.begin(p, sm, bars, abort_flag);
        float s_pend[KH];  // true h = s_pend * (h in TMEM)
#pragma unroll
        for (int hh = 0; hh < KH; ++hh) s_pend[hh] = 1.f;  // (indexed by constants only)
        Pos prev;
        prev.valid = false;
        bool prev_last = false;
        uint32_t npub = 0;  // segment end states published so far
        uint32_t nh = 0;    // exact-form tiles so far

        for (int k = 0;; ++k) {
            const bool have = w.s.valid;
            // ---- the state after tile k - 1: hand it off if its segment ends there
            if (k >= 1) {
                wait_bar(bars + kStatesDone, (k - 1) & 1, abort_flag, p.status);
                tc_fence_after_sync();
                if (prev_last) {
                    const bool fin = prev.tile == p.ntiles - 1;
#pragma unroll 1
                    for (int hh = 0; hh < KH; ++hh) {
                        uint32_t v[64];
                        tmem_ld64_sync(tmem + lane_off + kColH + hh * 64, v);
                        const float sp = s_pend[hh];
                        if (fin) {
                            if (p.final_state && n_live) {
                                float* dst = p.final_state +
                                             (static_cast<size_t>(prev.b) * p.Ht + prev.hs0 + hh) * kP * Nst + r;
#pragma unroll
                                for (int q = 0; q < 64; ++q) dst[q * Nst] = sp * __uint_as_float(v[q]);
                            }
                        } else {
                            float4* dst = reinterpret_cast<float4*>(
                                p.ring + ((static_cast<size_t>(prev.chain) * KH + hh) * kN + r) * kP);
#pragma unroll
                            for (int q = 0; q < 16; ++q)
                                dst[q] = make_float4(sp * __uint_as_float(v[4 * q]), sp * __uint_as_float(v[4 * q + 1]),
                                                     sp * __uint_as_float(v[4 * q + 2]),
                                                     sp * __uint_as_float(v[4 * q + 3]));
                        }
                    }
                    if (!fin) {
                        // every thread's part is visible GPU-wide before the four
                        // warps report to thread 0, which then releases the flag
                        __threadfence();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bars + kPub);
                        if (r == 0) {
                            wait_bar_1(bars + kPub, npub & 1, abort_flag, p.status);
                            __threadfence();
                            if (!p.skip_publish)
                                st_release_gpu_u64(p.flags + prev.chain,
                                                   tagged(p.epoch, static_cast<uint32_t>(prev.seg + 1)));
                        }
                        __syncwarp();
                        ++npub;
                    }
                }
            }
            if (!have) break;
            // ---- the record of tile k (released after the mask)
            const int st = k & 1;
            const uint32_t par = (k >> 1) & 1;
            const Rec& rc = recs[st];
            float f3[KH], ratio[KH], snext[KH];
            wait_bar(bars + kRecFull + st, par, abort_flag, p.status);
            const bool hard = rc.hard != 0;
            const bool first = w.s.tile == w.s.tile_begin;
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) {
                const float c = rc.cref[hh], ce = rc.csend[hh];
                if (first) s_pend[hh] = 1.f;
                // H' = 2^c s h (exact form: s h); the h the states MMA adds to is
                // the same 2^c s h (exact form: 2^cs_end s h)
                f3[hh] = (hard ? 1.f : ex2_approx(c)) * s_pend[hh];
                ratio[hh] = hard ? ex2_approx(ce) : 1.f;
                snext[hh] = hard ? 1.f : ex2_approx(ce - c);
            }
            // ---- H' (bf16 operand of MMA3) and the scaled state for tile k
            if (first && w.s.seg > 0) {
                // bounded acquire poll on the predecessor's flag, one per warp.
                // Giving up only records the status: the call's results are
                // then undefined, but every role still runs to its end.
                if (lane == 0 && !*abort_flag) {
                    const unsigned long long* f = p.flags + w.s.chain;
                    bool ok = false;
                    const uint64_t t0 = global_timer_ns();
                    for (unsigned long long it = 0; it < p.wait_limit; ++it) {
                        const uint64_t v = ld_acquire_gpu_u64(f);
                        if (static_cast<uint32_t>(v >> 32) == p.epoch &&
                            static_cast<uint32_t>(v) >= static_cast<uint32_t>(w.s.seg)) {
                            ok = true;
                            break;
                        }
                        if ((it & 255) == 255 && global_timer_ns() - t0 > 4000000000ull) break;
                        __nanosleep(64);
                    }
                    if (!ok) record_status(p.status, kDevWaitTimeout);
                }
                __syncwarp();
            }
            wait_bar(bars + kHpEmpty, (k & 1) ^ 1, abort_flag, p.status);
            tc_fence_after_sync();
            if (first) {
                // the piece's starting state goes into TMEM first: what the
                // predecessor published (row r of [kN][kP]), the chain's initial
                // state ([B][H][P][N]), or zero
#pragma unroll 1
                for (int j = 0; j < 4 * KH; ++j) {
                    const int hh = j >> 2, q0 = (j & 3) * 16;
                    uint32_t v[16];
                    if (w.s.seg > 0) {
                        const float4* src = reinterpret_cast<const float4*>(
                            p.ring + ((static_cast<size_t>(w.s.chain) * KH + hh) * kN + r) * kP + q0);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 u = __ldcg(src + q);
                            v[4 * q] = __float_as_uint(u.x);
                            v[4 * q + 1] = __float_as_uint(u.y);
                            v[4 * q + 2] = __float_as_uint(u.z);
                            v[4 * q + 3] = __float_as_uint(u.w);
                        }
                    } else if (p.init && n_live) {
                        const float* src =
                            p.init + (static_cast<size_t>(w.s.b) * p.Ht + w.s.hs0 + hh) * kP * Nst + q0 * Nst + r;
#pragma unroll
                        for (int q = 0; q < 16; ++q) v[q] = __float_as_uint(__ldg(src + q * Nst));
                    } else {
#pragma unroll
                        for (int q = 0; q < 16; ++q) v[q] = 0u;
                    }
                    tmem_st16(tmem + lane_off + kColH + hh * 64 + q0, v);
                }
                tmem_wait_st();
            }
            // 32 columns (a quarter of the heads' h) at a time: H' in shared
            // memory, the scaled h back into TMEM
#pragma unroll 1
            for (int j = 0; j < 2 * KH; ++j) {
                const int hh = j >> 1, half = j & 1;
                const float fh = (KH == 2 && hh) ? f3[KH - 1] : f3[0];
                const uint32_t a = tmem + lane_off + kColH + hh * 64 + half * 32;
                uint32_t v[32];  // fp32 bits of columns 32 half .. 32 half + 31 of row r
                tmem_ld32_sync(a, v);
#pragma unroll
                for (int q = 0; q < 32; ++q) v[q] = __float_as_uint(fh * __uint_as_float(v[q]));
                uint8_t* row = sm + Smem::kHp + hh * kHalf + r * 128;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int c = 4 * half + c4;
                    const uint32_t* u = v + c4 * 8;
                    const uint4 hv = make_uint4(pack_bf16x2(__uint_as_float(u[0]), __uint_as_float(u[1])),
                                                pack_bf16x2(__uint_as_float(u[2]), __uint_as_float(u[3])),
                                                pack_bf16x2(__uint_as_float(u[4]), __uint_as_float(u[5])),
                                                pack_bf16x2(__uint_as_float(u[6]), __uint_as_float(u[7])));
                    *reinterpret_cast<uint4*>(row + (((c ^ r) & 7) << 4)) = hv;
                }
                tmem_st32(a, v);
            }
            // exact form: the h the states MMA adds to is 2^cs_end s h
            if (__builtin_expect(hard, 0)) {
                tmem_wait_st();
                state_exact_rescale<KH>(tmem + lane_off + kColH, ratio[0], ratio[KH - 1]);
            }
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) s_pend[hh] = snext[hh];
            tmem_wait_st();
            fence_async_shared();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bars + kHReady);
                mbar_arrive(bars + kHpFull);
            }

            // ---- mask of tile k: S -> tril(S), as bf16 pairs over the first 64
            // columns of the S buffer
            wait_bar(bars + kSFull, k & 1, abort_flag, p.status);
            tc_fence_after_sync();
            const uint32_t s_col = tmem + lane_off + kColS;
            // 16 columns at a time: column block jc (fp32 columns 16 jc ..
            // 16 jc + 15) becomes bf16 pairs in columns 8 jc .. 8 jc + 7. Rows
            // of lane quadrant wq (i = 32 wq + lane) keep j <= i: blocks left of
            // 2 wq are packed whole, blocks 2 wq and 2 wq + 1 are cut at the
            // diagonal, the rest become zeros. A block's output columns lie in
            // a block read before it or in one this quadrant never reads.
            const int jd = 2 * wq;
#pragma unroll 1
            for (int jc = 0; jc < jd + 2; ++jc) {
                uint32_t sv[16];
                tmem_ld16_sync(s_col + jc * 16, sv);
                const int lim = jc < jd ? 16 : r - jc * 16;  // keep column offsets <= lim
                uint32_t pk[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    pk[q] = pack_bf16x2(2 * q <= lim ? __uint_as_float(sv[2 * q]) : 0.f,
                                        2 * q + 1 <= lim ? __uint_as_float(sv[2 * q + 1]) : 0.f);
                tmem_st8(s_col + jc * 8, pk);
            }
            {
                const uint32_t z8[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll 1
                for (int jc = jd + 2; jc < 8; ++jc) tmem_st8(s_col + jc * 8, z8);
            }
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kTrilFull + st);
            if (__builtin_expect(hard, 0)) {
                // exact form: S~_h,ij = tril(S)_ij 2^(cs_i - cs_j) dt_j into
                // columns 64-127, one head at a time
                state_exact_stilde<KH>(p, bars, abort_flag, rc, w.s.b, w.s.tile, w.s.hs0, s_col, nh, r, lane);
                ++nh;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kRecEmpty + st);
            prev = w.s;
            prev_last = w.s.tile == w.s.tile_end - 1;
            w.next(p, sm, bars, abort_flag);
        }
    } else if (warp >= kWgOut && warp < kWgOut + 4) {
        // ------------------------------------------- output: y = e Z (+ D x).
        // Thread r owns token row r of the tile. Scaled form: Z started from
        // D x / e, so y = e Z. Exact form: Z_r *= 2^(cs_r) first, which the
        // per-head masked products then add to, and y = Z + D x with x read
        // from global memory. Row r of y (128 bytes per head) goes into the
        // tile's C buffer in the 128-byte swizzle, and one TMA store per head
        // writes the tile (rows past L are clipped).
        const int wq = warp - kWgOut;
        const int r = wq * 32 + lane;  // token row i = TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        Walker<KH> w;
        w.begin(p, sm, bars, abort_flag);
        uint32_t nh = 0;
        for (int k = 0; w.s.valid; ++k, w.next(p, sm, bars, abort_flag)) {
            const Pos cur = w.s;
            const int st = k & 1;
            const uint32_t par = (k >> 1) & 1;
            const bool live = r < p.L - cur.tile * kT;
            const size_t row0 = (static_cast<size_t>(cur.b) * p.L + cur.tile * kT + r) * p.Ht + cur.hs0;
            const Rec& rc = recs[st];
            wait_bar(bars + kRecFull + st, par, abort_flag, p.status);
            const bool hard = rc.hard != 0;
            float e[KH], zs[KH];
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) {
                const float ci = rc.cs[hh][r];
                e[hh] = hard ? 1.f : ex2_approx(ci - rc.cref[hh]);
                zs[hh] = ex2_approx(ci);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kRecEmpty + st);
            if (__builtin_expect(hard, 0)) {
                out_exact_scale<KH>(bars, abort_flag, p.status, tmem + lane_off + kColZ + (k & 1) * 128, zs[0],
                                    zs[KH - 1], nh, lane);
                ++nh;
            }
            wait_bar(bars + kZFull + (k & 1), (k >> 1) & 1, abort_flag, p.status);
            tc_fence_after_sync();
            // y into the tile's C buffer (dead since MMA3), 32 columns of Z at a
            // time; this Z buffer is free for the initial value of tile k + 2
            // once the last columns are in registers
            uint8_t* ys = sm + Smem::kC + st * 2 * kHalf + r * 128;
            const bool add_dx = hard && p.D;
            if (__builtin_expect(!add_dx, 1)) {
#pragma unroll 1
                for (int j = 0; j < 2 * KH; ++j) {
                    const int hh = j >> 1, half = j & 1;
                    uint32_t zv[32];
                    tmem_ld32_sync(tmem + lane_off + kColZ + (k & 1) * 128 + hh * 64 + half * 32, zv);
                    if (j == 2 * KH - 1) {
                        tc_fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bars + kZEmpty + (k & 1));
                    }
                    const float eh = (KH == 2 && hh) ? e[KH - 1] : e[0];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t o[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int i = 8 * c4 + 2 * u;
                            const float2 yv = mul2(make_float2(__uint_as_float(zv[i]), __uint_as_float(zv[i + 1])),
                                                   make_float2(eh, eh));
                            o[u] = pack_bf16x2(yv.x, yv.y);
                        }
                        const int c = 4 * half + c4;
                        *reinterpret_cast<uint4*>(ys + hh * kHalf + (((c ^ r) & 7) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            } else {
                out_exact_epilogue<KH>(bars, tmem + lane_off + kColZ + (k & 1) * 128, ys, p.x, row0, p.D, cur.hs0,
                                       p.sub, live, r, lane, k & 1);
            }
            fence_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kYStaged);
            if (r == 0) {
                // one TMA store per head (rows past L are clipped); the C buffer
                // goes back to the producer once the stores have read it
                wait_bar_1(bars + kYStaged, k & 1, abort_flag, p.status);
#pragma unroll
                for (int hh = 0; hh < KH; ++hh)
                    tma_store_4d(&tmY, ys + hh * kHalf, 0, cur.hs0 + hh, cur.tile * kT, cur.b);
                tma_store_commit();
                tma_store_wait_read();
                mbar_arrive(bars + kEmptyCB + st);
            }
            __syncwarp();
        }
        if (r == 0) tma_store_wait_all();
    } else if (warp >= kWgScale) {
        // ----------------------- scale: X' = diag(f) X, and Z's initial value.
        // Thread r owns token row r: X'_r = f_r X_r in place (fp32 product, one
        // rounding), f_r = 2^(c - cs_r) dt_r (exact form: 2^(cs_end - cs_r) dt_r);
        // in the Z buffer the output warps have read for tile k - 2, Z_r starts from
        // D x_r / e_r = D x_r 2^(c - cs_r) (exact form: 0), so that MMA3 and
        // MMA2 accumulate onto the skip term.
        const int wq = warp - kWgScale;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        Walker<KH> w;
        w.begin(p, sm, bars, abort_flag);
        for (int k = 0; w.s.valid; ++k, w.next(p, sm, bars, abort_flag)) {
            const Pos cur = w.s;
            const int st = k & 1;
            const uint32_t par = (k >> 1) & 1;
            const bool live = r < p.L - cur.tile * kT;
            float dtr[KH], Dh[KH];
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) {
                const int hr = (cur.hs0 + hh) / p.sub;
                dtr[hh] = live ? __ldg(p.dt + (static_cast<size_t>(cur.b) * p.L + cur.tile * kT + r) * p.Hr + hr)
                               : 0.f;
                Dh[hh] = p.D ? __ldg(p.D + hr) : 0.f;
            }
            const Rec& rc = recs[st];
            wait_bar(bars + kRecFull + st, par, abort_flag, p.status);
            const bool hard = rc.hard != 0;
            float f[KH], ie[KH];
#pragma unroll
            for (int hh = 0; hh < KH; ++hh) {
                const float ci = rc.cs[hh][r];
                f[hh] = ex2_approx(hard ? rc.csend[hh] - ci : rc.cref[hh] - ci) * dtr[hh];
                ie[hh] = hard ? 0.f : Dh[hh] * ex2_approx(rc.cref[hh] - ci);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kRecEmpty + st);
            // one pass over row r, 16 columns at a time: X' in place in shared
            // memory, D x / e into Z buffer k & 1 (once the output warps have
            // read it for tile k - 2)
            wait_bar(bars + kZEmpty + (k & 1), ((k >> 1) & 1) ^ 1, abort_flag, p.status);
            wait_bar(bars + kFullX + st, par, abort_flag, p.status);
            tc_fence_after_sync();
            uint8_t* xrow = sm + Smem::kX + st * 2 * kHalf + r * 128;
#pragma unroll 1
            for (int j = 0; j < 4 * KH; ++j) {
                const int hh = j >> 2, c0 = 2 * (j & 3);
                const float fr = (KH == 2 && hh) ? f[KH - 1] : f[0];
                const float ih = (KH == 2 && hh) ? ie[KH - 1] : ie[0];
                uint32_t zv[16];
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint4* a = reinterpret_cast<uint4*>(xrow + hh * kHalf + ((((c0 + h2) ^ r) & 7) << 4));
                    const uint4 v = *a;
                    const uint32_t xw[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 xv = make_float2(bf16_lo(xw[u]), bf16_hi(xw[u]));
                        const float2 xs = mul2(xv, make_float2(fr, fr));
                        const float2 zs = mul2(xv, make_float2(ih, ih));
                        o[u] = pack_bf16x2(xs.x, xs.y);
                        zv[8 * h2 + 2 * u] = __float_as_uint(zs.x);
                        zv[8 * h2 + 2 * u + 1] = __float_as_uint(zs.y);
                    }
                    *a = make_uint4(o[0], o[1], o[2], o[3]);
                }
                tmem_st16(tmem + lane_off + kColZ + (k & 1) * 128 + hh * 64 + c0 * 8, zv);
            }
            fence_async_shared();
            tmem_wait_st();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(bars + kXpFull + st);
            if (lane == 0) mbar_arrive(bars + kZInit + (k & 1));
        }
    }

    // ---- teardown
    __syncwarp();
    tc_fence_before_sync();
    __syncthreads();
    if (warp == kWarpProducer) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ host side

int heads_per_tile(const FwdArgs& a)
{
    const int Ht = a.H * (a.P / kP);
    return (Ht / a.G) % 2 == 0 ? 2 : 1;
}

struct Plan {
    int KH, Ht, chains, ntiles, seg_len, nseg, items, grid, wrap;
    size_t ws_ctrl, ws_flags, ws_ring, ws_total;
};

// Segments per chain: about `per_cta` segments per CTA in all.
constexpr int kItemsPerCta = 4;

Plan make_plan(const FwdArgs& a, int ctas)
{
    Plan g;
    g.KH = heads_per_tile(a);
    g.Ht = a.H * (a.P / kP);
    g.chains = a.B * (g.Ht / g.KH);
    g.ntiles = (a.L + kT - 1) / kT;
    g.wrap = 0;
    if (g.chains >= ctas) {
        // every CTA owns an equal range of the chain-major tile order, at least
        // one chain long: at most one hand-off per CTA, none waited on long
        g.wrap = 1;
        g.seg_len = g.ntiles;
        g.nseg = 2;
        g.items = ctas;
        g.grid = ctas;
    } else {
        long long want = 1;
        if (g.chains < ctas / 2)  // else one chain per CTA: no hand-offs
            want = (static_cast<long long>(kItemsPerCta) * ctas + g.chains - 1) / g.chains;
        if (want > g.ntiles) want = g.ntiles;
        g.seg_len = static_cast<int>((g.ntiles + want - 1) / want);
        g.nseg = (g.ntiles + g.seg_len - 1) / g.seg_len;
        g.items = g.chains * g.nseg;
        g.grid = g.items < ctas ? g.items : ctas;
    }
    g.ws_ctrl = 0;
    g.ws_flags = 256;
    g.ws_ring = g.ws_flags + ((static_cast<size_t>(g.chains) * 8 + 255) / 256) * 256;
    g.ws_total = g.ws_ring + static_cast<size_t>(g.chains) * g.KH * kN * kP * sizeof(float);
    return g;
}

int g_skip_publish = 0;

template <int KH>
cudaError_t launch_kh(const CUtensorMap& tmX, const CUtensorMap& tmB, const CUtensorMap& tmC,
                      const CUtensorMap& tmY, const GParams& p, int grid, cudaStream_t stream)
{
    const uint32_t smem = Smem::kBytes;
    cudaError_t e = cudaFuncSetAttribute(grouped_forward_kernel<KH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    grouped_forward_kernel<KH><<<grid, kThreads, smem, stream>>>(tmX, tmB, tmC, tmY, p);
    return cudaGetLastError();
}

}  // namespace

bool supported(const FwdArgs& a)
{
    return a.bf16 && a.P % kP == 0 && a.P >= kP && a.N % 8 == 0 && a.N >= 8 && a.N <= kN &&
           (a.chunk == 64 || a.chunk == 128 || a.chunk == 256) &&
           static_cast<long long>(a.B) * a.L > 0;
}

bool preferred(const FwdArgs& a, int ctas)
{
    if (!supported(a)) return false;
    const Plan g = make_plan(a, ctas);
    // segments of one chain wait on each other in turn; with fewer chains than
    // CTAs they would run one after another, which the segment-parallel form
    // of the per-head kernel avoids
    return g.chains >= ctas / 2 || g.nseg == 1;
}

size_t workspace_bytes(const FwdArgs& a, int ctas) { return make_plan(a, ctas).ws_total; }

void set_skip_publish(int v) { g_skip_publish = v; }

cudaError_t forward(const FwdArgs& a, void* workspace, const LaunchCtx& ctx)
{
    if (!supported(a)) return cudaErrorInvalidValue;
    const int ctas = ctx.num_sms > 0 ? ctx.num_sms : 1;
    const Plan g = make_plan(a, ctas);
    CUtensorMap tmX, tmB, tmC, tmY;
    if (!make_map_bf16_4d(&tmX, a.x, kP, g.Ht, a.L, a.B) ||
        !make_map_bf16_4d(&tmY, a.y, kP, g.Ht, a.L, a.B) ||
        !make_map_bf16_4d(&tmB, a.Bm, a.N, a.G, a.L, a.B) ||
        !make_map_bf16_4d(&tmC, a.Cm, a.N, a.G, a.L, a.B))
        return cudaErrorInvalidValue;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    GParams p;
    p.dt = a.dt;
    p.A = a.A;
    p.D = a.D;
    p.init = a.init;
    p.x = static_cast<const __nv_bfloat16*>(a.x);
    p.y = static_cast<__nv_bfloat16*>(a.y);
    p.final_state = a.final_state;
    p.ctrl = reinterpret_cast<unsigned long long*>(ws + g.ws_ctrl);
    p.flags = reinterpret_cast<unsigned long long*>(ws + g.ws_flags);
    p.epoch = ctx.launch_tag(0);
    p.ring = reinterpret_cast<float*>(ws + g.ws_ring);
    p.status = ctx.status;
    p.wait_limit = ctx.wait_limit;
    for (int i = 0; i < Smem::kNumBars; ++i) p.bar_counts[i] = bar_count(i);
    p.B = a.B;
    p.L = a.L;
    p.Ht = g.Ht;
    p.Hr = a.H;
    p.sub = a.P / kP;
    p.G = a.G;
    p.N = a.N;
    p.nkh = a.N <= 64 ? 1 : 2;
    p.gpr = g.Ht / g.KH;
    p.hpg = g.Ht / a.G;
    p.ntiles = g.ntiles;
    p.chains = g.chains;
    p.seg_len = g.seg_len;
    p.nseg = g.nseg;
    p.items = g.items;
    p.wrap = g.wrap;
    p.grid = g.grid;
    p.skip_publish = g_skip_publish;
    return g.KH == 2 ? launch_kh<2>(tmX, tmB, tmC, tmY, p, g.grid, ctx.stream)
                     : launch_kh<1>(tmX, tmB, tmC, tmY, p, g.grid, ctx.stream);
}

}  // namespace grouped
}  // namespace ssd
