/*
 * ssd.h — C ABI of the B200-native Mamba-2 SSD layer library (libssd_b200.so).
 *
 * The operation. Per batch b and head h, with scalar A_h < 0, step sizes
 * dt[b,t,h] >= 0, group g = h / (H / G) and a P x N state starting at zero
 * (or at initial_state):
 *
 *     a_t = exp(dt_t * A_h)
 *     s_t = a_t * s_{t-1} + dt_t * x_t B_t^T          (x_t in R^P, B_t in R^N)
 *     y_t = s_t C_t + D_h * x_t
 *
 * which equals Y = (L o C B^T)(dt o X) + D X with L_ij = a_i * ... * a_{j+1}
 * for i >= j ("Mamba-2", docsaid.org, sections "Writing the SSM as one matrix"
 * and "Simplifying A to one number"; "Mamba-2 SSD note", 0h-n0.github.io,
 * section "SSD layer: equivalence under the scalar constraint"). The forward
 * pass evaluates it chunk by chunk: the quadratic form inside each chunk of
 * `chunk` tokens, the recurrence across chunks ("Mamba-2", section "Half of
 * each route"; "Mamba-2 SSD note", section "Chunked algorithm"). The decode
 * step applies the recurrence to one token ("Mamba-2", section "Computing
 * with four tokens", the recurrent route for generation). The discretisation
 * a = exp(dt A), B-bar = dt B is that of the simplified selective scan in
 * "Mamba paper review" (youngju.dev), section 3.3.
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense, row-major, contiguous, in device memory unless the
 *     name says host. x, Bm, Cm, y are in the I/O dtype (`ssd_dtype`); dt, A,
 *     D, state, initial_state and final_state are always fp32.
 *   - The caller owns every buffer, including the workspace. The library
 *     allocates no device memory on these paths.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *     the legacy default stream). Argument errors are returned before anything
 *     is enqueued. A launch failure returns SSD_ERR_CUDA.
 *   - Device-side waits are bounded. When one gives up, the kernel records a
 *     device status word and returns; ssd_poll_status() reports it as
 *     SSD_ERR_TIMEOUT. Results of that call are then undefined.
 *   - dt >= 0 and A <= 0 are the caller's contract (the decay is then in
 *     [0, 1]); they are not checked on the device.
 */
#ifndef SSD_B200_H
#define SSD_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ssd_stream_t; /* same object as cudaStream_t */

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,  /* null pointer, negative or inconsistent size */
    SSD_ERR_UNSUPPORTED = 2,  /* valid, but a size this build does not handle */
    SSD_ERR_MISALIGNED = 3,   /* a pointer is not 16-byte aligned */
    SSD_ERR_CUDA = 4,         /* a CUDA call failed (launch or copy) */
    SSD_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up */
    SSD_ERR_WORKSPACE = 6     /* workspace null or smaller than ssd_workspace_size() */
} ssd_status;

typedef enum {
    SSD_F32 = 0,   /* x, Bm, Cm, y in fp32: SIMT fp32 path (|rel err| ~1e-6) */
    SSD_BF16 = 1   /* x, Bm, Cm, y in bf16, fp32 accumulate: tensor-core path for the
                      sizes ssd_forward lists, SIMT path otherwise */
} ssd_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* ssd_status_string(ssd_status status);

/* Bytes of device workspace ssd_forward needs for these sizes (0 if the sizes
 * are invalid). On the tensor-core paths the size depends on the current
 * device's SM count, which decides how each (batch, head) chain is cut into
 * segments; ask on the device that will run the call. The workspace needs no
 * clearing, neither before its first use nor between calls: the control words
 * a call keeps there (look-back flags, a work ticket counter) carry a tag of
 * that call, so leftovers of any earlier call, of any path or size, read as
 * unwritten. Calls ordered on one stream may therefore share a workspace; two
 * calls that run concurrently must not. */
size_t ssd_workspace_size(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype);

/*
 * ssd_forward — chunked SSD forward pass (prefill / training forward).
 *   x        [B, L, H, P]  I/O dtype
 *   dt       [B, L, H]     fp32, step sizes after the softplus (>= 0)
 *   A        [H]           fp32, per-head decay rate (<= 0)
 *   Bm, Cm   [B, L, G, N]  I/O dtype, shared by the H/G heads of a group
 *   D        [H]           fp32, skip term; NULL means 0
 *   initial_state [B, H, P, N] fp32 state before token 0; NULL means zero
 *   y        [B, L, H, P]  I/O dtype, output (bf16 outputs are rounded to
 *                          nearest even from fp32)
 *   final_state [B, H, P, N] fp32 state after token L-1; NULL to skip
 *   chunk    tokens per chunk, 1..256
 *   Sizes: B, L >= 0 (B*L == 0 is a no-op apart from final_state =
 *   initial_state or 0), H >= 1, G >= 1, H % G == 0, P in [1, 256],
 *   N in [1, 256]. All pointers 16-byte aligned.
 *   The tensor-core paths are taken for bf16 with P a multiple of 64 (a head
 *   of P = 64m channels runs as m heads of 64 channels sharing dt, A and D:
 *   the rows of the P x N state evolve independently), N a multiple of 8
 *   with 8 <= N <= 256, and chunk in {64, 128, 256}; other valid sizes run
 *   the SIMT path. Both tensor-core kernels evaluate the chunked form on
 *   128-token tiles whatever `chunk` is (the result does not depend on the
 *   chunk length beyond rounding):
 *   - the head-group kernel (N <= 128, and enough (batch, head pair) chains
 *     to fill the GPU) takes two heads of one B/C group through each tile,
 *     sharing C B^T between them ("Mamba-2", section "Mamba-2 block", item
 *     2). Where a tile's total decay allows it, the decay mask is applied as
 *     a row and a column scaling around a reference point of the tile (the
 *     mask is a product of per-token decays); tiles of larger decay take an
 *     exact per-head form. The skip term D x enters as the initial value of
 *     the accumulator (up to fp32 rounding the same sum). Work is handed to
 *     CTAs through a ticket counter: with at least as many chains as SMs each
 *     CTA takes one ticket (its rank) and an equal range of the chain-major
 *     tile order, and the one piece it may wait on (the head of its first
 *     chain) is run first by the CTA of the rank before, which took its ticket
 *     earlier and so is running; with fewer chains, segments in ticket order.
 *     No wait depends on a CTA that is not resident.
 *   - the per-head kernel takes the other sizes. With N > 128 it runs two
 *     passes over the state columns (n < 128, then the rest; each state column
 *     evolves on its own and y is a sum over columns): the first stores y with
 *     the D term, the second adds its share into y in L2 (a bf16 add, so y is
 *     rounded twice), and each writes its columns of final_state. It hands its
 *     segments to CTAs statically and assumes every CTA of its grid (one per
 *     SM) is resident at once: if other work keeps some SMs busy for seconds
 *     (another stream, MPS), its bounded look-back waits give up and the call
 *     reports SSD_ERR_TIMEOUT through ssd_poll_status() with undefined results.
 */
ssd_status ssd_forward(const void* x, const float* dt, const float* A, const void* Bm,
                       const void* Cm, const float* D, const float* initial_state, void* y,
                       float* final_state, int B, int L, int H, int P, int G, int N,
                       int chunk, ssd_dtype dtype, void* workspace, size_t workspace_bytes,
                       ssd_stream_t stream);

/*
 * ssd_forward_noalloc — the forward pass for callers that cannot allocate
 * device memory. The pages describe no such entry point; it is a convenience
 * of this library. It takes the same arguments as ssd_forward without the
 * workspace and runs the per-head tensor-core kernel: its scratch (look-back
 * flags and the per-head state ring, with M = B*H*P/64: 256 + 8*M rounded to
 * 256, + 2*M*64*128*4 bytes) lives in a fixed 24 MiB device array inside the
 * library, which every GPU that loads the library holds until the process
 * exits. Nothing in the array needs clearing between calls (the flags carry
 * a tag of the call that wrote them). Only the tensor-core sizes are
 * handled (bf16, P a multiple of 64, N a multiple of 8 up to 256, chunk 64, 128 or 256,
 * B*L > 0); other sizes return SSD_ERR_UNSUPPORTED, and sizes whose scratch
 * exceeds the array (M > 383; or, in the segment-parallel form, the two
 * per-segment states, 2*M*nseg*64*128*4 more bytes, see ssd_workspace_size)
 * return SSD_ERR_WORKSPACE before anything is
 * enqueued. The call allocates nothing. The first call on each device looks
 * up the array's device address (make it before any stream capture). All
 * calls on a device share the array: calls that may overlap on the GPU race
 * and must not be issued concurrently; calls ordered on one stream are safe.
 */
ssd_status ssd_forward_noalloc(const void* x, const float* dt, const float* A, const void* Bm,
                               const void* Cm, const float* D, const float* initial_state,
                               void* y, float* final_state, int B, int L, int H, int P, int G,
                               int N, int chunk, ssd_dtype dtype, ssd_stream_t stream);

/*
 * ssd_forward_host — the same forward pass on HOST buffers (pinned memory
 * gives asynchronous copies). Copies the inputs into `device_buffer`, runs
 * the forward pass, copies y (and final_state if non-NULL) back, and
 * synchronises `stream` before returning. The batch runs in up to four slices
 * of rows on two internal streams of the library (created on the first call
 * on a device, after the work already queued on `stream`), so that one
 * slice's copies overlap another's forward pass and the two copy directions
 * overlap each other. `device_buffer` must hold at least
 * ssd_forward_host_buffer_size() bytes (the tensors plus one workspace per
 * internal stream); it needs no clearing.
 */
size_t ssd_forward_host_buffer_size(int B, int L, int H, int P, int G, int N, int chunk,
                                    ssd_dtype dtype);
ssd_status ssd_forward_host(const void* x_host, const float* dt_host, const float* A_host,
                            const void* Bm_host, const void* Cm_host, const float* D_host,
                            const float* initial_state_host, void* y_host,
                            float* final_state_host, int B, int L, int H, int P, int G,
                            int N, int chunk, ssd_dtype dtype, void* device_buffer,
                            size_t device_buffer_bytes, ssd_stream_t stream);

/*
 * ssd_step — one decode step for a batch of sequences (one token each).
 *   x [B, H, P] I/O dtype; dt [B, H] fp32; A [H] fp32; Bm, Cm [B, G, N] I/O
 *   dtype; D [H] fp32 or NULL; state [B, H, P, N] fp32, updated in place;
 *   y [B, H, P] I/O dtype. Sizes as for ssd_forward (L is 1).
 */
ssd_status ssd_step(const void* x, const float* dt, const float* A, const void* Bm,
                    const void* Cm, const float* D, float* state, void* y, int B, int H,
                    int P, int G, int N, ssd_dtype dtype, ssd_stream_t stream);

/* Number of kernels one ssd_forward call with these sizes enqueues (0 if the
 * sizes are invalid or there are no tokens): 1 for the tensor-core single
 * pass; 3 for the segment-parallel form (see ssd_forward_path: every
 * segment's local state, a scan over the segments, then the outputs); twice
 * that on the tensor-core path when N > 128 (one pass per 128 state
 * columns); 3 on the SIMT path. Host-side query; it reads the current device's SM count and
 * launches nothing. */
int ssd_forward_kernel_count(int B, int L, int H, int P, int G, int N, int chunk,
                             ssd_dtype dtype);

/* Which path one ssd_forward call with these sizes takes: 0 if the sizes are
 * invalid or there are no tokens, 1 the SIMT path, 2 the per-head tensor-core
 * kernel's single pass, 3 its segment-parallel form (fewer (batch, head)
 * chains than half the SMs, each cut into eight or more segments: few chains
 * on long sequences), 4 the head-group tensor-core kernel (two heads of one
 * B/C group per tile; N <= 128 with enough chains). Host-side query; it
 * reads the current device's SM count and launches nothing. */
int ssd_forward_path(int B, int L, int H, int P, int G, int N, int chunk, ssd_dtype dtype);

/* Synchronises `stream`, then reports and clears the device status word:
 * SSD_OK, SSD_ERR_TIMEOUT (a bounded wait gave up in an earlier call), or
 * SSD_ERR_CUDA (a CUDA error was pending on the stream). */
ssd_status ssd_poll_status(ssd_stream_t stream);

/* Test hook: sets the iteration limit of every device-side wait (0 restores
 * the default). A limit of 1 makes a wait that is not already satisfied give
 * up at once, which exercises the timeout path without hanging anything. */
void ssd_set_wait_limit(uint64_t iterations);

/* Test hook: when `skip_publish` is nonzero, forward calls on the tensor-core
 * path never publish tile end states, so every look-back wait runs into the
 * iteration limit and the call reports SSD_ERR_TIMEOUT through
 * ssd_poll_status(). Results of such calls are garbage. 0 restores normal
 * operation. */
void ssd_set_fault_injection(int skip_publish);

/* Test hook: which tensor-core kernel ssd_forward uses when both handle the
 * sizes. 0 (the default) picks the faster for the sizes, 1 forces the
 * per-head kernel, 2 the head-group kernel (bf16, P a multiple of 64,
 * N <= 128). Other values restore 0. ssd_workspace_size() already covers
 * either kernel. */
void ssd_set_forward_variant(int variant);

#ifdef __cplusplus
}
#endif

#endif /* SSD_B200_H */
