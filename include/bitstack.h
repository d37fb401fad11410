/*
 * bitstack.h -- C ABI of the B200 BitStack residual-block linear.
 *
 * What it computes.  A weight W (m x d, m = out_features, d = in_features) is held
 * as a stack of residual blocks.  Block i is a sign matrix S_i in {+1,-1}^{m x d},
 * packed one bit per entry, plus rank-k fp16 factors U_i (m x k) and V_i (d x k)
 * with sqrt(sigma) folded into both.  The weight the first n blocks describe is
 *
 *     W_hat_n = ( sum_{i < n} S_i (.) (U_i V_i^T) ) diag(1/s),
 *
 * where 1/s (length d, fp32) undoes the activation-aware per-input-channel scaling
 * applied before the decomposition.  bs_linear evaluates y = x W_hat_n^T for a
 * batch of rows x straight from the packed stack: the dense weight is never written
 * to device memory.
 *
 * Sources (page titles and the part of each page):
 *  - residual block = packed sign matrix + singular vectors from absolute value
 *    decomposition: "BitStack: Fine-Grained Size Control for Compressed Large
 *    Language Models in Variable Memory Environments" (paper-review page), Fig. 3
 *    caption; OpenReview discussion of "BitStack: Any-Size Compression of Large
 *    Language Models in Variable Memory Environments", reply A1.A.
 *  - W_hat as the sum of sign (.) (u_k vt_k) over the loaded blocks, starting from
 *    a zero accumulator: same OpenReview discussion, weight restoration snippet.
 *  - scaling undone per input channel: review page, Fig. 5 caption ("Eq. 4").
 *  - blocks loaded from storage when memory grows and offloaded when it shrinks,
 *    per weight, in a presorted order: review page, Fig. 2 caption; OpenReview
 *    reply A1.B.
 *
 * Device record layout (one block, bs_block_bytes(m, d, k) bytes):
 *   [ sign words : m*d/32 little-endian uint32, device tile order      ]
 *   [ U          : m x k fp16, row-major                               ]
 *   [ V          : d x k fp16, row-major                               ]
 * Sign bit value 1 means S = -1.  Device tile order: the m x d sign matrix is cut
 * into tiles of 128 rows x 256 columns stored row-tile-major (tile index
 * rt * (d/256) + g); a tile is 1024 words (4 KiB).  Row rr of a tile owns 8 words
 * p = 0..7 covering its 256 columns; word p of row rr is at index
 * (p / 4) * 512 + rr * 4 + (p % 4) within the tile, and bit 8*q + t of that word
 * (q = 0..3, t = 0..7) holds column 32*t + 4*p + q of the tile.  (This order lets a
 * kernel turn the bits of one K-step of 32 columns into int8 operands with one
 * shift-and-mask per 4 columns.)  bs_pack_record builds records from canonical
 * bits on the host.
 *
 * Conventions for every call.
 *  - Ownership: the caller allocates and owns all device memory (records, 1/s,
 *    workspace, x, y, W_out) and all pinned host records; the library never calls
 *    cudaMalloc or cudaFree.  A handle owns only its small host-side struct.
 *  - Streams: bs_stream_t is a cudaStream_t (NULL = the legacy default stream).
 *    Every device-side effect is ordered on the stream passed to the call.
 *  - Errors: every call returns a bs_status.  Arguments are validated on the host
 *    before anything is launched; a rejected call has no effect.  Launch failures
 *    return BS_ERR_CUDA.  Device-side waits are bounded; a wait that runs out sets a
 *    sticky device error word that bs_get_device_error reports as BS_ERR_TIMEOUT.
 *  - Shapes: m % 128 == 0, d % 256 == 0, 128 <= m, d <= 65536, k == 16 on the GPU
 *    path (bs_block_bytes and bs_pack_record accept any k >= 1); "w/o AVD" stacks
 *    (vanilla-SVD blocks, below) take any m, d up to 65536.
 *  - Alignment: device buffers 256-byte aligned; x, y, W_out and 1/s 16-byte
 *    aligned.  Violations return BS_ERR_ALIGNMENT.
 *  - Thread safety: a handle is not thread-safe; distinct handles are independent.
 */
#ifndef BITSTACK_B200_H
#define BITSTACK_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bs_stream_t; /* identical to cudaStream_t */
typedef struct bs_stack_s* bs_stack_t;   /* opaque handle of one weight's block stack */

typedef enum {
  BS_OK = 0,
  BS_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size, ... */
  BS_ERR_UNSUPPORTED_SHAPE = 2, /* m, d, k outside the supported set */
  BS_ERR_ALIGNMENT = 3,         /* a pointer misses its required alignment */
  BS_ERR_CAPACITY = 4,          /* append beyond capacity, buffer too small */
  BS_ERR_RANGE = 5,             /* n_loaded > blocks held, drop at zero, bad block index */
  BS_ERR_CUDA = 6,              /* a CUDA runtime call or launch failed */
  BS_ERR_TIMEOUT = 7,           /* a bounded device-side wait ran out */
  BS_ERR_NO_DEVICE = 8          /* no usable sm_100 device */
} bs_status;

typedef enum { BS_F16 = 0, BS_BF16 = 1, BS_F32 = 2 } bs_dtype;

/* ------------------------------------------------------------------ sizes ------ */

/* Bytes of one block record: m*d/8 + 2*k*(m + d).  This equals the fp16 size of a
 * rank-k' plain-SVD block with k' = k + m*d/(16*(m + d)) (review page, Fig. 5
 * caption), and gives 7,929,856 B = 7.56 MiB for 14336 x 4096 at k = 16, the
 * largest block of an 8B model (OpenReview discussion, reply A1.A).
 * Returns 0 for non-positive arguments or when d or m*d is not a multiple of 8. */
size_t bs_block_bytes(int m, int d, int k);

/* Device bytes the caller must provide for a stack of `capacity_blocks` blocks:
 * capacity * bs_block_bytes (block i at offset i * bs_block_bytes) rounded up to
 * 256, plus 256 bytes that hold the stack's device error word.  0 on invalid
 * arguments. */
size_t bs_stack_device_bytes(int m, int d, int k, int capacity_blocks);

/* Workspace bytes bs_linear needs for `n_loaded` blocks and `batch` rows (0 when the
 * call needs none).  Decode (batch <= 4): one arrival counter per 128-row tile (first,
 * so its place never moves), then one fp32 partial output per (128-row tile, chunk
 * group of 4 x 256 columns at batch 1, else 2 x 256) and batch row, about
 * m * d * n * batch / 256 bytes at batch 1 and m * d * n * batch / 128 above.
 * Prefill (batch > 4): none when its grid (128-row tiles x token tiles) fills the
 * current device's SMs; otherwise the kernel splits K into s parts of whole 256-column
 * groups, as many as fit beside the grid in one wave, and needs one counter per
 * (row tile, token tile), 256-aligned, then s fp32 partial tiles of 128 rows x the
 * token tile each (e.g. 16 tokens of a 4096 x 14336 weight on 148 SMs: s = 4, 2 MiB).
 * A prefill call given a smaller workspace (or none) runs one pass over K instead.
 * The caller zeroes a workspace once before its first use (e.g. cudaMemsetAsync); every
 * call that completes leaves its counters at zero again, so no clearing is needed
 * between calls, and calls captured in a CUDA graph may be replayed.  After a call
 * that reported BS_ERR_TIMEOUT the counters may be left non-zero: zero the workspace
 * again before reusing it.  One workspace may serve any number of stacks whose calls
 * are ordered on one stream; calls that may overlap on the GPU need distinct
 * workspaces. */
size_t bs_workspace_bytes(int m, int d, int k, int n_loaded, int batch);

/* ---------------------------------------------------------- host packing ------ */

/* Builds one block record on the host.
 * neg_bits: m rows of d/8 bytes, canonical order (column c in bit c%8 of byte c/8,
 *           1 = sign -1).  U: m x k fp16 bits, V: d x k fp16 bits, row-major.
 * record:   bs_block_bytes(m, d, k) bytes written in the device layout above.
 * Pure host code; needs no GPU.  m % 128 == 0 and d % 256 == 0 are required. */
bs_status bs_pack_record(int m, int d, int k, const uint8_t* neg_bits, const uint16_t* U, const uint16_t* V,
                         void* record);

/* ------------------------------------------------------------ stack life ------ */

/* Creates a handle over caller-owned device memory.
 * dev_blocks: >= bs_stack_device_bytes(m, d, k, capacity_blocks) bytes, 256-aligned;
 * dev_inv_scale: d fp32 values of 1/s, 16-aligned, read by every bs_linear call
 * (kept by pointer: it must stay valid and unchanged while the handle is used).
 * The stack starts with 0 blocks; the metadata area is cleared on `stream`.
 * Fails with BS_ERR_NO_DEVICE when the current device is not sm_100. */
bs_status bs_stack_create(int m, int d, int k, int capacity_blocks, void* dev_blocks, size_t dev_bytes,
                          const float* dev_inv_scale, bs_stream_t stream, bs_stack_t* out);

/* Frees the host handle only; device memory stays with the caller. */
bs_status bs_stack_destroy(bs_stack_t stack);

/* Number of blocks currently held (loaded). */
bs_status bs_stack_num_blocks(bs_stack_t stack, int* n_blocks);

/* Loads the next block when the memory budget grows: one cudaMemcpyAsync of the
 * record (ideally pinned host memory, which must stay valid until the stream passes
 * the copy) into slot n_blocks, with no repacking; n_blocks += 1.  BS_ERR_CAPACITY
 * when the stack is full.  Source: review page, Fig. 2 caption (blocks are loaded
 * from storage, in a presorted order, when the memory budget grows); OpenReview
 * discussion, reply A1.B (the stack adapts to the available memory at run time). */
bs_status bs_append_block(bs_stack_t stack, const void* host_record, bs_stream_t stream);

/* Offloads the last block when the budget shrinks: n_blocks -= 1, no transfer (the
 * host copy is the storage, and the blocks of one weight leave in the reverse order
 * of their loading).  BS_ERR_RANGE when the stack is empty.  Source: review page,
 * Fig. 2 caption (blocks are offloaded to storage when memory shrinks); OpenReview
 * discussion, reply A1.B. */
bs_status bs_drop_block(bs_stack_t stack);

/* ----------------------------------------------------------------- compute ----- */

/* y = x W_hat_n^T with n = n_loaded (0 <= n_loaded <= n_blocks; the decode path
 * takes up to 64 loaded blocks, the prefill path as many as its shared memory holds,
 * BS_ERR_RANGE / BS_ERR_CAPACITY beyond).  W_hat_n is the sum over the first n
 * blocks of sign (.) (U V^T), starting from zero, with the scaling undone per input
 * channel: OpenReview discussion, weight restoration snippet; review page, Fig. 5
 * caption ("Eq. 4").  The dense weight is never written to device memory.
 * x: batch x d row-major, y: batch x m row-major, both of dtype `dt` (BS_F16 or
 * BS_BF16), device pointers, 16-byte aligned.  n_loaded == 0 writes y = 0 (the
 * restoration accumulator starts at zero).  batch <= 4 runs the decode path (the
 * factored form y = sum_i U_i (S_i ((x (.) 1/s) V_i)) with the +-1 contraction on
 * int8 tensor cores, in one kernel that also quantises the activations); larger
 * batches run the prefill kernel (W_hat tiles rebuilt in shared memory, then a
 * tcgen05 GEMM; K split across CTAs when the grid would leave SMs idle and the
 * workspace holds the partials).  workspace: >= bs_workspace_bytes(m, d, k, n_loaded,
 * batch) device bytes, 256-aligned, zeroed before its first use (may be NULL when the
 * size is 0).  Asynchronous on `stream`; capturable in a CUDA graph.
 * The decode kernels are launched with programmatic dependent launch: they may start,
 * and read the stack's block area and the scale vector, before the kernel ahead of
 * them on `stream` has finished; they read x and touch the workspace and y only after
 * that kernel has completed.  The block area is written only by this library's own
 * copies (bs_append_block), which a dependent launch never overtakes. */
bs_status bs_linear(bs_stack_t stack, const void* x, int batch, bs_dtype dt, int n_loaded, void* y,
                    void* workspace, size_t workspace_bytes, bs_stream_t stream);

/* The same product as bs_linear for batch <= 4 (the decode path), for callers that
 * cannot allocate device memory and so cannot pass a workspace: plugin hosts that
 * give a kernel only its inputs and outputs, or serving loops that forbid
 * allocation after start-up (cudaMalloc may synchronise the device or fail under
 * memory pressure).  The pages have no counterpart to this call.
 * The scratch is an 8 MiB array inside the library, held by every GPU that loads
 * it until exit.  Calls whose scratch (bs_workspace_bytes) would exceed 8 MiB return
 * BS_ERR_CAPACITY (e.g. 4096 x 4096 needs 0.5 MiB at n = 8, batch 1, and fits up to
 * n = 64 at batch 1, 31 at batch 2, 21 at batch 3, 15 at batch 4); batch > 4 and
 * "w/o AVD" stacks return BS_ERR_INVALID_ARG; the current device must be the stack's
 * (BS_ERR_INVALID_ARG).
 * The first call on each device looks up the array's device address synchronously,
 * so make it before any stream capture.  All calls on a device, whatever their stack,
 * share the array: once bs_get_device_error has reported an error on any stack of a
 * device, the next call here on that device clears the whole array first.  Calls that
 * can overlap on the GPU race on the array; order them on one stream.  Allocates
 * nothing.  Otherwise as bs_linear. */
bs_status bs_linear_no_alloc(bs_stack_t stack, const void* x, int batch, bs_dtype dt, int n_loaded, void* y,
                             bs_stream_t stream);

/* W_out = W_hat_n (m x d row-major, dtype BS_F32, BS_F16 or BS_BF16), for tests and
 * for users who want the dense weight: the unfused path of the OpenReview
 * discussion's weight restoration snippet (a zero accumulator, then unpack(sign)
 * (.) (U V^T) added per loaded block), with the scaling undone per input channel
 * (review page, Fig. 5 caption).  n == 0 writes zeros.  Asynchronous on `stream`. */
bs_status bs_reconstruct(bs_stack_t stack, int n, void* W_out, bs_dtype dt, bs_stream_t stream);

/* out = S_block as int8 +-1, m x d row-major (block < n_blocks).  Asynchronous. */
bs_status bs_unpack_signs(bs_stack_t stack, int block, int8_t* out, bs_stream_t stream);

/* ------------------------------------------------------ GPU decomposition ----- */

/* Workspace bytes bs_decompose needs for an m x d weight (0 for an unsupported shape):
 * the fp32 residual (4 m d) plus sketches and small matrices, about 4 m d + 400 (m + d). */
size_t bs_decompose_workspace_bytes(int m, int d, int k);

/* Decomposes W into n_blocks BitStack records on the GPU (the offline step; review page
 * "BitStack: Fine-Grained Size Control...", Figs. 3 and 5; OpenReview discussion, reply
 * A3; README "Decomposition"): R_0 = W diag(s); for each block the sign bits of R
 * (bit 1 where R < 0), the rank-k SVD of |R| with sqrt(sigma) folded into both fp16
 * factors (each pair oriented so that the column sum of U is >= 0), and
 * R <- R - S (.) (U V^T) with the stored fp16 factors.  The SVD is randomized subspace
 * iteration with 32 columns, `power_iters` power iterations and a Gaussian sketch drawn
 * from `seed` by a counter-based generator, so results differ from an exact SVD by the
 * method's approximation, not by run.
 * W: m x d fp32 row-major, s: d fp32 (the scale itself; the stack wants fp32 1/s), both
 * device, 16-byte aligned.  records: device, >= n_blocks * bs_block_bytes(m, d, k),
 * 256-aligned; record i at i * bs_block_bytes.  res_norms_sq: device, n_blocks + 1
 * doubles, ||R_i||_F^2 for i = 0 .. n_blocks.  workspace: device, 256-aligned, at least
 * bs_decompose_workspace_bytes.  Shapes as the GPU path (k == 16).  Asynchronous on
 * `stream`; allocates nothing. */
bs_status bs_decompose(int m, int d, int k, int n_blocks, const float* W, const float* s, unsigned long long seed,
                       int power_iters, void* records, size_t records_bytes, double* res_norms_sq, void* workspace,
                       size_t workspace_bytes, bs_stream_t stream);

/* ------------------------------------------------- grouped decode (one launch) --- */

/* A decode token through many linears in one launch.  The pages' use case is a whole
 * model whose weights each hold a different number of loaded blocks, set by a memory
 * budget over the universal block stack (review page "BitStack: Fine-Grained Size
 * Control...", Fig. 2 caption; OpenReview discussion, reply A1.B); one launch over a
 * table of all its linears replaces one launch per linear.  The work of all linears is
 * split across the SMs as one list, so small and large linears share the machine.
 *
 * Workspace for bs_linear_group: the row-tile counters of all linears first (their
 * places depend only on the shapes, so a workspace stays valid as n_loaded changes
 * between tokens), then each linear's partials (about m d n batch / 256 bytes at batch
 * 1).  Zero it once before first use; completed calls leave the counters at zero.
 * 0 on invalid arguments (n_linears outside 1 .. 256, batch outside 1 .. 4, a null or
 * "w/o AVD" stack, a negative count). */
size_t bs_group_workspace_bytes(int n_linears, const bs_stack_t* stacks, const int* n_loaded, int batch);

/* y[l] = x[l] W_hat_{n_loaded[l]}(stacks[l])^T for l < n_linears (<= 256), every x[l]
 * batch x d_l and y[l] batch x m_l in one dtype, batch 1 .. 4, in one decode launch
 * (plus one cudaMemsetAsync per linear with n_loaded[l] == 0).  Host arrays of
 * n_linears entries, caller-owned.  All stacks must be BitStack stacks on the current
 * device.  Results are bit-identical to one bs_linear call per linear.  A bounded wait
 * that runs out is reported on stacks[0] (bs_get_device_error); zero the workspace
 * again after that.  Errors as bs_linear, checked for every linear before any launch. */
bs_status bs_linear_group(int n_linears, const bs_stack_t* stacks, const void* const* x, void* const* y,
                          const int* n_loaded, int batch, bs_dtype dt, void* workspace, size_t workspace_bytes,
                          bs_stream_t stream);

/* ------------------------------------------- "w/o AVD" blocks (vanilla SVD) ----- */

/* The ablation of the review page, Fig. 5 caption: every residual block is a plain
 * rank-k' factor pair from the vanilla SVD of the residual (no sign matrix), with
 * k' = k + m n / (16 (m + n)) so that a block takes the bytes of a BitStack block.
 * Record: [U, m x k' fp16 row-major][V, d x k' fp16 row-major], 2 k' (m + d) bytes,
 * sqrt(sigma) folded into both factors as for BitStack blocks.  Such a stack takes the
 * same calls as a BitStack stack (append, drop, num_blocks, linear, reconstruct,
 * get_device_error, destroy); bs_unpack_signs and bs_linear_no_alloc return
 * BS_ERR_INVALID_ARG for it.  Shapes: any m, d in 1 .. 65536; k' a multiple of 8 in
 * 8 .. 256 (whole 16-byte factor rows). */

/* k' for an m x d weight and BitStack rank k: k + m d / (16 (m + d)) rounded down to a
 * multiple of 8 (exact for 4096 x 4096, k = 16: 144).  0 on non-positive arguments. */
int bs_plain_rank(int m, int d, int k);

/* 2 k' (m + d); 0 for a shape outside the rules above. */
size_t bs_plain_block_bytes(int m, int d, int k_prime);

/* capacity * bs_plain_block_bytes rounded up to 256, plus 256 bytes for the stack's
 * device error word; 0 on invalid arguments. */
size_t bs_plain_stack_device_bytes(int m, int d, int k_prime, int capacity_blocks);

/* Workspace bs_linear needs on a "w/o AVD" stack (0 for n_loaded == 0): n arrival
 * counters, t = (x / s) V_i for up to 16 rows of x, and per-128-row slice parts of t,
 * about 4 k' n (d / 128 + 1) min(batch, 16) bytes.  Zero it once before first use; every
 * completed call leaves its counters at zero.  Any batch: x is taken in passes of 16
 * rows, ordered on the stream, which reuse the workspace. */
size_t bs_plain_workspace_bytes(int m, int d, int k_prime, int n_loaded, int batch);

/* As bs_stack_create, for "w/o AVD" blocks of rank k_prime
 * (dev_bytes >= bs_plain_stack_device_bytes). */
bs_status bs_plain_stack_create(int m, int d, int k_prime, int capacity_blocks, void* dev_blocks, size_t dev_bytes,
                                const float* dev_inv_scale, bs_stream_t stream, bs_stack_t* out);

/* ----------------------------------------------------------- load planning ----- */

/* Orders of the universal stack.  All blocks of all weights sit in one stack on the
 * storage device and are loaded or offloaded in a presorted order as the memory
 * budget changes (review page "BitStack: Fine-Grained Size Control...", Fig. 2
 * caption; OpenReview discussion, reply A1.B); the review page's Fig. 6 compares an
 * Average, a Greedy and a Random order. */
typedef enum {
  BS_ORDER_AVERAGE = 0, /* level-major: block 0 of every weight, then block 1, ...;
                           weights in index order within a level */
  BS_ORDER_GREEDY = 1,  /* repeatedly the weight whose next block has the highest
                           score; equal scores: the lower weight index */
  BS_ORDER_RANDOM = 2   /* step t: weight live[floor(draws[t] * |live|)] of the
                           weights with blocks left, in index order */
} bs_order_kind;

/* Writes the global load order of sum(n_blocks) blocks: step t loads block
 * out_block[t] of weight out_weight[t].  Within every weight the blocks come in
 * their own order 0, 1, 2, ... (each residual block corrects what the earlier ones
 * left; review page, Fig. 2), so only the interleaving of weights is chosen.
 * n_blocks: n_weights counts >= 0.  scores (GREEDY only, else may be NULL): row w
 *   holds weight w's per-block scores at scores[w * score_stride + i], i < n_blocks[w]
 *   (score_stride >= max n_blocks).  A natural score is the drop of the weight's
 *   scaled residual energy per byte, (|R_i|^2 - |R_{i+1}|^2) / block bytes.
 * draws (RANDOM only, else may be NULL): sum(n_blocks) numbers in [0, 1), the
 *   caller's random stream.
 * out_weight, out_block: caller-owned host arrays of sum(n_blocks) ints.
 * Host only; no device is touched.  BS_ERR_INVALID_ARG on null pointers the kind
 * needs, negative counts, a stride below the largest count, a draw outside [0, 1),
 * an unknown kind, or more than 2^30 blocks in total. */
bs_status bs_plan_order(int n_weights, const int* n_blocks, const double* scores, int score_stride,
                        bs_order_kind kind, const double* draws, int* out_weight, int* out_block);

/* Loads the longest prefix of a load order that fits a byte budget: walks
 * order_weight[0 .. n_steps) and counts a block of weight w (block_bytes[w] bytes)
 * until the next one would take the total above budget_bytes, then stops.
 * out_loaded: caller-owned array of n_weights ints, the blocks to keep loaded per
 * weight (blocks 0 .. out_loaded[w]-1).  Host only.  BS_ERR_INVALID_ARG on null
 * pointers, n_steps < 0, n_weights <= 0 or a weight index outside [0, n_weights). */
bs_status bs_plan_budget(long long n_steps, const int* order_weight, int n_weights,
                         const unsigned long long* block_bytes, unsigned long long budget_bytes, int* out_loaded);

/* ------------------------------------------------------------------ errors ----- */

/* Synchronises `stack`'s device, reads and clears the sticky device error word:
 * BS_OK, BS_ERR_TIMEOUT (a bounded wait ran out), or BS_ERR_CUDA. */
bs_status bs_get_device_error(bs_stack_t stack);

/* Static text for a status code. */
const char* bs_status_string(bs_status status);

/* Sets the bound (nanoseconds) on every device-side wait of this stack's kernels
 * (default 500 ms; values < 1000 are raised to 1000).  With `unreachable_flag`
 * non-zero, the next bs_linear decode call leaves out the first sign-tile copy of
 * its first CTA, so that CTA's waits for it (and everything behind them) run out
 * while the other CTAs complete: a host-side way to exercise the timeout path
 * without faulting the GPU.  Zero the workspace before reusing it after that call. */
bs_status bs_debug_set_wait(bs_stack_t stack, long long timeout_ns, int unreachable_flag);

#ifdef __cplusplus
}
#endif

#endif /* BITSTACK_B200_H */
