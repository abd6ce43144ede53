/*
 * ssa.h -- C ABI of libssa.so: Spatial Sparse Attention (SSA) forward on B200 (sm_100a).
 *
 * The operation (Direct3D-S2 summary page, "Technical principles of Direct3D-S2", SSA item;
 * Direct3D-S2 model page, "What is Direct3D-S2?"): sparse voxel tokens are partitioned by their
 * 3D coordinates into aligned 8^3 blocks; each query combines
 *   (a) attention over compressed block tokens (block mean of K/V times a D x D map Wc),
 *   (b) exact attention over the tokens of its own block plus the top (k-1) other blocks ranked
 *       by (a)'s attention scores,
 *   (c) attention over the tokens within Chebyshev radius r of it,
 * summed with per-(token, head) gates: out = g0*o_cmp + g1*o_sel + g2*o_win. Softmax scale is
 * 1/sqrt(D). Blocks are indexed in lexicographic (bx, by, bz) order inside each sequence and
 * sequences are independent.
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are CUDA device pointers owned by the caller; they must stay valid
 *     until the work queued on `stream` has finished. Pointers marked "host" are read before the
 *     call returns unless stated otherwise.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). All device work is queued on
 *     it; only ssa_plan*, ssa_plan_export, ssa_forward_host and ssa_last_device_status wait for
 *     the device.
 *   - Tensors are contiguous, row-major. Q, K, V, out: [N, H, D] elements of `dtype` (token-major,
 *     one row of H*D values per token). gates: [N, H, 3] fp32 in order (cmp, sel, win). Wc: [D, D]
 *     fp32, applied as a row vector times Wc (Kc[e] = sum_d mean(K)[d] * Wc[d][e]).
 *   - Errors: every function returns SSA_OK or an ssa_status_t code and leaves outputs
 *     unspecified on error. Argument errors are reported before any work is queued. Errors found
 *     by kernels (bad coordinates, bounded waits that ran out) are recorded in the plan's device
 *     status word, returned by the next call that waits for the device, and readable with
 *     ssa_last_device_status. No kernel traps or asserts.
 *   - Device memory is obtained through the allocator hook (ssa_set_allocator; default:
 *     stream-ordered allocation on the call's stream from a memory pool owned by the library,
 *     one per device, that keeps freed memory cached for reuse). A plan owns its buffers until
 *     ssa_plan_destroy; the forward workspace is cached in the plan and allocated on the first
 *     forward call for a given (H, D, dtype, k), so later calls of that shape allocate nothing.
 *   - Supported: block = 8; 0 <= r <= 8; 1 <= k <= 32; D in {32, 64, 96, 128};
 *     fp32 (CUDA-core path), bf16 and fp16 (tensor-core path, fp32 accumulation);
 *     grid extents 1..65535 per axis; N < 2^31 / H tokens.
 *   - There is no CPU fallback.
 */
#ifndef SSA_H
#define SSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSA_API __attribute__((visibility("default")))
#else
#define SSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ssa_plan_s* ssa_plan_t;

typedef enum { SSA_F32 = 0, SSA_BF16 = 1, SSA_F16 = 2 } ssa_dtype_t;

typedef enum {
    SSA_OK = 0,
    SSA_ERR_INVALID_ARG = 1,      /* bad pointer, size, or unsupported combination of sizes */
    SSA_ERR_COORD_RANGE = 2,      /* a coordinate outside [0, grid) of its sequence */
    SSA_ERR_DUPLICATE_COORD = 3,  /* two tokens of one sequence share a voxel */
    SSA_ERR_ALLOC = 4,            /* the allocator hook returned NULL */
    SSA_ERR_CUDA = 5,             /* a CUDA runtime call failed */
    SSA_ERR_UNSUPPORTED = 6,      /* block != 8, D/k/r outside the supported set, no sm_100 GPU */
    SSA_ERR_DEVICE_TIMEOUT = 7    /* a kernel's bounded wait ran out; its outputs are invalid */
} ssa_status_t;

/* Device allocator hook: return `bytes` of device memory usable on `stream` (a cudaStream_t),
 * or NULL on failure. `ctx` is passed through. */
typedef void* (*ssa_alloc_fn)(size_t bytes, void* stream, void* ctx);
typedef void (*ssa_free_fn)(void* ptr, void* stream, void* ctx);

/* Replace the process-wide allocator (NULL, NULL restores the default pool allocator).
 * Plans keep the hook they were created with. Not thread-safe against concurrent plan calls. */
SSA_API ssa_status_t ssa_set_allocator(ssa_alloc_fn alloc, ssa_free_fn release, void* ctx);

/*
 * Build the plan of one sequence: the block partition and the window neighbour lists.
 * Direct3D-S2 model page, "What is Direct3D-S2?": SSA partitions the sparse tokens into blocks
 * by their 3D coordinates. Direct3D-S2 summary page, "Technical principles of Direct3D-S2", SSA
 * item: the local window branch attends to nearby tokens. Blocks are the occupied aligned 8^3
 * cells in lexicographic (bx, by, bz) order; the window of a token is every token of its
 * sequence within Chebyshev distance r (itself included).
 *   coords: device int32 [n, 3] voxel coordinates (x, y, z), each in [0, grid[axis]).
 *   n:      number of tokens (>= 1).
 *   grid:   host int32[3] grid extent.
 *   block:  block edge, must be 8.
 *   r:      window radius (Chebyshev), 0..8.
 *   out:    receives the plan handle (owned by the caller; release with ssa_plan_destroy).
 * Waits for the device twice (to size the neighbour lists and to report coordinate errors).
 * Errors: SSA_ERR_COORD_RANGE, SSA_ERR_DUPLICATE_COORD, SSA_ERR_INVALID_ARG, SSA_ERR_ALLOC,
 * SSA_ERR_CUDA, SSA_ERR_UNSUPPORTED. The coords buffer is not retained.
 */
SSA_API ssa_status_t ssa_plan(const int32_t* coords, int64_t n, const int32_t grid[3], int32_t block,
                      int32_t r, void* stream, ssa_plan_t* out);

/*
 * Plan of a packed batch of `batch` independent sequences.
 *   coords:     device int32 [N, 3], sequence s occupying rows cu_seqlens[s]..cu_seqlens[s+1]-1.
 *   cu_seqlens: host int64 [batch + 1], cu_seqlens[0] = 0, non-decreasing, last = N.
 *   grids:      host int32 [batch, 3], per-sequence grid extent.
 * Blocks are numbered sequence by sequence (all blocks of sequence 0 first). Same errors as
 * ssa_plan.
 */
SSA_API ssa_status_t ssa_plan_varlen(const int32_t* coords, const int64_t* cu_seqlens, int32_t batch,
                             const int32_t* grids, int32_t block, int32_t r, void* stream,
                             ssa_plan_t* out);

/*
 * Recompute a plan in place for new coordinates with the same token count, sequence layout,
 * grids and radius (e.g. the next refinement pass over a re-voxelised support of equal size).
 * coords: device int32 [N, 3]. The forward workspace is kept when the block count and the row
 * count of the block-ordered key/value copies (padded block rows plus each sequence's pool of
 * blocks of at most 7 tokens) are unchanged, so a following ssa_forward allocates nothing. Waits
 * for the device like ssa_plan. On error the plan is left empty (only ssa_plan_destroy is valid).
 */
SSA_API ssa_status_t ssa_plan_rebuild(ssa_plan_t plan, const int32_t* coords, void* stream);

/* Sizes of a plan (host outputs; any may be NULL): tokens, occupied blocks, total neighbour
 * list length, number of sequences. The per-token neighbour lists are not needed by the 16-bit
 * forward, so they are counted on first request: asking for nnz may launch a kernel on the
 * plan's stream and wait for it. */
SSA_API ssa_status_t ssa_plan_info(ssa_plan_t plan, int64_t* n, int64_t* num_blocks, int64_t* nnz,
                           int32_t* batch);

/*
 * Copy the plan's canonical arrays into caller buffers (device pointers, any may be NULL):
 *   perm      int32 [N]       tokens in block order (ascending token index inside a block)
 *   tok_blk   int32 [N]       block index of every token
 *   blk_off   int32 [Mb + 1]  first position in perm of every block
 *   blk_coord int32 [Mb, 3]   block coordinates (bx, by, bz)
 *   blk_seq   int32 [Mb]      sequence of every block
 *   nbr_off   int64 [N + 1]   window CSR offsets
 *   nbr_idx   int32 [nnz]     window neighbours (global token indices), ascending per row
 * Waits for the device.
 */
SSA_API ssa_status_t ssa_plan_export(ssa_plan_t plan, int32_t* perm, int32_t* tok_blk, int32_t* blk_off,
                             int32_t* blk_coord, int32_t* blk_seq, int64_t* nbr_off,
                             int32_t* nbr_idx, void* stream);

/*
 * Forward pass: out = g0*o_cmp + g1*o_sel + g2*o_win for every token and head.
 * Direct3D-S2 summary page, "Technical principles of Direct3D-S2", SSA item: each block is
 * compressed into a block-level token (here block mean times Wc), important blocks are selected
 * from the compression module's attention scores (own block plus the top k-1 others), the local
 * window adds fine detail, and the three outputs are aggregated with gating scores (given here
 * as the `gates` input).
 *   q, k, v:  device [N, H, D] of dtype.
 *   gates:    device fp32 [N, H, 3].
 *   wc:       device fp32 [D, D].
 *   heads, head_dim: H and D.
 *   topk:     k, number of selected blocks including the own block (1..32).
 *   out:      device [N, H, D] of dtype (written in token order).
 * Queues work on `stream` and returns without waiting. The first call for a given
 * (H, D, dtype, k) allocates the plan's workspace; later calls allocate nothing.
 * Not reentrant on one plan: calls that share a plan must be ordered on one stream.
 * bf16 / fp16: a sequence may hold at most 65,536 * D / 32 occupied blocks (the union of the
 * selected blocks is built in on-chip memory); more returns SSA_ERR_UNSUPPORTED.
 */
SSA_API ssa_status_t ssa_forward(ssa_plan_t plan, const void* q, const void* k, const void* v,
                         const float* gates, const float* wc, int32_t heads, int32_t head_dim,
                         ssa_dtype_t dtype, int32_t topk, void* out, void* stream);

/*
 * As ssa_forward, and also writes what the three branches produced (same passage as
 * ssa_forward). Every extra output is optional (NULL = not written):
 *   sel_out: device int32 [N, H, k], the selected blocks (global block indices; slot 0 = own
 *            block, then the others by descending compressed score; -1 = empty slot);
 *   o_cmp, o_sel, o_win: device fp32 [N, H, D] in token order, each branch's normalised
 *            attention output before the gates (the kernels' fp32 accumulators).
 * Same errors and stream behaviour as ssa_forward.
 */
SSA_API ssa_status_t ssa_forward_debug(ssa_plan_t plan, const void* q, const void* k, const void* v,
                               const float* gates, const float* wc, int32_t heads,
                               int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* out,
                               int32_t* sel_out, float* o_cmp, float* o_sel, float* o_win,
                               void* stream);

/*
 * Forward pass with the attention prologue of the transformer that runs SSA (Hi3D v1.0 pipeline
 * page, "Stage 3: sparse flow sampling": rotary position embeddings and RMS normalisation of the
 * self-attention queries and keys). Before the method, q and k are each replaced, per token and
 * head, by
 *   u = x / sqrt(mean_d x_d^2 + eps) * gamma     (RMS normalisation over the head dimension)
 * followed by a 3D rotary embedding at the token's voxel coordinates (x, y, z) from the plan: the
 * head dimension is cut into an x part of D - 2c channels and y and z parts of c = 2*floor(D/6)
 * channels each; channel pair (2p, 2p+1), the j-th pair of a part of width w along axis a, turns
 * by the angle coords[a] * rope_theta^(-2j/w). V is not transformed.
 *   q_gamma, k_gamma: device fp32 [D] weights of the normalisation (shared by all heads).
 *   rope_theta: base of the rotary frequencies (> 1), e.g. 10000. eps: >= 0.
 *   sel_out: optional device int32 [N, H, k], as in ssa_forward_debug (NULL = not written).
 * Everything else as ssa_forward. bf16 / fp16: the transform runs inside the pooling kernel (keys)
 * and on each query tile after its load (queries), with fp32 arithmetic and the transformed
 * values rounded to the input type; fp32: a separate pass into workspace copies of q and k.
 * Errors: as ssa_forward, and SSA_ERR_INVALID_ARG for a NULL weight, rope_theta <= 1 or eps < 0.
 */
SSA_API ssa_status_t ssa_forward_prologue(ssa_plan_t plan, const void* q, const void* k, const void* v,
                                  const float* gates, const float* wc, const float* q_gamma,
                                  const float* k_gamma, float rope_theta, float eps, int32_t heads,
                                  int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* out,
                                  int32_t* sel_out, void* stream);

/*
 * Options of ssa_forward_ex; a NULL pointer (or a zero-initialised struct) turns a part off.
 *   q_gamma, k_gamma, rope_theta, rms_eps: the attention prologue of ssa_forward_prologue (both
 *       weights set, or neither).
 *   conv_w: device fp32 [27, D, D]. Compression by sparse 3D convolution over the block grid in
 *       place of the block mean times Wc (Direct3D-S2 summary page, "Technical principles of
 *       Direct3D-S2", SSA item: blocks become block-level tokens by sparse 3D convolution and
 *       pooling). The block means of K and V go through one 3x3x3 convolution over the occupied
 *       blocks of each sequence, stride 1, outputs at the occupied blocks only, an absent neighbour
 *       contributing nothing: Kc_b = sum_o mean(K_{b+o}) . W_o, with W_o = conv_w[9(dx+1) +
 *       3(dy+1) + (dz+1)] for the offset o = (dx, dy, dz), shared by K, V and all heads. The centre
 *       tap alone (W_(0,0,0) = Wc, others zero) is the plain method.
 *   gate_w, gate_b: device fp32 [D, 3] and [3]. Gates predicted from the queries (same item: the
 *       branches are aggregated with predicted gating scores): g = sigmoid(q . gate_w + gate_b) per
 *       token and head, q being the query as the attention sees it (after the prologue, in the
 *       input type), order (cmp, sel, win). Both set, or neither.
 *   select_share: 0 = every query selects its own blocks (the plain method); 1 = the queries of
 *       each 4x4x4 sub-block of cells (same (floor(x/4), floor(y/4), floor(z/4)) in one sequence;
 *       it lies in one 8x8x8 block) share one selection: their own block plus the top (k-1)
 *       other blocks by the sum over the sub-block's queries of their compressed-attention
 *       weights (softmax of the compressed logits), equal sums to the lower block index. The
 *       pages choose the blocks from the compression module's attention scores (same item)
 *       without saying whose; this pools them over neighbouring queries. bf16 / fp16 only
 *       (SSA_ERR_UNSUPPORTED for fp32). The first call builds the plan's sub-block order and
 *       its selection tiles (whole sub-blocks of a sequence, at most 128 rows and 32 sub-blocks
 *       each, packed on the host: the call waits for the stream twice).
 */
typedef struct {
    const float* q_gamma;
    const float* k_gamma;
    float rope_theta;
    float rms_eps;
    const float* conv_w;
    const float* gate_w;
    const float* gate_b;
    int32_t select_share;
} ssa_options_t;

/*
 * Forward pass with options (ssa_options_t; NULL = the plain ssa_forward). `gates` is not read,
 * and may be NULL, when the gates are predicted; `wc` likewise with a convolution compression.
 * sel_out: optional device int32 [N, H, k] (NULL = not written). Otherwise as ssa_forward; the
 * first call with a convolution builds the plan's block neighbour table (27 per block).
 * Errors: as ssa_forward, and SSA_ERR_INVALID_ARG for options set inconsistently.
 */
SSA_API ssa_status_t ssa_forward_ex(ssa_plan_t plan, const void* q, const void* k, const void* v,
                            const float* gates, const float* wc, int32_t heads, int32_t head_dim,
                            ssa_dtype_t dtype, int32_t topk, const ssa_options_t* options, void* out,
                            int32_t* sel_out, void* stream);

/*
 * ssa_forward on HOST buffers: copies q, k, v, gates, wc (host) to plan-owned device buffers,
 * runs the forward and copies the result into out (host). When H has a divisor h < H whose token
 * rows are at least 256 bytes (h D element size), the heads go in chunks of the smallest such h:
 * the copies of one chunk in, the forward of the previous one and the copy of the one before
 * that out overlap on two plan-owned side streams (first call: streams, events and two slots of
 * chunk buffers are created). Results equal the device forward's bit for bit. Pinned host memory
 * gives overlapped, full-speed copies; pageable memory works but is slower. The side streams
 * start after the work queued on `stream` before the call. Waits for the device before returning.
 */
SSA_API ssa_status_t ssa_forward_host(ssa_plan_t plan, const void* q, const void* k, const void* v,
                              const float* gates, const float* wc, int32_t heads,
                              int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* out,
                              void* stream);

/*
 * Backward pass (Direct3D-S2 model page, "What is Direct3D-S2?" and "Technical snapshot": the
 * method trains through SSA, with a faster backward than baseline sparse attention): gradients
 * of sum(dO * out) with respect to q, k, v, with the block
 * selection held fixed (it is not differentiable) and the compressed tokens' rounding treated as
 * identity. dq, dk, dv: device [N, H, D] of dtype. Runs the forward first (for the selection).
 * The compressed branch goes through cuBLAS strided-batched GEMMs per sequence (TF32 tensor cores
 * for bf16 / fp16, fp32 for fp32; the first call creates the plan's cuBLAS handle) with fp32
 * buffers of rows x blocks per head (up to 16 GB each, two of them); the selected and window
 * branches through CUDA-core kernels for the query side and, over inverted selection lists and
 * the window lists, the key side, with fp32 accumulation and no atomics. Queues work and returns
 * without waiting (the buffers are allocated and freed stream-ordered through the allocator).
 */
SSA_API ssa_status_t ssa_backward(ssa_plan_t plan, const void* q, const void* k, const void* v,
                          const float* gates, const float* wc, const void* dout, int32_t heads,
                          int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* dq, void* dk,
                          void* dv, void* stream);

/* Wait for `stream`, then read and clear the plan's device status word. */
SSA_API ssa_status_t ssa_last_device_status(ssa_plan_t plan, void* stream);

/*
 * Failure-detection check (measurement support, not part of the method): launches one warp that
 * waits, with the same bounded mbarrier wait every kernel of this library uses, on a barrier that
 * nothing arrives at, giving up after about max_cycles SM clock cycles (>= 1). The wait that runs
 * out records a device timeout in the plan's status word: the next ssa_last_device_status (or any
 * call that waits for the device) returns SSA_ERR_DEVICE_TIMEOUT and clears it; the context stays
 * usable. Queues work on `stream` and returns without waiting.
 */
SSA_API ssa_status_t ssa_debug_wait_timeout(ssa_plan_t plan, int64_t max_cycles, void* stream);

/* Release a plan and every buffer it owns (queued on the stream it was created on). */
SSA_API ssa_status_t ssa_plan_destroy(ssa_plan_t plan);

/* Static description of a status code. */
SSA_API const char* ssa_status_string(ssa_status_t status);

/*
 * Block offsets of one sequence without allocating device memory. The method has no counterpart
 * of this call: it is a convenience for callers that must not allocate (for example while other
 * work owns the allocator). It computes what the plan's block partition yields as blk_off: the
 * CSR token offsets of the occupied 8^3 blocks in block-key order (x-block major, then y, then z).
 *   coords:            device int32 [n, 3] voxel coordinates, n >= 1.
 *   grid:              host int32[3] grid extent, each in 1..65535.
 *   blk_off:           device int32 [blk_off_capacity]; receives n_blocks + 1 offsets
 *                      (blk_off[n_blocks] = number of tokens).
 *   blk_off_capacity:  must be >= min(n, number of grid blocks) + 1.
 *   n_blocks:          device int32 scalar; receives the number of occupied blocks, or -1 if a
 *                      coordinate lies outside the grid.
 * Scratch is one fixed device array inside the library (16.8 MB, enough for grids of up to
 * 2^21 blocks of 8^3 cells, i.e. 1024^3 cells). Each call clears what it uses first; nothing has
 * to start at zero. Calls that overlap in time share the array and race: serialise them (one
 * stream, or ordered with events). The first call on a device looks up the array's address.
 * Errors: SSA_ERR_INVALID_ARG (null pointer, n < 1, grid out of range, capacity too small),
 * SSA_ERR_UNSUPPORTED (more than 2^21 grid blocks), SSA_ERR_CUDA. Asynchronous on `stream`.
 */
SSA_API ssa_status_t ssa_block_offsets_noalloc(const int32_t* coords, int64_t n, const int32_t* grid,
                                               int32_t* blk_off, int64_t blk_off_capacity,
                                               int32_t* n_blocks, void* stream);

/* Number of kernels this library has launched in the process so far. */
SSA_API int64_t ssa_launch_count(void);

/*
 * Kernel timing (measurement support, not part of the method). When enabled, each hot step
 * (plan, pool, k_ssa_fwd) is bracketed by two CUDA
 * events recorded on the stream it is launched on. ssa_profile_read waits for the recorded
 * events, adds their durations to per-name totals and copies up to max_entries totals out:
 * names (host char[max_entries][64], NUL-terminated), total_ms and launches (host arrays; any
 * may be NULL). Returns the number of entries. ssa_profile_reset clears the totals.
 */
SSA_API ssa_status_t ssa_profile_enable(int32_t on);
SSA_API ssa_status_t ssa_profile_reset(void);
SSA_API int32_t ssa_profile_read(int32_t max_entries, char* names, double* total_ms,
                                 int64_t* launches);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H */
