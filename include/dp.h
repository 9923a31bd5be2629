/*
 * dp.h — C ABI of the DualParal window-step library for NVIDIA B200 (sm_100a).
 *
 * The method ("Minute-Long Videos with Dual Parallelisms", arXiv 2505.21070, abstract;
 * pith.science review of the same paper, Sections 3.1-3.2 and Figure 1) denoises a FIFO
 * queue of temporal blocks of latent frames, each block at its own (staggered) noise
 * level, in one DiT forward per step.  Every block's tokens attend to the window's own K/V
 * plus the cached K/V features of the block that last left the queue; each step pushes a
 * noisy block at the tail and pops a clean block at the head.  This library computes, on
 * one GPU, the per-step hot path of that scheme:
 *
 *   A0  per-block adaLN lookup (host)         dp_blocks_from_table, dp_queue_blocks
 *   A1  K/V modulation prepass                dp_adaln_modulate
 *   A2  window attention over [cache ; window] with the Q modulation fused into its
 *       prologue and the gate (+ residual) into its epilogue   dp_window_attention
 *   A3  queue and cache advance               dp_kvcache_advance, dp_queue_push/pop
 *   A4  the whole step A1 -> A2 -> A3         dp_window_step
 *   the queue's schedule over a whole video (host) and the coordinated noise
 *   initialisation's frame selection: dp_fifo_*, dp_coordinated_frames
 *   B   the DiT attention sublayer around A2 (pre-norm, q/k/v and output projections on
 *       caller-supplied weights): dp_ln_modulate, dp_linear, dp_qkv_project,
 *       dp_out_project, dp_sublayer_step
 *   C   the fresh-context variant of the cache (context K/V recomputed at the step that
 *       uses them, not reused from the block's last evaluation): dp_context_refresh,
 *       dp_context_refresh_sublayer
 *
 * Conventions (all entry points):
 *  - Token tensors are row-major [rows][hidden], hidden = n_heads * head_dim, channel
 *    c = h * head_dim + d.  Window rows are ordered head block (cleanest, smallest
 *    timestep) first.
 *  - Element types (dp_dtype): window inputs q, k, v, residual, out, noise and the latent
 *    queue are DP_BF16 (or DP_F32 for the fp32 path).  The modulated features k', v' and
 *    the cache are DP_F16 on the bf16 path (11-bit significand: with bf16 features the
 *    rounding of q', k', v' alone exceeds 2e-2 absolute on peaked softmaxes; f16 features
 *    saturate at +-65504) and DP_F32 on the fp32 path.  adaLN vectors are always float.
 *  - Ownership: the caller owns every device buffer; the library allocates no device
 *    memory on any call.  Descriptor structs are host-side plain data; the library
 *    updates their counters deterministically.
 *  - Asynchrony: work is enqueued on the given stream (a cudaStream_t; NULL = the legacy
 *    default stream) of the current device (see dp_set_device).  Argument errors are
 *    returned synchronously before anything is enqueued and leave descriptors unchanged.
 *  - Alignment: every device pointer must be 16-byte aligned and hidden * element size a
 *    multiple of 16 bytes.
 *  - Errors: launch failures return DP_ERR_CUDA (dp_last_error_detail() gives the CUDA
 *    message).  Bounded device-side waits that give up record DP_ERR_TIMEOUT in a device
 *    status word read by dp_device_status(); the kernel then returns without hanging.
 */
#ifndef DP_H
#define DP_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DP_MAX_BLOCKS 16   /* blocks in one window */
#define DP_MAX_SLOTS 16    /* slots of the latent queue and of the cache ring */

typedef enum {
  DP_OK = 0,
  DP_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, inconsistent sizes or offsets */
  DP_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. bf16 head_dim not 64/128) */
  DP_ERR_CUDA = -3,         /* a CUDA call or kernel launch failed */
  DP_ERR_CAPACITY = -4,     /* a block does not fit its cache slot / queue slot / queue */
  DP_ERR_TIMEOUT = -5,      /* a bounded device-side wait gave up (see dp_device_status) */
  DP_ERR_EMPTY = -6         /* pop from an empty queue */
} dp_status;

typedef enum { DP_F32 = 0, DP_BF16 = 1, DP_F16 = 2 } dp_dtype;

/* dp_window_attention flags */
#define DP_MOD_Q 1u     /* prologue: q' = q * (1 + scale_b) + shift_b, b = block of the row */
#define DP_GATE_OUT 2u  /* epilogue: out = gate_b * o (+ residual) */
/* Test hook for the failure path of the tensor-core kernel: its producer issues no K/V
 * loads, so every wait for them gives up at its bound (about 2 s of SM clock); the kernel
 * then stops, releases its resources and returns without writing `out`, and
 * dp_device_status() reports DP_ERR_TIMEOUT.  Nothing faults or hangs.  Use it with a
 * small launch (one CTA: n_win <= 256 rows and one head) so that one bound elapses. */
#define DP_TEST_SKIP_KV_LOADS 0x80000000u

/* dp_window_step flags */
#define DP_STEP_POP 1u  /* after attention, the head block exits: its K'/V' rows become the
                           cache (and the queue, if given, pops its head) */
#define DP_STEP_CACHE_ALL_SLOTS 2u  /* attention reads every slot of the cache ring that holds
                           rows (the K/V of the last n_slots exited blocks: a context of
                           several blocks, the pages' NumC frames), not only the most
                           recently written one */

/*
 * Window block table (host plain data, passed by pointer, copied into kernel arguments).
 * Block b owns window rows [row_offset[b], row_offset[b+1]); row_offset[0] = 0, offsets
 * non-decreasing, row_offset[n_blocks] = the window's row count.  mod[b] is a DEVICE
 * pointer to 3 * hidden floats: shift[hidden], scale[hidden], gate[hidden] — block b's
 * adaLN vectors for its own timestep (the review's Section 3.1: neighbouring blocks sit
 * at neighbouring noise levels; the DiT conditions each block on its own timestep).
 */
typedef struct {
  int32_t n_blocks;
  int32_t hidden;
  int32_t row_offset[DP_MAX_BLOCKS + 1];
  const float* mod[DP_MAX_BLOCKS];
} dp_blocks;

/*
 * Feature cache (the review's Section 3.2: the self-attention K/V features of the block
 * that just left, reused as context, one denoising step stale).  A ring of n_slots slots,
 * each [capacity][hidden] in k and in v (DEVICE, caller-owned, [n_slots][capacity][hidden]).
 * An advance writes slot (n_advances mod n_slots); attention reads the most recently
 * written slot (slot 0 before the first advance, whose contents the caller may preset
 * together with len[0]).
 */
typedef struct {
  void* k;
  void* v;
  int64_t capacity;
  int32_t hidden;
  int32_t n_slots;
  int64_t len[DP_MAX_SLOTS];
  int64_t n_advances;
  dp_dtype dtype;
} dp_kvcache;

/*
 * Latent block queue (the review's key machinery: a FIFO of blocks with noise levels
 * decreasing from tail to head).  latent is DEVICE memory [2 * n_slots][slot_rows][hidden],
 * a mirrored ring: a block pushed to physical slot p is written to slots p and p + n_slots,
 * so the live window, slots [head, head + count), is always one contiguous range.
 * rows[i] and evals[i] describe the block at logical position i (0 = head).  Only the
 * tail block may hold fewer than slot_rows rows (a ragged final block); no push may
 * follow it.
 */
typedef struct {
  void* latent;
  int64_t slot_rows;
  int32_t hidden;
  int32_t n_slots;
  int32_t head;
  int32_t count;
  int32_t rows[DP_MAX_SLOTS];
  int32_t evals[DP_MAX_SLOTS];
  int64_t n_pushed;
  int64_t n_popped;
  dp_dtype dtype;
} dp_queue;

/* ---------------------------------------------------------------- A0: host lookups */

/* Fill *out for n_blocks blocks: rows block_rows[b] (host), adaLN row table[timesteps[b]]
 * (the table is DEVICE memory [table_rows][3][hidden] float, standing in for the DiT's
 * timestep MLP).  INVALID_ARG on a timestep outside [0, table_rows) or n_blocks outside
 * [1, DP_MAX_BLOCKS]. */
dp_status dp_blocks_from_table(dp_blocks* out, const float* table, int32_t table_rows,
                               int32_t hidden, const int32_t* timesteps,
                               const int32_t* block_rows, int32_t n_blocks);

/* Block table of the queue's live window: block i gets rows[i] and adaLN row
 * table[tau[evals[i]]] (tau: host array of n_tau timesteps, noisiest first).  *window
 * receives the DEVICE address of the head block's first row (q = k = v of the window),
 * *n_win the window's row count.  EMPTY if no block is live; INVALID_ARG if a block has
 * already had n_tau evaluations. */
dp_status dp_queue_blocks(const dp_queue* q, const float* table, int32_t table_rows,
                          const int32_t* tau, int32_t n_tau, dp_blocks* out,
                          const void** window, int64_t* n_win);

/* ---------------------------------------------------------------- A1: modulation */

/* y[i, c] = x[i, c] * (1 + scale_b[c]) + shift_b[c] for every row i of block b, in fp32
 * (one fused multiply-add, 1 + scale rounded to float), rounded once to y's type (round to
 * nearest even; f16 saturates at +-65504).  x: DEVICE [n_rows][hidden] of x_dt; y: DEVICE
 * [n_rows][hidden] of y_dt; (x_dt, y_dt) is (bf16, bf16), (bf16, f16), (f16, f16) or
 * (f32, f32), else UNSUPPORTED.  y may equal x when the types match (in place), no other
 * overlap.  n_rows must equal blk->row_offset[blk->n_blocks]. */
dp_status dp_adaln_modulate(const void* x, void* y, int64_t n_rows, const dp_blocks* blk,
                            dp_dtype x_dt, dp_dtype y_dt, void* stream);

/* ---------------------------------------------------------------- A2: attention */

/* Window attention (the abstract's feature cache reused as context; the review's
 * Section 3.2 self-attention over the cached K/V of the neighbouring block):
 *   q'_i  = DP_MOD_Q ? q_i * (1 + scale_b) + shift_b : q_i          (b = block of row i)
 *   o_i,h = sum_j softmax_j(q'_i,h . K_j,h * softmax_scale) V_j,h,
 *           j over cache rows [0, cache_len) then window rows [0, n_win)
 *   out_i = (DP_GATE_OUT ? gate_b * o_i : o_i) + (residual ? residual_i : 0)
 * q, residual, out: DEVICE [n_win][hidden] of dt; k, v: DEVICE [n_win][hidden] of
 * feat_dt, entering as given (the window's modulated features); cache_k, cache_v: DEVICE
 * feat_dt, at least cache_len rows.  residual may be NULL.  out must not overlap any
 * input.  softmax_scale <= 0 selects 1/sqrt(head_dim).  (dt, feat_dt) = (bf16, f16) or
 * (bf16, bf16): tensor cores, head_dim 64 or 128, q' and P rounded to feat_dt, fp32
 * accumulation and softmax; (f32, f32): CUDA cores, full fp32, head_dim 4, 8, 16, 32, 64
 * or 128.  UNSUPPORTED otherwise. */
dp_status dp_window_attention(const void* q, const void* k, const void* v, int64_t n_win,
                              const void* cache_k, const void* cache_v, int64_t cache_len,
                              const void* residual, void* out, int32_t n_heads,
                              int32_t head_dim, float softmax_scale, const dp_blocks* blk,
                              uint32_t flags, dp_dtype dt, dp_dtype feat_dt, void* stream);

/* ---------------------------------------------------------------- A3: advance */

/* The exiting head block's features become the cache: rows [0, n_exit) of k_exit and
 * v_exit (DEVICE [n_exit][hidden]) are copied into slot (n_advances mod n_slots);
 * len[slot] = n_exit; n_advances += 1.  A byte copy (bit-exact).  CAPACITY if n_exit >
 * capacity.  n_exit = 0 empties the slot. */
dp_status dp_kvcache_advance(dp_kvcache* c, const void* k_exit, const void* v_exit,
                             int64_t n_exit, void* stream);

/* Push a fresh noise block (DEVICE [rows][hidden]) at the queue's tail (byte copy into the
 * mirrored ring); the new block has evals = 0.  CAPACITY if the queue is full or rows >
 * slot_rows; INVALID_ARG if the current tail is a short (final) block. */
dp_status dp_queue_push(dp_queue* q, const void* noise, int64_t rows, void* stream);

/* Coordinated noise initialisation's push (the abstract: initial noise patterns shared
 * without extra cost; the review: each new block drawn from the full noise space, shuffled so
 * that concatenated blocks do not repeat noise): the pushed block is the concatenation of
 * frames frame_idx[0 .. n_frames) (host array) of pool (DEVICE [pool_frames][frame_rows]
 * [hidden], the queue's type), written to the queue's tail slot like dp_queue_push (byte
 * copy, bit-exact).  Which frames (the shuffle) is the caller's choice;
 * dp_coordinated_frames implements the selection rule.  n_frames in [1, 16] (UNSUPPORTED
 * otherwise); INVALID_ARG for an index outside [0, pool_frames); CAPACITY as dp_queue_push
 * for n_frames * frame_rows rows. */
dp_status dp_queue_push_frames(dp_queue* q, const void* pool, int32_t pool_frames,
                               int64_t frame_rows, const int32_t* frame_idx, int32_t n_frames,
                               void* stream);

/* Pop the head block (metadata only: the slot becomes free).  EMPTY if no block. */
dp_status dp_queue_pop(dp_queue* q);

/* ---------------------------------------------------------------- the queue's schedule (host) */

/*
 * The FIFO schedule of a whole video (the review's key machinery and its Figure 1: blocks
 * enter at the tail one after another, every live block is evaluated once per step at its
 * own timestep, and a block leaves at the head after its last evaluation).  Block b enters
 * at step e_b = floor(b * T / W): with T evaluations per block and W blocks in the
 * steady-state window this gives exactly W live blocks in the steady state, T evaluations
 * of every block, and the exit of block b in the same step as the entry of block b + W
 * (the pages give no stagger; this is the plainest one with those properties).  The video
 * has n_blocks blocks; the run ends after step e_{n_blocks-1} + T - 1.  T >= W >= 1 (at
 * most one block enters per step), W <= DP_MAX_SLOTS.  Host plain data; the library
 * updates it in dp_fifo_commit.
 */
typedef struct {
  int32_t n_blocks;       /* blocks in the whole video */
  int32_t n_timesteps;    /* T: evaluations per block */
  int32_t window_blocks;  /* W: live blocks in the steady state */
  int32_t next_block;     /* the next block to enter (0: none has entered yet) */
  int64_t step;           /* schedule steps taken */
  int64_t exited_rows;    /* rows of the block that left last (0 before the first exit) */
} dp_fifo;

/* What one step of the schedule does, as dp_fifo_plan computes it. */
typedef struct {
  int32_t push_before;    /* block to push before the step (block 0 at step 0), else -1 */
  int32_t pop;            /* 1: the head block has its last evaluation in this step and
                             exits after it (DP_STEP_POP) */
  int32_t push_after;     /* block that enters after this step (pushed with or after it), else -1 */
  int32_t done;           /* 1: every block has left; there is no step to take */
  int64_t exit_rows;      /* rows of the head block when pop = 1, else 0 */
  const void* ctx_rows;   /* DEVICE address of the latent rows of the block that left last,
                             while the queue still holds them in the slot behind its head
                             (a queue with more slots than W), else NULL: the rows a fresh
                             context is recomputed from */
  int64_t ctx_n;          /* their row count (0 with ctx_rows NULL) */
} dp_fifo_step;

/* Entry step of block b: *step = floor(b * T / W).  INVALID_ARG unless b >= 0 and
 * T >= W >= 1. */
dp_status dp_fifo_entry_step(int32_t b, int32_t n_timesteps, int32_t window_blocks, int64_t* step);

/* A fresh schedule of n_blocks blocks (step 0, no block entered).  INVALID_ARG unless
 * n_blocks >= 1 and T >= W with 1 <= W <= DP_MAX_SLOTS. */
dp_status dp_fifo_init(dp_fifo* f, int32_t n_blocks, int32_t n_timesteps, int32_t window_blocks);

/* The next step of the schedule f for the queue q (host descriptor; its state after
 * push_before is what the step sees): whether the head block exits after the step, which
 * block enters, and the rows of the block that left last.  The queue must match the
 * schedule (its live count and its head block's evaluation count at this step, counting
 * push_before), else INVALID_ARG; done = 1 once every block has left.  Reads q only. */
dp_status dp_fifo_plan(const dp_fifo* f, const dp_queue* q, dp_fifo_step* out);

/* Record that the planned step ran (and its pushes were made): step += 1, next_block moves
 * past push_before and push_after, exited_rows = exit_rows when pop.  INVALID_ARG if the
 * plan is not the schedule's next step. */
dp_status dp_fifo_commit(dp_fifo* f, const dp_fifo_step* s);

/* Coordinated noise initialisation, the frame selection (the abstract: initial noise
 * patterns shared at no extra cost; the review: a full noise pool, shuffled assignment,
 * the last latents excluded).  The pool is the first window: the frames of blocks
 * 0 .. W-1, pool_frames = block_frames[0] + ... + block_frames[W-1] (W = min(window_blocks,
 * n_blocks)).  Block b < W takes its own frames of the pool in order; block b >= W takes
 * the pool frames in the order of perm (host, a permutation of [0, pool_frames), drawn by
 * the caller), skipping prev_frames (host, n_prev frames: the block just before it), the
 * first block_frames[b] of them.  frames_out (host) receives block_frames[b] pool frame
 * indices.  INVALID_ARG if perm is not a permutation (for b >= W), b is outside
 * [0, n_blocks), or the pool holds fewer than block_frames[b] frames outside prev_frames;
 * the result goes to dp_queue_push_frames. */
dp_status dp_coordinated_frames(const int32_t* block_frames, int32_t n_blocks, int32_t window_blocks,
                                int32_t b, const int32_t* prev_frames, int32_t n_prev,
                                const int32_t* perm, int32_t* frames_out);

/* ---------------------------------------------------------------- A4: window step */

/* One window step:
 *   1. k' = modulate(k), v' = modulate(v) into kv_work (DEVICE scratch, caller-allocated,
 *      2 * n_win * hidden feature elements: k' at element 0, v' at element n_win * hidden);
 *   2. out = dp_window_attention(q, k', v', cache, DP_MOD_Q | DP_GATE_OUT, residual);
 *   3. queue (if given): every live block's evals += 1;
 *   4. if flags & DP_STEP_POP: the head block (rows [0, row_offset[1])) exits — its k'/v'
 *      rows are written into the cache ring (dp_kvcache_advance), and the queue (if
 *      given) pops its head;
 *   5. if push_noise: it is pushed at the queue's tail (dp_queue_push; needs queue).
 * With DP_STEP_CACHE_ALL_SLOTS, step 2's cache rows are those of every slot with len > 0
 * (oldest first; the order does not change the result), else those of the most recently
 * written slot.  Steps 4 and 5 run as one copy kernel after the attention on the same stream.  All
 * argument checks (including capacities) happen before anything is enqueued.  q, k, v,
 * residual, out, push_noise and the queue are of type dt (bf16 or f32); kv_work and the
 * cache hold features (f16 for bf16, f32 for f32).  q, k and v may alias one another (the
 * queue's window); out and kv_work overlap nothing. */
dp_status dp_window_step(const void* q, const void* k, const void* v, int64_t n_win,
                         const dp_blocks* blk, dp_kvcache* cache, void* kv_work,
                         const void* residual, void* out, int32_t n_heads, int32_t head_dim,
                         uint32_t flags, dp_queue* queue, const void* push_noise,
                         int64_t push_rows, dp_dtype dt, void* stream);

/* ---------------------------------------------------------------- step without allocation */

/* Size in bytes of the fixed scratch array dp_window_step_noalloc uses on each device. */
#define DP_NOALLOC_SCRATCH_BYTES (32u << 20)

/* dp_window_step without the kv_work argument, for callers that cannot allocate device
 * memory: code embedded in a host that owns all device memory (a framework's caching
 * allocator, a plugin interface that hands over only inputs and outputs) or latency-bound
 * loops where cudaMalloc/cudaFree would synchronize the device.  The pages describe no
 * such entry point; it exists only for such integrations.
 * The window's k'/v' scratch is a fixed array of DP_NOALLOC_SCRATCH_BYTES inside the
 * library's device memory, held by every device that loads the library until the process
 * exits.  The call allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 * CAPACITY, before anything is enqueued, if 2 * n_win * n_heads * head_dim feature
 * elements (2 bytes each for bf16 windows, 4 for fp32) exceed that size (the sizes are
 * compared without forming the product, so no size overflows).  The first call on a
 * device, and the first after a device reset (a new CUDA context, recognised by its
 * context id), looks up the array's device address (cudaGetSymbolAddress, with that device
 * current); make that first call before any stream capture.  All calls share the one
 * array: calls whose work overlaps on the GPU (other streams, other threads) race on it;
 * order them on one stream.  Its contents from earlier calls are never read (the
 * modulation prepass overwrites every element it uses).  Arguments, results and errors are
 * otherwise those of dp_window_step. */
dp_status dp_window_step_noalloc(const void* q, const void* k, const void* v, int64_t n_win,
                                 const dp_blocks* blk, dp_kvcache* cache, const void* residual,
                                 void* out, int32_t n_heads, int32_t head_dim, uint32_t flags,
                                 dp_queue* queue, const void* push_noise, int64_t push_rows,
                                 dp_dtype dt, void* stream);

/* ---------------------------------------------------------------- B: DiT attention sublayer */

/*
 * The DiT layer around the window attention, with the adaLN conditioning of the pages'
 * DiT (the review's Section 3.1: each block is denoised at its own timestep; Section 3.2:
 * the self-attention K/V of the block that left are cached):
 *   B1  h   = LN(x) * (1 + scale_b) + shift_b          dp_ln_modulate
 *   B2  q, k, v = h W_qkv^T + b_qkv                     dp_qkv_project (dp_linear: plain)
 *   A2  o   = attention over [cache ; window k, v]     dp_window_attention, no flags
 *   B3  out = x + gate_b * (o W_o^T + b_o)              dp_out_project
 *   B4  the whole sublayer step and its advance         dp_sublayer_step
 * Weights are the caller's (trained weights are not part of this library): W_qkv DEVICE
 * [3 * hidden][hidden] bf16 and W_o [hidden][hidden] bf16, out-features by in-features
 * (row i of W holds output feature i's input weights), biases DEVICE float [3 * hidden] /
 * [hidden] or NULL.  Products run on the tensor cores with fp32 accumulation.
 */

/* B1: h_i = (x_i - mean_i) / sqrt(var_i + eps) * (1 + scale_b) + shift_b, mean and (biased)
 * variance over the row's hidden channels, computed in fp32 (two passes) and rounded once
 * to bf16; b = block of row i.  x, h: DEVICE [n_rows][hidden] bf16, h may equal x.
 * hidden = blk->hidden must be a multiple of 256 and at most 8192 (UNSUPPORTED
 * otherwise); eps > 0. */
dp_status dp_ln_modulate(const void* x, void* h, int64_t n_rows, const dp_blocks* blk, float eps,
                         void* stream);

/* y = a W^T + bias: a DEVICE [m][k] bf16, w DEVICE [n][k] bf16, bias DEVICE [n] float or
 * NULL, y DEVICE [m][n] of y_dt (bf16, or f16 saturating at +-65504), rounded once from
 * the fp32 sum (round to nearest even).  n a multiple of 128 and k of 8 (UNSUPPORTED
 * otherwise).  y overlaps no input. */
dp_status dp_linear(const void* a, const void* w, const float* bias, int64_t m, int32_t n,
                    int32_t k, void* y, dp_dtype y_dt, void* stream);

/* B2: [q | k | v] = h W_qkv^T + b_qkv, split by output column: q (columns [0, hidden))
 * DEVICE [n_rows][hidden] bf16 (the attention's raw query), k and v (columns [hidden,
 * 2 hidden) and [2 hidden, 3 hidden)) DEVICE [n_rows][hidden] f16 features (saturating).
 * hidden a multiple of 128. */
dp_status dp_qkv_project(const void* h, const void* w_qkv, const float* b_qkv, int64_t n_rows,
                         int32_t hidden, void* q, void* k, void* v, void* stream);

/* B3: out_i = residual_i + gate_b * (o_i W_o^T + b_o), b = block of row i, gate from
 * blk->mod[b] (after shift and scale), all in fp32, rounded once to bf16.  o, residual,
 * out: DEVICE [n_rows][hidden] bf16, hidden = blk->hidden a multiple of 128; out overlaps
 * no input. */
dp_status dp_out_project(const void* o, const void* w_o, const float* b_o, int64_t n_rows,
                         const dp_blocks* blk, const void* residual, void* out, void* stream);

/* B4: one sublayer step on the window x (DEVICE [n_win][hidden] bf16, e.g. the queue's
 * live window): B1, B2, the attention over [cache ; k, v] (softmax scale 1/sqrt(head_dim),
 * no modulation or gate inside it), B3 into out, then the advance of dp_window_step: every
 * live block's evals += 1; with DP_STEP_POP the head block's k and v rows (the projected
 * features of its last evaluation) become the cache and the queue pops; push_noise is
 * pushed at the tail.  work: DEVICE scratch of 4 * n_win * hidden 16-bit elements (h and
 * then the attention output, q, k, v); the cache holds f16 features; head_dim 64 or 128;
 * hidden a multiple of 256.  out overlaps neither x nor work.  All checks happen before
 * anything is enqueued. */
dp_status dp_sublayer_step(const void* x, int64_t n_win, const dp_blocks* blk, const void* w_qkv,
                           const float* b_qkv, const void* w_o, const float* b_o, float eps,
                           dp_kvcache* cache, void* work, void* out, int32_t n_heads,
                           int32_t head_dim, uint32_t flags, dp_queue* queue,
                           const void* push_noise, int64_t push_rows, void* stream);

/* ---------------------------------------------------------------- fresh context (cache ablation) */

/*
 * The cached variant reuses the context block's K/V as its last evaluation produced them,
 * one denoising step stale (the review's Section 3.2; the referee asks for an ablation
 * against K/V recomputed at the current step).  These calls recompute them instead: the
 * context rows go through the same feature projection as the window's own rows, with the
 * conditioning the caller gives for the current step, and the result overwrites the cache
 * slot the next step's attention reads (the most recently written slot; slot 0 before the
 * first advance).  That slot's len becomes n_ctx; n_advances and the other slots are
 * unchanged.  A following dp_window_step / dp_sublayer_step (same stream) attends to the
 * recomputed rows; with DP_STEP_CACHE_ALL_SLOTS the older slots keep their cached rows.
 * ctx_blk is the block table of the context rows (usually one block; mod[b] = that
 * block's adaLN vectors at the timestep it is conditioned on now); ctx_blk->hidden is
 * the hidden size.  n_ctx = 0 empties the slot and enqueues nothing.  CAPACITY if n_ctx
 * exceeds the cache capacity.  The context rows and scratch overlap no slot of the cache
 * ring (INVALID_ARG).
 */

/* Window-step features (identity projections, as in dp_window_step): k' = k_ctx (1 +
 * scale_b) + shift_b and v' likewise, b = the context block of the row, one fp32 fma
 * rounded once to the feature type.  k_ctx, v_ctx: DEVICE [n_ctx][hidden] of dt (DP_BF16
 * with an f16 cache, or DP_F32 with an f32 cache); they may be the same rows. */
dp_status dp_context_refresh(const void* k_ctx, const void* v_ctx, int64_t n_ctx, const dp_blocks* ctx_blk,
                             dp_kvcache* cache, dp_dtype dt, void* stream);

/* Sublayer features (as in dp_sublayer_step): h = LN(x_ctx) (1 + scale_b) + shift_b in bf16
 * (B1, eps as in dp_ln_modulate), then k = h W_k^T + b_k and v = h W_v^T + b_v in f16
 * (saturating), W_k and W_v rows [hidden, 2 hidden) and [2 hidden, 3 hidden) of w_qkv
 * (DEVICE [3 hidden][hidden] bf16), b_k and b_v the same entries of b_qkv (DEVICE float or
 * NULL).  x_ctx: DEVICE [n_ctx][hidden] bf16; work: DEVICE scratch of n_ctx * hidden bf16
 * elements, overlapping neither x_ctx nor the cache; the cache holds f16 features; hidden
 * a multiple of 256. */
dp_status dp_context_refresh_sublayer(const void* x_ctx, int64_t n_ctx, const dp_blocks* ctx_blk,
                                      const void* w_qkv, const float* b_qkv, float eps,
                                      dp_kvcache* cache, void* work, void* stream);

/* ---------------------------------------------------------------- profiling */

/* Stage timing of dp_window_step and dp_sublayer_step.  After dp_profile_begin(max_steps),
 * the next max_steps such calls on this thread record CUDA events (created and owned by the
 * library; no device memory) on their stream at the boundaries of the modulation prepass,
 * the attention and the advance.  dp_profile_end synchronizes on the last recorded event,
 * returns the summed times in milliseconds (any output pointer may be NULL) and the number
 * of steps recorded, and releases the events.  INVALID_ARG if max_steps < 1 or if
 * profiling is already active (begin) / not active (end). */
dp_status dp_profile_begin(int32_t max_steps);
dp_status dp_profile_end(float* ms_modulate, float* ms_attention, float* ms_advance,
                         int32_t* steps);
/* The same for any recorded step kind: ms[i] (i < max_stages) receives stage i's summed
 * time — for dp_window_step 0 modulation, 1 attention, 2 advance; for dp_sublayer_step
 * 0 pre-norm and modulation, 1 q/k/v projection, 2 attention, 3 out projection,
 * 4 advance — *n_stages the most stages any recorded step had. */
dp_status dp_profile_end_stages(float* ms, int32_t max_stages, int32_t* n_stages,
                                int32_t* steps);

/* ---------------------------------------------------------------- status */

/* Make device `ordinal` current for this thread's later calls. */
dp_status dp_set_device(int32_t ordinal);

/* Synchronize `stream`, then read and clear the device status word of the current device:
 * DP_ERR_TIMEOUT if a kernel's bounded wait gave up since the last call, else DP_OK
 * (or DP_ERR_CUDA if the synchronize failed). */
dp_status dp_device_status(void* stream);

/* Static text for a status code. */
const char* dp_status_string(dp_status s);

/* Detail of the most recent failure on this thread (CUDA error text, failed check). */
const char* dp_last_error_detail(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t dp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DP_H */
