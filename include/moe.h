/*
 * moe.h -- C ABI of libmoe: the routed mixture-of-experts expert FFN on one
 * NVIDIA B200 (sm_100a).
 *
 * The method (rocketrecap.com, "FlyDSL kernels in JAX" talk summary):
 *   paragraph 2 and timestamp 5:56 -- a two-stage routed MoE GEMM: gather of
 *     each expert's tokens, group GEMM with the gate/up projections (w1, w3),
 *     SwiGLU, group GEMM with the down projection (w2), scatter back to token
 *     order; it replaces a masked dense GEMM over all experts;
 *   timestamp 8:14 -- Mixtral-8x7B, top-2 routing, FP8, a one-time load-time
 *     preshuffle of the expert weights;
 *   timestamps 4:07 and 5:05 -- the host boundary: buffers, scalars and a
 *     stream handed to the kernel launcher.
 *
 * Conventions for every entry point
 *   - Pointers marked "device" must point to memory of the current CUDA device;
 *     pointers marked "host" to host memory.  The caller owns every buffer;
 *     the library allocates no device memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *     enqueued asynchronously; no entry point except moe_get_status waits for
 *     the device.
 *   - Arguments are validated on the host before anything is enqueued; on any
 *     return other than MOE_OK nothing was enqueued and outputs are untouched.
 *   - Faults a kernel detects (a wait that timed out, an index out of range)
 *     are recorded in a device status word read by moe_get_status.  Outputs of
 *     a call whose status is not MOE_OK are undefined.
 *   - Every device pointer must be 16-byte aligned (MOE_ERR_ALIGNMENT).
 *
 * Shapes: T tokens, H = d_model, F = d_ff, E experts, k experts per token,
 * A = T*k assignments (assignment a = t*k + j is token t's j-th choice).
 * Limits: 1 <= k <= min(E, 8), E <= 64, H % 128 == 0, F % 128 == 0,
 * 0 <= T, T*k <= 262144 (MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,    /* null pointer, bad dimension or k/E out of range */
    MOE_ERR_UNSUPPORTED = -2,    /* valid request outside what the kernels implement */
    MOE_ERR_ALIGNMENT = -3,      /* a device pointer is not 16-byte aligned */
    MOE_ERR_WORKSPACE = -4,      /* ws_bytes < moe_workspace_size(...) */
    MOE_ERR_CUDA = -5,           /* a CUDA runtime/driver call or launch failed */
    MOE_ERR_DEVICE_TIMEOUT = -6, /* a kernel's bounded wait ran out (device status) */
    MOE_ERR_DEVICE_BOUNDS = -7   /* a kernel saw an index out of range (device status) */
} moe_status;

typedef enum {
    MOE_BF16 = 0,      /* bf16 activations and weights */
    MOE_FP8_E4M3 = 1,  /* e4m3 weights with fp32 per-output-channel scales; bf16 activations
                          quantised per token to e4m3 inside the layer */
    MOE_MXFP4 = 2      /* MX FP4 weights: e2m1 codes with one UE8M0 (power-of-two) scale per 32
                          consecutive contraction elements (the kinachrichten.com page "PyTorch
                          erhaelt FlyDSL-Backend", its kernel list: MXFP4 scaled GEMM); activations
                          and h as in MOE_FP8_E4M3 */
} moe_dtype;

/* Bytes of device workspace moe_ffn_forward needs for this problem (0 on bad
 * arguments).  The same workspace also serves moe_route. */
size_t moe_workspace_size(int T, int H, int F, int E, int k, int dtype);

/*
 * One-time weight preshuffle (timestamp 8:14, "load-time preshuffle").
 * Produces the layout the group GEMMs stream from.  Each expert matrix
 * [rows, K] (K-contiguous, `eb` = 1 byte for e4m3, 2 for bf16) is cut into
 * blocks of 128 rows x 128 bytes of K, stored contiguously in the order
 * [expert][row block][K block], 16384 bytes each.  Inside a block, the 16-byte
 * chunk c of row r sits at byte r*128 + ((c ^ (r % 8)) * 16): the 128-byte
 * swizzle of the tensor cores' shared-memory operand, so one bulk copy of a
 * block is a ready operand tile.
 * w13 holds the gate and up projections interleaved in groups of 32 rows, so
 * that one tile of the first group GEMM holds matching gate/up channels:
 *   row 64*b + i      of w13[e] = row 32*b + i of w1[e]   (i in [0,32))
 *   row 64*b + 32 + i of w13[e] = row 32*b + i of w3[e]
 * and s13 (FP8 only) is interleaved the same way, unblocked: [E, 2F] fp32.
 *   w1, w3   device, [E,F,H] row-major (bf16 or e4m3 bytes), read only
 *   s1, s3   device, [E,F] fp32 (FP8) or NULL (BF16), read only
 *   w2       device, [E,H,F] row-major, read only
 *   w13_out  device, E*2F*H*eb bytes, written (blocked layout above)
 *   s13_out  device, [E,2F] fp32 (FP8) or NULL
 *   w2_out   device, E*H*F*eb bytes, written (blocked layout above)
 * The per-output-channel scales of w2 (s2, [E,H]) are used as they are.
 */
int moe_prepare_weights(const void* w1, const void* w3, const float* s1, const float* s3, const void* w2,
                        void* w13_out, float* s13_out, void* w2_out, int E, int F, int H, int dtype, void* stream);

/*
 * One-time preparation of MX FP4 expert weights (MOE_MXFP4; the load-time
 * preshuffle of timestamp 8:14 for this format).
 *   w1, w3   device, [E,F,H/2] bytes: e2m1 codes, two per byte, the even
 *            column (d_model index) in the low 4 bits; read only
 *   s1, s3   device, [E,F,H/32] bytes: UE8M0 exponents (scale 2^(s-127)) of the
 *            blocks of 32 consecutive columns; read only
 *   w2       device, [E,H,F/2] bytes; s2 device, [E,H,F/32] bytes (blocks along d_ff)
 *   w13_out  device, E*2F*H/2 bytes: w1/w3 rows interleaved in groups of 32 as
 *            for moe_prepare_weights, still packed, cut into contiguous
 *            blocks of 128 rows x 64 bytes (128 codes of K) in the order
 *            [expert][128-row block][128-column block], so that a TMA copy of
 *            half a block reads 4 KB in one run (it puts every 16 codes into
 *            16 bytes of shared memory); 32-byte aligned
 *   s13_out  device, E*2F*H/32 bytes: the scales of those rows regrouped into
 *            512-byte chunks per (expert, 128-row block, 128-column block),
 *            byte (r%32)*16 + (r/32)*4 + b = row r of the block, 32-column
 *            block b of the chunk (the order the MMA's scale copy takes)
 *   w2_out   device, E*H*F/2 bytes, the same blocks over [E,H] rows and d_ff
 *            columns (32-byte aligned); s2_out E*H*F/32 bytes, the same chunks
 * The layer is then called with dtype MOE_MXFP4, w13 = w13_out, s13 = s13_out,
 * w2 = w2_out, s2 = s2_out.
 */
int moe_prepare_weights_mx(const void* w1, const void* w3, const void* s1, const void* s3, const void* w2,
                           const void* s2, void* w13_out, void* s13_out, void* w2_out, void* s2_out, int E, int F,
                           int H, void* stream);

/*
 * Routing alone (timestamps 5:56 and 8:14): top-k selection, softmax over the
 * k selected logits, expert histogram, exclusive scan and stable permutation.
 *   logits    device, [T,E] fp32, read only.  Larger logit first; equal logits
 *             go to the lower expert index; NaN ranks as -inf.
 *   topk_ids  device, [T,k] int32, written: chosen experts, best first.
 *   topk_w    device, [T,k] fp32, written: exp(l_j - l_max) / sum_i exp(l_i - l_max)
 *             over the chosen logits (expf, so not bit-exact with an fp64 softmax).
 *   counts    device, [E] int32, written: assignments per expert.
 *   offsets   device, [E+1] int32, written: exclusive scan of counts.
 *   perm      device, [T*k] int32, written: sorted position -> assignment,
 *             grouped by expert, ascending assignment index within an expert.
 *   inv_perm  device, [T*k] int32, written: assignment -> sorted position.
 *   ws, ws_bytes  reserved; routing alone needs no workspace (may be NULL, 0).
 * ids, counts, offsets, perm and inv_perm are deterministic (bit-identical
 * from run to run).
 */
int moe_route(const float* logits, int T, int E, int k, int32_t* topk_ids, float* topk_w, int32_t* counts,
              int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes, void* stream);

/*
 * The whole MoE layer: out = sum_j topk_w[t,j] * W2_e (silu(W1_e x_t) * (W3_e x_t)),
 * e = topk_ids[t,j] (paragraph 2 and timestamp 5:56).
 *   x        device, [T,H] bf16, read only.
 *   logits   device, [T,E] fp32, read only (routed exactly as moe_route does).
 *   w13      device, w1/w3 prepared by moe_prepare_weights (blocked, interleaved).
 *   s13      device, [E,2F] fp32 (FP8) or NULL (BF16), from moe_prepare_weights;
 *            MXFP4: the scale chunks from moe_prepare_weights_mx.
 *   w2       device, w2 prepared by moe_prepare_weights (blocked; MXFP4: by
 *            moe_prepare_weights_mx).
 *   s2       device, [E,H] fp32 (FP8) or NULL (BF16); MXFP4: prepared chunks.
 *   out      device, [T,H] bf16, written.
 *   ws       device workspace, >= moe_workspace_size(T,H,F,E,k,dtype) bytes;
 *            scratch, contents undefined afterwards (moe_workspace_region
 *            gives the offsets of the intermediate buffers it holds; rows of
 *            the padded layout that hold no assignment are left unspecified).
 * Numerics: products accumulate in fp32 on the tensor cores.  FP8 mode:
 * x is quantised per token (sx = absmax/448 in IEEE fp32, e4m3 round to
 * nearest even with saturation); the intermediate h is rounded to bf16 and
 * re-quantised to e4m3 in blocks of 32 d_ff elements with a power-of-two
 * scale 2^ceil(log2(absmax/448)).  MXFP4 mode: the same, with the weights'
 * block scales applied inside the MMAs (128 x 128 one-CTA tiles whatever
 * MOE_OPT_PATH asks).  BF16 mode: h is rounded to bf16.  The k
 * weighted expert outputs are summed in fp32 and rounded once to bf16.
 * Execution: five kernels (six from 1024 tokens on) chained on `stream` with
 * programmatic dependent launch -- routing, the gather of each expert's token
 * rows into the expert-padded layout (with their per-token quantisation), the
 * first group GEMM, the second group GEMM with the scatter-add, and the bf16
 * rounding (MOE_OPT_GATHER can instead let the first GEMM gather the rows
 * itself by TMA after a quantisation pass); to the rest of the stream
 * the call is ordinary stream-ordered work (later work starts after `out` is
 * written).
 * The group GEMM tiles are chosen from the average rows per expert (see
 * MOE_OPT_PATH): small batches stream weights on one-CTA tiles, large ones
 * use 256 x 256 tiles on pairs of SMs.  The call makes no host<->device
 * synchronisation and may be captured in a CUDA graph.
 */
int moe_ffn_forward(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                    const void* s2, int T, int H, int F, int E, int k, int dtype, void* out, void* ws,
                    size_t ws_bytes, void* stream);

/*
 * The layer without a caller-supplied workspace, for callers that cannot
 * allocate device memory: code running while a stream is captured into a CUDA
 * graph (no cudaMalloc allowed then), hosts whose device memory belongs to an
 * allocator they cannot call, runtimes with a fixed memory budget.  The pages
 * have no counterpart of this entry point; it is a property of this library.
 *   Arguments, results and numerics are those of moe_ffn_forward, and the
 *   arguments are checked in the same order (MOE_ERR_INVALID_ARG,
 *   MOE_ERR_UNSUPPORTED, MOE_ERR_ALIGNMENT before MOE_ERR_WORKSPACE); the
 *   workspace is a device array built into the library,
 *   moe_static_workspace_bytes() long (64 MiB).  The driver reserves it on
 *   every GPU that loads the library's device code and keeps it until the
 *   process exits.  This call allocates nothing.
 *   Returns MOE_ERR_WORKSPACE, before enqueuing anything, when the problem
 *   needs more than that (moe_workspace_size(T,H,F,E,k,dtype) bytes); decode
 *   batches of Mixtral-8x7B experts fit (T = 16: about 22 MB FP8, 43 MB BF16).
 *   The first call in each CUDA context looks up the array's device address
 *   (cudaGetSymbolAddress) with that context current; make that first call
 *   before capturing a stream.  A device reset (cudaDeviceReset) ends the
 *   context: the next call is again a first call and looks the address up
 *   in the new context.
 *   All calls on a device share the one array, which keeps the last call's
 *   contents (every call rewrites all it reads; nothing needs to start at
 *   zero).  Calls whose work overlaps on the GPU -- e.g. on two streams at
 *   once -- race on it and give undefined results; serialise them.
 */
int moe_ffn_forward_static(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                           const void* s2, int T, int H, int F, int E, int k, int dtype, void* out, void* stream);
size_t moe_static_workspace_bytes(void);

/*
 * One rank's part of the d_ff-sharded layer (multi-GPU; the talk summary's
 * deployment, timestamp 8:14, runs the layer on 16 shards).  Each of n_ranks
 * GPUs holds an F_shard = d_ff / n_ranks slice of every expert: rows
 * [r*F_shard, (r+1)*F_shard) of w1 and w3 and the same columns of w2,
 * prepared by moe_prepare_weights with F = F_shard (F_shard % 128 == 0, so the
 * FP8 blocks of 32 d_ff channels never straddle two shards and the sharded
 * layer rounds h exactly as the whole layer does).  Every rank routes all T
 * tokens (the routing is deterministic, so all ranks agree), runs both group
 * GEMMs on its slice, and its second GEMM adds each token's partial output
 * straight into the combine rows of the rank that owns the token: rank
 * g = t / rows_per_rank owns tokens [g*rows_per_rank, (g+1)*rows_per_rank),
 * rows_per_rank = ceil(T / n_ranks) -- a GEMM and reduce-scatter in one pass,
 * through peer memory.  Then it adds 1 to every rank's arrival counter.
 *   x, logits, s2, T, H, E, k, dtype, ws, ws_bytes as in moe_ffn_forward (s2 is
 *            the full [E,H]); w13, s13, w2 are this rank's prepared slices.
 *   peer_out32   host array of n_ranks device pointers: rank g's fp32 combine
 *            rows [rows_per_rank, H] for this step (possibly another GPU's
 *            memory, mapped for peer access).  They must be zero before the
 *            first step; moe_dff_finalize zeroes the rows it rounds, so a
 *            caller that alternates two sets of combine rows between steps
 *            (set s % 2 at step s) always adds into zeroed rows.
 *   peer_counter host array of n_ranks device pointers: rank g's uint32
 *            arrival counter (zero before the first step).
 * Returns as moe_ffn_forward; 1 <= n_ranks <= 16, 0 <= rank < n_ranks.
 */
int moe_ffn_forward_dff(const void* x, const float* logits, const void* w13, const void* s13, const void* w2,
                        const void* s2, int T, int H, int F_shard, int E, int k, int dtype, int n_ranks, int rank,
                        float* const* peer_out32, unsigned int* const* peer_counter, void* ws, size_t ws_bytes,
                        void* stream);

/*
 * Closes a step of the d_ff-sharded layer on this rank: waits (bounded, like
 * every wait of this library) until this rank's arrival counter reaches
 * `target` -- n_ranks * step for the step-th call, counting from 1 -- then
 * rounds this rank's `rows` combine rows to bf16 into `out` [rows, H] and
 * zeroes them.  Enqueue it after moe_ffn_forward_dff on this rank's stream;
 * on one GPU standing in for several ranks, enqueue every rank's
 * moe_ffn_forward_dff before any rank's moe_dff_finalize.
 *   out32_rows  device, fp32 [rows, H]: this rank's combine rows of the step.
 *   out         device, bf16 [rows, H], written.
 *   counter     device, this rank's arrival counter.
 * A wait that runs out records MOE_ERR_DEVICE_TIMEOUT and leaves `out`
 * unwritten.
 */
int moe_dff_finalize(float* out32_rows, void* out, int rows, int H, const unsigned int* counter, unsigned int target,
                     void* stream);

/* Waits for `stream`, then returns and clears the device status word:
 * MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BOUNDS, or MOE_ERR_CUDA when
 * the wait itself failed. */
int moe_get_status(void* stream);

/* Regions of the workspace that moe_ffn_forward fills (for inspection and
 * tests).  Returns the byte offset of region `which` inside ws and its size in
 * *bytes, or -1 for a bad argument. */
typedef enum {
    MOE_WS_TOPK_IDS = 0,   /* int32 [T*k] */
    MOE_WS_TOPK_W = 1,     /* fp32 [T*k] */
    MOE_WS_COUNTS = 2,     /* int32 [E] */
    MOE_WS_OFFSETS = 3,    /* int32 [E+1] */
    MOE_WS_PERM = 4,       /* int32 [T*k] */
    MOE_WS_INV_PERM = 5,   /* int32 [T*k] */
    MOE_WS_SLOT_OF = 6,    /* int32 [T*k]: assignment -> row of the expert-padded layout */
    MOE_WS_XS = 7,         /* FP8: quantised activations, one row per token: e4m3 [T,H], written
                              when the first group GEMM gathers each expert's rows itself
                              (MOE_OPT_GATHER 1; BF16 then gathers from x itself); empty for BF16 */
    MOE_WS_SX = 8,         /* FP8: fp32 [T] per-token activation scale (empty for BF16) */
    MOE_WS_H = 9,          /* intermediate h [S,F]: e4m3 or bf16, rows F*eb + 128 bytes apart */
    MOE_WS_H_SF = 10,      /* UE8M0 block scales of h (FP8), tiled for the tensor cores */
    MOE_WS_OUT32 = 11,     /* fp32 [T,H] combine buffer */
    MOE_WS_NUM_MTILES = 12, /* int32: number of 128-row tiles in the padded layout */
    MOE_WS_SLOT_ASSIGN = 13, /* int32 [S]: padded row -> assignment, -1 for a padding row */
    MOE_WS_MTILE_EXPERT = 14, /* int32 [S/128]: 128-row tile -> expert */
    MOE_WS_ROUTE_BLOCKS = 15, /* int32 [ceil(T/256), E]: assignments per expert of each 256-token
                                 block (routing of large batches on many SMs) */
    MOE_WS_XG = 16,           /* gathered activations, one row per padded slot: e4m3 or bf16 [S,H],
                                 rows H*eb + 128 bytes apart (written by the gather pass; padding
                                 rows unspecified) */
    MOE_WS_SX_SLOT = 17       /* FP8: fp32 [S] activation scale of each padded row (gather pass) */
} moe_ws_region;

long long moe_workspace_region(int T, int H, int F, int E, int k, int dtype, int which, size_t* bytes);

/* Kernel selection for tests and tuning (host-side setting, process-wide).
 *   MOE_OPT_PATH:     0 = choose by problem size, 1 = force the throughput
 *                     tiles (256 x 256 tiles on pairs of SMs), 2 = force the
 *                     weight-streaming tiles (128 x 128 on one SM), 3 = force
 *                     128 x 256 tiles on one SM, 4 = force the tiny-batch
 *                     tiles (32 activation rows per stage; only for at most
 *                     32 assignments, else MOE_ERR_UNSUPPORTED).  MX FP4
 *                     weights run on 128 x 128 one-SM tiles only: 4 forces
 *                     their tiny-batch form, 1-3 the other one.  The
 *                     backward's GEMMs take 256 x 256 tiles on pairs of SMs
 *                     where the tile is 256 wide (0, 1) or one-SM tiles
 *                     only (2, 3, 4).
 *   MOE_OPT_SPLITK:   0 = automatic, n > 0 = split the second GEMM's K into n parts
 *                     (must divide F/128).
 *   MOE_OPT_TIMEOUT_MS: limit of every device-side wait (default 2000).
 *   MOE_OPT_TEST_STALL: 1 = test of the failure path: the first group GEMM
 *                     leaves out one operand copy of one CTA, so that CTA's
 *                     bounded waits run out, the call's outputs are undefined
 *                     and moe_get_status reports MOE_ERR_DEVICE_TIMEOUT; the
 *                     context stays usable.  0 (default) = off.
 *   MOE_OPT_TEST_CORRUPT: test of the bounds checks: after routing, the host
 *                     enqueues a 4-byte write of bytes 0x7F (an index far out
 *                     of range) over the first entry of one routing table --
 *                     1 = padded row -> assignment (read by the first GEMM's
 *                     token gather and the second GEMM's scatter),
 *                     2 = 128-row tile -> expert, 3 = the number of 128-row
 *                     tiles (both read by both GEMMs).  The kernel that reads it records
 *                     MOE_ERR_DEVICE_BOUNDS and skips the access; the call's
 *                     outputs are undefined and the context stays usable.
 *                     Also applies to moe_ffn_backward and
 *                     moe_ffn_forward_train (after their routing).
 *                     0 (default) = off.
 *   MOE_OPT_GATHER:   how the first group GEMM gets each expert's token rows:
 *                     0 = automatic (currently 2), 1 = the GEMM gathers them
 *                     itself with TMA tile::gather4 (four rows per copy) from
 *                     the per-token rows (MOE_WS_XS, or x for BF16) after a
 *                     per-token quantisation pass, 2 = a gather pass writes
 *                     them into the expert-padded layout (MOE_WS_XG) and the
 *                     GEMM copies whole tiles.
 * Returns the previous value, or MOE_ERR_INVALID_ARG. */
typedef enum {
    MOE_OPT_PATH = 0,
    MOE_OPT_SPLITK = 1,
    MOE_OPT_TIMEOUT_MS = 2,
    MOE_OPT_TEST_STALL = 3,
    MOE_OPT_TEST_CORRUPT = 4,
    MOE_OPT_GATHER = 5
} moe_option;
int moe_set_option(int option, int value);

/* Per-kernel device timing (tracing aid).  While enabled, moe_ffn_forward,
 * moe_ffn_backward and the weight preparations record a pair of CUDA events
 * around each step they enqueue (routing is one kernel for small batches and two from 1024 tokens
 * on; both are counted in `launches` and timed together; the backward's
 * routing, slot gather, rounding of dx and router gradient are timed
 * together as MOE_KERNEL_BWD_AUX).
 * moe_profile_enable returns the previous setting.  moe_profile_read waits for
 * the recorded events, adds up the elapsed time per kernel into
 * ms_total[MOE_KERNEL_COUNT] and the number of launches into
 * launches[MOE_KERNEL_COUNT] (both host arrays, either may be NULL), and
 * forgets the records when `reset` is nonzero.  Returns MOE_OK or MOE_ERR_CUDA. */
typedef enum {
    MOE_KERNEL_ROUTE = 0,
    MOE_KERNEL_QUANT = 1,  /* per-token FP8 quantisation + zeroing of the combine buffer */
    MOE_KERNEL_STAGE1 = 2, /* group GEMM with w1/w3 + SwiGLU */
    MOE_KERNEL_STAGE2 = 3, /* group GEMM with w2 + weighted scatter-add */
    MOE_KERNEL_FINALIZE = 4,
    MOE_KERNEL_BWD_GU = 5,   /* backward: g, u, h recomputed (group GEMM with w1/w3); the training forward
                              * counts its two GEMMs as STAGE1 and STAGE2 */
    MOE_KERNEL_BWD_DH = 6,   /* backward: dh = W2^T dy -> dg, du, routing-weight gradients */
    MOE_KERNEL_BWD_DX = 7,   /* backward: dx = W1^T dg + W3^T du, scatter-add per token */
    MOE_KERNEL_BWD_DW2 = 8,  /* backward: dW2 per expert */
    MOE_KERNEL_BWD_DW13 = 9, /* backward: dW1, dW3 per expert */
    MOE_KERNEL_BWD_AUX = 10, /* backward: routing, slot gather, dx rounding, router gradient */
    MOE_KERNEL_PREPARE = 11, /* moe_prepare_weights and _mx (weight layouts) */
    MOE_KERNEL_COUNT = 12
} moe_kernel_id;
int moe_profile_enable(int on);
int moe_profile_read(double* ms_total, int* launches, int reset);

/*
 * Backward pass (custom VJP) of the BF16 layer, for training.  The pages name
 * a custom VJP as the next step of the routed kernel without defining it
 * (rocketrecap.com "FlyDSL kernels in JAX", timestamp 10:07); this is the
 * gradient of the BF16 layer of moe_ffn_forward (h rounded to bf16 there;
 * the rounding passes gradients through unchanged) for an upstream gradient
 * dy = dL/dout.  For each assignment a = (t, j) of token t to expert e with
 * routing weight w_a, g = W1_e x_t, u = W3_e x_t, h = silu(g) u:
 *   dw_a = <dy_t, W2_e h>,  dh = w_a W2_e^T dy_t,  du = dh silu(g),
 *   dg = dh u s(g) (1 + g (1 - s(g)))  (s the logistic function),
 *   dx_t = sum_j (W1_e^T dg + W3_e^T du),
 *   dW1_e = sum dg x_t^T,  dW3_e = sum du x_t^T,  dW2_e = sum w_a dy_t h^T,
 *   dlogits[t, e_j] = w_j (dw_j - sum_i w_i dw_i) for the chosen experts, 0
 *   for the others (the routing weights are the softmax over the chosen
 *   logits; the choice is piecewise constant).
 * g and u are recomputed from x and w1/w3 (the forward keeps no
 * intermediates).  Every grouped GEMM reads its operands as they lie -- the
 * weights in the caller's row-major layout, the activations in the
 * expert-padded slot layout -- K-major or MN-major, so nothing is
 * transposed and the weights need no preparation.  Arithmetic: bf16
 * operands, fp32 accumulation; g and u are kept in fp32, h (as in the
 * forward), dg, du and the w_a dy_t entering dW2 are rounded to bf16 where
 * they are stored between kernels; dx is summed over the k experts in fp32
 * and rounded once.
 *
 * moe_backward_workspace_size: bytes of `ws` for moe_ffn_backward (0 if the
 *   dimensions are unsupported: bf16 only, d_model and d_ff multiples of 128,
 *   1 <= E <= 64, 1 <= k <= min(E, 8)).
 * moe_ffn_backward: x [T, H], dy [T, H] bf16, logits [T, E] fp32 (finite),
 *   w1, w3 [E, F, H] and w2 [E, H, F] bf16, row-major (as moe_prepare_weights
 *   takes them); outputs dx [T, H] bf16, dw1, dw3 [E, F, H] and dw2 [E, H, F]
 *   bf16 (fully written: zero for an expert with no tokens), dlogits [T, E]
 *   fp32.  Device pointers, 16-byte aligned (logits and dlogits 4-byte); ws
 *   >= moe_backward_workspace_size bytes.  Enqueued on `stream` (no host
 *   synchronisation; may be captured in a CUDA graph).  Returns MOE_OK,
 *   MOE_ERR_INVALID_ARG, MOE_ERR_ALIGNMENT, MOE_ERR_WORKSPACE or MOE_ERR_CUDA
 *   (a launch failed; device-side faults surface through moe_get_status as
 *   for the forward).
 */
size_t moe_backward_workspace_size(int T, int H, int F, int E, int k);
/*
 * Training pair.  moe_ffn_forward_train: the BF16 layer of moe_ffn_forward
 *   (same output, same arithmetic: h rounded to bf16, fp32 combine rounded
 *   once) computed from the caller's row-major w1, w3, w2 -- no
 *   moe_prepare_weights, which a training step would have to redo after every
 *   weight update -- and keeping in `ws` (moe_backward_workspace_size bytes)
 *   the routing, the gathered x and g, u, h of this call.
 * moe_ffn_backward_saved: the backward of the last moe_ffn_forward_train on
 *   the same `ws`, from what it kept (no routing, no recompute of g and u; x
 *   and logits are not needed again).  Same outputs and contract as
 *   moe_ffn_backward; T, H, F, E, k and the weights must be the forward's.
 */
int moe_ffn_forward_train(const void* x, const float* logits, const void* w1, const void* w3, const void* w2, int T,
                          int H, int F, int E, int k, void* out, void* ws, size_t ws_bytes, void* stream);
int moe_ffn_backward_saved(const void* w1, const void* w3, const void* w2, const void* dy, int T, int H, int F, int E,
                           int k, void* dx, void* dw1, void* dw3, void* dw2, float* dlogits, void* ws, size_t ws_bytes,
                           void* stream);
int moe_ffn_backward(const void* x, const float* logits, const void* w1, const void* w3, const void* w2,
                     const void* dy, int T, int H, int F, int E, int k, void* dx, void* dw1, void* dw3, void* dw2,
                     float* dlogits, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
