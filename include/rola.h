/*
 * rola.h — C ABI of the RoLA attention forward library for NVIDIA B200 (sm_100a).
 *
 * RoLA ("Rotary-Positioned Low-Rank Linear Attention", the sparse attention module of
 * SparkDiffusion) has two branches:
 *   - a block-sparse softmax branch that keeps, for every 64-token query block, the
 *     top-k fraction of key blocks by block energy;
 *   - a rank-r linear-attention branch with rotary (3D) positions over all keys, which
 *     restores the global context the sparse branch drops.
 * Sources: web page "SparkDiffusion: 265x Faster Video Generation on Consumer GPUs via
 * Sparse Attention & Distillation", section "RoLA: Preserving Global Context at Extreme
 * Sparsity"; news article on SparkDiffusion / SparkWan, section "What's New"; the
 * "AlibabaResearch/SparkDiffusion" README (inference section: topk is a keep ratio;
 * sparse-finetuning section: proj_q, proj_k, gate_proj, gate_bias; citation block:
 * RoLA and "RoPeSLR: 3D RoPE-driven Sparse-LowRank Attention").
 *
 * The pages fix only that structure.  The operator computed here, for every batch b
 * and head h (nb = ceil(N/64) blocks, the last one possibly short):
 *   1. qbar_i, kbar_j: fp32 means over the valid tokens of each 64-token block
 *      (token-order fp32 sums, one IEEE division by the count).
 *   2. s_ij = qbar_i . kbar_j as an fp32 fused multiply-add chain over channels 0..d-1.
 *      k = clamp(ceil(topk*nb - 1e-9), 1, nb) blocks with the largest s_ij are kept per
 *      query block; equal scores keep the lower key-block index.  Lists are ascending.
 *   3. O_sparse = softmax((q.k) * scale) v over the valid keys of the kept blocks.
 *   4. u = phi(q Wq_h), f = phi(k Wk_h), phi(x) = elu(x) + 1.  R(p) turns rotary pair
 *      (2c, 2c+1) by theta_c = pos_axis(c) * base^(-c'/P_axis) (pairs ordered t, h, w).
 *      S_h = sum_m R(p_m) f_m v_m^T (r x d), z_h = sum_m f_m over all N keys;
 *      O_lin = (R(p_n) u_n)^T S_h / (u_n^T z_h).
 *   5. out = O_sparse + g * O_lin, rounded once to the output type; g per head, per token
 *      and head, or sigmoid(q . wg_h + bg_h) from the query (rola_gate).
 *
 * Layouts (all row-major, contiguous, device memory owned by the caller):
 *   q, k, v, out : [B, N, H, d]  (fp32 for ROLA_F32, bf16 for ROLA_BF16 and ROLA_FP8_E4M3)
 *   Wq, Wk       : [H, d, r]     (same element type as q)
 *   g            : fp32, [H], [B, N, H] or [H*(d+1)] (rola_gate)
 *   workspace    : rola_workspace_size() bytes, 256-byte aligned, borrowed by the plan.
 * Every pointer must be 16-byte aligned; out must not overlap any input.
 *
 * Errors: every call returns a rola_status; nothing is thrown across the ABI.  Invalid
 * arguments are rejected on the host before any launch.  Calls are asynchronous on the
 * given stream and never synchronise, except rola_poll_device_status.  Device-side
 * waits are bounded: a wait that runs out records ROLA_ERR_DEVICE_TIMEOUT in a status
 * word in the workspace, and the kernel returns; rola_poll_device_status reports it.
 * The library never allocates device memory.
 */
#ifndef ROLA_H_
#define ROLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ROLA_API __attribute__((visibility("default")))
#else
#define ROLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; 0 means the legacy default stream. */
typedef struct CUstream_st* rola_stream_t;

typedef enum {
  ROLA_OK = 0,
  ROLA_ERR_INVALID_ARG = 1,     /* bad pointer, size, alignment or parameter            */
  ROLA_ERR_UNSUPPORTED = 2,     /* valid in principle, not built (e.g. d not 64/128)   */
  ROLA_ERR_WORKSPACE = 3,       /* workspace missing, misaligned or too small          */
  ROLA_ERR_CUDA = 4,            /* a CUDA runtime call or launch failed                */
  ROLA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait ran out (see poll)       */
  ROLA_ERR_DEVICE_BOUNDS = 6,   /* a device-side index check failed (see poll)         */
  ROLA_ERR_RANGE = 7            /* v holds a non-finite value (ROLA_BF16; reported by  */
                                /* poll: the kernels that copy v check every element)  */
} rola_status;

typedef enum {
  ROLA_F32 = 0,       /* fp32 in/out, fp32 arithmetic (correctness configuration)       */
  ROLA_BF16 = 1,      /* bf16 in/out, bf16 tensor-core products, fp32 accumulation      */
  ROLA_FP8_E4M3 = 2   /* bf16 in/out; q, k, v quantised inside to e4m3 with one absmax */
                      /* scale per (b, h, 64-token block) (scale = absmax/448, 1 when   */
                      /* absmax = 0; round to nearest even, saturating); fp8 tensor-core */
                      /* products, fp32 softmax; P is e4m3 too.  Block lists come from  */
                      /* the bf16 inputs, so they equal the ROLA_BF16 lists.  d = 128    */
                      /* only (ROLA_ERR_UNSUPPORTED otherwise).                          */
} rola_dtype;

/* The gain g that scales the linear branch (out = O_sparse + g * O_lin).  The pages name
 * gate_proj and gate_bias among RoLA's parameters (README, sparse-finetuning section)
 * without their form; ROLA_GATE_QPROJ takes the plainest reading that fits this
 * operator: a projection of each head's query to one logit, g = sigmoid(q . wg_h + bg_h). */
typedef enum {
  ROLA_GATE_HEAD = 0,   /* g: [H] fp32, one gain per head                                 */
  ROLA_GATE_TOKEN = 1,  /* g: [B, N, H] fp32, one gain per token and head, given           */
  ROLA_GATE_QPROJ = 2   /* g: fp32 gate_proj wg [H, d] followed by gate_bias bg [H]        */
                        /* (H*(d+1) values); the gain of token n, head h is computed as     */
                        /* sigmoid(sum_c q[b,n,h,c] * wg[h,c] + bg[h]) in fp32              */
} rola_gate;

typedef struct {
  int B, H, N, d, r;             /* batch, heads, tokens, head dim (64|128), rank (16|32)   */
  int block;                     /* tokens per block; must be 64                            */
  double topk;                   /* keep ratio in (0, 1]                                    */
  int grid_t, grid_h, grid_w;    /* latent grid, product == N; (1, 1, N) for 1D positions   */
  int rope_pairs_t, rope_pairs_h, rope_pairs_w; /* rotary pairs per axis, sum == r/2;      */
                                 /* all 0 = default: 1D grid -> all on w; else h = w =      */
                                 /* floor(r/6), t = r/2 - 2*floor(r/6)                      */
  double rope_base;              /* rotary frequency base, > 1 (10000)                      */
  float softmax_scale;           /* logit scale; 0 = 1/sqrt(d)                              */
  rola_dtype dtype;
  rola_gate gate;                /* how the gain g is given (default ROLA_GATE_HEAD)        */
} rola_params;

typedef struct rola_plan_s* rola_plan_t;

/* Fills *p with defaults: B=H=1, N=0, d=128, r=32, block 64, topk 0.1, grid (1,1,0),
 * default rotary split, base 10000, scale 0 (1/sqrt(d)), ROLA_BF16, ROLA_GATE_HEAD. */
ROLA_API rola_status rola_params_default(rola_params* p);

/* Number of 64-token blocks nb and kept blocks per query block k for *p. */
ROLA_API rola_status rola_keep_count(const rola_params* p, int* nb, int* k);

/* Bytes of device workspace a plan for *p needs (pooled means, block scores and key-block
 * norms, block lists, linear state, rotary table, the fp16 or fp8 copies, status word). */
ROLA_API rola_status rola_workspace_size(const rola_params* p, size_t* bytes);

/* Validates *p and binds it to `workspace` (device memory of at least
 * rola_workspace_size bytes, 256-byte aligned).  Host-only: no launch, no allocation
 * on the device.  The plan borrows the workspace until rola_plan_destroy. */
ROLA_API rola_status rola_plan(const rola_params* p, void* workspace, size_t workspace_bytes,
                      rola_plan_t* plan);

ROLA_API void rola_plan_destroy(rola_plan_t plan);

/* Steps 1-2 (block pooling, block scores, top-k): writes the block lists into the
 * workspace.  In ROLA_FP8_E4M3 mode also writes the e4m3 copies of q and k with their
 * per-block scales.  Reads q, k [B, N, H, d]. */
ROLA_API rola_status rola_select_blocks(rola_plan_t plan, const void* q, const void* k,
                               rola_stream_t stream);

/* Step 4, key side: S_h, z_h over all N keys into the workspace (fixed-order, run-to-run
 * deterministic reduction).  In ROLA_FP8_E4M3 mode also writes the e4m3 copy of v. */
ROLA_API rola_status rola_linear_state(rola_plan_t plan, const void* k, const void* v, const void* Wk,
                              rola_stream_t stream);

/* Steps 3-5: sparse attention over the kept blocks with the linear branch and the
 * combination fused into its epilogue; writes out [B, N, H, d] once.  g: fp32 gains [H],
 * [B, N, H], or the gate's wg [H, d] and bg [H], as p->gate says (device memory, 16-byte
 * aligned).  Uses the block
 * lists and the state the two calls above left in the workspace (in ROLA_FP8_E4M3 mode
 * also their e4m3 copies of q, k, v, which must come from the same q, k, v). */
ROLA_API rola_status rola_attend(rola_plan_t plan, const void* q, const void* k, const void* v,
                        const void* Wq, const float* g, void* out, rola_stream_t stream);

/* The whole forward pass: rola_select_blocks, rola_linear_state, rola_attend. */
ROLA_API rola_status rola_forward(rola_plan_t plan, const void* q, const void* k, const void* v,
                         const void* Wq, const void* Wk, const float* g, void* out,
                         rola_stream_t stream);

/* Steps 1-2 without any device allocation and without a plan or workspace (no
 * counterpart on the pages: this is a deployment variant of rola_select_blocks).
 * It is meant for callers that cannot allocate device memory at the point of the call
 * and have no workspace to lend -- code running inside a host framework whose pool owns
 * all device memory, or latency-critical paths where cudaMalloc's implicit device
 * synchronisation is not acceptable.  Writes the block lists [B, H, nb, k] int32 to the
 * caller's `col_idx` (q, k and col_idx as for rola_select_blocks; all 16-byte aligned).
 * Scratch: one 16 MiB array inside the library, which every GPU that loads the library
 * holds until the process exits; problems whose pooled means and block scores need more
 * (about 256 + 8*B*H*nb*d + 4*B*H*nb*ceil4(nb) bytes) are rejected with
 * ROLA_ERR_WORKSPACE before any launch.  col_idx must hold B*H*nb*k int32 and must not
 * overlap q or k (ROLA_ERR_INVALID_ARG otherwise).  Every call made outside stream capture
 * looks up the array's device address (cudaGetSymbolAddress) with the current device, so
 * calls after a device reset see the reloaded array; a call made while `stream` is being
 * captured reuses the address of the last uncaptured call on that device, so make at
 * least one call before any capture (a first call under capture fails with ROLA_ERR_CUDA).
 * All calls share the array: calls that overlap on the GPU (other streams, other host
 * threads) race and must be serialised by the caller.  Device-side index checks of this
 * variant are not reported. */
ROLA_API rola_status rola_select_blocks_noalloc(const rola_params* p, const void* q, const void* k,
                                                int32_t* col_idx, rola_stream_t stream);

/* Inspection (tests): copy, on `stream`, the block lists [B, H, nb, k] int32 (CSR column
 * indices; row i of (b, h) starts at ((b*H + h)*nb + i)*k), the pooled means [B, H, nb, d]
 * fp32, or the linear state S [B, H, r, d] and z [B, H, r] fp32 into caller buffers. */
ROLA_API rola_status rola_get_block_lists(rola_plan_t plan, int32_t* col_idx, rola_stream_t stream);
ROLA_API rola_status rola_get_pooled(rola_plan_t plan, float* qbar, float* kbar, rola_stream_t stream);
ROLA_API rola_status rola_get_linear_state(rola_plan_t plan, float* S, float* z, rola_stream_t stream);

/* Inspection (tests): copy, on `stream`, the tensor-core block scores of the last selection
 * [B, H, nb, nb] fp32 (row i of (b, h) at ((b*H + h)*nb + i)*nb; s~_ij = qbar_i . kbar_j from
 * tf32 operands: they only prune, the kept lists are decided on exact fp32 scores) and the
 * key-block norms ||kbar_j||_2 [B, H, nb] fp32 into caller device buffers. */
ROLA_API rola_status rola_get_block_scores(rola_plan_t plan, float* scores, float* knorm, rola_stream_t stream);

/* Inspection (tests), ROLA_FP8_E4M3 plans only (ROLA_ERR_INVALID_ARG otherwise): copy the
 * e4m3 copies q8, k8, v8 [B, N, H, d] (one byte per element, OCP E4M3 encoding) and their
 * scales sq, sk, sv [B, H, nb] fp32 (value = decoded byte * scale of its (b, h, block))
 * into caller device buffers on `stream`.  q8/k8/sq/sk are written by
 * rola_select_blocks, v8/sv by rola_linear_state. */
ROLA_API rola_status rola_get_fp8_copies(rola_plan_t plan, uint8_t* q8, uint8_t* k8, uint8_t* v8,
                                         float* sq, float* sk, float* sv, rola_stream_t stream);

/* Inspection (tests): the number of query-block tiles whose output the last attention
 * call recomputed in its careful pass (head dim 128, bf16 / fp8; 0 otherwise).  The fast
 * pass fixes each tile's softmax offsets from its first pair of key blocks; a tile where a
 * later score rises too far above them (P would leave fp16, or e4m3, range) is listed and
 * recomputed with per-pair offset updates.  Synchronises `stream`; writes a host int. */
ROLA_API rola_status rola_get_attend_redo_count(rola_plan_t plan, int* count, rola_stream_t stream);

/* Synchronises `stream`, reads and clears the device status word: ROLA_OK, or
 * ROLA_ERR_DEVICE_TIMEOUT / ROLA_ERR_DEVICE_BOUNDS if a kernel recorded one. */
ROLA_API rola_status rola_poll_device_status(rola_plan_t plan, rola_stream_t stream);

/* Debug hooks for tests of the failure path.  ROLA_DEBUG_STALL_WAIT makes the next
 * rola_attend wait on a barrier that nothing arrives on, with a wait limit of
 * `limit_us` microseconds; the kernel then records ROLA_ERR_DEVICE_TIMEOUT and returns.
 * 0 clears all hooks. */
#define ROLA_DEBUG_STALL_WAIT 1
ROLA_API rola_status rola_set_debug(rola_plan_t plan, int flags, int limit_us);

/* Stage timing (no counterpart on the pages; a measurement aid).  With `enable` != 0 every
 * later rola_forward on the plan records CUDA events on its stream between its stages
 * (at most ROLA_PROFILE_CALLS calls are kept; later calls run unrecorded).  It does not
 * change the work done.  Stages, for head dim 128 with bf16 or fp8 inputs:
 *   0: key/value pass and state reduction (state, k means, v copy / e4m3 k and v)
 *   1: query pass (q means, query features, e4m3 q)
 *   2: block scores and top-k selection
 *   3: attention (sparse branch with the fused linear epilogue)
 * and for the other configurations: 0 selection, 1 linear state, 2 attention.
 * Enabling creates the events (host call, synchronous); 0 destroys them.
 * rola_get_stage_times synchronises on the last recorded event, writes into ms[s] the
 * sum over the recorded calls of stage s's elapsed milliseconds (for s < max_stages),
 * and reports the stage and call counts; it then clears the record. */
#define ROLA_PROFILE_CALLS 64
ROLA_API rola_status rola_profile_stages(rola_plan_t plan, int enable);
ROLA_API rola_status rola_get_stage_times(rola_plan_t plan, float* ms, int max_stages, int* nstages,
                                          int* ncalls);

/* Backward of rola_forward (gradients for training; the pages' sparse-finetuning section
 * trains proj_q, proj_k, gate_proj and gate_bias with the attention).  Computes the
 * gradients of L = sum(dout * out) with the kept-block lists held fixed (the selection is
 * a discrete choice, so its gradient is zero almost everywhere):
 *   dq, dk, dv  [B, N, H, d] fp32      dWq, dWk  [H, d, r] fp32
 *   dg          the layout of g: [H] (ROLA_GATE_HEAD), [B, N, H] (ROLA_GATE_TOKEN), or
 *               d gate_proj [H, d] then d gate_bias [H] (ROLA_GATE_QPROJ), fp32.
 * q, k, v, Wq, Wk, g are the forward's inputs and dout [B, N, H, d] has the input dtype.
 * The call recomputes what it needs (block selection, the linear state, the softmax row
 * statistics) on the plan's workspace, so it needs no saved forward state; it overwrites
 * the plan's workspace as rola_forward does.  Configurations: ROLA_F32 and ROLA_BF16 (fp8
 * is a forward-only configuration: ROLA_ERR_UNSUPPORTED), every d, r and gate of the
 * forward.  Arithmetic: fp32 on the inputs' values.  Scratch: bwd_workspace, at least
 * rola_backward_workspace_size bytes, 16-byte aligned, caller-owned.  Every pointer is a
 * device pointer, 16-byte aligned; the gradients must not overlap each other or the
 * inputs (ROLA_ERR_INVALID_ARG).  Asynchronous on `stream`; deterministic (partial sums
 * are reduced in a fixed order). */
ROLA_API rola_status rola_backward_workspace_size(const rola_params* p, size_t* bytes);
ROLA_API rola_status rola_backward(rola_plan_t plan, const void* q, const void* k, const void* v,
                                   const void* Wq, const void* Wk, const float* g, const void* dout,
                                   float* dq, float* dk, float* dv, float* dWq, float* dWk, float* dg,
                                   void* bwd_workspace, size_t bwd_workspace_bytes,
                                   rola_stream_t stream);

/* Self-test of the softmax exponentials of the head-dim-128 attention kernels (a
 * measurement aid; the pages fix only P = exp(s - m)): y[i] = 2^x[i] for the n device
 * floats at x, computed by the same device functions the kernels call.  mode 0: the
 * special-function unit's ex2.approx (relative error about 2^-22; 2^-inf = 0).  mode 1: the
 * polynomial on the FMA pipe that the e4m3 path uses for a quarter of its exponentials
 * (x = n + f, n = round(x), a cubic in f, n added into the exponent field; relative error
 * below 7.8e-5 for -125 <= x <= 0; x below -125, -inf and NaN give 2^-125).  x and y are
 * device pointers of n floats (equal or disjoint); n >= 0.  Asynchronous on `stream`.
 * Returns ROLA_ERR_INVALID_ARG for a null pointer with n > 0, a negative n or another mode,
 * ROLA_ERR_CUDA if the launch fails. */
ROLA_API rola_status rola_eval_exp2(const float* x, float* y, int64_t n, int mode, rola_stream_t stream);

ROLA_API const char* rola_status_string(rola_status s);

#ifdef __cplusplus
}
#endif

#endif /* ROLA_H_ */
