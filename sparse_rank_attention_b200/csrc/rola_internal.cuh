// Internal declarations of the RoLA forward library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "rola.h"

namespace rola {

constexpr int kBlock = 64;         // tokens per block
constexpr int kStateChunk = 2048;  // tokens per linear-state partial sum (fp32 and d = 64 paths)

// Device status word values (mirror rola_status codes).
constexpr int kDevOk = 0;
constexpr int kDevTimeout = ROLA_ERR_DEVICE_TIMEOUT;
constexpr int kDevBounds = ROLA_ERR_DEVICE_BOUNDS;
constexpr int kDevRange = ROLA_ERR_RANGE;

// Everything a kernel needs to know about the problem, passed by value.
struct Dims {
  int B, H, N, d, r;
  int nb, k;                  // blocks, kept blocks per query block
  int gt, gh, gw;             // latent grid
  int pt, ph, pw;             // rotary pairs per axis
  int rope_off_h, rope_off_w; // table offsets of the h and w axes (t starts at 0)
  int chunk_tok;              // tokens per linear-state partial sum (a multiple of 64)
  int nchunk;                 // linear-state partial sums per (b, h)
  float scale;                // softmax logit scale
  double rope_base;
  int gate_mode;              // rola_gate: gain per head g[H], per token g[B, N, H], or
                              // computed from the query (g = gate_proj [H, d], gate_bias [H])
};

// The gain of token n of (b, h) for the gates that are read: g[H] (ROLA_GATE_HEAD) or
// g[B, N, H] (ROLA_GATE_TOKEN).
__host__ __device__ inline size_t gain_index(const Dims& dm, int b, int n, int h) {
  return dm.gate_mode == ROLA_GATE_TOKEN ? ((size_t)b * dm.N + n) * dm.H + h : (size_t)h;
}

// Partial dot product of channels [c0, c1) of a query row with the gate projection of
// head h (ROLA_GATE_QPROJ; g holds gate_proj [H, d] and then gate_bias [H]).
template <typename T>
__device__ __forceinline__ float gate_dot(const Dims& dm, const float* __restrict__ g, const T* q_row, int h,
                                          int c0, int c1) {
  const float* wg = g + (size_t)h * dm.d;
  float a = 0.f;
  for (int c = c0; c < c1; ++c) a = fmaf(static_cast<float>(q_row[c]), __ldg(wg + c), a);
  return a;
}

// sigmoid(dot + gate_bias_h): the gain of ROLA_GATE_QPROJ from the finished dot product.
__device__ __forceinline__ float gate_sigmoid(const Dims& dm, const float* __restrict__ g, int h, float dot) {
  const float a = dot + __ldg(g + (size_t)dm.H * dm.d + h);
  return 1.f / (1.f + __expf(-a));
}

// The gain of token n of (b, h) for any gate: read, or computed from the whole query row
// q_row (d channels) for ROLA_GATE_QPROJ.
template <typename T>
__device__ __forceinline__ float gate_value(const Dims& dm, const float* __restrict__ g, const T* q_row, int b,
                                            int n, int h) {
  if (dm.gate_mode == ROLA_GATE_QPROJ) return gate_sigmoid(dm, g, h, gate_dot(dm, g, q_row, h, 0, dm.d));
  return g[gain_index(dm, b, n, h)];
}

// Device pointers carved out of the caller's workspace.
struct Workspace {
  int* status;        // [64] ints; status[0] = first recorded device error
  float2* rope;       // (cos, sin) per (axis position, pair)
  float* qbar;        // [B, H, nb, d]
  float* kbar;        // [B, H, nb, d]
  int32_t* col_idx;   // [B, H, nb, k]
  float* scores;      // [B, H, nb, nbp] tensor-core block scores (nbp = nb rounded up to 4)
  float* knorm;       // [B, H, nbp] ||kbar_j||_2 (bounds the tensor-core scores' error)
  float* S_part;      // [B, H, nchunk, r, d]
  float* z_part;      // [B, H, nchunk, r]
  float* S;           // [B, H, r, d]
  float* z;           // [B, H, r]
  __nv_bfloat16* S_hi;  // [B, H, r, d] bf16(S)            } S = S_hi + S_lo to ~2^-17:
  __nv_bfloat16* S_lo;  // [B, H, r, d] bf16(S - S_hi)     } tensor-core operands of the epilogue
  __half* v16;          // [B, N, H, d] fp16 copy of v, each (b, h, block) as v * 2^-vexp
  int* vexp;            // [B, H, nb] the fp16 copy's power-of-two exponent per block
  uint8_t* simg;        // [B, H] S_h^T hi|lo as 128-byte-swizzled MN-major operand images
  uint8_t* uimg;        // [B, H, nb] (R u)^T hi|lo images ([r rows][64 tokens], swizzled)
  float* gden;          // [B, H, nb, 64] g_h / (u . z_h) per query token
  uint8_t* q8;        // [B, N, H, d] e4m3 (fp8 mode)
  uint8_t* k8;
  uint8_t* v8;
  int* redo;          // [1 + 2*B*H*nb]: count, then the tiles the attention's careful pass redoes
  float* sq;          // [B, H, nb] e4m3 scales (fp8 mode)
  float* sk;
  float* sv;
};

// Scratch of the backward (rola_backward), carved from the caller's second workspace.
struct BwdWorkspace {
  float* lse;       // [B, H, nb, 64] log-sum-exp of each query row's scaled logits (+inf past N)
  float* Drow;      // [B, H, nb, 64] dout . O_sparse per query row
  int* inv_off;     // [B, H, nb + 1] start of each key block's list of query blocks
  int* inv_idx;     // [B, H, nb * k] the query blocks that kept each key block, ascending
  float* dS_part;   // [B, H, nchunk, r, d] partial gradients of the state
  float* dz_part;   // [B, H, nchunk, r]
  float* dWq_part;  // [B, H, nchunk, d, r]
  float* dWk_part;  // [B, H, nchunk, d, r]
  float* dg_part;   // [B, H, nchunk, d + 1] gain: per head (entry 0), or gate_proj then gate_bias
  float* dS;        // [B, H, r, d]
  float* dz;        // [B, H, r]
  int* redo;        // [1 + B*H*nb]: count, then the query tiles whose row statistics are redone
};

size_t backward_workspace_bytes(const Dims& dm, BwdWorkspace* bw, char* base);
// Row statistics (lse, D) of every query tile on tcgen05; tiles it cannot take (a p above
// 2^64 against the first pair's column max) are listed in bw.redo (count zeroed here).
cudaError_t launch_bwd_rowstats_sm100(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                                     const Workspace& ws, const BwdWorkspace& bw, cudaStream_t st);
cudaError_t launch_bwd_dq_sm100(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                                const Workspace& ws, const BwdWorkspace& bw, float* dq, cudaStream_t st);
cudaError_t launch_bwd_dkv_sm100(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                                 const Workspace& ws, const BwdWorkspace& bw, float* dk, float* dv, cudaStream_t st);
cudaError_t launch_backward(const Dims& dm, rola_dtype dt, const void* q, const void* k, const void* v,
                            const void* Wq, const void* Wk, const float* g, const void* dout, float* dq, float* dk,
                            float* dv, float* dWq, float* dWk, float* dg, const Workspace& ws,
                            const BwdWorkspace& bw, cudaStream_t st);

}  // namespace rola

struct rola_plan_s {
  rola_params p;
  rola::Dims dm;
  rola::Workspace ws;
  void* ws_base;
  size_t ws_bytes;
  int debug_flags;
  int debug_limit_us;
  bool status_ready;  // status word zeroed on the device
  bool rope_ready;    // rotary table written
  // stage timing (rola_profile_stages): ROLA_PROFILE_CALLS x (stages + 1) events
  cudaEvent_t* prof_events;
  int prof_calls;     // forwards recorded since the last read
  int prof_stages;    // stages of the recorded configuration
};

namespace rola {

// ---- launchers (each returns cudaGetLastError() of its launch) ----
cudaError_t launch_pool(const Dims& dm, rola_dtype dt, const void* q, const void* k,
                        const Workspace& ws, cudaStream_t st);
cudaError_t launch_select(const Dims& dm, const Workspace& ws, cudaStream_t st);
cudaError_t launch_rope_table(const Dims& dm, const Workspace& ws, cudaStream_t st);
cudaError_t launch_linear_state(const Dims& dm, rola_dtype dt, const void* k, const void* v,
                                const void* Wk, const Workspace& ws, cudaStream_t st);
cudaError_t launch_attend_f32(const Dims& dm, const void* q, const void* k, const void* v,
                              const void* Wq, const float* g, void* out, const Workspace& ws,
                              cudaStream_t st);
cudaError_t launch_attend_bf16_warpmma(const Dims& dm, const void* q, const void* k,
                                       const void* v, const void* Wq, const float* g, void* out,
                                       const Workspace& ws, cudaStream_t st);
cudaError_t launch_attend_sm100(const Dims& dm, const void* q, const void* k, const Workspace& ws,
                                void* out, bool fp8, int debug_flags, int debug_limit_us, cudaStream_t st);
cudaError_t launch_eval_exp2(const float* x, float* y, int64_t n, int mode, cudaStream_t st);
cudaError_t launch_query_features(const Dims& dm, bool fp8, const void* q, const void* Wq, const float* g,
                                  const Workspace& ws, cudaStream_t st);
cudaError_t launch_kv_pass(const Dims& dm, bool fp8, const void* k, const void* v, const void* Wk,
                           const Workspace& ws, cudaStream_t st);
cudaError_t launch_state_reduce(const Dims& dm, const Workspace& ws, cudaStream_t st);
// TMA descriptor of a [B, N, H*d] activation tensor: boxes of box_rows tokens x 128
// bytes (64 channels of a 16-bit type, 128 of an 8-bit one).  False if encoding fails.
bool make_act_map(CUtensorMap* m, CUtensorMapDataType dt, uint32_t el_bytes, const void* ptr, const Dims& dm,
                  CUtensorMapSwizzle sw, uint32_t box_rows = 64);
bool make_map_3d(CUtensorMap* m, CUtensorMapDataType dt, uint32_t el_bytes, const void* ptr, uint64_t d0,
                 uint64_t d1, uint64_t d2, uint32_t box0, uint32_t box1, CUtensorMapSwizzle sw);
// Tensor-core block scores s~ = qbar kbar^T (tf32) into ws.scores and the key-block norms
// into ws.knorm: the input of the exact top-k (launch_select runs both).
cudaError_t launch_score_sm100(const Dims& dm, const Workspace& ws, int nbp, cudaStream_t st);
int score_row_stride(const Dims& dm);
size_t select_noalloc_bytes(const Dims& dm);
size_t select_noalloc_capacity();
cudaError_t select_blocks_noalloc(const Dims& dm, rola_dtype dt, const void* q, const void* k,
                                  int32_t* col_idx, cudaStream_t st);

// ---- device helpers ----
__device__ __forceinline__ void record_status(int* status, int code) {
  atomicCAS(status, kDevOk, code);
}

// Exponent e of the fp16 copy of a 64-token block of v (v is carried as v * 2^-e) from
// the block's largest |v|: 0 while that lies in [2^-6, 2^15) (every element then keeps
// fp16's precision down to 2^-8 of the largest), else the exponent that brings it into
// [2^14, 2^15).  Blocks of zeros, or with a non-finite value, take 0.
__device__ __forceinline__ int v16_exponent(float absmax) {
  if (!(absmax > 0.f) || !(absmax <= 3.402823466e38f) || (absmax >= 0x1p-6f && absmax < 32768.f)) return 0;
  int e2;
  frexpf(absmax, &e2);                 // absmax = m * 2^e2, m in [0.5, 1)
  return (e2 - 1) - 14;
}

// Largest |x| over the bf16 pairs of v, per 16-bit half: with the sign bit cleared, bf16
// patterns order as unsigned integers by magnitude (NaN above inf above every finite value),
// so one unsigned max per pair of halves does it.  bf16_absmax_value() folds the two halves
// into the float value (exact).
__device__ __forceinline__ uint32_t bf16x8_absmax_bits(const uint4& v) {
  const uint32_t m = 0x7fff7fffu;
  return __vmaxu2(__vmaxu2(v.x & m, v.y & m), __vmaxu2(v.z & m, v.w & m));
}
__device__ __forceinline__ float bf16_absmax_value(uint32_t halves) {
  return __uint_as_float(max(halves & 0xffffu, halves >> 16) << 16);
}

// Rotary cos/sin of pair c for token n.
__device__ __forceinline__ float2 rope_cs(const Dims& dm, const float2* __restrict__ rope, int n,
                                          int c) {
  if (c < dm.pt) {
    int t = n / (dm.gh * dm.gw);
    return rope[t * dm.pt + c];
  } else if (c < dm.pt + dm.ph) {
    int y = (n / dm.gw) % dm.gh;
    return rope[dm.rope_off_h + y * dm.ph + (c - dm.pt)];
  } else {
    int x = n % dm.gw;
    return rope[dm.rope_off_w + x * dm.pw + (c - dm.pt - dm.ph)];
  }
}

// Rotary-table offsets of token n's t, h and w positions (one division chain per token).
struct TokPos {
  int t, y, x;
};
__device__ __forceinline__ TokPos token_pos(const Dims& dm, int n) {
  const int hw = dm.gh * dm.gw;
  const int t = n / hw, rem = n - t * hw;
  const int y = rem / dm.gw;
  return {t * dm.pt, dm.rope_off_h + y * dm.ph, dm.rope_off_w + (rem - y * dm.gw) * dm.pw};
}

// Rotary cos/sin of pair c at a token position (same values as rope_cs).
__device__ __forceinline__ float2 rope_at(const Dims& dm, const float2* __restrict__ rope, const TokPos& p,
                                          int c) {
  if (c < dm.pt) return rope[p.t + c];
  if (c < dm.pt + dm.ph) return rope[p.y + (c - dm.pt)];
  return rope[p.x + (c - dm.pt - dm.ph)];
}

// phi(x) = elu(x) + 1.
__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : expf(x); }

// The same with e^x for x <= 0 as 2^(x log2 e) on the special-function unit (relative
// error ~2^-21: well inside what the bf16 paths keep of phi).
__device__ __forceinline__ float phi_fast(float x) {
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(x * 1.4426950408889634f));
  return x > 0.f ? x + 1.f : e;
}

}  // namespace rola
