// C ABI of the RoLA forward library: argument checks, workspace layout, launch order.
// The operator, layouts, ownership and error rules are stated in include/rola.h.
#include <cmath>
#include <cstring>
#include <new>

#include "rola_internal.cuh"

namespace {

using rola::Dims;
using rola::Workspace;

constexpr size_t kAlign = 256;

// The sparse-attention kernel of the head-dim-128 tensor-core path.
constexpr int kMaxBlocks = 6000;  // one score row per warp must fit shared memory

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Default rotary split: 1D grid -> every pair on w; else h = w = floor(P/3), t the rest.
void default_pairs(const rola_params& p, int* pt, int* ph, int* pw) {
  const int P = p.r / 2;
  if (p.grid_t == 1 && p.grid_h == 1) {
    *pt = 0; *ph = 0; *pw = P;
  } else {
    const int hw = P / 3;
    *pt = P - 2 * hw; *ph = hw; *pw = hw;
  }
}

int keep_count(int nb, double topk) {
  double x = std::ceil(topk * (double)nb - 1e-9);
  int k = (int)x;
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return k;
}

rola_status check_params(const rola_params* p) {
  if (!p) return ROLA_ERR_INVALID_ARG;
  if (p->B < 1 || p->H < 1 || p->N < 1) return ROLA_ERR_INVALID_ARG;
  if (p->block != rola::kBlock) return ROLA_ERR_UNSUPPORTED;
  if (p->d != 64 && p->d != 128) return ROLA_ERR_UNSUPPORTED;
  if (p->r != 16 && p->r != 32) return ROLA_ERR_UNSUPPORTED;
  if (!(p->topk > 0.0 && p->topk <= 1.0)) return ROLA_ERR_INVALID_ARG;
  if (p->grid_t < 1 || p->grid_h < 1 || p->grid_w < 1) return ROLA_ERR_INVALID_ARG;
  if ((long long)p->grid_t * p->grid_h * p->grid_w != p->N) return ROLA_ERR_INVALID_ARG;
  const int sp = p->rope_pairs_t + p->rope_pairs_h + p->rope_pairs_w;
  if (p->rope_pairs_t < 0 || p->rope_pairs_h < 0 || p->rope_pairs_w < 0) return ROLA_ERR_INVALID_ARG;
  if (sp != 0 && sp != p->r / 2) return ROLA_ERR_INVALID_ARG;
  if (!(p->rope_base > 1.0) || !std::isfinite(p->rope_base)) return ROLA_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.f) || !std::isfinite(p->softmax_scale)) return ROLA_ERR_INVALID_ARG;
  if (p->dtype != ROLA_F32 && p->dtype != ROLA_BF16 && p->dtype != ROLA_FP8_E4M3)
    return ROLA_ERR_INVALID_ARG;
  if (p->dtype == ROLA_FP8_E4M3 && p->d != 128) return ROLA_ERR_UNSUPPORTED;  // tcgen05 tile only
  if (p->gate != ROLA_GATE_HEAD && p->gate != ROLA_GATE_TOKEN && p->gate != ROLA_GATE_QPROJ)
    return ROLA_ERR_INVALID_ARG;
  const int nb = (p->N + rola::kBlock - 1) / rola::kBlock;
  if (nb > kMaxBlocks) return ROLA_ERR_UNSUPPORTED;
  if ((long long)p->B * p->H * nb > (1ll << 31) / 64) return ROLA_ERR_UNSUPPORTED;
  return ROLA_OK;
}

// Tokens per linear-state partial.  The head-dim-128 key/value pass runs one CTA per SM
// (148 SMs), so its chunk is chosen to fill the SMs in whole waves: the smallest
// makespan (waves x blocks per chunk, plus one block of per-CTA overhead) over all
// chunk lengths.  The other paths keep fixed 2048-token chunks.
int state_chunk_tokens(const rola_params& p, int nb) {
  if (!(p.d == 128 && p.dtype != ROLA_F32)) return rola::kStateChunk;
  constexpr long long kSMs = 2 * 148;   // CTA slots: two per SM
  const long long bh = (long long)p.B * p.H;
  long long best_cost = -1;
  int best = nb;
  for (int cb = 1; cb <= nb; ++cb) {
    const long long nchunk = (nb + cb - 1) / cb;
    const long long waves = (bh * nchunk + kSMs - 1) / kSMs;
    const long long cost = waves * (cb + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = cb;
    }
  }
  return best * rola::kBlock;
}

Dims make_dims(const rola_params& p) {
  Dims dm{};
  dm.B = p.B; dm.H = p.H; dm.N = p.N; dm.d = p.d; dm.r = p.r;
  dm.nb = (p.N + rola::kBlock - 1) / rola::kBlock;
  dm.k = keep_count(dm.nb, p.topk);
  dm.gt = p.grid_t; dm.gh = p.grid_h; dm.gw = p.grid_w;
  if (p.rope_pairs_t + p.rope_pairs_h + p.rope_pairs_w == 0) {
    default_pairs(p, &dm.pt, &dm.ph, &dm.pw);
  } else {
    dm.pt = p.rope_pairs_t; dm.ph = p.rope_pairs_h; dm.pw = p.rope_pairs_w;
  }
  dm.rope_off_h = dm.gt * dm.pt;
  dm.rope_off_w = dm.rope_off_h + dm.gh * dm.ph;
  dm.chunk_tok = state_chunk_tokens(p, dm.nb);
  dm.nchunk = (p.N + dm.chunk_tok - 1) / dm.chunk_tok;
  dm.scale = p.softmax_scale > 0.f ? p.softmax_scale : (float)(1.0 / std::sqrt((double)p.d));
  dm.rope_base = p.rope_base;
  dm.gate_mode = p.gate;
  return dm;
}

// Carves the workspace; with base == nullptr only the size is computed.
size_t carve(const rola_params& p, const Dims& dm, char* base, Workspace* ws) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* r = base ? base + off : nullptr;
    off = align_up(off + bytes);
    return r;
  };
  const size_t BH = (size_t)dm.B * dm.H;
  Workspace w{};
  w.status = reinterpret_cast<int*>(take(kAlign));
  w.rope = reinterpret_cast<float2*>(take(sizeof(float2) * (size_t)(dm.rope_off_w + dm.gw * dm.pw)));
  w.qbar = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb * dm.d));
  w.kbar = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb * dm.d));
  w.col_idx = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * BH * dm.nb * dm.k));
  w.scores = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb * rola::score_row_stride(dm)));
  w.knorm = reinterpret_cast<float*>(take(sizeof(float) * BH * rola::score_row_stride(dm)));
  w.S_part = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nchunk * dm.r * dm.d));
  w.z_part = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nchunk * dm.r));
  w.S = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.r * dm.d));
  w.z = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.r));
  w.S_hi = reinterpret_cast<__nv_bfloat16*>(take(sizeof(__nv_bfloat16) * BH * dm.r * dm.d));
  w.S_lo = reinterpret_cast<__nv_bfloat16*>(take(sizeof(__nv_bfloat16) * BH * dm.r * dm.d));
  if (p.dtype == ROLA_BF16) {
    w.v16 = reinterpret_cast<__half*>(take(sizeof(__half) * (size_t)dm.B * dm.N * dm.H * dm.d));
    w.vexp = reinterpret_cast<int*>(take(sizeof(int) * BH * dm.nb));
  }
  if (p.dtype != ROLA_F32 && p.d == 128) {
    w.redo = reinterpret_cast<int*>(take(sizeof(int) * (1 + 2 * BH * dm.nb)));
    w.simg = reinterpret_cast<uint8_t*>(take(BH * 4 * dm.r * 128));
    w.uimg = reinterpret_cast<uint8_t*>(take(BH * dm.nb * 2 * dm.r * 128));
    w.gden = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb * 64));
  }
  if (p.dtype == ROLA_FP8_E4M3) {
    const size_t elems = (size_t)dm.B * dm.N * dm.H * dm.d;
    w.q8 = reinterpret_cast<uint8_t*>(take(elems));
    w.k8 = reinterpret_cast<uint8_t*>(take(elems));
    w.v8 = reinterpret_cast<uint8_t*>(take(elems));
    w.sq = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb));
    w.sk = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb));
    w.sv = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb));
  }
  if (ws) *ws = w;
  return off;
}

rola_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA; }

// Zeroes the device status word the first time a plan issues work.
rola_status ensure_status_word(rola_plan_t plan, cudaStream_t st) {
  if (plan->status_ready) return ROLA_OK;
  cudaError_t e = cudaMemsetAsync(plan->ws.status, 0, kAlign, st);
  if (e != cudaSuccess) return ROLA_ERR_CUDA;
  plan->status_ready = true;
  return ROLA_OK;
}

size_t elem_size(rola_dtype dt) { return dt == ROLA_F32 ? 4 : 2; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

}  // namespace

extern "C" {

rola_status rola_params_default(rola_params* p) {
  if (!p) return ROLA_ERR_INVALID_ARG;
  std::memset(p, 0, sizeof(*p));
  p->B = 1; p->H = 1; p->N = 0; p->d = 128; p->r = 32;
  p->block = rola::kBlock;
  p->topk = 0.1;
  p->grid_t = 1; p->grid_h = 1; p->grid_w = 0;
  p->rope_base = 10000.0;
  p->softmax_scale = 0.f;
  p->dtype = ROLA_BF16;
  p->gate = ROLA_GATE_HEAD;
  return ROLA_OK;
}

rola_status rola_keep_count(const rola_params* p, int* nb, int* k) {
  rola_status s = check_params(p);
  if (s != ROLA_OK) return s;
  if (!nb || !k) return ROLA_ERR_INVALID_ARG;
  const Dims dm = make_dims(*p);
  *nb = dm.nb;
  *k = dm.k;
  return ROLA_OK;
}

rola_status rola_workspace_size(const rola_params* p, size_t* bytes) {
  rola_status s = check_params(p);
  if (s != ROLA_OK) return s;
  if (!bytes) return ROLA_ERR_INVALID_ARG;
  *bytes = carve(*p, make_dims(*p), nullptr, nullptr);
  return ROLA_OK;
}

rola_status rola_plan(const rola_params* p, void* workspace, size_t workspace_bytes,
                      rola_plan_t* plan) {
  rola_status s = check_params(p);
  if (s != ROLA_OK) return s;
  if (!plan) return ROLA_ERR_INVALID_ARG;
  *plan = nullptr;
  const Dims dm = make_dims(*p);
  const size_t need = carve(*p, dm, nullptr, nullptr);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kAlign) != 0 ||
      workspace_bytes < need)
    return ROLA_ERR_WORKSPACE;
  rola_plan_s* pl = new (std::nothrow) rola_plan_s();
  if (!pl) return ROLA_ERR_INVALID_ARG;
  pl->p = *p;
  pl->dm = dm;
  carve(*p, dm, static_cast<char*>(workspace), &pl->ws);
  pl->ws_base = workspace;
  pl->ws_bytes = workspace_bytes;
  *plan = pl;
  return ROLA_OK;
}

namespace {
constexpr int kProfSlots = 5;   // events per recorded forward (at most 4 stages)

void destroy_profile(rola_plan_t plan) {
  if (!plan->prof_events) return;
  for (int e = 0; e < ROLA_PROFILE_CALLS * kProfSlots; ++e)
    if (plan->prof_events[e]) cudaEventDestroy(plan->prof_events[e]);
  delete[] plan->prof_events;
  plan->prof_events = nullptr;
  plan->prof_calls = 0;
}

// Records the boundary event `k` of the current recorded call (no-op when not profiling).
void mark(rola_plan_t plan, int slot, int k, cudaStream_t st) {
  if (plan->prof_events && slot >= 0) cudaEventRecord(plan->prof_events[slot * kProfSlots + k], st);
}
}  // namespace

void rola_plan_destroy(rola_plan_t plan) {
  if (!plan) return;
  destroy_profile(plan);
  delete plan;
}

rola_status rola_profile_stages(rola_plan_t plan, int enable) {
  if (!plan) return ROLA_ERR_INVALID_ARG;
  destroy_profile(plan);
  if (!enable) return ROLA_OK;
  plan->prof_events = new (std::nothrow) cudaEvent_t[ROLA_PROFILE_CALLS * kProfSlots]();
  if (!plan->prof_events) return ROLA_ERR_INVALID_ARG;
  for (int e = 0; e < ROLA_PROFILE_CALLS * kProfSlots; ++e)
    if (cudaEventCreate(&plan->prof_events[e]) != cudaSuccess) {
      destroy_profile(plan);
      return ROLA_ERR_CUDA;
    }
  plan->prof_calls = 0;
  return ROLA_OK;
}

rola_status rola_get_stage_times(rola_plan_t plan, float* ms, int max_stages, int* nstages, int* ncalls) {
  if (!plan || !plan->prof_events || !nstages || !ncalls || (max_stages > 0 && !ms)) return ROLA_ERR_INVALID_ARG;
  const int calls = plan->prof_calls, ns = plan->prof_stages;
  *nstages = ns;
  *ncalls = calls;
  for (int s = 0; s < max_stages; ++s) ms[s] = 0.f;
  if (calls == 0) return ROLA_OK;
  if (cudaEventSynchronize(plan->prof_events[(calls - 1) * kProfSlots + ns]) != cudaSuccess) return ROLA_ERR_CUDA;
  for (int c = 0; c < calls; ++c)
    for (int s = 0; s < ns && s < max_stages; ++s) {
      float t = 0.f;
      if (cudaEventElapsedTime(&t, plan->prof_events[c * kProfSlots + s], plan->prof_events[c * kProfSlots + s + 1]) !=
          cudaSuccess)
        return ROLA_ERR_CUDA;
      ms[s] += t;
    }
  plan->prof_calls = 0;
  return ROLA_OK;
}

rola_status rola_select_blocks(rola_plan_t plan, const void* q, const void* k,
                               rola_stream_t stream) {
  if (!plan || !q || !k || !aligned16(q) || !aligned16(k)) return ROLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rola_status s = ensure_status_word(plan, st);
  if (s != ROLA_OK) return s;
  cudaError_t e = rola::launch_pool(plan->dm, plan->p.dtype, q, k, plan->ws, st);
  if (e != cudaSuccess) return ROLA_ERR_CUDA;
  return cuda_status(rola::launch_select(plan->dm, plan->ws, st));
}

rola_status rola_linear_state(rola_plan_t plan, const void* k, const void* v, const void* Wk,
                              rola_stream_t stream) {
  if (!plan || !k || !v || !Wk || !aligned16(k) || !aligned16(v) || !aligned16(Wk))
    return ROLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rola_status s = ensure_status_word(plan, st);
  if (s != ROLA_OK) return s;
  if (!plan->rope_ready) {
    if (rola::launch_rope_table(plan->dm, plan->ws, st) != cudaSuccess) return ROLA_ERR_CUDA;
    plan->rope_ready = true;
  }
  return cuda_status(rola::launch_linear_state(plan->dm, plan->p.dtype, k, v, Wk, plan->ws, st));
}

rola_status rola_attend(rola_plan_t plan, const void* q, const void* k, const void* v,
                        const void* Wq, const float* g, void* out, rola_stream_t stream) {
  if (!plan || !q || !k || !v || !Wq || !g || !out) return ROLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(Wq) || !aligned16(g) ||
      !aligned16(out))
    return ROLA_ERR_INVALID_ARG;
  const rola_params& p = plan->p;
  const size_t act = (size_t)p.B * p.N * p.H * p.d * elem_size(p.dtype);
  if (overlaps(out, act, q, act) || overlaps(out, act, k, act) || overlaps(out, act, v, act))
    return ROLA_ERR_INVALID_ARG;
  if (!plan->rope_ready) return ROLA_ERR_INVALID_ARG;  // rola_linear_state must run first
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rola_status s = ensure_status_word(plan, st);
  if (s != ROLA_OK) return s;
  cudaError_t e;
  if (p.dtype == ROLA_F32)
    e = rola::launch_attend_f32(plan->dm, q, k, v, Wq, g, out, plan->ws, st);
  else if (p.d == 128) {
    e = rola::launch_query_features(plan->dm, p.dtype == ROLA_FP8_E4M3, q, Wq, g, plan->ws, st);
    if (e == cudaSuccess)
      e = rola::launch_attend_sm100(plan->dm, q, k, plan->ws, out, p.dtype == ROLA_FP8_E4M3, plan->debug_flags,
                      plan->debug_limit_us, st);
  }
  else  // head dim 64: the transposed tcgen05 tile needs d = 128 rows
    e = rola::launch_attend_bf16_warpmma(plan->dm, q, k, v, Wq, g, out, plan->ws, st);
  return cuda_status(e);
}

rola_status rola_forward(rola_plan_t plan, const void* q, const void* k, const void* v,
                         const void* Wq, const void* Wk, const float* g, void* out,
                         rola_stream_t stream) {
  if (!plan || !q || !k || !v || !Wq || !Wk || !g || !out) return ROLA_ERR_INVALID_ARG;
  const rola_params& p = plan->p;
  const size_t act = (size_t)p.B * p.N * p.H * p.d * elem_size(p.dtype);
  if (overlaps(out, act, q, act) || overlaps(out, act, k, act) || overlaps(out, act, v, act))
    return ROLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(Wq) || !aligned16(Wk) || !aligned16(g) ||
      !aligned16(out))
    return ROLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int slot = -1;
  if (plan->prof_events && plan->prof_calls < ROLA_PROFILE_CALLS) slot = plan->prof_calls++;
  if (!(p.d == 128 && p.dtype != ROLA_F32)) {
    plan->prof_stages = 3;
    mark(plan, slot, 0, st);
    rola_status s = rola_select_blocks(plan, q, k, stream);
    if (s != ROLA_OK) return s;
    mark(plan, slot, 1, st);
    s = rola_linear_state(plan, k, v, Wk, stream);
    if (s != ROLA_OK) return s;
    mark(plan, slot, 2, st);
    s = rola_attend(plan, q, k, v, Wq, g, out, stream);
    mark(plan, slot, 3, st);
    return s;
  }
  // Head dim 128, bf16 / fp8: each input is read once before the attention kernel.
  //   key/value pass (state partials, k means, v copy / e4m3 k and v) -> state reduction
  //   -> query pass (q means, query features, e4m3 q) -> block scores -> top-k -> attention
  plan->prof_stages = 4;
  mark(plan, slot, 0, st);
  rola_status s = rola_linear_state(plan, k, v, Wk, stream);
  if (s != ROLA_OK) return s;
  mark(plan, slot, 1, st);
  const bool fp8 = p.dtype == ROLA_FP8_E4M3;
  cudaError_t e = rola::launch_query_features(plan->dm, fp8, q, Wq, g, plan->ws, st);
  mark(plan, slot, 2, st);
  if (e == cudaSuccess) e = rola::launch_select(plan->dm, plan->ws, st);
  mark(plan, slot, 3, st);
  if (e == cudaSuccess)
    e = rola::launch_attend_sm100(plan->dm, q, k, plan->ws, out, fp8, plan->debug_flags, plan->debug_limit_us, st);
  mark(plan, slot, 4, st);
  return cuda_status(e);
}

rola_status rola_select_blocks_noalloc(const rola_params* p, const void* q, const void* k,
                                       int32_t* col_idx, rola_stream_t stream) {
  rola_status s = check_params(p);
  if (s != ROLA_OK) return s;
  if (!q || !k || !col_idx || !aligned16(q) || !aligned16(k) || !aligned16(col_idx))
    return ROLA_ERR_INVALID_ARG;
  const Dims dm = make_dims(*p);
  if (rola::select_noalloc_bytes(dm) > rola::select_noalloc_capacity()) return ROLA_ERR_WORKSPACE;
  const size_t act = (size_t)p->B * p->N * p->H * p->d * elem_size(p->dtype);
  const size_t lists = sizeof(int32_t) * (size_t)dm.B * dm.H * dm.nb * dm.k;
  if (overlaps(col_idx, lists, q, act) || overlaps(col_idx, lists, k, act)) return ROLA_ERR_INVALID_ARG;
  return cuda_status(rola::select_blocks_noalloc(dm, p->dtype, q, k, col_idx,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

rola_status rola_get_block_lists(rola_plan_t plan, int32_t* col_idx, rola_stream_t stream) {
  if (!plan || !col_idx) return ROLA_ERR_INVALID_ARG;
  const Dims& dm = plan->dm;
  const size_t bytes = sizeof(int32_t) * (size_t)dm.B * dm.H * dm.nb * dm.k;
  return cuda_status(cudaMemcpyAsync(col_idx, plan->ws.col_idx, bytes, cudaMemcpyDeviceToDevice,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

rola_status rola_get_pooled(rola_plan_t plan, float* qbar, float* kbar, rola_stream_t stream) {
  if (!plan || !qbar || !kbar) return ROLA_ERR_INVALID_ARG;
  const Dims& dm = plan->dm;
  const size_t bytes = sizeof(float) * (size_t)dm.B * dm.H * dm.nb * dm.d;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(qbar, plan->ws.qbar, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ROLA_ERR_CUDA;
  return cuda_status(cudaMemcpyAsync(kbar, plan->ws.kbar, bytes, cudaMemcpyDeviceToDevice, st));
}

rola_status rola_get_block_scores(rola_plan_t plan, float* scores, float* knorm, rola_stream_t stream) {
  if (!plan || !scores || !knorm) return ROLA_ERR_INVALID_ARG;
  const Dims& dm = plan->dm;
  const size_t BH = (size_t)dm.B * dm.H, nbp = (size_t)rola::score_row_stride(dm);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpy2DAsync(scores, sizeof(float) * dm.nb, plan->ws.scores, sizeof(float) * nbp, sizeof(float) * dm.nb,
                        BH * dm.nb, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return ROLA_ERR_CUDA;
  return cuda_status(cudaMemcpy2DAsync(knorm, sizeof(float) * dm.nb, plan->ws.knorm, sizeof(float) * nbp,
                                       sizeof(float) * dm.nb, BH, cudaMemcpyDeviceToDevice, st));
}

rola_status rola_get_fp8_copies(rola_plan_t plan, uint8_t* q8, uint8_t* k8, uint8_t* v8, float* sq,
                                float* sk, float* sv, rola_stream_t stream) {
  if (!plan || !q8 || !k8 || !v8 || !sq || !sk || !sv) return ROLA_ERR_INVALID_ARG;
  if (plan->p.dtype != ROLA_FP8_E4M3) return ROLA_ERR_INVALID_ARG;
  const Dims& dm = plan->dm;
  const size_t elems = (size_t)dm.B * dm.N * dm.H * dm.d;
  const size_t sbytes = sizeof(float) * (size_t)dm.B * dm.H * dm.nb;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const struct { void* dst; const void* src; size_t n; } copies[6] = {
      {q8, plan->ws.q8, elems}, {k8, plan->ws.k8, elems}, {v8, plan->ws.v8, elems},
      {sq, plan->ws.sq, sbytes}, {sk, plan->ws.sk, sbytes}, {sv, plan->ws.sv, sbytes}};
  for (const auto& c : copies)
    if (cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyDeviceToDevice, st) != cudaSuccess) return ROLA_ERR_CUDA;
  return ROLA_OK;
}

rola_status rola_get_attend_redo_count(rola_plan_t plan, int* count, rola_stream_t stream) {
  if (!plan || !count) return ROLA_ERR_INVALID_ARG;
  *count = 0;
  if (!plan->ws.redo) return ROLA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(count, plan->ws.redo, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return ROLA_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(st));
}

rola_status rola_get_linear_state(rola_plan_t plan, float* S, float* z, rola_stream_t stream) {
  if (!plan || !S || !z) return ROLA_ERR_INVALID_ARG;
  const Dims& dm = plan->dm;
  const size_t BH = (size_t)dm.B * dm.H;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(S, plan->ws.S, sizeof(float) * BH * dm.r * dm.d, cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return ROLA_ERR_CUDA;
  return cuda_status(
      cudaMemcpyAsync(z, plan->ws.z, sizeof(float) * BH * dm.r, cudaMemcpyDeviceToDevice, st));
}

rola_status rola_poll_device_status(rola_plan_t plan, rola_stream_t stream) {
  if (!plan) return ROLA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!plan->status_ready) return ROLA_OK;
  int word = 0;
  if (cudaMemcpyAsync(&word, plan->ws.status, sizeof(int), cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return ROLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ROLA_ERR_CUDA;
  if (word == 0) return ROLA_OK;
  if (cudaMemsetAsync(plan->ws.status, 0, sizeof(int), st) != cudaSuccess) return ROLA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ROLA_ERR_CUDA;
  if (word == ROLA_ERR_DEVICE_TIMEOUT || word == ROLA_ERR_RANGE) return (rola_status)word;
  return ROLA_ERR_DEVICE_BOUNDS;
}

rola_status rola_set_debug(rola_plan_t plan, int flags, int limit_us) {
  if (!plan || flags < 0 || limit_us < 0) return ROLA_ERR_INVALID_ARG;
  plan->debug_flags = flags;
  plan->debug_limit_us = limit_us;
  return ROLA_OK;
}

rola_status rola_backward_workspace_size(const rola_params* p, size_t* bytes) {
  if (!bytes) return ROLA_ERR_INVALID_ARG;
  const rola_status s = check_params(p);
  if (s != ROLA_OK) return s;
  if (p->dtype != ROLA_F32 && p->dtype != ROLA_BF16) return ROLA_ERR_UNSUPPORTED;
  *bytes = rola::backward_workspace_bytes(make_dims(*p), nullptr, nullptr);
  return ROLA_OK;
}

rola_status rola_backward(rola_plan_t plan, const void* q, const void* k, const void* v, const void* Wq,
                          const void* Wk, const float* g, const void* dout, float* dq, float* dk, float* dv,
                          float* dWq, float* dWk, float* dg, void* bwd_workspace, size_t bwd_workspace_bytes,
                          rola_stream_t stream) {
  if (!plan) return ROLA_ERR_INVALID_ARG;
  const rola_params& p = plan->p;
  if (p.dtype != ROLA_F32 && p.dtype != ROLA_BF16) return ROLA_ERR_UNSUPPORTED;
  const void* in[] = {q, k, v, Wq, Wk, g, dout};
  const void* outp[] = {dq, dk, dv, dWq, dWk, dg, bwd_workspace};
  for (const void* x : in)
    if (!x || !aligned16(x)) return ROLA_ERR_INVALID_ARG;
  for (const void* x : outp)
    if (!x || !aligned16(x)) return ROLA_ERR_INVALID_ARG;
  const rola::Dims& dm = plan->dm;
  rola::BwdWorkspace bw;
  if (bwd_workspace_bytes < rola::backward_workspace_bytes(dm, nullptr, nullptr)) return ROLA_ERR_WORKSPACE;
  rola::backward_workspace_bytes(dm, &bw, static_cast<char*>(bwd_workspace));
  const size_t es = elem_size(p.dtype);
  const size_t act = (size_t)p.B * p.N * p.H * p.d;
  const size_t wsz = (size_t)p.H * p.d * p.r;
  const size_t gsz = p.gate == ROLA_GATE_HEAD ? (size_t)p.H
                     : p.gate == ROLA_GATE_TOKEN ? (size_t)p.B * p.N * p.H
                                                 : (size_t)p.H * (p.d + 1);
  // the gradients (and the scratch) overlap neither each other nor any input
  const void* ob[] = {dq, dk, dv, dWq, dWk, dg, bwd_workspace};
  const size_t on[] = {act * 4, act * 4, act * 4, wsz * 4, wsz * 4, gsz * 4, bwd_workspace_bytes};
  const size_t inn[] = {act * es, act * es, act * es, wsz * es, wsz * es, gsz * 4, act * es};
  for (int a = 0; a < 7; ++a) {
    for (int c = 0; c < 7; ++c)
      if (overlaps(ob[a], on[a], in[c], inn[c])) return ROLA_ERR_INVALID_ARG;
    for (int c = a + 1; c < 7; ++c)
      if (overlaps(ob[a], on[a], ob[c], on[c])) return ROLA_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  rola_status s = ensure_status_word(plan, st);
  if (s != ROLA_OK) return s;
  if (!plan->rope_ready) {
    if (rola::launch_rope_table(dm, plan->ws, st) != cudaSuccess) return ROLA_ERR_CUDA;
    plan->rope_ready = true;
  }
  cudaError_t e = rola::launch_pool(dm, p.dtype, q, k, plan->ws, st);
  if (e == cudaSuccess) e = rola::launch_select(dm, plan->ws, st);
  if (e == cudaSuccess) e = rola::launch_linear_state(dm, p.dtype, k, v, Wk, plan->ws, st);
  if (e == cudaSuccess)
    e = rola::launch_backward(dm, p.dtype, q, k, v, Wq, Wk, g, dout, dq, dk, dv, dWq, dWk, dg, plan->ws, bw, st);
  return cuda_status(e);
}

rola_status rola_eval_exp2(const float* x, float* y, int64_t n, int mode, rola_stream_t stream) {
  if (n < 0 || (mode != 0 && mode != 1) || (n > 0 && (!x || !y))) return ROLA_ERR_INVALID_ARG;
  return rola::launch_eval_exp2(x, y, n, mode, (cudaStream_t)stream) == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

const char* rola_status_string(rola_status s) {
  switch (s) {
    case ROLA_OK: return "ok";
    case ROLA_ERR_INVALID_ARG: return "invalid argument";
    case ROLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case ROLA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case ROLA_ERR_CUDA: return "CUDA runtime error";
    case ROLA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case ROLA_ERR_DEVICE_BOUNDS: return "a device-side index check failed";
    case ROLA_ERR_RANGE: return "an input value is outside the supported range";
  }
  return "unknown status";
}

}  // extern "C"
