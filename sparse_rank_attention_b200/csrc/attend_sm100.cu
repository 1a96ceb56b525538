// Sparse branch + fused linear epilogue + combination of RoLA (steps 3-5) on the sm_100a
// tensor cores (tcgen05 + TMEM + TMA), bf16 inputs, head dim 128.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (block-sparse softmax branch plus a
// low-rank linear branch with rotary positions); README sparse-finetuning section
// (proj_q, and the gate read here as a per-head gain g).
//
// Why the transposed tile: tcgen05.mma needs M = 128 rows for full rate, but a query
// block has 64 tokens and every query block keeps its own key blocks.  So the M side
// is taken by KEYS: each step multiplies one query block (N = 64) with a pair of its
// kept key blocks (M = 128 keys), and every MMA row does useful work:
//   S^T [128 keys x 64 q]  = [K_j1; K_j2] Q_i^T            (bf16, K-major A and B)
//   O^T [128 d x 64 q]    += [V_j1; V_j2]^T P^T            (fp16, MN-major A and B)
// Thread t of the 4 softmax warps owns TMEM lane t: key t of the pair for S^T and
// channel d = t for O^T.  The softmax max is per query (a TMEM column), so it is kept
// lazily: each query's exponent offset m only moves when a new score exceeds it by
// more than 8 (log2 units); that rare case takes an exact per-query max across the
// 128 lanes and rescales O^T.  Per-query sums l stay per thread (partials over that
// thread's keys) until the end.
//
// Roles (192 threads): warp 0 = TMA producer, warp 1 = MMA issuer (+ TMEM owner),
// warps 2-5 = softmax and epilogue.  K/V pairs are double-buffered, S^T is
// double-buffered in TMEM so the tensor cores run QK(it+1) and PV(it-1) while the
// softmax warps work on step it.
//
// Epilogue (per query block): u^T = Wq_h^T Q^T (Wq_h^T padded to 128 rows),
// phi, den = z.u, R(p) u split into bf16 hi + lo; num^T = S_h^T (R u)^T with S_h as
// bf16 hi + lo (three MMAs); out = O/l + g * num/den, staged in shared memory and
// written by one TMA store (rows past N are clipped by the tensor map).
//
// Every mbarrier wait is bounded (ROLA_ERR_DEVICE_TIMEOUT); on a timeout all roles
// leave their loops, in-flight MMAs and TMA copies are drained and TMEM is freed.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "rola_internal.cuh"
#include "sm100_ptx.cuh"

namespace rola {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;     // S^T buffers at columns 0 and 64
constexpr uint32_t kColO = 128;   // O^T
constexpr uint32_t kColU = 0;     // epilogue: u^T (reuses S buffer 0)
constexpr uint32_t kColNum = 64;  // epilogue: num^T (reuses S buffer 1)

constexpr uint32_t kOffQ = 0;              // 2 boxes [64 q][64 d] bf16, SW128 (16 KB)
constexpr uint32_t kOffK = 16384;          // 2 stages x 2 boxes [128 keys][64 d] (32 KB each)
constexpr uint32_t kOffV = 16384 + 65536;  // 2 stages x 2 boxes [128 keys][64 d] fp16
constexpr uint32_t kOffP = kOffV + 65536;  // P^T [128 keys][64 q] fp16, SW128 (16 KB)
constexpr uint32_t kOffCtl = kOffP + 16384;
constexpr uint32_t kStageBytes = 32768;
constexpr uint32_t kBoxKV = 16384;         // one [128][64] box of a K or V pair

struct Ctl {
  uint64_t q_full, k_full[2], v_full[2], kv_empty[2], s_full[2], s_empty[2];
  uint64_t p_full, pv_done, ep_bar, drain_bar, stall_bar;
  uint32_t tmem_base;
  int abort;
  float m_used[64];
  float fac[64];
  float red[4][64];
  float linv[64];
  float gden[64];
  float z[32];
};
constexpr size_t kSmemBytes = kOffCtl + sizeof(Ctl) + 1024;


// Reduce 64 per-lane values over the 32 lanes of a warp; lane l receives the results
// for entries 2l and 2l+1 (62 shuffles instead of 320).
template <bool kMax>
__device__ __forceinline__ float2 reduce_scatter64(const float* x, int lane) {
  const unsigned full = 0xffffffffu;
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  float a[32], b[16], c[8], d[4];
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4, h2 = lane & 2, h1 = lane & 1;
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const float mine = h16 ? x[32 + e] : x[e], send = h16 ? x[e] : x[32 + e];
    a[e] = op(mine, __shfl_xor_sync(full, send, 16));
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float mine = h8 ? a[16 + e] : a[e], send = h8 ? a[e] : a[16 + e];
    b[e] = op(mine, __shfl_xor_sync(full, send, 8));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float mine = h4 ? b[8 + e] : b[e], send = h4 ? b[e] : b[8 + e];
    c[e] = op(mine, __shfl_xor_sync(full, send, 4));
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float mine = h2 ? c[4 + e] : c[e], send = h2 ? c[e] : c[4 + e];
    d[e] = op(mine, __shfl_xor_sync(full, send, 2));
  }
  float r[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const float mine = h1 ? d[2 + e] : d[e], send = h1 ? d[e] : d[2 + e];
    r[e] = op(mine, __shfl_xor_sync(full, send, 1));
  }
  return make_float2(r[0], r[1]);
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_bf162(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Writes one 128-byte row (64 16-bit values given as 32 packed words) of a
// SW128 tile: 16-byte chunk c of row `row` goes to chunk position c ^ (row % 8).
__device__ __forceinline__ void st_row_sw128(uint8_t* tile, int row, const uint32_t* w) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 v = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    *reinterpret_cast<uint4*>(tile + row * 128 + ((c ^ (row & 7)) << 4)) = v;
  }
}

template <int RK>
__global__ void __launch_bounds__(kThreads, 1) attend_sm100_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
    const __nv_bfloat16* __restrict__ Wq, const float* __restrict__ g, Dims dm,
    const int32_t* __restrict__ col_idx, const __nv_bfloat16* __restrict__ S_hi,
    const __nv_bfloat16* __restrict__ S_lo, const float* __restrict__ z,
    const float2* __restrict__ rope, int* __restrict__ status, int debug_flags,
    unsigned long long limit_ns, unsigned long long debug_limit_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(base + kOffCtl);
  const uint32_t sbase = smem_addr(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const int kk_list = dm.k;
  const int npairs = (kk_list + 1) >> 1;
  const int32_t* L = col_idx + ((size_t)bh * dm.nb + i) * kk_list;
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };

  if (threadIdx.x == 0) {
    mbar_init(bar(ctl->q_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ctl->k_full[s]), 1);
      mbar_init(bar(ctl->v_full[s]), 1);
      mbar_init(bar(ctl->kv_empty[s]), 1);
      mbar_init(bar(ctl->s_full[s]), 1);
      mbar_init(bar(ctl->s_empty[s]), 128);
    }
    mbar_init(bar(ctl->p_full), 128);
    mbar_init(bar(ctl->pv_done), 1);
    mbar_init(bar(ctl->ep_bar), 1);
    mbar_init(bar(ctl->drain_bar), 1);
    mbar_init(bar(ctl->stall_bar), 1);
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 2 && lane < 32) {
    ctl->m_used[lane] = -INFINITY;
    ctl->m_used[lane + 32] = -INFINITY;
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtl wc{&ctl->abort, status, limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_out);
      const int xh = h * 128;
      mbar_expect_tx(bar(ctl->q_full), 16384);
      tma_load_3d(sbase + kOffQ, &tm_q, xh, i * 64, b, bar(ctl->q_full));
      tma_load_3d(sbase + kOffQ + 8192, &tm_q, xh + 64, i * 64, b, bar(ctl->q_full));
      int issued = 0;
      for (int it = 0; it < npairs; ++it) {
        const int s = it & 1;
        if (it >= 2 && !mbar_wait(bar(ctl->kv_empty[s]), ((it - 2) >> 1) & 1, wc)) break;
        int j1 = __ldg(L + 2 * it);
        int j2 = (2 * it + 1 < kk_list) ? __ldg(L + 2 * it + 1) : j1;
        if (j1 < 0 || j1 >= dm.nb || j2 < 0 || j2 >= dm.nb) {
          atomicCAS(status, 0, kDevBounds);
          j1 = j2 = 0;
        }
        const uint32_t kst = sbase + kOffK + s * kStageBytes, vst = sbase + kOffV + s * kStageBytes;
        mbar_expect_tx(bar(ctl->k_full[s]), kStageBytes);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(kst + c * kBoxKV, &tm_k, xh + 64 * c, j1 * 64, b, bar(ctl->k_full[s]));
          tma_load_3d(kst + c * kBoxKV + 8192, &tm_k, xh + 64 * c, j2 * 64, b, bar(ctl->k_full[s]));
        }
        mbar_expect_tx(bar(ctl->v_full[s]), kStageBytes);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(vst + c * kBoxKV, &tm_v, xh + 64 * c, j1 * 64, b, bar(ctl->v_full[s]));
          tma_load_3d(vst + c * kBoxKV + 8192, &tm_v, xh + 64 * c, j2 * 64, b, bar(ctl->v_full[s]));
        }
        issued = it + 1;
      }
      // Drain: every issued copy must land before the CTA can leave.
      mbar_wait(bar(ctl->q_full), 0, wc, false);
      for (int it = (issued >= 2 ? issued - 2 : 0); it < issued; ++it) {
        const int s = it & 1;
        mbar_wait(bar(ctl->k_full[s]), (it >> 1) & 1, wc, false);
        mbar_wait(bar(ctl->v_full[s]), (it >> 1) & 1, wc, false);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(1, 128, 64, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f16(0, 128, 64, 1, 1);
      bool ok = mbar_wait(bar(ctl->q_full), 0, wc);
      auto issue_pv = [&](int t) -> bool {
        const int s = t & 1;
        if (!mbar_wait(bar(ctl->v_full[s]), (t >> 1) & 1, wc)) return false;
        if (!mbar_wait(bar(ctl->p_full), t & 1, wc)) return false;
        tc_fence_after();
        const uint32_t va = sbase + kOffV + s * kStageBytes, pa = sbase + kOffP;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ss(tmem + kColO, sdesc_sw128(va + kk * 2048, kBoxKV, 1024),
                     sdesc_sw128(pa + kk * 2048, 8192, 1024), idesc_pv, (t > 0) || (kk > 0));
        mma_commit(bar(ctl->pv_done));
        mma_commit(bar(ctl->kv_empty[s]));
        return true;
      };
      for (int it = 0; ok && it < npairs; ++it) {
        const int s = it & 1;
        if (!mbar_wait(bar(ctl->k_full[s]), (it >> 1) & 1, wc)) { ok = false; break; }
        if (it >= 2 && !mbar_wait(bar(ctl->s_empty[s]), ((it - 2) >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ka = sbase + kOffK + s * kStageBytes, qa = sbase + kOffQ;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ss(tmem + kColS + 64 * s,
                     sdesc_sw128(ka + (kk >> 2) * kBoxKV + (kk & 3) * 32, 16, 1024),
                     sdesc_sw128(qa + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), idesc_qk, kk > 0);
        mma_commit(bar(ctl->s_full[s]));
        if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(npairs - 1);
      // Drain: no MMA may still be running when TMEM is freed.
      mma_commit(bar(ctl->drain_bar));
      mbar_wait(bar(ctl->drain_bar), 0, wc, false);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int wq = warp & 3;
    const int t = 32 * wq + lane;                  // TMEM lane: key of the pair / channel d
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * wq) << 16);
    const float sl2 = dm.scale * 1.4426950408889634f;
    uint8_t* sP = base + kOffP;
    bool fail = false;
    if (debug_flags & ROLA_DEBUG_STALL_WAIT) {
      WaitCtl dw{&ctl->abort, status, debug_limit_ns};
      fail = !mbar_wait(bar(ctl->stall_bar), 0, dw);
    }
    float lp[64];
#pragma unroll
    for (int q = 0; q < 64; ++q) lp[q] = 0.f;

    for (int it = 0; it < npairs; ++it) {
      const int s = it & 1;
      float x[64];
      const bool ok = !fail && mbar_wait(bar(ctl->s_full[s]), (it >> 1) & 1, wc);
      fail |= !ok;
      if (ok) {
        tc_fence_after();
        tmem_ld32(lane_addr + kColS + 64 * s, x);
        tmem_ld32(lane_addr + kColS + 64 * s + 32, x + 32);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(ctl->s_empty[s]));
      }
      const int jb = (t < 64) ? __ldg(L + 2 * it)
                              : ((2 * it + 1 < kk_list) ? __ldg(L + 2 * it + 1) : -1);
      const bool valid = ok && jb >= 0 && jb < dm.nb && jb * 64 + (t & 63) < dm.N;
      float dmax = -INFINITY;
#pragma unroll
      for (int q = 0; q < 64; ++q) {
        x[q] = valid ? x[q] * sl2 : -INFINITY;
        dmax = fmaxf(dmax, x[q] - ctl->m_used[q]);
      }
      if (named_vote_or(1, 128, fail || dmax > 8.f)) {
        if (named_vote_or(1, 128, fail)) break;
        // exact per-query max over the 128 keys of this pair
        const float2 wm = reduce_scatter64<true>(x, lane);
        ctl->red[wq][2 * lane] = wm.x;
        ctl->red[wq][2 * lane + 1] = wm.y;
        named_sync(1, 128);
        if (t < 64) {
          const float bm = fmaxf(fmaxf(ctl->red[0][t], ctl->red[1][t]), fmaxf(ctl->red[2][t], ctl->red[3][t]));
          const float mo = ctl->m_used[t];
          const float mn = fmaxf(mo, bm);
          ctl->fac[t] = exp2f(mo - mn);
          ctl->m_used[t] = mn;
        }
        named_sync(1, 128);
#pragma unroll
        for (int q = 0; q < 64; ++q) lp[q] *= ctl->fac[q];
        if (it > 0) {
          fail |= !mbar_wait(bar(ctl->pv_done), (it - 1) & 1, wc);
          if (!fail) {
            tc_fence_after();
            float o[32];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              tmem_ld32(lane_addr + kColO + 32 * half, o);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 32; ++q) o[q] *= ctl->fac[32 * half + q];
              tmem_st32(lane_addr + kColO + 32 * half, o);
            }
            tmem_wait_st();
          }
        }
      }
      uint32_t pw[32];
#pragma unroll
      for (int q = 0; q < 64; q += 2) {
        const float p0 = exp2f(x[q] - ctl->m_used[q]);
        const float p1 = exp2f(x[q + 1] - ctl->m_used[q + 1]);
        lp[q] += p0;
        lp[q + 1] += p1;
        pw[q >> 1] = pack_half2(p0, p1);
      }
      if (it > 0 && !fail) fail |= !mbar_wait(bar(ctl->pv_done), (it - 1) & 1, wc);
      st_row_sw128(sP, t, pw);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(ctl->p_full));
    }

    // ------------------------------------------------------------ epilogue
    if (!named_vote_or(1, 128, fail)) {
      fail |= !mbar_wait(bar(ctl->pv_done), (npairs - 1) & 1, wc);
    }
    if (!named_vote_or(1, 128, fail)) {
      tc_fence_after();
      // per-query sums l over the 128 threads
      const float2 ls = reduce_scatter64<false>(lp, lane);
      ctl->red[wq][2 * lane] = ls.x;
      ctl->red[wq][2 * lane + 1] = ls.y;
      // Wq_h^T padded to 128 rows -> K stage 0 (A operand, K-major SW128)
      {
        uint8_t* wt = base + kOffK;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float a0 = 0.f, a1 = 0.f;
            if (t < RK) {
              a0 = __bfloat162float(Wq[((size_t)h * 128 + 64 * c + 2 * e) * RK + t]);
              a1 = __bfloat162float(Wq[((size_t)h * 128 + 64 * c + 2 * e + 1) * RK + t]);
            }
            w[e] = pack_bf162(a0, a1);
          }
          st_row_sw128(wt + c * kBoxKV, t, w);
        }
      }
      // S_h^T hi / lo -> V stage 0 (A operands, MN-major SW128: row = rank a, 64 d per box)
      {
        uint8_t* sh = base + kOffV;
        uint8_t* sl = base + kOffV + 2 * RK * 128;
        for (int e = t; e < RK * 16; e += 128) {
          const int a = e >> 4, c = (e >> 3) & 1, cc = e & 7;
          const size_t src = ((size_t)bh * RK + a) * 128 + 64 * c + 8 * cc;
          const uint32_t off = c * (RK * 128) + a * 128 + ((cc ^ (a & 7)) << 4);
          *reinterpret_cast<uint4*>(sh + off) = *reinterpret_cast<const uint4*>(S_hi + src);
          *reinterpret_cast<uint4*>(sl + off) = *reinterpret_cast<const uint4*>(S_lo + src);
        }
      }
      if (t < RK) ctl->z[t] = z[(size_t)bh * RK + t];
      fence_proxy_async_smem();
      tc_fence_before();
      named_sync(1, 128);
      if (t < 64) ctl->linv[t] = 1.f / (ctl->red[0][t] + ctl->red[1][t] + ctl->red[2][t] + ctl->red[3][t]);
      if (t == 0) {
        tc_fence_after();
        constexpr uint32_t idesc_u = idesc_f16(1, 128, 64, 0, 0);
        const uint32_t wa = sbase + kOffK, qa = sbase + kOffQ;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ss(tmem + kColU, sdesc_sw128(wa + (kk >> 2) * kBoxKV + (kk & 3) * 32, 16, 1024),
                     sdesc_sw128(qa + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), idesc_u, kk > 0);
        mma_commit(bar(ctl->ep_bar));
      }
      fail |= !mbar_wait(bar(ctl->ep_bar), 0, wc);
      if (!named_vote_or(1, 128, fail)) {
        tc_fence_after();
        if (wq == 0) {
          // lane a holds u^T row a (rank a) for the 64 queries
          float u[64];
          tmem_ld32(lane_addr + kColU, u);
          tmem_ld32(lane_addr + kColU + 32, u + 32);
          tmem_wait_ld();
          const float za = lane < RK ? ctl->z[lane] : 0.f;
          float dz[64];
#pragma unroll
          for (int q = 0; q < 64; ++q) {
            u[q] = phi(u[q]);
            dz[q] = lane < RK ? u[q] * za : 0.f;
          }
          const float2 dn = reduce_scatter64<false>(dz, lane);
          const float gh = g[h];
          ctl->gden[2 * lane] = gh / dn.x;
          ctl->gden[2 * lane + 1] = gh / dn.y;
          uint32_t whi[32], wlo[32];
#pragma unroll
          for (int q = 0; q < 64; q += 2) {
            float r2[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float mine = u[q + e];
              const float other = __shfl_xor_sync(0xffffffffu, mine, 1);
              const int n = i * 64 + q + e;
              const float2 cs = (n < dm.N && lane < RK) ? rope_cs(dm, rope, n, lane >> 1) : make_float2(1.f, 0.f);
              r2[e] = (lane & 1) ? (cs.y * other + cs.x * mine) : (cs.x * mine - cs.y * other);
            }
            const uint32_t hi = pack_bf162(r2[0], r2[1]);
            const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
            whi[q >> 1] = hi;
            wlo[q >> 1] = pack_bf162(r2[0] - hf.x, r2[1] - hf.y);
          }
          if (lane < RK) {
            st_row_sw128(sP, lane, whi);
            st_row_sw128(sP + 8192, lane, wlo);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_sync(1, 128);
        if (t == 0) {
          tc_fence_after();
          constexpr uint32_t idesc_n = idesc_f16(1, 128, 64, 1, 1);
          const uint32_t sh = sbase + kOffV, sl = sbase + kOffV + 2 * RK * 128;
          const uint32_t uh = sbase + kOffP, ul = sbase + kOffP + 8192;
#pragma unroll
          for (int kk = 0; kk < RK / 16; ++kk) {
            const uint64_t ah = sdesc_sw128(sh + kk * 2048, RK * 128, 1024);
            const uint64_t al = sdesc_sw128(sl + kk * 2048, RK * 128, 1024);
            const uint64_t bhd = sdesc_sw128(uh + kk * 2048, 4096, 1024);
            const uint64_t bld = sdesc_sw128(ul + kk * 2048, 4096, 1024);
            mma_f16_ss(tmem + kColNum, ah, bhd, idesc_n, kk > 0);
            mma_f16_ss(tmem + kColNum, al, bhd, idesc_n, true);
            mma_f16_ss(tmem + kColNum, ah, bld, idesc_n, true);
          }
          mma_commit(bar(ctl->ep_bar));
        }
        fail |= !mbar_wait(bar(ctl->ep_bar), 1, wc);
        if (!named_vote_or(1, 128, fail)) {
          tc_fence_after();
          // out^T[d = t][q] = O^T / l + (g / den) num^T -> staging [2 boxes][64 q][64 d]
          uint8_t* stg = base + kOffQ;
          __nv_bfloat16* col = reinterpret_cast<__nv_bfloat16*>(stg + (t >> 6) * 8192) + (t & 63);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float o[32], nm[32];
            tmem_ld32(lane_addr + kColO + 32 * half, o);
            tmem_ld32(lane_addr + kColNum + 32 * half, nm);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const int qq = 32 * half + q;
              col[qq * 64] = __float2bfloat16_rn(o[q] * ctl->linv[qq] + nm[q] * ctl->gden[qq]);
            }
          }
          fence_proxy_async_smem();
          named_sync(1, 128);
          if (t == 0) {
            tma_store_3d(&tm_out, h * 128, i * 64, b, sbase + kOffQ);
            tma_store_3d(&tm_out, h * 128 + 64, i * 64, b, sbase + kOffQ + 8192);
            tma_store_commit();
            tma_store_wait0();
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [B, N, H*128] 16-bit tensor as a 3D map with [64 tokens x 64 channels] boxes.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, const Dims& dm,
              CUtensorMapSwizzle sw) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t HD = (cuuint64_t)dm.H * dm.d;
  cuuint64_t dims[3] = {HD, (cuuint64_t)dm.N, (cuuint64_t)dm.B};
  cuuint64_t strides[2] = {HD * 2, HD * 2 * (cuuint64_t)dm.N};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t attend_sm100_smem_bytes() { return kSmemBytes; }

cudaError_t launch_attend_sm100(const Dims& dm, const void* q, const void* k, const Workspace& ws,
                                const void* Wq, const float* g, void* out, int debug_flags,
                                int debug_limit_us, cudaStream_t st) {
  CUtensorMap tq, tk, tv, to;
  if (!make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws.v16, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, dm, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const unsigned long long limit_ns = 1000000000ull;  // 1 s per wait
  const unsigned long long dlimit = (unsigned long long)(debug_limit_us > 0 ? debug_limit_us : 1000) * 1000ull;
  dim3 grid(dm.nb, dm.B * dm.H);
  cudaError_t e;
  if (dm.r == 32) {
    e = cudaFuncSetAttribute(attend_sm100_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attend_sm100_kernel<32><<<grid, kThreads, kSmemBytes, st>>>(
        tq, tk, tv, to, static_cast<const __nv_bfloat16*>(Wq), g, dm, ws.col_idx, ws.S_hi, ws.S_lo,
        ws.z, ws.rope, ws.status, debug_flags, limit_ns, dlimit);
  } else {
    e = cudaFuncSetAttribute(attend_sm100_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attend_sm100_kernel<16><<<grid, kThreads, kSmemBytes, st>>>(
        tq, tk, tv, to, static_cast<const __nv_bfloat16*>(Wq), g, dm, ws.col_idx, ws.S_hi, ws.S_lo,
        ws.z, ws.rope, ws.status, debug_flags, limit_ns, dlimit);
  }
  return cudaGetLastError();
}

}  // namespace rola
