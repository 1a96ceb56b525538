// The backward's dq over the kept blocks on the sm_100a tensor cores (tcgen05 + TMEM + TMA),
// bf16 inputs, head dim 128: the same transposed tile as the forward's attention kernel.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (the block-sparse softmax branch whose
// gradient this is); README sparse-finetuning section (the attention is trained).
//
// With the softmax row statistics known (lse of each query row and D = dout . O, from the
// row-statistics kernel), each (query block i, pair of its kept key blocks j1, j2) needs
//   S^T  [128 keys x 64 q] = [K_j1; K_j2] Q_i^T            (bf16, K-major A and B)
//   dP^T [128 keys x 64 q] = [V_j1; V_j2] G_i^T            (G = dout; the same shape)
//   dA^T = P^T (dP^T - D_q),  P^T = 2^(S^T scale log2(e) - lse_q)    (elementwise: every
//          constant belongs to a column, so no reduction crosses the TMEM lanes)
//   dQ^T [128 d x 64 q]   += [K_j1; K_j2]^T dA^T             (A = the K pair read MN-major,
//          as the forward reads V; B = dA^T as bf16 hi + lo, two products)
// and dq += scale dQ at the tile's end (added to the linear part already in dq).
//
// Roles (384 threads): warp 0 = TMA producer of the tile's Q and dout (one slot) and of the
// K ring; warp 1 = issuer of S^T and dP^T (and TMEM owner); warp 2 = issuer of dQ^T;
// warp 3 = producer of the V ring; warps 4-11 = two groups of four, group g owning query
// columns [32 g, 32 g + 32): thread t of a group owns TMEM lane t (key t of the pair for
// S^T, dP^T; channel t for dQ^T).  K stages are freed after their dQ^T products (three of
// them), V stages after their dP^T products (two); S^T/dP^T are double-buffered in TMEM.
// Persistent: one CTA per SM walks the tiles tau = blockIdx.x + n * gridDim.x.
//
// The exponentials run on ex2.approx (relative error ~2^-22, far inside the gradients'
// tolerance), as in the forward's softmax.
//
// Every mbarrier wait is bounded (ROLA_ERR_DEVICE_TIMEOUT); on a timeout all roles leave
// their loops, in-flight MMAs and TMA copies are drained and TMEM is freed.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "rola_internal.cuh"
#include "sm100_ptx.cuh"
#include "softmax_exp.cuh"

namespace rola {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kSoftmaxWarps = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S^T, two buffers (0, 64)
constexpr uint32_t kColDP = 128;   // dP^T, two buffers (128, 192)
constexpr uint32_t kColQ = 256;    // dQ^T
constexpr int kKStages = 3;   // K is held until its dQ^T products: one more stage than V
constexpr int kVStages = 2;
constexpr int kABufs = 1;     // dA^T staging buffers (hi + lo each)

constexpr uint32_t kPairBytes = 128 * 128 * 2;   // K or V pair (two 64-channel boxes of 16 KB)
constexpr uint32_t kBoxKV = 16384;
constexpr uint32_t kStgBytes = 128 * 128;        // one dA^T half: 128 keys x 64 q bf16
constexpr uint32_t kOffQG = 0;                   // Q (16 KB) then dout (16 KB)
constexpr uint32_t kOffK = 32768;
constexpr uint32_t kOffV = kOffK + kKStages * kPairBytes;
constexpr uint32_t kOffA = kOffV + kVStages * kPairBytes;   // [kABufs][hi, lo] dA^T
constexpr uint32_t kOffCtl = kOffA + 2 * kABufs * kStgBytes;

struct Ctl {
  uint64_t qg_full, qg_free, k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_free[2], a_full[kABufs], a_free[kABufs], dq_done, dq_free, drain_s, drain_q;
  uint32_t tmem_base;
  int abort;
  alignas(16) float lse[2][64];   // per group: the tile's lse (log2 units) and D per query
  alignas(16) float dd[2][64];
};
constexpr size_t kSmemBytes = kOffCtl + sizeof(Ctl) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(x0, x1);
  const float2 bf = __bfloat1622float2(b);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - bf.x, x1 - bf.y);
  hi = *reinterpret_cast<const uint32_t*>(&b);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__global__ void __launch_bounds__(kThreads, 1) bwd_dq_sm100_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Dims dm,
    const int32_t* __restrict__ col_idx, const float* __restrict__ lse, const float* __restrict__ Drow,
    float* __restrict__ dq, int* __restrict__ status, unsigned long long limit_cycles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(base + kOffCtl);
  const uint32_t sbase = smem_addr(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = dm.nb * dm.B * dm.H;
  const int kk_list = dm.k, npairs = (kk_list + 1) >> 1;
  const int my_tiles = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };
  auto tile_of = [&](int jt) { return (int)blockIdx.x + jt * (int)gridDim.x; };
  auto list_of = [&](int tau) { return col_idx + (size_t)tau * kk_list; };

  if (threadIdx.x == 0) {
    mbar_init(bar(ctl->qg_full), 1);
    mbar_init(bar(ctl->qg_free), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(ctl->k_full[s]), 1);
      mbar_init(bar(ctl->k_empty[s]), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(ctl->v_full[s]), 1);
      mbar_init(bar(ctl->v_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ctl->s_full[s]), 1);
      mbar_init(bar(ctl->s_free[s]), kSoftmaxWarps);
    }
    for (int s = 0; s < kABufs; ++s) {
      mbar_init(bar(ctl->a_full[s]), kSoftmaxWarps);
      mbar_init(bar(ctl->a_free[s]), 1);
    }
    mbar_init(bar(ctl->dq_done), 1);
    mbar_init(bar(ctl->dq_free), kSoftmaxWarps);
    mbar_init(bar(ctl->drain_s), 1);
    mbar_init(bar(ctl->drain_q), 1);
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtl wc{&ctl->abort, status, limit_cycles};
  auto pair_blocks = [&](const int32_t* L, int it, int& j1, int& j2) {
    j1 = __ldg(L + 2 * it);
    j2 = (2 * it + 1 < kk_list) ? __ldg(L + 2 * it + 1) : j1;
    if (j1 < 0 || j1 >= dm.nb || j2 < 0 || j2 >= dm.nb) {
      atomicCAS(status, 0, kDevBounds);
      j1 = j2 = 0;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ Q, dout and the K ring
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_g);
      tma_prefetch_desc(&tm_k);
      int gp = 0, nqg = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        const int tau = tile_of(jt);
        const int bh = tau / dm.nb, i = tau - bh * dm.nb, b = bh / dm.H, xh = (bh % dm.H) * 128;
        const int32_t* L = list_of(tau);
        // one slot: the previous tile's S^T and dP^T products must be done with it
        if (jt > 0 && !mbar_wait(bar(ctl->qg_free), (jt - 1) & 1, wc)) break;
        mbar_expect_tx(bar(ctl->qg_full), 32768);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sbase + kOffQG + c * 8192, &tm_q, xh + 64 * c, i * 64, b, bar(ctl->qg_full));
          tma_load_3d(sbase + kOffQG + 16384 + c * 8192, &tm_g, xh + 64 * c, i * 64, b, bar(ctl->qg_full));
        }
        ++nqg;
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int s = gp % kKStages;
          if (gp >= kKStages && !mbar_wait(bar(ctl->k_empty[s]), ((gp / kKStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          int j1, j2;
          pair_blocks(L, it, j1, j2);
          const uint32_t st = sbase + kOffK + s * kPairBytes;
          mbar_expect_tx(bar(ctl->k_full[s]), kPairBytes);
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(st + c * kBoxKV, &tm_k, xh + 64 * c, j1 * 64, b, bar(ctl->k_full[s]));
            tma_load_3d(st + c * kBoxKV + 8192, &tm_k, xh + 64 * c, j2 * 64, b, bar(ctl->k_full[s]));
          }
        }
      }
      if (nqg > 0) mbar_wait(bar(ctl->qg_full), (nqg - 1) & 1, wc, false);
      for (int x = (gp > kKStages ? gp - kKStages : 0); x < gp; ++x)
        mbar_wait(bar(ctl->k_full[x % kKStages]), (x / kKStages) & 1, wc, false);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ the V ring
    if (lane == 0) {
      tma_prefetch_desc(&tm_v);
      int gp = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        const int tau = tile_of(jt);
        const int bh = tau / dm.nb, b = bh / dm.H, xh = (bh % dm.H) * 128;
        const int32_t* L = list_of(tau);
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int s = gp % kVStages;
          if (gp >= kVStages && !mbar_wait(bar(ctl->v_empty[s]), ((gp / kVStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          int j1, j2;
          pair_blocks(L, it, j1, j2);
          const uint32_t st = sbase + kOffV + s * kPairBytes;
          mbar_expect_tx(bar(ctl->v_full[s]), kPairBytes);
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(st + c * kBoxKV, &tm_v, xh + 64 * c, j1 * 64, b, bar(ctl->v_full[s]));
            tma_load_3d(st + c * kBoxKV + 8192, &tm_v, xh + 64 * c, j2 * 64, b, bar(ctl->v_full[s]));
          }
        }
      }
      for (int x = (gp > kVStages ? gp - kVStages : 0); x < gp; ++x)
        mbar_wait(bar(ctl->v_full[x % kVStages]), (x / kVStages) & 1, wc, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S^T and dP^T
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(1, 128, 64, 0, 0);
      int gp = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        if (!mbar_wait(bar(ctl->qg_full), jt & 1, wc)) break;
        const uint64_t dqd = sdesc_sw128(sbase + kOffQG, 16, 1024);
        const uint64_t dgd = sdesc_sw128(sbase + kOffQG + 16384, 16, 1024);
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int ks = gp % kKStages, vs = gp % kVStages, sb = gp & 1;
          if (!mbar_wait(bar(ctl->k_full[ks]), (gp / kKStages) & 1, wc) ||
              !mbar_wait(bar(ctl->v_full[vs]), (gp / kVStages) & 1, wc) ||
              (gp >= 2 && !mbar_wait(bar(ctl->s_free[sb]), ((gp - 2) >> 1) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dk = sdesc_sw128(sbase + kOffK + ks * kPairBytes, 16, 1024);
          const uint64_t dv = sdesc_sw128(sbase + kOffV + vs * kPairBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // K-step offsets: 32 B inside a box, boxes 16 KB / 8 KB apart
            const uint32_t ab = ((kk >> 2) * kBoxKV + (kk & 3) * 32) >> 4, bb = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
            mma_f16_ss(tmem + kColS + 64 * sb, dk + ab, dqd + bb, idesc, kk > 0);
            mma_f16_ss(tmem + kColDP + 64 * sb, dv + ab, dgd + bb, idesc, kk > 0);
          }
          mma_commit(bar(ctl->s_full[sb]));
          mma_commit(bar(ctl->v_empty[vs]));
        }
        if (ok) mma_commit(bar(ctl->qg_free));   // this tile's Q and dout are read
      }
      mma_commit(bar(ctl->drain_s));
      mbar_wait(bar(ctl->drain_s), 0, wc, false);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ dQ^T += K^T dA^T
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(1, 128, 64, 1, 1);
      int gp = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int s = gp % kKStages, ab = gp % kABufs;
          if (!mbar_wait(bar(ctl->a_full[ab]), (gp / kABufs) & 1, wc) ||
              (it == 0 && jt > 0 && !mbar_wait(bar(ctl->dq_free), (jt - 1) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = sdesc_sw128(sbase + kOffK + s * kPairBytes, kBoxKV, 1024);
          const uint64_t dh = sdesc_sw128(sbase + kOffA + ab * 2 * kStgBytes, 8192, 1024);
          const uint64_t dl = sdesc_sw128(sbase + kOffA + ab * 2 * kStgBytes + kStgBytes, 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // 16 keys per step: +2048 bytes in both operands
            mma_f16_ss(tmem + kColQ, da + 128 * kk, dh + 128 * kk, idesc, (it > 0) || (kk > 0));
            mma_f16_ss(tmem + kColQ, da + 128 * kk, dl + 128 * kk, idesc, true);
          }
          mma_commit(bar(ctl->a_free[ab]));
          mma_commit(bar(ctl->k_empty[s]));
          if (it == npairs - 1) mma_commit(bar(ctl->dq_done));
        }
      }
      mma_commit(bar(ctl->drain_q));
      mbar_wait(bar(ctl->drain_q), 0, wc, false);
    }
  } else {
    // ------------------------------------------------------------ dA^T and the tile's dq
    const int g = (warp - kSoftmaxWarp0) >> 2;
    const int wq = warp & 3;
    const int t = 32 * wq + lane;                  // TMEM lane: key of the pair / channel
    const int c0 = 32 * g;
    const uint32_t gbar = 1 + g;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * wq) << 16);
    const float sl2 = dm.scale * 1.4426950408889634f;
    bool fail = false;
    int gp = 0;
    for (int jt = 0; jt < my_tiles; ++jt) {
      const int tau = tile_of(jt);
      if (named_vote_or(gbar, 128, fail)) break;
      const int bh = tau / dm.nb, i = tau - bh * dm.nb, b = bh / dm.H, h = bh % dm.H;
      const int32_t* L = list_of(tau);
      // the group's 32 columns of lse and D (rows past N: lse = +inf, so P = 0)
      if (wq == 0) {
        const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + c0 + lane;
        ctl->lse[g][c0 + lane] = __ldg(lse + at);
        ctl->dd[g][c0 + lane] = __ldg(Drow + at);
      }
      named_sync(gbar, 128);
      const float4* l4 = reinterpret_cast<const float4*>(&ctl->lse[g][c0]);
      const float4* d4 = reinterpret_cast<const float4*>(&ctl->dd[g][c0]);
      for (int it = 0; it < npairs; ++it, ++gp) {
        const int sb = gp & 1;
        const bool ok = !fail && mbar_wait(bar(ctl->s_full[sb]), (gp >> 1) & 1, wc);
        fail |= !ok;
        tc_fence_after();
        float x[32], dp[32];
        tmem_ld32(lane_addr + kColS + 64 * sb + c0, x);
        tmem_ld32(lane_addr + kColDP + 64 * sb + c0, dp);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(ctl->s_free[sb]));
        // this thread's key: block j1 (t < 64) or j2 (the padding half of an odd list is a
        // repeat of j1 and contributes nothing), valid below N
        const int e = 2 * it + (t >> 6);
        const int jb = e < kk_list ? __ldg(L + e) : -1;
        const bool valid = jb >= 0 && jb < dm.nb && jb * 64 + (t & 63) < dm.N;
        // the staging buffer was last read by the dQ^T products kABufs pairs back
        const int ab = gp % kABufs;
        if (gp >= kABufs && !fail) fail |= !mbar_wait(bar(ctl->a_free[ab]), ((gp - kABufs) / kABufs) & 1, wc);
        uint8_t* stg = base + kOffA + ab * 2 * kStgBytes;
        // eight columns at a time: one 16-byte chunk of dA^T hi and one of lo
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const float4 lv = l4[2 * c8 + h2], dv = d4[2 * c8 + h2];
            const int q0 = 8 * c8 + 4 * h2;
            const float p0 = valid ? ex2_approx(fmaf(x[q0], sl2, -lv.x)) : 0.f;
            const float p1 = valid ? ex2_approx(fmaf(x[q0 + 1], sl2, -lv.y)) : 0.f;
            const float p2 = valid ? ex2_approx(fmaf(x[q0 + 2], sl2, -lv.z)) : 0.f;
            const float p3 = valid ? ex2_approx(fmaf(x[q0 + 3], sl2, -lv.w)) : 0.f;
            split_bf16x2(p0 * (dp[q0] - dv.x), p1 * (dp[q0 + 1] - dv.y), hw[2 * h2], lw[2 * h2]);
            split_bf16x2(p2 * (dp[q0 + 2] - dv.z), p3 * (dp[q0 + 3] - dv.w), hw[2 * h2 + 1], lw[2 * h2 + 1]);
          }
          const uint32_t off = t * 128 + (((4 * g + c8) ^ (t & 7)) << 4);
          *reinterpret_cast<uint4*>(stg + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(stg + kStgBytes + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ctl->a_full[ab]));
      }
      // the tile's dQ^T: lane = channel t, this group's 32 query columns
      fail |= !mbar_wait(bar(ctl->dq_done), jt & 1, wc);
      if (!named_vote_or(gbar, 128, fail)) {
        tc_fence_after();
        float o[32];
        tmem_ld32(lane_addr + kColQ + c0, o);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ctl->dq_free));
        // all 32 loads first (the compiler cannot tell the rows apart), then the stores
        float* col = dq + (((size_t)b * dm.N + i * 64 + c0) * dm.H + h) * 128 + t;
        const size_t rs = (size_t)dm.H * 128;
        const int nv = min(32, dm.N - (i * 64 + c0));
        float cur[32];
#pragma unroll
        for (int qq = 0; qq < 32; ++qq) cur[qq] = qq < nv ? col[qq * rs] : 0.f;
#pragma unroll
        for (int qq = 0; qq < 32; ++qq)
          if (qq < nv) col[qq * rs] = fmaf(dm.scale, o[qq], cur[qq]);
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

// ------------------------------------------------------------------ dk, dv
// Key-major: a tile is one key block j, walked over the query blocks that kept it (the
// key-major lists), two at a time on the M side:
//   S  [128 q x 64 keys] = [Q_i1; Q_i2] K_j^T,   dP = [G_i1; G_i2] V_j^T     (K-major)
//   P = 2^(S scale log2(e) - lse_row),  dA = P (dP - D_row)  (a constant per TMEM lane)
//   dV^T [128 d x 64 keys] += [G_i1; G_i2]^T P,  dK^T += [Q_i1; Q_i2]^T dA   (the query
//   pairs read MN-major, P and dA as bf16 hi + lo), and dk += scale dK, dv += dV at the end.
// Roles: warp 0 = producer of K_j, V_j (one slot) and of the ring of query pairs (Q and
// dout); warp 1 = issuer of S and dP (and TMEM owner); warp 2 = issuer of dV^T, dK^T;
// warps 4-11 = two groups of four (thread t: query row t of the pair for S, dP; channel t
// for dK^T, dV^T; group g: key columns [32 g, 32 g + 32)).  An odd list's last pair repeats
// its first block with every row masked (lse = +inf).
namespace kv {
constexpr uint32_t kKVBytes = 2 * 128 * 64 * 2;             // K_j then V_j, 16 KB each
constexpr uint32_t kQGBytes = 2 * kPairBytes;               // a query pair of Q, then of dout
constexpr int kStages = 2;
constexpr uint32_t kOffKV = 0;
constexpr uint32_t kOffQG = kKVBytes;
constexpr uint32_t kOffStg = kOffQG + kStages * kQGBytes;   // P hi, P lo, dA hi, dA lo
constexpr uint32_t kOffCtl = kOffStg + 4 * kStgBytes;
constexpr uint32_t kColS = 0, kColDP = 128, kColK = 256, kColV = 320;
struct Ctl {
  uint64_t kv_full, kv_free, qg_full[kStages], qg_empty[kStages], s_full[2], s_free[2], a_full, a_free;
  uint64_t dkv_done, dkv_free, drain_s, drain_d;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = kOffCtl + sizeof(Ctl) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace kv

__global__ void __launch_bounds__(kThreads, 1) bwd_dkv_sm100_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Dims dm,
    const int* __restrict__ inv_off, const int* __restrict__ inv_idx, const float* __restrict__ lse,
    const float* __restrict__ Drow, float* __restrict__ dk, float* __restrict__ dv, int* __restrict__ status,
    unsigned long long limit_cycles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  kv::Ctl* ctl = reinterpret_cast<kv::Ctl*>(base + kv::kOffCtl);
  const uint32_t sbase = smem_addr(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = dm.nb * dm.B * dm.H;
  const int my_tiles = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };
  auto tile_of = [&](int jt) { return (int)blockIdx.x + jt * (int)gridDim.x; };
  // the tile's list of query blocks: [e0, e1) of the (b, h) row of inv_idx
  auto list_of = [&](int tau, int& e0, int& e1) {
    const int bh = tau / dm.nb, j = tau - bh * dm.nb;
    e0 = __ldg(inv_off + (size_t)bh * (dm.nb + 1) + j);
    e1 = __ldg(inv_off + (size_t)bh * (dm.nb + 1) + j + 1);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(ctl->kv_full), 1);
    mbar_init(bar(ctl->kv_free), 1);
    for (int s = 0; s < kv::kStages; ++s) {
      mbar_init(bar(ctl->qg_full[s]), 1);
      mbar_init(bar(ctl->qg_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ctl->s_full[s]), 1);
      mbar_init(bar(ctl->s_free[s]), kSoftmaxWarps);
    }
    mbar_init(bar(ctl->a_full), kSoftmaxWarps);
    mbar_init(bar(ctl->a_free), 1);
    mbar_init(bar(ctl->dkv_done), 1);
    mbar_init(bar(ctl->dkv_free), kSoftmaxWarps);
    mbar_init(bar(ctl->drain_s), 1);
    mbar_init(bar(ctl->drain_d), 1);
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtl wc{&ctl->abort, status, limit_cycles};

  if (warp == 0) {
    // ------------------------------------------------------------ K_j, V_j and the query pairs
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_g);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int gp = 0, nt = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        const int tau = tile_of(jt);
        int e0, e1;
        list_of(tau, e0, e1);
        if (e1 <= e0) continue;   // a key block no query block kept: nothing to add
        const int bh = tau / dm.nb, j = tau - bh * dm.nb, b = bh / dm.H, xh = (bh % dm.H) * 128;
        if (nt > 0 && !mbar_wait(bar(ctl->kv_free), (nt - 1) & 1, wc)) break;
        mbar_expect_tx(bar(ctl->kv_full), kv::kKVBytes);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sbase + kv::kOffKV + c * 8192, &tm_k, xh + 64 * c, j * 64, b, bar(ctl->kv_full));
          tma_load_3d(sbase + kv::kOffKV + 16384 + c * 8192, &tm_v, xh + 64 * c, j * 64, b, bar(ctl->kv_full));
        }
        ++nt;
        const int* lst = inv_idx + (size_t)bh * dm.nb * dm.k;
        for (int e = e0; e < e1; e += 2, ++gp) {
          const int s = gp % kv::kStages;
          if (gp >= kv::kStages && !mbar_wait(bar(ctl->qg_empty[s]), ((gp / kv::kStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          int i1 = __ldg(lst + e), i2 = e + 1 < e1 ? __ldg(lst + e + 1) : i1;
          if (i1 < 0 || i1 >= dm.nb || i2 < 0 || i2 >= dm.nb) {
            atomicCAS(status, 0, kDevBounds);
            i1 = i2 = 0;
          }
          const uint32_t st = sbase + kv::kOffQG + s * kv::kQGBytes;
          mbar_expect_tx(bar(ctl->qg_full[s]), kv::kQGBytes);
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(st + c * kBoxKV, &tm_q, xh + 64 * c, i1 * 64, b, bar(ctl->qg_full[s]));
            tma_load_3d(st + c * kBoxKV + 8192, &tm_q, xh + 64 * c, i2 * 64, b, bar(ctl->qg_full[s]));
            tma_load_3d(st + kPairBytes + c * kBoxKV, &tm_g, xh + 64 * c, i1 * 64, b, bar(ctl->qg_full[s]));
            tma_load_3d(st + kPairBytes + c * kBoxKV + 8192, &tm_g, xh + 64 * c, i2 * 64, b, bar(ctl->qg_full[s]));
          }
        }
      }
      if (nt > 0) mbar_wait(bar(ctl->kv_full), (nt - 1) & 1, wc, false);
      for (int x = (gp > kv::kStages ? gp - kv::kStages : 0); x < gp; ++x)
        mbar_wait(bar(ctl->qg_full[x % kv::kStages]), (x / kv::kStages) & 1, wc, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S and dP
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(1, 128, 64, 0, 0);
      int gp = 0, nt = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        int e0, e1;
        list_of(tile_of(jt), e0, e1);
        if (e1 <= e0) continue;
        if (!mbar_wait(bar(ctl->kv_full), nt & 1, wc)) break;
        ++nt;
        const uint64_t dkd = sdesc_sw128(sbase + kv::kOffKV, 16, 1024);
        const uint64_t dvd = sdesc_sw128(sbase + kv::kOffKV + 16384, 16, 1024);
        for (int e = e0; e < e1; e += 2, ++gp) {
          const int s = gp % kv::kStages, sb = gp & 1;
          if (!mbar_wait(bar(ctl->qg_full[s]), (gp / kv::kStages) & 1, wc) ||
              (gp >= 2 && !mbar_wait(bar(ctl->s_free[sb]), ((gp - 2) >> 1) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dq = sdesc_sw128(sbase + kv::kOffQG + s * kv::kQGBytes, 16, 1024);
          const uint64_t dg = sdesc_sw128(sbase + kv::kOffQG + s * kv::kQGBytes + kPairBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t ab = ((kk >> 2) * kBoxKV + (kk & 3) * 32) >> 4, bb = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
            mma_f16_ss(tmem + kv::kColS + 64 * sb, dq + ab, dkd + bb, idesc, kk > 0);
            mma_f16_ss(tmem + kv::kColDP + 64 * sb, dg + ab, dvd + bb, idesc, kk > 0);
          }
          mma_commit(bar(ctl->s_full[sb]));
        }
        if (ok) mma_commit(bar(ctl->kv_free));   // K_j and V_j are read
      }
      mma_commit(bar(ctl->drain_s));
      mbar_wait(bar(ctl->drain_s), 0, wc, false);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ dV^T, dK^T
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(1, 128, 64, 1, 1);
      int gp = 0, nt = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        int e0, e1;
        list_of(tile_of(jt), e0, e1);
        if (e1 <= e0) continue;
        for (int e = e0; e < e1; e += 2, ++gp) {
          const int s = gp % kv::kStages;
          const bool first = e == e0;
          if (!mbar_wait(bar(ctl->a_full), gp & 1, wc) ||
              (first && nt > 0 && !mbar_wait(bar(ctl->dkv_free), (nt - 1) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dq = sdesc_sw128(sbase + kv::kOffQG + s * kv::kQGBytes, kBoxKV, 1024);
          const uint64_t dg = sdesc_sw128(sbase + kv::kOffQG + s * kv::kQGBytes + kPairBytes, kBoxKV, 1024);
          const uint32_t stg = sbase + kv::kOffStg;
          const uint64_t ph = sdesc_sw128(stg, 8192, 1024), pl = sdesc_sw128(stg + kStgBytes, 8192, 1024);
          const uint64_t ah = sdesc_sw128(stg + 2 * kStgBytes, 8192, 1024);
          const uint64_t al = sdesc_sw128(stg + 3 * kStgBytes, 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // 16 queries per step: +2048 bytes in every operand
            mma_f16_ss(tmem + kv::kColV, dg + 128 * kk, ph + 128 * kk, idesc, !first || kk > 0);
            mma_f16_ss(tmem + kv::kColV, dg + 128 * kk, pl + 128 * kk, idesc, true);
            mma_f16_ss(tmem + kv::kColK, dq + 128 * kk, ah + 128 * kk, idesc, !first || kk > 0);
            mma_f16_ss(tmem + kv::kColK, dq + 128 * kk, al + 128 * kk, idesc, true);
          }
          mma_commit(bar(ctl->a_free));
          mma_commit(bar(ctl->qg_empty[s]));
          if (e + 2 >= e1) mma_commit(bar(ctl->dkv_done));
        }
        ++nt;
      }
      mma_commit(bar(ctl->drain_d));
      mbar_wait(bar(ctl->drain_d), 0, wc, false);
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ P, dA and the tile's dk, dv
    const int g = (warp - kSoftmaxWarp0) >> 2;
    const int wq = warp & 3;
    const int t = 32 * wq + lane;                  // TMEM lane: query row of the pair / channel
    const int c0 = 32 * g;
    const uint32_t gbar = 1 + g;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * wq) << 16);
    const float sl2 = dm.scale * 1.4426950408889634f;
    bool fail = false;
    int gp = 0, nt = 0;
    for (int jt = 0; jt < my_tiles; ++jt) {
      const int tau = tile_of(jt);
      int e0, e1;
      list_of(tau, e0, e1);
      if (e1 <= e0) continue;
      if (named_vote_or(gbar, 128, fail)) break;
      const int bh = tau / dm.nb, j = tau - bh * dm.nb, b = bh / dm.H, h = bh % dm.H;
      const int* lst = inv_idx + (size_t)bh * dm.nb * dm.k;
      const int kvalid = min(64, dm.N - j * 64) - c0;   // this group's valid key columns
      for (int e = e0; e < e1; e += 2, ++gp) {
        const int sb = gp & 1;
        // this thread's query row: block i1 (t < 64) or i2 (the padding half of an odd
        // list is masked), its lse and D
        const int ee = e + (t >> 6);
        float lr = INFINITY, dr = 0.f;
        if (ee < e1) {
          const int ib = __ldg(lst + ee);
          if (ib >= 0 && ib < dm.nb) {
            const size_t at = (size_t)bh * dm.nb * 64 + (size_t)ib * 64 + (t & 63);
            lr = __ldg(lse + at);
            dr = __ldg(Drow + at);
          }
        }
        const bool ok = !fail && mbar_wait(bar(ctl->s_full[sb]), (gp >> 1) & 1, wc);
        fail |= !ok;
        tc_fence_after();
        float x[32], dp[32];
        tmem_ld32(lane_addr + kv::kColS + 64 * sb + c0, x);
        tmem_ld32(lane_addr + kv::kColDP + 64 * sb + c0, dp);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(ctl->s_free[sb]));
        // the staging was last read by the previous step's dV^T, dK^T products
        if (gp >= 1 && !fail) fail |= !mbar_wait(bar(ctl->a_free), (gp - 1) & 1, wc);
        uint8_t* stg = base + kv::kOffStg;
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint32_t ph[4], pl[4], ah[4], al[4];
#pragma unroll
          for (int w2 = 0; w2 < 4; ++w2) {
            const int k0 = 8 * c8 + 2 * w2;
            const float p0 = k0 < kvalid ? ex2_approx(fmaf(x[k0], sl2, -lr)) : 0.f;
            const float p1 = k0 + 1 < kvalid ? ex2_approx(fmaf(x[k0 + 1], sl2, -lr)) : 0.f;
            split_bf16x2(p0, p1, ph[w2], pl[w2]);
            split_bf16x2(p0 * (dp[k0] - dr), p1 * (dp[k0 + 1] - dr), ah[w2], al[w2]);
          }
          const uint32_t off = t * 128 + (((4 * g + c8) ^ (t & 7)) << 4);
          *reinterpret_cast<uint4*>(stg + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
          *reinterpret_cast<uint4*>(stg + kStgBytes + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
          *reinterpret_cast<uint4*>(stg + 2 * kStgBytes + off) = make_uint4(ah[0], ah[1], ah[2], ah[3]);
          *reinterpret_cast<uint4*>(stg + 3 * kStgBytes + off) = make_uint4(al[0], al[1], al[2], al[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ctl->a_full));
      }
      // the tile's dK^T, dV^T: lane = channel t, this group's 32 key columns
      fail |= !mbar_wait(bar(ctl->dkv_done), nt & 1, wc);
      ++nt;
      if (!named_vote_or(gbar, 128, fail)) {
        const size_t rs = (size_t)dm.H * 128;
        const size_t row0 = (((size_t)b * dm.N + j * 64 + c0) * dm.H + h) * 128 + t;
        // dK^T then dV^T, each: the TMEM columns, all loads of the rows, then the stores
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          tc_fence_after();
          float a[32];
          tmem_ld32(lane_addr + (which ? kv::kColV : kv::kColK) + c0, a);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (which == 1 && lane == 0) mbar_arrive(bar(ctl->dkv_free));
          float* col = (which ? dv : dk) + row0;
          const float f = which ? 1.f : dm.scale;
          float u[32];
#pragma unroll
          for (int kq = 0; kq < 32; ++kq) u[kq] = kq < kvalid ? col[kq * rs] : 0.f;
#pragma unroll
          for (int kq = 0; kq < 32; ++kq)
            if (kq < kvalid) col[kq * rs] = fmaf(f, a[kq], u[kq]);
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

// ------------------------------------------------------------------ row statistics
// Per query block i, over the pairs of its kept key blocks (as for dq):
//   S^T [128 keys x 64 q] = [K_j1; K_j2] Q_i^T,   dP^T = [V_j1; V_j2] dout_i^T
// and per query column c: m_c = the first pair's column max of s = S^T scale log2(e) over
// valid keys, p = 2^(s - m_c), l_c = sum p, e_c = sum p dP over every valid key of the list;
// lse_c = m_c + log2(l_c) (log2 units), D_c = e_c / l_c = dout . O_sparse.  Each thread keeps
// its TMEM lane's (its key's) partial sums for its group's 32 columns; one reduction per tile
// (a warp reduce-scatter, then the four warps in a fixed order).  A tile where some p would
// exceed 2^64 (a key far above the first pair's max) is listed for the warp-level kernel,
// which rescales block by block.
// Roles (384 threads): warp 0 = TMA producer of Q and dout (one slot) and the K ring; warp 1 =
// issuer of S^T and dP^T and TMEM owner; warp 3 = the V ring; warps 4-11 = two groups of four
// over query columns [32 g, 32 g + 32).
namespace rsx {
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTmemCols = 256;   // S^T (0, 64), dP^T (128, 192)
constexpr uint32_t kOffQG = 0;        // Q (16 KB) then dout (16 KB)
constexpr uint32_t kOffK = 32768;
constexpr uint32_t kOffV = kOffK + kKStages * kPairBytes;
constexpr uint32_t kOffCtl = kOffV + kVStages * kPairBytes;

struct Ctl {
  uint64_t qg_full, qg_free, k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_free[2], drain;
  uint32_t tmem_base;
  int abort;
  alignas(16) float red[2][2][4][32];   // per group: l and e (or the max), per warp, per column
  alignas(16) float mcol[2][32];        // per group: the tile's column offsets
};
constexpr size_t kSmemBytes = kOffCtl + sizeof(Ctl) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace rsx

__global__ void __launch_bounds__(kThreads, 1) bwd_rowstats_sm100_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_g,
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, Dims dm,
    const int32_t* __restrict__ col_idx, float* __restrict__ lse, float* __restrict__ Drow, int* __restrict__ redo,
    int* __restrict__ status, unsigned long long limit_cycles) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  rsx::Ctl* ctl = reinterpret_cast<rsx::Ctl*>(base + rsx::kOffCtl);
  const uint32_t sbase = smem_addr(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = dm.nb * dm.B * dm.H;
  const int kk_list = dm.k, npairs = (kk_list + 1) >> 1;
  const int my_tiles = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };
  auto tile_of = [&](int jt) { return (int)blockIdx.x + jt * (int)gridDim.x; };
  auto list_of = [&](int tau) { return col_idx + (size_t)tau * kk_list; };

  if (threadIdx.x == 0) {
    mbar_init(bar(ctl->qg_full), 1);
    mbar_init(bar(ctl->qg_free), 1);
    for (int s = 0; s < rsx::kKStages; ++s) {
      mbar_init(bar(ctl->k_full[s]), 1);
      mbar_init(bar(ctl->k_empty[s]), 1);
    }
    for (int s = 0; s < rsx::kVStages; ++s) {
      mbar_init(bar(ctl->v_full[s]), 1);
      mbar_init(bar(ctl->v_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ctl->s_full[s]), 1);
      mbar_init(bar(ctl->s_free[s]), kSoftmaxWarps);
    }
    mbar_init(bar(ctl->drain), 1);
    ctl->abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(&ctl->tmem_base), rsx::kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtl wc{&ctl->abort, status, limit_cycles};
  auto pair_blocks = [&](const int32_t* L, int it, int& j1, int& j2) {
    j1 = __ldg(L + 2 * it);
    j2 = (2 * it + 1 < kk_list) ? __ldg(L + 2 * it + 1) : j1;
    if (j1 < 0 || j1 >= dm.nb || j2 < 0 || j2 >= dm.nb) {
      atomicCAS(status, 0, kDevBounds);
      j1 = j2 = 0;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ Q, dout and the K ring
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_g);
      tma_prefetch_desc(&tm_k);
      int gp = 0, nqg = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        const int tau = tile_of(jt);
        const int bh = tau / dm.nb, i = tau - bh * dm.nb, b = bh / dm.H, xh = (bh % dm.H) * 128;
        const int32_t* L = list_of(tau);
        if (jt > 0 && !mbar_wait(bar(ctl->qg_free), (jt - 1) & 1, wc)) break;
        mbar_expect_tx(bar(ctl->qg_full), 32768);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sbase + rsx::kOffQG + c * 8192, &tm_q, xh + 64 * c, i * 64, b, bar(ctl->qg_full));
          tma_load_3d(sbase + rsx::kOffQG + 16384 + c * 8192, &tm_g, xh + 64 * c, i * 64, b, bar(ctl->qg_full));
        }
        ++nqg;
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int s = gp % rsx::kKStages;
          if (gp >= rsx::kKStages && !mbar_wait(bar(ctl->k_empty[s]), ((gp / rsx::kKStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          int j1, j2;
          pair_blocks(L, it, j1, j2);
          const uint32_t st = sbase + rsx::kOffK + s * kPairBytes;
          mbar_expect_tx(bar(ctl->k_full[s]), kPairBytes);
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(st + c * kBoxKV, &tm_k, xh + 64 * c, j1 * 64, b, bar(ctl->k_full[s]));
            tma_load_3d(st + c * kBoxKV + 8192, &tm_k, xh + 64 * c, j2 * 64, b, bar(ctl->k_full[s]));
          }
        }
      }
      if (nqg > 0) mbar_wait(bar(ctl->qg_full), (nqg - 1) & 1, wc, false);
      for (int x = (gp > rsx::kKStages ? gp - rsx::kKStages : 0); x < gp; ++x)
        mbar_wait(bar(ctl->k_full[x % rsx::kKStages]), (x / rsx::kKStages) & 1, wc, false);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ the V ring
    if (lane == 0) {
      tma_prefetch_desc(&tm_v);
      int gp = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        const int tau = tile_of(jt);
        const int bh = tau / dm.nb, b = bh / dm.H, xh = (bh % dm.H) * 128;
        const int32_t* L = list_of(tau);
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int s = gp % rsx::kVStages;
          if (gp >= rsx::kVStages && !mbar_wait(bar(ctl->v_empty[s]), ((gp / rsx::kVStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          int j1, j2;
          pair_blocks(L, it, j1, j2);
          const uint32_t st = sbase + rsx::kOffV + s * kPairBytes;
          mbar_expect_tx(bar(ctl->v_full[s]), kPairBytes);
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(st + c * kBoxKV, &tm_v, xh + 64 * c, j1 * 64, b, bar(ctl->v_full[s]));
            tma_load_3d(st + c * kBoxKV + 8192, &tm_v, xh + 64 * c, j2 * 64, b, bar(ctl->v_full[s]));
          }
        }
      }
      for (int x = (gp > rsx::kVStages ? gp - rsx::kVStages : 0); x < gp; ++x)
        mbar_wait(bar(ctl->v_full[x % rsx::kVStages]), (x / rsx::kVStages) & 1, wc, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S^T and dP^T
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(1, 128, 64, 0, 0);
      int gp = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        if (!mbar_wait(bar(ctl->qg_full), jt & 1, wc)) break;
        const uint64_t dqd = sdesc_sw128(sbase + rsx::kOffQG, 16, 1024);
        const uint64_t dgd = sdesc_sw128(sbase + rsx::kOffQG + 16384, 16, 1024);
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int ks = gp % rsx::kKStages, vs = gp % rsx::kVStages, sb = gp & 1;
          if (!mbar_wait(bar(ctl->k_full[ks]), (gp / rsx::kKStages) & 1, wc) ||
              !mbar_wait(bar(ctl->v_full[vs]), (gp / rsx::kVStages) & 1, wc) ||
              (gp >= 2 && !mbar_wait(bar(ctl->s_free[sb]), ((gp - 2) >> 1) & 1, wc))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dk = sdesc_sw128(sbase + rsx::kOffK + ks * kPairBytes, 16, 1024);
          const uint64_t dv = sdesc_sw128(sbase + rsx::kOffV + vs * kPairBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {   // K-step offsets: 32 B inside a box, boxes 16 KB / 8 KB apart
            const uint32_t ab = ((kk >> 2) * kBoxKV + (kk & 3) * 32) >> 4, bb = ((kk >> 2) * 8192 + (kk & 3) * 32) >> 4;
            mma_f16_ss(tmem + kColS + 64 * sb, dk + ab, dqd + bb, idesc, kk > 0);
            mma_f16_ss(tmem + kColDP + 64 * sb, dv + ab, dgd + bb, idesc, kk > 0);
          }
          mma_commit(bar(ctl->s_full[sb]));
          mma_commit(bar(ctl->k_empty[ks]));
          mma_commit(bar(ctl->v_empty[vs]));
        }
        if (ok) mma_commit(bar(ctl->qg_free));   // this tile's Q and dout are read
      }
      mma_commit(bar(ctl->drain));
      mbar_wait(bar(ctl->drain), 0, wc, false);
    }
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ the statistics
    const int g = (warp - kSoftmaxWarp0) >> 2;
    const int wq = warp & 3;
    const int t = 32 * wq + lane;                  // TMEM lane: key t of the pair
    const int c0 = 32 * g;
    const uint32_t gbar = 1 + g;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * wq) << 16);
    const float sl2 = dm.scale * 1.4426950408889634f;
    bool fail = false;
    int gp = 0;
    for (int jt = 0; jt < my_tiles; ++jt) {
      const int tau = tile_of(jt);
      const int bh = tau / dm.nb, i = tau - bh * dm.nb;
      const int32_t* L = list_of(tau);
      float m[32], ls[32], es[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        ls[c] = 0.f;
        es[c] = 0.f;
      }
      bool over = false;
      for (int it = 0; it < npairs; ++it, ++gp) {
        const int sb = gp & 1;
        const bool ok = !fail && mbar_wait(bar(ctl->s_full[sb]), (gp >> 1) & 1, wc);
        fail |= !ok;
        tc_fence_after();
        const int e = 2 * it + (t >> 6);
        const int jb = e < kk_list ? __ldg(L + e) : -1;
        const bool valid = jb >= 0 && jb < dm.nb && jb * 64 + (t & 63) < dm.N;
        if (it == 0) {
          // the tile's column offsets: the max of s over the first pair's valid keys
          float x[32];
          tmem_ld32(lane_addr + kColS + 64 * sb + c0, x);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) x[c] = valid ? x[c] * sl2 : -INFINITY;
          ctl->red[g][0][wq][lane] = reduce_scatter32<true>(x, lane);
          named_sync(gbar, 128);
          if (wq == 0)
            ctl->mcol[g][lane] = fmaxf(fmaxf(ctl->red[g][0][0][lane], ctl->red[g][0][1][lane]),
                                       fmaxf(ctl->red[g][0][2][lane], ctl->red[g][0][3][lane]));
          named_sync(gbar, 128);
          const float4* m4 = reinterpret_cast<const float4*>(ctl->mcol[g]);
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4) {
            const float4 v4 = m4[c4];
            m[4 * c4] = v4.x;
            m[4 * c4 + 1] = v4.y;
            m[4 * c4 + 2] = v4.z;
            m[4 * c4 + 3] = v4.w;
          }
        }
        // sixteen columns at a time: p = 2^(s - m), l += p, e += p dP
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float x[16], dp[16];
          tmem_ld16(lane_addr + kColS + 64 * sb + c0 + 16 * hh, x);
          tmem_ld16(lane_addr + kColDP + 64 * sb + c0 + 16 * hh, dp);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const float a = fmaf(x[c], sl2, -m[16 * hh + c]);
            over |= valid && a > 64.f;
            const float p = valid ? ex2_approx(a) : 0.f;
            ls[16 * hh + c] += p;
            es[16 * hh + c] = fmaf(p, dp[c], es[16 * hh + c]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(ctl->s_free[sb]));
      }
      // the tile's statistics: l and e summed over the 128 keys of every pair, in a fixed order.
      // Both votes span the two groups: they leave together on a failed wait, and a tile with
      // an overflowing p in either group is listed once and written by neither.
      if (named_vote_or(3, 256, fail)) break;
      const bool bad = named_vote_or(3, 256, over);
      const float lw = reduce_scatter32<false>(ls, lane), ew = reduce_scatter32<false>(es, lane);
      ctl->red[g][0][wq][lane] = lw;
      ctl->red[g][1][wq][lane] = ew;
      named_sync(gbar, 128);
      if (wq == 0) {
        const float lt = ((ctl->red[g][0][0][lane] + ctl->red[g][0][1][lane]) + ctl->red[g][0][2][lane]) +
                         ctl->red[g][0][3][lane];
        const float et = ((ctl->red[g][1][0][lane] + ctl->red[g][1][1][lane]) + ctl->red[g][1][2][lane]) +
                         ctl->red[g][1][3][lane];
        const int n = i * 64 + c0 + lane;
        const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + c0 + lane;
        if (!bad) {
          lse[at] = n < dm.N ? ctl->mcol[g][lane] + log2f(lt) : INFINITY;
          Drow[at] = n < dm.N ? et / lt : 0.f;
        } else if (g == 0 && lane == 0) {
          redo[1 + atomicAdd(redo, 1)] = tau;      // at most once per tile: the list holds every tile
        }
      }
      named_sync(gbar, 128);                         // red and mcol are rewritten next tile
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, rsx::kTmemCols);
  }
}

}  // namespace

cudaError_t launch_bwd_rowstats_sm100(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                                     const Workspace& ws, const BwdWorkspace& bw, cudaStream_t st) {
  CUtensorMap tq, tg, tk, tv;
  if (!make_act_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dout, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, dm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(bw.redo, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_rowstats_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)rsx::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long ntiles = (long long)dm.nb * dm.B * dm.H;
  dim3 grid((unsigned)(ntiles < sms ? ntiles : sms));
  // Wait limit in SM clock cycles: 2e9 cycles is 1 s at 2 GHz.
  bwd_rowstats_sm100_kernel<<<grid, kThreads, rsx::kSmemBytes, st>>>(tq, tg, tk, tv, dm, ws.col_idx, bw.lse, bw.Drow,
                                                                    bw.redo, ws.status, 2000000000ull);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq_sm100(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                                const Workspace& ws, const BwdWorkspace& bw, float* dq, cudaStream_t st) {
  CUtensorMap tq, tg, tk, tv;
  if (!make_act_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dout, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, dm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long ntiles = (long long)dm.nb * dm.B * dm.H;
  dim3 grid((unsigned)(ntiles < sms ? ntiles : sms));
  // Wait limit in SM clock cycles: 2e9 cycles is 1 s at 2 GHz.
  bwd_dq_sm100_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tg, tk, tv, dm, ws.col_idx, bw.lse, bw.Drow, dq,
                                                          ws.status, 2000000000ull);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkv_sm100(const Dims& dm, const void* q, const void* k, const void* v, const void* dout,
                                 const Workspace& ws, const BwdWorkspace& bw, float* dk, float* dv, cudaStream_t st) {
  CUtensorMap tq, tg, tk, tv;
  if (!make_act_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tg, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dout, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, dm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(bwd_dkv_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kv::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long ntiles = (long long)dm.nb * dm.B * dm.H;
  dim3 grid((unsigned)(ntiles < sms ? ntiles : sms));
  bwd_dkv_sm100_kernel<<<grid, kThreads, kv::kSmemBytes, st>>>(tq, tg, tk, tv, dm, bw.inv_off, bw.inv_idx, bw.lse,
                                                               bw.Drow, dk, dv, ws.status, 2000000000ull);
  return cudaGetLastError();
}

}  // namespace rola
