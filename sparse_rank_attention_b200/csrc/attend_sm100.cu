// Sparse branch + fused linear epilogue + combination of RoLA (steps 3-5) on the sm_100a
// tensor cores (tcgen05 + TMEM + TMA), bf16 inputs, head dim 128.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (block-sparse softmax branch plus a
// low-rank linear branch with rotary positions); README sparse-finetuning section
// (proj_q, and the gate read here as a gain g per head or per token and head).
//
// Why the transposed tile: tcgen05.mma needs M = 128 rows for full rate, but a query
// block has 64 tokens and every query block keeps its own key blocks.  So the M side
// is taken by KEYS: each step multiplies one query block (N = 64) with a pair of its
// kept key blocks (M = 128 keys), and every MMA row does useful work:
//   S^T [128 keys x 64 q]  = [K_j1; K_j2] Q_i^T            (bf16, K-major A and B)
//   O^T [128 d x 64 q]    += [V_j1; V_j2]^T P^T            (fp16, MN-major A and B)
// The softmax runs in two independent groups of four warps; group g owns the query
// columns [32g, 32g + 32) of S^T and O^T.  Thread t of a group owns TMEM lane t: key t of
// the pair for S^T and channel d = t for O^T.  The softmax max is per query (a TMEM
// column spread over 128 lanes), so it is kept lazily.  Fast pass: each query's exponent
// offset m is the exact column max of the tile's first pair and stays fixed; a tile whose
// per-thread partial row sums (which bound every P it made) pass the range of P (2^15 for
// fp16, 2^8 for e4m3) is listed for the careful pass, a second launch over the listed
// tiles in which m moves whenever a score exceeds it by more than 8 (log2 units), by an
// exact per-query max across the 128 lanes, rescaling the group's O^T columns and sums.
// Per-query sums l stay per thread (partials over that thread's keys) until the end.
//
// Roles (384 threads, one role per warp so that a sleeping wait never holds another
// role back): warp 0 = TMA producer of Q and the K ring, warp 1 = Q K^T issuer (and TMEM
// owner), warp 2 = P V issuer, warp 3 = producer of the epilogue operands and the V
// ring, warps 4-11 = the two softmax groups (two softmax warps per SM sub-partition).
// K and V pairs are double-buffered (K freed when its QK is done, V after its PV), S^T
// triple-buffered in TMEM, so QK runs up to two pairs ahead of the softmax warps.
//
// Epilogue (per query block): num^T = S_h^T (R u)^T on the tensor cores, with S_h and
// the rotated query features R u each as bf16 hi + lo (three MMAs); both operands, and
// g/den per query, arrive as ready-made shared-memory images (state reduction and the
// query-feature pre-pass write them) with one bulk copy issued in the prologue.
// out = O/l + (g/den) num, staged in shared memory and written by TMA stores, one per
// query group and channel half (rows past N are clipped by the tensor map).
//
// Every mbarrier wait is bounded (ROLA_ERR_DEVICE_TIMEOUT); on a timeout all roles
// leave their loops, in-flight MMAs and TMA copies are drained and TMEM is freed.
#include <climits>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp8.h>

#include "rola_internal.cuh"
#include "sm100_ptx.cuh"
#include "softmax_exp.cuh"

namespace rola {
namespace {

using namespace sm100;

// Softmax groups of four warps.  Four groups of 16 columns (640 threads, 96 registers)
// measured no faster than two of 32: a warp's per-pair chain, not the issue rate, sets
// the softmax side's pace.
constexpr int kGroups = 2;
constexpr int kCols = 64 / kGroups;            // query columns of a group
constexpr int kThreads = 128 + 128 * kGroups;
constexpr int kSoftmaxWarp0 = 4;  // group g = warps 4 + 4g .. 7 + 4g: query columns [kCols g, kCols (g + 1))
constexpr int kSoftmaxWarps = 4 * kGroups;
static_assert(kGroups == 2 || kGroups == 4, "softmax groups");
constexpr unsigned kGroupOffsetNs = 400;
constexpr uint32_t kTmemCols = 512;
constexpr int kSBufs = 3;         // S^T buffers at columns 0, 64, 128
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 192;   // O^T
constexpr uint32_t kColNum = 256; // epilogue: num^T (its own columns: the next tile's S^T
                                  // are computed while a tile's epilogue runs)
constexpr uint32_t kColM = 384;   // negated exponent offsets -m: every lane holds the 64
                                  // queries' -m, read with S^T (tensor memory, not shared
                                  // memory) and used as the addend of x = s * scale - m

constexpr int kMaxStages = 4;              // ring-depth bound (barrier arrays)

// Shared-memory geometry.  16-bit path: a tile row of 128 channels is two 128-byte
// swizzle boxes (channels 0-63, 64-127); fp8 path: one 128-byte box.  P^T is fp16 in
// 128-byte rows (SW128) or e4m3 in 64-byte rows (SW64).
template <bool FP8>
struct Geo {
  static constexpr uint32_t kEl = FP8 ? 1 : 2;                   // bytes per q/k/v element
  static constexpr uint32_t kQBytes = 64 * 128 * kEl;             // Q tile
  static constexpr uint32_t kPairBytes = 128 * 128 * kEl;         // K or V pair
  static constexpr uint32_t kBoxKV = FP8 ? 16384 : 16384;         // channel-box stride in a pair
  static constexpr uint32_t kPBytes = FP8 ? 8192 : 16384;         // one P^T buffer
  // K pairs are freed as soon as their QK is done, V pairs after their PV.  A pair's copy
  // from L2 takes longer than a pair's work, so the rings are as deep as shared memory
  // allows: 2 + 2 of 32 KB for 16-bit operands, 4 + 4 of 16 KB for e4m3.
  static constexpr int kKStages = FP8 ? 4 : 2;
  static constexpr int kVStages = FP8 ? 4 : 2;
  static constexpr uint32_t kOffQ = 0;                             // 2 Q slots of 16 KB (each
                                                                   // also its tile's out staging)
  static constexpr uint32_t kOffK = 32768;                         // K ring (1024-aligned)
  static constexpr uint32_t kOffV = kOffK + kKStages * kPairBytes;  // V ring
  static constexpr uint32_t kOffP = kOffV + kVStages * kPairBytes;  // 2 x P^T (also out staging)
  static constexpr uint32_t kOffSimg = kOffP + 2 * 16384;           // S_h^T hi | lo (<= 16 KB)
  static constexpr uint32_t kOffUimg = kOffSimg + 16384;            // (R u)^T hi | lo (<= 8 KB)
  static constexpr uint32_t kOffGden = kOffUimg + 8192;             // g/den per query (256 B)
  static constexpr uint32_t kOffCtl = kOffGden + 256;
};

struct Ctl {
  uint64_t q_full[2], q_free[2], k_full[kMaxStages], k_empty[kMaxStages], v_full[kMaxStages], v_empty[kMaxStages];
  uint64_t s_full[kSBufs], s_empty[kSBufs], p_full[2], pv_done[2], ep_full, ep_bar, drain_bar, stall_bar;
  uint32_t tmem_base;
  int abort;
  alignas(16) float fac[64];
  alignas(16) float red[kGroups][4][32];   // per query group: per-warp partial reductions
  alignas(16) float linv[64];
  float vref[kGroups][4];  // fp8: per-warp partial max of the kept blocks' V scales
  int emax[kGroups][4], emin[kGroups][4];  // 16-bit path: per-warp range of the kept blocks' v exponents
};
template <bool FP8>
constexpr size_t smem_bytes() { return Geo<FP8>::kOffCtl + sizeof(Ctl) + 1024; }


// Writes NC 16-byte chunks (4 packed words each), logical chunks c0 .. c0 + NC - 1 of
// row `row` of a SW128 tile (128-byte rows): chunk c goes to position c ^ (row % 8).
template <int NC>
__device__ __forceinline__ void st_chunks_sw128(uint8_t* tile, int row, int c0, const uint32_t* w) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    uint4 v = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    *reinterpret_cast<uint4*>(tile + row * 128 + (((c0 + c) ^ (row & 7)) << 4)) = v;
  }
}

// The same for a SW64 tile (64-byte rows): chunk c goes to position c ^ ((row / 2) % 4).
template <int NC>
__device__ __forceinline__ void st_chunks_sw64(uint8_t* tile, int row, int c0, const uint32_t* w) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    uint4 v = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    *reinterpret_cast<uint4*>(tile + row * 64 + (((c0 + c) ^ ((row >> 1) & 3)) << 4)) = v;
  }
}

// kCols consecutive fp32 columns of this thread's TMEM lane (warp-wide).
__device__ __forceinline__ void tmem_ldc(uint32_t taddr, float* v) {
  if constexpr (kCols == 32) tmem_ld32(taddr, v); else tmem_ld16(taddr, v);
}
__device__ __forceinline__ void tmem_stc(uint32_t taddr, const float* v) {
  if constexpr (kCols == 32) tmem_st32(taddr, v); else tmem_st16(taddr, v);
}

// Reduce kCols per-lane values over the warp into red[0 .. kCols): 32 columns with lane l
// writing entry l (31 shuffles); 16 columns by four halving steps and a last exchange,
// lane l then holding entry l / 2 (16 shuffles).
template <bool kMax>
__device__ __forceinline__ void reduce_cols(float* red, const float* x, int lane) {
  if constexpr (kCols == 32) {
    red[lane] = reduce_scatter32<kMax>(x, lane);
  } else {
    const unsigned full = 0xffffffffu;
    auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
    float b[8], c[4], d[2];
    const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4, h2 = lane & 2;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float mine = h16 ? x[8 + e] : x[e], send = h16 ? x[e] : x[8 + e];
      b[e] = op(mine, __shfl_xor_sync(full, send, 16));
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float mine = h8 ? b[4 + e] : b[e], send = h8 ? b[e] : b[4 + e];
      c[e] = op(mine, __shfl_xor_sync(full, send, 8));
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float mine = h4 ? c[2 + e] : c[e], send = h4 ? c[e] : c[2 + e];
      d[e] = op(mine, __shfl_xor_sync(full, send, 4));
    }
    const float mine = h2 ? d[1] : d[0], send = h2 ? d[0] : d[1];
    float r = op(mine, __shfl_xor_sync(full, send, 2));
    r = op(r, __shfl_xor_sync(full, r, 1));
    if (!(lane & 1)) red[lane >> 1] = r;
  }
}

template <int RK, bool FP8, bool CAREFUL>
__global__ void __launch_bounds__(kThreads, 1) attend_sm100_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out, Dims dm,
    const int32_t* __restrict__ col_idx, const uint8_t* __restrict__ simg,
    const uint8_t* __restrict__ uimg, const float* __restrict__ gden,
    const float* __restrict__ sq, const float* __restrict__ sk, const float* __restrict__ sv,
    const int* __restrict__ vexp, int* __restrict__ status, int* __restrict__ redo, int debug_flags,
    unsigned long long limit_cycles,
    unsigned long long debug_limit_cycles) {
  using G = Geo<FP8>;
  constexpr int kKStages = G::kKStages, kVStages = G::kVStages;
  static_assert(kKStages <= kMaxStages && kVStages <= kMaxStages, "ring depth");
  constexpr uint32_t kOffQ = G::kOffQ, kOffK = G::kOffK, kOffV = G::kOffV, kOffP = G::kOffP;
  constexpr uint32_t kOffSimg = G::kOffSimg, kOffUimg = G::kOffUimg, kOffGden = G::kOffGden;
  constexpr uint32_t kOffCtl = G::kOffCtl, kPairBytes = G::kPairBytes, kBoxKV = G::kBoxKV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(base + kOffCtl);
  const uint32_t sbase = smem_addr(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tile = (b, h, query block i).  The fast pass walks all tiles; the careful pass walks
  // the tiles the fast pass listed in redo[1..redo[0]] (each listed at most twice).
  const int ntiles_all = dm.nb * dm.B * dm.H;
  const int ntiles = CAREFUL ? min(*reinterpret_cast<volatile int*>(redo), 2 * ntiles_all) : ntiles_all;
  auto tile_at = [&](int idx) { return CAREFUL ? __ldg(redo + 1 + idx) : idx; };
  const int kk_list = dm.k;
  const int npairs = (kk_list + 1) >> 1;
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };
  // tile tau -> (b*H + h, i): consecutive tiles are consecutive query blocks of one head,
  // so the CTAs working at one time share that head's key/value blocks in L2
  auto tile_bh = [&](int tau) { return tau / dm.nb; };
  auto list_of = [&](int tau) { return col_idx + (size_t)tau * kk_list; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ctl->q_full[s]), 1);
      mbar_init(bar(ctl->q_free[s]), kGroups);           // one arrive per softmax group
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(ctl->k_full[s]), 1);
      mbar_init(bar(ctl->k_empty[s]), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(ctl->v_full[s]), 1);
      mbar_init(bar(ctl->v_empty[s]), 1);
    }
    for (int s = 0; s < kSBufs; ++s) {
      mbar_init(bar(ctl->s_full[s]), 1);
      mbar_init(bar(ctl->s_empty[s]), kSoftmaxWarps);   // one arrive per softmax warp
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ctl->p_full[s]), kSoftmaxWarps);
      mbar_init(bar(ctl->pv_done[s]), 1);
    }
    mbar_init(bar(ctl->ep_full), 1);
    mbar_init(bar(ctl->ep_bar), 1);
    mbar_init(bar(ctl->drain_bar), 2);
    mbar_init(bar(ctl->stall_bar), 1);
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
  // The producers read a pair's key blocks before they wait for its ring slot (the list
  // load then overlaps the wait) and check them after.
  auto pair_read = [&](const int32_t* L, int it, int& j1, int& j2) {
    j1 = __ldg(L + 2 * it);
    j2 = (2 * it + 1 < kk_list) ? __ldg(L + 2 * it + 1) : -2;
  };
  auto pair_check = [&](int& j1, int& j2) {
    if (j2 == -2) j2 = j1;
    if (j1 < 0 || j1 >= dm.nb || j2 < 0 || j2 >= dm.nb) {
      atomicCAS(status, 0, kDevBounds);
      j1 = j2 = 0;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ Q and the K ring
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      int nq = 0, gp = 0;               // Q tiles and K pairs issued
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < ntiles; idx += gridDim.x) {
        const int tau = tile_at(idx);
        const int bh = tile_bh(tau), i = tau - bh * dm.nb, b = bh / dm.H, xh = (bh % dm.H) * 128;
        const int32_t* L = list_of(tau);
        const int qb = nq & 1;
        // the Q slot doubles as the output staging of the tile two back: wait for its store
        if (nq >= 2 && !mbar_wait(bar(ctl->q_free[qb]), ((nq - 2) >> 1) & 1, wc)) break;
        mbar_expect_tx(bar(ctl->q_full[qb]), G::kQBytes);
        tma_load_3d(sbase + kOffQ + qb * 16384, &tm_q, xh, i * 64, b, bar(ctl->q_full[qb]));
        if (!FP8) tma_load_3d(sbase + kOffQ + qb * 16384 + 8192, &tm_q, xh + 64, i * 64, b, bar(ctl->q_full[qb]));
        ++nq;
        for (int it = 0; it < npairs; ++it) {
          const int s = gp % kKStages;
          int j1, j2;
          pair_read(L, it, j1, j2);
          if (gp >= kKStages && !mbar_wait(bar(ctl->k_empty[s]), ((gp / kKStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          pair_check(j1, j2);
          const uint32_t st = sbase + kOffK + s * kPairBytes;
          mbar_expect_tx(bar(ctl->k_full[s]), kPairBytes);
          for (int c = 0; c < (FP8 ? 1 : 2); ++c) {
            tma_load_3d(st + c * kBoxKV, &tm_k, xh + 64 * c, j1 * 64, b, bar(ctl->k_full[s]));
            tma_load_3d(st + c * kBoxKV + 8192, &tm_k, xh + 64 * c, j2 * 64, b, bar(ctl->k_full[s]));
          }
          ++gp;
        }
      }
      // Drain: every issued copy must land before the CTA leaves.
      for (int x = (nq > 2 ? nq - 2 : 0); x < nq; ++x) mbar_wait(bar(ctl->q_full[x & 1]), (x >> 1) & 1, wc, false);
      for (int x = (gp > kKStages ? gp - kKStages : 0); x < gp; ++x)
        mbar_wait(bar(ctl->k_full[x % kKStages]), (x / kKStages) & 1, wc, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ S^T = K_pair Q^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = FP8 ? idesc_f8(128, 64, 0, 0) : idesc_f16(1, 128, 64, 0, 0);
      int j = 0, gp = 0;
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < ntiles; idx += gridDim.x, ++j) {
        const int tau = tile_at(idx);
        const int qb = j & 1;
        if (!mbar_wait(bar(ctl->q_full[qb]), (j >> 1) & 1, wc)) break;
        const uint64_t dq = sdesc_sw128(sbase + kOffQ + qb * 16384, 16, 1024);
        for (int it = 0; it < npairs; ++it, ++gp) {
          const int ks = gp % kKStages, sb = gp % kSBufs;
          if (!mbar_wait(bar(ctl->k_full[ks]), (gp / kKStages) & 1, wc)) { ok = false; break; }
          if (gp >= kSBufs && !mbar_wait(bar(ctl->s_empty[sb]), ((gp / kSBufs) - 1) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = sdesc_sw128(sbase + kOffK + ks * kPairBytes, 16, 1024);
          if constexpr (FP8) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)   // 32 e4m3 channels (32 B) per step, one box
              mma_f8_ss(tmem + kColS + 64 * sb, da + ((kk * 32) >> 4), dq + ((kk * 32) >> 4), idesc_qk, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)   // K-step offsets: 32 B inside a box, boxes 16 KB / 8 KB apart
              mma_f16_ss(tmem + kColS + 64 * sb, da + (((kk >> 2) * kBoxKV + (kk & 3) * 32) >> 4),
                         dq + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), idesc_qk, kk > 0);
          }
          mma_commit(bar(ctl->s_full[sb]));
          mma_commit(bar(ctl->k_empty[ks]));
        }
      }
      mma_commit(bar(ctl->drain_bar));       // no MMA may run when TMEM is freed
      mbar_wait(bar(ctl->drain_bar), 0, wc, false);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ O^T += V^T P^T issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = FP8 ? idesc_f8(128, 64, 1, 1) : idesc_f16(0, 128, 64, 1, 1);
      constexpr uint32_t idesc_n = idesc_f16(1, 128, 64, 1, 1);
      const int t_num = npairs > 2 ? 2 : npairs - 1;   // the pair after which num^T is issued
      int gp = 0, j = 0;
      bool ok = true;
      for (int idx = blockIdx.x; ok && idx < ntiles; idx += gridDim.x, ++j) {
        const int tau = tile_at(idx);
        for (int t = 0; t < npairs; ++t, ++gp) {
          const int s = gp % kVStages, pb = gp & 1;
          if (!mbar_wait(bar(ctl->v_full[s]), (gp / kVStages) & 1, wc)) { ok = false; break; }
          if (!mbar_wait(bar(ctl->p_full[pb]), (gp >> 1) & 1, wc)) { ok = false; break; }
          const uint64_t db = FP8 ? sdesc_sw64(sbase + kOffP + pb * G::kPBytes, 4096, 512)
                                  : sdesc_sw128(sbase + kOffP + pb * G::kPBytes, 8192, 1024);
          tc_fence_after();
          // descriptors advance by 2048 bytes (16 K-rows) per step: +128 in the address field
          const uint64_t da = sdesc_sw128(sbase + kOffV + s * kPairBytes, kBoxKV, 1024);
          if constexpr (FP8) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)   // 32 keys per step: V rows of 128 B, P rows of 64 B
              mma_f8_ss(tmem + kColO, da + 256 * kk, db + 128 * kk, idesc_pv, (t > 0) || (kk > 0));
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_f16_ss(tmem + kColO, da + 128 * kk, db + 128 * kk, idesc_pv, (t > 0) || (kk > 0));
          }
          mma_commit(bar(ctl->pv_done[pb]));
          mma_commit(bar(ctl->v_empty[s]));
          if (t == t_num) {
            // num^T = S_h^T (R u)^T for the tile's epilogue, early: it needs only the
            // epilogue operands (by now loaded), and both groups are past the previous
            // tile's epilogue (they produced this tile's P), so its columns are free.
            if (!mbar_wait(bar(ctl->ep_full), j & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sh = sbase + kOffSimg, sl = sh + 2 * RK * 128;
            const uint32_t uh = sbase + kOffUimg, ul = uh + RK * 128;
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
        }
      }
      mma_commit(bar(ctl->drain_bar));
      mbar_wait(bar(ctl->drain_bar), 0, wc, false);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ V ring + epilogue operands
    if (lane == 0) {
      tma_prefetch_desc(&tm_v);
      tma_prefetch_desc(&tm_out);
      const uint32_t sbytes = 4 * RK * 128, ubytes = 2 * RK * 128;
      int gp = 0, j = 0, nep = 0, prev_bh = -1;
      bool ok = true;
      // Epilogue operands of tile j go into single buffers once tile j - 1's epilogue is
      // over (its output store has read the staging: everything before it is done too);
      // S_h only when the head changes.
      auto load_ep = [&](int tau) {
        if (j >= 1 && !mbar_wait(bar(ctl->q_free[(j - 1) & 1]), ((j - 1) >> 1) & 1, wc)) return false;
        const int bh = tile_bh(tau);
        const bool new_s = bh != prev_bh;
        mbar_expect_tx(bar(ctl->ep_full), (new_s ? sbytes : 0) + ubytes + 256);
        if (new_s) bulk_load(sbase + kOffSimg, simg + (size_t)bh * sbytes, sbytes, bar(ctl->ep_full));
        bulk_load(sbase + kOffUimg, uimg + (size_t)tau * ubytes, ubytes, bar(ctl->ep_full));
        bulk_load(sbase + kOffGden, gden + (size_t)tau * 64, 256, bar(ctl->ep_full));
        prev_bh = bh;
        ++nep;
        return true;
      };
      for (int idx = blockIdx.x; ok && idx < ntiles; idx += gridDim.x, ++j) {
        const int tau = tile_at(idx);
        const int bh = tile_bh(tau), b = bh / dm.H, xh = (bh % dm.H) * 128;
        const int32_t* L = list_of(tau);
        bool ep_done = false;
        for (int it = 0; it < npairs; ++it) {
          if (it == kVStages) {            // the tile's first V pairs are on their way
            if (!load_ep(tau)) { ok = false; break; }
            ep_done = true;
          }
          const int s = gp % kVStages;
          int j1, j2;
          pair_read(L, it, j1, j2);
          if (gp >= kVStages && !mbar_wait(bar(ctl->v_empty[s]), ((gp / kVStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          pair_check(j1, j2);
          const uint32_t st = sbase + kOffV + s * kPairBytes;
          mbar_expect_tx(bar(ctl->v_full[s]), kPairBytes);
          for (int c = 0; c < (FP8 ? 1 : 2); ++c) {
            tma_load_3d(st + c * kBoxKV, &tm_v, xh + 64 * c, j1 * 64, b, bar(ctl->v_full[s]));
            tma_load_3d(st + c * kBoxKV + 8192, &tm_v, xh + 64 * c, j2 * 64, b, bar(ctl->v_full[s]));
          }
          ++gp;
        }
        if (ok && !ep_done && !load_ep(tau)) ok = false;
      }
      for (int x = (gp > kVStages ? gp - kVStages : 0); x < gp; ++x)
        mbar_wait(bar(ctl->v_full[x % kVStages]), (x / kVStages) & 1, wc, false);
      if (nep > 0) mbar_wait(bar(ctl->ep_full), (nep - 1) & 1, wc, false);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Two independent groups of four warps: group g owns query columns [32g, 32g + 32)
    // of S^T and O^T (its own exponent offsets, sums, rescales and output rows), so two
    // softmax warps share each SM sub-partition and hide each other's latencies.
    const int g = (warp - kSoftmaxWarp0) >> 2;
    const int wq = warp & 3;                       // TMEM lane quadrant of this warp
    const int t = 32 * wq + lane;                  // TMEM lane: key of the pair / channel d
    const int c0 = kCols * g;                      // first query column of the group
    const uint32_t gbar = 1 + g;                   // the group's named barrier
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * wq) << 16);
    const float sl2 = dm.scale * 1.4426950408889634f;
    // fast pass: largest partial row sum (so largest P) a tile may reach, 2^15 for fp16 P
    // and 2^8 for e4m3 P (whose V-scale factor is at most 1; e4m3 saturates at 448)
    constexpr float kOverflow = FP8 ? 256.f : 32768.f;
    uint8_t* sP = base + kOffP;
    bool fail = false;
    if (debug_flags & ROLA_DEBUG_STALL_WAIT) {
      WaitCtl dw{&ctl->abort, status, debug_limit_cycles};
      fail = !mbar_wait(bar(ctl->stall_bar), 0, dw);
    }
    int gp = 0, j = 0;                             // pairs and tiles done by this CTA
    for (int idx = blockIdx.x; idx < ntiles; idx += gridDim.x, ++j) {
    const int tau = tile_at(idx);
    if (named_vote_or(gbar, 128, fail)) break;
    const int bh = tile_bh(tau), i = tau - bh * dm.nb, h = bh % dm.H;
    const int b = bh / dm.H;
    const int32_t* L = list_of(tau);
    float lp[kCols];
#pragma unroll
    for (int q = 0; q < kCols; ++q) lp[q] = 0.f;

    // fp8: the scores carry sq_i * sk_j, P carries sv_j / vref and the output vref, where
    // vref = the largest V scale of this row's kept blocks (so P * sv_j / vref <= 256).
    const size_t sbase_idx = (size_t)bh * dm.nb;
    float sqi = 1.f, vref = 1.f;
    int eref = 0;
    if constexpr (FP8) {
      sqi = __ldg(sq + sbase_idx + i);
      float mx = 0.f;
      for (int e = t; e < kk_list; e += 128) {
        const int jj = __ldg(L + e);
        if (jj >= 0 && jj < dm.nb) mx = fmaxf(mx, __ldg(sv + sbase_idx + jj));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) ctl->vref[g][wq] = mx;
      named_sync(gbar, 128);
      vref = fmaxf(fmaxf(ctl->vref[g][0], ctl->vref[g][1]), fmaxf(ctl->vref[g][2], ctl->vref[g][3]));
      if (!(vref > 0.f)) vref = 1.f;
    }
    // 16-bit path: v is carried in fp16 as v * 2^-vexp per key block.  The output takes
    // 2^eref / l (eref = the largest exponent of the row's kept blocks); a tile whose
    // blocks do not all share one exponent is listed by the fast pass (its P would need a
    // factor per pair) and redone by the careful pass, which scales each pair's P by
    // 2^(vexp_j - eref) <= 1.  The fast pass gathers the exponents here and reads the
    // group's range after its end-of-tile vote; the careful pass needs eref at once.
    if constexpr (!FP8) {
      int ex_hi = INT_MIN, ex_lo = INT_MAX;
      for (int e = t; e < kk_list; e += 128) {
        const int jj = __ldg(L + e);
        if (jj >= 0 && jj < dm.nb) {
          const int x = __ldg(vexp + sbase_idx + jj);
          ex_hi = max(ex_hi, x);
          ex_lo = min(ex_lo, x);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ex_hi = max(ex_hi, __shfl_xor_sync(0xffffffffu, ex_hi, o));
        ex_lo = min(ex_lo, __shfl_xor_sync(0xffffffffu, ex_lo, o));
      }
      if (lane == 0) {
        ctl->emax[g][wq] = ex_hi;
        ctl->emin[g][wq] = ex_lo;
      }
      if constexpr (CAREFUL) {
        named_sync(gbar, 128);
        int er = max(max(ctl->emax[g][0], ctl->emax[g][1]), max(ctl->emax[g][2], ctl->emax[g][3]));
        if (er == INT_MIN) er = 0;
        eref = er;
        vref = ldexpf(1.f, er);
      }
    }
    // The key block of this warp's half of each pair (warps 0-1 of a group hold the
    // pair's first block, warps 2-3 its second; -1: the padding half of an odd list).
    // fp8 (with the block's K and V scales, a chain of dependent loads): lane l holds
    // those of pair 32c + l, loaded once per 32 pairs and broadcast by a shuffle.  16-bit
    // path: one load per pair, a pair ahead (measured faster there).
    const int half = t >> 6;
    int lane_jb = -1;
    float lane_slt = sl2, lane_pf = 1.f;   // fp8: the pair's score scale and P factor
    auto stage_list = [&](int c) {
      const int pr = 32 * c + lane, e = 2 * pr + half;
      lane_jb = (pr < npairs && e < kk_list) ? __ldg(L + e) : -1;
      if constexpr (FP8) {
        const bool in = lane_jb >= 0 && lane_jb < dm.nb;
        const float skb = in ? __ldg(sk + sbase_idx + lane_jb) : 1.f;
        const float svb = in ? __ldg(sv + sbase_idx + lane_jb) : 1.f;
        lane_slt = sl2 * sqi * skb;   // scale * log2(e) * sq_i * sk_j
        lane_pf = svb / vref;         // sv_j / vref
      }
    };
    // keys of the last block past N (its rows come from the tensor map's zero fill)
    const bool ragged_tail = (dm.N & 63) != 0;
    auto key_block = [&](int it) {
      return (t < 64) ? __ldg(L + 2 * it) : ((2 * it + 1 < kk_list) ? __ldg(L + 2 * it + 1) : -1);
    };

    // fp8: the second group starts each tile a little later, so that the two groups'
    // phases (exponentials and e4m3 packing on the special-function unit, the rest on the
    // other pipes) interleave; this measured faster for fp8 only.
    if (FP8 && (g & 1)) __nanosleep(kGroupOffsetNs);
    bool s_seen = false;                           // the next pair's S was seen complete early
    // the queries' negated exponent offsets -m: set on a tile's first pair and kept in
    // registers by the fast pass (the careful pass moves them and reads its TMEM copy)
    float mn_tile[kCols];
    for (int it = 0; it < npairs; ++it, ++gp) {
      float mn_pair[kCols];
      float(&mn)[kCols] = CAREFUL ? mn_pair : mn_tile;
      const int sb = gp % kSBufs;
      const bool ok = !fail && (s_seen || mbar_wait(bar(ctl->s_full[sb]), (gp / kSBufs) & 1, wc));
      fail |= !ok;
      tc_fence_after();
      // tcgen05.ld is warp-collective: every lane loads; invalid keys are masked after.
      float x[kCols];
      tmem_ldc(lane_addr + kColS + 64 * sb + c0, x);
      if (CAREFUL && it > 0) tmem_ldc(lane_addr + kColM + c0, mn);
      // The P buffer was last read by the P V two pairs back (maybe in the previous tile):
      // its barrier is tested now and waited for only if that P V was not done yet.
      const bool p_free = gp < 2 || mbar_test_wait(bar(ctl->pv_done[gp & 1]), ((gp - 2) >> 1) & 1);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(bar(ctl->s_empty[sb]));   // S is in registers: buffer free
      int jb;                                        // uniform over the warp
      float slt = sl2, pf = 1.f;
      if constexpr (FP8) {
        if ((it & 31) == 0) stage_list(it >> 5);
        jb = __shfl_sync(0xffffffffu, lane_jb, it & 31);
        slt = __shfl_sync(0xffffffffu, lane_slt, it & 31);
        pf = __shfl_sync(0xffffffffu, lane_pf, it & 31);
      } else {
        // the fast pass needs the key block only on the last pair (below)
        jb = (CAREFUL || it + 1 == npairs) ? key_block(it) : 0;
      }
      // x = score * scale * log2(e) - m   (m = the query's exponent offset)
      if (it > 0) {
#pragma unroll
        for (int q = 0; q < kCols; q += 2) fma2(x[q], x[q + 1], x[q], x[q + 1], slt, slt, mn[q], mn[q + 1]);
      } else {
#pragma unroll
        for (int q = 0; q < kCols; q += 2) mul2(x[q], x[q + 1], slt, slt);
      }
      // keys past the end of the sequence and the padding half of an odd list: block lists
      // are ascending (the top-k writes them so), so only a tile's last pair can hold
      // either, and the fast pass checks only there (an out-of-range index is recorded by
      // the producers, ROLA_ERR_DEVICE_BOUNDS)
      const bool check = FP8 || CAREFUL || it + 1 == npairs;
      const bool valid = !check ? ok : (ok && jb >= 0 && jb < dm.nb && jb * 64 + (t & 63) < dm.N);
      bool any_invalid;
      if constexpr (FP8)   // the test is uniform over the warp but for a failed wait
        any_invalid = !ok || jb < 0 || jb >= dm.nb || (ragged_tail && jb == dm.nb - 1);
      else
        any_invalid = check ? __any_sync(0xffffffffu, !valid) : !ok;
      if (any_invalid) {
        if (!valid) {
#pragma unroll
          for (int q = 0; q < kCols; ++q) x[q] = -INFINITY;
        }
      }
      // The first pair of a tile sets the offsets (its exact column maxima).  Careful pass:
      // later pairs move them when a score exceeds its query's offset by more than 8 (P
      // then stays within [0, 256]), decided by a vote of the group on every pair.  Fast
      // pass: no per-pair test; the tile's partial row sums bound every P it made, and a
      // tile whose sums pass kOverflow (P may have left the range of fp16, or of e4m3
      // after the V-scale factor) is recomputed by the careful pass.
      bool slow;
      if constexpr (CAREFUL) {
        float dmax = -INFINITY;
#pragma unroll
        for (int q = 0; q < kCols; q += 2) dmax = max3f(dmax, x[q], x[q + 1]);
        slow = named_vote_or(gbar, 128, fail || it == 0 || dmax > 8.f);
      } else {
        slow = it == 0;
      }
      if (slow) {
        if (named_vote_or(gbar, 128, fail)) break;
        reduce_cols<true>(ctl->red[g][wq], x, lane);
        named_sync(gbar, 128);
        if (wq == 0 && lane < kCols) {               // lane = query column c0 + lane
          const float bm = fmaxf(fmaxf(ctl->red[g][0][lane], ctl->red[g][1][lane]),
                                 fmaxf(ctl->red[g][2][lane], ctl->red[g][3][lane]));
          const float delta = it == 0 ? bm : fmaxf(bm, 0.f);
          ctl->red[g][0][lane] = delta;              // reuse: shift of each query's offset
          ctl->fac[c0 + lane] = ex2_approx(-delta);
        }
        named_sync(gbar, 128);
        // new negated offsets -(m + delta) (m = 0 on a tile's first pair) into this lane's copy
        if (it > 0) tmem_ldc(lane_addr + kColM + c0, mn);
        const float4* d4 = reinterpret_cast<const float4*>(ctl->red[g][0]);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < kCols / 4; ++q4) {
          const float4 dd = d4[q4];
          const float d[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = 4 * q4 + e;
            x[q] -= d[e];
            mn[q] = it > 0 ? mn[q] - d[e] : -d[e];
          }
        }
        tmem_stc(lane_addr + kColM + c0, mn);
        tmem_wait_st();
        if (it > 0) {
          const float4* f4 = reinterpret_cast<const float4*>(ctl->fac + c0);
#pragma unroll
          for (int q4 = 0; q4 < kCols / 4; ++q4) {
            const float4 ff = f4[q4];
            lp[4 * q4 + 0] *= ff.x;
            lp[4 * q4 + 1] *= ff.y;
            lp[4 * q4 + 2] *= ff.z;
            lp[4 * q4 + 3] *= ff.w;
          }
          fail |= !mbar_wait(bar(ctl->pv_done[(gp - 1) & 1]), ((gp - 1) >> 1) & 1, wc);
          tc_fence_after();
          float o[kCols];
          tmem_ldc(lane_addr + kColO + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < kCols / 4; ++q4) {
            const float4 ff = f4[q4];
            o[4 * q4 + 0] *= ff.x;
            o[4 * q4 + 1] *= ff.y;
            o[4 * q4 + 2] *= ff.z;
            o[4 * q4 + 3] *= ff.w;
          }
          tmem_stc(lane_addr + kColO + c0, o);
          tmem_wait_st();
        }
        named_sync(gbar, 128);                       // red[g][0] is rewritten next time
      }
      // P = 2^x (fp16, or e4m3 times sv_j / vref) and the per-thread partial row sums
      uint32_t pw[kCols / 2];
      if constexpr (FP8) {
#pragma unroll
        for (int q = 0; q < kCols; q += 4) {
          // a quarter of the exponentials on the FMA pipe (see ex2_poly)
          const bool poly = (q & 12) == 12;
          float p0 = poly ? ex2_poly(x[q]) : ex2_approx(x[q]);
          float p1 = poly ? ex2_poly(x[q + 1]) : ex2_approx(x[q + 1]);
          float p2 = poly ? ex2_poly(x[q + 2]) : ex2_approx(x[q + 2]);
          float p3 = poly ? ex2_poly(x[q + 3]) : ex2_approx(x[q + 3]);
          add2(lp[q], lp[q + 1], p0, p1);
          add2(lp[q + 2], lp[q + 3], p2, p3);
          mul2(p0, p1, pf, pf);
          mul2(p2, p3, pf, pf);
          pw[q >> 2] = pack_e4m3x4(p0, p1, p2, p3);
        }
      } else {
        // every exponential on ex2 here (a quarter on the FMA pipe, as for fp8, measured
        // 1 % slower on this path)
        float vf = 1.f;                    // careful pass: 2^(vexp_j - eref) of this pair
        if constexpr (CAREFUL) {
          if (jb >= 0 && jb < dm.nb) vf = ldexpf(1.f, __ldg(vexp + sbase_idx + jb) - eref);
        }
#pragma unroll
        for (int q = 0; q < kCols; q += 2) {
          float p0 = ex2_approx(x[q]);
          float p1 = ex2_approx(x[q + 1]);
          add2(lp[q], lp[q + 1], p0, p1);
          if constexpr (CAREFUL) mul2(p0, p1, vf, vf);
          pw[q >> 1] = pack_half2(p0, p1);
        }
      }
      // the next pair's S, tested before this pair's stores so that the test's latency
      // overlaps them (a stale "not yet" only means a wait at the top of the loop)
      s_seen = it + 1 < npairs && !fail &&
               mbar_test_wait(bar(ctl->s_full[(gp + 1) % kSBufs]), ((gp + 1) / kSBufs) & 1);
      if (!p_free && !fail) fail |= !mbar_wait(bar(ctl->pv_done[gp & 1]), ((gp - 2) >> 1) & 1, wc);
      if constexpr (FP8)
        st_chunks_sw64<kCols / 16>(sP + (gp & 1) * G::kPBytes, t, (kCols / 16) * g, pw);
      else
        st_chunks_sw128<kCols / 8>(sP + (gp & 1) * G::kPBytes, t, (kCols / 8) * g, pw);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();                                  // the warp's P rows and O^T rescale are done
      if (lane == 0) mbar_arrive(bar(ctl->p_full[gp & 1]));
    }

    // ------------------------------------------------------------ epilogue
    if constexpr (!CAREFUL) {
      // each P of the tile is at most its thread's partial row sum
      bool overflow = false;
#pragma unroll
      for (int q = 0; q < kCols; ++q) overflow |= !(lp[q] <= kOverflow);   // (NaN counts too)
      const bool listed = named_vote_or(gbar, 128, overflow);
      bool mixed = false;                  // 16-bit path: the kept blocks' v exponents differ
      if constexpr (!FP8) {
        const int hi = max(max(ctl->emax[g][0], ctl->emax[g][1]), max(ctl->emax[g][2], ctl->emax[g][3]));
        const int lo = min(min(ctl->emin[g][0], ctl->emin[g][1]), min(ctl->emin[g][2], ctl->emin[g][3]));
        mixed = hi != lo && hi != INT_MIN;
        eref = hi == INT_MIN ? 0 : hi;
        vref = ldexpf(1.f, eref);
      }
      if ((listed || mixed) && t == 0) {
        const int slot = atomicAdd(redo, 1);
        if (slot < 2 * ntiles_all) redo[1 + slot] = tau;
      }
    }
    if (!named_vote_or(gbar, 128, fail)) {
      // per-query sums l over the group's 128 threads (final once the last P is made)
      reduce_cols<false>(ctl->red[g][wq], lp, lane);
      named_sync(gbar, 128);
      if (wq == 0 && lane < kCols)
        ctl->linv[c0 + lane] = vref / (ctl->red[g][0][lane] + ctl->red[g][1][lane] +
                                       ctl->red[g][2][lane] + ctl->red[g][3][lane]);
      // the tile's last P V (it also proves both groups are done with its S buffers), and
      // num^T (issued by the P V issuer early in the tile)
      fail |= !mbar_wait(bar(ctl->pv_done[(gp - 1) & 1]), ((gp - 1) >> 1) & 1, wc);
      fail |= !mbar_wait(bar(ctl->ep_bar), j & 1, wc);
      fail |= !mbar_wait(bar(ctl->ep_full), j & 1, wc);     // g/den copy visible to every thread
      if (!named_vote_or(gbar, 128, fail)) {
        tc_fence_after();
        // out^T[d = t][q] = O^T / l + (g / den) num^T -> staging [2 boxes][64 q][64 d],
        // this group's rows c0 .. c0 + 31
        const float* gd = reinterpret_cast<const float*>(base + kOffGden);
        uint8_t* stg = base + kOffQ + (j & 1) * 16384;   // the tile's Q slot
        __nv_bfloat16* col = reinterpret_cast<__nv_bfloat16*>(stg + (t >> 6) * 8192) + (t & 63);
        float o[kCols], nm[kCols];
        tmem_ldc(lane_addr + kColO + c0, o);
        tmem_ldc(lane_addr + kColNum + c0, nm);
        tmem_wait_ld();
#pragma unroll
        for (int qq4 = 0; qq4 < kCols / 4; ++qq4) {
          const float4 li = reinterpret_cast<const float4*>(ctl->linv + c0)[qq4];
          const float4 gg = reinterpret_cast<const float4*>(gd + c0)[qq4];
          const int q0 = c0 + 4 * qq4, e = 4 * qq4;
          col[(q0 + 0) * 64] = __float2bfloat16_rn(o[e + 0] * li.x + nm[e + 0] * gg.x);
          col[(q0 + 1) * 64] = __float2bfloat16_rn(o[e + 1] * li.y + nm[e + 1] * gg.y);
          col[(q0 + 2) * 64] = __float2bfloat16_rn(o[e + 2] * li.z + nm[e + 2] * gg.z);
          col[(q0 + 3) * 64] = __float2bfloat16_rn(o[e + 3] * li.w + nm[e + 3] * gg.w);
        }
        fence_proxy_async_smem();
        named_sync(gbar, 128);
        // rows at or past N are clipped by the tensor map; a box wholly past N is skipped
        if (t == 0) {
          const uint32_t src = sbase + kOffQ + (j & 1) * 16384 + c0 * 128;
          if (i * 64 + c0 < dm.N) {
            tma_store_3d(&tm_out, h * 128, i * 64 + c0, b, src);
            tma_store_3d(&tm_out, h * 128 + 64, i * 64 + c0, b, src + 8192);
            tma_store_commit();
            tma_store_wait_read0();
          }
          mbar_arrive(bar(ctl->q_free[j & 1]));      // the Q slot may be refilled
        }
      }
    }
    }   // tiles
  }


  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int RK, bool FP8>
cudaError_t launch_variant(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const Dims& dm, const Workspace& ws, int debug_flags,
                           int debug_limit_us, cudaStream_t st) {
  // Wait limits in SM clock cycles: 2e9 cycles is 1 s at 2 GHz (longer at lower clocks).
  const unsigned long long limit_cycles = 2000000000ull;
  const unsigned long long dlimit = (unsigned long long)(debug_limit_us > 0 ? debug_limit_us : 1000) * 2000ull;
  constexpr size_t smem = smem_bytes<FP8>();
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(attend_sm100_kernel<RK, FP8, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(attend_sm100_kernel<RK, FP8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)smem)) != cudaSuccess)
    return e;
  // persistent: one CTA per SM, each walking the tiles tau = blockIdx.x + n * gridDim.x
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long ntiles = (long long)dm.nb * dm.B * dm.H;
  dim3 grid((unsigned)(ntiles < sms ? ntiles : sms));
  // fast pass over every tile, then the careful pass over the tiles it listed (none, usually:
  // its CTAs then exit at once)
  if ((e = cudaMemsetAsync(ws.redo, 0, sizeof(int), st)) != cudaSuccess) return e;
  attend_sm100_kernel<RK, FP8, false><<<grid, kThreads, smem, st>>>(
      tq, tk, tv, to, dm, ws.col_idx, ws.simg, ws.uimg, ws.gden, ws.sq, ws.sk, ws.sv, ws.vexp, ws.status,
      ws.redo, debug_flags, limit_cycles, dlimit);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  attend_sm100_kernel<RK, FP8, true><<<grid, kThreads, smem, st>>>(
      tq, tk, tv, to, dm, ws.col_idx, ws.simg, ws.uimg, ws.gden, ws.sq, ws.sk, ws.sv, ws.vexp, ws.status,
      ws.redo, debug_flags, limit_cycles, dlimit);
  return cudaGetLastError();
}

}  // namespace

size_t attend_sm100_smem_bytes(bool fp8) { return fp8 ? smem_bytes<true>() : smem_bytes<false>(); }

cudaError_t launch_attend_sm100(const Dims& dm, const void* q, const void* k, const Workspace& ws,
                                void* out, bool fp8, int debug_flags, int debug_limit_us, cudaStream_t st) {
  CUtensorMap tq, tk, tv, to;
  bool ok;
  if (fp8)
    ok = make_act_map(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws.q8, dm, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_act_map(&tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws.k8, dm, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_act_map(&tv, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, ws.v8, dm, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = make_act_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dm, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_act_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, dm, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_act_map(&tv, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, ws.v16, dm, CU_TENSOR_MAP_SWIZZLE_128B);
  // output: [kCols tokens x 64 channels] boxes, one per query group and channel half
  ok = ok && make_act_map(&to, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, out, dm, CU_TENSOR_MAP_SWIZZLE_NONE, kCols);
  if (!ok) return cudaErrorInvalidValue;
  if (fp8)
    return dm.r == 32 ? launch_variant<32, true>(tq, tk, tv, to, dm, ws, debug_flags, debug_limit_us, st)
                      : launch_variant<16, true>(tq, tk, tv, to, dm, ws, debug_flags, debug_limit_us, st);
  return dm.r == 32 ? launch_variant<32, false>(tq, tk, tv, to, dm, ws, debug_flags, debug_limit_us, st)
                    : launch_variant<16, false>(tq, tk, tv, to, dm, ws, debug_flags, debug_limit_us, st);
}

}  // namespace rola
