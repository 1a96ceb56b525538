// Block scores of the selection (step 2) on the sm_100a tensor cores: for every (b, h),
// s~ = qbar kbar^T over all pairs of blocks, with tcgen05 kind::tf32 on a three-term split
// of the fp32 means (x = hi + lo, hi = x with its low 13 mantissa bits cleared, so exact in
// tf32; s~ = Ah Bh + Ah Bl + Al Bh), accumulated in TMEM and written to the score rows by
// TMA; and the key-block norms ||kbar_j||_2 that bound how far s~ can be from the exact
// score.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (the sparse branch keeps the query-key
// block pairs of highest energy); README inference section (topk = fraction kept).
//
// These scores only prune.  The kept lists are decided on exact fp32 scores (the chain of
// fused multiply-adds over channels 0..d-1, as stated for the selection), computed by the
// top-k kernel only for rows whose boundary s~ cannot settle.  Error of s~ against the
// exact score s, per pair (|.| summed over the channels c; |lo| <= 2^-10 |x|):
//   dropped Al Bl, lo read as tf32 (10 mantissa bits)      < 3 * 2^-20 sum |q_c k_c|
//   tensor-core fp32 accumulation (3 x d/8 steps of 8
//   products, taken as a few units of 2^-23 per step)      < 2^-17 sum |q_c k_c|
//   the exact chain's own rounding (d <= 128 FMAs)        < 2^-17 sum |q_c k_c|
//   operands or products below 2^-126 flushed to zero     < 2^-122 (|q| + |k|) + 2^-116
// and sum |q_c k_c| <= |q| |k| (Cauchy-Schwarz), so |s~ - s| <= 2^-14 |q| |k| + 2^-122 (|q| +
// |k|) + 2^-116, a factor of about three to spare (the tests check the measured error
// against half of it).
//
// Tiles: 128 query blocks (TMEM lanes, M) x 256 key blocks (TMEM columns, N), K = d in
// 32-channel chunks of 128 bytes (one 128-byte swizzle atom per row).  Rows past nb load as
// zeros; rows and columns past the score matrix are clipped by the TMA stores.
// Roles (320 threads): warp 0 = TMA producer (2-stage ring of A and B chunks); warps 6-9 =
// split of each landed chunk (hi in place, lo beside it); warp 1 = MMA issuer and TMEM owner
// (two accumulators of 256 columns); warps 2-5 = epilogue, warp w reading TMEM lanes
// 32 (w mod 4) .. +31: TMEM -> registers -> swizzled 32 x 32 staging box -> TMA store.  The
// tiles of the first row of query blocks also compute the key norms.
// Persistent: CTA c takes tiles c, c + gridDim.x, ...  Every wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "rola_internal.cuh"
#include "sm100_ptx.cuh"

namespace rola {
namespace {

using namespace sm100;

namespace sc {
constexpr int kM = 128;
constexpr int kN = 256;
constexpr int kStages = 2;
constexpr uint32_t kABytes = kM * 128;   // one 32-channel fp32 chunk of 128 query blocks
constexpr uint32_t kBBytes = kN * 128;
constexpr uint32_t kHalfBytes = kABytes + kBBytes;   // A then B: the hi parts; the lo parts follow
constexpr uint32_t kStageBytes = 2 * kHalfBytes;
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = 4;
constexpr int kSplitWarp0 = kEpiWarp0 + kEpiWarps;
constexpr int kSplitWarps = 4;
constexpr int kThreads = 32 * (kSplitWarp0 + kSplitWarps);
constexpr uint32_t kBoxBytes = 32 * 128;   // a 32 x 32 fp32 store box
constexpr uint32_t kOffStore = kStages * kStageBytes;
constexpr uint32_t kOffCtl = kOffStore + kEpiWarps * 2 * kBoxBytes;
constexpr uint32_t kTmemCols = 2 * kN;

struct Ctl {
  uint64_t full[kStages], split[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kSmemBytes = kOffCtl + sizeof(Ctl) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory");
}  // namespace sc

__global__ void __launch_bounds__(sc::kThreads, 1) score_sm100_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ CUtensorMap tm_s, Dims dm, const float* __restrict__ kbar, float* __restrict__ knorm,
    int nbp, int* __restrict__ status, unsigned long long limit_cycles) {
  using namespace sc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl* ctl = reinterpret_cast<Ctl*>(base + kOffCtl);
  const uint32_t sbase = smem_addr(base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = dm.nb, d = dm.d, nchunk = d / 32;
  const int nmt = (nb + kM - 1) / kM, nnt = (nb + kN - 1) / kN;
  const int ntiles = nmt * nnt * dm.B * dm.H;
  const int my_tiles = (int)blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };
  // tile jt of this CTA: key-block tiles innermost, so neighbouring tiles share A
  auto tile_of = [&](int jt, int& bh, int& mt, int& nt) {
    int tau = (int)blockIdx.x + jt * (int)gridDim.x;
    nt = tau % nnt;
    tau /= nnt;
    mt = tau % nmt;
    bh = tau / nmt;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(ctl->full[s]), 1);
      mbar_init(bar(ctl->split[s]), kSplitWarps);
      mbar_init(bar(ctl->empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(ctl->acc_full[s]), 1);
      mbar_init(bar(ctl->acc_empty[s]), kEpiWarps);
    }
    mbar_init(bar(ctl->drain), 1);
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
    // ------------------------------------------------------------ A and B chunks
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      int gc = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        int bh, mt, nt;
        tile_of(jt, bh, mt, nt);
        for (int c = 0; c < nchunk; ++c, ++gc) {
          const int s = gc % kStages;
          if (gc >= kStages && !mbar_wait(bar(ctl->empty[s]), ((gc / kStages) - 1) & 1, wc)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + s * kStageBytes;
          mbar_expect_tx(bar(ctl->full[s]), kHalfBytes);
          tma_load_3d(st, &tm_a, 32 * c, mt * kM, bh, bar(ctl->full[s]));
          tma_load_3d(st + kABytes, &tm_b, 32 * c, nt * kN, bh, bar(ctl->full[s]));
        }
      }
      // no copy may be in flight when the CTA exits
      for (int x = (gc > kStages ? gc - kStages : 0); x < gc; ++x)
        mbar_wait(bar(ctl->full[x % kStages]), (x / kStages) & 1, wc, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ s~ = A B^T into TMEM
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32(kM, kN);
      int gc = 0;
      bool ok = true;
      for (int jt = 0; ok && jt < my_tiles; ++jt) {
        const int acc = jt & 1;
        if (jt >= 2 && !mbar_wait(bar(ctl->acc_empty[acc]), ((jt - 2) >> 1) & 1, wc)) break;
        tc_fence_after();
        for (int c = 0; c < nchunk; ++c, ++gc) {
          const int s = gc % kStages;
          if (!mbar_wait(bar(ctl->split[s]), (gc / kStages) & 1, wc)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * kStageBytes;
          const uint64_t ah = sdesc_sw128(st, 16, 1024), bh = sdesc_sw128(st + kABytes, 16, 1024);
          const uint64_t al = sdesc_sw128(st + kHalfBytes, 16, 1024);
          const uint64_t bl = sdesc_sw128(st + kHalfBytes + kABytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // 8 channels (32 B) per MMA inside the 128-byte atom
            mma_tf32_ss(tmem + acc * kN, al + 2 * kk, bh + 2 * kk, idesc, (c | kk) != 0);
            mma_tf32_ss(tmem + acc * kN, ah + 2 * kk, bl + 2 * kk, idesc, true);
            mma_tf32_ss(tmem + acc * kN, ah + 2 * kk, bh + 2 * kk, idesc, true);
          }
          mma_commit(bar(ctl->empty[s]));
        }
        if (ok) mma_commit(bar(ctl->acc_full[acc]));
      }
      mma_commit(bar(ctl->drain));   // no MMA may run when TMEM is freed
      mbar_wait(bar(ctl->drain), 0, wc, false);
    }
  } else if (warp >= kSplitWarp0) {
    // ------------------------------------------------------------ hi / lo split
    const int t = threadIdx.x - 32 * kSplitWarp0;
    int gc = 0;
    bool fail = false;
    for (int jt = 0; jt < my_tiles && !fail; ++jt) {
      for (int c = 0; c < nchunk; ++c, ++gc) {
        const int s = gc % kStages;
        fail = __any_sync(0xffffffffu, !mbar_wait(bar(ctl->full[s]), (gc / kStages) & 1, wc));
        if (fail) break;
        uint8_t* hi = base + s * kStageBytes;
        uint8_t* lo = hi + kHalfBytes;
        for (uint32_t o = 16u * t; o < kHalfBytes; o += 16u * 32 * kSplitWarps) {
          const uint4 x = *reinterpret_cast<const uint4*>(hi + o);
          const uint4 h = make_uint4(x.x & 0xffffe000u, x.y & 0xffffe000u, x.z & 0xffffe000u, x.w & 0xffffe000u);
          *reinterpret_cast<uint4*>(hi + o) = h;
          *reinterpret_cast<float4*>(lo + o) =
              make_float4(__uint_as_float(x.x) - __uint_as_float(h.x), __uint_as_float(x.y) - __uint_as_float(h.y),
                          __uint_as_float(x.z) - __uint_as_float(h.z), __uint_as_float(x.w) - __uint_as_float(h.w));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if ((t & 31) == 0) mbar_arrive(bar(ctl->split[s]));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quad) << 16);
    uint8_t* stg = base + kOffStore + (warp - kEpiWarp0) * 2 * kBoxBytes;
    const uint32_t stg_addr = smem_addr(stg);
    int nst = 0;
    bool fail = false;
    for (int jt = 0; jt < my_tiles; ++jt) {
      int bh, mt, nt;
      tile_of(jt, bh, mt, nt);
      if (mt == 0) {
        // ||kbar_j||_2 of this tile's key blocks, once per block (fp32, channel order)
        for (int t = 32 * (warp - kEpiWarp0) + lane; t < kN; t += 32 * kEpiWarps) {
          const int j = nt * kN + t;
          if (j >= nb) break;
          const float4* kr = reinterpret_cast<const float4*>(kbar + ((size_t)bh * nb + j) * d);
          float ss = 0.f;
          for (int c4 = 0; c4 < d / 4; ++c4) {
            const float4 v = __ldg(kr + c4);
            ss = fmaf(v.x, v.x, ss);
            ss = fmaf(v.y, v.y, ss);
            ss = fmaf(v.z, v.z, ss);
            ss = fmaf(v.w, v.w, ss);
          }
          knorm[(size_t)bh * nbp + j] = sqrtf(ss);
        }
      }
      const int acc = jt & 1;
      fail = __any_sync(0xffffffffu, fail || !mbar_wait(bar(ctl->acc_full[acc]), (jt >> 1) & 1, wc));
      if (fail) break;
      tc_fence_after();
      const int y = mt * kM + 32 * quad;
#pragma unroll 1
      for (int c = 0; c < kN / 32; ++c) {
        const int x0 = nt * kN + 32 * c;
        if (x0 >= nbp || y >= nb) break;
        float v[32];
        tmem_ld32(lane_addr + acc * kN + 32 * c, v);
        tmem_wait_ld();
        // the box written two stores ago must have been read out
        if (lane == 0 && nst >= 2) tma_store_wait_read1();
        __syncwarp();
        uint8_t* sp = stg + (nst & 1) * kBoxBytes;
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4)
          *reinterpret_cast<float4*>(sp + lane * 128 + ((c4 ^ (lane & 7)) << 4)) =
              make_float4(v[4 * c4], v[4 * c4 + 1], v[4 * c4 + 2], v[4 * c4 + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tm_s, x0, y, bh, stg_addr + (nst & 1) * kBoxBytes);
          tma_store_commit();
        }
        ++nst;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ctl->acc_empty[acc]));
    }
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, sc::kTmemCols);
  }
}

}  // namespace

cudaError_t launch_score_sm100(const Dims& dm, const Workspace& ws, int nbp, cudaStream_t st) {
  if (dm.d % 32 != 0) return cudaErrorInvalidValue;
  const uint64_t BH = (uint64_t)dm.B * dm.H;
  CUtensorMap ta, tb, ts;
  if (!make_map_3d(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ws.qbar, dm.d, dm.nb, BH, 32, sc::kM,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&tb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ws.kbar, dm.d, dm.nb, BH, 32, sc::kN,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ws.scores, nbp, dm.nb, BH, 32, 32,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(score_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sc::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const long long ntiles = (long long)((dm.nb + sc::kM - 1) / sc::kM) * ((dm.nb + sc::kN - 1) / sc::kN) * (long long)BH;
  dim3 grid((unsigned)(ntiles < sms ? ntiles : sms));
  // Wait limit in SM clock cycles: 2e9 cycles is 1 s at 2 GHz.
  score_sm100_kernel<<<grid, sc::kThreads, sc::kSmemBytes, st>>>(ta, tb, ts, dm, ws.kbar, ws.knorm, nbp,
                                                                 ws.status, 2000000000ull);
  return cudaGetLastError();
}

}  // namespace rola
