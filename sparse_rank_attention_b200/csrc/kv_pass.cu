// Key/value pass of the RoLA forward for head dim 128 with bf16 inputs: one read of k
// and v computes everything the later steps need from them.
//   * the linear-branch state partials over a chunk of tokens (split-N; step 4, key side)
//       S_h += sum_m R(p_m) phi(k_m Wk_h) v_m^T,   z_h += sum_m phi(k_m Wk_h)
//     with both contractions on the tcgen05 tensor cores, accumulating in tensor memory;
//   * the block means of k (step 1, key side): fp32 sums in token order, one division;
//   * bf16 configuration: the fp16 copy of v that the attention kernel multiplies the
//     fp16 softmax weights with.  Each (b, h, block) of v is carried as v * 2^-e with one
//     power-of-two exponent e per block (0 for blocks whose largest |v| lies in
//     [2^-6, 2^15), else the exponent that brings it into [2^14, 2^15)), so every finite
//     bf16 value fits fp16 exactly as far as fp16's 11 bits allow; e goes to vexp.
//     Non-finite v sets ROLA_ERR_RANGE;
//   * fp8 configuration: the e4m3 copies of k and v with one scale per (b, h, block)
//     (scale = absmax / 448, 1 for an all-zero block; code = RN-sat(x * (1 / scale))).
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (high-energy block selection; low-rank
// linear branch with rotary positions); README sparse-finetuning section (proj_k).
//
// Layout of the work: a CTA owns one (b, h) and a chunk of whole 64-token blocks; the
// chunk length is chosen on the host so that the CTAs fill the SMs in whole waves (two
// CTAs per SM).  k and v tiles (one block each: two TMA boxes of 64 tokens x 64 channels,
// 128-byte swizzle) flow through a 2-stage ring filled by a producer warp; rows past N
// arrive as zeros.  Per tile:
//   F = K Wk           one tcgen05 MMA chain, M = 64 tokens, N = r, K = 128 channels
//                      (A = the k tile, B = Wk_h^T staged once per CTA), fp32 in TMEM,
//                      issued a tile ahead into one of two TMEM buffers;
//   F~ = R(p) phi(F)   warps 0-7 (two per TMEM lane quadrant), one token and a quarter
//                      of the r values per thread, stored as bf16 hi + lo into one of
//                      two K-major operand images;
//   S^T += V^T F~      M = 128 channels, N = r, K = 64 tokens (A = the v tile read
//                      MN-major, B = the hi and lo images), accumulated in TMEM over the
//                      whole chunk and read out once at its end;
// while warps 8-9 pool k (and write its e4m3 copy) and warps 10-11 write the copy of v.
// Every wait is bounded (ROLA_ERR_DEVICE_TIMEOUT).
#include "rola_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda_fp8.h>

namespace rola {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kTok = 64;                     // tokens per tile = one block
constexpr int kStages = 2;
constexpr int kThreads = 416;                // warps 0-7 features, 8-9 k means, 10-11 v copy, 12 TMA
constexpr uint32_t kTileBytes = kTok * kD * 2;   // 16 KB: two boxes of 64 rows x 128 bytes
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kColF = 0;                // F [64 tokens x r] (M = 64 layout), two buffers
constexpr uint32_t kColS = 64;               // S^T [128 channels x r]

// Byte offset of 16-byte chunk c (channels 8c .. 8c + 7, c = 0..15) of token row r in a
// tile: box c / 8 (8 KB each), 128-byte rows, chunk position (c % 8) ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((c >> 3) * 8192 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Byte offset of element (row, col) of a K-major 128-byte-swizzled bf16 operand image
// (rows of 64 elements; 8-row atoms of 1024 bytes).
__device__ __forceinline__ uint32_t img_off(int row, int col) {
  return (uint32_t)(row * 128 + ((((col >> 3) ^ row) & 7) << 4) + (col & 7) * 2);
}

template <int RK>
struct KVGeo {
  static constexpr uint32_t offK = 0;                                // kStages k tiles
  static constexpr uint32_t offV = offK + kStages * kTileBytes;      // kStages v tiles
  static constexpr uint32_t offW = offV + kStages * kTileBytes;      // Wk_h^T: 2 boxes [r][64 ch]
  static constexpr uint32_t kImg = 2 * RK * 128;                     // F~ hi [r][64 tok], then lo
  static constexpr uint32_t offF = offW + 2 * RK * 128;              // two F~ images
  static constexpr uint32_t offCtl = offF + 2 * kImg;
};

struct KVCtl {
  uint64_t full[kStages], freed[kStages], f_full[2], img_free[2], drain;
  uint32_t tmem_base;
  int abort;
  float zred[4][32];
  float red[8];
};

template <int RK>
constexpr size_t kv_smem_bytes() { return KVGeo<RK>::offCtl + sizeof(KVCtl) + 1024; }

__device__ __forceinline__ float absmax8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xffff0000u))));
  return m;
}

// 8 bf16 values times inv, rounded to e4m3 (nearest even, saturating), in element order.
__device__ __forceinline__ uint2 e4m3x8(const uint4& v, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[2] = {0, 0};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = make_float2(__uint_as_float(w[e] << 16) * inv, __uint_as_float(w[e] & 0xffff0000u) * inv);
    o[e >> 1] |= (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3) << (16 * (e & 1));
  }
  return make_uint2(o[0], o[1]);
}

// (x0, x1) as packed bf16 pairs hi + lo with |x - hi - lo| <= 2^-16 |x|.
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(x0, x1);
  const float2 bf = __bfloat1622float2(b);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - bf.x, x1 - bf.y);
  hi = *reinterpret_cast<const uint32_t*>(&b);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// TMEM lanes 0-15 of this warp's quadrant (the M = 64 layout): threads 0-15 read n
// consecutive fp32 columns, threads 16-31 the n columns after them.
__device__ __forceinline__ void tmem_ld16x2_x4(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x4.b32 {%0, %1, %2, %3}, [%4], 4;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_ld16x2_x8(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], 8;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane (all 32 lanes of the quadrant).
__device__ __forceinline__ void tmem_ld32x32_x16(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

template <int RK, bool FP8>
__global__ void __launch_bounds__(kThreads, 2) kv_pass_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __nv_bfloat16* __restrict__ Wk, Dims dm, const float2* __restrict__ rope,
    float* __restrict__ S_part, float* __restrict__ z_part, float* __restrict__ kbar,
    __half* __restrict__ v16, int* __restrict__ vexp, uint8_t* __restrict__ k8, uint8_t* __restrict__ v8,
    float* __restrict__ sk, float* __restrict__ sv, int* __restrict__ status) {
  using G = KVGeo<RK>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  KVCtl* ctl = reinterpret_cast<KVCtl*>(smem + G::offCtl);
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const int n_begin = chunk * dm.chunk_tok;
  const int n_end = min(dm.N, n_begin + dm.chunk_tok);
  const int ntiles = n_end > n_begin ? (n_end - n_begin + kTok - 1) / kTok : 0;
  const size_t rs = (size_t)dm.H * kD;           // elements between tokens

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(ctl->full[s]), 1);
      mbar_init(bar(ctl->freed[s]), 5);   // the S^T MMAs' commit + warps 8-11
    }
    for (int b2 = 0; b2 < 2; ++b2) {
      mbar_init(bar(ctl->f_full[b2]), 1);
      mbar_init(bar(ctl->img_free[b2]), 1);
    }
    mbar_init(bar(ctl->drain), 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  // Wk_h^T as the K-major B operand of F = K Wk: row a (rank), channel c in box c / 64
  for (int e = tid; e < kD * RK; e += kThreads) {
    const int c = e / RK, a = e % RK;
    *reinterpret_cast<__nv_bfloat16*>(smem + G::offW + (c >> 6) * (RK * 128) + img_off(a, c & 63)) =
        Wk[((size_t)h * kD + c) * RK + a];
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(smem_addr(&ctl->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const WaitCtl wc{&ctl->abort, status, 2000000000ull};

  if (warp == 12) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % kStages, n0 = n_begin + t * kTok;
        if (t >= kStages && !mbar_wait(bar(ctl->freed[s]), ((t / kStages) - 1) & 1, wc)) break;
        const uint32_t fb = bar(ctl->full[s]);
        mbar_expect_tx(fb, 2 * kTileBytes);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sbase + G::offK + s * kTileBytes + c * 8192, &tm_k, h * kD + 64 * c, n0, b, fb);
          tma_load_3d(sbase + G::offV + s * kTileBytes + c * 8192, &tm_v, h * kD + 64 * c, n0, b, fb);
        }
        issued = t + 1;
      }
      // every issued copy must land before the CTA leaves
      for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
        mbar_wait(bar(ctl->full[t % kStages]), (t / kStages) & 1, wc, false);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ features and the MMAs
    const bool issuer = warp == 0 && lane == 0;
    constexpr uint32_t idesc_f = idesc_f16(1, 64, RK, 0, 0);    // F = K Wk
    constexpr uint32_t idesc_s = idesc_f16(1, 128, RK, 1, 0);   // S^T += V^T F~
    constexpr int HR = RK / 4;                  // rank values per thread
    const int qd = warp & 3, hf = warp >> 2;    // TMEM lane quadrant; half of the ranks
    const int row = 16 * qd + (lane & 15);      // token of the tile
    const int a0 = hf * (RK / 2) + (lane >> 4) * HR;   // first rank value of this thread
    float zacc[HR];
#pragma unroll
    for (int a = 0; a < HR; ++a) zacc[a] = 0.f;
    bool ok = true;
    int done = 0;
    // F of tile t goes to TMEM buffer t & 1 and is issued one tile ahead, so that the
    // MMA's latency overlaps the features of the tile before; the F~ images alternate too.
    auto issue_f = [&](int t) {
      const int s = t % kStages;
      if (!mbar_wait(bar(ctl->full[s]), (t / kStages) & 1, wc)) return false;
      tc_fence_after();
      const uint32_t tk = sbase + G::offK + s * kTileBytes;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk)
        mma_f16_ss(tmem + kColF + 32 * (t & 1), sdesc_sw128(tk + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                   sdesc_sw128(sbase + G::offW + (kk >> 2) * (RK * 128) + (kk & 3) * 32, 16, 1024), idesc_f,
                   kk > 0);
      mma_commit(bar(ctl->f_full[t & 1]));
      return true;
    };
    // (the MMA of tile t + 1 is issued early only if its tile has already landed: waiting
    // for it here would hold the current tile back)
    int nf = 0;                                   // F MMAs issued (issuer thread)
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kStages, n = n_begin + t * kTok + row;
      if (issuer && ok) {
        if (nf == t) { ok = issue_f(t); ++nf; }
        if (ok && nf == t + 1 && t + 1 < ntiles &&
            mbar_test_wait(bar(ctl->full[(t + 1) % kStages]), ((t + 1) / kStages) & 1)) {
          ok = issue_f(t + 1);
          ++nf;
        }
      }
      // one barrier per tile (before the S^T MMAs): a failed wait is carried to it, and
      // tcgen05.ld runs on the whole converged warp whatever its lanes' waits returned
      if (ok) ok = mbar_wait(bar(ctl->f_full[t & 1]), (t >> 1) & 1, wc);
      __syncwarp();
      tc_fence_after();
      float f[HR];
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * qd) << 16) + kColF + 32 * (t & 1) + hf * (RK / 2);
      if constexpr (RK == 32) tmem_ld16x2_x8(lane_addr, f);
      else tmem_ld16x2_x4(lane_addr, f);
      tmem_wait_ld();
      // phi, z, rotation (pairs a0/2 ..) and the hi / lo split; tokens past the chunk
      // (or N) contribute nothing
      const bool valid = n < n_end;
      const TokPos pos = token_pos(dm, valid ? n : 0);
      uint32_t hi[HR / 2], lo[HR / 2];
#pragma unroll
      for (int p = 0; p < HR / 2; ++p) {
        const float x0 = valid ? phi_fast(f[2 * p]) : 0.f;
        const float x1 = valid ? phi_fast(f[2 * p + 1]) : 0.f;
        zacc[2 * p] += x0;
        zacc[2 * p + 1] += x1;
        const float2 cs = valid ? rope_at(dm, rope, pos, a0 / 2 + p) : make_float2(1.f, 0.f);
        split_bf16x2(cs.x * x0 - cs.y * x1, cs.y * x0 + cs.x * x1, hi[p], lo[p]);
      }
      // the S^T MMAs of tile t - 2 read this image: wait for them before rewriting it
      if (ok && t >= 2) ok = mbar_wait(bar(ctl->img_free[t & 1]), ((t - 2) >> 1) & 1, wc);
      uint8_t* ih = smem + G::offF + (t & 1) * G::kImg;
      if (ok) {
#pragma unroll
        for (int p = 0; p < HR / 2; ++p) {
          const int a = a0 + 2 * p;
          *reinterpret_cast<uint16_t*>(ih + img_off(a, row)) = (uint16_t)(hi[p] & 0xffffu);
          *reinterpret_cast<uint16_t*>(ih + img_off(a + 1, row)) = (uint16_t)(hi[p] >> 16);
          *reinterpret_cast<uint16_t*>(ih + RK * 128 + img_off(a, row)) = (uint16_t)(lo[p] & 0xffffu);
          *reinterpret_cast<uint16_t*>(ih + RK * 128 + img_off(a + 1, row)) = (uint16_t)(lo[p] >> 16);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      if (named_vote_or(1, 256, !ok)) { ok = false; break; }
      if (issuer) {
        tc_fence_after();
        const uint32_t tv = sbase + G::offV + s * kTileBytes;
        const uint32_t fi = sbase + G::offF + (t & 1) * G::kImg;
        const uint64_t da = sdesc_sw128(tv, 8192, 1024);
#pragma unroll
        for (int kk = 0; kk < kTok / 16; ++kk) {
          const uint64_t dh = sdesc_sw128(fi + kk * 32, 16, 1024);
          const uint64_t dl = sdesc_sw128(fi + RK * 128 + kk * 32, 16, 1024);
          mma_f16_ss(tmem + kColS, da + 128 * kk, dh, idesc_s, t > 0 || kk > 0);
          mma_f16_ss(tmem + kColS, da + 128 * kk, dl, idesc_s, true);
        }
        mma_commit(bar(ctl->freed[s]));
        mma_commit(bar(ctl->img_free[t & 1]));
      }
      done = t + 1;
    }
    // ---- chunk end: S^T (lane = channel) and z
    if (issuer) {
      mma_commit(bar(ctl->drain));             // every MMA of this CTA has completed
      mbar_wait(bar(ctl->drain), 0, wc, false);
    }
    named_sync(1, 256);
    tc_fence_after();
    float* Sp = S_part + ((size_t)bh * dm.nchunk + chunk) * RK * kD;
    if (hf == 0) {                               // S^T spans the 128 lanes: warps 0-3 read it
      if (ok && done == ntiles && ntiles > 0) {
        float sv_[RK];
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * qd) << 16);
        tmem_ld32x32_x16(lane_addr + kColS, sv_);
        if constexpr (RK == 32) tmem_ld32x32_x16(lane_addr + kColS + 16, sv_ + 16);
        tmem_wait_ld();
#pragma unroll
        for (int a = 0; a < RK; ++a) Sp[(size_t)a * kD + 32 * qd + lane] = sv_[a];
      } else {
#pragma unroll
        for (int a = 0; a < RK; ++a) Sp[(size_t)a * kD + 32 * qd + lane] = 0.f;
      }
    }
    // z: the 16 token lanes of each half-warp hold the same rank values
#pragma unroll
    for (int a = 0; a < HR; ++a) {
      float x = zacc[a];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      if ((lane & 15) == 0) ctl->zred[qd][a0 + a] = x;
    }
    named_sync(1, 256);
    if (tid < RK)
      z_part[((size_t)bh * dm.nchunk + chunk) * RK + tid] =
          ((ctl->zred[0][tid] + ctl->zred[1][tid]) + ctl->zred[2][tid]) + ctl->zred[3][tid];
    tc_fence_before();
  } else if (warp < 10) {
    // ------------------------------------------------------------ k means (+ e4m3 k)
    const int cp = tid - 256;                     // channel pair 0..63
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kStages, n0 = n_begin + t * kTok;
      const bool ok = mbar_wait(bar(ctl->full[s]), (t / kStages) & 1, wc);
      if (named_vote_or(2, 64, !ok)) break;
      const uint8_t* pK = smem + G::offK + s * kTileBytes;
      const int cnt = min(kTok, n_end - n0), blk = n0 / kTok;
      float a0 = 0.f, a1 = 0.f, am = 0.f;
      const uint8_t* col = pK + (cp >> 5) * 8192 + (cp & 3) * 4;   // box, word in chunk
      const int ch = (cp >> 2) & 7;                                 // chunk within the box
      for (int r = 0; r < cnt; ++r) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(col + r * 128 + ((ch ^ (r & 7)) << 4));
        const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xffff0000u);
        a0 = a0 + x0;
        a1 = a1 + x1;
        if (FP8) am = fmaxf(am, fmaxf(fabsf(x0), fabsf(x1)));
      }
      *reinterpret_cast<float2*>(kbar + ((size_t)bh * dm.nb + blk) * kD + 2 * cp) =
          make_float2(__fdiv_rn(a0, (float)cnt), __fdiv_rn(a1, (float)cnt));
      if constexpr (FP8) {
        // e4m3 copy of the k tile: block scale from the max over the two warps
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        if (lane == 0) ctl->red[warp - 8] = am;
        named_sync(2, 64);
        am = fmaxf(ctl->red[0], ctl->red[1]);
        const float sc = am > 0.f ? am / 448.f : 1.f, inv = 1.f / sc;
        if (cp == 0) sk[(size_t)bh * dm.nb + blk] = sc;
        for (int e = cp; e < cnt * 16; e += 64) {
          const int r = e >> 4, cv = e & 15;
          *reinterpret_cast<uint2*>(k8 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
              e4m3x8(*reinterpret_cast<const uint4*>(pK + swz(r, cv)), inv);
        }
        named_sync(2, 64);                         // red is rewritten next tile
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ctl->freed[s]));
    }
  } else {
    // ------------------------------------------------------------ copy of v
    const int tv = tid - 320;                     // 0..63
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kStages, n0 = n_begin + t * kTok;
      const bool ok = mbar_wait(bar(ctl->full[s]), (t / kStages) & 1, wc);
      if (named_vote_or(3, 64, !ok)) break;
      const uint8_t* pV = smem + G::offV + s * kTileBytes;
      const int cnt = min(kTok, n_end - n0), blk = n0 / kTok;
      float am = 0.f;
      bool finite = true;
      if constexpr (!FP8) {
        // one pass with the block exponent 0 (the common case): fp16 copy and the block's
        // largest |v| together; a block that needs another exponent is rewritten below
        for (int e = tv; e < cnt * 16; e += 64) {
          const int r = e >> 4, cv = e & 15;
          const uint4 raw = *reinterpret_cast<const uint4*>(pV + swz(r, cv));
          const float m = absmax8(raw);
          finite &= m <= 3.402823466e38f;           // false for inf and nan
          am = fmaxf(am, m);
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t o[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const __half2 hv = __floats2half2_rn(__uint_as_float(w[u] << 16), __uint_as_float(w[u] & 0xffff0000u));
            o[u] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(v16 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
      } else {
        for (int e = tv; e < cnt * 16; e += 64) {
          const float m = absmax8(*reinterpret_cast<const uint4*>(pV + swz(e >> 4, e & 15)));
          finite &= m <= 3.402823466e38f;
          am = fmaxf(am, m);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      if (lane == 0) ctl->red[4 + warp - 10] = am;
      finite = !named_vote_or(3, 64, !finite);     // also orders the red writes
      am = fmaxf(ctl->red[4], ctl->red[5]);
      if (!finite && tv == 0) record_status(status, kDevRange);
      if constexpr (!FP8) {
        // the block's exponent: v is carried as v * 2^-e in fp16
        const int ex = v16_exponent(am);
        if (tv == 0) vexp[(size_t)bh * dm.nb + blk] = ex;
        if (ex != 0) {
          for (int e = tv; e < cnt * 16; e += 64) {
            const int r = e >> 4, cv = e & 15;
            const uint4 raw = *reinterpret_cast<const uint4*>(pV + swz(r, cv));
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
            uint32_t o[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const __half2 hv = __floats2half2_rn(ldexpf(__uint_as_float(w[u] << 16), -ex),
                                                   ldexpf(__uint_as_float(w[u] & 0xffff0000u), -ex));
              o[u] = *reinterpret_cast<const uint32_t*>(&hv);
            }
            *reinterpret_cast<uint4*>(v16 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
                make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      } else {
        const float sc = am > 0.f ? am / 448.f : 1.f, inv = 1.f / sc;
        if (tv == 0) sv[(size_t)bh * dm.nb + blk] = sc;
        for (int e = tv; e < cnt * 16; e += 64) {
          const int r = e >> 4, cv = e & 15;
          *reinterpret_cast<uint2*>(v8 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
              e4m3x8(*reinterpret_cast<const uint4*>(pV + swz(r, cv)), inv);
        }
      }
      named_sync(3, 64);                           // red is rewritten next tile
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ctl->freed[s]));
    }
  }

  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int RK, bool FP8>
cudaError_t launch_variant(const Dims& dm, const void* k, const void* v, const void* Wk, const Workspace& ws,
                           cudaStream_t st) {
  constexpr size_t smem = kv_smem_bytes<RK>();
  cudaError_t e = cudaFuncSetAttribute(kv_pass_kernel<RK, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  CUtensorMap tk, tv;
  if (!make_act_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, dm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  dim3 grid(dm.nchunk, dm.B * dm.H);
  kv_pass_kernel<RK, FP8><<<grid, kThreads, smem, st>>>(
      tk, tv, static_cast<const __nv_bfloat16*>(Wk), dm, ws.rope, ws.S_part, ws.z_part, ws.kbar, ws.v16, ws.vexp,
      ws.k8, ws.v8, ws.sk, ws.sv, ws.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_pass(const Dims& dm, bool fp8, const void* k, const void* v, const void* Wk,
                           const Workspace& ws, cudaStream_t st) {
  if (dm.r == 32)
    return fp8 ? launch_variant<32, true>(dm, k, v, Wk, ws, st) : launch_variant<32, false>(dm, k, v, Wk, ws, st);
  return fp8 ? launch_variant<16, true>(dm, k, v, Wk, ws, st) : launch_variant<16, false>(dm, k, v, Wk, ws, st);
}

}  // namespace rola
