// Query pass of the RoLA forward for head dim 128 with bf16 inputs: one read of each
// (b, h, 64-token query block i) computes
//   * the block mean of q (step 1, query side): fp32 sums in token order, one division;
//   * fp8 configuration: the e4m3 copy of q with its block scale (absmax / 448, 1 for an
//     all-zero block; code = RN-sat(x * (1 / scale)));
//   * the query side of the linear branch (step 5):
//       u_n = phi(q_n Wq_h)            (r values per token, phi = elu + 1)
//       gden_n = g / (u_n . z_h)       (the gain over the unrotated normaliser; g = g_h,
//                                       g_{n,h} for a per-token gate, or the gate computed
//                                       from the query, sigmoid(q_n . wg_h + bg_h))
//       (R(p_n) u_n) split into bf16 hi + lo, stored transposed ([rank][64 tokens]) as the
//       exact 128-byte-swizzled shared-memory image the attention epilogue multiplies
//       with S_h on the tensor cores (one bulk copy there, no per-element work).
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (high-energy block selection; low-rank
// linear branch with rotary positions); README sparse-finetuning section (proj_q; the
// gate read as a gain per head, per token and head, or computed from the query by
// gate_proj and gate_bias).
//
// Layout of the work (as the key/value pass): a CTA owns one (b, h) and a chunk of whole
// query blocks; q tiles (two TMA boxes of 64 tokens x 64 channels, 128-byte swizzle) flow
// through a ring filled by a producer warp, two CTAs per SM.  One thread issues, a tile
// ahead and into one of two TMEM buffers,
//   U = Q [Wq_h | wg_h hi | wg_h lo]   tcgen05, M = 64 tokens, N = r (+ 8), K = 128
// (the gate's projection rides along as two extra B rows, gate_proj split into bf16 hi +
// lo, so q . wg comes out of the same MMA to ~2^-16); warps 0-7 then take one token
// and a quarter of the r values each (phi, den, rotation, the image, g/den: two warps
// per TMEM lane quadrant, so that twice as many warps hide the latencies of the per-token
// work), while warps 8-9 take the block mean and, fp8, warps 10-11 the block's absmax
// and the e4m3 copy.  Every wait is bounded.
#include "rola_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda_fp8.h>

namespace rola {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kStages = 3;
// warps 0-7 features, 8-9 means, (fp8: 10-11 the e4m3 copy), then the TMA producer
template <bool FP8>
struct QRoles {
  static constexpr int kTmaWarp = FP8 ? 12 : 10;
  static constexpr int kThreads = 32 * (kTmaWarp + 1);
};
constexpr uint32_t kTileBytes = kBlock * kD * 2;
constexpr uint32_t kTmemCols = 128;           // two U buffers of up to 40 columns, 64 apart

__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((c >> 3) * 8192 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Byte offset of element (row, col) of a K-major 128-byte-swizzled bf16 operand image.
__device__ __forceinline__ uint32_t img_off(int row, int col) {
  return (uint32_t)(row * 128 + ((((col >> 3) ^ row) & 7) << 4) + (col & 7) * 2);
}

// B rows of U = Q B^T: the r columns of Wq_h, then (gate from the query) wg hi, wg lo and
// zero rows up to a multiple of 8.
template <int RK, bool QG>
struct QGeo {
  static constexpr int NB = QG ? RK + 8 : RK;
  static constexpr uint32_t kBox = ((NB * 128 + 1023) / 1024) * 1024;    // one 64-channel box of B
  static constexpr uint32_t offQ = 0;                                    // kStages q tiles
  static constexpr uint32_t offW = offQ + kStages * kTileBytes;          // B: 2 boxes [NB][64 ch]
  static constexpr uint32_t kImg = 2 * RK * 128;                         // (R u)^T hi | lo
  static constexpr uint32_t offImg = offW + 2 * kBox;                    // two images
  static constexpr uint32_t offCtl = offImg + 2 * kImg;
};

struct QCtl {
  uint64_t full[kStages], freed[kStages], u_full[2], drain;
  uint32_t tmem_base;
  int abort;
  float red[4];
  float dpart[4][16];     // per quadrant and row: den over the upper half of the ranks
};

template <int RK, bool QG>
constexpr size_t q_smem_bytes() { return QGeo<RK, QG>::offCtl + sizeof(QCtl) + 1024; }

__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(x0, x1);
  const float2 bf = __bfloat1622float2(b);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - bf.x, x1 - bf.y);
  hi = *reinterpret_cast<const uint32_t*>(&b);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// TMEM lanes 0-15 of the warp's quadrant (the M = 64 layout): threads 0-15 read n
// consecutive columns, threads 16-31 the n columns after them.
template <int N>
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, float* v);
template <>
__device__ __forceinline__ void tmem_ld16x2<16>(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16], 16;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld16x2<8>(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], 8;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld16x2<4>(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x4.b32 {%0, %1, %2, %3}, [%4], 4;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld16x2<1>(uint32_t taddr, float* v) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x1.b32 {%0}, [%1], 1;" : "=r"(r[0]) : "r"(taddr) : "memory");
}

template <int RK, bool FP8, bool QG>
__global__ void __launch_bounds__(QRoles<FP8>::kThreads, 2) query_features_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __nv_bfloat16* __restrict__ Wq, const float* __restrict__ g,
    Dims dm, const float* __restrict__ z, const float2* __restrict__ rope, float* __restrict__ qbar,
    uint8_t* __restrict__ uimg, float* __restrict__ gden, uint8_t* __restrict__ q8, float* __restrict__ sq,
    int* __restrict__ status) {
  using G = QGeo<RK, QG>;
  constexpr int NB = G::NB;
  constexpr uint32_t kBox = G::kBox;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  QCtl* ctl = reinterpret_cast<QCtl*>(smem + G::offCtl);
  auto bar = [&](uint64_t& m) { return smem_addr(&m); };

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const int n_begin = chunk * dm.chunk_tok;
  const int n_end = min(dm.N, n_begin + dm.chunk_tok);
  const int ntiles = n_end > n_begin ? (n_end - n_begin + kBlock - 1) / kBlock : 0;
  const size_t rs = (size_t)dm.H * kD;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(ctl->full[s]), 1);
      mbar_init(bar(ctl->freed[s]), FP8 ? 5 : 3);   // the U MMAs' commit + warps 8-9 (10-11)
    }
    mbar_init(bar(ctl->u_full[0]), 1);
    mbar_init(bar(ctl->u_full[1]), 1);
    mbar_init(bar(ctl->drain), 1);
    ctl->abort = 0;
    fence_barrier_init();
  }
  // B = [Wq_h^T; wg hi; wg lo; 0]: row a, channel c in box c / 64 (K-major, 128-byte swizzle)
  for (int e = tid; e < kD * NB; e += QRoles<FP8>::kThreads) {
    const int c = e / NB, a = e % NB;
    __nv_bfloat16 val;
    if (a < RK) {
      val = Wq[((size_t)h * kD + c) * RK + a];
    } else {
      const float wg = (QG && a < RK + 2) ? __ldg(g + (size_t)h * kD + c) : 0.f;
      const __nv_bfloat16 whi = __float2bfloat16_rn(wg);
      val = a == RK ? whi : __float2bfloat16_rn(a == RK + 1 ? wg - __bfloat162float(whi) : 0.f);
    }
    *reinterpret_cast<__nv_bfloat16*>(smem + G::offW + (c >> 6) * kBox + img_off(a, c & 63)) = val;
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

  if (warp == QRoles<FP8>::kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % kStages;
        if (t >= kStages && !mbar_wait(bar(ctl->freed[s]), ((t / kStages) - 1) & 1, wc)) break;
        const uint32_t fb = bar(ctl->full[s]);
        mbar_expect_tx(fb, kTileBytes);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sbase + G::offQ + s * kTileBytes + c * 8192, &tm_q, h * kD + 64 * c, n_begin + t * kBlock, b,
                      fb);
        issued = t + 1;
      }
      for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
        mbar_wait(bar(ctl->full[t % kStages]), (t / kStages) & 1, wc, false);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ U and the features
    const bool issuer = warp == 0 && lane == 0;
    constexpr uint32_t idesc_u = idesc_f16(1, 64, NB, 0, 0);
    constexpr int HR = RK / 4;                  // rank values of a thread
    const int qd = warp & 3, hf = warp >> 2;    // TMEM lane quadrant; half of the ranks
    const int row = 16 * qd + (lane & 15);      // token of the tile
    const int a0 = hf * (RK / 2) + (lane >> 4) * HR;   // first rank value of this thread
    float zr[HR];
#pragma unroll
    for (int a = 0; a < HR; ++a) zr[a] = __ldg(z + (size_t)bh * RK + a0 + a);
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * qd) << 16);
    bool ok = true;
    // U of tile t goes to TMEM buffer t & 1 and is issued one tile ahead, so that the
    // MMA's latency overlaps the features of the tile before
    auto issue_u = [&](int t) {
      const int s = t % kStages;
      if (!mbar_wait(bar(ctl->full[s]), (t / kStages) & 1, wc)) return false;
      tc_fence_after();
      const uint32_t tq = sbase + G::offQ + s * kTileBytes;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk)
        mma_f16_ss(tmem + 64 * (t & 1), sdesc_sw128(tq + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                   sdesc_sw128(sbase + G::offW + (kk >> 2) * kBox + (kk & 3) * 32, 16, 1024), idesc_u, kk > 0);
      mma_commit(bar(ctl->u_full[t & 1]));
      mma_commit(bar(ctl->freed[s]));
      return true;
    };
    // (the MMA of tile t + 1 is issued early only if its tile has already landed)
    int nu = 0;                                   // U MMAs issued (issuer thread)
    for (int t = 0; t < ntiles; ++t) {
      const int i = n_begin / kBlock + t, n = i * kBlock + row;
      if (issuer && ok) {
        if (nu == t) { ok = issue_u(t); ++nu; }
        if (ok && nu == t + 1 && t + 1 < ntiles &&
            mbar_test_wait(bar(ctl->full[(t + 1) % kStages]), ((t + 1) / kStages) & 1)) {
          ok = issue_u(t + 1);
          ++nu;
        }
      }
      // one barrier per tile (after the image): a failed wait is carried to it, and
      // tcgen05.ld runs on the whole converged warp whatever its lanes' waits returned
      if (ok) ok = mbar_wait(bar(ctl->u_full[t & 1]), (t >> 1) & 1, wc);
      __syncwarp();
      tc_fence_after();
      float u[HR], gl = 0.f;
      const uint32_t ub = lane_addr + 64 * (t & 1);
      tmem_ld16x2<HR>(ub + hf * (RK / 2), u);
      // q . wg hi (threads 0-15), lo (16-31): read by the warps that write g/den
      if (QG && hf == 0) tmem_ld16x2<1>(ub + RK, &gl);
      tmem_wait_ld();
      tc_fence_before();       // U(t)'s buffer is next written by the MMA of tile t + 2, issued
                               // after this tile's closing barrier
      const bool valid = n < dm.N;
      if constexpr (QG) gl += __shfl_xor_sync(0xffffffffu, gl, 16);
      const TokPos pos = token_pos(dm, valid ? n : 0);
      uint8_t* img = smem + G::offImg + (t & 1) * G::kImg;
      float den = 0.f;
#pragma unroll
      for (int p = 0; p < HR / 2; ++p) {
        const float x0 = phi_fast(u[2 * p]), x1 = phi_fast(u[2 * p + 1]);
        den = fmaf(x0, zr[2 * p], fmaf(x1, zr[2 * p + 1], den));
        const float2 cs = valid ? rope_at(dm, rope, pos, a0 / 2 + p) : make_float2(1.f, 0.f);
        uint32_t hi, lo;
        split_bf16x2(cs.x * x0 - cs.y * x1, cs.y * x0 + cs.x * x1, hi, lo);
        const int a = a0 + 2 * p;
        *reinterpret_cast<uint16_t*>(img + img_off(a, row)) = (uint16_t)(hi & 0xffffu);
        *reinterpret_cast<uint16_t*>(img + img_off(a + 1, row)) = (uint16_t)(hi >> 16);
        *reinterpret_cast<uint16_t*>(img + RK * 128 + img_off(a, row)) = (uint16_t)(lo & 0xffffu);
        *reinterpret_cast<uint16_t*>(img + RK * 128 + img_off(a + 1, row)) = (uint16_t)(lo >> 16);
      }
      den += __shfl_xor_sync(0xffffffffu, den, 16);
      if (hf == 1 && lane < 16) ctl->dpart[qd][lane] = den;
      // the image and the partial dens are complete (and U(t) is read: its buffer may be
      // refilled)
      if (named_vote_or(1, 256, !ok)) { ok = false; break; }
      if (hf == 0 && lane < 16) {
        // gain of the token: read, or sigmoid(q . wg + bg)
        const float gh = QG ? gate_sigmoid(dm, g, h, gl) : (valid ? g[gain_index(dm, b, n, h)] : 0.f);
        den += ctl->dpart[qd][lane];
        gden[((size_t)bh * dm.nb + i) * kBlock + row] = valid ? gh / den : 0.f;
      }
      uint4* dst = reinterpret_cast<uint4*>(uimg + ((size_t)bh * dm.nb + i) * G::kImg);
      const uint4* src = reinterpret_cast<const uint4*>(img);
      for (int e = tid; e < (int)(G::kImg / 16); e += 256) dst[e] = src[e];
    }
    if (issuer) {
      mma_commit(bar(ctl->drain));             // no MMA may run when TMEM is freed
      mbar_wait(bar(ctl->drain), 0, wc, false);
    }
    tc_fence_before();
  } else if (warp < 10) {
    // ------------------------------------------------------------ block mean
    const int cp = tid - 256;                     // channel pair 0..63
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kStages, n0 = n_begin + t * kBlock, i = n0 / kBlock;
      const bool ok = mbar_wait(bar(ctl->full[s]), (t / kStages) & 1, wc);
      if (named_vote_or(2, 64, !ok)) break;
      const uint8_t* pQ = smem + G::offQ + s * kTileBytes;
      const int cnt = min(kBlock, dm.N - n0);
      float a0 = 0.f, a1 = 0.f;
      const uint8_t* col = pQ + (cp >> 5) * 8192 + (cp & 3) * 4;   // box, word in chunk
      const int ch = (cp >> 2) & 7;                                 // chunk within the box
      for (int r = 0; r < cnt; ++r) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(col + r * 128 + ((ch ^ (r & 7)) << 4));
        add2(a0, a1, __uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));   // token order, as fadd
      }
      *reinterpret_cast<float2*>(qbar + ((size_t)bh * dm.nb + i) * kD + 2 * cp) =
          make_float2(__fdiv_rn(a0, (float)cnt), __fdiv_rn(a1, (float)cnt));
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(ctl->freed[s]));
    }
  } else if (FP8) {
    // ------------------------------------------------------------ e4m3 copy of q
    // (its own warps, beside the means: the block's absmax, then every code)
    const int tq = tid - 320;                     // 0..63
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kStages, n0 = n_begin + t * kBlock, i = n0 / kBlock;
      const bool ok = mbar_wait(bar(ctl->full[s]), (t / kStages) & 1, wc);
      if (named_vote_or(3, 64, !ok)) break;
      const uint8_t* pQ = smem + G::offQ + s * kTileBytes;
      const int cnt = min(kBlock, dm.N - n0);
      uint32_t amb = 0;   // largest |q| of the thread's elements, as bf16 patterns
      for (int e = tq; e < cnt * 16; e += 64)
        amb = __vmaxu2(amb, bf16x8_absmax_bits(*reinterpret_cast<const uint4*>(pQ + swz(e >> 4, e & 15))));
      float am = bf16_absmax_value(amb);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      if (lane == 0) ctl->red[warp - 10] = am;
      named_sync(3, 64);
      am = fmaxf(ctl->red[0], ctl->red[1]);
      const float scale = am > 0.f ? am / 448.f : 1.f, inv = 1.f / scale;
      if (tq == 0) sq[(size_t)bh * dm.nb + i] = scale;
      for (int e = tq; e < cnt * 16; e += 64) {
        const int r = e >> 4, cv = e & 15;
        const uint4 v = *reinterpret_cast<const uint4*>(pQ + swz(r, cv));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[2] = {0, 0};
#pragma unroll
        for (int u = 0; u < 4; ++u) {   // each product rounded as a scalar multiply, two per f32x2
          float x0 = __uint_as_float(w[u] << 16), x1 = __uint_as_float(w[u] & 0xffff0000u);
          mul2(x0, x1, inv, inv);
          o[u >> 1] |= (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3) << (16 * (u & 1));
        }
        *reinterpret_cast<uint2*>(q8 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
            make_uint2(o[0], o[1]);
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

template <int RK, bool FP8, bool QG>
cudaError_t launch_variant(const Dims& dm, const void* q, const void* Wq, const float* g, const Workspace& ws,
                           cudaStream_t st) {
  constexpr size_t smem = q_smem_bytes<RK, QG>();
  cudaError_t e = cudaFuncSetAttribute(query_features_kernel<RK, FP8, QG>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  CUtensorMap tq;
  if (!make_act_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  dim3 grid(dm.nchunk, dm.B * dm.H);
  query_features_kernel<RK, FP8, QG><<<grid, QRoles<FP8>::kThreads, smem, st>>>(
      tq, static_cast<const __nv_bfloat16*>(Wq), g, dm, ws.z, ws.rope, ws.qbar, ws.uimg, ws.gden,
      FP8 ? ws.q8 : nullptr, FP8 ? ws.sq : nullptr, ws.status);
  return cudaGetLastError();
}

template <int RK, bool FP8>
cudaError_t launch_gate(const Dims& dm, const void* q, const void* Wq, const float* g, const Workspace& ws,
                        cudaStream_t st) {
  return dm.gate_mode == ROLA_GATE_QPROJ ? launch_variant<RK, FP8, true>(dm, q, Wq, g, ws, st)
                                         : launch_variant<RK, FP8, false>(dm, q, Wq, g, ws, st);
}

}  // namespace

cudaError_t launch_query_features(const Dims& dm, bool fp8, const void* q, const void* Wq, const float* g,
                                  const Workspace& ws, cudaStream_t st) {
  if (dm.r == 32)
    return fp8 ? launch_gate<32, true>(dm, q, Wq, g, ws, st) : launch_gate<32, false>(dm, q, Wq, g, ws, st);
  return fp8 ? launch_gate<16, true>(dm, q, Wq, g, ws, st) : launch_gate<16, false>(dm, q, Wq, g, ws, st);
}

}  // namespace rola
