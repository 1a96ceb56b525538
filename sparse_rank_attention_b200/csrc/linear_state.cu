// Linear-branch state of RoLA (key side of step 4): for every (b, h)
//   S_h = sum_m R(p_m) phi(k_m Wk_h) v_m^T   (r x d),   z_h = sum_m phi(k_m Wk_h)   (r)
// over all N keys, phi = elu + 1, R(p) the 3D rotary map on the r/2 adjacent pairs.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (low-rank linear branch with rotary
// positions restores global context); README sparse-finetuning section (proj_k);
// citation block "RoPeSLR: 3D RoPE-driven Sparse-LowRank Attention" (3D rotary).
//
// Split-N: each CTA sums one chunk of tokens into a partial; a second kernel adds the
// partials in chunk order, so the result does not depend on scheduling.  (For head dim
// 128 with bf16 inputs the key/value pass computes the partials instead.)
#include "rola_internal.cuh"
#include "warp_mma.cuh"

#include <cuda_fp8.h>

namespace rola {
namespace {

// (cos, sin) of pos * base^(-c'/P_axis) for every axis position and in-axis pair,
// evaluated in double and rounded to fp32.  Layout: t axis [gt][pt], then h [gh][ph],
// then w [gw][pw].
__global__ void rope_table_kernel(Dims dm, float2* __restrict__ rope) {
  const int total = dm.rope_off_w + dm.gw * dm.pw;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
    int pos, cp, cnt;
    if (e < dm.rope_off_h) {
      pos = e / dm.pt; cp = e % dm.pt; cnt = dm.pt;
    } else if (e < dm.rope_off_w) {
      const int e2 = e - dm.rope_off_h;
      pos = e2 / dm.ph; cp = e2 % dm.ph; cnt = dm.ph;
    } else {
      const int e2 = e - dm.rope_off_w;
      pos = e2 / dm.pw; cp = e2 % dm.pw; cnt = dm.pw;
    }
    const double theta = (double)pos * pow(dm.rope_base, -(double)cp / (double)cnt);
    double s, c;
    sincos(theta, &s, &c);
    rope[e] = make_float2((float)c, (float)s);
  }
}

// ------------------------------------------------------------------ bf16 inputs

constexpr int kLSTile = 64;

template <int D, int RK>
struct LSSmem {
  static constexpr int DP = D + 8;   // padded row (bf16 elements): ldmatrix without conflicts
  static constexpr int RP = RK + 8;
  static constexpr int kW = RK * DP;          // WkT [r][d]
  static constexpr int kTileElems = kLSTile * DP;
  static constexpr int kF = kLSTile * RP;     // rotated features [tok][r] (hi and lo parts)
  static constexpr size_t bytes = sizeof(__nv_bfloat16) * (kW + 4 * kTileElems + 2 * kF) +
                                  sizeof(float) * (4 * RK + 4);   // z partials, v block maxima
};

// grid: x = chunk, y = b*H + h; 128 threads (4 warps).
//   A: F = K_tile Wk       (warp w: tokens 16w..16w+15, all r)       mma m16n8k16
//   B: phi, z, rotation    (in registers; rotary pairs are adjacent accumulator columns);
//      the rotated features are split into bf16 hi + lo parts (F = hi + lo to ~2^-17)
//   C: S += R(F)^T V_tile  (warp w: d columns [w*D/4, (w+1)*D/4))    2 x mma m16n8k16
// The kernel also writes the fp16 copy of v that the attention kernel multiplies the
// fp16 softmax weights with (one power-of-two exponent per block, see v16_exponent), and
// flags non-finite values.
template <int D, int RK, bool FP8>
__global__ void __launch_bounds__(128) linear_state_bf16_kernel(
    const __nv_bfloat16* __restrict__ kin, const __nv_bfloat16* __restrict__ vin,
    const __nv_bfloat16* __restrict__ Wk, Dims dm, const float2* __restrict__ rope,
    float* __restrict__ S_part, float* __restrict__ z_part, __half* __restrict__ v16,
    int* __restrict__ vexp, uint8_t* __restrict__ v8, float* __restrict__ sv, int* __restrict__ status) {
  using L = LSSmem<D, RK>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __nv_bfloat16* sW = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sK = sW + L::kW;                     // [2][tile]
  __nv_bfloat16* sV = sK + 2 * L::kTileElems;         // [2][tile]
  __nv_bfloat16* sF = sV + 2 * L::kTileElems;       // hi part
  __nv_bfloat16* sFl = sF + L::kF;                    // lo part
  float* sZ = reinterpret_cast<float*>(sFl + L::kF);  // [4][RK] z partials, then 4 maxima of v

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const int n_begin = chunk * dm.chunk_tok;
  const int n_end = min(dm.N, n_begin + dm.chunk_tok);
  const int ntiles = (n_end - n_begin + kLSTile - 1) / kLSTile;
  const size_t row_stride = (size_t)dm.H * D;  // elements between tokens
  const __nv_bfloat16* kbase = kin + ((size_t)b * dm.N) * row_stride + (size_t)h * D;
  const __nv_bfloat16* vbase = vin + ((size_t)b * dm.N) * row_stride + (size_t)h * D;

  // WkT[a][c] = Wk[h][c][a]  (plain loads, once)
  for (int e = tid; e < D * RK; e += 128) {
    const int c = e / RK, a = e % RK;
    sW[a * L::DP + c] = Wk[((size_t)h * D + c) * RK + a];
  }

  auto load_tile = [&](int tile, int stage) {
    const int n0 = n_begin + tile * kLSTile;
    constexpr int kVecPerRow = D / 8;
    for (int e = tid; e < kLSTile * kVecPerRow; e += 128) {
      const int rr = e / kVecPerRow, cv = e % kVecPerRow;
      const int n = n0 + rr;
      const bool ok = n < n_end;
      const size_t off = (size_t)(ok ? n : n_begin) * row_stride + cv * 8;
      cp_async16(smem_u32(sK + stage * L::kTileElems + rr * L::DP + cv * 8), kbase + off, ok ? 16 : 0);
      cp_async16(smem_u32(sV + stage * L::kTileElems + rr * L::DP + cv * 8), vbase + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  constexpr int NT_F = RK / 8;        // n-tiles of F
  constexpr int MT_S = RK / 16;       // m-tiles of S
  constexpr int NT_S = D / 4 / 8;     // n-tiles of S per warp
  float sacc[MT_S][NT_S][4];
#pragma unroll
  for (int a = 0; a < MT_S; ++a)
#pragma unroll
    for (int c = 0; c < NT_S; ++c)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[a][c][e] = 0.f;
  float zacc[NT_F][2];
#pragma unroll
  for (int a = 0; a < NT_F; ++a) zacc[a][0] = zacc[a][1] = 0.f;

  load_tile(0, 0);
  for (int tile = 0; tile < ntiles; ++tile) {
    const int stage = tile & 1;
    if (tile + 1 < ntiles) {
      load_tile(tile + 1, stage ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* tK = sK + stage * L::kTileElems;
    const __nv_bfloat16* tV = sV + stage * L::kTileElems;

    if constexpr (!FP8) {
      // fp16 copy of the V tile (one 64-token block) as v * 2^-e, e from the block's
      // largest |v| (v16_exponent); non-finite values set ROLA_ERR_RANGE
      constexpr int kVecPerRow = D / 8;
      const int n0 = n_begin + tile * kLSTile;
      float amax = 0.f;
      bool finite = true;
      for (int e = tid; e < kLSTile * kVecPerRow; e += 128) {
        const int rr = e / kVecPerRow, cv = e % kVecPerRow;
        if (n0 + rr >= n_end) continue;
        const uint4 raw = *reinterpret_cast<const uint4*>(tV + rr * L::DP + cv * 8);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float m = fmaxf(fabsf(__uint_as_float(w[t] << 16)), fabsf(__uint_as_float(w[t] & 0xffff0000u)));
          finite &= m <= 3.402823466e38f;
          amax = fmaxf(amax, m);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (lane == 0) sZ[4 * RK + warp] = amax;
      finite = __syncthreads_and(finite);
      amax = fmaxf(fmaxf(sZ[4 * RK], sZ[4 * RK + 1]), fmaxf(sZ[4 * RK + 2], sZ[4 * RK + 3]));
      if (!finite && tid == 0) record_status(status, kDevRange);
      const int ex = finite ? v16_exponent(amax) : 0;
      if (tid == 0) vexp[(size_t)bh * dm.nb + n0 / kLSTile] = ex;
      for (int e = tid; e < kLSTile * kVecPerRow; e += 128) {
        const int rr = e / kVecPerRow, cv = e % kVecPerRow, n = n0 + rr;
        if (n >= n_end) continue;
        const uint4 raw = *reinterpret_cast<const uint4*>(tV + rr * L::DP + cv * 8);
        const __nv_bfloat162* src = reinterpret_cast<const __nv_bfloat162*>(&raw);
        uint4 packed;
        __half2* dst = reinterpret_cast<__half2*>(&packed);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          float2 f = __bfloat1622float2(src[t]);
          if (ex != 0) {
            f.x = ldexpf(f.x, -ex);
            f.y = ldexpf(f.y, -ex);
          }
          dst[t] = __floats2half2_rn(f.x, f.y);
        }
        *reinterpret_cast<uint4*>(v16 + ((size_t)b * dm.N + n) * row_stride + (size_t)h * D + cv * 8) =
            packed;
      }
      __syncthreads();                             // sZ's maxima are rewritten next tile
    } else {
      // e4m3 copy of the V tile: the tile is one 64-token block; scale = absmax / 448.
      constexpr int kVecPerRow = D / 8;
      const int n0 = n_begin + tile * kLSTile;
      float amax = 0.f;
      for (int e = tid; e < kLSTile * kVecPerRow; e += 128) {
        const int rr = e / kVecPerRow, cv = e % kVecPerRow;
        if (n0 + rr >= n_end) continue;
        const uint4 raw = *reinterpret_cast<const uint4*>(tV + rr * L::DP + cv * 8);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
          amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w[t] << 16)), fabsf(__uint_as_float(w[t] & 0xffff0000u))));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if (lane == 0) sZ[warp] = amax;   // sZ is free until the end of the chunk loop
      __syncthreads();
      amax = fmaxf(fmaxf(sZ[0], sZ[1]), fmaxf(sZ[2], sZ[3]));
      __syncthreads();
      const float scale = amax > 0.f ? amax / 448.f : 1.f, inv = 1.f / scale;
      if (tid == 0) sv[(size_t)bh * dm.nb + n0 / kLSTile] = scale;
      for (int e = tid; e < kLSTile * kVecPerRow; e += 128) {
        const int rr = e / kVecPerRow, cv = e % kVecPerRow, n = n0 + rr;
        if (n >= n_end) continue;
        const uint4 raw = *reinterpret_cast<const uint4*>(tV + rr * L::DP + cv * 8);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t o[2] = {0, 0};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float2 f = make_float2(__uint_as_float(w[t] << 16) * inv, __uint_as_float(w[t] & 0xffff0000u) * inv);
          o[t >> 1] |= (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3) << (16 * (t & 1));
        }
        *reinterpret_cast<uint2*>(v8 + ((size_t)b * dm.N + n) * row_stride + (size_t)h * D + cv * 8) =
            make_uint2(o[0], o[1]);
      }
    }

    // A: F = K Wk
    float f[NT_F][4];
#pragma unroll
    for (int a = 0; a < NT_F; ++a)
#pragma unroll
      for (int e = 0; e < 4; ++e) f[a][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(smem_u32(tK + (16 * warp + (lane & 15)) * L::DP + kk * 16 + (lane >> 4) * 8), af[0],
              af[1], af[2], af[3]);
#pragma unroll
      for (int nt = 0; nt < NT_F; nt += 2) {
        const int q = lane >> 3;
        uint32_t bf[4];
        ldsm_x4(smem_u32(sW + ((nt + (q >> 1)) * 8 + (lane & 7)) * L::DP + kk * 16 + (q & 1) * 8),
                bf[0], bf[1], bf[2], bf[3]);
        mma_bf16(f[nt], af, bf);
        mma_bf16(f[nt + 1], af, bf + 2);
      }
    }
    // B: phi, z, rotation -> sF (bf16)
    const int n_tile0 = n_begin + tile * kLSTile;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = 16 * warp + g + 8 * half;
      const int n = n_tile0 + row;
      const bool ok = n < n_end;
#pragma unroll
      for (int nt = 0; nt < NT_F; ++nt) {
        float x0 = ok ? phi(f[nt][2 * half]) : 0.f;
        float x1 = ok ? phi(f[nt][2 * half + 1]) : 0.f;
        zacc[nt][0] += x0;
        zacc[nt][1] += x1;
        const float2 cs = ok ? rope_cs(dm, rope, n, nt * 4 + t4) : make_float2(1.f, 0.f);
        const float y0 = cs.x * x0 - cs.y * x1;
        const float y1 = cs.y * x0 + cs.x * x1;
        const uint32_t hi = pack_bf16(y0, y1);
        const float2 hf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hi));
        *reinterpret_cast<uint32_t*>(sF + row * L::RP + nt * 8 + 2 * t4) = hi;
        *reinterpret_cast<uint32_t*>(sFl + row * L::RP + nt * 8 + 2 * t4) =
            pack_bf16(y0 - hf.x, y1 - hf.y);
      }
    }
    __syncthreads();
    // C: S += F^T V over the tile's 64 tokens
    const int colbase = warp * (D / 4);
#pragma unroll
    for (int kk = 0; kk < kLSTile / 16; ++kk) {
      const int q = lane >> 3;
      uint32_t af[MT_S][4], al[MT_S][4];
#pragma unroll
      for (int mt = 0; mt < MT_S; ++mt) {
        const int off = (kk * 16 + (q >> 1) * 8 + (lane & 7)) * L::RP + mt * 16 + (q & 1) * 8;
        ldsm_x4_t(smem_u32(sF + off), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
        ldsm_x4_t(smem_u32(sFl + off), al[mt][0], al[mt][1], al[mt][2], al[mt][3]);
      }
#pragma unroll
      for (int nt = 0; nt < NT_S; nt += 2) {
        uint32_t bf[4];
        ldsm_x4_t(smem_u32(tV + (kk * 16 + (q & 1) * 8 + (lane & 7)) * L::DP + colbase +
                           (nt + (q >> 1)) * 8),
                  bf[0], bf[1], bf[2], bf[3]);
#pragma unroll
        for (int mt = 0; mt < MT_S; ++mt) {
          mma_bf16(sacc[mt][nt], af[mt], bf);
          mma_bf16(sacc[mt][nt + 1], af[mt], bf + 2);
          mma_bf16(sacc[mt][nt], al[mt], bf);
          mma_bf16(sacc[mt][nt + 1], al[mt], bf + 2);
        }
      }
    }
    __syncthreads();
  }

  // partial S
  float* Sp = S_part + (((size_t)bh * dm.nchunk + chunk) * RK) * D;
  const int colbase = warp * (D / 4);
#pragma unroll
  for (int mt = 0; mt < MT_S; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT_S; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = mt * 16 + g + 8 * hh;
        const int col = colbase + nt * 8 + 2 * t4;
        *reinterpret_cast<float2*>(Sp + (size_t)row * D + col) =
            make_float2(sacc[mt][nt][2 * hh], sacc[mt][nt][2 * hh + 1]);
      }
  // partial z: lanes with equal t4 hold the same columns
#pragma unroll
  for (int nt = 0; nt < NT_F; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float x = zacc[nt][e];
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      if (g == 0) sZ[warp * RK + nt * 8 + 2 * t4 + e] = x;
    }
  __syncthreads();
  if (tid < RK) {
    const float x = ((sZ[tid] + sZ[RK + tid]) + sZ[2 * RK + tid]) + sZ[3 * RK + tid];
    z_part[((size_t)bh * dm.nchunk + chunk) * RK + tid] = x;
  }
}

// ------------------------------------------------------------------ fp32 inputs

// Plain fp32 arithmetic (the fp32 correctness configuration): same chunking.
template <int D, int RK>
__global__ void __launch_bounds__(128) linear_state_f32_kernel(
    const float* __restrict__ kin, const float* __restrict__ vin, const float* __restrict__ Wk,
    Dims dm, const float2* __restrict__ rope, float* __restrict__ S_part,
    float* __restrict__ z_part) {
  constexpr int T = 16;  // tokens per tile
  __shared__ float sK[T][D], sV[T][D], sW[D][RK], sFr[T][RK], sFu[T][RK];
  const int tid = threadIdx.x;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const int n_begin = chunk * dm.chunk_tok;
  const int n_end = min(dm.N, n_begin + dm.chunk_tok);
  const size_t row_stride = (size_t)dm.H * D;
  for (int e = tid; e < D * RK; e += 128) sW[e / RK][e % RK] = Wk[(size_t)h * D * RK + e];
  constexpr int kPer = (RK * D + 127) / 128;
  float sacc[kPer];
#pragma unroll
  for (int e = 0; e < kPer; ++e) sacc[e] = 0.f;
  float zacc = 0.f;
  for (int n0 = n_begin; n0 < n_end; n0 += T) {
    __syncthreads();
    for (int e = tid; e < T * D; e += 128) {
      const int rr = e / D, c = e % D, n = n0 + rr;
      const bool ok = n < n_end;
      const size_t off = ((size_t)b * dm.N + n) * row_stride + (size_t)h * D + c;
      sK[rr][c] = ok ? kin[off] : 0.f;
      sV[rr][c] = ok ? vin[off] : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < T * RK / 2; e += 128) {
      const int rr = e / (RK / 2), c = e % (RK / 2), n = n0 + rr;
      float f0 = 0.f, f1 = 0.f;
      for (int cc = 0; cc < D; ++cc) {
        f0 = fmaf(sK[rr][cc], sW[cc][2 * c], f0);
        f1 = fmaf(sK[rr][cc], sW[cc][2 * c + 1], f1);
      }
      const bool ok = n < n_end;
      f0 = ok ? phi(f0) : 0.f;
      f1 = ok ? phi(f1) : 0.f;
      const float2 cs = ok ? rope_cs(dm, rope, n, c) : make_float2(1.f, 0.f);
      sFu[rr][2 * c] = f0;
      sFu[rr][2 * c + 1] = f1;
      sFr[rr][2 * c] = cs.x * f0 - cs.y * f1;
      sFr[rr][2 * c + 1] = cs.y * f0 + cs.x * f1;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int idx = tid + e * 128;
      if (idx < RK * D) {
        const int a = idx / D, c = idx % D;
        float acc = sacc[e];
        for (int rr = 0; rr < T; ++rr) acc = fmaf(sFr[rr][a], sV[rr][c], acc);
        sacc[e] = acc;
      }
    }
    if (tid < RK)
      for (int rr = 0; rr < T; ++rr) zacc += sFu[rr][tid];
  }
  float* Sp = S_part + ((size_t)bh * dm.nchunk + chunk) * RK * D;
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int idx = tid + e * 128;
    if (idx < RK * D) Sp[idx] = sacc[e];
  }
  if (tid < RK) z_part[((size_t)bh * dm.nchunk + chunk) * RK + tid] = zacc;
}

// Adds the chunk partials in chunk order; writes S (fp32), its bf16 hi/lo split and z.
// With d = 128 it also writes S^T hi | lo as the attention epilogue's tensor-core operand
// image: MN-major, 128-byte swizzle, box c = channels 64c..64c+63, rank rows of 128 bytes.
__global__ void state_reduce_kernel(Dims dm, const float* __restrict__ S_part,
                                    const float* __restrict__ z_part, float* __restrict__ S,
                                    __nv_bfloat16* __restrict__ S_hi,
                                    __nv_bfloat16* __restrict__ S_lo, float* __restrict__ z,
                                    uint8_t* __restrict__ simg) {
  const int bh = blockIdx.y;
  const int rd = dm.r * dm.d;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < rd) {
    const float* p = S_part + (size_t)bh * dm.nchunk * rd + e;
    float acc = 0.f;
    for (int c = 0; c < dm.nchunk; ++c) acc += p[(size_t)c * rd];
    S[(size_t)bh * rd + e] = acc;
    const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
    const __nv_bfloat16 lo = __float2bfloat16_rn(acc - __bfloat162float(hi));
    S_hi[(size_t)bh * rd + e] = hi;
    S_lo[(size_t)bh * rd + e] = lo;
    if (simg != nullptr) {
      const int a = e / dm.d, dd = e % dm.d, c = dd >> 6, col = dd & 63;
      uint8_t* im = simg + (size_t)bh * 4 * dm.r * 128;
      const size_t off = (size_t)(c * dm.r + a) * 128 + (((col >> 3) ^ (a & 7)) << 4) + (col & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(im + off) = hi;
      *reinterpret_cast<__nv_bfloat16*>(im + 2 * dm.r * 128 + off) = lo;
    }
  } else if (e < rd + dm.r) {
    const int a = e - rd;
    const float* p = z_part + (size_t)bh * dm.nchunk * dm.r + a;
    float acc = 0.f;
    for (int c = 0; c < dm.nchunk; ++c) acc += p[(size_t)c * dm.r];
    z[(size_t)bh * dm.r + a] = acc;
  }
}

template <int D, int RK>
cudaError_t launch_ls(const Dims& dm, rola_dtype dt, const void* k, const void* v, const void* Wk,
                      const Workspace& ws, cudaStream_t st) {
  dim3 grid(dm.nchunk, dm.B * dm.H);
  if (dt == ROLA_F32) {
    linear_state_f32_kernel<D, RK><<<grid, 128, 0, st>>>(
        static_cast<const float*>(k), static_cast<const float*>(v), static_cast<const float*>(Wk),
        dm, ws.rope, ws.S_part, ws.z_part);
  } else {
    const size_t smem = LSSmem<D, RK>::bytes;
    if (dt == ROLA_FP8_E4M3) {
      cudaError_t e = cudaFuncSetAttribute(linear_state_bf16_kernel<D, RK, true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      linear_state_bf16_kernel<D, RK, true><<<grid, 128, smem, st>>>(
          static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
          static_cast<const __nv_bfloat16*>(Wk), dm, ws.rope, ws.S_part, ws.z_part, nullptr, nullptr, ws.v8,
          ws.sv, ws.status);
    } else {
      cudaError_t e = cudaFuncSetAttribute(linear_state_bf16_kernel<D, RK, false>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      linear_state_bf16_kernel<D, RK, false><<<grid, 128, smem, st>>>(
          static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
          static_cast<const __nv_bfloat16*>(Wk), dm, ws.rope, ws.S_part, ws.z_part, ws.v16, ws.vexp, nullptr,
          nullptr, ws.status);
    }
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_rope_table(const Dims& dm, const Workspace& ws, cudaStream_t st) {
  const int total = dm.rope_off_w + dm.gw * dm.pw;
  const int blocks = (total + 255) / 256;
  rope_table_kernel<<<blocks > 0 ? blocks : 1, 256, 0, st>>>(dm, ws.rope);
  return cudaGetLastError();
}

cudaError_t launch_linear_state(const Dims& dm, rola_dtype dt, const void* k, const void* v,
                                const void* Wk, const Workspace& ws, cudaStream_t st) {
  cudaError_t e;
  if (dm.d == 128 && dt != ROLA_F32) e = launch_kv_pass(dm, dt == ROLA_FP8_E4M3, k, v, Wk, ws, st);
  else if (dm.d == 128 && dm.r == 32) e = launch_ls<128, 32>(dm, dt, k, v, Wk, ws, st);
  else if (dm.d == 128 && dm.r == 16) e = launch_ls<128, 16>(dm, dt, k, v, Wk, ws, st);
  else if (dm.d == 64 && dm.r == 32) e = launch_ls<64, 32>(dm, dt, k, v, Wk, ws, st);
  else e = launch_ls<64, 16>(dm, dt, k, v, Wk, ws, st);
  if (e != cudaSuccess) return e;
  return launch_state_reduce(dm, ws, st);
}

cudaError_t launch_state_reduce(const Dims& dm, const Workspace& ws, cudaStream_t st) {
  const int rd = dm.r * dm.d + dm.r;
  dim3 grid((rd + 255) / 256, dm.B * dm.H);
  state_reduce_kernel<<<grid, 256, 0, st>>>(dm, ws.S_part, ws.z_part, ws.S, ws.S_hi, ws.S_lo,
                                            ws.z, ws.simg);
  return cudaGetLastError();
}

}  // namespace rola
