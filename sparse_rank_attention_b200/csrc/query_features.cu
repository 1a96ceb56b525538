// Query pass of the RoLA forward for head dim 128 with bf16 inputs: one read of each
// (b, h, 64-token query block i) computes
//   * the block mean of q (step 1, query side): fp32 sums in token order, one division;
//   * fp8 configuration: the e4m3 copy of q with its block scale (absmax / 448, 1 for an
//     all-zero block; code = RN-sat(x * (1 / scale)));
//   * the query side of the linear branch (step 5):
//       u_n = phi(q_n Wq_h)            (r values per token, phi = elu + 1)
//       gden_n = g / (u_n . z_h)       (the gain over the unrotated normaliser; g = g_h,
//                                       or g_{n,h} for a per-token gate)
//       (R(p_n) u_n) split into bf16 hi + lo, stored transposed ([rank][64 tokens]) as the
//       exact 128-byte-swizzled shared-memory image the attention epilogue multiplies
//       with S_h on the tensor cores (one bulk copy there, no per-element work).
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (high-energy block selection; low-rank
// linear branch with rotary positions); README sparse-finetuning section (proj_q; the
// gate read as a gain per head or per token and head).
#include "rola_internal.cuh"
#include "warp_mma.cuh"

#include <cuda_fp8.h>

namespace rola {
namespace {

// grid: x = query block i, y = b*H + h; 128 threads (4 warps x 16 tokens).
template <int RK, bool FP8>
__global__ void __launch_bounds__(128) query_features_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ Wq,
    const float* __restrict__ g, Dims dm, const float* __restrict__ z,
    const float2* __restrict__ rope, float* __restrict__ qbar, uint8_t* __restrict__ uimg,
    float* __restrict__ gden, uint8_t* __restrict__ q8, float* __restrict__ sq) {
  constexpr int D = 128, DP = D + 8, WP = RK + 8;
  __shared__ __align__(16) __nv_bfloat16 sQ[kBlock * DP];
  __shared__ __align__(16) __nv_bfloat16 sW[D * WP];     // Wq_h [d][r], padded rows
  __shared__ __align__(1024) uint8_t img[2 * RK * 128];   // (R u)^T hi | lo, SW128 rows
  __shared__ float sz[RK];
  __shared__ float sred[4];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const size_t rs = (size_t)dm.H * D;
  const int n0 = i * kBlock, cnt = min(kBlock, dm.N - n0);
  const __nv_bfloat16* qb = q + (size_t)b * dm.N * rs + (size_t)h * D;
  for (int e = tid; e < kBlock * (D / 8); e += 128) {
    const int rr = e / (D / 8), cv = e % (D / 8), n = n0 + rr;
    const bool ok = n < dm.N;
    cp_async16(smem_u32(sQ + rr * DP + cv * 8), qb + (size_t)(ok ? n : 0) * rs + cv * 8, ok ? 16 : 0);
  }
  for (int e = tid; e < D * RK / 8; e += 128) {
    const int c = e / (RK / 8), a8 = e % (RK / 8);
    cp_async16(smem_u32(sW + c * WP + a8 * 8), Wq + ((size_t)h * D + c) * RK + a8 * 8, 16);
  }
  cp_async_commit();
  if (tid < RK) sz[tid] = z[(size_t)bh * RK + tid];
  cp_async_wait<0>();
  __syncthreads();

  // block mean of q: threads 0-63 own two adjacent channels each, tokens added in order
  {
    float am = 0.f;
    if (tid < 64) {
      float a0 = 0.f, a1 = 0.f;
      const uint32_t* col = reinterpret_cast<const uint32_t*>(sQ) + tid;
      for (int r = 0; r < cnt; ++r) {
        const uint32_t w = col[r * (DP / 2)];
        const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xffff0000u);
        a0 = a0 + x0;
        a1 = a1 + x1;
        if (FP8) am = fmaxf(am, fmaxf(fabsf(x0), fabsf(x1)));
      }
      *reinterpret_cast<float2*>(qbar + ((size_t)bh * dm.nb + i) * D + 2 * tid) =
          make_float2(__fdiv_rn(a0, (float)cnt), __fdiv_rn(a1, (float)cnt));
    }
    if constexpr (FP8) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      if (lane == 0) sred[warp] = am;
      __syncthreads();
      am = fmaxf(fmaxf(sred[0], sred[1]), fmaxf(sred[2], sred[3]));
      const float scale = am > 0.f ? am / 448.f : 1.f, inv = 1.f / scale;
      if (tid == 0) sq[(size_t)bh * dm.nb + i] = scale;
      for (int e = tid; e < cnt * (D / 8); e += 128) {
        const int rr = e / (D / 8), cv = e % (D / 8);
        const uint4 v = *reinterpret_cast<const uint4*>(sQ + rr * DP + cv * 8);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[2] = {0, 0};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 f = make_float2(__uint_as_float(w[u] << 16) * inv, __uint_as_float(w[u] & 0xffff0000u) * inv);
          o[u >> 1] |= (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3) << (16 * (u & 1));
        }
        *reinterpret_cast<uint2*>(q8 + ((size_t)b * dm.N + n0 + rr) * rs + (size_t)h * D + cv * 8) =
            make_uint2(o[0], o[1]);
      }
    }
  }

  constexpr int NT = RK / 8;
  float f[NT][4];
#pragma unroll
  for (int a = 0; a < NT; ++a)
#pragma unroll
    for (int e = 0; e < 4; ++e) f[a][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t af[4];
    ldsm_x4(smem_u32(sQ + (16 * warp + (lane & 15)) * DP + kk * 16 + (lane >> 4) * 8), af[0], af[1],
            af[2], af[3]);
#pragma unroll
    for (int nt = 0; nt < NT; nt += 2) {
      uint32_t bf[4];
      const int row = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
      ldsm_x4_t(smem_u32(sW + row * WP + nt * 8 + (lane >> 4) * 8), bf[0], bf[1], bf[2], bf[3]);
      mma_bf16(f[nt], af, bf);
      mma_bf16(f[nt + 1], af, bf + 2);
    }
  }
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = 16 * warp + g8 + 8 * half;     // token within the block
    const int n = i * kBlock + row;
    const bool ok = n < dm.N;
    const float gh = ok ? g[gain_index(dm, b, n, h)] : 0.f;
    const TokPos pos = token_pos(dm, ok ? n : 0);
    float den = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float u0 = phi_fast(f[nt][2 * half]), u1 = phi_fast(f[nt][2 * half + 1]);
      const int a = nt * 8 + 2 * t4;
      den = fmaf(u0, sz[a], fmaf(u1, sz[a + 1], den));
      const float2 cs = ok ? rope_at(dm, rope, pos, nt * 4 + t4) : make_float2(1.f, 0.f);
      const float r0 = cs.x * u0 - cs.y * u1;
      const float r1 = cs.y * u0 + cs.x * u1;
      const __nv_bfloat16 h0 = __float2bfloat16_rn(r0), h1 = __float2bfloat16_rn(r1);
      const uint32_t c0 = (((row >> 3) ^ (a & 7)) << 4) + (row & 7) * 2;
      const uint32_t c1 = (((row >> 3) ^ ((a + 1) & 7)) << 4) + (row & 7) * 2;
      *reinterpret_cast<__nv_bfloat16*>(img + a * 128 + c0) = h0;
      *reinterpret_cast<__nv_bfloat16*>(img + (a + 1) * 128 + c1) = h1;
      *reinterpret_cast<__nv_bfloat16*>(img + RK * 128 + a * 128 + c0) =
          __float2bfloat16_rn(r0 - __bfloat162float(h0));
      *reinterpret_cast<__nv_bfloat16*>(img + RK * 128 + (a + 1) * 128 + c1) =
          __float2bfloat16_rn(r1 - __bfloat162float(h1));
    }
    den += __shfl_xor_sync(0xffffffffu, den, 1);
    den += __shfl_xor_sync(0xffffffffu, den, 2);
    if (t4 == 0) gden[((size_t)bh * dm.nb + i) * kBlock + row] = gh / den;
  }
  __syncthreads();
  uint4* dst = reinterpret_cast<uint4*>(uimg + ((size_t)bh * dm.nb + i) * (2 * RK * 128));
  const uint4* src = reinterpret_cast<const uint4*>(img);
  for (int e = tid; e < 2 * RK * 128 / 16; e += 128) dst[e] = src[e];
}

}  // namespace

cudaError_t launch_query_features(const Dims& dm, bool fp8, const void* q, const void* Wq, const float* g,
                                  const Workspace& ws, cudaStream_t st) {
  dim3 grid(dm.nb, dm.B * dm.H);
  auto qq = static_cast<const __nv_bfloat16*>(q);
  auto ww = static_cast<const __nv_bfloat16*>(Wq);
  if (dm.r == 32) {
    if (fp8)
      query_features_kernel<32, true><<<grid, 128, 0, st>>>(qq, ww, g, dm, ws.z, ws.rope, ws.qbar, ws.uimg,
                                                            ws.gden, ws.q8, ws.sq);
    else
      query_features_kernel<32, false><<<grid, 128, 0, st>>>(qq, ww, g, dm, ws.z, ws.rope, ws.qbar, ws.uimg,
                                                             ws.gden, nullptr, nullptr);
  } else {
    if (fp8)
      query_features_kernel<16, true><<<grid, 128, 0, st>>>(qq, ww, g, dm, ws.z, ws.rope, ws.qbar, ws.uimg,
                                                            ws.gden, ws.q8, ws.sq);
    else
      query_features_kernel<16, false><<<grid, 128, 0, st>>>(qq, ww, g, dm, ws.z, ws.rope, ws.qbar, ws.uimg,
                                                             ws.gden, nullptr, nullptr);
  }
  return cudaGetLastError();
}

}  // namespace rola
