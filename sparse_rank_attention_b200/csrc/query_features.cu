// Query side of the linear branch of RoLA (part of step 5), as a pre-pass of the
// attention kernel: for every (b, h, 64-token query block i)
//   u_n = phi(q_n Wq_h)            (r values per token, phi = elu + 1)
//   gden_n = g_h / (u_n . z_h)     (the gain over the unrotated normaliser)
//   (R(p_n) u_n) split into bf16 hi + lo, stored transposed ([rank][64 tokens]) as the
//   exact 128-byte-swizzled shared-memory image the attention epilogue multiplies with
//   S_h on the tensor cores (one bulk copy there, no per-element work).
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (low-rank linear branch with rotary
// positions); README sparse-finetuning section (proj_q; the gate read as a per-head gain).
#include "rola_internal.cuh"
#include "warp_mma.cuh"

namespace rola {
namespace {

// grid: x = query block i, y = b*H + h; 128 threads (4 warps x 16 tokens).
template <int RK>
__global__ void __launch_bounds__(128) query_features_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ Wq,
    const float* __restrict__ g, Dims dm, const float* __restrict__ z,
    const float2* __restrict__ rope, uint8_t* __restrict__ uimg, float* __restrict__ gden) {
  constexpr int D = 128, DP = D + 8;
  __shared__ __align__(16) __nv_bfloat16 sQ[kBlock * DP];
  __shared__ __align__(16) __nv_bfloat16 sW[RK * DP];     // Wq_h^T [r][d]
  __shared__ __align__(1024) uint8_t img[2 * RK * 128];   // (R u)^T hi | lo, SW128 rows
  __shared__ float sz[RK];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const size_t rs = (size_t)dm.H * D;
  const __nv_bfloat16* qb = q + (size_t)b * dm.N * rs + (size_t)h * D;
  for (int e = tid; e < kBlock * (D / 8); e += 128) {
    const int rr = e / (D / 8), cv = e % (D / 8), n = i * kBlock + rr;
    const bool ok = n < dm.N;
    cp_async16(smem_u32(sQ + rr * DP + cv * 8), qb + (size_t)(ok ? n : 0) * rs + cv * 8, ok ? 16 : 0);
  }
  cp_async_commit();
  for (int e = tid; e < D * RK; e += 128) {
    const int c = e / RK, a = e % RK;
    sW[a * DP + c] = Wq[((size_t)h * D + c) * RK + a];
  }
  if (tid < RK) sz[tid] = z[(size_t)bh * RK + tid];
  cp_async_wait<0>();
  __syncthreads();

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
      const int qd = lane >> 3;
      uint32_t bf[4];
      ldsm_x4(smem_u32(sW + ((nt + (qd >> 1)) * 8 + (lane & 7)) * DP + kk * 16 + (qd & 1) * 8), bf[0],
              bf[1], bf[2], bf[3]);
      mma_bf16(f[nt], af, bf);
      mma_bf16(f[nt + 1], af, bf + 2);
    }
  }
  const float gh = g[h];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = 16 * warp + g8 + 8 * half;     // token within the block
    const int n = i * kBlock + row;
    const bool ok = n < dm.N;
    float den = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float u0 = phi(f[nt][2 * half]), u1 = phi(f[nt][2 * half + 1]);
      const int a = nt * 8 + 2 * t4;
      den = fmaf(u0, sz[a], fmaf(u1, sz[a + 1], den));
      const float2 cs = ok ? rope_cs(dm, rope, n, nt * 4 + t4) : make_float2(1.f, 0.f);
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

cudaError_t launch_query_features(const Dims& dm, const void* q, const void* Wq, const float* g,
                                  const Workspace& ws, cudaStream_t st) {
  dim3 grid(dm.nb, dm.B * dm.H);
  if (dm.r == 32)
    query_features_kernel<32><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                    static_cast<const __nv_bfloat16*>(Wq), g, dm,
                                                    ws.z, ws.rope, ws.uimg, ws.gden);
  else
    query_features_kernel<16><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                    static_cast<const __nv_bfloat16*>(Wq), g, dm,
                                                    ws.z, ws.rope, ws.uimg, ws.gden);
  return cudaGetLastError();
}

}  // namespace rola
