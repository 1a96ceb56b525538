// Sparse branch + fused linear epilogue + combination of RoLA (steps 3-5), bf16 inputs,
// warp-level tensor cores (mma.sync m16n8k16).
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (block-sparse softmax branch plus a
// low-rank linear branch with rotary positions); README sparse-finetuning section
// (proj_q, and the gate read here as a gain g per head or per token and head).
//
// One CTA per (b, h, 64-token query block), 4 warps x 16 query rows:
//   for each kept key block j (ascending):  S = Q K_j^T, online softmax, O += P V_j
//   epilogue: u = phi(Q Wq), den = u.z, num = (R u) S_h, out = O/l + g * num/den
// Precision: Q K^T in bf16 (exact products, fp32 sums); the softmax weights P are
// rounded to fp16 and multiplied with the fp16 copy of v (bf16 P would cost up to
// ~1e-3 absolute on peaked rows); R u and S_h enter the epilogue products as bf16
// hi + lo pairs (three products), so the linear branch keeps ~fp32 accuracy.
// K_j / V_j are double-buffered with cp.async; out is staged in shared memory and
// written with 16-byte stores, once.
#include <climits>

#include "rola_internal.cuh"
#include "warp_mma.cuh"

namespace rola {
namespace {

template <int D, int RK>
struct AttSmem {
  static constexpr int DP = D + 8;            // padded row, bf16 elements
  static constexpr int kTile = kBlock * DP;
  static constexpr int kWq = RK * DP;         // WqT [r][d]
  static constexpr int kS = RK * DP;          // S_h [r][d] (hi and lo)
  static constexpr size_t bytes = sizeof(__nv_bfloat16) * (5 * kTile + kWq + 2 * kS) + sizeof(float) * RK;
};

template <int D, int RK>
__global__ void __launch_bounds__(128, 2) attend_bf16_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __half* __restrict__ v, const __nv_bfloat16* __restrict__ Wq,
    const float* __restrict__ g, __nv_bfloat16* __restrict__ out, Dims dm,
    const int32_t* __restrict__ col_idx, const __nv_bfloat16* __restrict__ S_hi,
    const __nv_bfloat16* __restrict__ S_lo, const float* __restrict__ z,
    const float2* __restrict__ rope, const int* __restrict__ vexp, int* __restrict__ status) {
  using L = AttSmem<D, RK>;
  constexpr int DP = L::DP;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sK = sQ + L::kTile;          // [2][tile]
  __half* sV = reinterpret_cast<__half*>(sK + 2 * L::kTile);      // [2][tile] fp16
  __nv_bfloat16* sW = reinterpret_cast<__nv_bfloat16*>(sV + 2 * L::kTile);
  __nv_bfloat16* sS = sW + L::kWq;        // S_hi
  __nv_bfloat16* sSl = sS + L::kS;        // S_lo
  float* sz = reinterpret_cast<float*>(sSl + L::kS);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3, quad = lane >> 3;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const size_t rs = (size_t)dm.H * D;
  const __nv_bfloat16* qb = q + (size_t)b * dm.N * rs + (size_t)h * D;
  const __nv_bfloat16* kb = k + (size_t)b * dm.N * rs + (size_t)h * D;
  const __half* vb = v + (size_t)b * dm.N * rs + (size_t)h * D;
  const int32_t* Lst = col_idx + ((size_t)bh * dm.nb + i) * dm.k;
  constexpr int VPR = D / 8;  // 16-byte vectors per row

  // Q tile, S_h (cp.async); WqT and z (plain loads)
  for (int e = tid; e < kBlock * VPR; e += 128) {
    const int rr = e / VPR, cv = e % VPR, n = i * kBlock + rr;
    const bool ok = n < dm.N;
    cp_async16(smem_u32(sQ + rr * DP + cv * 8), qb + (size_t)(ok ? n : 0) * rs + cv * 8, ok ? 16 : 0);
  }
  for (int e = tid; e < RK * VPR; e += 128) {
    const int a = e / VPR, cv = e % VPR;
    cp_async16(smem_u32(sS + a * DP + cv * 8), S_hi + ((size_t)bh * RK + a) * D + cv * 8, 16);
    cp_async16(smem_u32(sSl + a * DP + cv * 8), S_lo + ((size_t)bh * RK + a) * D + cv * 8, 16);
  }
  cp_async_commit();
  for (int e = tid; e < D * RK; e += 128) {
    const int c = e / RK, a = e % RK;
    sW[a * DP + c] = Wq[((size_t)h * D + c) * RK + a];
  }
  if (tid < RK) sz[tid] = z[(size_t)bh * RK + tid];

  auto block_of = [&](int jj) {
    int j = Lst[jj];
    if (j < 0 || j >= dm.nb) {
      if (tid == 0) record_status(status, kDevBounds);
      j = 0;
    }
    return j;
  };
  auto load_kv = [&](int j, int stage) {
    for (int e = tid; e < kBlock * VPR; e += 128) {
      const int rr = e / VPR, cv = e % VPR, m = j * kBlock + rr;
      const bool ok = m < dm.N;
      const size_t off = (size_t)(ok ? m : 0) * rs + cv * 8;
      cp_async16(smem_u32(sK + stage * L::kTile + rr * DP + cv * 8), kb + off, ok ? 16 : 0);
      cp_async16(smem_u32(sV + stage * L::kTile + rr * DP + cv * 8), vb + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  // v is carried in fp16 as v * 2^-vexp per key block: P of block j is scaled by
  // 2^(vexp_j - eref) (at most 1) and the output by 2^eref, eref = the row's largest vexp
  const int* ve = vexp + (size_t)bh * dm.nb;
  int eref = INT_MIN;
  for (int jj = 0; jj < dm.k; ++jj) {
    const int j = Lst[jj];
    if (j >= 0 && j < dm.nb) eref = max(eref, __ldg(ve + j));
  }
  if (eref == INT_MIN) eref = 0;

  int j_next = block_of(0);
  load_kv(j_next, 0);
  cp_async_wait<1>();
  __syncthreads();

  uint32_t qf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    ldsm_x4(smem_u32(sQ + (16 * warp + (lane & 15)) * DP + kk * 16 + (lane >> 4) * 8), qf[kk][0],
            qf[kk][1], qf[kk][2], qf[kk][3]);

  float o[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  const float sl2 = dm.scale * 1.4426950408889634f;

  for (int jj = 0; jj < dm.k; ++jj) {
    const int stage = jj & 1;
    const int j = j_next;
    if (jj + 1 < dm.k) {
      j_next = block_of(jj + 1);
      load_kv(j_next, stage ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* tK = sK + stage * L::kTile;
    const __half* tV = sV + stage * L::kTile;

    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t bf[4];
        ldsm_x4(smem_u32(tK + ((nt + (quad >> 1)) * 8 + (lane & 7)) * DP + kk * 16 + (quad & 1) * 8),
                bf[0], bf[1], bf[2], bf[3]);
        mma_bf16(s[nt], qf[kk], bf);
        mma_bf16(s[nt + 1], qf[kk], bf + 2);
      }
    }
    const int nvalid = min(kBlock, dm.N - j * kBlock);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nt * 8 + 2 * t4 + (e & 1);
        s[nt][e] = col < nvalid ? s[nt][e] * sl2 : -INFINITY;
      }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * hh], s[nt][2 * hh + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(mrow[hh], mx);
      const float corr = exp2f(mrow[hh] - mnew);
      float rsum = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = exp2f(s[nt][2 * hh] - mnew);
        const float p1 = exp2f(s[nt][2 * hh + 1] - mnew);
        s[nt][2 * hh] = p0;
        s[nt][2 * hh + 1] = p1;
        rsum += p0 + p1;
      }
      lrow[hh] = lrow[hh] * corr + rsum;
      mrow[hh] = mnew;
#pragma unroll
      for (int nt = 0; nt < D / 8; ++nt) {
        o[nt][2 * hh] *= corr;
        o[nt][2 * hh + 1] *= corr;
      }
    }
    const int ej = __ldg(ve + j);
    if (ej != eref) {
      const float fac = ldexpf(1.f, ej - eref);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] *= fac;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_f16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_f16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_f16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_f16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < D / 8; nt += 2) {
        uint32_t bf[4];
        ldsm_x4_t(smem_u32(tV + (kk * 16 + (quad & 1) * 8 + (lane & 7)) * DP + (nt + (quad >> 1)) * 8),
                  bf[0], bf[1], bf[2], bf[3]);
        mma_f16(o[nt], pa, bf);
        mma_f16(o[nt + 1], pa, bf + 2);
      }
    }
    __syncthreads();
  }

  float inv_l[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float l = lrow[hh];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    inv_l[hh] = ldexpf(1.f / l, eref);
  }

  // ---- linear branch epilogue
  constexpr int NTU = RK / 8;
  float u[NTU][4];
#pragma unroll
  for (int nt = 0; nt < NTU; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) u[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
    for (int nt = 0; nt < NTU; nt += 2) {
      uint32_t bf[4];
      ldsm_x4(smem_u32(sW + ((nt + (quad >> 1)) * 8 + (lane & 7)) * DP + kk * 16 + (quad & 1) * 8),
              bf[0], bf[1], bf[2], bf[3]);
      mma_bf16(u[nt], qf[kk], bf);
      mma_bf16(u[nt + 1], qf[kk], bf + 2);
    }
  float den[2] = {0.f, 0.f};
#pragma unroll
  for (int nt = 0; nt < NTU; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      u[nt][e] = phi(u[nt][e]);
      den[e >> 1] += u[nt][e] * sz[nt * 8 + 2 * t4 + (e & 1)];
    }
  float coef[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float dd = den[hh];
    dd += __shfl_xor_sync(0xffffffffu, dd, 1);
    dd += __shfl_xor_sync(0xffffffffu, dd, 2);
    const int n = i * kBlock + 16 * warp + g8 + 8 * hh;
    const bool ok = n < dm.N;
    // the query row of token n is still in sQ (the output is staged there only later)
    coef[hh] = (ok ? gate_value(dm, g, sQ + (16 * warp + g8 + 8 * hh) * DP, b, n, h) : 0.f) / dd;
#pragma unroll
    for (int nt = 0; nt < NTU; ++nt) {
      const float2 cs = ok ? rope_cs(dm, rope, n, nt * 4 + t4) : make_float2(1.f, 0.f);
      const float x0 = u[nt][2 * hh], x1 = u[nt][2 * hh + 1];
      u[nt][2 * hh] = cs.x * x0 - cs.y * x1;
      u[nt][2 * hh + 1] = cs.y * x0 + cs.x * x1;
    }
  }
  uint32_t ua[RK / 16][4], ul[RK / 16][4];
#pragma unroll
  for (int kk = 0; kk < RK / 16; ++kk) {
    split_bf16(u[2 * kk][0], u[2 * kk][1], ua[kk][0], ul[kk][0]);
    split_bf16(u[2 * kk][2], u[2 * kk][3], ua[kk][1], ul[kk][1]);
    split_bf16(u[2 * kk + 1][0], u[2 * kk + 1][1], ua[kk][2], ul[kk][2]);
    split_bf16(u[2 * kk + 1][2], u[2 * kk + 1][3], ua[kk][3], ul[kk][3]);
  }
#pragma unroll
  for (int nt = 0; nt < D / 8; nt += 2) {
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < RK / 16; ++kk) {
      uint32_t bf[4], bl[4];
      const int off = (kk * 16 + (quad & 1) * 8 + (lane & 7)) * DP + (nt + (quad >> 1)) * 8;
      ldsm_x4_t(smem_u32(sS + off), bf[0], bf[1], bf[2], bf[3]);
      ldsm_x4_t(smem_u32(sSl + off), bl[0], bl[1], bl[2], bl[3]);
      mma_bf16(acc[0], ua[kk], bf);
      mma_bf16(acc[1], ua[kk], bf + 2);
      mma_bf16(acc[0], ua[kk], bl);
      mma_bf16(acc[1], ua[kk], bl + 2);
      mma_bf16(acc[0], ul[kk], bf);
      mma_bf16(acc[1], ul[kk], bf + 2);
    }
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const float y0 = o[nt + t][2 * hh] * inv_l[hh] + coef[hh] * acc[t][2 * hh];
        const float y1 = o[nt + t][2 * hh + 1] * inv_l[hh] + coef[hh] * acc[t][2 * hh + 1];
        *reinterpret_cast<uint32_t*>(sQ + (16 * warp + g8 + 8 * hh) * DP + (nt + t) * 8 + 2 * t4) =
            pack_bf16(y0, y1);
      }
  }
  __syncthreads();
  __nv_bfloat16* ob = out + (size_t)b * dm.N * rs + (size_t)h * D;
  for (int e = tid; e < kBlock * VPR; e += 128) {
    const int rr = e / VPR, cv = e % VPR, n = i * kBlock + rr;
    if (n < dm.N)
      *reinterpret_cast<uint4*>(ob + (size_t)n * rs + cv * 8) =
          *reinterpret_cast<const uint4*>(sQ + rr * DP + cv * 8);
  }
}

template <int D, int RK>
cudaError_t launch_bf16(const Dims& dm, const void* q, const void* k, const void* v,
                        const void* Wq, const float* g, void* out, const Workspace& ws,
                        cudaStream_t st) {
  const size_t smem = AttSmem<D, RK>::bytes;
  cudaError_t e = cudaFuncSetAttribute(attend_bf16_kernel<D, RK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(dm.nb, dm.B * dm.H);
  attend_bf16_kernel<D, RK><<<grid, 128, smem, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      ws.v16, static_cast<const __nv_bfloat16*>(Wq), g, static_cast<__nv_bfloat16*>(out), dm,
      ws.col_idx, ws.S_hi, ws.S_lo, ws.z, ws.rope, ws.vexp, ws.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_bf16_warpmma(const Dims& dm, const void* q, const void* k,
                                       const void* v, const void* Wq, const float* g, void* out,
                                       const Workspace& ws, cudaStream_t st) {
  if (dm.d == 128 && dm.r == 32) return launch_bf16<128, 32>(dm, q, k, v, Wq, g, out, ws, st);
  if (dm.d == 128 && dm.r == 16) return launch_bf16<128, 16>(dm, q, k, v, Wq, g, out, ws, st);
  if (dm.d == 64 && dm.r == 32) return launch_bf16<64, 32>(dm, q, k, v, Wq, g, out, ws, st);
  return launch_bf16<64, 16>(dm, q, k, v, Wq, g, out, ws, st);
}

}  // namespace rola
