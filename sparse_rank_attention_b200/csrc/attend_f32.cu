// Sparse branch + linear epilogue + combination of RoLA (steps 3-5) for fp32 inputs.
//
// This is the fp32 correctness configuration: plain fp32 FMA arithmetic, one thread per
// query token, the kept key blocks staged through shared memory.  The bf16 and fp8
// configurations use the tensor-core kernel instead.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (block-sparse softmax branch plus a
// low-rank linear branch with rotary positions); README sparse-finetuning section
// (proj_q and the gate parameters; the gate is read here as a gain g per head or per
// token and head).
#include "rola_internal.cuh"

namespace rola {
namespace {

// grid: x = query block i, y = b*H + h; 64 threads, thread t owns token 64*i + t.
template <int D, int RK>
__global__ void __launch_bounds__(64) attend_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ Wq, const float* __restrict__ g, float* __restrict__ out, Dims dm,
    const int32_t* __restrict__ col_idx, const float* __restrict__ S,
    const float* __restrict__ z, const float2* __restrict__ rope, int* __restrict__ status) {
  extern __shared__ float sm[];
  float* sQ = sm;                      // [64][D+1]
  float* sK = sQ + kBlock * (D + 1);   // [64][D+1]
  float* sV = sK + kBlock * (D + 1);   // [64][D]
  float* sW = sV + kBlock * D;         // [D][RK]
  float* sS = sW + D * RK;             // [RK][D]
  float* sz = sS + RK * D;             // [RK]
  float* sP = sz + RK;                 // [64][65] scaled logits of each thread's token
  const int tid = threadIdx.x;
  const int i = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const size_t rs = (size_t)dm.H * D;
  const float* qb = q + (size_t)b * dm.N * rs + (size_t)h * D;
  const float* kb = k + (size_t)b * dm.N * rs + (size_t)h * D;
  const float* vb = v + (size_t)b * dm.N * rs + (size_t)h * D;
  const int n = i * kBlock + tid;
  const bool valid = n < dm.N;

  for (int e = tid; e < kBlock * D; e += 64) {
    const int rr = e / D, c = e % D, nn = i * kBlock + rr;
    sQ[rr * (D + 1) + c] = nn < dm.N ? qb[(size_t)nn * rs + c] : 0.f;
  }
  for (int e = tid; e < D * RK; e += 64) sW[e] = Wq[(size_t)h * D * RK + e];
  for (int e = tid; e < RK * D; e += 64) sS[e] = S[(size_t)bh * RK * D + e];
  if (tid < RK) sz[tid] = z[(size_t)bh * RK + tid];

  float o[D];
#pragma unroll
  for (int c = 0; c < D; ++c) o[c] = 0.f;
  float m = -INFINITY, l = 0.f;
  const float sl2 = dm.scale * 1.4426950408889634f;  // logits in log2 units
  const int32_t* L = col_idx + ((size_t)bh * dm.nb + i) * dm.k;
  for (int jj = 0; jj < dm.k; ++jj) {
    int j = L[jj];
    if (j < 0 || j >= dm.nb) {
      if (tid == 0) record_status(status, kDevBounds);
      j = 0;
    }
    __syncthreads();
    for (int e = tid; e < kBlock * D; e += 64) {
      const int rr = e / D, c = e % D, mm = j * kBlock + rr;
      sK[rr * (D + 1) + c] = mm < dm.N ? kb[(size_t)mm * rs + c] : 0.f;
      sV[rr * D + c] = mm < dm.N ? vb[(size_t)mm * rs + c] : 0.f;
    }
    __syncthreads();
    const int nvalid = min(kBlock, dm.N - j * kBlock);
    float* srow = sP + tid * (kBlock + 1);
    float mx = -INFINITY;
    for (int t = 0; t < nvalid; ++t) {
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) acc = fmaf(sQ[tid * (D + 1) + c], sK[t * (D + 1) + c], acc);
      srow[t] = acc * sl2;
      mx = fmaxf(mx, srow[t]);
    }
    const float mnew = fmaxf(m, mx);
    const float corr = exp2f(m - mnew);
    l *= corr;
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] *= corr;
    for (int t = 0; t < nvalid; ++t) {
      const float p = exp2f(srow[t] - mnew);
      l += p;
#pragma unroll
      for (int c = 0; c < D; ++c) o[c] = fmaf(p, sV[t * D + c], o[c]);
    }
    m = mnew;
  }

  // linear branch: u = phi(q Wq), den = u . z, num = (R u) . S
  float u[RK];
#pragma unroll
  for (int a = 0; a < RK; ++a) {
    float acc = 0.f;
    for (int c = 0; c < D; ++c) acc = fmaf(sQ[tid * (D + 1) + c], sW[c * RK + a], acc);
    u[a] = phi(acc);
  }
  float den = 0.f;
#pragma unroll
  for (int a = 0; a < RK; ++a) den = fmaf(u[a], sz[a], den);
  float ur[RK];
#pragma unroll
  for (int c = 0; c < RK / 2; ++c) {
    const float2 cs = valid ? rope_cs(dm, rope, n, c) : make_float2(1.f, 0.f);
    ur[2 * c] = cs.x * u[2 * c] - cs.y * u[2 * c + 1];
    ur[2 * c + 1] = cs.y * u[2 * c] + cs.x * u[2 * c + 1];
  }
  if (!valid) return;
  const float gh = gate_value(dm, g, sQ + tid * (D + 1), b, n, h);
  const float inv_l = 1.f / l, inv_den = 1.f / den;
  float* ob = out + ((size_t)b * dm.N + n) * rs + (size_t)h * D;
#pragma unroll
  for (int c = 0; c < D; ++c) {
    float num = 0.f;
#pragma unroll
    for (int a = 0; a < RK; ++a) num = fmaf(ur[a], sS[a * D + c], num);
    ob[c] = o[c] * inv_l + gh * (num * inv_den);
  }
}

template <int D, int RK>
cudaError_t launch_f32(const Dims& dm, const void* q, const void* k, const void* v,
                       const void* Wq, const float* g, void* out, const Workspace& ws,
                       cudaStream_t st) {
  const size_t smem =
      sizeof(float) * (2 * kBlock * (D + 1) + kBlock * D + 2 * D * RK + RK + kBlock * (kBlock + 1));
  cudaError_t e = cudaFuncSetAttribute(attend_f32_kernel<D, RK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(dm.nb, dm.B * dm.H);
  attend_f32_kernel<D, RK><<<grid, 64, smem, st>>>(
      static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
      static_cast<const float*>(Wq), g, static_cast<float*>(out), dm, ws.col_idx, ws.S, ws.z,
      ws.rope, ws.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_f32(const Dims& dm, const void* q, const void* k, const void* v,
                              const void* Wq, const float* g, void* out, const Workspace& ws,
                              cudaStream_t st) {
  if (dm.d == 128 && dm.r == 32) return launch_f32<128, 32>(dm, q, k, v, Wq, g, out, ws, st);
  if (dm.d == 128 && dm.r == 16) return launch_f32<128, 16>(dm, q, k, v, Wq, g, out, ws, st);
  if (dm.d == 64 && dm.r == 32) return launch_f32<64, 32>(dm, q, k, v, Wq, g, out, ws, st);
  return launch_f32<64, 16>(dm, q, k, v, Wq, g, out, ws, st);
}

}  // namespace rola
