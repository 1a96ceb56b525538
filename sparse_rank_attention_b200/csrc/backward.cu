// Backward of the RoLA forward: the gradients of L = sum(dout * out) with respect to q, k,
// v, Wq, Wk and the gain parameters, with the kept-block lists held fixed (the selection
// is a discrete choice).  fp32 arithmetic throughout, on bf16 or fp32 inputs.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (block-sparse softmax branch plus a
// low-rank linear branch with rotary positions); README sparse-finetuning section
// (proj_q, proj_k, gate_proj, gate_bias: the trained parameters whose gradients these are).
//
// Chain rule of the forward's definition (each line a kernel below):
//   sparse branch, per query token n over the keys m of its kept blocks, with
//   P_nm = exp(scale q_n.k_m - lse_n), O_n = sum_m P_nm v_m, D_n = dout_n . O_n:
//     dA_nm = P_nm (dout_n . v_m - D_n)
//     dq_n += scale sum_m dA_nm k_m                        (query-major: its kept list)
//     dk_m += scale sum_n dA_nm q_n,  dv_m += sum_n P_nm dout_n   (key-major: the query
//                                                           blocks that kept block m)
//   linear branch and gain, with x = q Wq, u = phi(x), y = R(p) u, den = u.z,
//   L = y^T S / den, out = O + g L:
//     dg_n = dout_n . L_n;  gG = g dout;  dS += y gG^T / den;  dy = S gG / den;
//     dden = -(gG . L) / den;  du = R^T dy + dden z;  dz += dden u;  dx = phi'(x) du;
//     dq += Wq dx;  dWq += q dx^T;  (gate from the query: dlogit = dg g (1 - g),
//     dq += dlogit wg, dwg += dlogit q, dbg += dlogit)
//   key side, with w = k Wk, f = phi(w), yk = R(p) f:
//     dv += dS^T yk;  df = R^T (dS v) + dz;  dw = phi'(w) df;  dk += Wk dw;  dWk += k dw^T.
//
// Tiles of 64 tokens in shared memory as fp32, 256 threads; in the 64 x 64 and 64 x d
// products thread (ty, tx) = (tid / 16, tid % 16) holds rows 4 ty .. 4 ty + 3 and columns
// tx + 16 j.  Partial sums over token chunks are reduced in a fixed order, so the result
// is the same from run to run.  Every wait is a __syncthreads; no kernel spins.
#include <type_traits>

#include "rola_internal.cuh"
#include "sm100_ptx.cuh"
#include "warp_mma.cuh"

namespace rola {
namespace {

constexpr int kT = 256;

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float dphi_f(float x) { return x > 0.f ? 1.f : expf(x); }

// Loads rows [n0, n0 + 64) of head h of a [B, N, H, D] tensor into s[64][D + 1] as fp32;
// rows at or past N are zero.
template <typename T, int D>
__device__ __forceinline__ void load_tile(float* s, const T* __restrict__ x, const Dims& dm, int b, int h,
                                          int n0) {
  for (int e = threadIdx.x; e < 64 * D; e += kT) {
    const int r = e / D, c = e % D, n = n0 + r;
    s[r * (D + 1) + c] = n < dm.N ? to_f(x[(((size_t)b * dm.N + n) * dm.H + h) * D + c]) : 0.f;
  }
}

// sum over the 16 threads of a half-warp (the tx of one ty)
__device__ __forceinline__ float sum16(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float max16(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// s[i][j] = sum_e A[4 ty + i][e] B[tx + 16 j][e]  (A, B: [64][D + 1])
template <int D>
__device__ __forceinline__ void mm_abt(float (&s)[4][4], const float* A, const float* B, int ty, int tx) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll 4
  for (int e = 0; e < D; ++e) {
    float a[4], bb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = A[(4 * ty + i) * (D + 1) + e];
#pragma unroll
    for (int j = 0; j < 4; ++j) bb[j] = B[(tx + 16 * j) * (D + 1) + e];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = fmaf(a[i], bb[j], s[i][j]);
  }
}

// acc[i][c] += sum_e A[4 ty + i][e] B[e][tx + 16 c]  (A: [64][65], B: [64][D + 1])
template <int D>
__device__ __forceinline__ void mm_ab(float (&acc)[4][D / 16], const float* A, const float* B, int ty, int tx) {
#pragma unroll 4
  for (int e = 0; e < 64; ++e) {
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = A[(4 * ty + i) * 65 + e];
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      const float bv = B[e * (D + 1) + tx + 16 * c];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][c] = fmaf(a[i], bv, acc[i][c]);
    }
  }
}

// acc[i][c] += sum_e A[e][4 ty + i] B[e][tx + 16 c]  (A: [64][65], B: [64][D + 1])
template <int D>
__device__ __forceinline__ void mm_atb(float (&acc)[4][D / 16], const float* A, const float* B, int ty, int tx) {
#pragma unroll 4
  for (int e = 0; e < 64; ++e) {
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = A[e * 65 + 4 * ty + i];
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      const float bv = B[e * (D + 1) + tx + 16 * c];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i][c] = fmaf(a[i], bv, acc[i][c]);
    }
  }
}

__device__ __forceinline__ int checked_block(const Dims& dm, int j, int* status) {
  if (j < 0 || j >= dm.nb) {
    if (threadIdx.x == 0) record_status(status, kDevBounds);
    return 0;
  }
  return j;
}

// ------------------------------------------------------------------ sparse branch
// Per query tile: the row statistics of the forward's softmax, lse = m + log l of the
// scaled logits (+inf for rows past N), and D = dout . O.
template <typename T, int D>
__global__ void __launch_bounds__(kT) bwd_rowstats_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                          const T* __restrict__ v, const T* __restrict__ dout,
                                                          Dims dm, const int32_t* __restrict__ col_idx,
                                                          float* __restrict__ lse, float* __restrict__ Drow,
                                                          int* __restrict__ status) {
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sK = sQ + 64 * (D + 1);
  float* sV = sK + 64 * (D + 1);
  float* sP = sV + 64 * (D + 1);   // [64][65]
  const int i = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int32_t* L = col_idx + ((size_t)bh * dm.nb + i) * dm.k;
  load_tile<T, D>(sQ, q, dm, b, h, i * 64);
  float m[4], l[4], o[4][D / 16];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) o[r][c] = 0.f;
  }
  for (int jj = 0; jj < dm.k; ++jj) {
    const int j = checked_block(dm, L[jj], status);
    __syncthreads();
    load_tile<T, D>(sK, k, dm, b, h, j * 64);
    load_tile<T, D>(sV, v, dm, b, h, j * 64);
    __syncthreads();
    float s[4][4];
    mm_abt<D>(s, sQ, sK, ty, tx);
    const int nvalid = min(64, dm.N - j * 64);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        s[r][c] = tx + 16 * c < nvalid ? s[r][c] * dm.scale : -INFINITY;
        mx = fmaxf(mx, s[r][c]);
      }
      mx = max16(mx);
      const float mnew = fmaxf(m[r], mx);
      const float corr = m[r] == -INFINITY ? 0.f : expf(m[r] - mnew);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = expf(s[r][c] - mnew);
        sP[(4 * ty + r) * 65 + tx + 16 * c] = p;
        rs += p;
      }
      l[r] = l[r] * corr + sum16(rs);
      m[r] = mnew;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) o[r][c] *= corr;
    }
    __syncthreads();
    mm_ab<D>(o, sP, sV, ty, tx);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int n = i * 64 + 4 * ty + r;
    float dsum = 0.f;
    if (n < dm.N) {
      const T* G = dout + (((size_t)b * dm.N + n) * dm.H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 16; ++c) dsum = fmaf(to_f(G[tx + 16 * c]), o[r][c] / l[r], dsum);
    }
    dsum = sum16(dsum);
    if (tx == 0) {
      const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + 4 * ty + r;
      lse[at] = n < dm.N ? m[r] + logf(l[r]) : INFINITY;
      Drow[at] = n < dm.N ? dsum : 0.f;
    }
  }
}

// dq += scale sum_m dA_nm k_m over the query tile's kept blocks (added to the linear part
// already in dq).
template <typename T, int D>
__global__ void __launch_bounds__(kT) bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                    const T* __restrict__ v, const T* __restrict__ dout, Dims dm,
                                                    const int32_t* __restrict__ col_idx,
                                                    const float* __restrict__ lse, const float* __restrict__ Drow,
                                                    float* __restrict__ dq, int* __restrict__ status) {
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sG = sQ + 64 * (D + 1);
  float* sK = sG + 64 * (D + 1);
  float* sV = sK + 64 * (D + 1);
  float* sA = sV + 64 * (D + 1);   // [64][65]
  const int i = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  const int32_t* L = col_idx + ((size_t)bh * dm.nb + i) * dm.k;
  load_tile<T, D>(sQ, q, dm, b, h, i * 64);
  load_tile<T, D>(sG, dout, dm, b, h, i * 64);
  float ls[4], dd[4], acc[4][D / 16];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + 4 * ty + r;
    ls[r] = lse[at];
    dd[r] = Drow[at];
#pragma unroll
    for (int c = 0; c < D / 16; ++c) acc[r][c] = 0.f;
  }
  for (int jj = 0; jj < dm.k; ++jj) {
    const int j = checked_block(dm, L[jj], status);
    __syncthreads();
    load_tile<T, D>(sK, k, dm, b, h, j * 64);
    load_tile<T, D>(sV, v, dm, b, h, j * 64);
    __syncthreads();
    float s[4][4], dp[4][4];
    mm_abt<D>(s, sQ, sK, ty, tx);
    mm_abt<D>(dp, sG, sV, ty, tx);
    const int nvalid = min(64, dm.N - j * 64);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = tx + 16 * c < nvalid ? expf(s[r][c] * dm.scale - ls[r]) : 0.f;
        sA[(4 * ty + r) * 65 + tx + 16 * c] = p * (dp[r][c] - dd[r]);
      }
    __syncthreads();
    mm_ab<D>(acc, sA, sK, ty, tx);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int n = i * 64 + 4 * ty + r;
    if (n >= dm.N) continue;
    float* row = dq + (((size_t)b * dm.N + n) * dm.H + h) * D;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) row[tx + 16 * c] += dm.scale * acc[r][c];
  }
}

// dk, dv of one key tile over the query blocks that kept it (added to the linear parts).
template <typename T, int D>
__global__ void __launch_bounds__(kT) bwd_dkv_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                     const T* __restrict__ v, const T* __restrict__ dout, Dims dm,
                                                     const int* __restrict__ inv_off, const int* __restrict__ inv_idx,
                                                     const float* __restrict__ lse, const float* __restrict__ Drow,
                                                     float* __restrict__ dk, float* __restrict__ dv) {
  extern __shared__ float sm[];
  float* sK = sm;
  float* sV = sK + 64 * (D + 1);
  float* sQ = sV + 64 * (D + 1);
  float* sG = sQ + 64 * (D + 1);
  float* sP = sG + 64 * (D + 1);   // [64 q][65]
  float* sA = sP + 64 * 65;        // [64 q][65]
  float* sL = sA + 64 * 65;        // [64] lse of the query tile
  float* sD = sL + 64;             // [64] D of the query tile
  const int j = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  load_tile<T, D>(sK, k, dm, b, h, j * 64);
  load_tile<T, D>(sV, v, dm, b, h, j * 64);
  const int nvalid = min(64, dm.N - j * 64);
  float ak[4][D / 16], av[4][D / 16];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < D / 16; ++c) ak[r][c] = av[r][c] = 0.f;
  const int* lst = inv_idx + (size_t)bh * dm.nb * dm.k;
  const int e0 = inv_off[(size_t)bh * (dm.nb + 1) + j], e1 = inv_off[(size_t)bh * (dm.nb + 1) + j + 1];
  for (int e = e0; e < e1; ++e) {
    const int i = lst[e];
    __syncthreads();
    load_tile<T, D>(sQ, q, dm, b, h, i * 64);
    load_tile<T, D>(sG, dout, dm, b, h, i * 64);
    if (threadIdx.x < 64) {
      const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + threadIdx.x;
      sL[threadIdx.x] = lse[at];
      sD[threadIdx.x] = Drow[at];
    }
    __syncthreads();
    float s[4][4], dp[4][4];     // rows: queries 4 ty + r; columns: keys tx + 16 c
    mm_abt<D>(s, sQ, sK, ty, tx);
    mm_abt<D>(dp, sG, sV, ty, tx);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float lr = sL[4 * ty + r], dr = sD[4 * ty + r];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float p = tx + 16 * c < nvalid ? expf(s[r][c] * dm.scale - lr) : 0.f;
        sP[(4 * ty + r) * 65 + tx + 16 * c] = p;
        sA[(4 * ty + r) * 65 + tx + 16 * c] = p * (dp[r][c] - dr);
      }
    }
    __syncthreads();
    mm_atb<D>(av, sP, sG, ty, tx);   // rows: keys
    mm_atb<D>(ak, sA, sQ, ty, tx);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int m = j * 64 + 4 * ty + r;
    if (m >= dm.N) continue;
    const size_t at = (((size_t)b * dm.N + m) * dm.H + h) * D;
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      dk[at + tx + 16 * c] += dm.scale * ak[r][c];
      dv[at + tx + 16 * c] += av[r][c];
    }
  }
}

// ------------------------------------------------------------------ sparse branch, bf16
// The same three kernels for bf16 inputs on the warp-level tensor cores (mma.sync
// m16n8k16, fp32 accumulation): 128 threads, warp w owning rows 16 w .. 16 w + 15 of its
// tile, tiles in shared memory as bf16 [64][D + 8].  Q, K, V and dout enter exactly; P and
// dA enter the second products as bf16 hi + lo pairs (two products each, ~2^-16 relative),
// so the gradients keep fp32-level accuracy.
template <int D>
struct MmaTiles {
  static constexpr int DP = D + 8;
  static constexpr int kTile = 64 * DP;
  static constexpr size_t bytes = sizeof(__nv_bfloat16) * 4 * kTile + sizeof(float) * 128;
};

// rows [n0, n0 + 64) of head h of a [B, N, H, D] bf16 tensor -> s[64][D + 8] (cp.async;
// rows at or past N zero-filled)
template <int D>
__device__ __forceinline__ void load_tile_bf16(__nv_bfloat16* s, const __nv_bfloat16* __restrict__ x, const Dims& dm,
                                               int b, int h, int n0) {
  constexpr int VPR = D / 8;
  for (int e = threadIdx.x; e < 64 * VPR; e += 128) {
    const int r = e / VPR, cv = e % VPR, n = n0 + r;
    const bool ok = n < dm.N;
    cp_async16(smem_u32(s + r * (D + 8) + cv * 8), x + (((size_t)b * dm.N + (ok ? n : 0)) * dm.H + h) * D + cv * 8,
               ok ? 16 : 0);
  }
}

// acc[nt] (16 x 64 per warp) = A (rows 16 w.. of sA) times B^T (rows of sB), K = D
template <int D>
__device__ __forceinline__ void mma_rows_abt(float (&acc)[8][4], const __nv_bfloat16* sA, const __nv_bfloat16* sB,
                                             int warp, int lane) {
  constexpr int DP = D + 8;
  const int quad = lane >> 3;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t af[4];
    ldsm_x4(smem_u32(sA + (16 * warp + (lane & 15)) * DP + kk * 16 + (lane >> 4) * 8), af[0], af[1], af[2], af[3]);
#pragma unroll
    for (int nt = 0; nt < 8; nt += 2) {
      uint32_t bf[4];
      ldsm_x4(smem_u32(sB + ((nt + (quad >> 1)) * 8 + (lane & 7)) * DP + kk * 16 + (quad & 1) * 8), bf[0], bf[1],
              bf[2], bf[3]);
      mma_bf16(acc[nt], af, bf);
      mma_bf16(acc[nt + 1], af, bf + 2);
    }
  }
}

// acc (16 x D per warp) += X (16 x 64, accumulator layout, as bf16 hi + lo) times sB (64 x D)
template <int D>
__device__ __forceinline__ void mma_rows_xb(float (&acc)[D / 8][4], const float (&x)[8][4], const __nv_bfloat16* sB,
                                            int lane) {
  constexpr int DP = D + 8;
  const int quad = lane >> 3;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t hi[4], lo[4];
    split_bf16(x[2 * kk][0], x[2 * kk][1], hi[0], lo[0]);
    split_bf16(x[2 * kk][2], x[2 * kk][3], hi[1], lo[1]);
    split_bf16(x[2 * kk + 1][0], x[2 * kk + 1][1], hi[2], lo[2]);
    split_bf16(x[2 * kk + 1][2], x[2 * kk + 1][3], hi[3], lo[3]);
#pragma unroll
    for (int nt = 0; nt < D / 8; nt += 2) {
      uint32_t bf[4];
      ldsm_x4_t(smem_u32(sB + (kk * 16 + (quad & 1) * 8 + (lane & 7)) * DP + (nt + (quad >> 1)) * 8), bf[0], bf[1],
                bf[2], bf[3]);
      mma_bf16(acc[nt], hi, bf);
      mma_bf16(acc[nt + 1], hi, bf + 2);
      mma_bf16(acc[nt], lo, bf);
      mma_bf16(acc[nt + 1], lo, bf + 2);
    }
  }
}

// Row statistics on the tensor cores.  D_n = dout_n . O_n = sum_m P_nm (dout_n . v_m), so the
// row's D is accumulated online like its softmax sum, from dP = dout V^T (one exact bf16
// product per block) instead of forming O.
template <int D>
__device__ __forceinline__ void rowstats_mma_tile(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const __nv_bfloat16* __restrict__ dout, const Dims& dm, const int32_t* __restrict__ col_idx,
    float* __restrict__ lse, float* __restrict__ Drow, int* __restrict__ status, int i, int bh, unsigned char* smb) {
  using L = MmaTiles<D>;
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smb);
  __nv_bfloat16* sG = sQ + L::kTile;
  __nv_bfloat16* sK = sG + L::kTile;
  __nv_bfloat16* sV = sK + L::kTile;
  const int b = bh / dm.H, h = bh % dm.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g8 = lane >> 2, t4 = lane & 3;
  const int32_t* Lst = col_idx + ((size_t)bh * dm.nb + i) * dm.k;
  const float sl2 = dm.scale * 1.4426950408889634f;
  load_tile_bf16<D>(sQ, q, dm, b, h, i * 64);
  load_tile_bf16<D>(sG, dout, dm, b, h, i * 64);
  cp_async_commit();
  // per row half hh: running max m (log2 units), sum l and sum of p dP (this thread's columns)
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, pd[2] = {0.f, 0.f};
  for (int jj = 0; jj < dm.k; ++jj) {
    const int j = checked_block(dm, Lst[jj], status);
    __syncthreads();
    load_tile_bf16<D>(sK, k, dm, b, h, j * 64);
    load_tile_bf16<D>(sV, v, dm, b, h, j * 64);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    float s[8][4], dp[8][4];
    mma_rows_abt<D>(s, sQ, sK, warp, lane);
    mma_rows_abt<D>(dp, sG, sV, warp, lane);
    const int nvalid = min(64, dm.N - j * 64);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 2 * hh; e < 2 * hh + 2; ++e) {
          s[nt][e] = nt * 8 + 2 * t4 + (e & 1) < nvalid ? s[nt][e] * sl2 : -INFINITY;
          mx = fmaxf(mx, s[nt][e]);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float mnew = fmaxf(m[hh], mx);
      const float corr = m[hh] == -INFINITY ? 0.f : exp2f(m[hh] - mnew);
      float rs = 0.f, rd = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 2 * hh; e < 2 * hh + 2; ++e) {
          const float p = exp2f(s[nt][e] - mnew);
          rs += p;
          rd = fmaf(p, dp[nt][e], rd);
        }
      l[hh] = l[hh] * corr + rs;
      pd[hh] = pd[hh] * corr + rd;
      m[hh] = mnew;
    }
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float lt = l[hh], dt = pd[hh];
    lt += __shfl_xor_sync(0xffffffffu, lt, 1);
    lt += __shfl_xor_sync(0xffffffffu, lt, 2);
    dt += __shfl_xor_sync(0xffffffffu, dt, 1);
    dt += __shfl_xor_sync(0xffffffffu, dt, 2);
    const int row = 16 * warp + g8 + 8 * hh, n = i * 64 + row;
    if (t4 == 0) {
      const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + row;
      lse[at] = n < dm.N ? m[hh] + log2f(lt) : INFINITY;   // log2 units of scale * log2(e) * q.k
      Drow[at] = n < dm.N ? dt / lt : 0.f;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(128) bwd_rowstats_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const __nv_bfloat16* __restrict__ dout, Dims dm, const int32_t* __restrict__ col_idx, float* __restrict__ lse,
    float* __restrict__ Drow, int* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smb[];
  rowstats_mma_tile<D>(q, k, v, dout, dm, col_idx, lse, Drow, status, blockIdx.x, blockIdx.y, smb);
}

// The query tiles listed in redo (count, then tiles b*H*nb + h*nb + i), grid-strided.
template <int D>
__global__ void __launch_bounds__(128) bwd_rowstats_redo_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const __nv_bfloat16* __restrict__ dout, Dims dm, const int32_t* __restrict__ col_idx, float* __restrict__ lse,
    float* __restrict__ Drow, const int* __restrict__ redo, int* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smb[];
  const int count = min(redo[0], dm.B * dm.H * dm.nb);   // each tile is listed at most once
  for (int e = blockIdx.x; e < count; e += gridDim.x) {
    const int tau = redo[1 + e];
    if (tau < 0 || tau >= dm.B * dm.H * dm.nb) {
      if (threadIdx.x == 0) record_status(status, kDevBounds);
      continue;
    }
    __syncthreads();   // the previous tile's shared memory is read out
    rowstats_mma_tile<D>(q, k, v, dout, dm, col_idx, lse, Drow, status, tau % dm.nb, tau / dm.nb, smb);
  }
}

template <int D>
__global__ void __launch_bounds__(128) bwd_dq_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const __nv_bfloat16* __restrict__ dout, Dims dm, const int32_t* __restrict__ col_idx,
    const float* __restrict__ lse, const float* __restrict__ Drow, float* __restrict__ dq, int* __restrict__ status) {
  using L = MmaTiles<D>;
  extern __shared__ __align__(16) unsigned char smb[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smb);
  __nv_bfloat16* sG = sQ + L::kTile;
  __nv_bfloat16* sK = sG + L::kTile;
  __nv_bfloat16* sV = sK + L::kTile;
  const int i = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g8 = lane >> 2, t4 = lane & 3;
  const int32_t* Lst = col_idx + ((size_t)bh * dm.nb + i) * dm.k;
  const float sl2 = dm.scale * 1.4426950408889634f;
  load_tile_bf16<D>(sQ, q, dm, b, h, i * 64);
  load_tile_bf16<D>(sG, dout, dm, b, h, i * 64);
  cp_async_commit();
  float ls[2], dd[2], acc[D / 8][4];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + 16 * warp + g8 + 8 * hh;
    ls[hh] = lse[at];
    dd[hh] = Drow[at];
  }
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  for (int jj = 0; jj < dm.k; ++jj) {
    const int j = checked_block(dm, Lst[jj], status);
    __syncthreads();
    load_tile_bf16<D>(sK, k, dm, b, h, j * 64);
    load_tile_bf16<D>(sV, v, dm, b, h, j * 64);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    float s[8][4], dp[8][4];
    mma_rows_abt<D>(s, sQ, sK, warp, lane);
    mma_rows_abt<D>(dp, sG, sV, warp, lane);
    const int nvalid = min(64, dm.N - j * 64);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hh = e >> 1;
        const float p = nt * 8 + 2 * t4 + (e & 1) < nvalid ? exp2f(s[nt][e] * sl2 - ls[hh]) : 0.f;
        s[nt][e] = p * (dp[nt][e] - dd[hh]);
      }
    mma_rows_xb<D>(acc, s, sK, lane);
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int n = i * 64 + 16 * warp + g8 + 8 * hh;
    if (n >= dm.N) continue;
    float2* row = reinterpret_cast<float2*>(dq + (((size_t)b * dm.N + n) * dm.H + h) * D);
    float2 cur[D / 8];               // all loads first, then the stores
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) cur[nt] = row[nt * 4 + t4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
      row[nt * 4 + t4] = make_float2(fmaf(dm.scale, acc[nt][2 * hh], cur[nt].x),
                                     fmaf(dm.scale, acc[nt][2 * hh + 1], cur[nt].y));
  }
}

template <int D>
__global__ void __launch_bounds__(128) bwd_dkv_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const __nv_bfloat16* __restrict__ dout, Dims dm, const int* __restrict__ inv_off, const int* __restrict__ inv_idx,
    const float* __restrict__ lse, const float* __restrict__ Drow, float* __restrict__ dk, float* __restrict__ dv) {
  using L = MmaTiles<D>;
  extern __shared__ __align__(16) unsigned char smb[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smb);
  __nv_bfloat16* sV = sK + L::kTile;
  __nv_bfloat16* sQ = sV + L::kTile;
  __nv_bfloat16* sG = sQ + L::kTile;
  float* sL = reinterpret_cast<float*>(sG + L::kTile);   // [64] lse of the query tile
  float* sD = sL + 64;                                     // [64] D of the query tile
  const int j = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g8 = lane >> 2, t4 = lane & 3;
  const float sl2 = dm.scale * 1.4426950408889634f;
  load_tile_bf16<D>(sK, k, dm, b, h, j * 64);
  load_tile_bf16<D>(sV, v, dm, b, h, j * 64);
  cp_async_commit();
  float ak[D / 8][4], av[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) ak[nt][e] = av[nt][e] = 0.f;
  const int* lst = inv_idx + (size_t)bh * dm.nb * dm.k;
  const int e0 = inv_off[(size_t)bh * (dm.nb + 1) + j], e1 = inv_off[(size_t)bh * (dm.nb + 1) + j + 1];
  for (int e = e0; e < e1; ++e) {
    const int i = lst[e];
    __syncthreads();
    load_tile_bf16<D>(sQ, q, dm, b, h, i * 64);
    load_tile_bf16<D>(sG, dout, dm, b, h, i * 64);
    cp_async_commit();
    if (threadIdx.x < 64) {
      const size_t at = (size_t)bh * dm.nb * 64 + (size_t)i * 64 + threadIdx.x;
      sL[threadIdx.x] = lse[at];
      sD[threadIdx.x] = Drow[at];
    }
    cp_async_wait<0>();
    __syncthreads();
    float st[8][4], dpt[8][4];          // rows: keys 16 w + g8 (+ 8); columns: queries
    mma_rows_abt<D>(st, sK, sQ, warp, lane);
    mma_rows_abt<D>(dpt, sV, sG, warp, lane);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int qc = nt * 8 + 2 * t4 + (x & 1);
        const float p = exp2f(st[nt][x] * sl2 - sL[qc]);   // 0 for queries past N (lse = +inf)
        st[nt][x] = p;
        dpt[nt][x] = p * (dpt[nt][x] - sD[qc]);
      }
    mma_rows_xb<D>(av, st, sG, lane);
    mma_rows_xb<D>(ak, dpt, sQ, lane);
  }
  const int nvalid = min(64, dm.N - j * 64);
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r = 16 * warp + g8 + 8 * hh;
    if (r >= nvalid) continue;
    const size_t at = (((size_t)b * dm.N + j * 64 + r) * dm.H + h) * D;
    float2* rk = reinterpret_cast<float2*>(dk + at);
    float2* rv = reinterpret_cast<float2*>(dv + at);
    float2 ck[D / 8], cv[D / 8];     // all loads first, then the stores
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      ck[nt] = rk[nt * 4 + t4];
      cv[nt] = rv[nt * 4 + t4];
    }
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      rk[nt * 4 + t4] = make_float2(fmaf(dm.scale, ak[nt][2 * hh], ck[nt].x), fmaf(dm.scale, ak[nt][2 * hh + 1], ck[nt].y));
      rv[nt * 4 + t4] = make_float2(cv[nt].x + av[nt][2 * hh], cv[nt].y + av[nt][2 * hh + 1]);
    }
  }
}

// For each (b, h): the query blocks that kept each key block, ascending (the key-major
// view of the lists).  Counts, an exclusive scan, a scatter, then each list sorted.
__global__ void __launch_bounds__(kT) bwd_inverse_lists_kernel(Dims dm, const int32_t* __restrict__ col_idx,
                                                               int* __restrict__ inv_off, int* __restrict__ inv_idx) {
  extern __shared__ int cnt[];   // [nb + 1]
  const int bh = blockIdx.x;
  const int32_t* L = col_idx + (size_t)bh * dm.nb * dm.k;
  int* off = inv_off + (size_t)bh * (dm.nb + 1);
  int* idx = inv_idx + (size_t)bh * dm.nb * dm.k;
  for (int j = threadIdx.x; j <= dm.nb; j += kT) cnt[j] = 0;
  __syncthreads();
  const int total = dm.nb * dm.k;
  for (int e = threadIdx.x; e < total; e += kT) {
    const int j = L[e];
    if (j >= 0 && j < dm.nb) atomicAdd(&cnt[j], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int j = 0; j < dm.nb; ++j) {
      const int c = cnt[j];
      off[j] = run;
      cnt[j] = run;            // becomes the scatter cursor
      run += c;
    }
    off[dm.nb] = run;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < total; e += kT) {
    const int j = L[e];
    if (j >= 0 && j < dm.nb) idx[atomicAdd(&cnt[j], 1)] = e / dm.k;
  }
  __syncthreads();
  __threadfence_block();
  for (int j = threadIdx.x; j < dm.nb; j += kT) {   // insertion sort of each list
    const int a = off[j], z = off[j + 1];
    for (int x = a + 1; x < z; ++x) {
      const int val = idx[x];
      int y = x - 1;
      while (y >= a && idx[y] > val) {
        idx[y + 1] = idx[y];
        --y;
      }
      idx[y + 1] = val;
    }
  }
}

// ------------------------------------------------------------------ linear branch
// Per chunk of tokens, 64-token tiles; the small products (64 x r x d) run as 4 x 4
// register tiles per thread over shared-memory operands (tile t = tid + 256 s: rows
// 4 (t / NT) .. + 3, columns t % NT + NT j), the per-row steps (phi, the rotation, the
// normaliser, the gain) one row or one rank pair per thread.
// The two token tiles stay in the inputs' type (bf16 rows padded by 2 elements, fp32 by 1),
// so that two CTAs fit an SM; everything else is fp32.
template <typename T, int D, int RK>
struct LinSmem {
  static constexpr int TT = D + (sizeof(T) == 2 ? 2 : 1);                       // tile row stride
  static constexpr size_t kTileBytes = (sizeof(T) * 64 * TT + 15) / 16 * 16;
  static constexpr int kW = D * (RK + 1);      // Wq or Wk [D][RK]
  static constexpr int kS = RK * (D + 1);      // S or dS [RK][D]
  static constexpr int kR = 64 * (RK + 1);     // [64][RK] row vectors
  static constexpr size_t bytes = 2 * kTileBytes + sizeof(float) * (kW + kS + 4 * kR + RK + 6 * 64);
};

// rows [n0, n0 + 64) of head h of a [B, N, H, D] tensor into s[64][TT] in its own type, by
// 16-byte loads; rows at or past N are zero
template <typename T, int D, int TT>
__device__ __forceinline__ void load_tile_t(T* s, const T* __restrict__ x, const Dims& dm, int b, int h, int n0) {
  constexpr int EV = 16 / sizeof(T);           // elements per 16-byte load
  for (int e = threadIdx.x; e < 64 * (D / EV); e += kT) {
    const int r = e / (D / EV), c = (e % (D / EV)) * EV, n = n0 + r;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (n < dm.N) val = *reinterpret_cast<const uint4*>(x + (((size_t)b * dm.N + n) * dm.H + h) * D + c);
    const uint32_t w[4] = {val.x, val.y, val.z, val.w};
    uint32_t* dst = reinterpret_cast<uint32_t*>(s + r * TT + c);   // 4-byte aligned for both types
#pragma unroll
    for (int u = 0; u < 4; ++u) dst[u] = w[u];
  }
}

// acc[s][i][j] += sum_k a(m, k) b(k, n) for the tiles of this thread of an M x N product
// (m = 4 (t / NT) + i, n = t % NT + NT j).
template <int M, int N, int K, int S_, class FA, class FB>
__device__ __forceinline__ void tile_gemm(float (&acc)[S_][4][4], FA a, FB b) {
  constexpr int NT = N / 4, TILES = (M / 4) * NT;
#pragma unroll
  for (int s = 0; s < S_; ++s) {
    const int t = threadIdx.x + kT * s;
    if (t >= TILES) break;
    const int m0 = 4 * (t / NT), n0 = t % NT;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = a(m0 + i, k);
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = b(k, n0 + NT * j);
#pragma unroll
      for (int i = 0; i < 4; ++i)   // two columns per packed f32x2 FMA, each rounded as fmaf
#pragma unroll
        for (int j = 0; j < 4; j += 2)
          sm100::fma2(acc[s][i][j], acc[s][i][j + 1], av[i], av[i], bv[j], bv[j + 1], acc[s][i][j], acc[s][i][j + 1]);
    }
  }
}

template <int M, int N>
constexpr int tiles_per_thread() { return ((M / 4) * (N / 4) + kT - 1) / kT; }

template <int S_>
__device__ __forceinline__ void zero_acc(float (&acc)[S_][4][4]) {
#pragma unroll
  for (int s = 0; s < S_; ++s)
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[s][i][j] = 0.f;
}

// Visits the elements of this thread's tiles: f(m, n, value).
template <int M, int N, int S_, class F>
__device__ __forceinline__ void tile_each(const float (&acc)[S_][4][4], F f) {
  constexpr int NT = N / 4, TILES = (M / 4) * NT;
#pragma unroll
  for (int s = 0; s < S_; ++s) {
    const int t = threadIdx.x + kT * s;
    if (t >= TILES) break;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) f(4 * (t / NT) + i, t % NT + NT * j, acc[s][i][j]);
  }
}

// (cos, sin) of rank pair p at token n (identity past N)
__device__ __forceinline__ float2 pair_cs(const Dims& dm, const float2* __restrict__ rope, int n, int p) {
  if (n >= dm.N) return make_float2(1.f, 0.f);
  return rope_at(dm, rope, token_pos(dm, n), p);
}

// Query side: per chunk of query tokens, the linear branch's dq (written; the sparse part
// is added later), the chunk's partial dS, dz, dWq and gain gradients.  With T = G S^T
// (the row's dout against each rank of the state), dg = y . T / den and dy = g T / den, so
// the linear output itself is never formed.
template <typename T, int D, int RK>
__global__ void __launch_bounds__(kT, 2) bwd_linear_query_kernel(
    const T* __restrict__ q, const T* __restrict__ dout, const T* __restrict__ Wq, const float* __restrict__ g,
    Dims dm, const float* __restrict__ S, const float* __restrict__ z, const float2* __restrict__ rope,
    float* __restrict__ dq, float* __restrict__ dg, float* __restrict__ dS_part, float* __restrict__ dz_part,
    float* __restrict__ dWq_part, float* __restrict__ dg_part) {
  using Lsm = LinSmem<T, D, RK>;
  constexpr int WS = RK + 1, TS = D + 1, TT = Lsm::TT;
  extern __shared__ __align__(16) unsigned char smraw[];
  T* sQ = reinterpret_cast<T*>(smraw);
  T* sG = reinterpret_cast<T*>(smraw + Lsm::kTileBytes);
  float* sW = reinterpret_cast<float*>(smraw + 2 * Lsm::kTileBytes);   // Wq [D][RK + 1]
  float* sS = sW + Lsm::kW;           // S [RK][D + 1]
  float* sX = sS + Lsm::kS;           // x, then dx [64][RK + 1]
  float* sU = sX + Lsm::kR;           // u
  float* sY = sU + Lsm::kR;           // R u
  float* sT = sY + Lsm::kR;           // G S^T
  float* sz = sT + Lsm::kR;           // z [RK]
  float* sgd = sz + RK;               // g / den per row [64]
  float* sdd = sgd + 64;              // dden per row
  float* sdl = sdd + 64;              // dlogit per row (gate from the query)
  float* sdg = sdl + 64;              // dg per row
  float* sdot = sdg + 64;             // q . wg per row
  float* sden = sdot + 64;            // den per row
  const int chunk = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int tid = threadIdx.x;
  const int n_begin = chunk * dm.chunk_tok, n_end = min(dm.N, n_begin + dm.chunk_tok);
  const bool qproj = dm.gate_mode == ROLA_GATE_QPROJ;
  for (int e = tid; e < D * RK; e += kT) sW[(e / RK) * WS + e % RK] = to_f(Wq[(size_t)h * D * RK + e]);
  for (int e = tid; e < RK * D; e += kT) sS[(e / D) * TS + e % D] = S[(size_t)bh * RK * D + e];
  if (tid < RK) sz[tid] = z[(size_t)bh * RK + tid];
  constexpr int SP = tiles_per_thread<RK, D>(), WP = tiles_per_thread<D, RK>();
  constexpr int XP = tiles_per_thread<64, RK>(), QP = tiles_per_thread<64, D>();
  float aS[SP][4][4], aW[WP][4][4];
  zero_acc(aS);
  zero_acc(aW);
  float az = 0.f, awg = 0.f, adg = 0.f, abg = 0.f;   // rank tid (dz), channel tid (dwg), sums
  for (int n0 = n_begin; n0 < n_end; n0 += 64) {
    __syncthreads();
    load_tile_t<T, D, TT>(sQ, q, dm, b, h, n0);
    load_tile_t<T, D, TT>(sG, dout, dm, b, h, n0);
    __syncthreads();
    // x = q Wq and T = G S^T
    {
      float ax[XP][4][4], at[XP][4][4];
      zero_acc(ax);
      zero_acc(at);
      tile_gemm<64, RK, D>(ax, [&](int m, int c) { return to_f(sQ[m * TT + c]); }, [&](int c, int a) { return sW[c * WS + a]; });
      tile_gemm<64, RK, D>(at, [&](int m, int c) { return to_f(sG[m * TT + c]); }, [&](int c, int a) { return sS[a * TS + c]; });
      tile_each<64, RK>(ax, [&](int m, int a, float x) {
        sX[m * WS + a] = x;
        sU[m * WS + a] = phi_f(x);
      });
      tile_each<64, RK>(at, [&](int m, int a, float x) { sT[m * WS + a] = x; });
    }
    if (qproj && tid < 64) {
      float dot = 0.f;
      for (int c = 0; c < D; ++c) dot = fmaf(to_f(sQ[tid * TT + c]), __ldg(g + (size_t)h * D + c), dot);
      sdot[tid] = dot;
    }
    __syncthreads();
    // y = R u (one rank pair per item) and the row's den = u . z
    for (int e = tid; e < 64 * (RK / 2); e += kT) {
      const int m = e / (RK / 2), p = e % (RK / 2);
      const float2 cs = pair_cs(dm, rope, n0 + m, p);
      const float x0 = sU[m * WS + 2 * p], x1 = sU[m * WS + 2 * p + 1];
      sY[m * WS + 2 * p] = cs.x * x0 - cs.y * x1;
      sY[m * WS + 2 * p + 1] = cs.y * x0 + cs.x * x1;
    }
    if (tid < 64) {
      float den = 0.f;
      for (int a = 0; a < RK; ++a) den = fmaf(sU[tid * WS + a], sz[a], den);
      sden[tid] = den;
    }
    __syncthreads();
    // per row: dg = y . T / den, the gain, g / den, dden = -g dg / den, dlogit
    if (tid < 64) {
      const int n = n0 + tid;
      const bool valid = n < n_end;
      const float den = sden[tid];
      float dgn = 0.f;
      for (int a = 0; a < RK; ++a) dgn = fmaf(sY[tid * WS + a], sT[tid * WS + a], dgn);
      dgn = valid ? dgn / den : 0.f;
      const float gn = qproj ? gate_sigmoid(dm, g, h, sdot[tid]) : g[gain_index(dm, b, valid ? n : n_begin, h)];
      sdg[tid] = dgn;
      sgd[tid] = valid ? gn / den : 0.f;
      sdd[tid] = -gn * dgn / den;
      sdl[tid] = valid ? dgn * gn * (1.f - gn) : 0.f;
      if (valid && dm.gate_mode == ROLA_GATE_TOKEN) dg[((size_t)b * dm.N + n) * dm.H + h] = dgn;
    }
    __syncthreads();
    // dy = (g / den) T, du = R^T dy + dden z, dx = phi'(x) du (one rank pair per item)
    for (int e = tid; e < 64 * (RK / 2); e += kT) {
      const int m = e / (RK / 2), p = e % (RK / 2);
      const float2 cs = pair_cs(dm, rope, n0 + m, p);
      const float gd = sgd[m], dd = sdd[m];
      const float y0 = gd * sT[m * WS + 2 * p], y1 = gd * sT[m * WS + 2 * p + 1];
      const float u0 = cs.x * y0 + cs.y * y1 + dd * sz[2 * p];
      const float u1 = -cs.y * y0 + cs.x * y1 + dd * sz[2 * p + 1];
      const bool valid = n0 + m < n_end;
      sX[m * WS + 2 * p] = valid ? dphi_f(sX[m * WS + 2 * p]) * u0 : 0.f;
      sX[m * WS + 2 * p + 1] = valid ? dphi_f(sX[m * WS + 2 * p + 1]) * u1 : 0.f;
    }
    __syncthreads();
    // dq = dx Wq^T (+ dlogit wg) for the valid rows
    {
      float aq[QP][4][4];
      zero_acc(aq);
      tile_gemm<64, D, RK>(aq, [&](int m, int a) { return sX[m * WS + a]; }, [&](int a, int c) { return sW[c * WS + a]; });
      tile_each<64, D>(aq, [&](int m, int c, float x) {
        const int n = n0 + m;
        if (n < n_end) {
          if (qproj) x = fmaf(sdl[m], __ldg(g + (size_t)h * D + c), x);
          dq[(((size_t)b * dm.N + n) * dm.H + h) * D + c] = x;
        }
      });
    }
    // dS += y^T (G g / den), dWq += Q^T dx, dz += dden u, the gains' sums (rows in order)
    tile_gemm<RK, D, 64>(aS, [&](int a, int m) { return sY[m * WS + a]; },
                         [&](int m, int c) { return to_f(sG[m * TT + c]) * sgd[m]; });
    tile_gemm<D, RK, 64>(aW, [&](int c, int m) { return to_f(sQ[m * TT + c]); }, [&](int m, int a) { return sX[m * WS + a]; });
    if (tid < RK)
      for (int m = 0; m < 64; ++m) az = fmaf(sdd[m], sU[m * WS + tid], az);
    if (qproj && tid < D)
      for (int m = 0; m < 64; ++m) awg = fmaf(sdl[m], to_f(sQ[m * TT + tid]), awg);
    if (tid == 0)
      for (int m = 0; m < 64; ++m) {
        adg += sdg[m];
        abg += sdl[m];
      }
  }
  const size_t pbase = (size_t)bh * dm.nchunk + chunk;
  tile_each<RK, D>(aS, [&](int a, int c, float x) { dS_part[pbase * RK * D + (size_t)a * D + c] = x; });
  tile_each<D, RK>(aW, [&](int c, int a, float x) { dWq_part[pbase * D * RK + (size_t)c * RK + a] = x; });
  if (tid < RK) dz_part[pbase * RK + tid] = az;
  float* gp = dg_part + pbase * (D + 1);
  if (qproj) {
    if (tid < D) gp[tid] = awg;
    if (tid == 0) gp[D] = abg;
  } else if (tid == 0) {
    gp[0] = adg;
  }
}

// dS, dz per (b, h): the chunks' partials summed in order.
template <int D, int RK>
__global__ void __launch_bounds__(kT) bwd_state_grad_reduce_kernel(Dims dm, const float* __restrict__ dS_part,
                                                                   const float* __restrict__ dz_part,
                                                                   float* __restrict__ dS, float* __restrict__ dz) {
  const int bh = blockIdx.x;
  for (int e = threadIdx.x; e < RK * D + RK; e += kT) {
    float acc = 0.f;
    if (e < RK * D) {
      for (int c = 0; c < dm.nchunk; ++c) acc += dS_part[((size_t)bh * dm.nchunk + c) * RK * D + e];
      dS[(size_t)bh * RK * D + e] = acc;
    } else {
      const int a = e - RK * D;
      for (int c = 0; c < dm.nchunk; ++c) acc += dz_part[((size_t)bh * dm.nchunk + c) * RK + a];
      dz[(size_t)bh * RK + a] = acc;
    }
  }
}

// Key side: per chunk of key tokens, the linear branch's dk and dv (written; the sparse
// parts are added later) and the chunk's partial dWk.  With Tk = V dS^T:
// dv = (R f) dS, df = R^T Tk + dz, dw = phi'(w) df, dk = dw Wk^T, dWk += K^T dw.
template <typename T, int D, int RK>
__global__ void __launch_bounds__(kT, 2) bwd_linear_key_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                            const T* __restrict__ Wk, Dims dm,
                                                            const float* __restrict__ dS, const float* __restrict__ dz,
                                                            const float2* __restrict__ rope, float* __restrict__ dk,
                                                            float* __restrict__ dv, float* __restrict__ dWk_part) {
  using Lsm = LinSmem<T, D, RK>;
  constexpr int WS = RK + 1, TS = D + 1, TT = Lsm::TT;
  extern __shared__ __align__(16) unsigned char smraw[];
  T* sK = reinterpret_cast<T*>(smraw);
  T* sV = reinterpret_cast<T*>(smraw + Lsm::kTileBytes);
  float* sW = reinterpret_cast<float*>(smraw + 2 * Lsm::kTileBytes);   // Wk [D][RK + 1]
  float* sS = sW + Lsm::kW;           // dS [RK][D + 1]
  float* sX = sS + Lsm::kS;           // w, then dw [64][RK + 1]
  float* sY = sX + Lsm::kR;           // R f
  float* sT = sY + Lsm::kR;           // V dS^T
  float* sz = sT + 2 * Lsm::kR;       // dz [RK]
  const int chunk = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int tid = threadIdx.x;
  const int n_begin = chunk * dm.chunk_tok, n_end = min(dm.N, n_begin + dm.chunk_tok);
  for (int e = tid; e < D * RK; e += kT) sW[(e / RK) * WS + e % RK] = to_f(Wk[(size_t)h * D * RK + e]);
  for (int e = tid; e < RK * D; e += kT) sS[(e / D) * TS + e % D] = dS[(size_t)bh * RK * D + e];
  if (tid < RK) sz[tid] = dz[(size_t)bh * RK + tid];
  constexpr int WP = tiles_per_thread<D, RK>(), XP = tiles_per_thread<64, RK>(), QP = tiles_per_thread<64, D>();
  float aW[WP][4][4];
  zero_acc(aW);
  for (int n0 = n_begin; n0 < n_end; n0 += 64) {
    __syncthreads();
    load_tile_t<T, D, TT>(sK, k, dm, b, h, n0);
    load_tile_t<T, D, TT>(sV, v, dm, b, h, n0);
    __syncthreads();
    {
      float ax[XP][4][4], at[XP][4][4];
      zero_acc(ax);
      zero_acc(at);
      tile_gemm<64, RK, D>(ax, [&](int m, int c) { return to_f(sK[m * TT + c]); }, [&](int c, int a) { return sW[c * WS + a]; });
      tile_gemm<64, RK, D>(at, [&](int m, int c) { return to_f(sV[m * TT + c]); }, [&](int c, int a) { return sS[a * TS + c]; });
      tile_each<64, RK>(ax, [&](int m, int a, float x) { sX[m * WS + a] = x; });
      tile_each<64, RK>(at, [&](int m, int a, float x) { sT[m * WS + a] = x; });
    }
    __syncthreads();
    // R f and dw = phi'(w) (R^T Tk + dz), one rank pair per item
    for (int e = tid; e < 64 * (RK / 2); e += kT) {
      const int m = e / (RK / 2), p = e % (RK / 2);
      const float2 cs = pair_cs(dm, rope, n0 + m, p);
      const float w0 = sX[m * WS + 2 * p], w1 = sX[m * WS + 2 * p + 1];
      const float f0 = phi_f(w0), f1 = phi_f(w1);
      sY[m * WS + 2 * p] = cs.x * f0 - cs.y * f1;
      sY[m * WS + 2 * p + 1] = cs.y * f0 + cs.x * f1;
      const float t0 = sT[m * WS + 2 * p], t1 = sT[m * WS + 2 * p + 1];
      const bool valid = n0 + m < n_end;
      sX[m * WS + 2 * p] = valid ? dphi_f(w0) * (cs.x * t0 + cs.y * t1 + sz[2 * p]) : 0.f;
      sX[m * WS + 2 * p + 1] = valid ? dphi_f(w1) * (-cs.y * t0 + cs.x * t1 + sz[2 * p + 1]) : 0.f;
    }
    __syncthreads();
    {
      float avv[QP][4][4], akk[QP][4][4];
      zero_acc(avv);
      zero_acc(akk);
      tile_gemm<64, D, RK>(avv, [&](int m, int a) { return sY[m * WS + a]; }, [&](int a, int c) { return sS[a * TS + c]; });
      tile_gemm<64, D, RK>(akk, [&](int m, int a) { return sX[m * WS + a]; }, [&](int a, int c) { return sW[c * WS + a]; });
      tile_each<64, D>(avv, [&](int m, int c, float x) {
        if (n0 + m < n_end) dv[(((size_t)b * dm.N + n0 + m) * dm.H + h) * D + c] = x;
      });
      tile_each<64, D>(akk, [&](int m, int c, float x) {
        if (n0 + m < n_end) dk[(((size_t)b * dm.N + n0 + m) * dm.H + h) * D + c] = x;
      });
    }
    tile_gemm<D, RK, 64>(aW, [&](int c, int m) { return to_f(sK[m * TT + c]); }, [&](int m, int a) { return sX[m * WS + a]; });
  }
  const size_t pbase = (size_t)bh * dm.nchunk + chunk;
  tile_each<D, RK>(aW, [&](int c, int a, float x) { dWk_part[pbase * D * RK + (size_t)c * RK + a] = x; });
}

// Per head: dWq, dWk and the per-head gain gradients summed over the batch and the chunks
// in order.
template <int D, int RK>
__global__ void __launch_bounds__(kT) bwd_head_reduce_kernel(Dims dm, const float* __restrict__ dWq_part,
                                                             const float* __restrict__ dWk_part,
                                                             const float* __restrict__ dg_part,
                                                             float* __restrict__ dWq, float* __restrict__ dWk,
                                                             float* __restrict__ dg) {
  const int h = blockIdx.x;
  for (int e = threadIdx.x; e < D * RK; e += kT) {
    float aq = 0.f, ak = 0.f;
    for (int b = 0; b < dm.B; ++b)
      for (int c = 0; c < dm.nchunk; ++c) {
        const size_t pb = ((size_t)(b * dm.H + h) * dm.nchunk + c) * D * RK + e;
        aq += dWq_part[pb];
        ak += dWk_part[pb];
      }
    dWq[(size_t)h * D * RK + e] = aq;
    dWk[(size_t)h * D * RK + e] = ak;
  }
  if (dm.gate_mode == ROLA_GATE_TOKEN) return;
  const int ng = dm.gate_mode == ROLA_GATE_QPROJ ? D + 1 : 1;
  for (int e = threadIdx.x; e < ng; e += kT) {
    float acc = 0.f;
    for (int b = 0; b < dm.B; ++b)
      for (int c = 0; c < dm.nchunk; ++c) acc += dg_part[((size_t)(b * dm.H + h) * dm.nchunk + c) * (D + 1) + e];
    if (dm.gate_mode == ROLA_GATE_QPROJ)
      (e < D ? dg[(size_t)h * D + e] : dg[(size_t)dm.H * D + h]) = acc;
    else
      dg[h] = acc;
  }
}

template <typename T, int D, int RK>
cudaError_t launch_all(const Dims& dm, const void* q_, const void* k_, const void* v_, const void* Wq_,
                       const void* Wk_, const float* g, const void* dout_, float* dq, float* dk, float* dv,
                       float* dWq, float* dWk, float* dg, const Workspace& ws, const BwdWorkspace& bw,
                       cudaStream_t st) {
  const T* q = static_cast<const T*>(q_);
  const T* k = static_cast<const T*>(k_);
  const T* v = static_cast<const T*>(v_);
  const T* Wq = static_cast<const T*>(Wq_);
  const T* Wk = static_cast<const T*>(Wk_);
  const T* dout = static_cast<const T*>(dout_);
  const int BH = dm.B * dm.H;
  cudaError_t e;
  constexpr size_t lin_smem = LinSmem<T, D, RK>::bytes;
  constexpr size_t tile = sizeof(float) * 64 * (D + 1), ptile = sizeof(float) * 64 * 65;
  constexpr size_t rs_smem = 3 * tile + ptile, dq_smem = 4 * tile + ptile, dkv_smem = 4 * tile + 2 * ptile + 128 * 4;
  if ((e = cudaFuncSetAttribute(bwd_linear_query_kernel<T, D, RK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)lin_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_linear_key_kernel<T, D, RK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)lin_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_inverse_lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(int) * (dm.nb + 1)))) != cudaSuccess)
    return e;
  dim3 gchunk(dm.nchunk, BH), gtile(dm.nb, BH);
  // linear branch: query side (writes dq and the token gains), the state gradient, key
  // side (writes dk, dv)
  bwd_linear_query_kernel<T, D, RK><<<gchunk, kT, lin_smem, st>>>(q, dout, Wq, g, dm, ws.S, ws.z, ws.rope, dq, dg,
                                                                  bw.dS_part, bw.dz_part, bw.dWq_part, bw.dg_part);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_state_grad_reduce_kernel<D, RK><<<BH, kT, 0, st>>>(dm, bw.dS_part, bw.dz_part, bw.dS, bw.dz);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_linear_key_kernel<T, D, RK><<<gchunk, kT, lin_smem, st>>>(k, v, Wk, dm, bw.dS, bw.dz, ws.rope, dk, dv,
                                                                bw.dWk_part);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_head_reduce_kernel<D, RK><<<dm.H, kT, 0, st>>>(dm, bw.dWq_part, bw.dWk_part, bw.dg_part, dWq, dWk, dg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // sparse branch: row statistics, the key-major lists, dq, then dk and dv
  bwd_inverse_lists_kernel<<<BH, kT, sizeof(int) * (dm.nb + 1), st>>>(dm, ws.col_idx, bw.inv_off, bw.inv_idx);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    constexpr size_t mm_smem = MmaTiles<D>::bytes;
    if ((e = cudaFuncSetAttribute(bwd_rowstats_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)mm_smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_dq_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)mm_smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_dkv_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)mm_smem)) != cudaSuccess)
      return e;
    if constexpr (D == 128) {   // tcgen05, with the rare overflowing tiles redone block by block
      if ((e = cudaFuncSetAttribute(bwd_rowstats_redo_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)mm_smem)) != cudaSuccess)
        return e;
      if ((e = launch_bwd_rowstats_sm100(dm, q, k, v, dout, ws, bw, st)) != cudaSuccess) return e;
      bwd_rowstats_redo_kernel<D><<<296, 128, mm_smem, st>>>(q, k, v, dout, dm, ws.col_idx, bw.lse, bw.Drow, bw.redo,
                                                             ws.status);
    } else {
      bwd_rowstats_mma_kernel<D><<<gtile, 128, mm_smem, st>>>(q, k, v, dout, dm, ws.col_idx, bw.lse, bw.Drow,
                                                              ws.status);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if constexpr (D == 128) {   // the forward's transposed tcgen05 tile
      if ((e = launch_bwd_dq_sm100(dm, q, k, v, dout, ws, bw, dq, st)) != cudaSuccess) return e;
    } else {
      bwd_dq_mma_kernel<D><<<gtile, 128, mm_smem, st>>>(q, k, v, dout, dm, ws.col_idx, bw.lse, bw.Drow, dq,
                                                        ws.status);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if constexpr (D == 128) return launch_bwd_dkv_sm100(dm, q, k, v, dout, ws, bw, dk, dv, st);
    bwd_dkv_mma_kernel<D><<<gtile, 128, mm_smem, st>>>(q, k, v, dout, dm, bw.inv_off, bw.inv_idx, bw.lse, bw.Drow,
                                                       dk, dv);
    return cudaGetLastError();
  } else {
    if ((e = cudaFuncSetAttribute(bwd_rowstats_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)rs_smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_dq_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)dq_smem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_dkv_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)dkv_smem)) != cudaSuccess)
      return e;
    bwd_rowstats_kernel<T, D><<<gtile, kT, rs_smem, st>>>(q, k, v, dout, dm, ws.col_idx, bw.lse, bw.Drow,
                                                          ws.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_dq_kernel<T, D><<<gtile, kT, dq_smem, st>>>(q, k, v, dout, dm, ws.col_idx, bw.lse, bw.Drow, dq, ws.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_dkv_kernel<T, D><<<gtile, kT, dkv_smem, st>>>(q, k, v, dout, dm, bw.inv_off, bw.inv_idx, bw.lse, bw.Drow,
                                                       dk, dv);
    return cudaGetLastError();
  }
}

template <typename T>
cudaError_t launch_dtype(const Dims& dm, const void* q, const void* k, const void* v, const void* Wq, const void* Wk,
                         const float* g, const void* dout, float* dq, float* dk, float* dv, float* dWq, float* dWk,
                         float* dg, const Workspace& ws, const BwdWorkspace& bw, cudaStream_t st) {
#define ROLA_BWD(D_, R_) launch_all<T, D_, R_>(dm, q, k, v, Wq, Wk, g, dout, dq, dk, dv, dWq, dWk, dg, ws, bw, st)
  if (dm.d == 128) return dm.r == 32 ? ROLA_BWD(128, 32) : ROLA_BWD(128, 16);
  return dm.r == 32 ? ROLA_BWD(64, 32) : ROLA_BWD(64, 16);
#undef ROLA_BWD
}

}  // namespace

size_t backward_workspace_bytes(const Dims& dm, BwdWorkspace* bw, char* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* r = base ? base + off : nullptr;
    off = (off + bytes + 255) / 256 * 256;
    return r;
  };
  const size_t BH = (size_t)dm.B * dm.H;
  BwdWorkspace w{};
  w.lse = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb * 64));
  w.Drow = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nb * 64));
  w.inv_off = reinterpret_cast<int*>(take(sizeof(int) * BH * (dm.nb + 1)));
  w.inv_idx = reinterpret_cast<int*>(take(sizeof(int) * BH * dm.nb * dm.k));
  w.dS_part = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nchunk * dm.r * dm.d));
  w.dz_part = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nchunk * dm.r));
  w.dWq_part = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nchunk * dm.d * dm.r));
  w.dWk_part = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nchunk * dm.d * dm.r));
  w.dg_part = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.nchunk * (dm.d + 1)));
  w.dS = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.r * dm.d));
  w.dz = reinterpret_cast<float*>(take(sizeof(float) * BH * dm.r));
  w.redo = reinterpret_cast<int*>(take(sizeof(int) * (1 + BH * dm.nb)));
  if (bw) *bw = w;
  return off;
}

cudaError_t launch_backward(const Dims& dm, rola_dtype dt, const void* q, const void* k, const void* v,
                            const void* Wq, const void* Wk, const float* g, const void* dout, float* dq, float* dk,
                            float* dv, float* dWq, float* dWk, float* dg, const Workspace& ws,
                            const BwdWorkspace& bw, cudaStream_t st) {
  if (dt == ROLA_F32)
    return launch_dtype<float>(dm, q, k, v, Wq, Wk, g, dout, dq, dk, dv, dWq, dWk, dg, ws, bw, st);
  return launch_dtype<__nv_bfloat16>(dm, q, k, v, Wq, Wk, g, dout, dq, dk, dv, dWq, dWk, dg, ws, bw, st);
}

}  // namespace rola
