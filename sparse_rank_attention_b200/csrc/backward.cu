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
#include "rola_internal.cuh"

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
template <int D, int RK>
struct LinSmem {
  static constexpr int kTile = 64 * (D + 1);
  static constexpr int kW = D * (RK + 1);      // Wq or Wk [D][RK]
  static constexpr int kS = RK * (D + 1);      // S or dS [RK][D]
  static constexpr int kR = 64 * (RK + 1);     // [64][RK] row vectors
  static constexpr size_t bytes = sizeof(float) * (2 * kTile + kW + kS + 3 * kR + RK + 3 * 64);
};

// Rotation of the rank pairs of row `n` (this thread's RK / 4 ranks from a0): y = R x, or
// R^T x when back is set.
template <int Q>
__device__ __forceinline__ void rotate_q(const Dims& dm, const float2* __restrict__ rope, int n, int a0,
                                         const float (&x)[Q], float (&y)[Q], bool back) {
  const TokPos pos = token_pos(dm, n < dm.N ? n : 0);
#pragma unroll
  for (int p = 0; p < Q / 2; ++p) {
    const float2 cs = n < dm.N ? rope_at(dm, rope, pos, a0 / 2 + p) : make_float2(1.f, 0.f);
    const float sn = back ? -cs.y : cs.y;
    y[2 * p] = cs.x * x[2 * p] - sn * x[2 * p + 1];
    y[2 * p + 1] = sn * x[2 * p] + cs.x * x[2 * p + 1];
  }
}

// Query side: per chunk of query tokens, the linear branch's dq (written, the sparse part
// is added later), the chunk's partial dS, dz, dWq and gain gradients.
template <typename T, int D, int RK>
__global__ void __launch_bounds__(kT) bwd_linear_query_kernel(
    const T* __restrict__ q, const T* __restrict__ dout, const T* __restrict__ Wq, const float* __restrict__ g,
    Dims dm, const float* __restrict__ S, const float* __restrict__ z, const float2* __restrict__ rope,
    float* __restrict__ dq, float* __restrict__ dg, float* __restrict__ dS_part, float* __restrict__ dz_part,
    float* __restrict__ dWq_part, float* __restrict__ dg_part) {
  using Lsm = LinSmem<D, RK>;
  constexpr int QR = RK / 4, QC = D / 4, PT = D * RK / kT;
  extern __shared__ float sm[];
  float* sQ = sm;
  float* sG = sQ + Lsm::kTile;
  float* sW = sG + Lsm::kTile;        // Wq [D][RK + 1]
  float* sS = sW + Lsm::kW;           // S [RK][D + 1]
  float* sY = sS + Lsm::kS;           // R u [64][RK + 1]
  float* sX = sY + Lsm::kR;           // dx [64][RK + 1]
  float* sZr = sX + Lsm::kR;          // dz partials of the last tile [64][RK + 1]
  float* sz = sZr + Lsm::kR;          // z [RK]
  float* sgd = sz + RK;               // g / den per row [64]
  float* sdl = sgd + 64;              // dlogit per row (gate from the query) [64]
  float* sdg = sdl + 64;              // dg per row [64]
  const int chunk = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int tid = threadIdx.x, row = tid >> 2, qt = tid & 3, a0 = qt * QR, c0 = qt * QC;
  const int n_begin = chunk * dm.chunk_tok, n_end = min(dm.N, n_begin + dm.chunk_tok);
  for (int e = tid; e < D * RK; e += kT) sW[(e / RK) * (RK + 1) + e % RK] = to_f(Wq[(size_t)h * D * RK + e]);
  for (int e = tid; e < RK * D; e += kT) sS[(e / D) * (D + 1) + e % D] = S[(size_t)bh * RK * D + e];
  if (tid < RK) sz[tid] = z[(size_t)bh * RK + tid];
  // per-thread accumulators: dS[a][c] and dWq[c][a] for c = tid % D, a in the thread's
  // block of PT ranks; dz over this thread's rows; the gain's parts
  const int pc = tid % D, pa = (tid / D) * PT;
  float aS[PT], aW[PT], aZ[QR], adg = 0.f, awg = 0.f, abg = 0.f;
#pragma unroll
  for (int x = 0; x < PT; ++x) aS[x] = aW[x] = 0.f;
#pragma unroll
  for (int x = 0; x < QR; ++x) aZ[x] = 0.f;
  for (int n0 = n_begin; n0 < n_end; n0 += 64) {
    __syncthreads();
    load_tile<T, D>(sQ, q, dm, b, h, n0);
    load_tile<T, D>(sG, dout, dm, b, h, n0);
    __syncthreads();
    const int n = n0 + row;
    const bool valid = n < n_end;
    // x = q Wq (this thread's ranks), u = phi(x), y = R u, den = u . z
    float x[QR], u[QR], y[QR];
#pragma unroll
    for (int a = 0; a < QR; ++a) x[a] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float qv = sQ[row * (D + 1) + c];
#pragma unroll
      for (int a = 0; a < QR; ++a) x[a] = fmaf(qv, sW[c * (RK + 1) + a0 + a], x[a]);
    }
    float den = 0.f;
#pragma unroll
    for (int a = 0; a < QR; ++a) {
      u[a] = phi_f(x[a]);
      den = fmaf(u[a], sz[a0 + a], den);
    }
    den += __shfl_xor_sync(0xffffffffu, den, 1);
    den += __shfl_xor_sync(0xffffffffu, den, 2);
    rotate_q<QR>(dm, rope, n, a0, u, y, false);
#pragma unroll
    for (int a = 0; a < QR; ++a) sY[row * (RK + 1) + a0 + a] = y[a];
    // the gain of the token
    float gn;
    if (dm.gate_mode == ROLA_GATE_QPROJ) {
      float dot = 0.f;
      for (int c = c0; c < c0 + QC; ++c) dot = fmaf(sQ[row * (D + 1) + c], __ldg(g + (size_t)h * D + c), dot);
      dot += __shfl_xor_sync(0xffffffffu, dot, 1);
      dot += __shfl_xor_sync(0xffffffffu, dot, 2);
      gn = gate_sigmoid(dm, g, h, dot);
    } else {
      gn = g[gain_index(dm, b, valid ? n : n_begin, h)];
    }
    __syncthreads();
    // L = y^T S / den on this thread's columns; dg = dout . L
    float dgn = 0.f;
    float Lc[QC];
#pragma unroll
    for (int c = 0; c < QC; ++c) Lc[c] = 0.f;
    for (int a = 0; a < RK; ++a) {
      const float ya = sY[row * (RK + 1) + a];
#pragma unroll
      for (int c = 0; c < QC; ++c) Lc[c] = fmaf(ya, sS[a * (D + 1) + c0 + c], Lc[c]);
    }
#pragma unroll
    for (int c = 0; c < QC; ++c) dgn = fmaf(sG[row * (D + 1) + c0 + c], Lc[c] / den, dgn);
    dgn += __shfl_xor_sync(0xffffffffu, dgn, 1);
    dgn += __shfl_xor_sync(0xffffffffu, dgn, 2);
    if (!valid) dgn = 0.f;
    // dy = S gG / den on this thread's ranks; dden = -g dg / den
    const float gd = valid ? gn / den : 0.f;
    float dy[QR];
#pragma unroll
    for (int a = 0; a < QR; ++a) dy[a] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float gv = sG[row * (D + 1) + c];
#pragma unroll
      for (int a = 0; a < QR; ++a) dy[a] = fmaf(sS[(a0 + a) * (D + 1) + c], gv, dy[a]);
    }
    const float dden = -gn * dgn / den;
    float du[QR];
#pragma unroll
    for (int a = 0; a < QR; ++a) dy[a] *= gd;
    rotate_q<QR>(dm, rope, n, a0, dy, du, true);
#pragma unroll
    for (int a = 0; a < QR; ++a) {
      du[a] = fmaf(dden, sz[a0 + a], du[a]);
      aZ[a] = fmaf(dden, u[a], aZ[a]);
      sX[row * (RK + 1) + a0 + a] = valid ? dphi_f(x[a]) * du[a] : 0.f;
    }
    if (qt == 0) {
      sgd[row] = gd;
      sdg[row] = dgn;
      sdl[row] = valid ? dgn * gn * (1.f - gn) : 0.f;
    }
    __syncthreads();
    // dq = Wq dx (+ dlogit wg), this thread's columns; the token's dg
    if (valid) {
      float* dqrow = dq + (((size_t)b * dm.N + n) * dm.H + h) * D;
#pragma unroll 4
      for (int c = 0; c < QC; ++c) {
        float acc = 0.f;
#pragma unroll
        for (int a = 0; a < RK; ++a) acc = fmaf(sW[(c0 + c) * (RK + 1) + a], sX[row * (RK + 1) + a], acc);
        if (dm.gate_mode == ROLA_GATE_QPROJ) acc = fmaf(sdl[row], __ldg(g + (size_t)h * D + c0 + c), acc);
        dqrow[c0 + c] = acc;
      }
      if (dm.gate_mode == ROLA_GATE_TOKEN && qt == 0) dg[((size_t)b * dm.N + n) * dm.H + h] = dgn;
    }
    // dS[a][c] += sum_rows y gG / den;  dWq[c][a] += sum_rows q dx  (c = pc, a from pa)
    for (int rr = 0; rr < 64; ++rr) {
      const float gq = sG[rr * (D + 1) + pc] * sgd[rr];
      const float qv = sQ[rr * (D + 1) + pc];
#pragma unroll
      for (int x2 = 0; x2 < PT; ++x2) {
        aS[x2] = fmaf(sY[rr * (RK + 1) + pa + x2], gq, aS[x2]);
        aW[x2] = fmaf(qv, sX[rr * (RK + 1) + pa + x2], aW[x2]);
      }
    }
    if (tid < D)
      for (int rr = 0; rr < 64; ++rr) awg = fmaf(sdl[rr], sQ[rr * (D + 1) + tid], awg);
    if (tid == 0)
      for (int rr = 0; rr < 64; ++rr) {
        adg += sdg[rr];
        abg += sdl[rr];
      }
  }
  // the chunk's partials: dS, dWq (fixed per thread), dz (rows summed in order), gain
  const size_t pbase = (size_t)bh * dm.nchunk + chunk;
#pragma unroll
  for (int x2 = 0; x2 < PT; ++x2) {
    dS_part[pbase * RK * D + (size_t)(pa + x2) * D + pc] = aS[x2];
    dWq_part[pbase * D * RK + (size_t)pc * RK + pa + x2] = aW[x2];
  }
  __syncthreads();
#pragma unroll
  for (int a = 0; a < QR; ++a) sZr[row * (RK + 1) + a0 + a] = aZ[a];
  __syncthreads();
  if (tid < RK) {
    float acc = 0.f;
    for (int rr = 0; rr < 64; ++rr) acc += sZr[rr * (RK + 1) + tid];
    dz_part[pbase * RK + tid] = acc;
  }
  float* gp = dg_part + pbase * (D + 1);
  if (dm.gate_mode == ROLA_GATE_QPROJ) {
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
// parts are added later) and the chunk's partial dWk.
template <typename T, int D, int RK>
__global__ void __launch_bounds__(kT) bwd_linear_key_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                                            const T* __restrict__ Wk, Dims dm,
                                                            const float* __restrict__ dS, const float* __restrict__ dz,
                                                            const float2* __restrict__ rope, float* __restrict__ dk,
                                                            float* __restrict__ dv, float* __restrict__ dWk_part) {
  using Lsm = LinSmem<D, RK>;
  constexpr int QR = RK / 4, QC = D / 4, PT = D * RK / kT;
  extern __shared__ float sm[];
  float* sK = sm;
  float* sV = sK + Lsm::kTile;
  float* sW = sV + Lsm::kTile;        // Wk [D][RK + 1]
  float* sS = sW + Lsm::kW;           // dS [RK][D + 1]
  float* sY = sS + Lsm::kS;           // R f [64][RK + 1]
  float* sX = sY + Lsm::kR;           // dw [64][RK + 1]
  float* sz = sX + 2 * Lsm::kR;       // dz [RK]
  const int chunk = blockIdx.x, bh = blockIdx.y, b = bh / dm.H, h = bh % dm.H;
  const int tid = threadIdx.x, row = tid >> 2, qt = tid & 3, a0 = qt * QR, c0 = qt * QC;
  const int n_begin = chunk * dm.chunk_tok, n_end = min(dm.N, n_begin + dm.chunk_tok);
  for (int e = tid; e < D * RK; e += kT) sW[(e / RK) * (RK + 1) + e % RK] = to_f(Wk[(size_t)h * D * RK + e]);
  for (int e = tid; e < RK * D; e += kT) sS[(e / D) * (D + 1) + e % D] = dS[(size_t)bh * RK * D + e];
  if (tid < RK) sz[tid] = dz[(size_t)bh * RK + tid];
  const int pc = tid % D, pa = (tid / D) * PT;
  float aW[PT];
#pragma unroll
  for (int x2 = 0; x2 < PT; ++x2) aW[x2] = 0.f;
  for (int n0 = n_begin; n0 < n_end; n0 += 64) {
    __syncthreads();
    load_tile<T, D>(sK, k, dm, b, h, n0);
    load_tile<T, D>(sV, v, dm, b, h, n0);
    __syncthreads();
    const int n = n0 + row;
    const bool valid = n < n_end;
    float w[QR], f[QR], y[QR];
#pragma unroll
    for (int a = 0; a < QR; ++a) w[a] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float kv = sK[row * (D + 1) + c];
#pragma unroll
      for (int a = 0; a < QR; ++a) w[a] = fmaf(kv, sW[c * (RK + 1) + a0 + a], w[a]);
    }
#pragma unroll
    for (int a = 0; a < QR; ++a) f[a] = phi_f(w[a]);
    rotate_q<QR>(dm, rope, n, a0, f, y, false);
#pragma unroll
    for (int a = 0; a < QR; ++a) sY[row * (RK + 1) + a0 + a] = y[a];
    // R^T (dS v) + dz on this thread's ranks
    float dyk[QR];
#pragma unroll
    for (int a = 0; a < QR; ++a) dyk[a] = 0.f;
    for (int c = 0; c < D; ++c) {
      const float vv = sV[row * (D + 1) + c];
#pragma unroll
      for (int a = 0; a < QR; ++a) dyk[a] = fmaf(sS[(a0 + a) * (D + 1) + c], vv, dyk[a]);
    }
    float df[QR];
    rotate_q<QR>(dm, rope, n, a0, dyk, df, true);
#pragma unroll
    for (int a = 0; a < QR; ++a) sX[row * (RK + 1) + a0 + a] = valid ? dphi_f(w[a]) * (df[a] + sz[a0 + a]) : 0.f;
    __syncthreads();
    if (valid) {
      const size_t at = (((size_t)b * dm.N + n) * dm.H + h) * D;
#pragma unroll 4
      for (int c = 0; c < QC; ++c) {
        float av = 0.f, ak = 0.f;
#pragma unroll
        for (int a = 0; a < RK; ++a) {
          av = fmaf(sY[row * (RK + 1) + a], sS[a * (D + 1) + c0 + c], av);
          ak = fmaf(sW[(c0 + c) * (RK + 1) + a], sX[row * (RK + 1) + a], ak);
        }
        dv[at + c0 + c] = av;
        dk[at + c0 + c] = ak;
      }
    }
    for (int rr = 0; rr < 64; ++rr) {
      const float kv = sK[rr * (D + 1) + pc];
#pragma unroll
      for (int x2 = 0; x2 < PT; ++x2) aW[x2] = fmaf(kv, sX[rr * (RK + 1) + pa + x2], aW[x2]);
    }
  }
  const size_t pbase = (size_t)bh * dm.nchunk + chunk;
#pragma unroll
  for (int x2 = 0; x2 < PT; ++x2) dWk_part[pbase * D * RK + (size_t)pc * RK + pa + x2] = aW[x2];
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
  constexpr size_t lin_smem = LinSmem<D, RK>::bytes;
  constexpr size_t tile = sizeof(float) * 64 * (D + 1), ptile = sizeof(float) * 64 * 65;
  constexpr size_t rs_smem = 3 * tile + ptile, dq_smem = 4 * tile + ptile, dkv_smem = 4 * tile + 2 * ptile + 128 * 4;
  if ((e = cudaFuncSetAttribute(bwd_linear_query_kernel<T, D, RK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)lin_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_linear_key_kernel<T, D, RK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)lin_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_rowstats_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)rs_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_dq_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dq_smem)) !=
          cudaSuccess ||
      (e = cudaFuncSetAttribute(bwd_dkv_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)dkv_smem)) != cudaSuccess ||
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
  // sparse branch
  bwd_rowstats_kernel<T, D><<<gtile, kT, rs_smem, st>>>(q, k, v, dout, dm, ws.col_idx, bw.lse, bw.Drow, ws.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_inverse_lists_kernel<<<BH, kT, sizeof(int) * (dm.nb + 1), st>>>(dm, ws.col_idx, bw.inv_off, bw.inv_idx);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dq_kernel<T, D><<<gtile, kT, dq_smem, st>>>(q, k, v, dout, dm, ws.col_idx, bw.lse, bw.Drow, dq, ws.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dkv_kernel<T, D><<<gtile, kT, dkv_smem, st>>>(q, k, v, dout, dm, bw.inv_off, bw.inv_idx, bw.lse, bw.Drow, dk,
                                                     dv);
  return cudaGetLastError();
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
