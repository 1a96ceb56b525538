// Block pooling (step 1) and block scores + top-k selection (step 2) of RoLA.
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (the sparse branch keeps the high-energy
// query-key blocks); "AlibabaResearch/SparkDiffusion" README, inference section (topk is
// the fraction of key blocks kept).  Block size, pooling rule and tie-break are this
// library's reading: 64-token blocks, fp32 means, lowest key-block index wins a tie.
//
// Both kernels reproduce a stated fp32 order exactly, so the block lists are bit-exact:
//   qbar = (fp32 sum of the block's tokens in token order) / count   (IEEE division)
//   s_ij = fma chain over channels 0..d-1 starting from 0
#include "rola_internal.cuh"

namespace rola {
namespace {

// ------------------------------------------------------------------ pooling

template <typename T>
struct PoolTraits;
template <>
struct PoolTraits<float> {
  static constexpr int kEPV = 4;  // elements per 16-byte vector
  __device__ static void add(float* acc, const uint4& v) {
    acc[0] = acc[0] + __uint_as_float(v.x);
    acc[1] = acc[1] + __uint_as_float(v.y);
    acc[2] = acc[2] + __uint_as_float(v.z);
    acc[3] = acc[3] + __uint_as_float(v.w);
  }
};
template <>
struct PoolTraits<__nv_bfloat16> {
  static constexpr int kEPV = 8;
  __device__ static void add(float* acc, const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc[2 * e] = acc[2 * e] + __uint_as_float(w[e] << 16);
      acc[2 * e + 1] = acc[2 * e + 1] + __uint_as_float(w[e] & 0xffff0000u);
    }
  }
};

// grid: x = vector-column tiles of 128 threads over H*d, y = block i, z = 2*b + tensor.
// One thread owns one 16-byte column vector and adds the block's tokens in order.
template <typename T>
__global__ void __launch_bounds__(128) pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                   Dims dm, float* __restrict__ qbar,
                                                   float* __restrict__ kbar) {
  constexpr int EPV = PoolTraits<T>::kEPV;
  constexpr int kBatch = 8;
  const int tensor = blockIdx.z & 1, b = blockIdx.z >> 1;
  const T* __restrict__ x = tensor ? k : q;
  float* __restrict__ xb = tensor ? kbar : qbar;
  const int HD = dm.H * dm.d;
  const int vcol = blockIdx.x * blockDim.x + threadIdx.x;
  if (vcol * EPV >= HD) return;
  const int i = blockIdx.y;
  const int n0 = i * kBlock, cnt = min(dm.N - n0, kBlock);
  const uint4* __restrict__ src =
      reinterpret_cast<const uint4*>(x + ((size_t)b * dm.N + n0) * HD) + vcol;
  const size_t vstride = (size_t)HD / EPV;
  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
  for (int t0 = 0; t0 < cnt; t0 += kBatch) {
    uint4 buf[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (t0 + u < cnt) buf[u] = __ldg(src + (size_t)(t0 + u) * vstride);
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (t0 + u < cnt) PoolTraits<T>::add(acc, buf[u]);
  }
  const int c0 = vcol * EPV;
  const int h = c0 / dm.d, ch = c0 % dm.d;
  float* dst = xb + (((size_t)b * dm.H + h) * dm.nb + i) * dm.d + ch;
  const float fc = (float)cnt;
#pragma unroll
  for (int e = 0; e < EPV; ++e) dst[e] = __fdiv_rn(acc[e], fc);
}

// ------------------------------------------------------------------ scores + top-k

constexpr int kSelThreads = 256;
constexpr int kKeyChunk = 64;
constexpr int kKTStride = kKeyChunk + 4;  // padded row of the transposed key chunk

__host__ __device__ inline int select_rows_per_cta(int nb) { return nb <= 1300 ? 32 : 16; }

__host__ __device__ inline size_t select_smem(int R, int d, int nb) {
  const int nbp = (nb + kKeyChunk - 1) / kKeyChunk * kKeyChunk;
  return sizeof(float) * ((size_t)R * (d + 1) + (size_t)d * kKTStride + (size_t)R * nbp) +
         sizeof(uint32_t) * 256 * (kSelThreads / 32);
}

// grid: x = row tiles of R query blocks, y = b*H + h.
// Phase 1: scores of R query blocks against all key blocks into shared memory.
// Phase 2: one warp per row: 4-pass 8-bit radix select of the k-th largest score,
// then one pass in index order emits the kept indices (ties -> lower index).
template <int R>
__global__ void __launch_bounds__(kSelThreads) select_kernel(Dims dm, const float* __restrict__ qbar,
                                                             const float* __restrict__ kbar,
                                                             int32_t* __restrict__ col_idx,
                                                             int* __restrict__ status) {
  constexpr int RPT = R / 16;  // rows per thread in phase 1
  extern __shared__ float smem[];
  const int d = dm.d, nb = dm.nb, kk = dm.k;
  const int nbp = (nb + kKeyChunk - 1) / kKeyChunk * kKeyChunk;
  float* qs = smem;                         // [R][d+1]
  float* kT = qs + R * (d + 1);             // [d][kKTStride]
  float* sc = kT + d * kKTStride;           // [R][nbp]
  uint32_t* hist_all = reinterpret_cast<uint32_t*>(sc + R * nbp);  // [8][256]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int bh = blockIdx.y;
  const int row0 = blockIdx.x * R;
  const float* qsrc = qbar + (size_t)bh * nb * d;
  const float* ksrc = kbar + (size_t)bh * nb * d;

  for (int e = tid; e < R * d; e += kSelThreads) {
    const int rr = e / d, c = e % d;
    qs[rr * (d + 1) + c] = (row0 + rr < nb) ? qsrc[(size_t)(row0 + rr) * d + c] : 0.f;
  }
  const int rg = tid / 16, kg = tid % 16;
  for (int j0 = 0; j0 < nb; j0 += kKeyChunk) {
    __syncthreads();
    for (int e = tid; e < kKeyChunk * d; e += kSelThreads) {
      const int jj = e / d, c = e % d;
      kT[c * kKTStride + jj] = (j0 + jj < nb) ? ksrc[(size_t)(j0 + jj) * d + c] : 0.f;
    }
    __syncthreads();
    float acc[RPT][4];
#pragma unroll
    for (int a = 0; a < RPT; ++a)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[a][e] = 0.f;
#pragma unroll 4
    for (int c = 0; c < d; ++c) {
      const float4 kv = *reinterpret_cast<const float4*>(&kT[c * kKTStride + kg * 4]);
#pragma unroll
      for (int a = 0; a < RPT; ++a) {
        const float qv = qs[(rg * RPT + a) * (d + 1) + c];
        acc[a][0] = fmaf(qv, kv.x, acc[a][0]);
        acc[a][1] = fmaf(qv, kv.y, acc[a][1]);
        acc[a][2] = fmaf(qv, kv.z, acc[a][2]);
        acc[a][3] = fmaf(qv, kv.w, acc[a][3]);
      }
    }
#pragma unroll
    for (int a = 0; a < RPT; ++a)
      *reinterpret_cast<float4*>(&sc[(rg * RPT + a) * nbp + j0 + kg * 4]) =
          make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
  }
  __syncthreads();

  uint32_t* hist = hist_all + warp * 256;
  const unsigned full = 0xffffffffu;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int rr = warp; rr < R; rr += kSelThreads / 32) {
    const int i = row0 + rr;
    if (i >= nb) break;
    uint32_t* key = reinterpret_cast<uint32_t*>(sc + rr * nbp);
    // Order-preserving map float -> uint32 (both zeros map to the key of +0).
    for (int j = lane; j < nb; j += 32) {
      float f = sc[rr * nbp + j];
      if (f == 0.f) f = 0.f;
      const uint32_t u = __float_as_uint(f);
      key[j] = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    __syncwarp();
    uint32_t prefix = 0, pmask = 0;
    int need = kk;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int bb = lane; bb < 256; bb += 32) hist[bb] = 0;
      __syncwarp();
      for (int j = lane; j < nb; j += 32) {
        const uint32_t u = key[j];
        if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
      }
      __syncwarp();
      int cntv[8], local = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {  // lane owns bins 255-8*lane-e, in descending order
        cntv[e] = (int)hist[255 - 8 * lane - e];
        local += cntv[e];
      }
      int incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(full, incl, off);
        if (lane >= off) incl += t;
      }
      const int excl = incl - local;
      const unsigned hit = __ballot_sync(full, excl < need && need <= incl);
      const int src = hit ? (__ffs(hit) - 1) : 0;
      int digit = 0, above = 0;
      if (lane == src) {
        int c = excl;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (c + cntv[e] >= need) {
            digit = 255 - 8 * lane - e;
            above = c;
            break;
          }
          c += cntv[e];
        }
      }
      digit = __shfl_sync(full, digit, src);
      above = __shfl_sync(full, above, src);
      need -= above;
      prefix |= (uint32_t)digit << shift;
      pmask |= 255u << shift;
      __syncwarp();
    }
    // prefix is the k-th largest key; `need` elements equal to it are kept.
    int32_t* out = col_idx + ((size_t)bh * nb + i) * kk;
    int written = 0, eqseen = 0;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t u = (j < nb) ? key[j] : 0u;
      const bool gt = (j < nb) && u > prefix;
      const bool eq = (j < nb) && u == prefix;
      const unsigned beq = __ballot_sync(full, eq);
      const bool keep = gt || (eq && eqseen + __popc(beq & lt_mask) < need);
      const unsigned bk = __ballot_sync(full, keep);
      const int pos = written + __popc(bk & lt_mask);
      if (keep) {
        if (pos < kk) out[pos] = j;
      }
      written += __popc(bk);
      eqseen += __popc(beq);
    }
    if (lane == 0 && written != kk) record_status(status, kDevBounds);
    __syncwarp();
  }
}

}  // namespace

cudaError_t launch_pool(const Dims& dm, rola_dtype dt, const void* q, const void* k,
                        const Workspace& ws, cudaStream_t st) {
  const int HD = dm.H * dm.d;
  if (dt == ROLA_F32) {
    dim3 grid((HD / 4 + 127) / 128, dm.nb, 2 * dm.B);
    pool_kernel<float><<<grid, 128, 0, st>>>(static_cast<const float*>(q),
                                             static_cast<const float*>(k), dm, ws.qbar, ws.kbar);
  } else {
    dim3 grid((HD / 8 + 127) / 128, dm.nb, 2 * dm.B);
    pool_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                     static_cast<const __nv_bfloat16*>(k), dm,
                                                     ws.qbar, ws.kbar);
  }
  return cudaGetLastError();
}

size_t select_smem_bytes(const Dims& dm) {
  return select_smem(select_rows_per_cta(dm.nb), dm.d, dm.nb);
}

cudaError_t launch_select(const Dims& dm, const Workspace& ws, cudaStream_t st) {
  const int R = select_rows_per_cta(dm.nb);
  const size_t smem = select_smem(R, dm.d, dm.nb);
  dim3 grid((dm.nb + R - 1) / R, dm.B * dm.H);
  cudaError_t e;
  if (R == 32) {
    e = cudaFuncSetAttribute(select_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<32><<<grid, kSelThreads, smem, st>>>(dm, ws.qbar, ws.kbar, ws.col_idx, ws.status);
  } else {
    e = cudaFuncSetAttribute(select_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<16><<<grid, kSelThreads, smem, st>>>(dm, ws.qbar, ws.kbar, ws.col_idx, ws.status);
  }
  return cudaGetLastError();
}

}  // namespace rola
