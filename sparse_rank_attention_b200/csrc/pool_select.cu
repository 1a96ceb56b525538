// Block pooling (step 1) and the top-k selection (step 2) of RoLA; the block scores that
// prune the selection come from the tensor cores (score_sm100.cu).
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (the sparse branch keeps the high-energy
// query-key blocks); "AlibabaResearch/SparkDiffusion" README, inference section (topk is
// the fraction of key blocks kept).  Block size, pooling rule and tie-break are this
// library's reading: 64-token blocks, fp32 means, lowest key-block index wins a tie.
//
// The kernels reproduce a stated fp32 order exactly, so the block lists are bit-exact:
//   qbar = (fp32 sum of the block's tokens in token order) / count   (IEEE division)
//   s_ij = fma chain over channels 0..d-1 starting from 0
// (s_ij is computed exactly for every block that the tensor-core scores cannot rule out).
#include <cuda_fp8.h>

#include <mutex>

#include "rola_internal.cuh"
#include "sm100_ptx.cuh"

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
  __device__ static float absmax(const uint4&) { return 0.f; }        // fp8 takes bf16 only
  __device__ static uint2 to_e4m3(const uint4&, float) { return make_uint2(0, 0); }
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
  __device__ static float absmax(const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e)
      m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xffff0000u))));
    return m;
  }
  // 8 bf16 values times `inv`, rounded to e4m3 (nearest, saturating), in element order.
  __device__ static uint2 to_e4m3(const uint4& v, float inv) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0, 0};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = make_float2(__uint_as_float(w[e] << 16) * inv, __uint_as_float(w[e] & 0xffff0000u) * inv);
      const uint32_t pair = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
      out[e >> 1] |= pair << (16 * (e & 1));
    }
    return make_uint2(out[0], out[1]);
  }
};

// grid: x = vector-column tiles of 128 threads over H*d, y = block i, z = 2*b + tensor.
// One thread owns one 16-byte column vector and adds the block's tokens in order.
// With FP8 (bf16 inputs only) the same CTA also quantises the block to e4m3: per
// (b, h, block) scale = absmax / 448 (1 if the block is all zero), x8 = RN-sat(x / scale).
template <typename T, bool FP8>
__global__ void __launch_bounds__(128) pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                   Dims dm, float* __restrict__ qbar,
                                                   float* __restrict__ kbar, uint8_t* __restrict__ q8,
                                                   uint8_t* __restrict__ k8, float* __restrict__ sq,
                                                   float* __restrict__ sk) {
  constexpr int EPV = PoolTraits<T>::kEPV;
  constexpr int kBatch = 8;
  const int tensor = blockIdx.z & 1, b = blockIdx.z >> 1;
  const T* __restrict__ x = tensor ? k : q;
  float* __restrict__ xb = tensor ? kbar : qbar;
  const int HD = dm.H * dm.d;
  const int vcol = blockIdx.x * blockDim.x + threadIdx.x;
  const bool active = vcol * EPV < HD;
  if (!FP8 && !active) return;
  const int i = blockIdx.y;
  const int n0 = i * kBlock, cnt = min(dm.N - n0, kBlock);
  const uint4* __restrict__ src =
      reinterpret_cast<const uint4*>(x + ((size_t)b * dm.N + n0) * HD) + vcol;
  const size_t vstride = (size_t)HD / EPV;
  float acc[EPV];
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
  if (active) {
    for (int t0 = 0; t0 < cnt; t0 += kBatch) {
      uint4 buf[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (t0 + u < cnt) buf[u] = __ldg(src + (size_t)(t0 + u) * vstride);
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (t0 + u < cnt) {
          PoolTraits<T>::add(acc, buf[u]);
          if (FP8) amax = fmaxf(amax, PoolTraits<T>::absmax(buf[u]));
        }
    }
    const int c0 = vcol * EPV;
    const int h = c0 / dm.d, ch = c0 % dm.d;
    float* dst = xb + (((size_t)b * dm.H + h) * dm.nb + i) * dm.d + ch;
    const float fc = (float)cnt;
#pragma unroll
    for (int e = 0; e < EPV; ++e) dst[e] = __fdiv_rn(acc[e], fc);
  }
  if constexpr (FP8) {
    // a head's d channels are d/8 consecutive threads (16 for d = 128, 8 for d = 64)
    const int per_head = dm.d / EPV;
    for (int off = 1; off < per_head; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (!active) return;
    const int h = vcol * EPV / dm.d;
    const float scale = amax > 0.f ? amax / 448.f : 1.f;
    const float inv = 1.f / scale;
    if ((vcol % per_head) == 0) (tensor ? sk : sq)[((size_t)b * dm.H + h) * dm.nb + i] = scale;
    uint8_t* dst8 = (tensor ? k8 : q8) + ((size_t)b * dm.N + n0) * HD + (size_t)vcol * EPV;
    for (int t = 0; t < cnt; ++t) {
      const uint4 v = __ldg(src + (size_t)t * vstride);
      *reinterpret_cast<uint2*>(dst8 + (size_t)t * HD) = PoolTraits<T>::to_e4m3(v, inv);
    }
  }
}

// ------------------------------------------------------------------ top-k per row

constexpr int kTopkWarps = 8;
constexpr int kTopkBatch = 3;    // float4 loads of a score row in flight per lane

// Bound on |s~ - s| between the tensor-core score s~ and the exact score s of a pair:
//   kBoundRel |qbar_i| |kbar_j| + kBoundAbs (|qbar_i| + |kbar_j|) + kBoundFloor
// (split tf32 operands, fp32 accumulation, flushed subnormals; derived where the scores
// are made).
constexpr float kBoundRel = 0x1p-14f;
constexpr float kBoundAbs = 0x1p-122f;
constexpr float kBoundFloor = 0x1p-116f;

// Candidate blocks (or keys) a warp keeps apart: room for k and a margin, 64 to 256.
__host__ __device__ inline int topk_cand(int k) {
  const int c = (k + 32 + 31) / 32 * 32;
  return c < 64 ? 64 : (c > 256 ? 256 : c);
}

__host__ __device__ inline size_t topk_smem(int nbp, int d, int cand) {
  return sizeof(uint32_t) * ((size_t)kTopkWarps * (nbp + 256 + 2 * cand + d));
}

// Order-preserving map float -> uint32 (both zeros map to the key of +0) and its inverse.
__device__ __forceinline__ uint32_t float_key(float f) {
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Bitonic sort (ascending) of 64 keys across the warp, two per lane: element i sits in lane
// i mod 32, register i / 32 (v0 for i < 32).
__device__ __forceinline__ void warp_sort64(uint32_t& v0, uint32_t& v1, int lane) {
#pragma unroll
  for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j == 32) {   // partners in the same lane; the final merge is ascending
        const uint32_t a = min(v0, v1), b = max(v0, v1);
        v0 = a;
        v1 = b;
      } else {
        const uint32_t p0 = __shfl_xor_sync(0xffffffffu, v0, j), p1 = __shfl_xor_sync(0xffffffffu, v1, j);
        const bool lower = (lane & j) == 0;
        const bool up0 = (lane & k) == 0, up1 = ((lane + 32) & k) == 0;
        v0 = (lower == up0) ? min(v0, p0) : max(v0, p0);
        v1 = (lower == up1) ? min(v1, p1) : max(v1, p1);
      }
    }
  }
}

// Exact scores of key blocks j1 and j2 against the query block's mean (in shared memory):
// each a chain of fused multiply-adds over channels 0..d-1 starting from 0.  The key rows
// are read kExactStep float4 at a time, the next step's loads issued before this step's
// multiply-adds, so that one L2 round trip is exposed per step rather than per load.
constexpr int kExactStep = 2;
__device__ __forceinline__ void exact_scores(const float* qrow, const float* __restrict__ kb, int d, int j1, int j2,
                                             float& s1, float& s2) {
  const float4* k1 = reinterpret_cast<const float4*>(kb + (size_t)j1 * d);
  const float4* k2 = reinterpret_cast<const float4*>(kb + (size_t)j2 * d);
  const float4* q4 = reinterpret_cast<const float4*>(qrow);
  const int n4 = d / 4;
  float a = 0.f, b = 0.f;
  float4 x[kExactStep], y[kExactStep];
#pragma unroll
  for (int u = 0; u < kExactStep; ++u) {
    x[u] = __ldg(k1 + u);
    y[u] = __ldg(k2 + u);
  }
  for (int c4 = 0; c4 < n4; c4 += kExactStep) {
    float4 xn[kExactStep], yn[kExactStep];
    const bool more = c4 + kExactStep < n4;
#pragma unroll
    for (int u = 0; u < kExactStep; ++u) {
      xn[u] = more ? __ldg(k1 + c4 + kExactStep + u) : x[u];
      yn[u] = more ? __ldg(k2 + c4 + kExactStep + u) : y[u];
    }
#pragma unroll
    for (int u = 0; u < kExactStep; ++u) {
      const float4 q = q4[c4 + u];
      a = fmaf(q.x, x[u].x, a);
      b = fmaf(q.x, y[u].x, b);
      a = fmaf(q.y, x[u].y, a);
      b = fmaf(q.y, y[u].y, b);
      a = fmaf(q.z, x[u].z, a);
      b = fmaf(q.z, y[u].z, b);
      a = fmaf(q.w, x[u].w, a);
      b = fmaf(q.w, y[u].w, b);
    }
#pragma unroll
    for (int u = 0; u < kExactStep; ++u) {
      x[u] = xn[u];
      y[u] = yn[u];
    }
  }
  s1 = a;
  s2 = b;
}

// One warp per row (b, h, i).  The tensor-core scores s~ and the bound e_j give for every
// key block an interval [lo_j, hi_j] = [s~_j - e_j, s~_j + e_j] that holds its exact score.
// L = the k-th largest lo (radix select): at least k blocks score >= L, so a block with
// hi_j < L is below k others and is not kept.  The others are the candidates: when there
// are exactly k of them (most rows) they are the kept set; otherwise they get their exact
// fp32 scores and a radix select over those picks the kept set (ties -> lower index) in
// index order.  A row with a non-finite score or bound, or with more than `cand`
// candidates, takes the exact score of every block instead.
__global__ void __launch_bounds__(kTopkWarps * 32, 4) topk_kernel(Dims dm, const float* __restrict__ scores,
                                                               int nbp, const float* __restrict__ qbar,
                                                               const float* __restrict__ kbar,
                                                               const float* __restrict__ knorm,
                                                               int32_t* __restrict__ col_idx,
                                                               int* __restrict__ status) {
  extern __shared__ __align__(16) uint32_t tsm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kTopkWarps + warp;
  const long long nrows = (long long)dm.B * dm.H * dm.nb;
  if (row >= nrows) return;
  const int nb = dm.nb, kk = dm.k, d = dm.d;
  int32_t* out = col_idx + row * kk;
  if (kk >= nb) {   // every block is kept
    for (int j = lane; j < nb; j += 32) out[j] = j;
    return;
  }
  uint32_t* key = tsm + warp * nbp;
  uint32_t* hist = tsm + kTopkWarps * nbp + warp * 256;
  const int cand = topk_cand(kk);
  uint32_t* ckey = tsm + kTopkWarps * (nbp + 256) + warp * cand;
  int* cidx = reinterpret_cast<int*>(tsm + kTopkWarps * (nbp + 256 + cand) + warp * cand);
  float* qrow = reinterpret_cast<float*>(tsm + kTopkWarps * (nbp + 256 + 2 * cand) + warp * d);
  const size_t bh = (size_t)(row / nb);
  const float* kb = kbar + bh * nb * d;
  const float* kn = knorm + bh * nbp;
  const unsigned full = 0xffffffffu;
  const unsigned lt_mask = (1u << lane) - 1u;

  // the query block's mean (to shared memory) and its norm
  float ss = 0.f;
  for (int c = 4 * lane; c < d; c += 128) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(qbar + (size_t)row * d + c));
    *reinterpret_cast<float4*>(qrow + c) = v;
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(full, ss, off);
  const float qn = sqrtf(ss);
  const float cq = fmaf(kBoundRel, qn, kBoundAbs);   // e_j = cq |kbar_j| + c0
  const float c0 = fmaf(kBoundAbs, qn, kBoundFloor);

  // One 8-bit radix step over keys[0, n) that match (prefix, pmask): picks the digit at
  // `shift` of the need-th largest and updates prefix, pmask and need (the count still to
  // take among keys equal to the prefix so far).  Lanes with equal digits are merged first
  // (__match_any_sync), so a bin shared by most keys costs one atomic per step.
  auto radix_step = [&](const uint32_t* keys, int n, int shift, uint32_t& prefix, uint32_t& pmask,
                        int& need) {
    for (int bb = lane; bb < 256; bb += 32) hist[bb] = 0;
    __syncwarp();
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t u = j < n ? keys[j] : 0u;
      const uint32_t digit = (j < n && (u & pmask) == prefix) ? ((u >> shift) & 255u) : 256u;
      const unsigned peers = __match_any_sync(full, digit);
      if (digit != 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
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
    const int srcl = hit ? (__ffs(hit) - 1) : 0;
    int digit = 0, above = 0;
    if (lane == srcl) {
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
    digit = __shfl_sync(full, digit, srcl);
    above = __shfl_sync(full, above, srcl);
    need -= above;
    prefix |= (uint32_t)digit << shift;
    pmask |= 255u << shift;
    __syncwarp();
  };
  // The kk-th largest of keys[0, n) (prefix) and how many keys equal to it are kept (need):
  // every key through the first digit; the keys still matching it are gathered into ckey
  // (when they fit) for the other three.
  auto select_kth = [&](const uint32_t* keys, int n, uint32_t& prefix, int& need) {
    uint32_t pmask = 0;
    prefix = 0;
    need = kk;
    radix_step(keys, n, 24, prefix, pmask, need);
    int nc = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t u = j < n ? keys[j] : 0u;
      const bool take = j < n && (u & pmask) == prefix;
      const unsigned bin = __ballot_sync(full, take);
      const int pos = nc + __popc(bin & lt_mask);
      if (take && pos < cand) ckey[pos] = u;
      nc += __popc(bin);
    }
    __syncwarp();
    const uint32_t* src = nc <= cand ? ckey : keys;
    const int ns = nc <= cand ? nc : n;
    for (int pass = 1; pass < 4; ++pass) radix_step(src, ns, 24 - 8 * pass, prefix, pmask, need);
  };

  // The kk-th largest (kk <= 64) of 64 keys held two per lane (0 = absent: no finite score
  // maps to key 0).
  auto kth_of64 = [&](uint32_t v0, uint32_t v1) -> uint32_t {
    warp_sort64(v0, v1, lane);
    const int e = 64 - kk;
    return __shfl_sync(full, (e >> 5) ? v1 : v0, e & 31);
  };

  // Lower bounds lo_j as keys in shared memory; each lane keeps the two largest and the
  // smallest of its keys and the largest e_j.  lo_j = s~_j - e_j with e_j > 0 is never -0, so
  // its key needs no zero fix-up; a NaN lo has a key above +inf's or below -inf's.  The row
  // is read as float4 (rows are nbp floats, nbp a multiple of 4), kTopkBatch per lane in
  // flight.
  const float4* src4 = reinterpret_cast<const float4*>(scores + row * nbp);
  const float4* kn4 = reinterpret_cast<const float4*>(kn);
  const int n4 = (nb + 3) >> 2;
  uint32_t top1 = 0, top2 = 0, kmin = 0xffffffffu;
  float emax = 0.f;
  auto lo_key = [](float lo) {
    const uint32_t u = __float_as_uint(lo);
    return u ^ ((uint32_t)((int32_t)u >> 31) | 0x80000000u);
  };
  for (int t0 = 0; t0 < n4; t0 += 32 * kTopkBatch) {
    float4 sv[kTopkBatch], kv[kTopkBatch];
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) {
      const int t = t0 + 32 * u + lane;
      if (t < n4) {
        sv[u] = __ldcs(src4 + t);
        kv[u] = __ldg(kn4 + t);
      }
    }
#pragma unroll
    for (int u = 0; u < kTopkBatch; ++u) {
      const int t = t0 + 32 * u + lane;
      if (t < n4) {
        const float s4[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
        const float k4[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
        const int nin = min(4, nb - 4 * t);   // blocks of this float4 below nb
        uint32_t l4[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (c < nin) {
            const float e = fmaf(cq, k4[c], c0);
            l4[c] = lo_key(s4[c] - e);
            emax = fmaxf(emax, e);
            kmin = min(kmin, l4[c]);
            top2 = max(top2, min(top1, l4[c]));
            top1 = max(top1, l4[c]);
          } else {
            l4[c] = 0u;
          }
        }
        *reinterpret_cast<uint4*>(key + 4 * t) = make_uint4(l4[0], l4[1], l4[2], l4[3]);
      }
    }
  }
  __syncwarp();
  uint32_t kmax = top1;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    emax = fmaxf(emax, __shfl_xor_sync(full, emax, off));
    kmin = min(kmin, __shfl_xor_sync(full, kmin, off));
    kmax = max(kmax, __shfl_xor_sync(full, kmax, off));
  }
  // every lo_j is finite when the keys lie strictly between those of -inf and +inf (a NaN e
  // or s~ makes lo NaN), and every hi_j <= max lo + 2 max e is finite when that sum is
  const bool finite = kmin > 0x007fffffu && kmax < 0xff800000u && isfinite(key_float(kmax) + 2.f * emax);
  uint32_t prefix = 0;
  int need = kk;
  if (finite) {
    // L = the kk-th largest lo; candidates C = {lo_j >= L - 2 emax}: only they can have
    // hi_j >= L, every other block scores below the kk blocks whose lo >= L.
    // T0 = the kk-th largest of the 64 lane top-twos is at most L (kk keys reach it), so
    // G = {lo_j >= T0 - 2 emax} (usually little more than kk blocks) holds both the top kk
    // lo and C: L is selected within G and C filtered out of it, in index order.
    bool have_c = false;
    int nc = 0;
    if (kk <= 64) {
      const uint32_t T0 = kth_of64(top1, top2);   // 0 when fewer than kk blocks: take all
      const uint32_t t0 = T0 ? lo_key(key_float(T0) - 2.f * emax) : 0u;
      int ng = 0;
#pragma unroll 4
      for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        const uint32_t u = j < nb ? key[j] : 0u;
        const bool take = j < nb && u >= t0;
        const unsigned bin = __ballot_sync(full, take);
        const int pos = ng + __popc(bin & lt_mask);
        if (take && pos < cand) {
          ckey[pos] = u;
          cidx[pos] = j;
        }
        ng += __popc(bin);
      }
      __syncwarp();
      if (ng <= cand) {
        if (ng <= 64) {
          prefix = kth_of64(lane < ng ? ckey[lane] : 0u, lane + 32 < ng ? ckey[lane + 32] : 0u);
        } else {
          uint32_t pmask = 0;
          for (int pass = 0; pass < 4; ++pass) radix_step(ckey, ng, 24 - 8 * pass, prefix, pmask, need);
        }
        const uint32_t TL = lo_key(key_float(prefix) - 2.f * emax);
        for (int e0 = 0; e0 < ng; e0 += 32) {   // compaction in place: entries are read first
          const int e = e0 + lane;
          const bool take = e < ng && ckey[e] >= TL;
          const int j = take ? cidx[e] : 0;
          const unsigned bin = __ballot_sync(full, take);
          const int pos = nc + __popc(bin & lt_mask);
          __syncwarp();
          if (take) cidx[pos] = j;
          nc += __popc(bin);
        }
        __syncwarp();
        have_c = true;
      }
    }
    if (!have_c) {
      select_kth(key, nb, prefix, need);
      const uint32_t TL = lo_key(key_float(prefix) - 2.f * emax);
#pragma unroll 4
      for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        const bool take = j < nb && key[j] >= TL;
        const unsigned bin = __ballot_sync(full, take);
        const int pos = nc + __popc(bin & lt_mask);
        if (take && pos < cand) cidx[pos] = j;
        nc += __popc(bin);
      }
      __syncwarp();
    }
    if (nc == kk) {
      // no block outside the kk can reach them: the boundary is settled without exact scores
      for (int e = lane; e < kk; e += 32) out[e] = cidx[e];
      return;
    }
    if (nc <= cand) {
      for (int e0 = 0; e0 < nc; e0 += 64) {
        const int a = e0 + lane, b = e0 + 32 + lane;
        const int ja = a < nc ? cidx[a] : cidx[0];
        const int jb = b < nc ? cidx[b] : ja;
        float sa, sb;
        exact_scores(qrow, kb, d, ja, jb, sa, sb);
        if (a < nc) ckey[a] = float_key(sa);
        if (b < nc) ckey[b] = float_key(sb);
      }
      __syncwarp();
      if (kk <= 64 && nc <= 64) {
        // the kk-th largest exact key, and how many equal to it are kept
        prefix = kth_of64(lane < nc ? ckey[lane] : 0u, lane + 32 < nc ? ckey[lane + 32] : 0u);
        const int above = __popc(__ballot_sync(full, lane < nc && ckey[lane] > prefix)) +
                          __popc(__ballot_sync(full, lane + 32 < nc && ckey[lane + 32] > prefix));
        need = kk - above;
      } else {
        uint32_t pmask = 0;
        prefix = 0;
        need = kk;
        for (int pass = 0; pass < 4; ++pass) radix_step(ckey, nc, 24 - 8 * pass, prefix, pmask, need);
      }
      // the kept candidates in index order: above the k-th largest, or equal to it and
      // among the first `need` such
      int written = 0, eqseen = 0;
      for (int e0 = 0; e0 < nc; e0 += 32) {
        const int e = e0 + lane;
        const uint32_t u = e < nc ? ckey[e] : 0u;
        const bool gt = e < nc && u > prefix;
        const bool eq = e < nc && u == prefix;
        const unsigned beq = __ballot_sync(full, eq);
        const bool keep = gt || (eq && eqseen + __popc(beq & lt_mask) < need);
        const unsigned bk = __ballot_sync(full, keep);
        const int pos = written + __popc(bk & lt_mask);
        if (keep && pos < kk) out[pos] = cidx[e];
        written += __popc(bk);
        eqseen += __popc(beq);
      }
      if (lane == 0 && written != kk) record_status(status, kDevBounds);
      return;
    }
  }

  // every block's exact score, then the same select over the whole row
  for (int j0 = 0; j0 < nb; j0 += 64) {
    const int a = j0 + lane, b = j0 + 32 + lane;
    const int ja = a < nb ? a : 0;
    const int jb = b < nb ? b : ja;
    float sa, sb;
    exact_scores(qrow, kb, d, ja, jb, sa, sb);
    if (a < nb) key[a] = float_key(sa);
    if (b < nb) key[b] = float_key(sb);
  }
  __syncwarp();
  select_kth(key, nb, prefix, need);
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
    if (keep && pos < kk) out[pos] = j;
    written += __popc(bk);
    eqseen += __popc(beq);
  }
  if (lane == 0 && written != kk) record_status(status, kDevBounds);
}

}  // namespace

cudaError_t launch_pool(const Dims& dm, rola_dtype dt, const void* q, const void* k,
                        const Workspace& ws, cudaStream_t st) {
  const int HD = dm.H * dm.d;
  if (dt == ROLA_F32) {
    dim3 grid((HD / 4 + 127) / 128, dm.nb, 2 * dm.B);
    pool_kernel<float, false><<<grid, 128, 0, st>>>(static_cast<const float*>(q),
                                                    static_cast<const float*>(k), dm, ws.qbar,
                                                    ws.kbar, nullptr, nullptr, nullptr, nullptr);
  } else if (dt == ROLA_FP8_E4M3) {
    dim3 grid((HD / 8 + 127) / 128, dm.nb, 2 * dm.B);
    pool_kernel<__nv_bfloat16, true><<<grid, 128, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), dm, ws.qbar,
        ws.kbar, ws.q8, ws.k8, ws.sq, ws.sk);
  } else {
    dim3 grid((HD / 8 + 127) / 128, dm.nb, 2 * dm.B);
    pool_kernel<__nv_bfloat16, false><<<grid, 128, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), dm, ws.qbar,
        ws.kbar, nullptr, nullptr, nullptr, nullptr);
  }
  return cudaGetLastError();
}

int score_row_stride(const Dims& dm) { return (dm.nb + 3) / 4 * 4; }

cudaError_t launch_select(const Dims& dm, const Workspace& ws, cudaStream_t st) {
  const int nbp = score_row_stride(dm);
  cudaError_t e = launch_score_sm100(dm, ws, nbp, st);
  if (e != cudaSuccess) return e;
  const size_t smem = topk_smem(nbp, dm.d, topk_cand(dm.k));
  e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)dm.B * dm.H * dm.nb;
  topk_kernel<<<(unsigned)((rows + kTopkWarps - 1) / kTopkWarps), kTopkWarps * 32, smem, st>>>(
      dm, ws.scores, nbp, ws.qbar, ws.kbar, ws.knorm, ws.col_idx, ws.status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ allocation-free variant
//
// Block selection for callers that cannot allocate device memory and have no workspace
// to lend.  Its scratch (status word, pooled means, block scores and key norms) lives in
// one file-scope device array of kSelectScratchBytes; every GPU that loads this library holds that array
// until the process exits.  In host code `g_select_scratch` only names a host-side
// stand-in, so its device address is looked up with cudaGetSymbolAddress, once per device
// (on the first call made with that device current), and passed to the kernels.

namespace {

constexpr size_t kSelectScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_select_scratch[kSelectScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

size_t select_noalloc_bytes(const Dims& dm) {
  const size_t BH = (size_t)dm.B * dm.H;
  return 256 + 2 * align256(sizeof(float) * BH * dm.nb * dm.d) +
         align256(sizeof(float) * BH * dm.nb * score_row_stride(dm)) + align256(sizeof(float) * BH * score_row_stride(dm));
}

size_t select_noalloc_capacity() { return kSelectScratchBytes; }

cudaError_t select_blocks_noalloc(const Dims& dm, rola_dtype dt, const void* q, const void* k,
                                  int32_t* col_idx, cudaStream_t st) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  // The array's device address is looked up with this device current: on the first call
  // on a device, and again on every call made outside stream capture (so that a device
  // reset, which reloads the module, cannot leave a stale address behind).  A call made
  // while `st` is being captured uses the address of the last uncaptured call.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  e = cudaStreamIsCapturing(st, &cap);
  if (e != cudaSuccess) return e;
  char* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr || cap == cudaStreamCaptureStatusNone) {
      if (cap != cudaStreamCaptureStatusNone) return cudaErrorStreamCaptureUnsupported;
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_select_scratch);
      if (e != cudaSuccess) return e;
      g_scratch_addr[dev] = ptr;
    }
    base = static_cast<char*>(g_scratch_addr[dev]);
  }
  const size_t BH = (size_t)dm.B * dm.H;
  Workspace w{};
  w.status = reinterpret_cast<int*>(base);
  w.qbar = reinterpret_cast<float*>(base + 256);
  w.kbar = reinterpret_cast<float*>(base + 256 + align256(sizeof(float) * BH * dm.nb * dm.d));
  w.scores = reinterpret_cast<float*>(base + 256 + 2 * align256(sizeof(float) * BH * dm.nb * dm.d));
  w.knorm = reinterpret_cast<float*>(reinterpret_cast<char*>(w.scores) +
                                     align256(sizeof(float) * BH * dm.nb * score_row_stride(dm)));
  w.col_idx = col_idx;
  // The array keeps the previous call's contents: the status word must start at zero.
  e = cudaMemsetAsync(w.status, 0, 256, st);
  if (e != cudaSuccess) return e;
  // The selection does not depend on the fp8 copies; pool as for bf16 inputs.
  e = launch_pool(dm, dt == ROLA_FP8_E4M3 ? ROLA_BF16 : dt, q, k, w, st);
  if (e != cudaSuccess) return e;
  return launch_select(dm, w, st);
}

}  // namespace rola
