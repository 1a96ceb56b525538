// Block pooling (step 1) and block scores + top-k selection (step 2) of RoLA.
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

// ------------------------------------------------------------------ block scores

constexpr int kTS = 128;  // score tile: 128 query blocks x 128 key blocks
constexpr int kKC = 16;   // channels staged per step

// grid: x = key-block tile, y = query-block tile, z = b*H + h; 256 threads, 8x8 scores each.
// s_ij accumulates q_i[c] * k_j[c] with fmaf in channel order 0..d-1 (the stated order).
// The next 16-channel chunk is loaded into registers (float4 per row and channel quad)
// while the current one is multiplied, then stored transposed into the other buffer.
constexpr size_t kScoreSmem = sizeof(float) * 2 * 2 * kKC * (kTS + 4);

__global__ void __launch_bounds__(256, 2) score_kernel(Dims dm, const float* __restrict__ qbar,
                                                       const float* __restrict__ kbar,
                                                       float* __restrict__ scores, int nbp) {
  extern __shared__ __align__(16) float ssm[];
  float (*As)[kKC][kTS + 4] = reinterpret_cast<float (*)[kKC][kTS + 4]>(ssm);
  float (*Bs)[kKC][kTS + 4] = reinterpret_cast<float (*)[kKC][kTS + 4]>(ssm + 2 * kKC * (kTS + 4));
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int i0 = blockIdx.y * kTS, j0 = blockIdx.x * kTS, bh = blockIdx.z;
  const int nb = dm.nb, d = dm.d;
  const float* qb = qbar + (size_t)bh * nb * d;
  const float* kb = kbar + (size_t)bh * nb * d;
  constexpr int kQuads = kKC / 4, kPer = kTS * kQuads / 256;   // float4 loads per thread
  float4 ra[kPer], rb[kPer];
  auto load = [&](int c0) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + 256 * u, r = e / kQuads, cq = e % kQuads;
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      ra[u] = (i0 + r < nb) ? *reinterpret_cast<const float4*>(qb + (size_t)(i0 + r) * d + c0 + 4 * cq) : z;
      rb[u] = (j0 + r < nb) ? *reinterpret_cast<const float4*>(kb + (size_t)(j0 + r) * d + c0 + 4 * cq) : z;
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = tid + 256 * u, r = e / kQuads, c = 4 * (e % kQuads);
      As[buf][c][r] = ra[u].x; As[buf][c + 1][r] = ra[u].y; As[buf][c + 2][r] = ra[u].z; As[buf][c + 3][r] = ra[u].w;
      Bs[buf][c][r] = rb[u].x; Bs[buf][c + 1][r] = rb[u].y; Bs[buf][c + 2][r] = rb[u].z; Bs[buf][c + 3][r] = rb[u].w;
    }
  };
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
  const int nch = d / kKC;
  load(0);
  store(0);
  __syncthreads();
  for (int ch = 0; ch < nch; ++ch) {
    const int buf = ch & 1;
    if (ch + 1 < nch) load((ch + 1) * kKC);
#pragma unroll 1
    for (int c = 0; c < kKC; ++c) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][c][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][c][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][c][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][c][tx * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
      // two scores per packed f32x2 FMA (each rounded as fmaf: the chains stay exact)
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int e = 0; e < 8; e += 2)
          sm100::fma2(acc[a][e], acc[a][e + 1], av[a], av[a], bv[e], bv[e + 1], acc[a][e], acc[a][e + 1]);
    }
    if (ch + 1 < nch) store(buf ^ 1);   // the other buffer was last read before the barrier below
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int i = i0 + ty * 8 + a;
    if (i >= nb) continue;
    float* row = scores + ((size_t)bh * nb + i) * nbp + j0 + tx * 8;
    if (j0 + tx * 8 + 8 <= nbp) {
      *reinterpret_cast<float4*>(row) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
      *reinterpret_cast<float4*>(row + 4) = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (j0 + tx * 8 + e < nbp) row[e] = acc[a][e];
    }
  }
}

// ------------------------------------------------------------------ top-k per row

constexpr int kTopkWarps = 8;
constexpr int kTopkCand = 256;   // keys left after the first digit, kept apart (if they fit)

__host__ __device__ inline size_t topk_smem(int nbp) {
  return sizeof(uint32_t) * ((size_t)kTopkWarps * (nbp + 256 + kTopkCand));
}

// One warp per row (b, h, i): 4-pass 8-bit radix select of the k-th largest score, then
// one pass in index order emits the kept block indices (ties -> lower index).  For
// k <= 64 the select runs over few keys: the k-th largest of the 64 lane top-twos is a
// lower bound of the answer, and only the keys at or above it (when at most kTopkCand)
// are gathered and selected from.  Otherwise the first pass reads every key and the keys
// still matching its digit are gathered for the other three.
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(Dims dm, const float* __restrict__ scores,
                                                               int nbp, int32_t* __restrict__ col_idx,
                                                               int* __restrict__ status) {
  extern __shared__ uint32_t tsm[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * kTopkWarps + warp;
  const long long nrows = (long long)dm.B * dm.H * dm.nb;
  if (row >= nrows) return;
  const int nb = dm.nb, kk = dm.k;
  uint32_t* key = tsm + warp * nbp;
  uint32_t* hist = tsm + kTopkWarps * nbp + warp * 256;
  uint32_t* cand = tsm + kTopkWarps * (nbp + 256) + warp * kTopkCand;
  const float* src = scores + row * nbp;
  const unsigned full = 0xffffffffu;
  const unsigned lt_mask = (1u << lane) - 1u;
  // Order-preserving map float -> uint32 (both zeros map to the key of +0); each lane
  // also keeps the two largest of its keys.
  uint32_t top1 = 0, top2 = 0;
  for (int j = lane; j < nb; j += 32) {
    float f = src[j];
    if (f == 0.f) f = 0.f;
    const uint32_t u = __float_as_uint(f);
    const uint32_t kj = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    key[j] = kj;
    top2 = max(top2, min(top1, kj));
    top1 = max(top1, kj);
  }
  __syncwarp();

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
  // Gathers the keys that satisfy `in` into cand (in any order; counts are all the radix
  // steps take from them).  Returns their number (those past kTopkCand are not stored).
  auto gather = [&](auto in) {
    int nc = 0;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t u = j < nb ? key[j] : 0u;
      const bool take = j < nb && in(u);
      const unsigned bin = __ballot_sync(full, take);
      const int pos = nc + __popc(bin & lt_mask);
      if (take && pos < kTopkCand) cand[pos] = u;
      nc += __popc(bin);
    }
    __syncwarp();
    return nc;
  };

  uint32_t prefix = 0, pmask = 0;
  int need = kk;
  bool done = false;
  if (kk <= 64 && nb >= 64) {
    // Bound from below: T = the kk-th largest of the 64 lane top-twos is a key with at least
    // kk keys at or above it, so the kk-th largest key is >= T; the keys >= T (usually little
    // more than kk) are gathered and the exact select runs over them alone.
    cand[lane] = top1;
    cand[32 + lane] = top2;
    __syncwarp();
    uint32_t tp = 0, tm = 0;
    int tn = kk;
    for (int pass = 0; pass < 4; ++pass) radix_step(cand, 64, 24 - 8 * pass, tp, tm, tn);
    const int nc = gather([&](uint32_t u) { return u >= tp; });
    if (nc <= kTopkCand) {
      for (int pass = 0; pass < 4; ++pass) radix_step(cand, nc, 24 - 8 * pass, prefix, pmask, need);
      done = true;
    }
  }
  if (!done) {
    // every key through the first digit; then the keys still matching it are gathered
    // (when they fit) for the other three
    radix_step(key, nb, 24, prefix, pmask, need);
    const int nc = gather([&](uint32_t u) { return (u & pmask) == prefix; });
    const uint32_t* src_keys = nc <= kTopkCand ? cand : key;
    const int nsrc = nc <= kTopkCand ? nc : nb;
    for (int pass = 1; pass < 4; ++pass) radix_step(src_keys, nsrc, 24 - 8 * pass, prefix, pmask, need);
  }
  // prefix is the k-th largest key; `need` elements equal to it are kept.
  int32_t* out = col_idx + row * kk;
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

size_t select_smem_bytes(const Dims& dm) { return topk_smem(score_row_stride(dm)); }

cudaError_t launch_select(const Dims& dm, const Workspace& ws, cudaStream_t st) {
  const int nbp = score_row_stride(dm);
  dim3 g1((dm.nb + kTS - 1) / kTS, (dm.nb + kTS - 1) / kTS, dm.B * dm.H);
  cudaError_t e = cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScoreSmem);
  if (e != cudaSuccess) return e;
  score_kernel<<<g1, 256, kScoreSmem, st>>>(dm, ws.qbar, ws.kbar, ws.scores, nbp);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = topk_smem(nbp);
  e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)dm.B * dm.H * dm.nb;
  topk_kernel<<<(unsigned)((rows + kTopkWarps - 1) / kTopkWarps), kTopkWarps * 32, smem, st>>>(
      dm, ws.scores, nbp, ws.col_idx, ws.status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ allocation-free variant
//
// Block selection for callers that cannot allocate device memory and have no workspace
// to lend.  Its scratch (status word, pooled means, block scores) lives in one file-scope
// device array of kSelectScratchBytes; every GPU that loads this library holds that array
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
         align256(sizeof(float) * BH * dm.nb * score_row_stride(dm));
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
