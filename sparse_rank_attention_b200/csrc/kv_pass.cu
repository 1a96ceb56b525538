// Key/value pass of the RoLA forward for head dim 128 with bf16 inputs: one read of k
// and v computes everything the later steps need from them.
//   * the linear-branch state partials over a chunk of tokens (split-N; step 4, key side)
//       S_h += sum_m R(p_m) phi(k_m Wk_h) v_m^T,   z_h += sum_m phi(k_m Wk_h)
//   * the block means of k (step 1, key side): fp32 sums in token order, one division
//   * bf16 configuration: the fp16 copy of v that the attention kernel multiplies the
//     fp16 softmax weights with (values outside the fp16 range set ROLA_ERR_RANGE)
//   * fp8 configuration: the e4m3 copies of k and v with one scale per (b, h, block)
//     (scale = absmax / 448, 1 for an all-zero block; code = RN-sat(x * (1 / scale))).
//
// Sources: "SparkDiffusion: 265x Faster Video Generation ..." page, section "RoLA:
// Preserving Global Context at Extreme Sparsity" (high-energy block selection; low-rank
// linear branch with rotary positions); README sparse-finetuning section (proj_k).
//
// Layout of the work: a CTA owns one (b, h) and a chunk of whole 64-token blocks; the
// chunk length is chosen on the host so that the CTAs fill the SMs in whole waves.  k and
// v tiles (one block each: two TMA boxes of 64 tokens x 64 channels, 128-byte swizzle)
// flow through a 2-stage ring of TMA copies completing on mbarriers, so the next tile is in
// flight while one is processed, with two CTAs per SM (two tiles in flight per SM); rows
// past N arrive as zeros.
// Per tile: warps 0-3 compute F = K Wk (mma.sync), phi, z and the rotation and store
// the rotated features as bf16 hi + lo; meanwhile warps 4-5 pool k (and write its e4m3
// copy) and warps 6-7 write the copy of v; then all 8 warps add F^T V into their 16
// columns of S.
#include "rola_internal.cuh"
#include "sm100_ptx.cuh"
#include "warp_mma.cuh"

#include <cuda_fp8.h>

namespace rola {
namespace {

constexpr int kD = 128;
constexpr int kTok = 64;                     // tokens per tile = one block
constexpr int kStages = 2;
constexpr int kThreads = 256;
constexpr uint32_t kTileBytes = kTok * kD * 2;   // 16 KB, 64 rows of 256 bytes

// Byte offset of 16-byte chunk c (channels 8c .. 8c + 7, c = 0..15) of token row r in a
// tile: box c / 8 (8 KB each), 128-byte rows, chunk position (c % 8) ^ (r % 8).
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((c >> 3) * 8192 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int RK>
struct KVSmem {
  static constexpr int WP = RK + 8;          // Wk rows [d][r], padded (conflict-free ldmatrix)
  static constexpr int RP = RK + 8;          // F rows [token][r], padded
  static constexpr size_t offK = 0;
  static constexpr size_t offV = offK + (size_t)kStages * kTileBytes;
  static constexpr size_t offW = offV + (size_t)kStages * kTileBytes;
  static constexpr size_t offF = offW + (size_t)kD * WP * 2;
  static constexpr size_t offFl = offF + (size_t)kTok * RP * 2;
  static constexpr size_t offZ = offFl + (size_t)kTok * RP * 2;   // [4][RK] fp32
  static constexpr size_t offRed = offZ + (size_t)4 * RK * 4;      // [2][4] fp32
  static constexpr size_t offBar = offRed + 2 * 4 * 4;              // full[kStages], abort flag
  static constexpr size_t bytes = offBar + kStages * 8 + 16 + 1024;   // + alignment slack
};

__device__ __forceinline__ float absmax8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[e] << 16)), fabsf(__uint_as_float(w[e] & 0xffff0000u))));
  return m;
}

// 8 bf16 values times inv, rounded to e4m3 (nearest even, saturating), in element order.
__device__ __forceinline__ uint2 e4m3x8(const uint4& v, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[2] = {0, 0};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = make_float2(__uint_as_float(w[e] << 16) * inv, __uint_as_float(w[e] & 0xffff0000u) * inv);
    o[e >> 1] |= (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3) << (16 * (e & 1));
  }
  return make_uint2(o[0], o[1]);
}

template <int RK, bool FP8>
__global__ void __launch_bounds__(kThreads, 2) kv_pass_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const __nv_bfloat16* __restrict__ Wk, Dims dm, const float2* __restrict__ rope,
    float* __restrict__ S_part, float* __restrict__ z_part, float* __restrict__ kbar,
    __half* __restrict__ v16, uint8_t* __restrict__ k8, uint8_t* __restrict__ v8,
    float* __restrict__ sk, float* __restrict__ sv, int* __restrict__ status) {
  using L = KVSmem<RK>;
  using namespace sm100;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::offBar);
  int* abort_flag = reinterpret_cast<int*>(smem + L::offBar + kStages * 8);
  const __nv_bfloat16* sW = reinterpret_cast<const __nv_bfloat16*>(smem + L::offW);
  __nv_bfloat16* sF = reinterpret_cast<__nv_bfloat16*>(smem + L::offF);
  __nv_bfloat16* sFl = reinterpret_cast<__nv_bfloat16*>(smem + L::offFl);
  float* sZ = reinterpret_cast<float*>(smem + L::offZ);
  float* sRed = reinterpret_cast<float*>(smem + L::offRed);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g8 = lane >> 2, t4 = lane & 3;
  const int chunk = blockIdx.x, bh = blockIdx.y;
  const int b = bh / dm.H, h = bh % dm.H;
  const int n_begin = chunk * dm.chunk_tok;
  const int n_end = min(dm.N, n_begin + dm.chunk_tok);
  const int ntiles = n_end > n_begin ? (n_end - n_begin + kTok - 1) / kTok : 0;
  const size_t rs = (size_t)dm.H * kD;           // elements between tokens
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&full[s]), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const WaitCtl wc{abort_flag, status, 2000000000ull};

  // Wk_h [d][r] (contiguous in global) -> padded rows; part of the first copy group
  for (int e = tid; e < kD * RK / 8; e += kThreads) {
    const int c = e / (RK / 8), a8 = e % (RK / 8);
    cp_async16(sbase + (uint32_t)(L::offW + (c * L::WP + a8 * 8) * 2), Wk + ((size_t)h * kD + c) * RK + a8 * 8, 16);
  }
  cp_async_commit();
  // one thread issues the tile copies: 4 boxes (k, v x two channel halves) per tile
  auto load_tile = [&](int t) {
    const int s = t % kStages, n0 = n_begin + t * kTok;
    const uint32_t bar = smem_u32(&full[s]);
    mbar_expect_tx(bar, 2 * kTileBytes);
    for (int c = 0; c < 2; ++c) {
      tma_load_3d(sbase + (uint32_t)(L::offK + s * kTileBytes) + c * 8192, &tm_k, h * kD + 64 * c, n0, b, bar);
      tma_load_3d(sbase + (uint32_t)(L::offV + s * kTileBytes) + c * 8192, &tm_v, h * kD + 64 * c, n0, b, bar);
    }
  };
  if (tid == 0) {
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    for (int t = 0; t < kStages - 1 && t < ntiles; ++t) load_tile(t);
  }
  cp_async_wait<0>();               // Wk (visible after the loop's first barrier)
  int issued = ntiles < kStages - 1 ? ntiles : kStages - 1;

  constexpr int NT_F = RK / 8;     // n-tiles of F (warps 0-3)
  constexpr int MT_S = RK / 16;    // m-tiles of S
  float sacc[MT_S][2][4];
#pragma unroll
  for (int a = 0; a < MT_S; ++a)
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[a][c][e] = 0.f;
  float zacc[NT_F][2];
#pragma unroll
  for (int a = 0; a < NT_F; ++a) zacc[a][0] = zacc[a][1] = 0.f;

  int consumed = 0;
  for (int t = 0; t < ntiles; ++t) {
    const int s = t % kStages, n0 = n_begin + t * kTok;
    const bool ok = mbar_wait(smem_u32(&full[s]), (t / kStages) & 1, wc);
    // tile t landed; every warp is done with tile t - 1 (its stage may be refilled)
    if (__syncthreads_or(!ok)) break;
    consumed = t + 1;
    if (tid == 0 && issued < ntiles) {
      fence_proxy_async_smem();
      load_tile(issued++);
    }
    const int cnt = min(kTok, n_end - n0);
    const uint32_t tK = sbase + (uint32_t)(L::offK + s * kTileBytes);
    const uint32_t tV = sbase + (uint32_t)(L::offV + s * kTileBytes);
    const uint8_t* pK = smem + L::offK + s * kTileBytes;
    const uint8_t* pV = smem + L::offV + s * kTileBytes;

    if (warp < 4) {
      // ---- F = K Wk for tokens 16*warp .. +15, all r; phi, z, rotation -> sF (hi, lo)
      float f[NT_F][4];
#pragma unroll
      for (int a = 0; a < NT_F; ++a)
#pragma unroll
        for (int e = 0; e < 4; ++e) f[a][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        uint32_t af[4];
        ldsm_x4(tK + swz(16 * warp + (lane & 15), 2 * kk + (lane >> 4)), af[0], af[1], af[2], af[3]);
#pragma unroll
        for (int nt = 0; nt < NT_F; nt += 2) {
          uint32_t bf[4];
          const int row = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
          ldsm_x4_t(smem_u32(sW + row * L::WP + nt * 8 + (lane >> 4) * 8), bf[0], bf[1], bf[2], bf[3]);
          mma_bf16(f[nt], af, bf);
          mma_bf16(f[nt + 1], af, bf + 2);
        }
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int row = 16 * warp + g8 + 8 * half;
        const int n = n0 + row;
        const bool valid = n < n_end;
        const TokPos pos = token_pos(dm, valid ? n : 0);
#pragma unroll
        for (int nt = 0; nt < NT_F; ++nt) {
          const float x0 = valid ? phi_fast(f[nt][2 * half]) : 0.f;
          const float x1 = valid ? phi_fast(f[nt][2 * half + 1]) : 0.f;
          zacc[nt][0] += x0;
          zacc[nt][1] += x1;
          const float2 cs = valid ? rope_at(dm, rope, pos, nt * 4 + t4) : make_float2(1.f, 0.f);
          const float y0 = cs.x * x0 - cs.y * x1;
          const float y1 = cs.y * x0 + cs.x * x1;
          uint32_t hi, lo;
          split_bf16(y0, y1, hi, lo);
          *reinterpret_cast<uint32_t*>(sF + row * L::RP + nt * 8 + 2 * t4) = hi;
          *reinterpret_cast<uint32_t*>(sFl + row * L::RP + nt * 8 + 2 * t4) = lo;
        }
      }
    } else if (warp < 6) {
      // ---- pooling of k: thread = two adjacent channels, tokens added in order
      const int cp = tid - 128;                     // channel pair 0..63
      const int blk = n0 / kTok;
      float a0 = 0.f, a1 = 0.f, am = 0.f;
      const uint8_t* col = pK + (cp >> 5) * 8192 + (cp & 3) * 4;   // box, word in chunk
      const int ch = (cp >> 2) & 7;                                 // chunk within the box
      for (int r = 0; r < cnt; ++r) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(col + r * 128 + ((ch ^ (r & 7)) << 4));
        const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xffff0000u);
        a0 = a0 + x0;
        a1 = a1 + x1;
        if (FP8) am = fmaxf(am, fmaxf(fabsf(x0), fabsf(x1)));
      }
      *reinterpret_cast<float2*>(kbar + ((size_t)bh * dm.nb + blk) * kD + 2 * cp) =
          make_float2(__fdiv_rn(a0, (float)cnt), __fdiv_rn(a1, (float)cnt));
      if constexpr (FP8) {
        // e4m3 copy of the k tile: block scale from the max over the two warps
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        if (lane == 0) sRed[warp - 4] = am;
        asm volatile("bar.sync 1, 64;" ::: "memory");
        am = fmaxf(sRed[0], sRed[1]);
        const float sc = am > 0.f ? am / 448.f : 1.f, inv = 1.f / sc;
        if (cp == 0) sk[(size_t)bh * dm.nb + blk] = sc;
        for (int e = cp; e < cnt * 16; e += 64) {
          const int r = e >> 4, cv = e & 15;
          *reinterpret_cast<uint2*>(k8 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
              e4m3x8(*reinterpret_cast<const uint4*>(pK + swz(r, cv)), inv);
        }
        asm volatile("bar.sync 1, 64;" ::: "memory");   // sRed is rewritten next tile
      }
    } else {
      // ---- copy of v: fp16 (bf16 configuration) or e4m3 with its block scale (fp8)
      const int tv = tid - 192;                     // 0..63
      if constexpr (!FP8) {
        bool bad = false;
        for (int e = tv; e < cnt * 16; e += 64) {
          const int r = e >> 4, cv = e & 15;
          const uint4 raw = *reinterpret_cast<const uint4*>(pV + swz(r, cv));
          const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
          uint32_t o[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            // |x| >= 65536 (bf16 0x4780 and up, inf, nan) does not fit fp16; below that
            // every bf16 value rounds to fp16 within its range
            bad |= ((w[u] & 0x7fffu) >= 0x4780u) || (((w[u] >> 16) & 0x7fffu) >= 0x4780u);
            const __half2 hv = __floats2half2_rn(__uint_as_float(w[u] << 16), __uint_as_float(w[u] & 0xffff0000u));
            o[u] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(v16 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
        if (bad) record_status(status, kDevRange);
      } else {
        float am = 0.f;
        for (int e = tv; e < cnt * 16; e += 64) {
          const int r = e >> 4, cv = e & 15;
          am = fmaxf(am, absmax8(*reinterpret_cast<const uint4*>(pV + swz(r, cv))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        if (lane == 0) sRed[4 + warp - 6] = am;
        asm volatile("bar.sync 2, 64;" ::: "memory");
        am = fmaxf(sRed[4], sRed[5]);
        const float sc = am > 0.f ? am / 448.f : 1.f, inv = 1.f / sc;
        const int blk = n0 / kTok;
        if (tv == 0) sv[(size_t)bh * dm.nb + blk] = sc;
        for (int e = tv; e < cnt * 16; e += 64) {
          const int r = e >> 4, cv = e & 15;
          *reinterpret_cast<uint2*>(v8 + ((size_t)b * dm.N + n0 + r) * rs + (size_t)h * kD + cv * 8) =
              e4m3x8(*reinterpret_cast<const uint4*>(pV + swz(r, cv)), inv);
        }
        asm volatile("bar.sync 2, 64;" ::: "memory");
      }
    }
    __syncthreads();                 // sF complete

    // ---- S += F^T V: warp w owns channels 16w .. 16w + 15
#pragma unroll
    for (int kk = 0; kk < kTok / 16; ++kk) {
      const int q = lane >> 3;
      uint32_t af[MT_S][4], al[MT_S][4];
#pragma unroll
      for (int mt = 0; mt < MT_S; ++mt) {
        const int off = (kk * 16 + (q >> 1) * 8 + (lane & 7)) * L::RP + mt * 16 + (q & 1) * 8;
        ldsm_x4_t(smem_u32(sF + off), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
        ldsm_x4_t(smem_u32(sFl + off), al[mt][0], al[mt][1], al[mt][2], al[mt][3]);
      }
      uint32_t bf[4];
      ldsm_x4_t(tV + swz(kk * 16 + (q & 1) * 8 + (lane & 7), 2 * warp + (q >> 1)), bf[0], bf[1], bf[2], bf[3]);
#pragma unroll
      for (int mt = 0; mt < MT_S; ++mt) {
        mma_bf16(sacc[mt][0], af[mt], bf);
        mma_bf16(sacc[mt][1], af[mt], bf + 2);
        mma_bf16(sacc[mt][0], al[mt], bf);
        mma_bf16(sacc[mt][1], al[mt], bf + 2);
      }
    }
  }
  // every issued copy must land before the CTA leaves (only a failed wait leaves some)
  if (tid == 0)
    for (int t = consumed; t < issued; ++t) mbar_wait(smem_u32(&full[t % kStages]), (t / kStages) & 1, wc, false);

  // ---- partials of this chunk (zeros for an empty chunk)
  float* Sp = S_part + ((size_t)bh * dm.nchunk + chunk) * RK * kD;
#pragma unroll
  for (int mt = 0; mt < MT_S; ++mt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int row = mt * 16 + g8 + 8 * hh;
        const int col = 16 * warp + nt * 8 + 2 * t4;
        *reinterpret_cast<float2*>(Sp + (size_t)row * kD + col) =
            make_float2(sacc[mt][nt][2 * hh], sacc[mt][nt][2 * hh + 1]);
      }
  __syncthreads();
  if (warp < 4) {
    // lanes with equal t4 hold the same columns: add over the 8 row groups
#pragma unroll
    for (int nt = 0; nt < NT_F; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float x = zacc[nt][e];
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        if (g8 == 0) sZ[warp * RK + nt * 8 + 2 * t4 + e] = x;
      }
  }
  __syncthreads();
  if (tid < RK)
    z_part[((size_t)bh * dm.nchunk + chunk) * RK + tid] =
        ((sZ[tid] + sZ[RK + tid]) + sZ[2 * RK + tid]) + sZ[3 * RK + tid];
}

template <int RK, bool FP8>
cudaError_t launch_variant(const Dims& dm, const void* k, const void* v, const void* Wk, const Workspace& ws,
                           cudaStream_t st) {
  constexpr size_t smem = KVSmem<RK>::bytes;
  cudaError_t e = cudaFuncSetAttribute(kv_pass_kernel<RK, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  CUtensorMap tk, tv;
  if (!make_act_map(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k, dm, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_act_map(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, v, dm, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  dim3 grid(dm.nchunk, dm.B * dm.H);
  kv_pass_kernel<RK, FP8><<<grid, kThreads, smem, st>>>(
      tk, tv, static_cast<const __nv_bfloat16*>(Wk), dm, ws.rope, ws.S_part, ws.z_part, ws.kbar, ws.v16, ws.k8, ws.v8,
      ws.sk, ws.sv, ws.status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kv_pass(const Dims& dm, bool fp8, const void* k, const void* v, const void* Wk,
                           const Workspace& ws, cudaStream_t st) {
  if (dm.r == 32)
    return fp8 ? launch_variant<32, true>(dm, k, v, Wk, ws, st) : launch_variant<32, false>(dm, k, v, Wk, ws, st);
  return fp8 ? launch_variant<16, true>(dm, k, v, Wk, ws, st) : launch_variant<16, false>(dm, k, v, Wk, ws, st);
}

}  // namespace rola
