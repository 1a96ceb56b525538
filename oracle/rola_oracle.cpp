// RoLA forward — CPU oracle (test infrastructure, NOT part of the product).
//
// Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
// load this library.  It shares no code, header, table or constant with the
// CUDA library: every quantity below is recomputed here from the definition with
// plain loops and no blocking, fusion or reordering -- in double precision, except
// the block selection, which is taken in fp32 (item 2 below).
//
// Sources (web pages about SparkDiffusion / RoLA; cited by page title and section):
//   [README]  "AlibabaResearch/SparkDiffusion" (GitHub README mirror):
//             - inference section: topk is a keep ratio (0.1/0.05/0.03 = 90/95/97 % sparsity);
//             - sparse-finetuning section: RoLA adds proj_q, proj_k, gate_proj, gate_bias;
//             - citation block: "RoLA: Rotary-Positioned Low-Rank Linear Attention",
//               "RoPeSLR: 3D RoPE-driven Sparse-LowRank Attention".
//   [NEWS]    "SparkDiffusion ... SparkWan" news article, section "What's New":
//             RoLA = a sparse branch over high-energy query-key blocks plus a light
//             low-rank path that restores global context.
//   [BLOG]    "SparkDiffusion: 265x Faster Video Generation on Consumer GPUs via Sparse
//             Attention & Distillation", section "RoLA: Preserving Global Context at
//             Extreme Sparsity": block-sparse branch keeps the high-energy interactions,
//             a low-rank linear branch with rotary positions recovers the dropped context.
//
// The pages fix only that structure.  The concrete operator this oracle computes
// (each reading is listed again in the design notes of the repository):
//   1. 64-token blocks of the flattened (t,h,w) token order; the last block may be short.
//   2. Block energy s_ij = mean(q over block i) . mean(k over block j), no scale.  The
//      selection is an integer decision taken from floating point, so it is taken in
//      the precision of the GPU kernels (fp32), in a stated order: token sums in token
//      order, one division by the count, a fused multiply-add chain over channels.
//   3. Each query block keeps k = clamp(ceil(topk*nb - 1e-9), 1, nb) key blocks with the
//      largest s_ij; equal scores rank the lower key-block index first; the kept list is
//      stored in ascending order.
//   4. Sparse branch: exact softmax attention of every query token of block i over all
//      valid key tokens of its kept blocks, logits (q.k)*scale, scale = 1/sqrt(d) by default.
//   5. Linear branch over ALL N keys: u = phi(q Wq_h), f = phi(k Wk_h), phi(x) = elu(x)+1;
//      R(p) rotates the r/2 adjacent pairs (2c, 2c+1) by theta_c = pos_axis(c)(p) *
//      base^(-c'/P_axis); numerator = (R(p_n) u_n)^T sum_m R(p_m) f_m v_m^T,
//      denominator = u_n^T sum_m f_m (unrotated), O_lin = numerator / denominator.
//   6. out = O_sparse + g * O_lin, with one of three gains: g_h per head; g_{n,h} per
//      token and head, given; or the gate computed from the query, g_{n,h} =
//      sigmoid(q_{n,h} . wg_h + bg_h), from the gate_proj (wg, [H][d]) and gate_bias (bg,
//      [H]) parameters the README's sparse-finetuning section adds.
//
// Build: g++ -O3 -fopenmp -shared -fPIC (no -march, no fast-math: no FMA contraction).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

constexpr int kBlock = 64;  // tokens per block (reading 1)

}  // namespace

extern "C" {

// Problem description as the oracle sees it.  Plain struct, own definition.
struct rola_oracle_shape {
  int B, H, N, d, r;
  int grid_t, grid_h, grid_w;     // grid_t*grid_h*grid_w == N
  int pairs_t, pairs_h, pairs_w;  // rotary pairs per axis, sum == r/2
  double rope_base;               // frequency base (10000)
  double scale;                   // softmax logit scale
  double topk;                    // keep ratio in (0, 1]
  int gate_mode;                  // 0: g is [H] (a gain per head); 1: g is [B][N][H] (a gain
                                  // per token and head); 2: g holds gate_proj [H][d] then
                                  // gate_bias [H], and the gain is sigmoid(q . wg_h + bg_h)
};

int rola_oracle_num_blocks(int N) { return (N + kBlock - 1) / kBlock; }

// Reading 3 / [README] inference section: topk is the fraction of key blocks kept.
int rola_oracle_keep_count(int nb, double topk) {
  double x = std::ceil(topk * (double)nb - 1e-9);
  int k = (int)x;
  if (k < 1) k = 1;
  if (k > nb) k = nb;
  return k;
}

// Positions of the flattened (t, h, w) grid: token n = (t*grid_h + y)*grid_w + x.
// pos is [N][3] = (t, y, x).
void rola_oracle_positions(const rola_oracle_shape* s, double* pos) {
  for (int n = 0; n < s->N; ++n) {
    int x = n % s->grid_w;
    int y = (n / s->grid_w) % s->grid_h;
    int t = n / (s->grid_w * s->grid_h);
    pos[3 * n + 0] = t;
    pos[3 * n + 1] = y;
    pos[3 * n + 2] = x;
  }
}

// Mean of x over the valid tokens of each block (reading 2), in the precision the
// selection decision is taken in (fp32): the tokens of the block are added one after
// the other in token order into an fp32 sum, then the sum is divided by the count
// (one IEEE fp32 division).  x: [B, N, H, d] (float values), xbar: [B, H, nb, d].
void rola_oracle_pool(const rola_oracle_shape* s, const float* x, float* xbar) {
  const int B = s->B, H = s->H, N = s->N, d = s->d;
  const int nb = rola_oracle_num_blocks(N);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < nb; ++i) {
        int n0 = i * kBlock, n1 = std::min(N, n0 + kBlock);
        float* o = xbar + (((size_t)b * H + h) * nb + i) * d;
        for (int c = 0; c < d; ++c) {
          volatile float acc = 0.0f;  // volatile: one rounding per addition, in order
          for (int n = n0; n < n1; ++n) acc = acc + x[(((size_t)b * N + n) * H + h) * d + c];
          o[c] = acc / (float)(n1 - n0);
        }
      }
}

// Block energy s_ij = qbar_i . kbar_j (reading 2) in fp32: a chain of fused
// multiply-adds over the channels in order 0..d-1, starting from 0.
static float block_score(const float* qb, const float* kb, int d) {
  float acc = 0.0f;
  for (int c = 0; c < d; ++c) acc = std::fmaf(qb[c], kb[c], acc);
  return acc;
}

// Top-k with lowest-index tie-break, ascending lists (reading 3).
// col_idx: [B, H, nb, k].  kth: the k-th largest score of each row.  next: the
// (k+1)-th largest (-inf when k == nb).  amax: max_j |s_ij|.  All per row [B, H, nb].
void rola_oracle_select(const rola_oracle_shape* s, const float* qbar, const float* kbar,
                        int32_t* col_idx, double* kth, double* next, double* amax) {
  const int B = s->B, H = s->H, d = s->d;
  const int nb = rola_oracle_num_blocks(s->N);
  const int k = rola_oracle_keep_count(nb, s->topk);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      std::vector<float> sc(nb);
      std::vector<int> order(nb);
      const float* Qb = qbar + ((size_t)b * H + h) * nb * d;
      const float* Kb = kbar + ((size_t)b * H + h) * nb * d;
      for (int i = 0; i < nb; ++i) {
        double m = 0.0;
        for (int j = 0; j < nb; ++j) {
          sc[j] = block_score(Qb + (size_t)i * d, Kb + (size_t)j * d, d);
          m = std::max(m, std::fabs((double)sc[j]));
        }
        for (int j = 0; j < nb; ++j) order[j] = j;
        std::sort(order.begin(), order.end(), [&](int a, int c) {
          if (sc[a] != sc[c]) return sc[a] > sc[c];
          return a < c;
        });
        size_t row = ((size_t)b * H + h) * nb + i;
        kth[row] = sc[order[k - 1]];
        next[row] = (k < nb) ? (double)sc[order[k]] : -std::numeric_limits<double>::infinity();
        amax[row] = m;
        std::vector<int> kept(order.begin(), order.begin() + k);
        std::sort(kept.begin(), kept.end());
        for (int t = 0; t < k; ++t) col_idx[row * k + t] = kept[t];
      }
    }
}

// phi(x) = elu(x) + 1 (alpha = 1): x + 1 for x > 0, exp(x) otherwise (reading 5).
static double phi(double x) { return x > 0.0 ? x + 1.0 : std::exp(x); }

// Axis and in-axis index of rotary pair c: pairs are ordered t, then h, then w.
static void pair_axis(const rola_oracle_shape* s, int c, int* axis, int* cprime, int* count) {
  if (c < s->pairs_t) {
    *axis = 0; *cprime = c; *count = s->pairs_t;
  } else if (c < s->pairs_t + s->pairs_h) {
    *axis = 1; *cprime = c - s->pairs_t; *count = s->pairs_h;
  } else {
    *axis = 2; *cprime = c - s->pairs_t - s->pairs_h; *count = s->pairs_w;
  }
}

// y = R(p) x for one position p (3 coordinates), x, y of length r.
// Pair (2c, 2c+1) is turned counter-clockwise by theta_c.
static void rotate(const rola_oracle_shape* s, const double* p, const double* x, double* y) {
  for (int c = 0; c < s->r / 2; ++c) {
    int axis, cp, cnt;
    pair_axis(s, c, &axis, &cp, &cnt);
    double theta = p[axis] * std::pow(s->rope_base, -(double)cp / (double)cnt);
    double cs = std::cos(theta), sn = std::sin(theta);
    y[2 * c] = cs * x[2 * c] - sn * x[2 * c + 1];
    y[2 * c + 1] = sn * x[2 * c] + cs * x[2 * c + 1];
  }
}

// phi(x_n W_h) for one token row x (length d), W: [H, d, r] (float values).
static void feature(const rola_oracle_shape* s, const float* xrow, const float* W, int h,
                    double* out) {
  const int d = s->d, r = s->r;
  for (int a = 0; a < r; ++a) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += (double)xrow[c] * (double)W[((size_t)h * d + c) * r + a];
    out[a] = phi(acc);
  }
}

// Linear-branch state over all N keys (reading 5):
//   S_h = sum_m R(p_m) phi(k_m Wk_h) v_m^T   -> S: [B, H, r, d]
//   z_h = sum_m phi(k_m Wk_h)                -> z: [B, H, r]
// pos: [N][3] positions (any values; the grid helper gives the default ones).
void rola_oracle_linear_state(const rola_oracle_shape* s, const float* k, const float* v,
                              const float* Wk, const double* pos, double* S, double* z) {
  const int B = s->B, H = s->H, N = s->N, d = s->d, r = s->r;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      std::vector<double> f(r), fr(r);
      double* Sh = S + ((size_t)b * H + h) * r * d;
      double* zh = z + ((size_t)b * H + h) * r;
      for (int a = 0; a < r * d; ++a) Sh[a] = 0.0;
      for (int a = 0; a < r; ++a) zh[a] = 0.0;
      for (int m = 0; m < N; ++m) {
        const float* km = k + (((size_t)b * N + m) * H + h) * d;
        const float* vm = v + (((size_t)b * N + m) * H + h) * d;
        feature(s, km, Wk, h, f.data());
        rotate(s, pos + 3 * (size_t)m, f.data(), fr.data());
        for (int a = 0; a < r; ++a) {
          zh[a] += f[a];
          for (int c = 0; c < d; ++c) Sh[(size_t)a * d + c] += fr[a] * (double)vm[c];
        }
      }
    }
}

// The gain of token n of (b, h) (reading 6): g_h; g_{n,h} given per token; or the gate
// from the query, sigmoid(q_n . wg_h + bg_h) (README sparse-finetuning section: gate_proj,
// gate_bias), with the dot product and the sigmoid in double.
static double gain(const rola_oracle_shape* s, const double* g, const float* qn, int b, int n, int h) {
  if (s->gate_mode == 1) return g[((size_t)b * s->N + n) * s->H + h];
  if (s->gate_mode == 2) {
    const double* wg = g + (size_t)h * s->d;
    double a = g[(size_t)s->H * s->d + h];
    for (int c = 0; c < s->d; ++c) a += (double)qn[c] * wg[c];
    return 1.0 / (1.0 + std::exp(-a));
  }
  return g[h];
}

// Output of the listed query blocks.  blocks: nrows triples (b, h, i).
// For each listed block, rows [0, 64) of the three outputs (each [nrows][64][d]) hold
//   sparse: O_sparse, lin: O_lin, out: O_sparse + g * O_lin
// with g the gain of the token (see gain above), for the valid tokens of the block; rows
// past N are left at 0.
void rola_oracle_attend_blocks(const rola_oracle_shape* s, const float* q, const float* k,
                               const float* v, const float* Wq, const double* g,
                               const int32_t* col_idx, const double* S, const double* z,
                               const double* pos, int nrows, const int32_t* blocks,
                               double* sparse, double* lin, double* out) {
  const int H = s->H, N = s->N, d = s->d, r = s->r;
  const int nb = rola_oracle_num_blocks(N);
  const int kk = rola_oracle_keep_count(nb, s->topk);
#pragma omp parallel for schedule(dynamic)
  for (int t = 0; t < nrows; ++t) {
    const int b = blocks[3 * t], h = blocks[3 * t + 1], i = blocks[3 * t + 2];
    const int32_t* L = col_idx + (((size_t)b * H + h) * nb + i) * kk;
    const double* Sh = S + ((size_t)b * H + h) * r * d;
    const double* zh = z + ((size_t)b * H + h) * r;
    std::vector<int> keys;
    for (int a = 0; a < kk; ++a)
      for (int m = L[a] * kBlock; m < std::min(N, (L[a] + 1) * kBlock); ++m) keys.push_back(m);
    std::vector<double> logit(keys.size()), u(r), ur(r);
    double* os = sparse + (size_t)t * kBlock * d;
    double* ol = lin + (size_t)t * kBlock * d;
    double* oo = out + (size_t)t * kBlock * d;
    std::memset(os, 0, sizeof(double) * kBlock * d);
    std::memset(ol, 0, sizeof(double) * kBlock * d);
    std::memset(oo, 0, sizeof(double) * kBlock * d);
    for (int n = i * kBlock; n < std::min(N, (i + 1) * kBlock); ++n) {
      const int row = n - i * kBlock;
      const float* qn = q + (((size_t)b * N + n) * H + h) * d;
      // Sparse branch: exact softmax over the kept keys (reading 4).
      double mx = -std::numeric_limits<double>::infinity();
      for (size_t a = 0; a < keys.size(); ++a) {
        const float* km = k + (((size_t)b * N + keys[a]) * H + h) * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += (double)qn[c] * (double)km[c];
        logit[a] = acc * s->scale;
        mx = std::max(mx, logit[a]);
      }
      double den = 0.0;
      for (size_t a = 0; a < keys.size(); ++a) {
        logit[a] = std::exp(logit[a] - mx);
        den += logit[a];
      }
      for (size_t a = 0; a < keys.size(); ++a) {
        const float* vm = v + (((size_t)b * N + keys[a]) * H + h) * d;
        double w = logit[a] / den;
        for (int c = 0; c < d; ++c) os[(size_t)row * d + c] += w * (double)vm[c];
      }
      // Linear branch (reading 5).
      feature(s, qn, Wq, h, u.data());
      rotate(s, pos + 3 * (size_t)n, u.data(), ur.data());
      double lden = 0.0;
      for (int a = 0; a < r; ++a) lden += u[a] * zh[a];
      for (int c = 0; c < d; ++c) {
        double num = 0.0;
        for (int a = 0; a < r; ++a) num += ur[a] * Sh[(size_t)a * d + c];
        ol[(size_t)row * d + c] = num / lden;
      }
      // Combination (reading 6).
      const double gn = gain(s, g, qn, b, n, h);
      for (int c = 0; c < d; ++c)
        oo[(size_t)row * d + c] = os[(size_t)row * d + c] + gn * ol[(size_t)row * d + c];
    }
  }
}

// Whole forward pass: out [B, N, H, d] (double) and col_idx [B, H, nb, k].
void rola_oracle_forward(const rola_oracle_shape* s, const float* q, const float* k,
                         const float* v, const float* Wq, const float* Wk, const double* g,
                         double* out, int32_t* col_idx) {
  const int B = s->B, H = s->H, N = s->N, d = s->d, r = s->r;
  const int nb = rola_oracle_num_blocks(N);
  std::vector<float> qbar((size_t)B * H * nb * d), kbar((size_t)B * H * nb * d);
  std::vector<double> kth((size_t)B * H * nb), nxt((size_t)B * H * nb), amax((size_t)B * H * nb);
  std::vector<double> pos((size_t)N * 3), S((size_t)B * H * r * d), z((size_t)B * H * r);
  rola_oracle_pool(s, q, qbar.data());
  rola_oracle_pool(s, k, kbar.data());
  rola_oracle_select(s, qbar.data(), kbar.data(), col_idx, kth.data(), nxt.data(), amax.data());
  rola_oracle_positions(s, pos.data());
  rola_oracle_linear_state(s, k, v, Wk, pos.data(), S.data(), z.data());
  std::vector<int32_t> blocks;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < nb; ++i) {
        blocks.push_back(b); blocks.push_back(h); blocks.push_back(i);
      }
  const int nrows = B * H * nb;
  std::vector<double> os((size_t)nrows * kBlock * d), ol((size_t)nrows * kBlock * d),
      oo((size_t)nrows * kBlock * d);
  rola_oracle_attend_blocks(s, q, k, v, Wq, g, col_idx, S.data(), z.data(), pos.data(), nrows,
                            blocks.data(), os.data(), ol.data(), oo.data());
  for (int t = 0; t < nrows; ++t) {
    const int b = blocks[3 * t], h = blocks[3 * t + 1], i = blocks[3 * t + 2];
    for (int n = i * kBlock; n < std::min(N, (i + 1) * kBlock); ++n)
      for (int c = 0; c < d; ++c)
        out[(((size_t)b * N + n) * H + h) * d + c] =
            oo[((size_t)t * kBlock + (n - i * kBlock)) * d + c];
  }
}

// ------------------------------------------------------------------ fp8 (e4m3) variant
//
// OCP 8-bit floating point, E4M3 flavour: 1 sign bit, 4 exponent bits (bias 7), 3
// mantissa bits.  Exponent field 0 holds subnormals m/8 * 2^-6; fields 1..15 hold
// (1 + m/8) * 2^(e-7), except field 15 with mantissa 7, which is NaN.  There are no
// infinities; the largest finite magnitude is 448 (field 15, mantissa 6).
//
// Encoding of a finite float y: round |y| to the nearest representable magnitude, ties
// to the even mantissa; magnitudes above 448 saturate to 448.  Written from the format
// definition: within the binade [2^E, 2^(E+1)) (E >= -6) the spacing is 2^(E-3); below
// 2^-6 it is the subnormal spacing 2^-9.
static uint8_t e4m3_encode(float y) {
  const uint8_t sign = std::signbit(y) ? 0x80 : 0x00;
  const double a = std::fabs((double)y);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int E = (int)std::floor(std::log2(a));
  // log2 of a double can land one off near powers of two: correct it exactly.
  while (std::ldexp(1.0, E) > a) --E;
  while (std::ldexp(1.0, E + 1) <= a) ++E;
  if (E < -6) E = -6;                                // subnormal range shares 2^-9 spacing
  const double step = std::ldexp(1.0, E - 3);
  const double n = a / step;                         // exact: a power-of-two division
  double r = std::floor(n);
  const double frac = n - r;
  if (frac > 0.5 || (frac == 0.5 && std::fmod(r, 2.0) != 0.0)) r += 1.0;
  const double v = r * step;                         // the rounded magnitude (<= 448)
  if (v < std::ldexp(1.0, -6)) return sign | (uint8_t)(v / std::ldexp(1.0, -9));   // subnormal
  int Ev = (int)std::floor(std::log2(v));
  while (std::ldexp(1.0, Ev) > v) --Ev;
  while (std::ldexp(1.0, Ev + 1) <= v) ++Ev;
  const int mant = (int)((v / std::ldexp(1.0, Ev) - 1.0) * 8.0);
  return sign | (uint8_t)(((Ev + 7) << 3) | mant);
}

static double e4m3_decode(uint8_t c) {
  const double sgn = (c & 0x80) ? -1.0 : 1.0;
  const int e = (c >> 3) & 0xF, m = c & 7;
  if (e == 15 && m == 7) return std::numeric_limits<double>::quiet_NaN();
  if (e == 0) return sgn * std::ldexp((double)m / 8.0, -6);
  return sgn * std::ldexp(1.0 + m / 8.0, e - 7);
}

void rola_oracle_e4m3_encode(const float* y, uint8_t* code, size_t n) {
  for (size_t e = 0; e < n; ++e) code[e] = e4m3_encode(y[e]);
}

void rola_oracle_e4m3_decode(const uint8_t* code, double* y, size_t n) {
  for (size_t e = 0; e < n; ++e) y[e] = e4m3_decode(code[e]);
}

// Per-(b, h, 64-token block) quantisation of x [B, N, H, d] (float values) to e4m3:
// absmax over the block's valid tokens and all d channels; scale = absmax / 448 (1 when
// absmax = 0); code = encode(x * (1 / scale)).  The integer codes are decided from
// floating point, so this is done in the precision the kernels use: the division, the
// reciprocal and the product are each one fp32 operation rounded to nearest.
// codes: [B, N, H, d]; scales: [B, H, nb].
void rola_oracle_quantize_blocks(const rola_oracle_shape* s, const float* x, uint8_t* codes,
                                 float* scales) {
  const int B = s->B, H = s->H, N = s->N, d = s->d;
  const int nb = rola_oracle_num_blocks(N);
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int i = 0; i < nb; ++i) {
        const int n0 = i * kBlock, n1 = std::min(N, n0 + kBlock);
        float amax = 0.0f;
        for (int n = n0; n < n1; ++n)
          for (int c = 0; c < d; ++c) amax = std::max(amax, std::fabs(x[(((size_t)b * N + n) * H + h) * d + c]));
        volatile float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
        volatile float inv = 1.0f / scale;
        scales[((size_t)b * H + h) * nb + i] = scale;
        for (int n = n0; n < n1; ++n)
          for (int c = 0; c < d; ++c) {
            const size_t at = (((size_t)b * N + n) * H + h) * d + c;
            volatile float y = x[at] * inv;
            codes[at] = e4m3_encode(y);
          }
      }
}

// ------------------------------------------------------------------ backward (next row f2)
//
// Gradients of L = sum_n dout_n . out_n with respect to q, k, v, Wq, Wk and the gain
// parameters, the kept-block lists held fixed (the selection is a discrete choice; its
// gradient is zero almost everywhere).  Derived by the chain rule from steps 4-6 above:
//   sparse (each query token n, kept keys m):  P_nm = softmax_m(scale q_n . k_m),
//     O_n = sum_m P_nm v_m;  D_n = dout_n . O_n;  dA_nm = P_nm (dout_n . v_m - D_n);
//     dv_m += P_nm dout_n;  dq_n += scale sum_m dA_nm k_m;  dk_m += scale sum_n dA_nm q_n;
//   combination: out_n = O_n + g_n L_n;  dg_n = dout_n . L_n; with gG_n = g_n dout_n
//   linear, query side (x_n = q_n Wq, u_n = phi(x_n), y_n = R(p_n) u_n, den_n = u_n . z,
//     L_n = y_n^T S / den_n):  dS += y_n gG_n^T / den_n;  dy_n = S gG_n / den_n;
//     dden_n = -(gG_n . L_n) / den_n;  du_n = R(p_n)^T dy_n + dden_n z;  dz += dden_n u_n;
//     dx_n = phi'(x_n) du_n (phi'(x) = 1 for x > 0, e^x otherwise);  dq_n += Wq dx_n;
//     dWq += q_n dx_n^T;
//   linear, key side (w_m = k_m Wk, f_m = phi(w_m), S = sum_m R(p_m) f_m v_m^T,
//     z = sum_m f_m):  dv_m += dS^T R(p_m) f_m;  df_m = R(p_m)^T (dS v_m) + dz;
//     dw_m = phi'(w_m) df_m;  dk_m += Wk dw_m;  dWk += k_m dw_m^T;
//   gain from the query (gate_mode 2, g_n = sigmoid(q_n . wg + bg)): dlogit_n =
//     dg_n g_n (1 - g_n);  dq_n += dlogit_n wg;  dwg += dlogit_n q_n;  dbg += dlogit_n.
// Inputs as for the forward; dout [B,N,H,d] (double); col_idx the forward's lists.
// Outputs (double, overwritten): dq, dk, dv [B,N,H,d]; dWq, dWk [H,d,r]; dg with the
// layout of g ([H], [B,N,H], or gate_proj [H][d] then gate_bias [H]).
static double phi_grad(double x) { return x > 0.0 ? 1.0 : std::exp(x); }

// y = R(p)^T x: pair (2c, 2c+1) turned clockwise by theta_c.
static void rotate_back(const rola_oracle_shape* s, const double* p, const double* x, double* y) {
  for (int c = 0; c < s->r / 2; ++c) {
    int axis, cp, cnt;
    pair_axis(s, c, &axis, &cp, &cnt);
    double theta = p[axis] * std::pow(s->rope_base, -(double)cp / (double)cnt);
    double cs = std::cos(theta), sn = std::sin(theta);
    y[2 * c] = cs * x[2 * c] + sn * x[2 * c + 1];
    y[2 * c + 1] = -sn * x[2 * c] + cs * x[2 * c + 1];
  }
}

void rola_oracle_backward(const rola_oracle_shape* s, const float* q, const float* k,
                          const float* v, const float* Wq, const float* Wk, const double* g,
                          const double* dout, const int32_t* col_idx, double* dq, double* dk,
                          double* dv, double* dWq, double* dWk, double* dg) {
  const int B = s->B, H = s->H, N = s->N, d = s->d, r = s->r;
  const int nb = rola_oracle_num_blocks(N);
  const int kk = rola_oracle_keep_count(nb, s->topk);
  std::vector<double> pos((size_t)N * 3);
  rola_oracle_positions(s, pos.data());
  const size_t nact = (size_t)B * N * H * d;
  std::fill(dq, dq + nact, 0.0);
  std::fill(dk, dk + nact, 0.0);
  std::fill(dv, dv + nact, 0.0);
  std::fill(dWq, dWq + (size_t)H * d * r, 0.0);
  std::fill(dWk, dWk + (size_t)H * d * r, 0.0);
  const size_t ng = s->gate_mode == 0 ? (size_t)H : s->gate_mode == 1 ? (size_t)B * N * H : (size_t)H * (d + 1);
  std::fill(dg, dg + ng, 0.0);
  auto at = [&](int b, int n, int h) { return (((size_t)b * N + n) * H + h) * d; };
  // heads are independent, and dWq, dWk and a per-head dg sum over the batch inside one head
#pragma omp parallel for schedule(dynamic)
  for (int h = 0; h < H; ++h)
    for (int b = 0; b < B; ++b) {
      // key-side features and the state (as the forward computes them, in double)
      std::vector<double> w((size_t)N * r), f((size_t)N * r), yk((size_t)N * r);
      std::vector<double> S((size_t)r * d, 0.0), z(r, 0.0);
      for (int m = 0; m < N; ++m) {
        const float* km = k + at(b, m, h);
        const float* vm = v + at(b, m, h);
        for (int a = 0; a < r; ++a) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += (double)km[c] * (double)Wk[((size_t)h * d + c) * r + a];
          w[(size_t)m * r + a] = acc;
          f[(size_t)m * r + a] = phi(acc);
        }
        rotate(s, &pos[3 * (size_t)m], &f[(size_t)m * r], &yk[(size_t)m * r]);
        for (int a = 0; a < r; ++a) {
          z[a] += f[(size_t)m * r + a];
          for (int c = 0; c < d; ++c) S[(size_t)a * d + c] += yk[(size_t)m * r + a] * (double)vm[c];
        }
      }
      std::vector<double> dS((size_t)r * d, 0.0), dz(r, 0.0);
      std::vector<double> x(r), u(r), yq(r), L(d), O(d), gG(d), dy(r), du(r), dx(r);
      std::vector<int> keys;
      std::vector<double> P;
      for (int i = 0; i < nb; ++i) {
        const int32_t* Li = col_idx + (((size_t)b * H + h) * nb + i) * kk;
        keys.clear();
        for (int a = 0; a < kk; ++a)
          for (int m = Li[a] * kBlock; m < std::min(N, (Li[a] + 1) * kBlock); ++m) keys.push_back(m);
        P.resize(keys.size());
        for (int n = i * kBlock; n < std::min(N, (i + 1) * kBlock); ++n) {
          const float* qn = q + at(b, n, h);
          const double* G = dout + at(b, n, h);
          // sparse branch: P and O
          double mx = -std::numeric_limits<double>::infinity();
          for (size_t a = 0; a < keys.size(); ++a) {
            const float* km = k + at(b, keys[a], h);
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += (double)qn[c] * (double)km[c];
            P[a] = acc * s->scale;
            mx = std::max(mx, P[a]);
          }
          double sum = 0.0;
          for (size_t a = 0; a < keys.size(); ++a) {
            P[a] = std::exp(P[a] - mx);
            sum += P[a];
          }
          for (int c = 0; c < d; ++c) O[c] = 0.0;
          for (size_t a = 0; a < keys.size(); ++a) {
            P[a] /= sum;
            const float* vm = v + at(b, keys[a], h);
            for (int c = 0; c < d; ++c) O[c] += P[a] * (double)vm[c];
          }
          double Dn = 0.0;
          for (int c = 0; c < d; ++c) Dn += G[c] * O[c];
          for (size_t a = 0; a < keys.size(); ++a) {
            const int m = keys[a];
            const float* km = k + at(b, m, h);
            const float* vm = v + at(b, m, h);
            double dP = 0.0;
            for (int c = 0; c < d; ++c) dP += G[c] * (double)vm[c];
            const double dA = P[a] * (dP - Dn);
            for (int c = 0; c < d; ++c) {
              dv[at(b, m, h) + c] += P[a] * G[c];
              dq[at(b, n, h) + c] += s->scale * dA * (double)km[c];
              dk[at(b, m, h) + c] += s->scale * dA * (double)qn[c];
            }
          }
          // linear branch, query side
          for (int a = 0; a < r; ++a) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += (double)qn[c] * (double)Wq[((size_t)h * d + c) * r + a];
            x[a] = acc;
            u[a] = phi(acc);
          }
          rotate(s, &pos[3 * (size_t)n], u.data(), yq.data());
          double den = 0.0;
          for (int a = 0; a < r; ++a) den += u[a] * z[a];
          for (int c = 0; c < d; ++c) {
            double num = 0.0;
            for (int a = 0; a < r; ++a) num += yq[a] * S[(size_t)a * d + c];
            L[c] = num / den;
          }
          const double gn = gain(s, g, qn, b, n, h);
          double dgn = 0.0;
          for (int c = 0; c < d; ++c) dgn += G[c] * L[c];
          if (s->gate_mode == 0) {
            dg[h] += dgn;
          } else if (s->gate_mode == 1) {
            dg[((size_t)b * N + n) * H + h] = dgn;
          } else {
            const double dlogit = dgn * gn * (1.0 - gn);
            const double* wg = g + (size_t)h * d;
            for (int c = 0; c < d; ++c) {
              dq[at(b, n, h) + c] += dlogit * wg[c];
              dg[(size_t)h * d + c] += dlogit * (double)qn[c];
            }
            dg[(size_t)H * d + h] += dlogit;
          }
          for (int c = 0; c < d; ++c) gG[c] = gn * G[c];
          double gGL = 0.0;
          for (int c = 0; c < d; ++c) gGL += gG[c] * L[c];
          const double dden = -gGL / den;
          for (int a = 0; a < r; ++a) {
            double acc = 0.0;
            for (int c = 0; c < d; ++c) {
              dS[(size_t)a * d + c] += yq[a] * gG[c] / den;
              acc += S[(size_t)a * d + c] * gG[c];
            }
            dy[a] = acc / den;
          }
          rotate_back(s, &pos[3 * (size_t)n], dy.data(), du.data());
          for (int a = 0; a < r; ++a) {
            du[a] += dden * z[a];
            dz[a] += dden * u[a];
            dx[a] = phi_grad(x[a]) * du[a];
          }
          for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int a = 0; a < r; ++a) {
              acc += (double)Wq[((size_t)h * d + c) * r + a] * dx[a];
              dWq[((size_t)h * d + c) * r + a] += (double)qn[c] * dx[a];
            }
            dq[at(b, n, h) + c] += acc;
          }
        }
      }
      // linear branch, key side
      std::vector<double> dyk(r), df(r);
      for (int m = 0; m < N; ++m) {
        const float* km = k + at(b, m, h);
        const float* vm = v + at(b, m, h);
        for (int c = 0; c < d; ++c) {
          double acc = 0.0;
          for (int a = 0; a < r; ++a) acc += dS[(size_t)a * d + c] * yk[(size_t)m * r + a];
          dv[at(b, m, h) + c] += acc;
        }
        for (int a = 0; a < r; ++a) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += dS[(size_t)a * d + c] * (double)vm[c];
          dyk[a] = acc;
        }
        rotate_back(s, &pos[3 * (size_t)m], dyk.data(), df.data());
        for (int a = 0; a < r; ++a) df[a] = phi_grad(w[(size_t)m * r + a]) * (df[a] + dz[a]);
        for (int c = 0; c < d; ++c) {
          double acc = 0.0;
          for (int a = 0; a < r; ++a) {
            acc += (double)Wk[((size_t)h * d + c) * r + a] * df[a];
            dWk[((size_t)h * d + c) * r + a] += (double)km[c] * df[a];
          }
          dk[at(b, m, h) + c] += acc;
        }
      }
    }
}

// The same gradients on a sample, for problems too large for the whole backward: for the
// listed heads h (all batch entries) the per-head dWq[h], dWk[h] and dg[h] (gate_mode 0
// only), and for the listed blocks (b, h, i) the 64 rows of dq (qblocks) or of dk, dv
// (kblocks).  Every listed block's head must be listed.  Same definition and arithmetic as
// rola_oracle_backward, restricted to what the sample needs: the linear branch over all
// tokens of the listed heads, the softmax of every query row that touches a listed block.
// Outputs: dq [nq][64][d], dk, dv [nk][64][d] (rows past N zero), dWq, dWk [nh][d][r],
// dg [nh].
void rola_oracle_backward_sample(const rola_oracle_shape* s, const float* q, const float* k,
                                 const float* v, const float* Wq, const float* Wk, const double* g,
                                 const double* dout, const int32_t* col_idx, int nh, const int32_t* heads,
                                 int nq, const int32_t* qblocks, int nk, const int32_t* kblocks,
                                 double* dq, double* dk, double* dv, double* dWq, double* dWk, double* dg) {
  const int B = s->B, H = s->H, N = s->N, d = s->d, r = s->r;
  const int nb = rola_oracle_num_blocks(N);
  const int kk = rola_oracle_keep_count(nb, s->topk);
  std::vector<double> pos((size_t)N * 3);
  rola_oracle_positions(s, pos.data());
  std::fill(dq, dq + (size_t)nq * kBlock * d, 0.0);
  std::fill(dk, dk + (size_t)nk * kBlock * d, 0.0);
  std::fill(dv, dv + (size_t)nk * kBlock * d, 0.0);
  std::fill(dWq, dWq + (size_t)nh * d * r, 0.0);
  std::fill(dWk, dWk + (size_t)nh * d * r, 0.0);
  std::fill(dg, dg + nh, 0.0);
  auto at = [&](int b, int n, int h) { return (((size_t)b * N + n) * H + h) * d; };
  // softmax row of query token n of (b, h): probabilities over its kept keys, and D_n
  auto softmax_row = [&](int b, int h, int n, std::vector<int>& keys, std::vector<double>& P, double& Dn) {
    const int i = n / kBlock;
    const int32_t* Li = col_idx + (((size_t)b * H + h) * nb + i) * kk;
    keys.clear();
    for (int a = 0; a < kk; ++a)
      for (int m = Li[a] * kBlock; m < std::min(N, (Li[a] + 1) * kBlock); ++m) keys.push_back(m);
    P.resize(keys.size());
    const float* qn = q + at(b, n, h);
    double mx = -std::numeric_limits<double>::infinity();
    for (size_t a = 0; a < keys.size(); ++a) {
      const float* km = k + at(b, keys[a], h);
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += (double)qn[c] * (double)km[c];
      P[a] = acc * s->scale;
      mx = std::max(mx, P[a]);
    }
    double sum = 0.0;
    for (size_t a = 0; a < keys.size(); ++a) {
      P[a] = std::exp(P[a] - mx);
      sum += P[a];
    }
    Dn = 0.0;
    const double* G = dout + at(b, n, h);
    for (size_t a = 0; a < keys.size(); ++a) {
      P[a] /= sum;
      const float* vm = v + at(b, keys[a], h);
      double gv = 0.0;
      for (int c = 0; c < d; ++c) gv += G[c] * (double)vm[c];
      Dn += P[a] * gv;
    }
  };
#pragma omp parallel for schedule(dynamic)
  for (int t = 0; t < nh; ++t) {
    const int h = heads[t];
    std::vector<int> keys;
    std::vector<double> P;
    for (int b = 0; b < B; ++b) {
      std::vector<double> w((size_t)N * r), yk((size_t)N * r), f(r);
      std::vector<double> S((size_t)r * d, 0.0), z(r, 0.0), dS((size_t)r * d, 0.0), dz(r, 0.0);
      for (int m = 0; m < N; ++m) {
        const float* km = k + at(b, m, h);
        const float* vm = v + at(b, m, h);
        for (int a = 0; a < r; ++a) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += (double)km[c] * (double)Wk[((size_t)h * d + c) * r + a];
          w[(size_t)m * r + a] = acc;
          f[a] = phi(acc);
        }
        rotate(s, &pos[3 * (size_t)m], f.data(), &yk[(size_t)m * r]);
        for (int a = 0; a < r; ++a) {
          z[a] += f[a];
          for (int c = 0; c < d; ++c) S[(size_t)a * d + c] += yk[(size_t)m * r + a] * (double)vm[c];
        }
      }
      // linear branch, query side, every token of (b, h)
      std::vector<double> x(r), u(r), yq(r), L(d), dy(r), du(r), dx(r);
      for (int n = 0; n < N; ++n) {
        const float* qn = q + at(b, n, h);
        const double* G = dout + at(b, n, h);
        for (int a = 0; a < r; ++a) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += (double)qn[c] * (double)Wq[((size_t)h * d + c) * r + a];
          x[a] = acc;
          u[a] = phi(acc);
        }
        rotate(s, &pos[3 * (size_t)n], u.data(), yq.data());
        double den = 0.0;
        for (int a = 0; a < r; ++a) den += u[a] * z[a];
        double dgn = 0.0;
        for (int c = 0; c < d; ++c) {
          double num = 0.0;
          for (int a = 0; a < r; ++a) num += yq[a] * S[(size_t)a * d + c];
          L[c] = num / den;
          dgn += G[c] * L[c];
        }
        const double gn = g[h];
        dg[t] += dgn;
        for (int a = 0; a < r; ++a) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) {
            dS[(size_t)a * d + c] += yq[a] * gn * G[c] / den;
            acc += S[(size_t)a * d + c] * gn * G[c];
          }
          dy[a] = acc / den;
        }
        const double dden = -gn * dgn / den;
        rotate_back(s, &pos[3 * (size_t)n], dy.data(), du.data());
        for (int a = 0; a < r; ++a) {
          du[a] += dden * z[a];
          dz[a] += dden * u[a];
          dx[a] = phi_grad(x[a]) * du[a];
        }
        for (int c = 0; c < d; ++c)
          for (int a = 0; a < r; ++a) dWq[((size_t)t * d + c) * r + a] += (double)qn[c] * dx[a];
        for (int e = 0; e < nq; ++e)   // the listed query blocks' linear part of dq
          if (qblocks[3 * e] == b && qblocks[3 * e + 1] == h && qblocks[3 * e + 2] == n / kBlock)
            for (int c = 0; c < d; ++c) {
              double acc = 0.0;
              for (int a = 0; a < r; ++a) acc += (double)Wq[((size_t)h * d + c) * r + a] * dx[a];
              dq[((size_t)e * kBlock + n % kBlock) * d + c] += acc;
            }
      }
      // linear branch, key side, every key of (b, h)
      std::vector<double> dyk(r), df(r);
      for (int m = 0; m < N; ++m) {
        const float* km = k + at(b, m, h);
        const float* vm = v + at(b, m, h);
        for (int a = 0; a < r; ++a) {
          double acc = 0.0;
          for (int c = 0; c < d; ++c) acc += dS[(size_t)a * d + c] * (double)vm[c];
          dyk[a] = acc;
        }
        rotate_back(s, &pos[3 * (size_t)m], dyk.data(), df.data());
        for (int a = 0; a < r; ++a) df[a] = phi_grad(w[(size_t)m * r + a]) * (df[a] + dz[a]);
        for (int c = 0; c < d; ++c)
          for (int a = 0; a < r; ++a) dWk[((size_t)t * d + c) * r + a] += (double)km[c] * df[a];
        for (int e = 0; e < nk; ++e)
          if (kblocks[3 * e] == b && kblocks[3 * e + 1] == h && kblocks[3 * e + 2] == m / kBlock)
            for (int c = 0; c < d; ++c) {
              double ak = 0.0, av = 0.0;
              for (int a = 0; a < r; ++a) {
                ak += (double)Wk[((size_t)h * d + c) * r + a] * df[a];
                av += dS[(size_t)a * d + c] * yk[(size_t)m * r + a];
              }
              dk[((size_t)e * kBlock + m % kBlock) * d + c] += ak;
              dv[((size_t)e * kBlock + m % kBlock) * d + c] += av;
            }
      }
      // sparse branch: dq of the listed query blocks
      double Dn;
      for (int e = 0; e < nq; ++e) {
        if (qblocks[3 * e] != b || qblocks[3 * e + 1] != h) continue;
        const int i = qblocks[3 * e + 2];
        for (int n = i * kBlock; n < std::min(N, (i + 1) * kBlock); ++n) {
          softmax_row(b, h, n, keys, P, Dn);
          const double* G = dout + at(b, n, h);
          for (size_t a = 0; a < keys.size(); ++a) {
            const float* km = k + at(b, keys[a], h);
            const float* vm = v + at(b, keys[a], h);
            double dP = 0.0;
            for (int c = 0; c < d; ++c) dP += G[c] * (double)vm[c];
            const double dA = P[a] * (dP - Dn);
            for (int c = 0; c < d; ++c) dq[((size_t)e * kBlock + n % kBlock) * d + c] += s->scale * dA * (double)km[c];
          }
        }
      }
      // sparse branch: dk, dv of the listed key blocks, over the query blocks that kept them
      for (int e = 0; e < nk; ++e) {
        if (kblocks[3 * e] != b || kblocks[3 * e + 1] != h) continue;
        const int j = kblocks[3 * e + 2];
        for (int i = 0; i < nb; ++i) {
          const int32_t* Li = col_idx + (((size_t)b * H + h) * nb + i) * kk;
          bool kept = false;
          for (int a = 0; a < kk; ++a) kept |= Li[a] == j;
          if (!kept) continue;
          for (int n = i * kBlock; n < std::min(N, (i + 1) * kBlock); ++n) {
            softmax_row(b, h, n, keys, P, Dn);
            const float* qn = q + at(b, n, h);
            const double* G = dout + at(b, n, h);
            for (size_t a = 0; a < keys.size(); ++a) {
              if (keys[a] / kBlock != j) continue;
              const float* vm = v + at(b, keys[a], h);
              double dP = 0.0;
              for (int c = 0; c < d; ++c) dP += G[c] * (double)vm[c];
              const double dA = P[a] * (dP - Dn);
              const size_t row = (size_t)e * kBlock + keys[a] % kBlock;
              for (int c = 0; c < d; ++c) {
                dk[row * d + c] += s->scale * dA * (double)qn[c];
                dv[row * d + c] += P[a] * G[c];
              }
            }
          }
        }
      }
    }
  }
}

int rola_oracle_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
