// CPU oracle for the FP8 block-scaled GEMM, its quantizers and dequantizer,
// the K-grouped GEMM and the expert FFN's activation.
//
// TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
// load this file or the library built from it: only tests/, the smoke check
// in __graft_entry__.py and bench.py's CPU legs (the CPU baseline and the
// reference arm) use it. It shares no code, header, table or constant
// generator with the CUDA library.
//
// What it computes (all plain definitions, written out without blocking,
// fusion or reordering beyond what the definition states):
//
//  * The e4m3 code: OCP 8-bit floating point specification, format E4M3
//    ("fn" variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
//    no infinities, S.1111.111 is NaN, largest finite magnitude 448. The pages
//    use FP8 operands without defining the bit layout ("DeepGEMM" overview,
//    zixun.chuxinyishu.com/article/345.html, section "FP8与细粒度缩放").
//  * Fine-grained scaling: activations get one fp32 scale per token per
//    128-channel slice, weights one fp32 scale per 128x128 block (same page
//    and section; DeepSeek-V3 review "28.5 倍压缩 + 1/10 成本",
//    developer.cloud.tencent.cn/article/2686109, "创新之处" item 4: one scale
//    per 128 elements and 128x128 block scaling; its "风险与不足" item 6 names
//    448.0 as the FP8 upper bound used by the quantizer).
//    Reading taken: s = amax_c / 448 with amax_c = max(amax, 1e-4) in fp32,
//    q = e4m3(x * (448 / amax_c)), the product rounded once in fp32, the
//    conversion round-to-nearest-even with saturation to +-448.
//  * The GEMM D = (A*sa)(B*sb)^T with two-level accumulation: the FP8 products
//    of every 128-wide K block are summed and then added into a higher
//    precision accumulator with both scales applied ("一文看懂 DeepSeek
//    開源項目第三彈" on animattoys.com, section "為現代 AI 計算而造", the
//    two-step FP8-multiply / high-precision-accumulate description, and the
//    deployment guide's note on two-level accumulation (promotion)).
//    The oracle reaches the exact value of that definition: each block sum of
//    128 products of e4m3 values is exact in fp64 (every product is a multiple
//    of 2^-18 below 2^18, so any partial sum needs fewer than 53 bits), and
//    only the two scale multiplies and the outer sum over K blocks round in
//    fp64. The result is kept in fp64, not rounded to bf16.
//
//  * Weight dequantization (the review's quantize / dequantize / GEMM trio):
//    x = bf16(fp32(dec(q) * s)) per element with the block's scale s.
//  * The K-grouped GEMM of FP8 training's expert weight gradients (the
//    animattoys.com page, section "為現代 AI 計算而造", names FP8 training
//    among DeepGEMM's uses; the DeepSeek-V3 review's quantize / dequantize /
//    GEMM trio, "创新之处" item 4, scales every operand per 128 elements of
//    the contraction). Reading taken: the contraction runs over tokens, the
//    experts' token ranges are stacked along it (each a multiple of 128), and
//    both operands carry one scale per row per 128-token block:
//      D[e][m][n] = sum over expert e's token blocks tb of
//                   sa[m][tb] * sb[n][tb] * sum_{t in tb} a[m][t] * b[n][t].
//    Exact block sums, fp64 result (as for the GEMM above).
//  * The expert FFN's activation (the "Mega MoE" kernel fuses both expert
//    GEMMs with the SwiGLU activation: "DeepGEMM" overview, section
//    "swapAB与Mega MoE"; the pages name SwiGLU without a formula). Reading
//    taken: h = silu(gate) * up with silu(g) = g / (1 + exp(-g)), gate and up
//    the bf16 outputs of the first GEMM, evaluated in fp32 and rounded once to
//    bf16. exp is evaluated by one fixed sequence of IEEE fp32 operations
//    (Cody and Waite's argument reduction, "Software Manual for the
//    Elementary Functions", 1980, then the degree-7 Taylor polynomial in
//    Horner form with fused multiply-adds), so that a second implementation
//    of the same method can agree with it bit for bit.
//
// Build: g++ -O2 -std=c++17 -fPIC -shared -pthread -ffp-contract=off
// (no fast-math: the quantizer's fp32 divide and multiply must be IEEE).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

constexpr int kBlock = 128;  // scale granularity along K and along N

// ---- e4m3 ------------------------------------------------------------------

struct E4M3Table {
  double value[256];
  E4M3Table() {
    for (int c = 0; c < 256; ++c) {
      const int sign = c >> 7;
      const int exponent = (c >> 3) & 0xF;
      const int mantissa = c & 0x7;
      double v;
      if (exponent == 0xF && mantissa == 0x7) {
        v = std::numeric_limits<double>::quiet_NaN();
      } else if (exponent == 0) {
        // subnormal: (mantissa / 8) * 2^(1 - 7)
        v = std::ldexp(static_cast<double>(mantissa), -9);
      } else {
        // normal: (1 + mantissa / 8) * 2^(exponent - 7)
        v = std::ldexp(static_cast<double>(8 + mantissa), exponent - 10);
      }
      value[c] = sign ? -v : v;
    }
  }
};

const E4M3Table& table() {
  static const E4M3Table t;
  return t;
}

// Round a float to the nearest e4m3 value, ties to the even code, saturating
// magnitudes at or above 448 to 448. NaN maps to 0x7F. The sign of zero is
// kept. Codes 0x00..0x7E hold the non-negative finite values in increasing
// order, so the nearest value is found by bisection over that range.
uint8_t encode(float v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(static_cast<double>(v));
  const double* t = table().value;
  if (a >= t[0x7E]) return sign | 0x7E;
  int lo = 0, hi = 0x7E;  // invariant: t[lo] <= a < t[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (t[mid] <= a) lo = mid; else hi = mid;
  }
  const double dlo = a - t[lo];
  const double dhi = t[hi] - a;
  int code;
  if (dlo < dhi) code = lo;
  else if (dhi < dlo) code = hi;
  else code = (lo % 2 == 0) ? lo : hi;
  return sign | static_cast<uint8_t>(code);
}

float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// Smallest power of two >= r, for a positive normal float r: 2^E if r is
// exactly 2^E (zero mantissa field), else 2^(E+1).
float pow2_ceil(float r) {
  uint32_t u;
  std::memcpy(&u, &r, sizeof u);
  uint32_t e = (u >> 23) & 0xFFu;
  if ((u & 0x007FFFFFu) != 0) e += 1;
  const uint32_t v = e << 23;
  float out;
  std::memcpy(&out, &v, sizeof out);
  return out;
}

// One scaling group: amax -> scale -> codes. `vals` holds the group's
// elements (already widened from bf16, which is exact).
// ue8m0 = 0: s = amax_c / 448, codes of x * (448 / amax_c) (one fp32 rounding).
// ue8m0 = 1 (the power-of-two scales of the DeepSeek-V3 review, "创新之处"
// item 4: UE8M0 scales are powers of two): s = the smallest power of two at
// or above amax_c / 448, codes of x / s (exact: s is a power of two), so no
// element exceeds 448 before rounding.
float quantize_group(const std::vector<float>& vals, std::vector<uint8_t>& codes, int ue8m0) {
  float amax = 0.0f;
  for (float x : vals) amax = std::max(amax, std::fabs(x));
  const float amax_c = std::max(amax, 1e-4f);
  codes.resize(vals.size());
  if (ue8m0) {
    const float scale = pow2_ceil(amax_c / 448.0f);
    for (size_t i = 0; i < vals.size(); ++i) codes[i] = encode(vals[i] / scale);
    return scale;
  }
  const float scale = amax_c / 448.0f;
  const float inv = 448.0f / amax_c;
  for (size_t i = 0; i < vals.size(); ++i) {
    const float y = vals[i] * inv;  // one fp32 rounding (no contraction)
    codes[i] = encode(y);
  }
  return scale;
}

// ---- SwiGLU -------------------------------------------------------------------

// exp(x) in fp32: x clamped to [-87, 88] (so that 2^n below stays a normal
// number), n = nearest integer to x * log2(e), r = x - n * ln2 with ln2 split
// into C1 = 355/512 (n * C1 is exact) and C2 = ln2 - C1, then
// exp(r) = sum_{k<=7} r^k / k! by Horner's rule with fused multiply-adds, and
// the result p * 2^n (one rounding).
float exp_f32(float x) {
  x = std::fmin(std::fmax(x, -87.0f), 88.0f);
  const float n = std::nearbyint(x * 1.44269504088896341f);
  const float c1 = 0.693359375f;
  const float c2 = -2.12194440e-4f;
  float r = std::fma(-n, c1, x);
  r = std::fma(-n, c2, r);
  float p = 1.0f / 5040.0f;
  p = std::fma(p, r, 1.0f / 720.0f);
  p = std::fma(p, r, 1.0f / 120.0f);
  p = std::fma(p, r, 1.0f / 24.0f);
  p = std::fma(p, r, 1.0f / 6.0f);
  p = std::fma(p, r, 0.5f);
  p = std::fma(p, r, 1.0f);
  p = std::fma(p, r, 1.0f);
  uint32_t bits = static_cast<uint32_t>(static_cast<int>(n) + 127) << 23;  // 2^n, n in [-126, 127]
  float two_n;
  std::memcpy(&two_n, &bits, 4);
  return p * two_n;
}

float silu_f32(float g) { return g / (1.0f + exp_f32(-g)); }

template <typename F>
void parallel_for(int64_t n, int threads, F&& body) {
  if (threads <= 0) threads = static_cast<int>(std::max(1u, std::thread::hardware_concurrency()));
  threads = static_cast<int>(std::min<int64_t>(threads, std::max<int64_t>(n, 1)));
  if (threads <= 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(threads);
  for (int t = 0; t < threads; ++t) {
    pool.emplace_back([&, t]() {
      for (int64_t i = t; i < n; i += threads) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

// Exact value of one output element: sum over K blocks of
// sa * sb * (exact sum of the block's 128 code products).
double dot_blocked(const uint8_t* qa_row, const float* sa_row, const uint8_t* qb_row,
                   const float* sb_row, int K) {
  const double* t = table().value;
  double acc = 0.0;
  for (int kb = 0; kb < K / kBlock; ++kb) {
    double s = 0.0;
    for (int k = kb * kBlock; k < (kb + 1) * kBlock; ++k) s += t[qa_row[k]] * t[qb_row[k]];
    acc += static_cast<double>(sa_row[kb]) * static_cast<double>(sb_row[kb]) * s;
  }
  return acc;
}

}  // namespace

extern "C" {

double oracle_e4m3_decode(uint8_t code) { return table().value[code]; }

uint8_t oracle_e4m3_encode(float v) { return encode(v); }

void oracle_e4m3_encode_array(const float* v, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = encode(v[i]);
}

// Activation quantizer, one scale per token per 128-channel slice.
// x: bf16 bits [G][M][K]; q: e4m3 codes [G][M][K]; s: fp32 [G][M][K/128]
// (logical order: token, then K block). Returns 0, or -1 on bad sizes.
int oracle_per_token_cast(const uint16_t* x, uint8_t* q, float* s, int G, int M, int K,
                          int threads, int ue8m0) {
  if (G < 0 || M < 0 || K <= 0 || K % kBlock != 0) return -1;
  const int KB = K / kBlock;
  parallel_for(static_cast<int64_t>(G) * M, threads, [&](int64_t row) {
    std::vector<float> vals(kBlock);
    std::vector<uint8_t> codes;
    for (int kb = 0; kb < KB; ++kb) {
      const int64_t base = row * K + static_cast<int64_t>(kb) * kBlock;
      for (int i = 0; i < kBlock; ++i) vals[i] = bf16_to_float(x[base + i]);
      s[row * KB + kb] = quantize_group(vals, codes, ue8m0);
      std::memcpy(q + base, codes.data(), kBlock);
    }
  });
  return 0;
}

// Weight quantizer, one scale per 128x128 block.
// x: bf16 bits [G][N][K]; q: [G][N][K]; s: fp32 [G][ceil(N/128)][K/128].
// A last block that covers fewer than 128 rows uses only its valid rows.
int oracle_per_block_cast(const uint16_t* x, uint8_t* q, float* s, int G, int N, int K,
                          int threads, int ue8m0) {
  if (G < 0 || N < 0 || K <= 0 || K % kBlock != 0) return -1;
  const int KB = K / kBlock;
  const int NB = (N + kBlock - 1) / kBlock;
  parallel_for(static_cast<int64_t>(G) * NB * KB, threads, [&](int64_t blk) {
    const int64_t g = blk / (static_cast<int64_t>(NB) * KB);
    const int nb = static_cast<int>((blk / KB) % NB);
    const int kb = static_cast<int>(blk % KB);
    const int n0 = nb * kBlock;
    const int n1 = std::min(N, n0 + kBlock);
    std::vector<float> vals;
    vals.reserve(static_cast<size_t>(kBlock) * kBlock);
    for (int n = n0; n < n1; ++n) {
      const int64_t base = (g * N + n) * K + static_cast<int64_t>(kb) * kBlock;
      for (int i = 0; i < kBlock; ++i) vals.push_back(bf16_to_float(x[base + i]));
    }
    std::vector<uint8_t> codes;
    s[blk] = quantize_group(vals, codes, ue8m0);
    size_t j = 0;
    for (int n = n0; n < n1; ++n) {
      const int64_t base = (g * N + n) * K + static_cast<int64_t>(kb) * kBlock;
      std::memcpy(q + base, codes.data() + j, kBlock);
      j += kBlock;
    }
  });
  return 0;
}

// bf16 bits of a float, round to nearest with ties to even (IEEE 754
// binary32 -> bfloat16: keep the upper 16 bits after adding half a unit in
// the last kept place, plus one if that place is odd). NaN stays NaN (quiet,
// sign kept).
uint16_t float_to_bf16_rne(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
    return static_cast<uint16_t>((u >> 16) | 0x0040u);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return static_cast<uint16_t>(u >> 16);
}

// Weight dequantization, the third kernel of the FP8 trio (quantize,
// dequantize, GEMM; DeepSeek-V3 review "28.5 倍压缩 + 1/10 成本",
// "创新之处" item 4 and "可复用的模式与技巧" item 3): every code times the
// fp32 scale of its 128x128 block. Reading taken: the product dec(q) * s is
// rounded once in fp32 and then to bf16, both round to nearest even.
// q [G][N][K], s [G][ceil(N/128)][K/128], x (bf16 bits) [G][N][K].
int oracle_per_block_dequant(const uint8_t* q, const float* s, uint16_t* x, int G, int N, int K,
                             int threads) {
  if (G < 0 || N < 0 || K <= 0 || K % kBlock != 0) return -1;
  const int KB = K / kBlock;
  const int NB = (N + kBlock - 1) / kBlock;
  parallel_for(static_cast<int64_t>(G) * N, threads, [&](int64_t row) {
    const int64_t g = row / N;
    const int n = static_cast<int>(row % N);
    const float* srow = s + (g * NB + n / kBlock) * KB;
    for (int k = 0; k < K; ++k) {
      const float v = static_cast<float>(table().value[q[row * K + k]]) * srow[k / kBlock];
      x[row * K + k] = float_to_bf16_rne(v);
    }
  });
  return 0;
}

// Dense GEMM, D = (A*sa)(B*sb)^T in fp64.
// qa [M][K], sa [M][K/128], qb [N][K], sb [ceil(N/128)][K/128], out [M][N].
int oracle_gemm_nt(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                   double* out, int M, int N, int K, int threads) {
  if (M < 0 || N < 0 || K <= 0 || K % kBlock != 0) return -1;
  const int KB = K / kBlock;
  parallel_for(M, threads, [&](int64_t m) {
    for (int n = 0; n < N; ++n) {
      out[m * N + n] = dot_blocked(qa + m * K, sa + m * KB, qb + static_cast<int64_t>(n) * K,
                                   sb + static_cast<int64_t>(n / kBlock) * KB, K);
    }
  });
  return 0;
}

// MoE grouped GEMM, contiguous layout: row m of A uses expert m_indices[m]'s
// weights; rows with m_indices[m] < 0 are padding and come out as NaN
// (undefined). qa [M_total][K], sa [M_total][K/128], qb [G][N][K],
// sb [G][ceil(N/128)][K/128], out [M_total][N].
int oracle_grouped_contiguous(const uint8_t* qa, const float* sa, const uint8_t* qb,
                              const float* sb, const int32_t* m_indices, double* out,
                              int M_total, int N, int K, int G, int threads) {
  if (M_total < 0 || N < 0 || G <= 0 || K <= 0 || K % kBlock != 0) return -1;
  const int KB = K / kBlock;
  const int NB = (N + kBlock - 1) / kBlock;
  for (int m = 0; m < M_total; ++m)
    if (m_indices[m] >= G) return -1;
  parallel_for(M_total, threads, [&](int64_t m) {
    const int g = m_indices[m];
    for (int n = 0; n < N; ++n) {
      if (g < 0) {
        out[m * N + n] = std::numeric_limits<double>::quiet_NaN();
        continue;
      }
      const uint8_t* brow = qb + (static_cast<int64_t>(g) * N + n) * K;
      const float* srow = sb + (static_cast<int64_t>(g) * NB + n / kBlock) * KB;
      out[m * N + n] = dot_blocked(qa + m * K, sa + m * KB, brow, srow, K);
    }
  });
  return 0;
}

// MoE grouped GEMM, masked layout: expert e owns rows [0, masked_m[e]) of its
// M_max-row slab; the other rows come out as NaN (undefined).
// qa [G][M_max][K], sa [G][M_max][K/128], qb [G][N][K], sb [G][ceil(N/128)][K/128],
// out [G][M_max][N].
int oracle_grouped_masked(const uint8_t* qa, const float* sa, const uint8_t* qb,
                          const float* sb, const int32_t* masked_m, double* out, int G,
                          int M_max, int N, int K, int threads) {
  if (G <= 0 || M_max < 0 || N < 0 || K <= 0 || K % kBlock != 0) return -1;
  for (int e = 0; e < G; ++e)
    if (masked_m[e] < 0 || masked_m[e] > M_max) return -1;
  const int KB = K / kBlock;
  const int NB = (N + kBlock - 1) / kBlock;
  parallel_for(static_cast<int64_t>(G) * M_max, threads, [&](int64_t row) {
    const int e = static_cast<int>(row / M_max);
    const int m = static_cast<int>(row % M_max);
    for (int n = 0; n < N; ++n) {
      if (m >= masked_m[e]) {
        out[row * N + n] = std::numeric_limits<double>::quiet_NaN();
        continue;
      }
      const uint8_t* brow = qb + (static_cast<int64_t>(e) * N + n) * K;
      const float* srow = sb + (static_cast<int64_t>(e) * NB + n / kBlock) * KB;
      out[row * N + n] = dot_blocked(qa + row * K, sa + row * KB, brow, srow, K);
    }
  });
  return 0;
}

// Selected output elements of any of the three forms: element p is row
// a_row[p] of qa/sa against row n[p] of expert e[p]'s weights.
// qa [*][K], sa [*][K/128], qb [G][N][K], sb [G][ceil(N/128)][K/128].
int oracle_gemm_points(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                       const int64_t* a_row, const int64_t* e, const int64_t* n, int64_t P,
                       double* out, int N, int K, int G, int threads) {
  if (N <= 0 || G <= 0 || K <= 0 || K % kBlock != 0 || P < 0) return -1;
  for (int64_t p = 0; p < P; ++p)
    if (e[p] < 0 || e[p] >= G || n[p] < 0 || n[p] >= N || a_row[p] < 0) return -1;
  const int KB = K / kBlock;
  const int NB = (N + kBlock - 1) / kBlock;
  parallel_for(P, threads, [&](int64_t p) {
    const uint8_t* brow = qb + (e[p] * N + n[p]) * K;
    const float* srow = sb + (e[p] * NB + n[p] / kBlock) * KB;
    out[p] = dot_blocked(qa + a_row[p] * K, sa + a_row[p] * KB, brow, srow, K);
  });
  return 0;
}

// K-grouped GEMM. qa: e4m3 [M][T]; sa: fp32 [M][T/128]; qb: e4m3 [N][T];
// sb: fp32 [N][T/128]; ks: int32 [G] token counts (multiples of 128, summing
// to T); out: fp64 [G][M][N]. Returns 0, or -1 on bad sizes or counts.
int oracle_k_grouped(const uint8_t* qa, const float* sa, const uint8_t* qb, const float* sb,
                     const int32_t* ks, double* out, int G, int M, int N, int T, int threads) {
  if (G < 1 || M < 0 || N < 0 || T < 0 || T % kBlock != 0) return -1;
  int64_t total = 0;
  for (int e = 0; e < G; ++e) {
    if (ks[e] < 0 || ks[e] % kBlock != 0) return -1;
    total += ks[e];
  }
  if (total != T) return -1;
  const int TB = T / kBlock;
  int64_t t0 = 0;
  for (int e = 0; e < G; ++e) {
    const int64_t tb0 = t0 / kBlock;
    const int len = ks[e];
    double* oe = out + static_cast<int64_t>(e) * M * N;
    parallel_for(M, threads, [&](int64_t m) {
      for (int n = 0; n < N; ++n) {
        oe[m * N + n] = len == 0 ? 0.0
                                 : dot_blocked(qa + m * T + t0, sa + m * TB + tb0,
                                               qb + static_cast<int64_t>(n) * T + t0,
                                               sb + static_cast<int64_t>(n) * TB + tb0, len);
      }
    });
    t0 += len;
  }
  return 0;
}

float oracle_exp_f32(float x) { return exp_f32(x); }
float oracle_silu_f32(float g) { return silu_f32(g); }

// h = bf16(silu(g) * u) elementwise; g, u, h bf16 bit patterns.
void oracle_swiglu(const uint16_t* g, const uint16_t* u, uint16_t* h, int64_t n) {
  for (int64_t i = 0; i < n; ++i)
    h[i] = float_to_bf16_rne(silu_f32(bf16_to_float(g[i])) * bf16_to_float(u[i]));
}

// bf16 nearest-even rounding of fp64 values (one rounding from the exact
// value; magnitudes beyond the largest finite bf16 round to infinity).
void oracle_f64_to_bf16(const double* v, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) {
    const double x = v[i];
    if (std::isnan(x)) {
      out[i] = 0x7FC0;
      continue;
    }
    const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
    const double a = std::fabs(x);
    if (a == 0.0) {
      out[i] = sign;
      continue;
    }
    // spacing of bf16 values at a's binade (subnormals share the smallest)
    int e;
    std::frexp(a, &e);                 // a = f * 2^e, f in [0.5, 1)
    int q = std::max(e - 8, -133);     // bf16: 8 significant bits; subnormal spacing 2^-133
    const double unit = std::ldexp(1.0, q);
    const double m = a / unit;         // exact (power-of-two scaling)
    double r = std::nearbyint(m);      // ties to even (default rounding mode)
    const double y = r * unit;
    const float f = y > 3.3895313892515355e38 ? std::numeric_limits<float>::infinity()
                                              : static_cast<float>(y);  // exact: <= 8 significant bits
    uint32_t b;
    std::memcpy(&b, &f, 4);
    out[i] = static_cast<uint16_t>(sign | ((b >> 16) & 0x7FFF));
  }
}

int oracle_hardware_threads(void) {
  return static_cast<int>(std::max(1u, std::thread::hardware_concurrency()));
}

}  // extern "C"
