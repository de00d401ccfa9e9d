// Plain CPU oracle of the fine-grained FP8 linear layer, in C++17.
//
// TEST INFRASTRUCTURE ONLY: built into oracle/liboracle.so and called from the
// tests, the smoke check and the CPU baseline of the benchmark. It shares no
// code, header or table with the CUDA library and includes nothing from it.
//
// What it computes, and where the pages say so (by page title and section):
//
//  * "FP8 à granularité fine" (Hugging Face transformers docs), opening
//    bullets: weights are quantized per 2-D block of 128 x 128
//    (weight_block_size=(128, 128)); activations per token in groups of 128
//    input channels. Section "Chemin rapide de DeepGEMM": the activation scales
//    are computed at run time (activation_scheme="dynamic"). Section "Format
//    d'échelle UE8M0": scale_fmt="float" keeps the scales as plain fp32.
//  * "Déployer la parcimonie 2:4 avec FP8 sur Hopper", pipeline steps 2, 4
//    and 6 and "Exemples pratiques 1": groups of 4 contiguous weights along
//    K, the two of largest magnitude kept, FP8 scales recomputed after
//    pruning. "Combiner élagage et quantification ...", section on 2:4
//    sparsity: keep the two largest of every 4.
//
// The readings taken where the pages are silent (each one is listed with its
// reason in the design notes):
//
//  * the 8-bit format is OCP FP8 E4M3 "fn" (bias 7, no infinities, largest
//    finite 448); conversion rounds to nearest, ties to even, and saturates
//    to +-448;
//  * scale s = fl32(amax / 448) with an IEEE fp32 division; element code =
//    e4m3(fl32(x / s)), one IEEE fp32 division then one rounding to E4M3;
//    amax == 0 gives s == 0 and every element encodes as a zero carrying the
//    element's sign;
//  * a ragged last row block of a weight (N % 128 != 0) takes its amax over
//    its valid rows only;
//  * 2:4 ties in magnitude go to the lower index; pruned positions become +0;
//  * the GEMM is Y[m,n] = sum_kb sA[m,kb] * sW[n/128,kb] * sum_{k in kb}
//    qA[m,k] * qW[n,k], evaluated here in double: each K-block partial is a
//    sum of 128 products of E4M3 values and is exact in double; the scale
//    product and the running sum over K-blocks are rounded to double in the
//    order written.
//
// Floating point: compiled without fast-math and with -ffp-contract=off, so
// every float and double operation is the IEEE operation written (no fused
// multiply-add, no flush to zero).
//
// Layouts are dense row-major: X, qA [M][K]; sA [M][K/128]; W, qW [N][K];
// sW [ceil(N/128)][K/128]; vals [N][K/2]; meta [N][K/8] (byte j holds group
// 2j in bits 0-3 and group 2j+1 in bits 4-7, each nibble = i0 | i1 << 2 with
// i0 < i1 the kept positions); Y [M][N] double.
//
// Work is spread over threads by independent outputs only (rows, blocks or
// output columns); no thread ever combines another thread's partial results,
// so the answer does not depend on the thread count.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

namespace {

constexpr int kGroup = 128;        // 1x128 activation groups, 128x128 weight blocks
constexpr double kE4M3Max = 448.0; // 1.75 * 2^8
constexpr float kE4M3MaxF = 448.0f;

std::atomic<int> g_threads{0};     // 0 = every hardware thread

int thread_count() {
  int t = g_threads.load();
  if (t <= 0) {
    t = static_cast<int>(std::thread::hardware_concurrency());
    if (t <= 0) t = 1;
  }
  return t;
}

// Run body(i) for i in [0, n), spread over the worker threads in contiguous
// chunks.
void parallel_for(int64_t n, const std::function<void(int64_t)>& body) {
  if (n <= 0) return;
  const int64_t t = std::min<int64_t>(thread_count(), n);
  if (t == 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  pool.reserve(static_cast<size_t>(t));
  for (int64_t w = 0; w < t; ++w) {
    const int64_t lo = n * w / t, hi = n * (w + 1) / t;
    pool.emplace_back([lo, hi, &body] {
      for (int64_t i = lo; i < hi; ++i) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------- E4M3 codec
// OCP 8-bit floating point, E4M3 ("fn"): sign bit, 4 exponent bits (bias 7),
// 3 mantissa bits. Exponent field 0 is subnormal: (m / 8) * 2^-6. Otherwise
// (1 + m / 8) * 2^(e - 7). S.1111.111 is NaN; there are no infinities.

double e4m3_value(uint8_t code) {
  const int s = code >> 7, e = (code >> 3) & 0xF, m = code & 0x7;
  if (e == 15 && m == 7) return std::nan("");
  const double mag = e == 0 ? std::ldexp(static_cast<double>(m), -9)
                            : (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
  return s ? -mag : mag;
}

// Round an fp32 value to E4M3: nearest, ties to even, saturating to +-448;
// the sign of zero is kept; NaN (outside the contract) gives 0x7F.
uint8_t e4m3_encode(float v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  double a = std::fabs(static_cast<double>(v));   // exact widening
  if (a > kE4M3Max) a = kE4M3Max;                  // saturation (Inf included)
  // Spacing of E4M3 values in the binade of a: 2^(floor(log2 a) - 3) for
  // normal magnitudes (>= 2^-6), 2^-9 below. Dividing by a power of two is
  // exact, so nearbyint (round half to even in the default rounding mode)
  // performs the one rounding.
  double step = std::ldexp(1.0, -9);
  if (a >= std::ldexp(1.0, -6)) {
    int ex = 0;
    std::frexp(a, &ex);                            // a = f * 2^ex, f in [0.5, 1)
    step = std::ldexp(1.0, ex - 1 - 3);
  }
  const double q = std::nearbyint(a / step) * step;   // <= 448, which is a code
  if (q == 0.0) return sign;
  if (q < std::ldexp(1.0, -6)) {                       // subnormal
    return static_cast<uint8_t>(sign | static_cast<int>(std::nearbyint(q / std::ldexp(1.0, -9))));
  }
  int ex = 0;
  std::frexp(q, &ex);
  const int e = ex - 1;                                // floor(log2 q)
  const int m = static_cast<int>(std::nearbyint((std::ldexp(q, -e) - 1.0) * 8.0));
  return static_cast<uint8_t>(sign | ((e + 7) << 3) | m);
}

// Codes of the elements x[0..n) against one scale s: e4m3(fl32(x / s)); a
// zero scale (an all-zero group or block) gives each element's signed zero.
uint8_t quantize_one(float x, float s) {
  if (s == 0.0f) return std::signbit(x) ? 0x80 : 0x00;
  const float ratio = x / s;                           // IEEE fp32 division
  return e4m3_encode(ratio);
}

// UE8M0 ("float8_e8m0fnu": 8 exponent bits, no sign, no mantissa): code c
// stands for 2^(c - 127); 0xFF is NaN. The scale of a group or block is the
// smallest power of two s with 448 * s >= amax, so no element saturates;
// amax == 0 (and any amax below 448 * 2^-127) takes the smallest code, 0.
int ue8m0_code_of_amax(float amax) {
  if (!(amax > 0.0f)) return 0;
  int e = 0;
  std::frexp(static_cast<double>(amax) / 448.0, &e);   // amax / 448 < 2^e (approximately)
  // settle e exactly: 448 * 2^e >= amax and 448 * 2^(e-1) < amax
  while (e > -127 && std::ldexp(448.0, e - 1) >= static_cast<double>(amax)) --e;
  while (std::ldexp(448.0, e) < static_cast<double>(amax)) ++e;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e + 127;
}

float ue8m0_scale(int code) { return static_cast<float>(std::ldexp(1.0, code - 127)); }

}  // namespace

extern "C" {

void orc_set_threads(int n) { g_threads.store(n); }

int orc_threads(void) { return thread_count(); }

void orc_e4m3_encode(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(v[i]);
}

void orc_e4m3_decode(const uint8_t* code, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_value(code[i]);
}

// Dynamic activation quantization, 1x128 groups along K: for token m and
// group g, sa[m][g] = fl32(max_{k in g} |x[m][k]| / 448) and
// qa[m][k] = e4m3(fl32(x[m][k] / sa[m][g])).
void orc_quant_act_group128(const float* x, int64_t M, int64_t K, uint8_t* qa, float* sa) {
  const int64_t KB = K / kGroup;
  parallel_for(M, [&](int64_t m) {
    for (int64_t g = 0; g < KB; ++g) {
      const float* xg = x + m * K + g * kGroup;
      float amax = 0.0f;
      for (int i = 0; i < kGroup; ++i) amax = std::max(amax, std::fabs(xg[i]));
      const float s = amax / kE4M3MaxF;                // IEEE fp32 division
      sa[m * KB + g] = s;
      for (int i = 0; i < kGroup; ++i) qa[m * K + g * kGroup + i] = quantize_one(xg[i], s);
    }
  });
}

// Weight quantization, 128x128 blocks: for block (nb, kb),
// sw[nb][kb] = fl32(max |w| over the block's valid rows / 448) and
// qw = e4m3(fl32(w / sw)).
void orc_quant_weight_block128(const float* w, int64_t N, int64_t K, uint8_t* qw, float* sw) {
  const int64_t KB = K / kGroup, NB = (N + kGroup - 1) / kGroup;
  parallel_for(NB * KB, [&](int64_t blk) {
    const int64_t nb = blk / KB, kb = blk % KB;
    const int64_t r0 = nb * kGroup, r1 = std::min<int64_t>(N, r0 + kGroup);
    float amax = 0.0f;
    for (int64_t r = r0; r < r1; ++r)
      for (int i = 0; i < kGroup; ++i) amax = std::max(amax, std::fabs(w[r * K + kb * kGroup + i]));
    const float s = amax / kE4M3MaxF;
    sw[nb * KB + kb] = s;
    for (int64_t r = r0; r < r1; ++r)
      for (int i = 0; i < kGroup; ++i) {
        const int64_t k = kb * kGroup + i;
        qw[r * K + k] = quantize_one(w[r * K + k], s);
      }
  });
}

// Kept positions of one group of 4: member i is kept when fewer than two
// others beat it; j beats i when |w_j| > |w_i|, or |w_j| == |w_i| and j < i
// (ties go to the lower index; +0 and -0 are equal). Exactly two are kept.
static void select24(const float* g, int* i0, int* i1) {
  int kept[2], nk = 0;
  for (int i = 0; i < 4; ++i) {
    int beaten = 0;
    for (int j = 0; j < 4; ++j) {
      if (j == i) continue;
      const float aj = std::fabs(g[j]), ai = std::fabs(g[i]);
      if (aj > ai || (aj == ai && j < i)) ++beaten;
    }
    if (beaten < 2) kept[nk++] = i;
  }
  *i0 = kept[0];
  *i1 = kept[1];
}

// 2:4 magnitude pruning along K, then 128x128 block quantization of the
// pruned matrix (scales recomputed after pruning), then compression: the two
// kept codes of each group in position order and one index nibble per group.
// w_pruned (may be null) receives the pruned weights as floats (bf16-exact).
void orc_prune24_compress(const float* w, int64_t N, int64_t K, uint8_t* vals, uint8_t* meta,
                          float* sw, float* w_pruned) {
  const int64_t G = K / 4;
  std::vector<float> wp(static_cast<size_t>(N * K));
  std::vector<uint8_t> sel(static_cast<size_t>(N * G * 2));   // kept positions i0, i1
  parallel_for(N, [&](int64_t n) {
    for (int64_t g = 0; g < G; ++g) {
      const float* grp = w + n * K + 4 * g;
      int i0 = 0, i1 = 0;
      select24(grp, &i0, &i1);
      sel[2 * (n * G + g)] = static_cast<uint8_t>(i0);
      sel[2 * (n * G + g) + 1] = static_cast<uint8_t>(i1);
      for (int i = 0; i < 4; ++i) wp[n * K + 4 * g + i] = (i == i0 || i == i1) ? grp[i] : 0.0f;
    }
  });
  std::vector<uint8_t> q(static_cast<size_t>(N * K));
  orc_quant_weight_block128(wp.data(), N, K, q.data(), sw);
  parallel_for(N, [&](int64_t n) {
    for (int64_t g = 0; g < G; ++g) {
      const int i0 = sel[2 * (n * G + g)], i1 = sel[2 * (n * G + g) + 1];
      vals[n * (K / 2) + 2 * g] = q[n * K + 4 * g + i0];
      vals[n * (K / 2) + 2 * g + 1] = q[n * K + 4 * g + i1];
      const uint8_t nib = static_cast<uint8_t>(i0 | (i1 << 2));
      uint8_t& byte = meta[n * (K / 8) + g / 2];
      if (g % 2 == 0) byte = nib;
      else byte = static_cast<uint8_t>(byte | (nib << 4));
    }
    if (w_pruned) std::memcpy(w_pruned + n * K, wp.data() + n * K, sizeof(float) * K);
  });
}

// Dense codes [N][K] from the compressed form: the kept codes at positions
// i0, i1 of every group of 4, code 0x00 (+0) at the two pruned positions.
void orc_decompress24(const uint8_t* vals, const uint8_t* meta, int64_t N, int64_t K, uint8_t* q) {
  const int64_t G = K / 4;
  parallel_for(N, [&](int64_t n) {
    for (int64_t g = 0; g < G; ++g) {
      const uint8_t byte = meta[n * (K / 8) + g / 2];
      const int nib = g % 2 == 0 ? (byte & 0xF) : (byte >> 4);
      const int i0 = nib & 3, i1 = nib >> 2;
      uint8_t* dst = q + n * K + 4 * g;
      dst[0] = dst[1] = dst[2] = dst[3] = 0;
      dst[i0] = vals[n * (K / 2) + 2 * g];
      dst[i1] = vals[n * (K / 2) + 2 * g + 1];
    }
  });
}

// Value of UE8M0 scale codes as fp32 (2^(c - 127), exact; NaN for 0xFF).
void orc_ue8m0_decode(const uint8_t* code, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i)
    out[i] = code[i] == 0xFF ? std::nanf("") : ue8m0_scale(code[i]);
}

// UE8M0 scale codes of the given amax values.
void orc_ue8m0_of_amax(const float* amax, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = static_cast<uint8_t>(ue8m0_code_of_amax(amax[i]));
}

// The UE8M0 variant of the activation quantizer: per 1x128 group the scale
// is the power of two 2^(c - 127) of ue8m0_code_of_amax(amax), stored as its
// code sa8[m][g]; the elements are e4m3(fl32(x / s)) as before.
void orc_quant_act_group128_ue8m0(const float* x, int64_t M, int64_t K, uint8_t* qa,
                                  uint8_t* sa8) {
  const int64_t KB = K / kGroup;
  parallel_for(M, [&](int64_t m) {
    for (int64_t g = 0; g < KB; ++g) {
      const float* xg = x + m * K + g * kGroup;
      float amax = 0.0f;
      for (int i = 0; i < kGroup; ++i) amax = std::max(amax, std::fabs(xg[i]));
      const int c = ue8m0_code_of_amax(amax);
      sa8[m * KB + g] = static_cast<uint8_t>(c);
      const float s = ue8m0_scale(c);
      for (int i = 0; i < kGroup; ++i) qa[m * K + g * kGroup + i] = quantize_one(xg[i], s);
    }
  });
}

// The UE8M0 variant of the weight quantizer (128x128 blocks, ragged last row
// block over its valid rows).
void orc_quant_weight_block128_ue8m0(const float* w, int64_t N, int64_t K, uint8_t* qw,
                                     uint8_t* sw8) {
  const int64_t KB = K / kGroup, NB = (N + kGroup - 1) / kGroup;
  parallel_for(NB * KB, [&](int64_t blk) {
    const int64_t nb = blk / KB, kb = blk % KB;
    const int64_t r0 = nb * kGroup, r1 = std::min<int64_t>(N, r0 + kGroup);
    float amax = 0.0f;
    for (int64_t r = r0; r < r1; ++r)
      for (int i = 0; i < kGroup; ++i) amax = std::max(amax, std::fabs(w[r * K + kb * kGroup + i]));
    const int c = ue8m0_code_of_amax(amax);
    sw8[nb * KB + kb] = static_cast<uint8_t>(c);
    const float s = ue8m0_scale(c);
    for (int64_t r = r0; r < r1; ++r)
      for (int i = 0; i < kGroup; ++i) {
        const int64_t k = kb * kGroup + i;
        qw[r * K + k] = quantize_one(w[r * K + k], s);
      }
  });
}

// The block-scaled GEMM, one 128-deep K-block at a time:
//   y[m][j] = sum_kb (sa[m][kb] * sw[n/128][kb]) * sum_{k in kb} a[m][k] * w[n][k]
// for the weight rows n = cols[j] (all rows, n = j, when cols is null); a, w
// the E4M3 values of the codes. Output y [M][ncols] in double.
void orc_block_gemm(const uint8_t* qa, const float* sa, int64_t M, const uint8_t* qw,
                    const float* sw, int64_t N, int64_t K, const int64_t* cols, int64_t ncols,
                    double* y) {
  const int64_t KB = K / kGroup;
  (void)N;
  double table[256];
  for (int c = 0; c < 256; ++c) table[c] = e4m3_value(static_cast<uint8_t>(c));
  parallel_for(ncols, [&](int64_t j) {
    const int64_t n = cols ? cols[j] : j;
    const uint8_t* wrow = qw + n * K;
    const float* srow = sw + (n / kGroup) * KB;
    for (int64_t m = 0; m < M; ++m) {
      const uint8_t* arow = qa + m * K;
      double acc = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        double partial = 0.0;   // exact: 128 products of E4M3 values
        for (int i = 0; i < kGroup; ++i) {
          const int64_t k = kb * kGroup + i;
          partial += table[arow[k]] * table[wrow[k]];
        }
        const double scale = static_cast<double>(sa[m * KB + kb]) * static_cast<double>(srow[kb]);
        acc += scale * partial;
      }
      y[m * ncols + j] = acc;
    }
  });
}

// The same GEMM with the weights in 2:4 compressed form: each weight row used
// is rebuilt by decompression, then multiplied as above.
void orc_sparse24_gemm(const uint8_t* qa, const float* sa, int64_t M, const uint8_t* vals,
                       const uint8_t* meta, const float* sw, int64_t N, int64_t K,
                       const int64_t* cols, int64_t ncols, double* y) {
  std::vector<uint8_t> qw(static_cast<size_t>(ncols * K));
  std::vector<int64_t> rows(static_cast<size_t>(ncols));
  for (int64_t j = 0; j < ncols; ++j) rows[j] = cols ? cols[j] : j;
  // decompress the used rows one by one into a compact [ncols][K] matrix
  parallel_for(ncols, [&](int64_t j) {
    orc_decompress24(vals + rows[j] * (K / 2), meta + rows[j] * (K / 8), 1, K,
                     qw.data() + j * K);
  });
  // each compact row j keeps the scale row of its original row
  const int64_t KB = K / kGroup;
  std::vector<float> swj(static_cast<size_t>(ncols * KB));
  for (int64_t j = 0; j < ncols; ++j)
    for (int64_t kb = 0; kb < KB; ++kb) swj[j * KB + kb] = sw[(rows[j] / kGroup) * KB + kb];
  // multiply row j of the compact matrix with its own scale row: a weight
  // "block" of one row
  double table[256];
  for (int c = 0; c < 256; ++c) table[c] = e4m3_value(static_cast<uint8_t>(c));
  (void)N;
  parallel_for(ncols, [&](int64_t j) {
    const uint8_t* wrow = qw.data() + j * K;
    const float* srow = swj.data() + j * KB;
    for (int64_t m = 0; m < M; ++m) {
      const uint8_t* arow = qa + m * K;
      double acc = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        double partial = 0.0;
        for (int i = 0; i < kGroup; ++i) {
          const int64_t k = kb * kGroup + i;
          partial += table[arow[k]] * table[wrow[k]];
        }
        const double scale = static_cast<double>(sa[m * KB + kb]) * static_cast<double>(srow[kb]);
        acc += scale * partial;
      }
      y[m * ncols + j] = acc;
    }
  });
}

// The grouped (mixture-of-experts) GEMM: row m of the tokens is multiplied by
// the weights of its expert e = m_indices[m] (weights [E][N][K], scales
// [E][ceil(N/128)][K/128]) with the block-scaled formula above; rows with
// e outside [0, E) (padding) get NaN, i.e. no defined result.
void orc_grouped_gemm(const uint8_t* qa, const float* sa, int64_t M, const uint8_t* qw,
                      const float* sw, const int32_t* m_indices, int64_t E, int64_t N, int64_t K,
                      double* y) {
  const int64_t KB = K / kGroup, NB = (N + kGroup - 1) / kGroup;
  double table[256];
  for (int c = 0; c < 256; ++c) table[c] = e4m3_value(static_cast<uint8_t>(c));
  parallel_for(M, [&](int64_t m) {
    const int64_t e = m_indices[m];
    for (int64_t n = 0; n < N; ++n) {
      if (e < 0 || e >= E) {
        y[m * N + n] = std::nan("");
        continue;
      }
      const uint8_t* wrow = qw + (e * N + n) * K;
      const float* srow = sw + (e * NB + n / kGroup) * KB;
      const uint8_t* arow = qa + m * K;
      double acc = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        double partial = 0.0;
        for (int i = 0; i < kGroup; ++i) {
          const int64_t k = kb * kGroup + i;
          partial += table[arow[k]] * table[wrow[k]];
        }
        const double scale = static_cast<double>(sa[m * KB + kb]) * static_cast<double>(srow[kb]);
        acc += scale * partial;
      }
      y[m * N + n] = acc;
    }
  });
}

// SwiGLU of the gated MLP: h = silu(g) * u with silu(g) = g / (1 + e^-g),
// in double (g, u the gate and up outputs of the GEMM).
void orc_swiglu(const double* g, const double* u, int64_t n, double* h) {
  for (int64_t i = 0; i < n; ++i) h[i] = g[i] / (1.0 + std::exp(-g[i])) * u[i];
}

// Tolerance of h given tolerances tg, tu of g and u: silu has a slope of
// magnitude below 1.1 everywhere (its derivative sigma(g) (1 + g (1 -
// sigma(g))) lies in (-0.11, 1.1)), so
//   |h - h_ref| <= 1.1 tg (|u| + tu) + |silu(g)| tu + 1e-5 |h|
// with the last term for the fp32 evaluation of silu and the product.
void orc_swiglu_bound(const double* g, const double* u, const double* tg, const double* tu,
                      int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) {
    const double sg = g[i] / (1.0 + std::exp(-g[i]));
    out[i] = 1.1 * tg[i] * (std::fabs(u[i]) + tu[i]) + std::fabs(sg) * tu[i] +
             1e-5 * std::fabs(sg * u[i]);
  }
}

// The magnitude sum behind the GEMM's error bound:
//   S[m][j] = sum_k |a[m][k] * sa[m][k/128]| * |w[n][k] * sw[n/128][k/128]|
// for n = cols[j] (all rows when null), the dequantized operands in double.
void orc_gemm_abs_sum(const uint8_t* qa, const float* sa, int64_t M, const uint8_t* qw,
                      const float* sw, int64_t N, int64_t K, const int64_t* cols, int64_t ncols,
                      double* out) {
  const int64_t KB = K / kGroup;
  (void)N;
  double table[256];
  for (int c = 0; c < 256; ++c) table[c] = std::fabs(e4m3_value(static_cast<uint8_t>(c)));
  parallel_for(ncols, [&](int64_t j) {
    const int64_t n = cols ? cols[j] : j;
    const uint8_t* wrow = qw + n * K;
    const float* srow = sw + (n / kGroup) * KB;
    for (int64_t m = 0; m < M; ++m) {
      const uint8_t* arow = qa + m * K;
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const double a = table[arow[k]] * static_cast<double>(std::fabs(sa[m * KB + k / kGroup]));
        const double w = table[wrow[k]] * static_cast<double>(std::fabs(srow[k / kGroup]));
        acc += a * w;
      }
      out[m * ncols + j] = acc;
    }
  });
}

}  // extern "C"
