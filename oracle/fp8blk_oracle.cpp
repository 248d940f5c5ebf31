// CPU oracle for the block-FP8 linear layer. TEST INFRASTRUCTURE ONLY.
//
// Only the tests, the smoke check and the benchmark's CPU-baseline leg may
// load this library. The product path (the CUDA library) never calls it and
// shares no code with it: not a header, a table or a helper. It is written to
// be read against the definitions, not to be fast: plain loops, one element
// at a time, products summed in double precision.
//
// What it computes follows FastVideo PR #1829 ("MiniMax H3: block-FP8 text
// encoder on Hopper, its converter, and a 4xH100 FastH3 profile"):
//   * section "Changes", converter bullet: weights are E4M3 codes plus one
//     float weight_scale_inv per 128x128 block, grid [N/128, K/128];
//   * section "Purpose": each linear multiplies the activations by the
//     dequantized weight, which the page states is the same computation the
//     Blackwell groupwise GEMM carries out inside;
//   * section "Changes", tests bullet: the dequantizer equals the scale
//     broadcast over its block times the code.
// Steps the page leaves open are read as follows: scale_inv = amax / 448 in float; a code is E4M3(W / s) with
// a float division, round-to-nearest-even and saturation to +-448; an
// all-zero block gets s = 0 and sign-preserving zero codes; the scale grid is
// ceil-divided and amax covers in-bounds elements only; activations use
// 1 x 128 K-groups with the same recipe; E4M3 is OCP E4M3FN (bias 7, no
// infinities, 0x7F/0xFF are NaN, max 448).
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math (SSE float arithmetic, so
// each float operation is one IEEE-754 correctly rounded operation).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- E4M3 codec
// OCP 8-bit floating point specification (OFP8), E4M3 variant: sign bit,
// 4 exponent bits with bias 7, 3 mantissa bits. Exponent field 0 encodes
// subnormals m/8 * 2^-6; S.1111.111 is NaN; there is no infinity.
double e4m3_value_from_fields(int code) {
  const int sign = (code >> 7) & 1;
  const int e = (code >> 3) & 0xF;
  const int m = code & 0x7;
  if (e == 0xF && m == 0x7) return std::nan("");
  double mag = (e == 0) ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -mag : mag;
}

struct E4M3Table {
  double v[256];
  E4M3Table() {
    for (int c = 0; c < 256; ++c) v[c] = e4m3_value_from_fields(c);
  }
};
const E4M3Table& table() {
  static const E4M3Table t;
  return t;
}

// Encode by search: saturate the magnitude to 448, take the nearest finite
// non-negative table value (codes 0x00..0x7E are increasing in value), break
// an exact tie towards the code whose mantissa LSB (= code bit 0) is 0, and
// put the input's sign bit on the result (so -0 and tiny negatives give 0x80).
uint8_t e4m3_encode_search(float f) {
  if (std::isnan(f)) return 0x7F;
  const double* T = table().v;
  double a = std::fabs(static_cast<double>(f));
  if (a > 448.0) a = 448.0;
  // smallest code c in [0, 0x7E] with T[c] >= a
  int lo = 0, hi = 0x7E;
  while (lo < hi) {
    int mid = (lo + hi) / 2;
    if (T[mid] >= a) hi = mid; else lo = mid + 1;
  }
  int c = lo;
  if (c > 0) {
    double up = T[c] - a, down = a - T[c - 1];
    if (down < up || (down == up && ((c - 1) & 1) == 0)) c = c - 1;
  }
  return static_cast<uint8_t>(c | (std::signbit(f) ? 0x80 : 0x00));
}

// Independent encoder working on the float's bit fields (no table): used only
// to cross-check the search encoder over every float bit pattern.
uint8_t e4m3_encode_fields(float f) {
  uint32_t b;
  std::memcpy(&b, &f, 4);
  const uint32_t sign = (b >> 31) << 7;
  const uint32_t a = b & 0x7FFFFFFFu;
  if (a > 0x7F800000u) return 0x7F;                 // NaN
  if (a >= 0x43E00000u) return uint8_t(sign | 0x7E);  // >= 448 (and inf): saturate
  if (a >= 0x3C800000u) {                            // >= 2^-6: E4M3 normal range
    const uint32_t fexp = (a >> 23) - 127 + 7;       // 1..15
    const uint32_t mant = a & 0x7FFFFFu;
    uint32_t x = (fexp << 3) | (mant >> 20);
    const uint32_t rem = mant & 0xFFFFFu, half = 0x80000u;
    if (rem > half || (rem == half && (x & 1u))) x += 1;  // carry may bump exponent
    if (x > 0x7E) x = 0x7E;
    return uint8_t(sign | x);
  }
  // below 2^-6: the result is an integer multiple of 2^-9, i.e. code = RNE(a * 2^9)
  const uint32_t fe = a >> 23;
  if (fe == 0) return uint8_t(sign);  // float zero / subnormal (< 2^-126)
  const uint32_t sig = 0x800000u | (a & 0x7FFFFFu);  // value = sig * 2^(fe-150)
  const uint32_t r = 141u - fe;                       // value*2^9 = sig >> r (r >= 21)
  if (r >= 32) return uint8_t(sign);
  uint32_t q = sig >> r;
  const uint32_t rem = sig & ((1u << r) - 1u), half = 1u << (r - 1u);
  if (rem > half || (rem == half && (q & 1u))) q += 1;
  return uint8_t(sign | q);
}

// ------------------------------------------------------------- BF16 helpers
float bf16_to_float(uint16_t h) {
  uint32_t b = uint32_t(h) << 16;
  float f;
  std::memcpy(&f, &b, 4);
  return f;
}

// float -> bfloat16, round to nearest, ties to even; NaN stays a quiet NaN.
uint16_t float_to_bf16_rne(float f) {
  uint32_t b;
  std::memcpy(&b, &f, 4);
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return uint16_t((b >> 16) | 0x40u);
  const uint32_t lsb = (b >> 16) & 1u;
  b += 0x7FFFu + lsb;
  return uint16_t(b >> 16);
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

template <class F>
void parallel_for(int64_t n, int nthreads, F fn) {
  if (nthreads < 1) nthreads = 1;
  if (n < nthreads) nthreads = int(n > 0 ? n : 1);
  if (nthreads == 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::vector<std::thread> th;
  for (int t = 0; t < nthreads; ++t)
    th.emplace_back([=] {
      for (int64_t i = t; i < n; i += nthreads) fn(i);
    });
  for (auto& x : th) x.join();
}

// One block-scaled group: amax over the in-bounds elements, s = amax / 448,
// codes = E4M3(v / s). Used for a 128x128 weight block and for a 1x128
// activation group alike (the recipe is the same; only the extent differs).
void quantize_group(const uint16_t* src, int64_t ld_src, int64_t rows, int64_t cols,
                    uint8_t* dst, int64_t ld_dst, float* scale_out) {
  float amax = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      float a = std::fabs(bf16_to_float(src[r * ld_src + c]));
      if (a > amax) amax = a;
    }
  const float s = amax / 448.0f;
  *scale_out = s;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      const float v = bf16_to_float(src[r * ld_src + c]);
      uint8_t code;
      if (amax == 0.0f)
        code = std::signbit(v) ? 0x80 : 0x00;
      else
        code = e4m3_encode_search(v / s);
      dst[r * ld_dst + c] = code;
    }
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------- codec API
void orc_e4m3_table(double* out256) {
  for (int c = 0; c < 256; ++c) out256[c] = table().v[c];
}

uint8_t orc_e4m3_encode(float f) { return e4m3_encode_search(f); }
uint8_t orc_e4m3_encode_fields(float f) { return e4m3_encode_fields(f); }
uint16_t orc_bf16_rne(float f) { return float_to_bf16_rne(f); }

void orc_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode_search(v[i]);
}

void orc_bf16_rne_array(const float* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = float_to_bf16_rne(v[i]);
}

// Number of float bit patterns in [lo, hi) where the two encoders disagree.
// `planted` is a test hook: at that bit pattern the bit-field encoder's code
// is taken with its lowest bit flipped, so a test can check that one planted
// disagreement is counted exactly once (no bit pattern equals the default,
// which is above 2^32).
static int64_t crosscheck_encoders(uint64_t lo, uint64_t hi, uint64_t planted, int nthreads) {
  if (hi <= lo) return 0;
  const uint64_t chunk = 1ull << 20;
  const int64_t nchunks = int64_t((hi - lo + chunk - 1) / chunk);
  std::vector<int64_t> bad(size_t(nchunks), 0);
  parallel_for(nchunks, nthreads, [&](int64_t ci) {
    uint64_t a = lo + uint64_t(ci) * chunk, b = a + chunk < hi ? a + chunk : hi;
    int64_t cnt = 0;
    for (uint64_t u = a; u < b; ++u) {
      uint32_t bits = uint32_t(u);
      float f;
      std::memcpy(&f, &bits, 4);
      uint8_t by_fields = e4m3_encode_fields(f);
      if (u == planted) by_fields ^= 1u;
      cnt += e4m3_encode_search(f) != by_fields;
    }
    bad[size_t(ci)] = cnt;
  });
  int64_t total = 0;
  for (auto c : bad) total += c;
  return total;
}

int64_t orc_crosscheck_encoders(uint64_t lo, uint64_t hi, int nthreads) {
  return crosscheck_encoders(lo, hi, ~0ull, nthreads);
}

int64_t orc_crosscheck_encoders_planted(uint64_t lo, uint64_t hi, uint64_t planted, int nthreads) {
  return crosscheck_encoders(lo, hi, planted, nthreads);
}

// Mismatches between given codes and the oracle's encoding of the float bit
// patterns lo, lo+1, ..., lo+n-1 (for checking a device codec in chunks).
int64_t orc_count_code_mismatches(uint64_t lo, int64_t n, const uint8_t* codes, int nthreads) {
  const int64_t chunk = 1 << 20;
  const int64_t nchunks = (n + chunk - 1) / chunk;
  std::vector<int64_t> bad(size_t(nchunks > 0 ? nchunks : 1), 0);
  parallel_for(nchunks, nthreads, [&](int64_t ci) {
    int64_t a = ci * chunk, b = a + chunk < n ? a + chunk : n, cnt = 0;
    for (int64_t i = a; i < b; ++i) {
      uint32_t bits = uint32_t(lo + uint64_t(i));
      float f;
      std::memcpy(&f, &bits, 4);
      cnt += e4m3_encode_fields(f) != codes[i];
    }
    bad[size_t(ci)] = cnt;
  });
  int64_t total = 0;
  for (auto c : bad) total += c;
  return total;
}

// ----------------------------------------------------- (a1) weight converter
// FastVideo PR #1829, "Changes", converter bullet: the checkpoint holds the
// E4M3 codes and a float weight_scale_inv grid of shape [N/128, K/128]. w is BF16 [N][ldw]; q is [N][ldq];
// scale_inv is dense [ceil(N/128)][ceil(K/128)].
void orc_quantize_weight(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q,
                         int64_t ldq, float* scale_inv, int nthreads) {
  const int64_t NB = cdiv(N, 128), KB = cdiv(K, 128);
  parallel_for(NB * KB, nthreads, [&](int64_t b) {
    const int64_t nb = b / KB, kb = b % KB;
    const int64_t n0 = nb * 128, k0 = kb * 128;
    const int64_t rows = (N - n0) < 128 ? (N - n0) : 128;
    const int64_t cols = (K - k0) < 128 ? (K - k0) : 128;
    quantize_group(w + n0 * ldw + k0, ldw, rows, cols, q + n0 * ldq + k0, ldq,
                   &scale_inv[nb * KB + kb]);
  });
}

// ------------------------------------------------------------ (a2) dequantize
// FastVideo PR #1829, "Purpose" and the tests bullet of "Changes": the code
// times its block's scale (the scale broadcast over the block), in float,
// rounded once to BF16.
void orc_dequantize(const uint8_t* q, int64_t ldq, const float* scale_inv, int64_t N, int64_t K,
                    uint16_t* w, int64_t ldw, int nthreads) {
  const int64_t KB = cdiv(K, 128);
  parallel_for(N, nthreads, [&](int64_t n) {
    for (int64_t k = 0; k < K; ++k) {
      const float code_value = float(table().v[q[n * ldq + k]]);
      const float s = scale_inv[(n / 128) * KB + (k / 128)];
      const float prod = code_value * s;
      w[n * ldw + k] = float_to_bf16_rne(prod);
    }
  });
}

// --------------------------------------------------- (a3) activation quantize
// The Blackwell route quantizes activations before the groupwise GEMM
// (FastVideo PR #1829, "Changes", loader bullet, which names a Triton
// activation quantizer for the Blackwell runtime).
// Groups are 1 x 128 along K with the weight recipe. sx is [M][ceil(K/128)].
void orc_act_quant(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, uint8_t* qx,
                   int64_t ldqx, float* sx, int nthreads) {
  const int64_t KB = cdiv(K, 128);
  parallel_for(M, nthreads, [&](int64_t m) {
    for (int64_t kb = 0; kb < KB; ++kb) {
      const int64_t k0 = kb * 128, cols = (K - k0) < 128 ? (K - k0) : 128;
      quantize_group(x + m * ldx + k0, ldx, 1, cols, qx + m * ldqx + k0, ldqx, &sx[m * KB + kb]);
    }
  });
}

// ------------------------------------------------- (a4..a7) linear, W8A16
// ref[i][n] = sum_k x[m][k] * E4M3(q[n][k]) * s[n/128][k/128] in double,
// m = rows[i] (rows == NULL: m = i, nrows = M). Products are exact in double.
void orc_linear_w8a16(const uint16_t* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                      const float* scale_inv, int64_t M, int64_t N, int64_t K, const int64_t* rows,
                      int64_t nrows, double* ref, int nthreads) {
  (void)M;
  const int64_t KB = cdiv(K, 128);
  const double* T = table().v;
  parallel_for(nrows, nthreads, [&](int64_t i) {
    const int64_t m = rows ? rows[i] : i;
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const double xv = double(bf16_to_float(x[m * ldx + k]));
        const double wv = T[q[n * ldq + k]] * double(scale_inv[(n / 128) * KB + (k / 128)]);
        acc += xv * wv;
      }
      ref[i * N + n] = acc;
    }
  });
}

// -------------------------------------------------- (a4..a7) linear, W8A8
// ref[i][n] = sum_kb sx[m][kb] * s[n/128][kb] * sum_{k in kb} E4M3(qx[m][k]) * E4M3(q[n][k]),
// in double (the inner sums of code products are exact in double).
void orc_linear_w8a8(const uint8_t* qx, int64_t ldqx, const float* sx, const uint8_t* q,
                     int64_t ldq, const float* scale_inv, int64_t M, int64_t N, int64_t K,
                     const int64_t* rows, int64_t nrows, double* ref, int nthreads) {
  (void)M;
  const int64_t KB = cdiv(K, 128);
  const double* T = table().v;
  parallel_for(nrows, nthreads, [&](int64_t i) {
    const int64_t m = rows ? rows[i] : i;
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t kb = 0; kb < KB; ++kb) {
        const int64_t k0 = kb * 128, k1 = (k0 + 128) < K ? (k0 + 128) : K;
        double part = 0.0;
        for (int64_t k = k0; k < k1; ++k) part += T[qx[m * ldqx + k]] * T[q[n * ldq + k]];
        acc += double(sx[m * KB + kb]) * double(scale_inv[(n / 128) * KB + kb]) * part;
      }
      ref[i * N + n] = acc;
    }
  });
}

}  // extern "C"
