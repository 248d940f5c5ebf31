// Elementwise stages of the block-FP8 linear: the weight converter, the
// dequantizer, the 1 x 128 activation quantizer and the bare E4M3 codec.
// All are HBM-bound streams: 16-byte vector loads and stores, one pass over
// the data (the converter keeps its 128 x 128 block in registers between the
// amax reduction and the encoding).
#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {
namespace {

// Per-halfword |bf16| maximum. For non-NaN values the magnitude order equals
// the unsigned order of (bits & 0x7FFF), so integer maxima give the exact amax.
__device__ __forceinline__ uint32_t absmax2(uint32_t acc, uint32_t w) {
  return __vmaxu2(acc, w & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t absmax_u4(uint32_t acc, const uint4& v) {
  acc = absmax2(acc, v.x);
  acc = absmax2(acc, v.y);
  acc = absmax2(acc, v.z);
  return absmax2(acc, v.w);
}

// The codes are E4M3(RN_f32(v / d)): the float quotient (IEEE division,
// round to nearest even) rounded again to E4M3 with saturation.
//
// Division is the converter's costliest step, so when d >= 2^-125 a cheaper
// route gives the same codes: with y = RN(1 / d), q = RN(v * y) lies within a
// few float ulps of RN(v / d). E4M3 rounding can only tell them apart near one
// of its decision points -- floats whose low 20 mantissa bits are 0x80000
// (midpoints of the 3-bit mantissa grid) -- or in E4M3's subnormal range;
// when any element of a warp's chunk is there (|low20 - 0x80000| <= 16 ulps,
// or 0 < |q| < 2^-5) the whole chunk takes the exact quotient instead (a
// warp-uniform branch; rare for real data). Checked exhaustively against the
// exact quotient over every BF16 value v and every BF16 block maximum
// (d = amax / 448).
__device__ __forceinline__ bool near_e4m3_decision(float q) {
  const uint32_t b = __float_as_uint(q) & 0x7FFFFFFFu;
  return b != 0u && (b < 0x3D000000u || ((b & 0xFFFFFu) - 0x7FFF0u) <= 0x20u);
}

// Eight BF16 values -> eight E4M3 codes of RN_f32(v / d) (code i in byte i).
// All 32 lanes of the warp must call this together.
__device__ __forceinline__ uint2 encode8(const uint4& v, float d) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = bf16_lo_to_f32(w[i]);
    f[2 * i + 1] = bf16_hi_to_f32(w[i]);
  }
  float q[8];
  bool exact = d < 2.35098870e-38f;  // 2^-125: 1/d would not be a finite normal
  if (!exact) {
    const float y = __frcp_rn(d);
    bool near = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      q[i] = __fmul_rn(f[i], y);
      near |= near_e4m3_decision(q[i]);
    }
    exact = __any_sync(0xFFFFFFFFu, near);
  }
  if (exact) {
#pragma unroll
    for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(f[i], d);
  }
  return make_uint2(cvt_e4m3x2(q[1], q[0]) | (cvt_e4m3x2(q[3], q[2]) << 16),
                    cvt_e4m3x2(q[5], q[4]) | (cvt_e4m3x2(q[7], q[6]) << 16));
}

// Loads 8 BF16 values at p (16-byte aligned); elements at or past `valid`
// read as +0, which never changes an amax.
__device__ __forceinline__ uint4 load8_bf16(const uint16_t* p, int valid) {
  if (valid >= 8) return __ldcs(reinterpret_cast<const uint4*>(p));
  uint32_t e[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) e[t] = (t < valid) ? static_cast<uint32_t>(p[t]) : 0u;
  return make_uint4(e[0] | (e[1] << 16), e[2] | (e[3] << 16), e[4] | (e[5] << 16),
                    e[6] | (e[7] << 16));
}

__device__ __forceinline__ void store8_codes(uint8_t* p, uint2 c, int valid) {
  if (valid >= 8) {
    __stcs(reinterpret_cast<uint2*>(p), c);
    return;
  }
#pragma unroll
  for (int t = 0; t < 8; ++t)
    if (t < valid) p[t] = static_cast<uint8_t>(((t < 4 ? c.x : c.y) >> (8 * (t & 3))) & 0xFFu);
}

// ------------------------------------------------------------- converter
// One CTA per 128 x 128 block (FastVideo PR #1829, "Changes", converter
// bullet): 256 threads x 8 chunks of 8 BF16 values stay in registers; the
// block amax is reduced across the CTA; every element is then divided by
// s = amax / 448 and encoded.
__global__ void __launch_bounds__(256) quantize_weight_kernel(
    const uint16_t* __restrict__ w, int64_t N, int64_t K, int64_t ldw, uint8_t* __restrict__ q,
    int64_t ldq, float* __restrict__ scale_inv, int KB) {
  const int64_t blk = blockIdx.x;
  const int64_t nb = blk / KB, kb = blk - nb * KB;
  const int64_t n0 = nb * 128, k0 = kb * 128;
  const int rows = static_cast<int>((N - n0 < 128 ? N - n0 : 128));
  const int cols = static_cast<int>((K - k0 < 128 ? K - k0 : 128));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  uint4 v[8];
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = tid + 256 * i;
    const int r = c >> 4, kk = (c & 15) * 8;
    v[i] = make_uint4(0, 0, 0, 0);
    if (r < rows && kk < cols) v[i] = load8_bf16(w + (n0 + r) * ldw + k0 + kk, cols - kk);
    m2 = absmax_u4(m2, v[i]);
  }
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t red[8];
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = max(m, red[i]);

  const float amax = __uint_as_float(m << 16);
  const float s = __fdiv_rn(amax, 448.0f);
  if (tid == 0) scale_inv[blk] = s;
  // An all-zero block has s = 0: its +-0 elements keep their sign under a
  // division by 1 instead.
  const float d = (amax == 0.0f) ? 1.0f : s;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = tid + 256 * i;
    const int r = c >> 4, kk = (c & 15) * 8;
    const uint2 codes = encode8(v[i], d);  // every lane encodes (warp vote inside)
    if (r < rows && kk < cols) store8_codes(q + (n0 + r) * ldq + k0 + kk, codes, cols - kk);
  }
}

// ----------------------------------------------------------- dequantizer
// w[n][k] = BF16(float(E4M3(q[n][k])) * s[n/128][k/128]): one warp per row at
// a time, 16 codes (one 16-byte load, two 16-byte stores) per lane-step.
__device__ __forceinline__ uint32_t dequant2(uint32_t codes16, float s) {
  const uint32_t h2 = e4m3x2_to_f16x2(codes16);
  return cvt_bf16x2(__fmul_rn(f16_hi_to_f32(h2), s), __fmul_rn(f16_lo_to_f32(h2), s));
}

__global__ void __launch_bounds__(256) dequantize_kernel(const uint8_t* __restrict__ q, int64_t ldq,
                                                         const float* __restrict__ scale_inv,
                                                         int64_t N, int64_t K, int KB,
                                                         uint16_t* __restrict__ w, int64_t ldw) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t n = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); n < N; n += warps) {
    const uint8_t* qrow = q + n * ldq;
    uint16_t* wrow = w + n * ldw;
    const float* srow = scale_inv + (n >> 7) * KB;
    // Four 16-code chunks per lane per step: all four loads are issued before
    // any conversion, so each warp keeps 2 KB of reads in flight.
    for (int64_t base = 0; base < K; base += 4 * 32 * 16) {
      uint4 c[4];
      float s[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t k = base + u * 512 + lane * 16;
        c[u] = make_uint4(0, 0, 0, 0);
        s[u] = 0.0f;
        if (k < K) s[u] = __ldg(srow + (k >> 7));
        if (k + 16 <= K) c[u] = __ldcs(reinterpret_cast<const uint4*>(qrow + k));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t k = base + u * 512 + lane * 16;
        if (k + 16 <= K) {
          const uint4 o0 = make_uint4(dequant2(c[u].x, s[u]), dequant2(c[u].x >> 16, s[u]),
                                      dequant2(c[u].y, s[u]), dequant2(c[u].y >> 16, s[u]));
          const uint4 o1 = make_uint4(dequant2(c[u].z, s[u]), dequant2(c[u].z >> 16, s[u]),
                                      dequant2(c[u].w, s[u]), dequant2(c[u].w >> 16, s[u]));
          __stcs(reinterpret_cast<uint4*>(wrow + k), o0);
          __stcs(reinterpret_cast<uint4*>(wrow + k + 8), o1);
        } else if (k < K) {
          for (int64_t t = k; t < K; ++t)
            wrow[t] = static_cast<uint16_t>(dequant2(qrow[t], s[u]) & 0xFFFFu);
        }
      }
    }
  }
}

// -------------------------------------------------- activation quantizer
// 1 x 128 K-groups: a half-warp per group (16 lanes x 8 BF16), amax by
// shuffles, s = amax / 448, codes = E4M3(x / s). Groups are numbered row-major
// (g = m * KB + kb) and spread over the whole grid, 16 per CTA; lanes past
// the last group still take part in the shuffles.
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t* __restrict__ x,
                                                           int64_t M, int64_t K, int64_t ldx,
                                                           uint8_t* __restrict__ qx, int64_t ldqx,
                                                           float* __restrict__ sx, int64_t ldsx,
                                                           int KB) {
  const int j = threadIdx.x & 15;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 16 + (threadIdx.x >> 4);
  const bool live = g < M * KB;
  const int64_t m = live ? g / KB : 0;
  const int kb = live ? static_cast<int>(g - m * KB) : 0;
  const int64_t k = static_cast<int64_t>(kb) * 128 + 8 * j;
  const bool valid = live && k < K;
  const int nvalid = valid ? static_cast<int>((K - k < 8 ? K - k : 8)) : 0;
  const uint4 v = valid ? load8_bf16(x + m * ldx + k, nvalid) : make_uint4(0, 0, 0, 0);
  const uint32_t m2 = absmax_u4(0u, v);
  uint32_t mx = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
  const float amax = __uint_as_float(mx << 16);
  const float s = __fdiv_rn(amax, 448.0f);
  const uint2 codes = encode8(v, (amax == 0.0f) ? 1.0f : s);  // every lane (warp vote)
  if (valid) store8_codes(qx + m * ldqx + k, codes, nvalid);
  if (live && j == 0) sx[static_cast<int64_t>(kb) * ldsx + m] = s;
}

// ------------------------------------------------------------------ codec
__global__ void __launch_bounds__(256) encode_kernel(const float* __restrict__ v, int64_t n,
                                                     uint8_t* __restrict__ out) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x * 4;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4; i < n;
       i += stride) {
    if (i + 4 <= n) {
      const float4 f = __ldcs(reinterpret_cast<const float4*>(v + i));
      const uint32_t c = cvt_e4m3x2(f.y, f.x) | (cvt_e4m3x2(f.w, f.z) << 16);
      __stcs(reinterpret_cast<unsigned int*>(out + i), c);
    } else {
      for (int64_t t = i; t < n; ++t) out[t] = static_cast<uint8_t>(cvt_e4m3x2(0.0f, v[t]) & 0xFFu);
    }
  }
}

int grid_for_rows(int64_t rows, int num_sms) {
  const int64_t ctas = cdiv(rows, 8);
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  return static_cast<int>(ctas < cap ? ctas : cap);
}

}  // namespace

cudaError_t launch_quantize_weight(const Launch& L, const uint16_t* w, int64_t N, int64_t K,
                                   int64_t ldw, uint8_t* q, int64_t ldq, float* scale_inv) {
  const int64_t NB = cdiv(N, 128), KB = cdiv(K, 128);
  if (NB * KB > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  quantize_weight_kernel<<<static_cast<unsigned>(NB * KB), 256, 0, L.stream>>>(
      w, N, K, ldw, q, ldq, scale_inv, static_cast<int>(KB));
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const Launch& L, const uint8_t* q, int64_t ldq,
                              const float* scale_inv, int64_t N, int64_t K, uint16_t* w,
                              int64_t ldw) {
  dequantize_kernel<<<grid_for_rows(N, L.num_sms), 256, 0, L.stream>>>(
      q, ldq, scale_inv, N, K, static_cast<int>(cdiv(K, 128)), w, ldw);
  return cudaGetLastError();
}

cudaError_t launch_quantize_act(const Launch& L, const uint16_t* x, int64_t M, int64_t K,
                                int64_t ldx, uint8_t* qx, int64_t ldqx, float* sx, int64_t ldsx) {
  const int64_t ctas = cdiv(M * cdiv(K, 128), 16);
  if (ctas > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  quantize_act_kernel<<<static_cast<unsigned>(ctas), 256, 0, L.stream>>>(
      x, M, K, ldx, qx, ldqx, sx, ldsx, static_cast<int>(cdiv(K, 128)));
  return cudaGetLastError();
}

cudaError_t launch_encode_e4m3(const Launch& L, const float* v, int64_t n, uint8_t* codes) {
  const int64_t ctas = cdiv(n, 1024);
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 16;
  encode_kernel<<<static_cast<unsigned>(ctas < cap ? ctas : cap), 256, 0, L.stream>>>(v, n, codes);
  return cudaGetLastError();
}

}  // namespace fp8blk
