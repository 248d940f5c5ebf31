// Elementwise stages of the block-FP8 linear: the weight converter, the
// dequantizer, the 1 x 128 activation quantizer and the bare E4M3 codec.
// All are HBM-bound streams with one pass over the data: the converter and
// the dequantizer move tiles with TMA (the converter keeps its 128 x 128
// block in registers between the amax reduction and the encoding), the
// activation quantizer and the codec use 16-byte vector loads and stores.
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
// Division is the converter's costliest step, so when d >= 2^-125 a bracket
// gives the same codes from two products: with y = RN(1 / d),
// ylo = RN(y (1 - 2^-21)) and yhi = RN(y (1 + 2^-21)), the products
// RN(v ylo) and RN(v yhi) lie on either side of RN(v / d) (each of y, ylo,
// RN(v ylo) adds at most 2^-24 relative error, 3 x 2^-24 < 2^-21 - 2^-24).
// E4M3 rounding is monotone, so when both ends give the same code, so does
// the quotient; elements whose bracket straddles a decision point take the
// exact quotient instead. Checked exhaustively against the exact quotient
// over every BF16 value v and every BF16 block maximum (d = amax / 448).
struct E4M3Divisor {
  float d;         // the divisor
  uint64_t ylo2;   // RN(y (1 - 2^-21)) in both halves
  uint64_t yhi2;   // RN(y (1 + 2^-21)) in both halves
  bool exact;      // 1 / d is not a finite normal: always divide
};

__device__ __forceinline__ E4M3Divisor make_divisor(float d) {
  E4M3Divisor r;
  r.d = d;
  r.exact = d < 2.35098870e-38f;  // 2^-125
  const float y = __frcp_rn(r.exact ? 1.0f : d);
  const float ylo = __fmul_rn(y, 0.99999952316284180f);  // 1 - 2^-21
  const float yhi = __fmul_rn(y, 1.00000047683715820f);  // 1 + 2^-21
  r.ylo2 = pack_f32x2(ylo, ylo);
  r.yhi2 = pack_f32x2(yhi, yhi);
  return r;
}

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// E4M3 codes of the two floats packed in p (low half -> low byte).
__device__ __forceinline__ uint32_t cvt_e4m3x2_packed(uint64_t p) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
  return cvt_e4m3x2(hi, lo);
}

// Two BF16 values (low half -> low byte) -> the E4M3 codes of the bracket's
// lower end; `diff` gets the bytes where the upper end gives another code
// (a straddle, settled by the exact quotient).
__device__ __forceinline__ uint32_t bracket2(uint32_t w2, const E4M3Divisor& dv, uint32_t& diff) {
  const uint64_t f2 = pack_u32x2(w2 << 16, w2 & 0xFFFF0000u);
  const uint32_t clo = cvt_e4m3x2_packed(fmul2(f2, dv.ylo2));
  const uint32_t chi = cvt_e4m3x2_packed(fmul2(f2, dv.yhi2));
  diff = clo ^ chi;
  return clo;
}

// The exact codes of two BF16 values (two IEEE divisions).
__device__ __forceinline__ uint32_t divide2(uint32_t w2, float d) {
  return cvt_e4m3x2(__fdiv_rn(bf16_hi_to_f32(w2), d), __fdiv_rn(bf16_lo_to_f32(w2), d));
}

// Eight BF16 values -> eight E4M3 codes of RN_f32(v / d) (code i in byte i).
// All 32 lanes of the warp must call this together. Element positions where
// some lane's bracket straddles a decision point take the exact quotient
// (for the other lanes it gives the same code); BF16 data hit such near-ties
// often, since v / (amax / 448) is a ratio of two 8-bit mantissas times 7.
__device__ __forceinline__ uint2 encode8(const uint4& v, const E4M3Divisor& dv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t code[4], diff[4];
  if (dv.exact) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      diff[i] = 0u;
      code[i] = divide2(w[i], dv.d);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) code[i] = bracket2(w[i], dv, diff[i]);
  }
  if (__any_sync(0xFFFFFFFFu, (diff[0] | diff[1] | diff[2] | diff[3]) != 0u)) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (__any_sync(0xFFFFFFFFu, (diff[i] & 0xFFu) != 0u))
        code[i] = (code[i] & 0xFF00u) | (cvt_e4m3x2(0.0f, __fdiv_rn(bf16_lo_to_f32(w[i]), dv.d)) & 0xFFu);
      if (__any_sync(0xFFFFFFFFu, (diff[i] >> 8) != 0u))
        code[i] = (code[i] & 0x00FFu) | (cvt_e4m3x2(__fdiv_rn(bf16_hi_to_f32(w[i]), dv.d), 0.0f) & 0xFF00u);
    }
  }
  return make_uint2(code[0] | (code[1] << 16), code[2] | (code[3] << 16));
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
// Per 128 x 128 block (FastVideo PR #1829, "Changes", converter bullet): the
// block amax over the BF16 values, s = amax / 448, and every element divided
// by s and encoded. Persistent CTAs (two per SM) walk the blocks b =
// blockIdx.x, + gridDim.x, ... in row-major block order. Thread 0 keeps a
// 3-deep ring of TMA loads in flight (box 128 x 128 BF16, unswizzled; parts
// past N or K read as 0, which never changes an amax). Each of the eight
// warps takes 16 rows of a block: lane l reads elements 4l..4l+3 of each row
// (8-byte shared loads, conflict-free), the warps' maxima meet in shared
// memory, and each lane then encodes its 64 values and writes 4 codes per row
// (128 contiguous bytes per warp and row). The encoding is one multiply per
// element by a multiplier checked for the block (below), or, for the blocks
// where no candidate passes, the product bracket: elements whose bracket
// straddles a decision point are then settled after the block, each lane
// re-reading its values from the stage. A stage is refilled (by thread 0)
// only once the next block's amax barrier shows every warp done with it:
// two loads stay in flight per CTA.

// A single multiplier per block. For a block divisor d, write each BF16
// value as v = 1.m x 2^e. Scaling v by 2^e scales RN(v / d) and RN(v * c)
// exactly, as long as neither leaves the FP32 normal range. So whether
// E4M3(RN(v * c)) equals E4M3(RN(v / d)) depends only on the 7-bit mantissa
// m and on which E4M3 binade the quotient falls in:
//  - all normal binades round alike up to a shift of the exponent field;
//  - each subnormal binade from 2^-12 to 2^-6 has its own grid;
//  - quotients below 2^-12 are far from every decision point (the lowest,
//    2^-10, is four times larger) and give a zero code either way.
// verify_multiplier checks one mantissa: the quotient and the product of
// v_m = 1.m x 2^-e(c), placed in [1, 4), then scaled by 2^0 and by
// 2^-7 ... 2^-12, must give equal codes. When every mantissa passes for some
// c, the block is encoded with one multiply and one conversion per element
// and no check. A search over every BF16 block maximum and every BF16 value
// (1.06 x 10^9 pairs, FP32 arithmetic as here) found: c = RN(1/d) passes for
// 80% of the maxima, its upper neighbour for 12%, its lower one for 3%;
// with a passing c, all codes equal the quotient's. Blocks where no
// candidate passes keep the product bracket.
__device__ __forceinline__ bool verify_multiplier(float c, float d, int m) {
  const int ec = static_cast<int>((__float_as_uint(c) >> 23) & 0xFFu) - 127;
  const float vm = __uint_as_float((static_cast<uint32_t>(127 - ec) << 23) |
                                   (static_cast<uint32_t>(m) << 16));
  const float r = __fdiv_rn(vm, d);
  const float rp = __fmul_rn(vm, c);
  uint32_t x = cvt_e4m3x2(r, rp);
  bool ok = (x & 0xFFu) == (x >> 8);
  float scale = 0.0078125f;  // 2^-7
#pragma unroll
  for (int k = 0; k < 6; ++k) {
    x = cvt_e4m3x2(__fmul_rn(r, scale), __fmul_rn(rp, scale));
    ok = ok && ((x & 0xFFu) == (x >> 8));
    scale *= 0.5f;
  }
  return ok;
}

// Divisors below this go to the bracket (and, below 2^-125, to division):
// c ~ 1/d would reach values where v_m = 1.m x 2^-e(c) leaves the range.
constexpr float kMinMultiplierDivisor = 7.88860905e-31f;  // 2^-100

// A warp's 16 rows of one block with a verified multiplier: codes of
// RN(v * c), stored row by row (4 per lane).
template <bool Interior>
__device__ __forceinline__ void encode_rows_fast(const uint2 (&v)[16], uint64_t c2, uint8_t* dst,
                                                 int64_t ldq, int rows_left, int cols_left) {
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const uint32_t w0 = v[r].x, w1 = v[r].y;
    const uint32_t c01 = cvt_e4m3x2_packed(fmul2(pack_u32x2(w0 << 16, w0 & 0xFFFF0000u), c2));
    const uint32_t c23 = cvt_e4m3x2_packed(fmul2(pack_u32x2(w1 << 16, w1 & 0xFFFF0000u), c2));
    const uint32_t codes = c01 | (c23 << 16);
    if (Interior) {
      __stcs(reinterpret_cast<unsigned int*>(dst), codes);
    } else if (r < rows_left && cols_left > 0) {
      if (cols_left >= 4) {
        __stcs(reinterpret_cast<unsigned int*>(dst), codes);
      } else {
        for (int t = 0; t < cols_left; ++t) dst[t] = static_cast<uint8_t>(codes >> (8 * t));
      }
    }
    dst += ldq;
  }
}

// A warp's 16 rows of one block: codes of the bracket's lower end stored
// row by row (4 per lane), returning one bit per row pair with a straddle.
// Interior blocks store without bounds checks; otherwise rows_left and
// cols_left are the rows and columns of this lane's part inside the matrix.
template <bool Interior>
__device__ __forceinline__ uint32_t encode_rows(const uint2 (&v)[16], const E4M3Divisor& dv,
                                                uint8_t* dst, int64_t ldq, int rows_left,
                                                int cols_left) {
  uint32_t straddled = 0u;
#pragma unroll
  for (int g = 0; g < 8; ++g) {
    const uint32_t w4[4] = {v[2 * g].x, v[2 * g].y, v[2 * g + 1].x, v[2 * g + 1].y};
    uint32_t code[4], diff[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) code[k] = bracket2(w4[k], dv, diff[k]);
    straddled |= ((diff[0] | diff[1] | diff[2] | diff[3]) != 0u ? 1u : 0u) << g;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t codes = code[2 * h] | (code[2 * h + 1] << 16);
      if (Interior) {
        __stcs(reinterpret_cast<unsigned int*>(dst), codes);
      } else if (2 * g + h < rows_left && cols_left > 0) {
        if (cols_left >= 4) {
          __stcs(reinterpret_cast<unsigned int*>(dst), codes);
        } else {
          for (int t = 0; t < cols_left; ++t) dst[t] = static_cast<uint8_t>(codes >> (8 * t));
        }
      }
      dst += ldq;
    }
  }
  return straddled;
}

constexpr int kCvtStages = 3;
constexpr int kCvtStageBytes = 128 * 128 * 2;
constexpr size_t kCvtSmem = 128 + static_cast<size_t>(kCvtStages) * kCvtStageBytes;

__global__ void __launch_bounds__(256, 2) quantize_weight_kernel(
    const __grid_constant__ CUtensorMap tm_w, int64_t N, int64_t K, uint8_t* __restrict__ q,
    int64_t ldq, float* __restrict__ scale_inv, int KB, int nblocks, unsigned* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  __shared__ uint64_t full[kCvtStages];
  __shared__ uint32_t red[2][8];
  __shared__ uint32_t vote[2][8], vote2[2][8];
  __shared__ int abort_flag;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // Launched as a programmatic dependent: the launch overlaps the kernel
  // before, and nothing is read or written until that kernel has completed.
  pdl_launch_dependents();
  pdl_wait();
  if (tid == 0) {
    for (int s = 0; s < kCvtStages; ++s) mbar_init(&full[s], 1);
    mbar_init_fence();
    abort_flag = 0;
  }
  __syncthreads();
  // Thread 0: load this CTA's i-th block into stage i % kCvtStages.
  auto issue = [&](int i) {
    const int b = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    if (b >= nblocks) return;
    const int nb = b / KB, kb = b - nb * KB;
    uint64_t* bar = &full[i % kCvtStages];
    mbar_arrive_expect_tx(bar, kCvtStageBytes);
    tma_load_2d(smem + (i % kCvtStages) * kCvtStageBytes, &tm_w, bar, kb * 128, nb * 128);
  };
  if (tid == 0) {
    tma_prefetch_map(&tm_w);
    for (int i = 0; i < kCvtStages; ++i) issue(i);
  }
  int i = 0;
  for (;; ++i) {
    const int b = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    if (b >= nblocks) break;
    const int st = i % kCvtStages;
    const bool landed = mbar_wait_warp(&full[st], static_cast<uint32_t>((i / kCvtStages) & 1), err,
                                       kErrWaitLoad);
    const uint8_t* rows16 = smem + st * kCvtStageBytes + warp * 16 * 256 + lane * 8;
    uint2 v[16];
    uint32_t m2 = 0;
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      v[r] = *reinterpret_cast<const uint2*>(rows16 + r * 256);
      m2 = absmax2(absmax2(m2, v[r].x), v[r].y);
    }
    uint32_t m = __reduce_max_sync(0xFFFFFFFFu, max(m2 & 0xFFFFu, m2 >> 16));
    if (lane == 0) {
      red[i & 1][warp] = m;
      if (!landed) abort_flag = 1;
    }
    __syncthreads();
    if (abort_flag) break;
    // Every warp is done with the previous block's stage (its straddles
    // included): refill it.
    if (tid == 0 && i > 0) issue(i + kCvtStages - 1);
    m = red[i & 1][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = max(m, red[i & 1][w]);
    const float amax = __uint_as_float(m << 16);
    const float s = __fdiv_rn(amax, 448.0f);
    if (tid == 0) scale_inv[b] = s;
    const int nb = b / KB, kb = b - nb * KB;
    const int64_t n0 = static_cast<int64_t>(nb) * 128, k0 = static_cast<int64_t>(kb) * 128;
    const int rows = static_cast<int>(N - n0 < 128 ? N - n0 : 128);
    const int cols = static_cast<int>(K - k0 < 128 ? K - k0 : 128);
    const int col = 4 * lane;
    uint8_t* dst0 = q + (n0 + warp * 16) * ldq + k0 + col;
    // The multiplier: an all-zero block encodes +-0 with any c. Otherwise
    // warps 0-3 check RN(1/s) and warps 4-7 its upper neighbour, one
    // mantissa per thread; if both fail, warps 0-3 check the lower one.
    // Every branch below is the same for the whole CTA.
    float c = 1.0f;
    bool fast = amax == 0.0f;
    if (!fast && s >= kMinMultiplierDivisor) {
      const float c0 = __frcp_rn(s);
      const float cu = __uint_as_float(__float_as_uint(c0) + 1u);
      const bool okw = __all_sync(0xFFFFFFFFu, verify_multiplier(tid < 128 ? c0 : cu, s, tid & 127));
      if (lane == 0) vote[i & 1][warp] = okw ? 1u : 0u;
      __syncthreads();
      const uint32_t* vt = vote[i & 1];
      if (vt[0] & vt[1] & vt[2] & vt[3]) {
        c = c0;
        fast = true;
      } else if (vt[4] & vt[5] & vt[6] & vt[7]) {
        c = cu;
        fast = true;
      } else {
        const float cd = __uint_as_float(__float_as_uint(c0) - 1u);
        const bool ok2 = __all_sync(0xFFFFFFFFu, tid < 128 ? verify_multiplier(cd, s, tid & 127) : true);
        if (lane == 0) vote2[i & 1][warp] = ok2 ? 1u : 0u;
        __syncthreads();
        const uint32_t* v2 = vote2[i & 1];
        if (v2[0] & v2[1] & v2[2] & v2[3]) {
          c = cd;
          fast = true;
        }
      }
    }
    if (fast) {
      const uint64_t c2 = pack_f32x2(c, c);
      if (rows == 128 && cols == 128)
        encode_rows_fast<true>(v, c2, dst0, ldq, 16, 4);
      else
        encode_rows_fast<false>(v, c2, dst0, ldq, rows - warp * 16, cols - col);
      continue;
    }
    const E4M3Divisor dv = make_divisor(s);
    // Provisional codes from the bracket's lower end, with one bit per row
    // pair in which this lane saw a straddle (every pair when d is too small
    // for the bracket).
    uint32_t straddled = dv.exact ? 0xFFu : 0u;
    if (rows == 128 && cols == 128)
      straddled |= encode_rows<true>(v, dv, dst0, ldq, 16, 4);
    else
      straddled |= encode_rows<false>(v, dv, dst0, ldq, rows - warp * 16, cols - col);
    // Straddles (rare): each lane re-reads its row pairs that had one from
    // the stage (still resident: it is refilled only after the next amax
    // barrier) and writes the exact quotient's code over the provisional one.
    while (straddled != 0u) {
      const int g = __ffs(straddled) - 1;
      straddled &= straddled - 1u;
      const uint8_t* src = smem + st * kCvtStageBytes + (warp * 16 + 2 * g) * 256 + lane * 8;
      const uint2 a = *reinterpret_cast<const uint2*>(src);
      const uint2 c = *reinterpret_cast<const uint2*>(src + 256);
      const uint32_t w4[4] = {a.x, a.y, c.x, c.y};
      uint32_t elems = 0;  // bit 2k + h: half h of word k straddles
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t diff;
        bracket2(w4[k], dv, diff);
        if (dv.exact) diff = 0xFFFFu;
        elems |= (((diff & 0xFFu) != 0u ? 1u : 0u) | ((diff >> 8) != 0u ? 2u : 0u)) << (2 * k);
      }
      // one element per lane and pass: the lanes' divisions run side by side
      while (elems != 0u) {
        const int t = __ffs(elems) - 1;
        elems &= elems - 1u;
        const int k = t >> 1;
        const uint32_t wd = (k & 2) ? ((k & 1) ? w4[3] : w4[2]) : ((k & 1) ? w4[1] : w4[0]);
        const float x = (t & 1) ? bf16_hi_to_f32(wd) : bf16_lo_to_f32(wd);
        const uint32_t code = cvt_e4m3x2(0.0f, __fdiv_rn(x, dv.d)) & 0xFFu;
        const int r = warp * 16 + 2 * g + (k >> 1), cc = col + 2 * (k & 1) + (t & 1);
        if (r < rows && cc < cols) q[(n0 + r) * ldq + k0 + cc] = static_cast<uint8_t>(code);
      }
    }
  }
  // After a time-out, the loads still in flight land before the CTA exits.
  if (tid == 0 && abort_flag) {
    // issued so far: blocks 0 .. max(kCvtStages - 1, i + kCvtStages - 2)
    const int last = i + kCvtStages - 2 > kCvtStages - 1 ? i + kCvtStages - 2 : kCvtStages - 1;
    for (int k = i; k <= last; ++k) {
      const int b = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
      if (b < nblocks) mbar_wait(&full[k % kCvtStages], static_cast<uint32_t>((k / kCvtStages) & 1), err, kErrWaitLoad);
    }
  }
}

// ----------------------------------------------------------- dequantizer
// w[n][k] = BF16(float(E4M3(q[n][k])) * s[n/128][k/128]), one float multiply
// and one round to nearest even. Persistent, one CTA of 512 threads per SM,
// over tiles of 64 rows x 256 codes (tile t: row tile t / tiles_k, column
// tile t % tiles_k). Thread 0 keeps a 4-stage ring of TMA loads of code
// tiles (16 KB, unswizzled; parts past N or K read as 0) and TMA-stores each
// finished BF16 tile (32 KB, three staging buffers; the store clips at N and
// K), so the bytes in flight sit in shared memory, not in registers. Every
// thread converts two 16-code chunks per tile (chunk c = thread + 512 u:
// row c / 16, codes 16 (c % 16) ...), reading the stage conflict-free and
// writing its 32 bytes of BF16 in the half order that keeps a quarter warp
// on distinct banks. A tile's two block scales are loaded two tiles ahead.
__device__ __forceinline__ uint32_t dequant2(uint32_t codes16, float s) {
  const uint32_t h2 = e4m3x2_to_f16x2(codes16);
  return cvt_bf16x2(__fmul_rn(f16_hi_to_f32(h2), s), __fmul_rn(f16_lo_to_f32(h2), s));
}

constexpr int kDqRows = 64, kDqCols = 256;
constexpr int kDqInBytes = kDqRows * kDqCols;       // one code tile
constexpr int kDqOutBytes = kDqRows * kDqCols * 2;  // its BF16 tile
constexpr int kDqStages = 4, kDqOutBufs = 3, kDqThreads = 512;
constexpr size_t kDqSmem = 128 + static_cast<size_t>(kDqStages) * kDqInBytes +
                           static_cast<size_t>(kDqOutBufs) * kDqOutBytes;

__global__ void __launch_bounds__(kDqThreads, 1) dequantize_kernel(
    const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_w,
    const float* __restrict__ scale_inv, int KB, int tiles_k, int ntiles, unsigned* __restrict__ err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  uint8_t* s_in = smem;                                 // kDqStages code tiles
  uint8_t* s_out = smem + kDqStages * kDqInBytes;       // kDqOutBufs BF16 tiles
  __shared__ uint64_t full[kDqStages];
  __shared__ int abort_flag;
  const int tid = threadIdx.x;
  // Launched as a programmatic dependent: the launch overlaps the kernel
  // before, and nothing is read or written until that kernel has completed.
  pdl_launch_dependents();
  pdl_wait();
  if (tid == 0) {
    for (int st = 0; st < kDqStages; ++st) mbar_init(&full[st], 1);
    mbar_init_fence();
    abort_flag = 0;
  }
  __syncthreads();
  // Thread 0: load this CTA's i-th tile into stage i % kDqStages.
  auto issue = [&](int i) {
    const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    if (t >= ntiles) return;
    const int tr = t / tiles_k, tc = t - tr * tiles_k;
    uint64_t* bar = &full[i % kDqStages];
    mbar_arrive_expect_tx(bar, kDqInBytes);
    tma_load_2d(s_in + (i % kDqStages) * kDqInBytes, &tm_q, bar, tc * kDqCols, tr * kDqRows);
  };
  if (tid == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_w);
    for (int i = 0; i < kDqStages; ++i) issue(i);
  }
  const int h = (tid >> 2) & 1;  // which 16-byte half of its 32 output bytes a thread writes first
  // The block scales of this CTA's i-th tile (0 past K).
  auto scales = [&](int i, float& s0, float& s1) {
    const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    s0 = s1 = 0.0f;
    if (t >= ntiles) return;
    const int tr = t / tiles_k, tc = t - tr * tiles_k;
    const float* srow = scale_inv + static_cast<int64_t>((tr * kDqRows) >> 7) * KB;
    const int kb0 = tc * (kDqCols / 128);
    if (kb0 < KB) s0 = __ldg(srow + kb0);
    if (kb0 + 1 < KB) s1 = __ldg(srow + kb0 + 1);
  };
  float s0, s1, n0, n1;
  scales(0, s0, s1);
  scales(1, n0, n1);
  int i = 0;
  for (;; ++i) {
    const int t = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    if (t >= ntiles) break;
    const int st = i % kDqStages;
    const bool landed = mbar_wait_warp(&full[st], static_cast<uint32_t>((i / kDqStages) & 1), err,
                                       kErrWaitLoad);
    if (tid == 0) tma_store_wait_read<kDqOutBufs - 1>();  // the store that last used this buffer has read it
    if ((tid & 31) == 0 && !landed) abort_flag = 1;
    __syncthreads();
    if (abort_flag) break;
    float p0, p1;
    scales(i + 2, p0, p1);
    const int tr = t / tiles_k, tc = t - tr * tiles_k;
    const uint8_t* in = s_in + st * kDqInBytes;
    uint8_t* out = s_out + (i % kDqOutBufs) * kDqOutBytes;
#pragma unroll
    for (int u = 0; u < kDqInBytes / 16 / kDqThreads; ++u) {
      const int c = tid + kDqThreads * u;
      const uint4 v = *reinterpret_cast<const uint4*>(in + 16 * c);
      const float sc = (c & 15) < 8 ? s0 : s1;
      const uint4 o0 = make_uint4(dequant2(v.x, sc), dequant2(v.x >> 16, sc), dequant2(v.y, sc),
                                  dequant2(v.y >> 16, sc));
      const uint4 o1 = make_uint4(dequant2(v.z, sc), dequant2(v.z >> 16, sc), dequant2(v.w, sc),
                                  dequant2(v.w >> 16, sc));
      uint8_t* dst = out + (c >> 4) * (2 * kDqCols) + (c & 15) * 32;
      *reinterpret_cast<uint4*>(dst + 16 * h) = h ? o1 : o0;
      *reinterpret_cast<uint4*>(dst + 16 * (1 - h)) = h ? o0 : o1;
    }
    s0 = n0;
    s1 = n1;
    n0 = p0;
    n1 = p1;
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tma_store_2d(&tm_w, out, tc * kDqCols, tr * kDqRows);
      tma_store_commit();
      issue(i + kDqStages);  // every thread is done with stage st
    }
  }
  if (tid == 0) {
    // After a time-out, the loads still in flight land before the CTA exits.
    if (abort_flag) {
      for (int k = i; k < i + kDqStages; ++k) {
        const int t = static_cast<int>(blockIdx.x) + k * static_cast<int>(gridDim.x);
        if (t < ntiles) mbar_wait(&full[k % kDqStages], static_cast<uint32_t>((k / kDqStages) & 1), err, kErrWaitLoad);
      }
    }
    tma_store_wait_all();
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
  // The W8A8 GEMM launched after this kernel may be scheduled now: it reads
  // the codes and scales only after griddepcontrol.wait. When this kernel is
  // itself a programmatic dependent (inside a sequence of linears), x may be
  // the previous linear's output: wait for that kernel first.
  pdl_launch_dependents();
  pdl_wait();
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
  const uint2 codes = encode8(v, make_divisor((amax == 0.0f) ? 1.0f : s));  // every lane (warp vote)
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

// A launch as a programmatic dependent of the kernel before it in the stream.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace

cudaError_t launch_quantize_weight(const Launch& L, const uint16_t* w, int64_t N, int64_t K,
                                   int64_t ldw, uint8_t* q, int64_t ldq, float* scale_inv) {
  const int64_t NB = cdiv(N, 128), KB = cdiv(K, 128);
  if (NB * KB > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  CUtensorMap tw;
  if (!make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, K, N, 2 * ldw, 128, 128,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(quantize_weight_kernel), kCvtSmem);
  if (e != cudaSuccess) return e;
  const int64_t nblocks = NB * KB, cap = 2 * static_cast<int64_t>(L.num_sms);
  return launch_pdl(quantize_weight_kernel, static_cast<unsigned>(nblocks < cap ? nblocks : cap),
                    256, kCvtSmem, L.stream, tw, N, K, q, ldq, scale_inv, static_cast<int>(KB),
                    static_cast<int>(nblocks), L.err);
}

cudaError_t launch_dequantize(const Launch& L, const uint8_t* q, int64_t ldq,
                              const float* scale_inv, int64_t N, int64_t K, uint16_t* w,
                              int64_t ldw) {
  const int64_t tiles_k = cdiv(K, kDqCols), ntiles = cdiv(N, kDqRows) * tiles_k;
  if (ntiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  CUtensorMap tq, tw;
  if (!make_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, ldq, kDqCols, kDqRows,
                    CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w, K, N, 2 * ldw, kDqCols, kDqRows,
                    CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(dequantize_kernel), kDqSmem);
  if (e != cudaSuccess) return e;
  const int64_t grid = ntiles < L.num_sms ? ntiles : L.num_sms;
  return launch_pdl(dequantize_kernel, static_cast<unsigned>(grid), kDqThreads, kDqSmem, L.stream, tq, tw,
                    scale_inv, static_cast<int>(cdiv(K, 128)), static_cast<int>(tiles_k),
                    static_cast<int>(ntiles), L.err);
}

cudaError_t launch_quantize_act(const Launch& L, const uint16_t* x, int64_t M, int64_t K,
                                int64_t ldx, uint8_t* qx, int64_t ldqx, float* sx, int64_t ldsx,
                                bool pdl) {
  const int64_t ctas = cdiv(M * cdiv(K, 128), 16);
  if (ctas > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, quantize_act_kernel, x, M, K, ldx, qx, ldqx, sx, ldsx,
                            static_cast<int>(cdiv(K, 128)));
}

cudaError_t launch_encode_e4m3(const Launch& L, const float* v, int64_t n, uint8_t* codes) {
  const int64_t ctas = cdiv(n, 1024);
  const int64_t cap = static_cast<int64_t>(L.num_sms) * 16;
  encode_kernel<<<static_cast<unsigned>(ctas < cap ? ctas : cap), 256, 0, L.stream>>>(v, n, codes);
  return cudaGetLastError();
}

}  // namespace fp8blk
