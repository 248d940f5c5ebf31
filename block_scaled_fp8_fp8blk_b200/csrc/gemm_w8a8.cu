// Block-scaled FP8 x FP8 linear (W8A8) on tcgen05:
//   y[m][n] = BF16( sum_kb sx[kb][m] * s[n/128][kb] * P_kb[m][n] ),
//   P_kb = (128-wide K slab of qx) . (same slab of q)^T, E4M3 x E4M3 -> FP32.
// FastVideo PR #1829, "Purpose": the linear is x times the dequantized weight,
// computed the way the Blackwell groupwise GEMM does it (scales applied per
// 128-wide K group). The scales are arbitrary floats, not powers of two, and
// the weight blocks are 128 x 128, so they are applied in software to each
// slab's FP32 partial ("promotion") rather than by the MMA.
//
// One CTA computes a 128 (m) x BN (n) tile:
//   warp 0      TMA producer: qx tile [128 x 128 B] + q tile [BN x 128 B] per
//               slab into a STAGES-deep shared-memory ring (128-byte swizzle);
//   warp 1      TMEM allocator and MMA issuer: 4 x (M=128, N=BN, K=32) per
//               slab into one of two TMEM partial buffers (fresh, no
//               accumulation across slabs);
//   warps 2..   promotion/epilogue: each thread owns one tile row and 128
//               columns, reads the slab partial from TMEM, accumulates
//               acc += P * (sx * s) in registers, releases the TMEM buffer, and
//               finally rounds to BF16 and stores.
// Every wait is bounded (kWaitLimitCycles) and reports to the error word.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {
namespace {

template <int BN>
struct W8A8Cfg {
  static constexpr int BM = 128;
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int EPI_WARPS = 4 * (BN / 128);
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr size_t BAR_BYTES = 256;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = make_idesc(0u, 0u, 128, BN);  // E4M3 x E4M3 -> F32
  static_assert(2 * STAGES * 8 + 4 * 8 + 8 <= BAR_BYTES, "barrier area");
};

template <int BN>
__global__ void __launch_bounds__(W8A8Cfg<BN>::THREADS, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const float* __restrict__ sx, int64_t ldsx, const float* __restrict__ sw,
                     __nv_bfloat16* __restrict__ y, int64_t ldy, int M, int N, int KB,
                     unsigned* __restrict__ err) {
  using C = W8A8Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Token tiles of one weight tile are adjacent in the grid, so they run
  // together and read the weight tile from DRAM once.
  const int m0 = blockIdx.x * C::BM, n0 = blockIdx.y * BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], C::EPI_WARPS);
    }
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_map(&tm_a);
      tma_prefetch_map(&tm_b);
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, err, kErrWaitLoad)) break;
        mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
        tma_load_2d(sA + stage * C::A_BYTES, &tm_a, &full[stage], kb * 128, m0);
        tma_load_2d(sB + stage * C::B_BYTES, &tm_b, &full[stage], kb * 128, n0);
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // Drain: the last load into every used stage has landed before exit
      // (immediate on the normal path, where the MMA warp consumed them all).
      for (int s = 0; s < C::STAGES && s < issued; ++s)
        mbar_wait(&full[s], last_parity((issued - s + C::STAGES - 1) / C::STAGES), err, kErrWaitLoad);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // Descriptors are formed once; stepping through shared memory adds
      // (bytes >> 4) to their start-address field.
      const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(sA));
      const uint64_t bdesc0 = sw128_kmajor_desc(smem_addr(sB));
      int stage = 0, buf = 0, issued = 0;
      uint32_t phase = 0, tphase = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&tempty[buf], tphase ^ 1u, err, kErrWaitMma)) break;
        if (!mbar_wait(&full[stage], phase, err, kErrWaitMma)) break;
        tc_fence_after_sync();
        const uint64_t ad = adesc0 + static_cast<uint64_t>((stage * C::A_BYTES) >> 4);
        const uint64_t bd = bdesc0 + static_cast<uint64_t>((stage * C::B_BYTES) >> 4);
        const uint32_t d = tmem + static_cast<uint32_t>(buf * BN);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_f8f6f4_ss(d, ad + 2u * k, bd + 2u * k, C::IDESC, k > 0 ? 1u : 0u);
        tc_commit(&empty[stage]);
        tc_commit(&tfull[buf]);
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        if (++buf == 2) {
          buf = 0;
          tphase ^= 1u;
        }
      }
      // Drain: all issued MMAs have completed before TMEM is released.
      if (issued > 0) {
        const int b = (issued - 1) & 1;
        mbar_wait(&tfull[b], last_parity((issued - b + 1) / 2), err, kErrWaitMma);
      }
    }
  } else {
    const int e = warp - 2;
    const int quad = warp & 3;           // TMEM lanes this warp may access
    const int half = e >> 2;             // which 128 columns of the tile
    const int row = quad * 32 + lane;    // tile row == TMEM lane
    const int col0 = half * 128;
    const int ncol0 = n0 + col0;
    const bool cols_live = ncol0 < N;
    const float* sw_row = sw + static_cast<int64_t>(cols_live ? (ncol0 >> 7) : 0) * KB;
    const float* sx_col = sx + m0 + row;  // sx[kb][m]: ldsx covers whole 128-row tiles
    const uint32_t t_row = tmem + (static_cast<uint32_t>(quad * 32) << 16) + col0;

    uint64_t acc[64];  // column pairs
#pragma unroll
    for (int i = 0; i < 64; ++i) acc[i] = 0ull;

    int buf = 0;
    uint32_t tphase = 0;
    float c_next = __ldg(sx_col) * __ldg(sw_row);
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      const float c = c_next;
      if (kb + 1 < KB) c_next = __ldg(sx_col + (kb + 1) * ldsx) * __ldg(sw_row + kb + 1);
      if (!mbar_wait_warp(&tfull[buf], tphase, err, kErrWaitEpilogue)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      tmem_axpy2<4>(t_row + static_cast<uint32_t>(buf * BN), c, acc);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      if (++buf == 2) {
        buf = 0;
        tphase ^= 1u;
      }
    }

    const int m = m0 + row;
    if (ok && m < M && cols_live) {
      __nv_bfloat16* yrow = y + static_cast<int64_t>(m) * ldy + ncol0;
      const int ncols = min(128, N - ncol0);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int c = 8 * j;
        uint4 o;
        o.x = cvt_bf16x2_pair(acc[c / 2 + 0]);
        o.y = cvt_bf16x2_pair(acc[c / 2 + 1]);
        o.z = cvt_bf16x2_pair(acc[c / 2 + 2]);
        o.w = cvt_bf16x2_pair(acc[c / 2 + 3]);
        if (c + 8 <= ncols) {
          *reinterpret_cast<uint4*>(yrow + c) = o;
        } else if (c < ncols) {
          const uint32_t wv[4] = {o.x, o.y, o.z, o.w};
          uint16_t* yr = reinterpret_cast<uint16_t*>(yrow);
          for (int t = c; t < ncols; ++t)
            yr[t] = static_cast<uint16_t>((wv[(t - c) >> 1] >> (16 * ((t - c) & 1))) & 0xFFFFu);
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN>
cudaError_t launch_bn(const Launch& L, const uint8_t* qx, int64_t ldqx, const float* sx,
                      int64_t ldsx, const uint8_t* q, int64_t ldq, const float* sw, uint16_t* y,
                      int64_t ldy, int64_t M, int64_t N, int64_t K) {
  using C = W8A8Cfg<BN>;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, K, M, ldqx, 128, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, ldq, 128, BN))
    return cudaErrorInvalidValue;
  auto kern = w8a8_gemm_kernel<BN>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(cdiv(M, 128)), static_cast<unsigned>(cdiv(N, BN)));
  kern<<<grid, C::THREADS, C::SMEM, L.stream>>>(ta, tb, sx, ldsx, sw,
                                                reinterpret_cast<__nv_bfloat16*>(y), ldy,
                                                static_cast<int>(M), static_cast<int>(N),
                                                static_cast<int>(cdiv(K, 128)), L.err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w8a8_gemm(const Launch& L, const uint8_t* qx, int64_t ldqx, const float* sx,
                             int64_t ldsx, const uint8_t* q, int64_t ldq, const float* sw,
                             uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K) {
  if (cdiv(N, 256) > 65535) return cudaErrorInvalidValue;
  return launch_bn<256>(L, qx, ldqx, sx, ldsx, q, ldq, sw, y, ldy, M, N, K);
}

}  // namespace fp8blk
