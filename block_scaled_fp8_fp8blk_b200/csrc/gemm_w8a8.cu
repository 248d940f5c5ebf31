// Block-scaled FP8 x FP8 linear (W8A8) on tcgen05:
//   y[m][n] = BF16( sum_kb sx[kb][m] * s[n/128][kb] * P_kb[m][n] ),
//   P_kb = (128-wide K slab of qx) . (same slab of q)^T, E4M3 x E4M3 -> FP32.
// FastVideo PR #1829, "Purpose": the linear is x times the dequantized weight,
// computed the way the Blackwell groupwise GEMM does it (scales applied per
// 128-wide K group). The scales are arbitrary floats, not powers of two, and
// the weight blocks are 128 x 128, so they are applied in software to each
// slab's FP32 partial ("promotion") rather than by the MMA.
//
// Persistent kernel: one CTA per SM walks output tiles of NSUB x 128 tokens
// by 128 weight rows (one weight block, so the weight scale is one number per
// slab), tile index t = m-tile + (#m-tiles) * n-tile (token tiles of one weight
// tile are neighbours and share it through L2). All rings run on across
// tiles, so the next tile's loads and MMAs overlap this tile's stores.
//   warp 0     TMA producer: per slab one q tile [128 x 128 B] into the B ring
//              and NSUB qx sub-tiles [128 x 128 B] into the A ring;
//   warp 1     TMEM allocator and MMA issuer: per slab and sub-tile
//              4 x (M=128, N=128, K=32) into a 4-deep ring of TMEM partials;
//   warps 2-9  promotion/epilogue: warp (2 + 4t + q') owns TMEM quadrant
//              q = warp % 4 of sub-tile t; each thread owns one token row:
//              acc += P * (sx[m] * s) with packed FP32x2 FMAs, then 16-byte
//              BF16 row stores.
// Every wait is bounded (kWaitLimitCycles) and reports to the error word.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {
namespace {

template <int NSUB>
struct W8A8Cfg {
  static constexpr int TILE_BYTES = 128 * 128;  // one 128 x 128 FP8 operand tile
  static constexpr int AS = NSUB == 2 ? 8 : 6;  // A (activation) ring depth
  static constexpr int BS = NSUB == 2 ? 4 : 6;  // B (weight) ring depth
  static constexpr int PB = 4;                  // TMEM partial ring depth (x 128 columns)
  static constexpr int THREADS = 320;
  static constexpr int NBAR = 2 * AS + 2 * BS + 2 * PB;
  static constexpr size_t SMEM_TILES = static_cast<size_t>(AS + BS) * TILE_BYTES;
  static constexpr size_t SMEM = 1024 + SMEM_TILES + 8 * NBAR + 16;
  static constexpr uint32_t IDESC = make_idesc(0u, 0u, 128, 128);  // E4M3 x E4M3 -> F32
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int NSUB>
__global__ void __launch_bounds__(320, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const float* __restrict__ sx, int64_t ldsx, const float* __restrict__ sw,
                     __nv_bfloat16* __restrict__ y, int64_t ldy, int M, int N, int KB, int mtiles,
                     int ntiles_total, unsigned* __restrict__ err) {
  using C = W8A8Cfg<NSUB>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sA = smem;                              // AS x 16 KB
  uint8_t* sB = smem + C::AS * C::TILE_BYTES;      // BS x 16 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_TILES);
  uint64_t* afull = bars;               // qx sub-tile landed   (1 arrival + tx)
  uint64_t* aempty = afull + C::AS;     // qx sub-tile consumed (1 commit)
  uint64_t* bfull = aempty + C::AS;     // q tile landed        (1 arrival + tx)
  uint64_t* bempty = bfull + C::BS;     // q tile consumed      (1 commit)
  uint64_t* pfull = bempty + C::BS;     // partial ready        (1 commit)
  uint64_t* pempty = pfull + C::PB;     // partial consumed     (4 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + C::PB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::AS; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int s = 0; s < C::BS; ++s) {
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], 1);
    }
    for (int b = 0; b < C::PB; ++b) {
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], 4);
    }
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
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
      Ring ar, br;
      int a_issued = 0, b_issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles_total && ok; tile += gridDim.x) {
        const int m0 = (tile % mtiles) * (128 * NSUB), n0 = (tile / mtiles) * 128;
        for (int kb = 0; kb < KB && ok; ++kb) {
          if (!mbar_wait(&bempty[br.slot], br.phase ^ 1u, err, kErrWaitLoad)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bfull[br.slot], C::TILE_BYTES);
          tma_load_2d(sB + br.slot * C::TILE_BYTES, &tm_b, &bfull[br.slot], kb * 128, n0);
          ++b_issued;
          br.next(C::BS);
          for (int t = 0; t < NSUB; ++t) {
            if (!mbar_wait(&aempty[ar.slot], ar.phase ^ 1u, err, kErrWaitLoad)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&afull[ar.slot], C::TILE_BYTES);
            tma_load_2d(sA + ar.slot * C::TILE_BYTES, &tm_a, &afull[ar.slot], kb * 128, m0 + 128 * t);
            ++a_issued;
            ar.next(C::AS);
          }
        }
      }
      // Drain: the last load into every used slot has landed before exit.
      for (int s = 0; s < C::AS && s < a_issued; ++s)
        mbar_wait(&afull[s], last_parity((a_issued - s + C::AS - 1) / C::AS), err, kErrWaitLoad);
      for (int s = 0; s < C::BS && s < b_issued; ++s)
        mbar_wait(&bfull[s], last_parity((b_issued - s + C::BS - 1) / C::BS), err, kErrWaitLoad);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // Descriptors are formed once; stepping through shared memory adds
      // (bytes >> 4) to their start-address field.
      const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(sA));
      const uint64_t bdesc0 = sw128_kmajor_desc(smem_addr(sB));
      Ring ar, br, pr;
      int issued = 0, last_p = 0;
      uint32_t last_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles_total && ok; tile += gridDim.x) {
        for (int kb = 0; kb < KB && ok; ++kb) {
          if (!mbar_wait(&bfull[br.slot], br.phase, err, kErrWaitMma)) {
            ok = false;
            break;
          }
          const uint64_t bd = bdesc0 + static_cast<uint64_t>((br.slot * C::TILE_BYTES) >> 4);
          for (int t = 0; t < NSUB; ++t) {
            if (!mbar_wait(&afull[ar.slot], ar.phase, err, kErrWaitMma) ||
                !mbar_wait(&pempty[pr.slot], pr.phase ^ 1u, err, kErrWaitMma)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint64_t ad = adesc0 + static_cast<uint64_t>((ar.slot * C::TILE_BYTES) >> 4);
            const uint32_t d = tmem + static_cast<uint32_t>(pr.slot * 128);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_f8f6f4_ss(d, ad + 2u * k, bd + 2u * k, C::IDESC, k > 0 ? 1u : 0u);
            tc_commit(&aempty[ar.slot]);
            tc_commit(&pfull[pr.slot]);
            last_p = pr.slot;
            last_phase = pr.phase;
            ++issued;
            ar.next(C::AS);
            pr.next(C::PB);
          }
          if (!ok) break;
          tc_commit(&bempty[br.slot]);
          br.next(C::BS);
        }
      }
      // Drain: all issued MMAs have completed before TMEM is released.
      if (issued > 0) mbar_wait(&pfull[last_p], last_phase, err, kErrWaitMma);
    }
  } else if (((warp - 2) >> 2) < NSUB) {
    // -------------------------------------------------- promotion/epilogue
    const int t = (warp - 2) >> 2;  // token sub-tile
    const int quad = warp & 3;      // TMEM lanes this warp may access
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    Ring pr;
    for (int i = 0; i < t; ++i) pr.next(C::PB);
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles_total && ok; tile += gridDim.x) {
      const int m0 = (tile % mtiles) * (128 * NSUB), n0 = (tile / mtiles) * 128;
      const int m = m0 + 128 * t + row;
      // sx is group-major with ldsx covering whole 128-row tiles, so rows
      // past M read padding (their results are never stored).
      const float* sx_col = sx + (m < M ? m : 0);
      const float* sw_row = sw + static_cast<int64_t>(n0 >> 7) * KB;
      uint64_t acc[64];  // column pairs
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = 0ull;
      float c_next = __ldg(sx_col) * __ldg(sw_row);
      for (int kb = 0; kb < KB; ++kb) {
        const float c = c_next;
        if (kb + 1 < KB) c_next = __ldg(sx_col + (kb + 1) * ldsx) * __ldg(sw_row + kb + 1);
        if (!mbar_wait_warp(&pfull[pr.slot], pr.phase, err, kErrWaitEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        tmem_axpy2<4>(t_lane + static_cast<uint32_t>(pr.slot * 128), c, acc);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[pr.slot]);
        for (int i = 0; i < NSUB; ++i) pr.next(C::PB);
      }
      if (ok && m < M && n0 < N) {
        __nv_bfloat16* yrow = y + static_cast<int64_t>(m) * ldy + n0;
        const int ncols = min(128, N - n0);
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
            for (int e = c; e < ncols; ++e)
              yr[e] = static_cast<uint16_t>((wv[(e - c) >> 1] >> (16 * ((e - c) & 1))) & 0xFFFFu);
          }
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

template <int NSUB>
cudaError_t launch_nsub(const Launch& L, const uint8_t* qx, int64_t ldqx, const float* sx,
                        int64_t ldsx, const uint8_t* q, int64_t ldq, const float* sw, uint16_t* y,
                        int64_t ldy, int64_t M, int64_t N, int64_t K) {
  using C = W8A8Cfg<NSUB>;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, K, M, ldqx, 128, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, ldq, 128, 128))
    return cudaErrorInvalidValue;
  auto kern = w8a8_gemm_kernel<NSUB>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  const int64_t mtiles = cdiv(M, 128 * NSUB), tiles = mtiles * cdiv(N, 128);
  if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(tiles < L.num_sms ? tiles : L.num_sms);
  kern<<<grid, C::THREADS, C::SMEM, L.stream>>>(
      ta, tb, sx, ldsx, sw, reinterpret_cast<__nv_bfloat16*>(y), ldy, static_cast<int>(M),
      static_cast<int>(N), static_cast<int>(cdiv(K, 128)), static_cast<int>(mtiles),
      static_cast<int>(tiles), L.err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_w8a8_gemm(const Launch& L, const uint8_t* qx, int64_t ldqx, const float* sx,
                             int64_t ldsx, const uint8_t* q, int64_t ldq, const float* sw,
                             uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K) {
  if (M <= 128) return launch_nsub<1>(L, qx, ldqx, sx, ldsx, q, ldq, sw, y, ldy, M, N, K);
  return launch_nsub<2>(L, qx, ldqx, sx, ldsx, q, ldq, sw, y, ldy, M, N, K);
}

}  // namespace fp8blk
