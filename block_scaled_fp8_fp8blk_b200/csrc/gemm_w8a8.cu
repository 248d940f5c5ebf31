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
// tiles, so the next tile's loads and MMAs overlap this tile's stores. The
// MMA thread commits once per sub-tile group ("item" i = NSUB * slab + t) to
// a ring of "item done" barriers read by every consumer (the producer
// recycling operand slots, the promotion warps reading partials).
//   warp 0     TMA producer: per slab one q tile [128 x 128 B] into the B ring
//              and NSUB qx sub-tiles [128 x 128 B] into the A ring;
//   warp 1     TMEM allocator and MMA issuer: per item 4 x (M=128, N=128,
//              K=32) into a 4-deep ring of TMEM partials;
//   warps 2-3  idle (they complete the first warpgroup);
//   warps 4..  promotion/epilogue, one warpgroup per sub-tile: warp 4 + 4t + q
//              owns TMEM lane quadrant q of sub-tile t; each thread owns one
//              token row:
//              acc += P * (sx[m] * s) with packed FP32x2 FMAs; at the end of
//              a tile the warp writes its 32 x 128 BF16 block into a
//              128B-swizzled staging buffer and TMA-stores it. The store
//              clips rows at M and columns at N rounded down to 8 (the bulk
//              copy moves whole 16-byte chunks); the last < 8 columns of a
//              ragged N are written from the staging buffer with plain stores.
// Every wait is bounded (kWaitLimitCycles) and reports to the error word.
#include <cuda_bf16.h>

#include <cstring>

#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {
namespace {

template <int NSUB>
struct W8A8Cfg {
  static constexpr int TILE_BYTES = 128 * 128;  // one 128 x 128 FP8 operand tile
  static constexpr int AS = 6;                  // A (activation) ring depth (items)
  static constexpr int BS = NSUB == 2 ? 4 : 6;  // B (weight) ring depth (slabs)
  static constexpr int PB = 4;                  // TMEM partial ring depth (x 128 columns)
  static constexpr int RD = 8;                  // "item done" barrier ring depth
  static constexpr int EPI_WARPS = 4 * NSUB;
  static constexpr int THREADS = 128 + 32 * EPI_WARPS;
  // With two epilogue warpgroups the registers are rebalanced with setmaxnreg:
  // the launch gives 384 threads x 168 registers, the control warpgroup keeps
  // 56 and the epilogue warpgroups take 224 each (128 x (56 + 2 x 224)).
  static constexpr int REG_CTRL = 56, REG_EPI = 224, REG_LAUNCH = 168;
  static_assert(NSUB == 1 || 128 * (REG_CTRL + 2 * REG_EPI) <= THREADS * REG_LAUNCH,
                "register split");
  static constexpr int STAGE_BYTES = 2 * 32 * 128;  // per epilogue warp: 32 rows x 128 BF16
  static constexpr int NBAR = AS + BS + RD + PB;
  static constexpr size_t SMEM_TILES =
      static_cast<size_t>(AS + BS) * TILE_BYTES + static_cast<size_t>(EPI_WARPS) * STAGE_BYTES;
  static constexpr size_t SMEM = 1024 + SMEM_TILES + 8 * NBAR + 16;
  static constexpr uint32_t IDESC = make_idesc(0u, 0u, 128, 128);  // E4M3 x E4M3 -> F32
  static_assert(SMEM <= 227 * 1024, "shared memory");
  // Item i's "done" barrier is reused by item i + RD; every waiter on item i
  // must pass its wait before item i + RD can complete. The producer waits on
  // item i - AS before loading A for item i and on the last item of slab
  // j - BS before loading B for slab j; the promotion warps of sub-tile t
  // consume item i + RD - PB (same t) before the MMA may write its slot again.
  static_assert(RD >= AS && RD >= NSUB * BS && RD >= PB && (RD - PB) % NSUB == 0,
                "done ring depth");
};

__device__ __forceinline__ uint32_t ring_parity(int item, int depth) {
  return static_cast<uint32_t>((item / depth) & 1);
}

template <int NSUB>
__global__ void __launch_bounds__(W8A8Cfg<NSUB>::THREADS, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_y, const float* __restrict__ sx,
                     int64_t ldsx, const float* __restrict__ sw, uint16_t* __restrict__ y,
                     int64_t ldy, int M, int N, int n_tma, int KB, int mtiles, int ntiles_total,
                     unsigned* __restrict__ err) {
  using C = W8A8Cfg<NSUB>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sA = smem;                              // AS x 16 KB
  uint8_t* sB = smem + C::AS * C::TILE_BYTES;      // BS x 16 KB
  uint8_t* sY = sB + C::BS * C::TILE_BYTES;        // EPI_WARPS x 8 KB output staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_TILES);
  uint64_t* afull = bars;               // qx sub-tile landed   (1 arrival + tx)
  uint64_t* bfull = afull + C::AS;      // q tile landed        (1 arrival + tx)
  uint64_t* done = bfull + C::BS;       // item's MMAs complete (1 commit)
  uint64_t* pempty = done + C::RD;      // partial consumed     (4 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + C::PB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int my_tiles =
      static_cast<int>(blockIdx.x) < ntiles_total ? (ntiles_total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int total_slabs = my_tiles * KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::AS; ++s) mbar_init(&afull[s], 1);
    for (int s = 0; s < C::BS; ++s) mbar_init(&bfull[s], 1);
    for (int b = 0; b < C::RD; ++b) mbar_init(&done[b], 1);
    for (int b = 0; b < C::PB; ++b) mbar_init(&pempty[b], 4);
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

  // Each warpgroup sets its register budget at the top of its role.
  if (warp < 4) {
    if constexpr (NSUB == 2) setmaxnreg_dec<C::REG_CTRL>();
    if (warp == 0) {
      if (lane == 0) {
        tma_prefetch_map(&tm_a);
        tma_prefetch_map(&tm_b);
        int j = 0, a_issued = 0, b_issued = 0;  // slab counter (across tiles)
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles_total && ok; tile += gridDim.x) {
          const int m0 = (tile % mtiles) * (128 * NSUB), n0 = (tile / mtiles) * 128;
          for (int kb = 0; kb < KB && ok; ++kb, ++j) {
            const int bs = j % C::BS;
            // A slot is refilled once the last item that read it has finished.
            const int ib = NSUB * (j - C::BS) + NSUB - 1;
            if (j >= C::BS &&
                !mbar_wait_sleepy(&done[ib % C::RD], ring_parity(ib, C::RD), err, kErrWaitLoad)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bfull[bs], C::TILE_BYTES);
            tma_load_2d(sB + bs * C::TILE_BYTES, &tm_b, &bfull[bs], kb * 128, n0);
            ++b_issued;
            for (int t = 0; t < NSUB; ++t) {
              const int i = j * NSUB + t, as = i % C::AS;
              if (i >= C::AS) {
                const int io = i - C::AS;
                if (!mbar_wait_sleepy(&done[io % C::RD], ring_parity(io, C::RD), err, kErrWaitLoad)) {
                  ok = false;
                  break;
                }
              }
              mbar_arrive_expect_tx(&afull[as], C::TILE_BYTES);
              tma_load_2d(sA + as * C::TILE_BYTES, &tm_a, &afull[as], kb * 128, m0 + 128 * t);
              ++a_issued;
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
        int i = 0;  // items issued
        bool ok = true;
        for (int j = 0; j < total_slabs && ok; ++j) {
          if (!mbar_wait(&bfull[j % C::BS], ring_parity(j, C::BS), err, kErrWaitMma)) break;
          const uint64_t bd = bdesc0 + static_cast<uint64_t>(((j % C::BS) * C::TILE_BYTES) >> 4);
#pragma unroll
          for (int t = 0; t < NSUB; ++t) {
            ok = mbar_wait(&afull[i % C::AS], ring_parity(i, C::AS), err, kErrWaitMma) &&
                 (i < C::PB ||
                  mbar_wait(&pempty[i % C::PB], ring_parity(i - C::PB, C::PB), err, kErrWaitMma));
            if (!ok) break;
            tc_fence_after_sync();
            const uint64_t ad = adesc0 + static_cast<uint64_t>(((i % C::AS) * C::TILE_BYTES) >> 4);
            const uint32_t d = tmem + static_cast<uint32_t>((i % C::PB) * 128);
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_f8f6f4_ss(d, ad + 2u * k, bd + 2u * k, C::IDESC, k > 0 ? 1u : 0u);
            tc_commit(&done[i % C::RD]);
            ++i;
          }
        }
        // Drain: all issued MMAs have completed before TMEM is released.
        if (i > 0) mbar_wait(&done[(i - 1) % C::RD], ring_parity(i - 1, C::RD), err, kErrWaitMma);
      }
    }
  } else {
    if constexpr (NSUB == 2) setmaxnreg_inc<C::REG_EPI>();
    // -------------------------------------------------- promotion/epilogue
    const int t = (warp - 4) >> 2;  // token sub-tile
    const int quad = warp & 3;      // TMEM lanes this warp may access
    const int row = quad * 32 + lane;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    uint8_t* stage = sY + (warp - 4) * C::STAGE_BYTES;
    int j = 0;
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
      for (int kb = 0; kb < KB; ++kb, ++j) {
        const float c = c_next;
        if (kb + 1 < KB) c_next = __ldg(sx_col + (kb + 1) * ldsx) * __ldg(sw_row + kb + 1);
        const int i = j * NSUB + t;
        if (!mbar_wait_warp(&done[i % C::RD], ring_parity(i, C::RD), err, kErrWaitEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        const int slot = i % C::PB;
        tmem_axpy2<4>(t_lane + static_cast<uint32_t>(slot * 128), c, acc);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[slot]);
      }
      if (!ok) break;
      // Output: the staging buffer's previous store has been read out; rows
      // are 128 B (64 columns) per half, 16-byte chunk c of row r sits at
      // chunk position c ^ (r % 8) (the 128-byte swizzle the store expects).
      const int r0 = m0 + 128 * t + quad * 32;
      if (lane == 0) tma_store_wait_read<0>();
      __syncwarp();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint8_t* srow = stage + h * 4096 + lane * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int p = 32 * h + 4 * c;
          uint4 o;
          o.x = cvt_bf16x2_pair(acc[p + 0]);
          o.y = cvt_bf16x2_pair(acc[p + 1]);
          o.z = cvt_bf16x2_pair(acc[p + 2]);
          o.w = cvt_bf16x2_pair(acc[p + 3]);
          *reinterpret_cast<uint4*>(srow + ((c ^ (lane & 7)) << 4)) = o;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && r0 < M && n0 < n_tma) {
        tma_store_2d(&tm_y, stage, n0, r0);
        if (n0 + 64 < n_tma) tma_store_2d(&tm_y, stage + 4096, n0 + 64, r0);
        tma_store_commit();
      }
      if (n_tma < N && n_tma >= n0 && n_tma < n0 + 128 && m < M) {
        const int cl = n_tma - n0;  // first tail column within the tile
        const uint16_t* src = reinterpret_cast<const uint16_t*>(
            stage + (cl >> 6) * 4096 + lane * 128 + ((((cl & 63) >> 3) ^ (lane & 7)) << 4));
        uint16_t* dst = y + static_cast<int64_t>(m) * ldy + n_tma;
        for (int e = 0; e < N - n_tma; ++e) dst[e] = src[e];
      }
    }
    if (lane == 0) tma_store_wait_all();
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
  CUtensorMap ta, tb, ty;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, K, M, ldqx, 128, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, ldq, 128, 128))
    return cudaErrorInvalidValue;
  // The output map covers columns [0, N rounded down to 8); none if N < 8.
  const int64_t n_tma = N & ~int64_t{7};
  if (n_tma > 0) {
    if (!make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, n_tma, M, 2 * ldy, 64, 32))
      return cudaErrorInvalidValue;
  } else {
    memset(&ty, 0, sizeof(ty));
  }
  auto kern = w8a8_gemm_kernel<NSUB>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  if (NSUB == 2) {
    // The register split needs the launch allocation it was sized for.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kern));
    if (e != cudaSuccess) return e;
    if (fa.numRegs < C::REG_LAUNCH) return cudaErrorInvalidConfiguration;
  }
  const int64_t mtiles = cdiv(M, 128 * NSUB), tiles = mtiles * cdiv(N, 128);
  if (tiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(tiles < L.num_sms ? tiles : L.num_sms);
  kern<<<grid, C::THREADS, C::SMEM, L.stream>>>(
      ta, tb, ty, sx, ldsx, sw, y, ldy, static_cast<int>(M), static_cast<int>(N),
      static_cast<int>(n_tma), static_cast<int>(cdiv(K, 128)), static_cast<int>(mtiles),
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
