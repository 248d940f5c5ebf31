// Block-scaled linear with BF16 activations and E4M3 weights (W8A16) on
// tcgen05:
//   y[m][n] = BF16( sum_kb s[n/128][kb] * P_kb[n][m] ),
//   P_kb[n][m] = sum_{k in slab kb} BF16(E4M3(q[n][k])) * x[m][k]   (FP32),
// i.e. y = x . dequant(W)^T (FastVideo PR #1829, "Purpose") with the block
// scale applied to each 128-wide K slab's FP32 partial. Every E4M3 value is
// exactly representable in BF16, so the tensor cores see the exact weights.
//
// The product is computed transposed ("swap AB"): the 128 weight rows of a
// CTA are the MMA's M dimension and a tile of BT tokens is its N dimension,
// so small token counts (decode-like M = 1..64) still fill the 128-row MMA.
// The weight slab is expanded FP8 -> BF16 by converter warps straight into
// TMEM, where tcgen05.mma reads its A operand; shared memory only holds the
// FP8 bytes (read once) and the BF16 activation tile.
//
// Warp roles (320 threads):
//   warp 0     TMA producer: q tile [128 x 128 B] + x tile [BT x 128 BF16]
//              (two 64-element, 128-byte-swizzled atoms) per slab;
//   warp 1     TMEM allocator and MMA issuer: 8 x (M=128, N=BT, K=16) per
//              slab, A from TMEM, B from shared memory, fresh partial;
//   warps 2-5  expansion: one weight row per thread, 128 codes -> 64 bf16x2
//              words -> tcgen05.st into one of two TMEM A buffers;
//   warps 6-9  promotion/epilogue: acc[BT] += P * s in registers, then BF16
//              stores of y (coalesced along n).
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {
namespace {

template <int BT>
struct W8A16Cfg {
  static constexpr int Q_BYTES = 128 * 128;      // FP8 weight slab
  static constexpr int X_ATOM = BT * 128;         // BT rows x 64 BF16 (128 B)
  static constexpr int X_BYTES = 2 * X_ATOM;
  static constexpr int STAGE_BYTES = Q_BYTES + X_BYTES;
  static constexpr int STAGES = BT >= 128 ? 4 : (BT >= 64 ? 6 : 8);
  static constexpr int THREADS = 320;
  static constexpr int TMEM_A = 0;                // 2 buffers x 64 columns
  static constexpr int TMEM_P = 128;              // 2 buffers x BT columns
  static constexpr int TMEM_USED = 128 + 2 * BT;
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static constexpr size_t BAR_BYTES = 256;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = make_idesc(1u, 1u, 128, BT);  // BF16 x BF16 -> F32
  static_assert(BT % 16 == 0 && BT >= 16 && BT <= 128, "MMA N for M=128");
  static_assert(2 * STAGES * 8 + 8 * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(STAGES * STAGE_BYTES + 1024 + BAR_BYTES <= 227 * 1024, "shared memory");
};

// Expand 16 E4M3 codes (one 16-byte chunk) into 8 bf16x2 words.
__device__ __forceinline__ void expand16(const uint4& c, uint32_t* o) {
  o[0] = e4m3x2_to_bf16x2(c.x);
  o[1] = e4m3x2_to_bf16x2(c.x >> 16);
  o[2] = e4m3x2_to_bf16x2(c.y);
  o[3] = e4m3x2_to_bf16x2(c.y >> 16);
  o[4] = e4m3x2_to_bf16x2(c.z);
  o[5] = e4m3x2_to_bf16x2(c.z >> 16);
  o[6] = e4m3x2_to_bf16x2(c.w);
  o[7] = e4m3x2_to_bf16x2(c.w >> 16);
}

template <int BT>
__global__ void __launch_bounds__(320, 1)
    w8a16_gemm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_x,
                      const float* __restrict__ sw, __nv_bfloat16* __restrict__ y, int64_t ldy,
                      int M, int N, int KB, unsigned* __restrict__ err) {
  using C = W8A16Cfg<BT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sQ = smem;                                   // STAGES x Q_BYTES
  uint8_t* sX = smem + C::STAGES * C::Q_BYTES;          // STAGES x X_BYTES
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                  // TMA landed            (1 arrival + tx)
  uint64_t* empty = bars + C::STAGES;     // stage reusable        (4 expanders + 1 commit)
  uint64_t* afull = bars + 2 * C::STAGES; // A buffer written      (4 expanders)
  uint64_t* aempty = afull + 2;           // A buffer consumed     (1 commit)
  uint64_t* pfull = afull + 4;            // partial ready         (1 commit)
  uint64_t* pempty = afull + 6;           // partial consumed      (4 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(afull + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Token tiles of one weight tile are adjacent in the grid (shared through L2).
  const int m0 = blockIdx.x * BT, n0 = blockIdx.y * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 5);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 4);
      mbar_init(&aempty[b], 1);
      mbar_init(&pfull[b], 1);
      mbar_init(&pempty[b], 4);
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
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_x);
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, err, kErrWaitLoad)) break;
        mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
        uint8_t* xs = sX + stage * C::X_BYTES;
        tma_load_2d(sQ + stage * C::Q_BYTES, &tm_q, &full[stage], kb * 128, n0);
        tma_load_2d(xs, &tm_x, &full[stage], kb * 128, m0);
        tma_load_2d(xs + C::X_ATOM, &tm_x, &full[stage], kb * 128 + 64, m0);
        ++issued;
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      for (int s = 0; s < C::STAGES && s < issued; ++s)
        mbar_wait(&full[s], last_parity((issued - s + C::STAGES - 1) / C::STAGES), err, kErrWaitLoad);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // The x tile of a stage has landed once the expansion warps report the
      // A buffer full (they waited on the stage's TMA barrier first), so the
      // MMA thread waits only on afull and pempty. Descriptors are formed
      // once; stepping through shared memory adds (bytes >> 4) to them.
      const uint64_t xdesc0 = sw128_kmajor_desc(smem_addr(sX));
      int stage = 0, buf = 0, issued = 0;
      uint32_t bphase = 0;
      for (int kb = 0; kb < KB; ++kb) {
        if (!mbar_wait(&afull[buf], bphase, err, kErrWaitMma)) break;
        if (!mbar_wait(&pempty[buf], bphase ^ 1u, err, kErrWaitMma)) break;
        tc_fence_after_sync();
        const uint64_t xd = xdesc0 + static_cast<uint64_t>((stage * C::X_BYTES) >> 4);
        const uint32_t d = tmem + static_cast<uint32_t>(C::TMEM_P + buf * BT);
        const uint32_t a = tmem + static_cast<uint32_t>(C::TMEM_A + buf * 64);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_f16_ts(d, a + 8u * k, xd + static_cast<uint64_t>(((k >> 2) * C::X_ATOM + (k & 3) * 32) >> 4),
                     C::IDESC, k > 0 ? 1u : 0u);
        tc_commit(&empty[stage]);
        tc_commit(&aempty[buf]);
        tc_commit(&pfull[buf]);
        ++issued;
        if (++stage == C::STAGES) stage = 0;
        if (++buf == 2) {
          buf = 0;
          bphase ^= 1u;
        }
      }
      if (issued > 0) {
        const int b = (issued - 1) & 1;
        mbar_wait(&pfull[b], last_parity((issued - b + 1) / 2), err, kErrWaitMma);
      }
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------- expansion
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // weight row within the tile == TMEM lane
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    int stage = 0, buf = 0;
    uint32_t phase = 0, bphase = 0;
    for (int kb = 0; kb < KB; ++kb) {
      if (!mbar_wait_warp(&full[stage], phase, err, kErrWaitExpand)) break;
      // Row r of the 128-byte-swizzled slab: 16-byte chunk c sits at chunk
      // position c ^ (r & 7).
      const uint8_t* qrow = sQ + stage * C::Q_BYTES + r * 128;
      uint4 c[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        c[j] = *reinterpret_cast<const uint4*>(qrow + ((j ^ (r & 7)) << 4));
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (!mbar_wait_warp(&aempty[buf], bphase ^ 1u, err, kErrWaitExpand)) break;
      tc_fence_after_sync();
      const uint32_t ta = t_lane + static_cast<uint32_t>(C::TMEM_A + buf * 64);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
#pragma unroll
        for (int j = 0; j < 4; ++j) expand16(c[4 * h + j], o + 8 * j);
        tmem_st32x32(ta + 32u * h, o);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[buf]);
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1u;
      }
    }
  } else {
    // -------------------------------------------------- promotion/epilogue
    const int quad = warp & 3;
    const int n = n0 + quad * 32 + lane;
    const float* sw_row = sw + static_cast<int64_t>(blockIdx.y) * KB;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16) + C::TMEM_P;
    float acc[BT];
#pragma unroll
    for (int i = 0; i < BT; ++i) acc[i] = 0.0f;
    int buf = 0;
    uint32_t bphase = 0;
    float s_next = __ldg(sw_row);
    bool ok = true;
    for (int kb = 0; kb < KB; ++kb) {
      const float s = s_next;
      if (kb + 1 < KB) s_next = __ldg(sw_row + kb + 1);
      if (!mbar_wait_warp(&pfull[buf], bphase, err, kErrWaitEpilogue)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t = t_lane + static_cast<uint32_t>(buf * BT);
      if constexpr (BT == 16) {
        uint32_t p[16];
        tmem_ld32x16(t, p);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = fmaf(__uint_as_float(p[i]), s, acc[i]);
      } else {
        tmem_axpy<BT / 32>(t, s, acc);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pempty[buf]);
      if (++buf == 2) {
        buf = 0;
        bphase ^= 1u;
      }
    }
    if (ok && n < N) {
      uint16_t* ycol = reinterpret_cast<uint16_t*>(y) + n;
      const int mcount = min(BT, M - m0);
#pragma unroll
      for (int j = 0; j < BT; ++j)
        if (j < mcount)
          ycol[static_cast<int64_t>(m0 + j) * ldy] =
              static_cast<uint16_t>(cvt_bf16x2(0.0f, acc[j]) & 0xFFFFu);
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

template <int BT>
cudaError_t launch_bt(const Launch& L, const uint16_t* x, int64_t ldx, const uint8_t* q,
                      int64_t ldq, const float* sw, uint16_t* y, int64_t ldy, int64_t M,
                      int64_t N, int64_t K) {
  using C = W8A16Cfg<BT>;
  CUtensorMap tq, tx;
  if (!make_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, ldq, 128, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, ldx * 2, 64, BT))
    return cudaErrorInvalidValue;
  auto kern = w8a16_gemm_kernel<BT>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(cdiv(M, BT)), static_cast<unsigned>(cdiv(N, 128)));
  kern<<<grid, C::THREADS, C::SMEM, L.stream>>>(tq, tx, sw, reinterpret_cast<__nv_bfloat16*>(y),
                                                ldy, static_cast<int>(M), static_cast<int>(N),
                                                static_cast<int>(cdiv(K, 128)), L.err);
  return cudaGetLastError();
}

}  // namespace

size_t w8a16_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

cudaError_t launch_w8a16_gemm(const Launch& L, const uint16_t* x, int64_t ldx, const uint8_t* q,
                              int64_t ldq, const float* sw, uint16_t* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, void*, size_t) {
  if (cdiv(N, 128) > 65535) return cudaErrorInvalidValue;
  if (M <= 16) return launch_bt<16>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K);
  if (M <= 32) return launch_bt<32>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K);
  if (M <= 64) return launch_bt<64>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K);
  return launch_bt<128>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K);
}

}  // namespace fp8blk
