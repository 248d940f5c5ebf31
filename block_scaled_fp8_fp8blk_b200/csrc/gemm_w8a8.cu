// Block-scaled FP8 x FP8 linear (W8A8) on tcgen05:
//   y[m][n] = BF16( sum_kb sx[kb][m] * s[n/128][kb] * P_kb[m][n] ),
//   P_kb = (128-wide K slab of qx) . (same slab of q)^T, E4M3 x E4M3 -> FP32.
// FastVideo PR #1829, "Purpose": the linear is x times the dequantized weight,
// computed the way the Blackwell groupwise GEMM does it (scales applied per
// 128-wide K group). The scales are arbitrary floats, not powers of two, and
// the weight blocks are 128 x 128, so they are applied in software to each
// slab's FP32 partial ("promotion") rather than by the MMA.
//
// Persistent kernel: one CTA per SM walks output tiles of 128 tokens by 256
// weight rows (two weight blocks) in raster groups (tile_coords): the token
// tiles of one weight tile are neighbours and share it through L2, and a
// group of token tiles (at most 24 MB of activation codes) meets every
// weight tile before the next group starts.
// Every ring runs on across tiles, so the next tile's loads and MMAs overlap
// this tile's stores.
//
// The single-thread control loops set the pace on this part: a commit stalls
// its issuer's MMA stream for a few hundred cycles and every barrier or TMA
// operation costs on the order of a hundred cycles of that thread's time. So
// the work per control operation is made large (one N=256 MMA covers a whole
// 128 x 256 x 32 step; one stage barrier covers a whole slab), the control
// work is spread over four threads, and ring positions are powers of two.
//   warp 0     TMA producer of the activation slab [128 x 128 B] per stage;
//   warp 1     TMA producer of the weight slab [256 x 128 B] per stage;
//   warp 2, 3  MMA issuers: issuer e takes the slabs j with j % 2 == e, each
//              4 x (M=128, N=256, K=32) into its own 256-column TMEM partial,
//              then one commit to the slab's "done" barrier. While one issuer
//              waits or commits, the other's MMAs keep the tensor pipe busy.
//              (warp 2 also allocates TMEM.)
//   warps 4-11 promotion/epilogue: warp 4 + 4h + q owns TMEM lane quadrant q
//              (32 token rows) and partial columns [128h, 128h + 128), i.e.
//              weight block n0/128 + h, so each thread's scale per slab is
//              c = sx[kb][m] * s[n0/128 + h][kb]: acc += P * c with packed
//              FP32x2 FMAs. At the end of a tile the warp writes its 32 x 128
//              BF16 block, 64 columns at a time, into a 128B-swizzled staging
//              buffer and TMA-stores it. The store clips rows at M and columns
//              at N rounded down to 8 (the bulk copy moves whole 16-byte
//              chunks); the last < 8 columns of a ragged N are written from
//              the staging buffer with plain stores.
// Every wait is bounded (kWaitLimitCycles) and reports to the error word.
#include <cuda_bf16.h>

#include <cstring>

#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {
namespace {

struct W8A8Cfg {
  static constexpr int BM = 128;                          // tokens per tile (MMA M)
  static constexpr int BN = 256;                          // weight rows per tile (MMA N)
  static constexpr int A_BYTES = BM * 128;                // activation slab
  static constexpr int B_BYTES = BN * 128;                // weight slab
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // one K slab of both operands
  static constexpr int ST = 4;                            // stages (power of two)
  static constexpr int RD = 8;                            // "slab done" ring (power of two)
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 128 + 32 * EPI_WARPS;
  static constexpr int OUT_BYTES = 32 * 128;              // per epilogue warp: 32 rows x 64 BF16
  static constexpr int NBAR = ST + RD + 2;
  static constexpr size_t SMEM_TILES =
      static_cast<size_t>(ST) * STAGE_BYTES + static_cast<size_t>(EPI_WARPS) * OUT_BYTES;
  static constexpr size_t SMEM = 1024 + SMEM_TILES + 8 * NBAR + 16;
  static constexpr uint32_t IDESC = make_idesc(0u, 0u, BM, BN);  // E4M3 x E4M3 -> F32
  // The launch gives 384 threads x 168 registers; the control warpgroup keeps
  // 56 and the two epilogue warpgroups take 224 each (128 x (56 + 2 x 224)).
  static constexpr int REG_CTRL = 56, REG_EPI = 224, REG_LAUNCH = 168;
  static_assert(128 * (REG_CTRL + 2 * REG_EPI) <= THREADS * REG_LAUNCH, "register split");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert((ST & (ST - 1)) == 0 && (RD & (RD - 1)) == 0, "power-of-two rings");
  // Slab j's "done" barrier is reused by slab j + RD, which must not complete
  // before every waiter on slab j has passed: the producers wait on slab j
  // before loading slab j + ST (RD >= ST keeps slab j + RD's loads behind
  // that wait), and the promotion warps wait on slab j before releasing the
  // partial of slab j, which slab j + 2 (same issuer, same TMEM slot) waits
  // for (RD >= 2).
  static_assert(RD >= ST && RD >= 2 && RD % 2 == 0, "done ring depth");
};

// Bounded wait on `bar` for the phase parity of its use `use` (0, 1, 2, ...).
__device__ __forceinline__ bool wait_use(uint64_t* bar, int use, unsigned* err, unsigned flag) {
  return mbar_wait(bar, static_cast<uint32_t>(use & 1), err, flag);
}

__global__ void __launch_bounds__(W8A8Cfg::THREADS, 1)
    w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_y, const float* __restrict__ sx,
                     int64_t ldsx, const float* __restrict__ sw, uint16_t* __restrict__ y,
                     int64_t ldy, int M, int N, int n_tma, int KB, int mtiles, int ntiles_total,
                     int gm, int a_bytes, unsigned* __restrict__ err) {
  using C = W8A8Cfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;                            // ST stages: A then B
  uint8_t* sOut = smem + C::ST * C::STAGE_BYTES;             // EPI_WARPS x 4 KB staging
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_TILES);
  uint64_t* full = bars;               // stage landed       (2 producers + tx)
  uint64_t* done = full + C::ST;       // slab's MMAs done   (1 commit)
  uint64_t* pempty = done + C::RD;     // partial consumed   (8 epilogue warps), one per issuer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles_n = ntiles_total / mtiles;
  const int my_tiles =
      static_cast<int>(blockIdx.x) < ntiles_total ? (ntiles_total - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int total_slabs = my_tiles * KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::ST; ++s) mbar_init(&full[s], 2);
    for (int b = 0; b < C::RD; ++b) mbar_init(&done[b], 1);
    for (int b = 0; b < 2; ++b) mbar_init(&pempty[b], C::EPI_WARPS);
    mbar_init_fence();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // The next kernel in the stream may be scheduled now; it reads y after its
  // own griddepcontrol.wait.
  pdl_launch_dependents();

  // Each warpgroup sets its register budget at the top of its role.
  if (warp < 4) {
    setmaxnreg_dec<C::REG_CTRL>();
    if (warp < 2 && lane == 0) {
      // ------------------------------------------------- producers (A, B)
      const bool is_a = warp == 0;
      const CUtensorMap* map = is_a ? &tm_a : &tm_b;
      const uint32_t bytes = is_a ? static_cast<uint32_t>(a_bytes) : C::B_BYTES;
      uint8_t* dst0 = smem + (is_a ? 0 : C::A_BYTES);
      tma_prefetch_map(map);
      // Launched as a programmatic dependent of the activation quantizer:
      // the weights may stream at once, the activation codes only once that
      // kernel has completed (a no-op for an ordinary launch).
      if (is_a) pdl_wait();
      int j = 0;  // slab counter (across tiles)
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles_total && ok; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, mtiles, ntiles_n, gm, mt, nt);
        const int row0 = is_a ? mt * C::BM : nt * C::BN;
        for (int kb = 0; kb < KB; ++kb, ++j) {
          const int stage = j & (C::ST - 1);
          if (j >= C::ST) {  // the slab that last used this stage has finished
            const int jo = j - C::ST;
            if (!wait_use(&done[jo & (C::RD - 1)], jo / C::RD, err, kErrWaitLoad)) {
              ok = false;
              break;
            }
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(dst0 + stage * C::STAGE_BYTES, map, &full[stage], kb * 128, row0);
        }
      }
      // Drain: the loads of the last stages have landed before the CTA may
      // exit (on a time-out the other producer's half may be missing; the
      // waits are bounded).
      for (int jj = (j > C::ST ? j - C::ST : 0); jj < j; ++jj)
        wait_use(&full[jj & (C::ST - 1)], jj / C::ST, err, kErrWaitLoad);
    } else if (warp >= 2 && lane == 0) {
      // ----------------------------------------------------- MMA issuers
      const int e = warp - 2;
      const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(smem));
      const uint64_t bdesc0 = sw128_kmajor_desc(smem_addr(smem + C::A_BYTES));
      const uint32_t d = tmem + static_cast<uint32_t>(e * C::BN);
      int last = -1;
      for (int j = e; j < total_slabs; j += 2) {
        if (!wait_use(&full[j & (C::ST - 1)], j / C::ST, err, kErrWaitMma)) break;
        const int u = j >> 1;  // use of this issuer's partial
        if (u >= 1 && !wait_use(&pempty[e], u - 1, err, kErrWaitMma)) break;
        tc_fence_after_sync();
        const uint64_t soff = static_cast<uint64_t>(((j & (C::ST - 1)) * C::STAGE_BYTES) >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_f8f6f4_ss(d, adesc0 + soff + 2u * k, bdesc0 + soff + 2u * k, C::IDESC, k > 0 ? 1u : 0u);
        tc_commit(&done[j & (C::RD - 1)]);
        last = j;
      }
      // Drain: this issuer's MMAs have completed before TMEM is released.
      if (last >= 0) wait_use(&done[last & (C::RD - 1)], last / C::RD, err, kErrWaitMma);
    }
  } else {
    setmaxnreg_inc<C::REG_EPI>();
    // -------------------------------------------------- promotion/epilogue
    pdl_wait();  // the activation scales come from the kernel before
    const int ew = warp - 4;
    const int quad = warp & 3;  // TMEM lanes this warp may access
    const int h = ew >> 2;      // partial columns [128h, 128h + 128)
    const int row = quad * 32 + lane;
    const uint32_t t_lane =
        tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(h * 128);
    uint8_t* stage = sOut + ew * C::OUT_BYTES;
    uint8_t* srow = stage + lane * 128;
    int j = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles_total && ok; tile += gridDim.x) {
      int mt, nt;
      tile_coords(tile, mtiles, ntiles_n, gm, mt, nt);
      const int m0 = mt * C::BM;
      const int col0 = nt * C::BN + 128 * h;  // first output column of this warp
      const bool has_cols = col0 < N;
      const int m = m0 + row;
      // sx is group-major with ldsx covering whole 128-row tiles, so rows
      // past M read padding (their results are never stored).
      const float* sx_col = sx + (m < M ? m : 0);
      const float* sw_row = sw + static_cast<int64_t>(has_cols ? (col0 >> 7) : 0) * KB;
      uint64_t acc[64];  // column pairs
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = 0ull;
      // The two scale factors of a slab are loaded one slab ahead and only
      // multiplied when used, so the product does not wait on the loads.
      float fx = has_cols ? __ldg(sx_col) : 0.0f, fw = has_cols ? __ldg(sw_row) : 0.0f;
      for (int kb = 0; kb < KB; ++kb, ++j) {
        const float c = fx * fw;
        if (has_cols && kb + 1 < KB) { fx = __ldg(sx_col + (kb + 1) * ldsx); fw = __ldg(sw_row + kb + 1); }
        if (!mbar_wait_warp(&done[j & (C::RD - 1)], static_cast<uint32_t>((j / C::RD) & 1), err,
                            kErrWaitEpilogue)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        tmem_axpy2<4>(t_lane + static_cast<uint32_t>((j & 1) * C::BN), c, acc);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[j & 1]);
      }
      if (!ok) break;
      // Output, 64 columns at a time: the staging buffer's previous store has
      // been read out; 16-byte chunk c of row r sits at chunk position
      // c ^ (r % 8) (the 128-byte swizzle the store expects).
      const int r0 = m0 + quad * 32;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int base = col0 + 64 * hh;
        if (lane == 0) tma_store_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int p = 32 * hh + 4 * c;
          uint4 o;
          o.x = cvt_bf16x2_pair(acc[p + 0]);
          o.y = cvt_bf16x2_pair(acc[p + 1]);
          o.z = cvt_bf16x2_pair(acc[p + 2]);
          o.w = cvt_bf16x2_pair(acc[p + 3]);
          *reinterpret_cast<uint4*>(srow + ((c ^ (lane & 7)) << 4)) = o;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && r0 < M && base < n_tma) {
          tma_store_2d(&tm_y, stage, base, r0);
          tma_store_commit();
        }
        if (n_tma < N && n_tma >= base && n_tma < base + 64 && m < M) {
          const int cl = n_tma - base;  // first tail column within these 64
          const uint16_t* src =
              reinterpret_cast<const uint16_t*>(srow + (((cl >> 3) ^ (lane & 7)) << 4));
          uint16_t* dst = y + static_cast<int64_t>(m) * ldy + n_tma;
          for (int e = 0; e < N - n_tma; ++e) dst[e] = src[e];
        }
      }
    }
    if (lane == 0) tma_store_wait_all();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_w8a8_gemm(const Launch& L, const uint8_t* qx, int64_t ldqx, const float* sx,
                             int64_t ldsx, const uint8_t* q, int64_t ldq, const float* sw,
                             uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                             bool after_act_quant) {
  using C = W8A8Cfg;
  CUtensorMap ta, tb, ty;
  // Fewer than BM tokens: load only the first round_up(M, 8) activation rows
  // of a slab. The MMA still reads BM rows; the rows past those only reach
  // output rows >= M, which are never stored.
  const int64_t a_rows = M < C::BM ? round_up(M, 8) : C::BM;
  if (!make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, K, M, ldqx, 128,
                    static_cast<uint32_t>(a_rows)))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, ldq, 128, C::BN))
    return cudaErrorInvalidValue;
  // The output map covers columns [0, N rounded down to 8); none if N < 8.
  const int64_t n_tma = N & ~int64_t{7};
  if (n_tma > 0) {
    if (!make_tmap_2d(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, n_tma, M, 2 * ldy, 64, 32))
      return cudaErrorInvalidValue;
  } else {
    memset(&ty, 0, sizeof(ty));
  }
  auto kern = w8a8_gemm_kernel;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  {
    // The register split needs the launch allocation it was sized for
    // (checked once).
    static const cudaError_t regs = [&] {
      cudaFuncAttributes fa;
      cudaError_t r = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kern));
      if (r != cudaSuccess) return r;
      return fa.numRegs < C::REG_LAUNCH ? cudaErrorInvalidConfiguration : cudaSuccess;
    }();
    if (regs != cudaSuccess) return regs;
  }
  const int64_t mtiles = cdiv(M, C::BM), tiles = mtiles * cdiv(N, C::BN);
  // Slab counters are 32-bit per CTA.
  if (tiles * cdiv(K, 128) > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int grid = static_cast<int>(tiles < L.num_sms ? tiles : L.num_sms);
  // After the activation quantizer: a programmatic dependent launch, so the
  // GEMM's set-up and weight loads overlap that kernel.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = after_act_quant ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, sx, ldsx, sw, y, ldy, static_cast<int>(M),
                            static_cast<int>(N), static_cast<int>(n_tma),
                            static_cast<int>(cdiv(K, 128)), static_cast<int>(mtiles),
                            static_cast<int>(tiles), raster_group(mtiles, C::BM * K, kRasterBytesW8A8),
                            static_cast<int>(a_rows * 128), L.err);
}

}  // namespace fp8blk
