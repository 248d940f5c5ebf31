// Block-scaled linear with BF16 activations and E4M3 weights (W8A16) on
// tcgen05:
//   y[m][n] = BF16( sum_kb s[n/128][kb] * P_kb[n][m] ),
//   P_kb[n][m] = sum_{k in slab kb} BF16(E4M3(q[n][k])) * x[m][k]   (FP32),
// i.e. y = x . dequant(W)^T (FastVideo PR #1829, "Purpose") with the block
// scale applied to each 128-wide K slab's FP32 partial. Every E4M3 value is
// exactly representable in BF16, so the tensor cores see the exact weights.
//
// The product is computed transposed ("swap AB"): the 128 weight rows of a
// tile are the MMA's M dimension and the tokens its N dimension, so small
// token counts still fill the 128-row MMA. A weight slab is expanded
// FP8 -> BF16 once, straight into TMEM (the MMA's A operand), and used for
// NSUB token sub-tiles of BT tokens each; the expansion costs no
// shared-memory write traffic.
//
// Persistent kernel: one CTA per SM walks tiles (NSUB x BT tokens by 128
// weight rows) in raster groups (tile_coords: token tiles of one weight tile
// are neighbours in the order, so they share it through L2, and a group of
// token tiles, at most 48 MB of activations, meets every weight tile before
// the next group starts), and every ring runs on across tiles. Each
// sub-tile group ("item" i = NSUB * slab + t) is issued and committed by its
// own MMA thread to a ring of "item done" barriers that every consumer reads
// (the activation producer recycling slots, the expansion warps recycling A
// buffers, the promotion warps reading partials): a commit stalls its
// issuer's MMA stream for a few hundred cycles, and with one issuer per
// sub-tile the other issuer's MMAs fill that gap.
//
// Warp roles (16 warps; registers rebalanced per warpgroup with setmaxnreg):
//   warp 0       TMA producer of weight-code slabs [128 x 128 B] (q ring);
//   warp 1       TMA producer of activation sub-tiles [BT x 128 BF16] (x ring);
//   warps 2, 3   MMA issuers of alternate items: per item 8 x (M=128, N=BT,
//                K=16), A from TMEM, B from shared memory, into a ring of TMEM
//                partials shared in item order (warp 2 also allocates TMEM);
//   warps 4-7    expansion: one weight row per thread (TMEM lane), 128 codes
//                -> 64 bf16x2 words -> tcgen05.st into one of AB A buffers
//                (with one sub-tile, of the even slabs only);
//   warps 8-15   two sub-tiles: promotion/epilogue, acc += P * s with packed
//                FP32x2 FMAs, then BF16 stores of y (coalesced along n);
//                one sub-tile: warps 8-11 promote and store, warps 12-15
//                expand the odd slabs (the conversion is the per-slab cost
//                at small token counts, so two groups overlap it).
// Every wait is bounded (kWaitLimitCycles) and reports to the error word.
#include <cuda_bf16.h>

#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {
namespace {

template <int BT, int NSUB>
struct W8A16Cfg {
  static constexpr int Q_BYTES = 128 * 128;  // FP8 weight slab
  static constexpr int X_ATOM = BT * 128;    // BT rows x 64 BF16 (128 B)
  static constexpr int X_BYTES = 2 * X_ATOM; // one sub-tile slab
  // With one sub-tile two warpgroups expand alternate slabs; the q ring is
  // then even, so each q slot (and its barriers) belongs to one of them.
  static constexpr int NEXP = NSUB == 1 ? 2 : 1;
  // Ring depths (slots of 16 KB weight codes, of BT x 128 activations): at
  // one sub-tile the weight stream from HBM is the cost, and the activations
  // (at most 128 tokens) come from L2, so the weight ring gets the shared
  // memory -- with four weight slots at BT = 64 the expansion warps waited
  // on HBM latency (six: 15% faster on a 262 MB layer at 64 tokens).
  static constexpr int QS = NSUB == 2 ? 3 : (BT >= 64 ? 6 : 8);
  static constexpr int XS = BT >= 128 ? (NSUB == 2 ? 5 : 2) : (BT >= 64 ? 4 : 7);
  static constexpr int THREADS = 512;
  static constexpr int PB = 3;                  // TMEM partial ring depth (items)
  static constexpr int RD = 8;                  // "group done" barrier ring depth (items)
  // Expanded-weight (A) buffers in TMEM, 64 columns each; with one sub-tile
  // the two issuers take alternate slabs, each over AB / 2 of them.
  static constexpr int AB = (NSUB == 1 && BT <= 64) ? 4 : 2;
  static constexpr int TMEM_A = 0;              // AB buffers x 64 columns
  static constexpr int TMEM_P = 64 * AB;        // PB buffers x BT columns
  static constexpr int TMEM_USED = TMEM_P + PB * BT;
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static constexpr int NBAR = 2 * QS + XS + AB + RD + PB * 2;
  static constexpr int OUT_BYTES = 16 * 64;     // per epilogue warp: 16 tokens x 32 BF16
  static constexpr size_t SMEM_TILES = static_cast<size_t>(QS) * Q_BYTES +
                                       static_cast<size_t>(XS) * X_BYTES + 4 * NSUB * OUT_BYTES;
  static constexpr size_t SMEM = 1024 + SMEM_TILES + 8 * NBAR + 16;
  static constexpr uint32_t IDESC = make_idesc(1u, 1u, 128, BT);  // BF16 x BF16 -> F32
  static_assert(BT % 16 == 0 && BT >= 16 && BT <= 128, "MMA N for M=128");
  static_assert(NSUB == 1 || NSUB == 2, "sub-tiles");
  static_assert(TMEM_USED <= 512, "TMEM");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  // Item i = NSUB * slab + sub-tile. Every consumer of item i's "done"
  // barrier waits on it before item i + RD can be committed. The activation
  // producer recycles an x slot XS items later (RD >= XS keeps the loads of
  // item i + RD behind its wait on item i). The expansion waits for the items
  // of slab j - AB before filling slab j's A buffer (RD >= AB * NSUB puts
  // item i + RD in that slab or a later one; with two expansion groups the
  // items a group waits on have one parity, and so do the items of one
  // "done" barrier, RD being even). The promotion warps of
  // sub-tile t release a partial after waiting on its item; partials are used
  // in item order across both issuers, so item k waits for the promotion of
  // item k - PB, and with PB = 3 and two issuers each issuer waits on the
  // other sub-tile's promotions: item i + RD needs the A buffer of slab
  // (i + RD) / NSUB, whose expansion waited for both items of an earlier
  // slab, one of which waited for the promotion of an item of sub-tile t at
  // or after i (checked for RD = 8, PB = 3, NSUB <= 2).
  static_assert(RD >= XS && RD >= AB * NSUB && RD - PB >= NSUB - 1, "done ring depth");
  // Two issuers own alternate items (item i: issuer i % 2). The x slot of
  // item i last held item i - XS; the issuer of item i has already waited
  // on the promotion of item i - 5 (at its previous item), so item i - XS
  // has been issued and its load waited on whenever XS is even (same
  // issuer) or odd and at least 5 (the other issuer, which issues in order).
  static_assert(XS % 2 == 0 || XS >= 5, "x ring depth with two issuers");
  static_assert(AB % 2 == 0 && RD % 2 == 0, "rings shared by alternating issuers");
  static_assert(NEXP == 1 || QS % NEXP == 0, "q ring shared by alternating expansion groups");
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

__device__ __forceinline__ uint32_t ring_parity(int item, int depth) {
  return static_cast<uint32_t>((item / depth) & 1);
}

// The slabs one CTA runs, as a run of segments (tile, [kb0, kb1)). Tiles
// [0, dp_tiles) run whole, round robin (CTA c takes c, c + G, ...; G =
// gridDim.x); the U = (tiles - dp_tiles) x KB slabs of the other tiles, in
// tile-major order, run stream-K: CTA c takes the contiguous range
// [c U / G, (c + 1) U / G), so every CTA gets the same share within one slab.
// A stream-K tile may be split across consecutive CTAs; only a CTA's first
// and last stream-K segments can be partial. dp_tiles = 0 is pure stream-K,
// dp_tiles = tiles pure round robin.
// (Slab counts fit in 32 bits: the host checks tiles x KB.)
struct Schedule {
  int u, end, first;
  int tile, KB, dp_tiles;
  __device__ Schedule(int kb_per_tile, int tiles, int dp)
      : tile(static_cast<int>(blockIdx.x)), KB(kb_per_tile), dp_tiles(dp) {
    const int64_t U = static_cast<int64_t>(tiles - dp) * kb_per_tile;
    first = u = static_cast<int>(U * blockIdx.x / gridDim.x);
    end = static_cast<int>(U * (blockIdx.x + 1) / gridDim.x);
  }
  __device__ int slabs() const {
    const int dp = tile < dp_tiles ? ((dp_tiles - 1 - tile) / static_cast<int>(gridDim.x) + 1) * KB : 0;
    return dp + (end - first);
  }
  __device__ bool next(int& t, int& kb0, int& kb1) {
    if (tile < dp_tiles) {
      t = tile;
      kb0 = 0;
      kb1 = KB;
      tile += static_cast<int>(gridDim.x);
      return true;
    }
    if (u >= end) return false;
    const int lt = u / KB;
    t = dp_tiles + lt;
    kb0 = u - lt * KB;
    kb1 = min(KB, kb0 + (end - u));
    u += kb1 - kb0;
    return true;
  }
};

// ------------------------------------------------------------------ expansion
// One warpgroup expands the slabs j = eg, eg + NEXP, ... of its CTA: thread r
// (TMEM lane r) turns weight row r's 128 codes into 64 bf16x2 words and
// stores them with tcgen05.st into A buffer j % AB.
template <class C, int NSUB>
__device__ __forceinline__ void expand_slabs(int eg, int total_slabs, const uint8_t* sQ,
                                             uint32_t tmem, uint64_t* qfull, uint64_t* qempty,
                                             uint64_t* afull, uint64_t* done, unsigned* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int r = quad * 32 + lane;  // weight row within the tile == TMEM lane
  const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  for (int j = eg; j < total_slabs; j += C::NEXP) {
    const int qs = j % C::QS;
    if (!mbar_wait_warp(&qfull[qs], ring_parity(j, C::QS), err, kErrWaitExpand)) break;
    // Row r of the 128-byte-swizzled slab: 16-byte chunk c sits at chunk
    // position c ^ (r & 7).
    const uint8_t* qrow = sQ + qs * C::Q_BYTES + r * 128;
    uint4 c[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      c[u] = *reinterpret_cast<const uint4*>(qrow + ((u ^ (r & 7)) << 4));
    uint32_t o[32];
#pragma unroll
    for (int u = 0; u < 4; ++u) expand16(c[u], o + 8 * u);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      c[u] = *reinterpret_cast<const uint4*>(qrow + (((4 + u) ^ (r & 7)) << 4));
    // A buffer j % AB was last read by the items of slab j - AB.
    bool free_a = true;
    if (j >= C::AB) {
#pragma unroll
      for (int t = 0; t < NSUB; ++t) {
        const int ia = NSUB * (j - C::AB) + t;
        free_a = free_a && mbar_wait_warp(&done[ia % C::RD], ring_parity(ia, C::RD), err, kErrWaitExpand);
      }
    }
    if (!free_a) break;
    tc_fence_after_sync();
    const uint32_t ta = t_lane + static_cast<uint32_t>(C::TMEM_A + (j % C::AB) * 64);
    tmem_st32x32(ta, o);
    tmem_st_wait();  // the source registers are refilled below
#pragma unroll
    for (int u = 0; u < 4; ++u) expand16(c[u], o + 8 * u);
    // The codes have been consumed (shared-memory loads complete): the
    // slab's q slot may be refilled.
    __syncwarp();
    if (lane == 0) mbar_arrive(&qempty[qs]);
    tmem_st32x32(ta + 32u, o);
    tmem_st_wait();
    tc_fence_before_sync();
    __syncwarp();
    if (lane == 0) mbar_arrive(&afull[j % C::AB]);
  }
}

// Tile t -> (token tile, weight tile): in raster groups of gm token tiles
// (GROUPED), else token tile t % mtiles of weight tile t / mtiles (one group;
// the cheaper form keeps the epilogue within its registers).
template <bool GROUPED>
__device__ __forceinline__ void tile_of(int t, int mtiles, int ntiles_total, int gm, int& mt,
                                        int& nt) {
  if constexpr (GROUPED) {
    tile_coords(t, mtiles, ntiles_total / mtiles, gm, mt, nt);
  } else {
    nt = t / mtiles;
    mt = t % mtiles;
  }
}

template <int BT, int NSUB, bool GROUPED>
__global__ void __launch_bounds__(512, 1)
    w8a16_gemm_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_x,
                      const float* __restrict__ sw, __nv_bfloat16* __restrict__ y, int64_t ldy,
                      int M, int N, int KB, int mtiles, int ntiles_total, int gm, int dp_tiles,
                      int early_weights, float* __restrict__ part, unsigned* __restrict__ err) {
  using C = W8A16Cfg<BT, NSUB>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sQ = smem;                       // QS x Q_BYTES
  uint8_t* sX = smem + C::QS * C::Q_BYTES;  // XS x X_BYTES
  uint8_t* sOut = sX + C::XS * C::X_BYTES;  // 4 NSUB x OUT_BYTES output transposition
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::SMEM_TILES);
  uint64_t* qfull = bars;              // codes landed          (1 arrival + tx)
  uint64_t* qempty = qfull + C::QS;    // codes read            (4 expansion warps)
  uint64_t* xfull = qempty + C::QS;    // x sub-tile landed     (1 arrival + tx)
  uint64_t* afull = xfull + C::XS;     // A buffer written      (4 expansion warps)
  uint64_t* done = afull + C::AB;      // item's MMAs complete  (1 commit)
  uint64_t* pempty = done + C::RD;     // partial consumed      (4 or 8 epilogue warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pempty + C::PB * 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_slabs = Schedule(KB, ntiles_total, dp_tiles).slabs();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::QS; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 4);
    }
    for (int s = 0; s < C::XS; ++s) mbar_init(&xfull[s], 1);
    for (int b = 0; b < C::AB; ++b) mbar_init(&afull[b], 4);
    for (int b = 0; b < C::RD; ++b) mbar_init(&done[b], 1);
    // One barrier per (partial slot, issuer). NSUB == 2: all eight epilogue
    // warps promote every item.
    for (int b = 0; b < C::PB * 2; ++b) mbar_init(&pempty[b], NSUB == 2 ? 8 : 4);
    mbar_init_fence();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  // The kernel after this one in the stream (the stream-K fix-up, or the
  // next linear) may be scheduled now: whatever it reads of this kernel's
  // output it reads after griddepcontrol.wait. This kernel in turn reads the
  // activations, and writes y and the workspace, only after its own wait for
  // the kernel before it; the weights too, unless the caller has promised
  // that the kernel before does not write them (early_weights).
  pdl_launch_dependents();

  // Each warpgroup sets its register budget at the top of its role:
  // 128 x (64 + 72 + 184 + 184) = 64512 of the 65536 the block holds.
  const int wg = warp >> 2;
  if (wg == 0) {
    setmaxnreg_dec<64>();
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------ weight-code producer
      tma_prefetch_map(&tm_q);
      if (!early_weights) pdl_wait();
      int j = 0;  // slab counter (across tiles)
      bool ok = true;
      Schedule sc(KB, ntiles_total, dp_tiles);
      int tile, kb0, kb1;
      while (ok && sc.next(tile, kb0, kb1)) {
        int mt, nt;
        tile_of<GROUPED>(tile, mtiles, ntiles_total, gm, mt, nt);
        const int n0 = nt * 128;
        for (int kb = kb0; kb < kb1; ++kb, ++j) {
          const int qs = j % C::QS;
          if (!mbar_wait_sleepy(&qempty[qs], ring_parity(j, C::QS) ^ 1u, err, kErrWaitLoad)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&qfull[qs], C::Q_BYTES);
          tma_load_2d(sQ + qs * C::Q_BYTES, &tm_q, &qfull[qs], kb * 128, n0);
        }
      }
      // Drain: every load issued has landed before the CTA may exit.
      for (int s = 0; s < C::QS && s < j; ++s)
        mbar_wait(&qfull[s], last_parity((j - s + C::QS - 1) / C::QS), err, kErrWaitLoad);
    } else if (warp == 1 && lane == 0) {
      // ------------------------------------------------- activation producer
      tma_prefetch_map(&tm_x);
      pdl_wait();
      int i = 0;  // item counter (across tiles)
      bool ok = true;
      Schedule sc(KB, ntiles_total, dp_tiles);
      int tile, kb0, kb1;
      while (ok && sc.next(tile, kb0, kb1)) {
        int mt, nt;
        tile_of<GROUPED>(tile, mtiles, ntiles_total, gm, mt, nt);
        const int m0 = mt * (BT * NSUB);
        for (int kb = kb0; kb < kb1 && ok; ++kb) {
          for (int t = 0; t < NSUB; ++t, ++i) {
            const int xs = i % C::XS;
            if (i >= C::XS) {  // the item that last used this slot has finished
              const int io = i - C::XS;
              if (!mbar_wait_sleepy(&done[io % C::RD], ring_parity(io, C::RD), err, kErrWaitLoad)) {
                ok = false;
                break;
              }
            }
            uint8_t* xsm = sX + xs * C::X_BYTES;
            mbar_arrive_expect_tx(&xfull[xs], C::X_BYTES);
            tma_load_2d(xsm, &tm_x, &xfull[xs], kb * 128, m0 + t * BT);
            tma_load_2d(xsm + C::X_ATOM, &tm_x, &xfull[xs], kb * 128 + 64, m0 + t * BT);
          }
        }
      }
      for (int s = 0; s < C::XS && s < i; ++s)
        mbar_wait(&xfull[s], last_parity((i - s + C::XS - 1) / C::XS), err, kErrWaitLoad);
    } else if (warp >= 2 && warp < 4 && lane == 0) {
      // ------------------------------------------------------- MMA issuers
      // Issuer u runs the items i with i % 2 == u: sub-tile u of every slab
      // (NSUB == 2), or every other slab (NSUB == 1). One issuer's waits and
      // commits hide behind the other's MMAs. Descriptors are formed once;
      // stepping through shared memory adds (bytes >> 4) to their
      // start-address field.
      const int u = warp - 2;
      const uint64_t xdesc0 = sw128_kmajor_desc(smem_addr(sX));
      int last = -1;
      for (int j = NSUB == 1 ? u : 0; j < total_slabs; j += NSUB == 1 ? 2 : 1) {
        const int i = NSUB == 1 ? j : 2 * j + u;
        if (!mbar_wait(&afull[j % C::AB], ring_parity(j, C::AB), err, kErrWaitMma)) break;
        if (!mbar_wait(&xfull[i % C::XS], ring_parity(i, C::XS), err, kErrWaitMma)) break;
        // Partial slot i % PB last held item k = i - PB, whose promotion
        // arrives on that slot's barrier for k's issuer. Each issuer meets
        // every phase of the barriers it waits on, in order (a parity wait
        // cannot tell a phase from the one two before or after).
        if (i >= C::PB) {
          const int k = i - C::PB;
          if (!mbar_wait(&pempty[(k % C::PB) * 2 + (k & 1)], ring_parity(k, C::PB * 2), err,
                         kErrWaitMma))
            break;
        }
        tc_fence_after_sync();
        const uint32_t a = tmem + static_cast<uint32_t>(C::TMEM_A + (j % C::AB) * 64);
        const uint64_t xd = xdesc0 + static_cast<uint64_t>(((i % C::XS) * C::X_BYTES) >> 4);
        const uint32_t d = tmem + static_cast<uint32_t>(C::TMEM_P + (i % C::PB) * BT);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_f16_ts(d, a + 8u * k,
                     xd + static_cast<uint64_t>(((k >> 2) * C::X_ATOM + (k & 3) * 32) >> 4),
                     C::IDESC, k > 0 ? 1u : 0u);
        tc_commit(&done[i % C::RD]);
        last = i;
      }
      // Drain: this issuer's MMAs have completed before TMEM is released.
      if (last >= 0) mbar_wait(&done[last % C::RD], ring_parity(last, C::RD), err, kErrWaitMma);
    }
  } else if (wg == 1) {
    setmaxnreg_dec<72>();
    expand_slabs<C, NSUB>(0, total_slabs, sQ, tmem, qfull, qempty, afull, done, err);
  } else {
    setmaxnreg_inc<184>();
    if constexpr (NSUB == 2) {
      // ------------------------------------ promotion/epilogue (two sub-tiles)
      pdl_wait();  // y may still be read by the kernel before
      // All eight warps promote every item: warp 8 + 4h + q owns TMEM lane
      // quadrant q and token columns [64h, 64h + 64) of each item's partial,
      // so a partial is read by eight warps at once (two 32-column loads
      // each) and its slot is released sooner.
      const int ew = warp - 8, quad = warp & 3, h = ew >> 2;
      const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16) + C::TMEM_P +
                              static_cast<uint32_t>(64 * h);
      uint8_t* stg = sOut + ew * C::OUT_BYTES;
      const int rr = lane >> 1, hh = lane & 1;  // row and half this lane stores
      int j = 0;
      bool ok = true;
      bool first_sk = true;  // the next stream-K segment is this CTA's first
      Schedule sc(KB, ntiles_total, dp_tiles);
      int tile, kb0, kb1;
      while (ok && sc.next(tile, kb0, kb1)) {
        int mt, nt;
        tile_of<GROUPED>(tile, mtiles, ntiles_total, gm, mt, nt);
        const int m0 = mt * (BT * NSUB), n0 = nt * 128;
        const float* sw_row = sw + static_cast<int64_t>(n0 >> 7) * KB;
        uint64_t acc[64];  // acc[32t + p]: tokens 128t + 64h + 2p and 2p + 1
#pragma unroll
        for (int e = 0; e < 64; ++e) acc[e] = 0ull;
        float s_next = __ldg(sw_row + kb0);
        for (int kb = kb0; kb < kb1 && ok; ++kb, ++j) {
          const float s = s_next;
          if (kb + 1 < kb1) s_next = __ldg(sw_row + kb + 1);
          const uint64_t s2 = pack_f32x2(s, s);
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int i = 2 * j + t;
            if (!mbar_wait_warp(&done[i % C::RD], ring_parity(i, C::RD), err, kErrWaitEpilogue)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t tp = t_lane + static_cast<uint32_t>((i % C::PB) * BT);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              uint32_t p[32];
              tmem_ld32x32(tp + 32u * c, p);
#pragma unroll
              for (int e = 0; e < 16; ++e)
                ffma2(acc[32 * t + 16 * c + e], pack_u32x2(p[2 * e], p[2 * e + 1]), s2);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&pempty[(i % C::PB) * 2 + t]);
          }
        }
        if (!ok) break;
        const int slot = first_sk ? 0 : 1;
        if (tile >= dp_tiles) first_sk = false;
        if (kb0 != 0 || kb1 != KB) {
          // Part of a stream-K tile: the FP32 partial goes to slot (CTA,
          // first or last stream-K segment) of the workspace, [256 tokens]
          // [128 weight rows] with the weight row fastest;
          // w8a16_streamk_fixup adds the slots.
          float* dst = part + (static_cast<int64_t>(blockIdx.x) * 2 + slot) * (BT * NSUB * 128) +
                       quad * 32 + lane;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) {
              float lo, hi;
              asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[32 * t + pp]));
              const int mloc = 128 * t + 64 * h + 2 * pp;
              dst[mloc * 128] = lo;
              dst[(mloc + 1) * 128] = hi;
            }
          }
          continue;
        }
        // Output: sixteen tokens at a time through shared memory as rows of
        // 32 BF16 (this warp's columns of y), then 32-byte stores per lane.
        const int nw = n0 + quad * 32;  // first column of this warp
#pragma unroll
        for (int t = 0; t < 2; ++t) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t b2 = cvt_bf16x2_pair(acc[32 * t + 8 * g + e]);
              *reinterpret_cast<uint16_t*>(stg + (2 * e) * 64 + lane * 2) = static_cast<uint16_t>(b2 & 0xFFFFu);
              *reinterpret_cast<uint16_t*>(stg + (2 * e + 1) * 64 + lane * 2) = static_cast<uint16_t>(b2 >> 16);
            }
            __syncwarp();
            const uint8_t* src = stg + rr * 64 + hh * 32;
            const int m = m0 + 128 * t + 64 * h + 16 * g + rr, c0 = nw + 16 * hh;
            if (m < M && c0 < N) {
              uint16_t* dst = reinterpret_cast<uint16_t*>(y) + static_cast<int64_t>(m) * ldy + c0;
              if (c0 + 16 <= N) {
                reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<const uint4*>(src)[0];
                reinterpret_cast<uint4*>(dst)[1] = reinterpret_cast<const uint4*>(src)[1];
              } else {
                for (int c = 0; c < N - c0; ++c) dst[c] = reinterpret_cast<const uint16_t*>(src)[c];
              }
            }
            __syncwarp();  // the next group overwrites the buffer
          }
        }
      }
    } else if (((warp - 8) >> 2) < NSUB) {
      // ------------------------------------------------ promotion/epilogue
      pdl_wait();  // y and the workspace may still be in use by the kernel before
      const int t = (warp - 8) >> 2;  // token sub-tile
      const int quad = warp & 3;
      const uint32_t t_lane = tmem + (static_cast<uint32_t>(quad * 32) << 16) + C::TMEM_P;
      int j = 0;
      bool ok = true;
      Schedule sc(KB, ntiles_total, dp_tiles);
      int tile, kb0, kb1;
      bool first_segment = true;
      while (ok && sc.next(tile, kb0, kb1)) {
        int tm, tn;
        tile_of<GROUPED>(tile, mtiles, ntiles_total, gm, tm, tn);
        const int m0 = tm * (BT * NSUB), n0 = tn * 128;
        const float* sw_row = sw + static_cast<int64_t>(n0 >> 7) * KB;
        uint64_t acc[BT / 2];
#pragma unroll
        for (int e = 0; e < BT / 2; ++e) acc[e] = 0ull;
        float s_next = __ldg(sw_row + kb0);
        for (int kb = kb0; kb < kb1; ++kb, ++j) {
          const float s = s_next;
          if (kb + 1 < kb1) s_next = __ldg(sw_row + kb + 1);
          const int i = j * NSUB + t;
          if (!mbar_wait_warp(&done[i % C::RD], ring_parity(i, C::RD), err, kErrWaitEpilogue)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint64_t s2 = pack_f32x2(s, s);
          const uint32_t tp = t_lane + static_cast<uint32_t>((i % C::PB) * BT);
          if constexpr (BT == 16) {
            uint32_t p[16];
            tmem_ld32x16(tp, p);
#pragma unroll
            for (int e = 0; e < 8; ++e) ffma2(acc[e], pack_u32x2(p[2 * e], p[2 * e + 1]), s2);
          } else {
#pragma unroll
            for (int h = 0; h < BT / 32; ++h) {
              uint32_t p[32];
              tmem_ld32x32(tp + 32u * h, p);
#pragma unroll
              for (int e = 0; e < 16; ++e)
                ffma2(acc[16 * h + e], pack_u32x2(p[2 * e], p[2 * e + 1]), s2);
            }
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pempty[(i % C::PB) * 2 + (i & 1)]);
        }
        if (!ok) break;
        const bool whole = kb0 == 0 && kb1 == KB;
        const int slot = first_segment ? 0 : 1;
        first_segment = false;
        if (!whole) {
          // Part of a tile split across CTAs (stream-K): the FP32 partial goes
          // to slot (CTA, first or last segment) of the workspace, [BT][128]
          // with the weight row fastest; w8a16_streamk_fixup adds the slots.
          float* dst = part + (static_cast<int64_t>(blockIdx.x) * 2 + slot) * (BT * 128) + quad * 32 + lane;
#pragma unroll
          for (int e = 0; e < BT / 2; ++e) {
            float lo, hi;
            asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc[e]));
            dst[(2 * e) * 128] = lo;
            dst[(2 * e + 1) * 128] = hi;
          }
          continue;
        }
        // Output: the warp holds y[mt .. mt + BT)[n0 + 32q .. + 32) with one
        // weight row (column of y) per lane. Sixteen tokens at a time go
        // through shared memory as rows of 32 BF16, so that each lane then
        // stores 16 contiguous values (32 bytes) of one row of y.
        const int mt = m0 + t * BT;
        const int nw = n0 + quad * 32;  // first column of this warp
        uint8_t* stg = sOut + (warp - 8) * C::OUT_BYTES;
        const int rr = lane >> 1, hh = lane & 1;  // row and half this lane stores
#pragma unroll
        for (int g = 0; g < BT / 16; ++g) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t b2 = cvt_bf16x2_pair(acc[8 * g + e]);
            *reinterpret_cast<uint16_t*>(stg + (2 * e) * 64 + lane * 2) = static_cast<uint16_t>(b2 & 0xFFFFu);
            *reinterpret_cast<uint16_t*>(stg + (2 * e + 1) * 64 + lane * 2) = static_cast<uint16_t>(b2 >> 16);
          }
          __syncwarp();
          const uint8_t* src = stg + rr * 64 + hh * 32;
          const int m = mt + 16 * g + rr, c0 = nw + 16 * hh;
          if (m < M && c0 < N) {
            uint16_t* dst = reinterpret_cast<uint16_t*>(y) + static_cast<int64_t>(m) * ldy + c0;
            if (c0 + 16 <= N) {
              reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<const uint4*>(src)[0];
              reinterpret_cast<uint4*>(dst)[1] = reinterpret_cast<const uint4*>(src)[1];
            } else {
              for (int c = 0; c < N - c0; ++c) dst[c] = reinterpret_cast<const uint16_t*>(src)[c];
            }
          }
          __syncwarp();  // the next group overwrites the buffer
        }
      }
    } else {
      // One sub-tile: warps 12-15 are the second expansion group (odd slabs).
      expand_slabs<C, NSUB>(1, total_slabs, sQ, tmem, qfull, qempty, afull, done, err);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 2) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// CTAs a stream-K launch may use (the workspace is sized for this many).
constexpr int kStreamKMaxCtas = 160;

// The tiles a stream-K launch splits across CTAs, worked out on the host:
// CTA c holds slabs [c U / G, (c + 1) U / G) of the U = tiles x KB slabs, so
// a tile is split when a range boundary falls inside it. Each split tile
// lists its first contributor c0 (whose last segment it is), the number of
// contributors, and the workspace slot c0 wrote (0 if the tile was also
// c0's first segment, else 1); later contributors wrote slot 0.
struct SplitTiles {
  int count;
  int tile[kStreamKMaxCtas];
  short c0[kStreamKMaxCtas];
  unsigned char ncontrib[kStreamKMaxCtas];
  unsigned char slot0[kStreamKMaxCtas];
};

SplitTiles split_tiles(int64_t ntiles, int64_t KB, int64_t G) {
  SplitTiles st{};
  const int64_t U = ntiles * KB;
  for (int64_t c0 = 0; c0 + 1 < G; ++c0) {
    const int64_t x = U * (c0 + 1) / G;  // first slab of CTA c0 + 1
    const int64_t t = x / KB, s0 = t * KB;
    const int64_t c0_start = U * c0 / G;
    if (x == s0 || c0_start > s0) continue;  // no split here, or not the tile's first boundary
    const int64_t c1 = ((s0 + KB) * G - 1) / U;  // holds the tile's last slab
    st.tile[st.count] = static_cast<int>(t);
    st.c0[st.count] = static_cast<short>(c0);
    st.ncontrib[st.count] = static_cast<unsigned char>(c1 - c0 + 1);
    st.slot0[st.count] = static_cast<unsigned char>(c0_start == s0 ? 0 : 1);
    ++st.count;
  }
  return st;
}

// Stream-K fix-up: y of every split tile, the sum of its contributors' FP32
// partials in slab order, rounded once to BF16. Block (i, g) handles split
// tile i for tokens [8 g, 8 g + 8) of its TOK with one thread per weight row
// and token parity, every partial load issued before the sums. Tiles run by
// a single CTA were written directly. Launched as a programmatic dependent
// of the GEMM: it waits for the GEMM grid to complete before it reads a
// partial.
template <int TOK>
__global__ void __launch_bounds__(256) w8a16_streamk_fixup(const __grid_constant__ SplitTiles st,
                                                           const float* __restrict__ part,
                                                           uint16_t* __restrict__ y, int64_t ldy,
                                                           int M, int N, int mtiles, int gm) {
  pdl_launch_dependents();  // the next linear may be scheduled; it waits for this grid
  pdl_wait();
  const int i = static_cast<int>(blockIdx.x);
  const int r = threadIdx.x & 127;
  int mt, nt;
  tile_coords(st.tile[i], mtiles, (N + 127) / 128, gm, mt, nt);
  const int n = nt * 128 + r;
  if (n >= N) return;
  const int m0 = mt * TOK;
  const int c0 = st.c0[i], nc = st.ncontrib[i], slot0 = st.slot0[i];
  const int mbase = static_cast<int>(blockIdx.y) * 8 + (threadIdx.x >> 7);
  float acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = 0.0f;
  for (int c = 0; c < nc; ++c) {
    const float* p = part + (static_cast<int64_t>(c0 + c) * 2 + (c == 0 ? slot0 : 0)) * (TOK * 128) + r;
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int m = mbase + 2 * u;
      v[u] = m < TOK && m0 + m < M ? p[m * 128] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] += v[u];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int m = mbase + 2 * u;
    if (m < TOK && m0 + m < M)
      y[static_cast<int64_t>(m0 + m) * ldy + n] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[u]));
  }
}

// Workspace bytes of a stream-K launch with grid CTAs and TOK-token tiles:
// two FP32 partial slots of [TOK][128] per CTA.
size_t streamk_bytes(int64_t grid, int tok) {
  return static_cast<size_t>(grid) * 2 * tok * 128 * sizeof(float);
}

template <int BT, int NSUB, bool GROUPED>
cudaError_t launch_bt(const Launch& L, const uint16_t* x, int64_t ldx, const uint8_t* q,
                      int64_t ldq, const float* sw, uint16_t* y, int64_t ldy, int64_t M,
                      int64_t N, int64_t K, void* ws, size_t ws_bytes, bool early_weights) {
  using C = W8A16Cfg<BT, NSUB>;
  constexpr int TOK = BT * NSUB;
  CUtensorMap tq, tx;
  if (!make_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, K, N, ldq, 128, 128))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, ldx * 2, 64, BT))
    return cudaErrorInvalidValue;
  auto kern = w8a16_gemm_kernel<BT, NSUB, GROUPED>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  {
    // The setmaxnreg split (64512 registers) needs 128 per thread at launch
    // (checked once per kernel).
    static const cudaError_t regs = [&] {
      cudaFuncAttributes fa;
      cudaError_t r = cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kern));
      if (r != cudaSuccess) return r;
      return fa.numRegs * C::THREADS < 128 * (64 + 72 + 184 + 184) ? cudaErrorInvalidConfiguration
                                                                   : cudaSuccess;
    }();
    if (regs != cudaSuccess) return regs;
  }
  const int64_t mtiles = cdiv(M, TOK), tiles = mtiles * cdiv(N, 128);
  const int gm = GROUPED ? raster_group(mtiles, TOK * K * 2, kRasterBytesW8A16) : static_cast<int>(mtiles);
  // Slab and item counters are 32-bit per CTA.
  if (tiles * cdiv(K, 128) * NSUB > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int64_t KB = cdiv(K, 128);
  const int64_t G = L.num_sms < kStreamKMaxCtas ? L.num_sms : kStreamKMaxCtas;
  int64_t dp_tiles, grid;
  if (NSUB == 1) {
    // One token tile (M <= 128): stream-K over all the slabs, so every SM
    // streams the same share of the weights however few tiles there are.
    dp_tiles = 0;
    grid = tiles * KB < G ? tiles * KB : G;
    if (!ws || ws_bytes < streamk_bytes(grid, TOK)) return cudaErrorInvalidValue;
  } else {
    // Whole tiles round robin. When the last wave of tiles would leave at
    // least 15% of the SM time idle, and the workspace allows, the tiles of
    // that wave run stream-K over all CTAs instead. (Below that the partial
    // round trip and the fix-up cost what the even split saves: at 10% idle
    // -- 400 tiles on 148 SMs -- both ran in the same time.)
    const int64_t waves = tiles / G, rem = tiles - waves * G;
    const int64_t tail_grid = waves > 0 ? G : (rem * KB < G ? rem * KB : G);
    const bool tail_sk = rem > 0 && (G - rem) * 100 >= 15 * (waves + 1) * G && tail_grid >= 2 && ws &&
                         reinterpret_cast<uintptr_t>(ws) % 256 == 0 &&
                         ws_bytes >= streamk_bytes(tail_grid, TOK);
    if (tail_sk) {
      dp_tiles = waves * G;
      grid = tail_grid;
    } else {
      dp_tiles = tiles;
      grid = tiles < L.num_sms ? tiles : L.num_sms;
    }
  }
  // A programmatic dependent of the kernel before it in the stream (its set-up
  // overlaps that kernel's tail; see the kernel for what waits).
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = L.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tq, tx, sw, reinterpret_cast<__nv_bfloat16*>(y), ldy,
                           static_cast<int>(M), static_cast<int>(N), static_cast<int>(KB),
                           static_cast<int>(mtiles), static_cast<int>(tiles), gm,
                           static_cast<int>(dp_tiles), early_weights ? 1 : 0,
                           static_cast<float*>(ws), L.err);
    if (e != cudaSuccess) return e;
  }
  if (dp_tiles == tiles || grid < 2) return cudaSuccess;
  SplitTiles st = split_tiles(tiles - dp_tiles, KB, grid);
  if (st.count == 0) return cudaSuccess;
  for (int i = 0; i < st.count; ++i) st.tile[i] += static_cast<int>(dp_tiles);
  const int mt = static_cast<int>(M < TOK ? M : TOK);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(st.count), static_cast<unsigned>((mt + 7) / 8));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = L.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, w8a16_streamk_fixup<TOK>, st, static_cast<const float*>(ws), y,
                            ldy, static_cast<int>(M), static_cast<int>(N), static_cast<int>(mtiles),
                            gm);
}

}  // namespace

namespace {
int token_tile(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128)); }
}  // namespace

// M <= 128 runs stream-K: FP32 partials of split tiles, two slots per CTA
// (required). M > 128 runs whole 256-token tiles and may run its last wave
// stream-K: the same slots of [256][128] for up to 160 CTAs (optional).
size_t w8a16_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 128) return streamk_bytes(kStreamKMaxCtas, token_tile(M));
  const int64_t units = cdiv(M, 256) * cdiv(N, 128) * cdiv(K, 128);
  return streamk_bytes(units < kStreamKMaxCtas ? units : kStreamKMaxCtas, 256);
}

size_t w8a16_workspace_required(int64_t M, int64_t N, int64_t K) {
  return M <= 128 ? w8a16_workspace_bytes(M, N, K) : 0;
}

cudaError_t launch_w8a16_gemm(const Launch& L, const uint16_t* x, int64_t ldx, const uint8_t* q,
                              int64_t ldq, const float* sw, uint16_t* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, void* ws, size_t ws_bytes, bool early_weights) {
  if (M <= 16) return launch_bt<16, 1, false>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K, ws, ws_bytes, early_weights);
  if (M <= 32) return launch_bt<32, 1, false>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K, ws, ws_bytes, early_weights);
  if (M <= 64) return launch_bt<64, 1, false>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K, ws, ws_bytes, early_weights);
  if (M <= 128) return launch_bt<128, 1, false>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K, ws, ws_bytes, early_weights);
  // Activations larger than the raster budget run in raster groups.
  if (raster_group(cdiv(M, 256), 256 * K * 2, kRasterBytesW8A16) < cdiv(M, 256))
    return launch_bt<128, 2, true>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K, ws, ws_bytes, early_weights);
  return launch_bt<128, 2, false>(L, x, ldx, q, ldq, sw, y, ldy, M, N, K, ws, ws_bytes, early_weights);
}

}  // namespace fp8blk
