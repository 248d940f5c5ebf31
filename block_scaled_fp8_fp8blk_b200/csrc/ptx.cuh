// Hand-written PTX for sm_100a: mbarriers, TMA tile loads, tcgen05 (TMEM
// allocation, MMA, commit, TMEM loads/stores) and the FP8 conversions.
// Written from the PTX ISA's descriptions of these instructions.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fp8blk {

// Bounded waits give up after this many SM cycles (about 2 s at 1.9 GHz),
// set a flag in the device error word and let the kernel wind down.
constexpr long long kWaitLimitCycles = 4000000000LL;

enum DeviceErrorBits : unsigned {
  kErrWaitLoad = 1u,
  kErrWaitMma = 2u,
  kErrWaitEpilogue = 4u,
  kErrWaitExpand = 8u,
  kErrWaitSelfTest = 16u,
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes the initialized barriers visible to the async proxy (TMA, tcgen05).
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase with the given parity to complete, at most
// limit_cycles; on time-out OR `flag` into *err and return false.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, unsigned* err,
                                              unsigned flag, long long limit_cycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      if (mbar_try_wait(bar, parity)) return true;
#ifdef FP8BLK_WAIT_BACKOFF_NS
      __nanosleep(FP8BLK_WAIT_BACKOFF_NS);
#endif
    }
    if (clock64() - t0 > limit_cycles) {
      atomicOr(err, flag);
      return false;
    }
  }
}

// The kernels' wait: at most kWaitLimitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* err,
                                          unsigned flag) {
  return mbar_wait_for(bar, parity, err, flag, kWaitLimitCycles);
}

// Bounded wait for a thread that is normally far ahead of the barrier it
// waits on (a TMA producer): it sleeps between polls instead of spinning,
// leaving issue slots to the other warps of its SM sub-partition.
__device__ __forceinline__ bool mbar_wait_sleepy(uint64_t* bar, uint32_t parity, unsigned* err,
                                                 unsigned flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
      __nanosleep(64);
      if (mbar_try_wait(bar, parity)) return true;
    }
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(err, flag);
      return false;
    }
  }
}

// Warp-uniform bounded wait: lane 0 polls, every lane gets the same answer
// and the warp is converged afterwards (needed before .sync.aligned ops).
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, unsigned* err,
                                               unsigned flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, err, flag) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// Programmatic dependent launch (sm_90 and later): let the kernel launched
// after this one in the stream be scheduled now, and, in that kernel, wait
// until the kernel before it has completed with its memory visible.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Position in a ring of mbarrier-guarded slots: slot index and the parity of
// the phase that slot is on.
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int depth) {
    if (++slot == depth) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// Parity of the most recent phase of a ring slot that was used `uses` times.
__device__ __forceinline__ uint32_t last_parity(int uses) { return static_cast<uint32_t>((uses - 1) & 1); }

// ----------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tile load global -> shared, completion counted on `bar` in bytes.
// c0 is the innermost coordinate (elements); c0 * element size must be a
// multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Same, with an L2 eviction-priority hint (a createpolicy result).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map,
                                                 uint64_t* bar, int32_t c0, int32_t c1,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 2-D tile store shared -> global (out-of-bounds parts of the box are not
// written); completion tracked with bulk async-groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t c0,
                                             int32_t c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_addr(src)), "r"(c0), "r"(c1)
               : "memory");
}
__device__ __forceinline__ void tma_store_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed store groups still read their shared source.
template <int N>
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until all committed store groups have completed.
__device__ __forceinline__ void tma_store_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (tcgen05.mma / TMA) reads of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------- tcgen05
// TMEM allocation is done by one whole warp; the base address is written to
// shared memory. ncols is a power of two >= 32.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The barrier gets one arrival when all tcgen05.mma issued so far by this
// thread have completed (their smem reads and TMEM writes are done).
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, E4M3 x E4M3 -> FP32 (K = 32 per instruction).
__device__ __forceinline__ void mma_f8f6f4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, BF16 x BF16 -> FP32 (K = 16 per instruction).
__device__ __forceinline__ void mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with 128-byte swizzling: rows of 128 bytes, 8-row (1024-byte) swizzle atoms
// stacked along M/N (stride byte offset 1024). The tile base must be
// 1024-byte aligned; stepping along K inside the 128-byte row adds bytes to
// the start address. Fields: start >> 4 [0,14), leading byte offset >> 4
// [16,30) (unused for swizzled K-major; 1), stride byte offset >> 4 [32,46),
// descriptor version 1 [46,48), base offset 0 [49,52), layout 2 = 128-byte
// swizzle [61,64).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor (kind::f16 / kind::f8f6f4, dense): D format [4,6)
// (1 = F32), A format [7,10), B format [10,13) (f8f6f4: 0 = E4M3; f16: 1 =
// BF16), A/B major [15], [16] (0 = K-major), N >> 3 [17,23), M >> 4 [24,29).
constexpr uint32_t make_idesc(uint32_t a_fmt, uint32_t b_fmt, int M, int N) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

#define FP8BLK_R8(p, i) \
  "=r"(p[i]), "=r"(p[i + 1]), "=r"(p[i + 2]), "=r"(p[i + 3]), "=r"(p[i + 4]), "=r"(p[i + 5]), \
      "=r"(p[i + 6]), "=r"(p[i + 7])
#define FP8BLK_W8(p, i) \
  "+r"(p[i]), "+r"(p[i + 1]), "+r"(p[i + 2]), "+r"(p[i + 3]), "+r"(p[i + 4]), "+r"(p[i + 5]), \
      "+r"(p[i + 6]), "+r"(p[i + 7])
#define FP8BLK_I8(p, i) \
  "r"(p[i]), "r"(p[i + 1]), "r"(p[i + 2]), "r"(p[i + 3]), "r"(p[i + 4]), "r"(p[i + 5]), \
      "r"(p[i + 6]), "r"(p[i + 7])

// 32 lanes x 32 consecutive 32-bit columns (one register per column per
// thread), then wait for the load. Thread t of the warp reads lane
// (lane base + t). The wait carries the registers as in/out operands so no
// use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld32x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FP8BLK_R8(r, 0), FP8BLK_R8(r, 8), FP8BLK_R8(r, 16), FP8BLK_R8(r, 24)
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : FP8BLK_W8(r, 0), FP8BLK_W8(r, 8), FP8BLK_W8(r, 16), FP8BLK_W8(r, 24)
               :
               : "memory");
}

__device__ __forceinline__ void tmem_ld32x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : FP8BLK_R8(r, 0), FP8BLK_R8(r, 8)
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" : FP8BLK_W8(r, 0), FP8BLK_W8(r, 8) : : "memory");
}

// Split form of the 32x32b.x32 load: issue, then wait carrying the
// destination registers as in/out operands (no use can move above the wait).
__device__ __forceinline__ void tmem_ld32x32_issue(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : FP8BLK_R8(r, 0), FP8BLK_R8(r, 8), FP8BLK_R8(r, 16), FP8BLK_R8(r, 24)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : FP8BLK_W8(r, 0), FP8BLK_W8(r, 8), FP8BLK_W8(r, 16), FP8BLK_W8(r, 24)
               :
               : "memory");
}

// Empty volatile statement that claims to rewrite r: code reading r cannot
// be scheduled above it (used to keep a load issued before the work that
// should overlap it).
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
  asm volatile("" : FP8BLK_W8(r, 0), FP8BLK_W8(r, 8), FP8BLK_W8(r, 16), FP8BLK_W8(r, 24));
}

// acc[j] += float(TMEM[lane, t + j]) * c for j < 32 * NCH: 32 columns per
// load, the next load in flight while the current chunk is consumed.
template <int NCH>
__device__ __forceinline__ void tmem_axpy(uint32_t t, float c, float* acc) {
  uint32_t pa[32], pb[32];
  tmem_ld32x32_issue(t, pa);
  tmem_ld_wait(pa);
#pragma unroll
  for (int j = 0; j < NCH; j += 2) {
    if (j + 1 < NCH) {
      tmem_ld32x32_issue(t + 32u * (j + 1), pb);
      reg_fence(pa);
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[32 * j + i] = fmaf(__uint_as_float(pa[i]), c, acc[32 * j + i]);
    if (j + 1 < NCH) {
      tmem_ld_wait(pb);
      if (j + 2 < NCH) {
        tmem_ld32x32_issue(t + 32u * (j + 2), pa);
        reg_fence(pb);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i)
        acc[32 * (j + 1) + i] = fmaf(__uint_as_float(pb[i]), c, acc[32 * (j + 1) + i]);
      if (j + 2 < NCH) tmem_ld_wait(pa);
    }
  }
}

// 32 lanes x 32 consecutive columns store (thread t writes lane base + t).
// Completion is awaited separately with tmem_st_wait().
__device__ __forceinline__ void tmem_st32x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      FP8BLK_I8(r, 0), FP8BLK_I8(r, 8), FP8BLK_I8(r, 16), FP8BLK_I8(r, 24)
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------- registers and FP32x2
// Warpgroup-wide register budget changes (all 128 threads of an aligned
// warpgroup execute the same one). The per-warpgroup budgets of a kernel
// must add up to no more than the registers it was launched with.
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ uint64_t pack_u32x2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
// acc = p * c + acc on two FP32 lanes at once (each lane one rounded FMA).
__device__ __forceinline__ void ffma2(uint64_t& acc, uint64_t p, uint64_t c) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(p), "l"(c));
}

// acc2[j] += (TMEM[lane, t + 2j], TMEM[lane, t + 2j + 1]) * (c, c) for
// j < 16 * NCH, with packed FP32x2 FMAs (acc2 holds column pairs).
template <int NCH>
__device__ __forceinline__ void tmem_axpy2(uint32_t t, float c, uint64_t* acc2) {
  const uint64_t c2 = pack_f32x2(c, c);
#pragma unroll
  for (int j = 0; j < NCH; ++j) {
    uint32_t p[32];
    tmem_ld32x32(t + 32u * j, p);
#pragma unroll
    for (int i = 0; i < 16; ++i) ffma2(acc2[16 * j + i], pack_u32x2(p[2 * i], p[2 * i + 1]), c2);
  }
}

// ------------------------------------------------------- FP8 conversions
// Two floats -> two E4M3 codes, round to nearest even, saturating to +-448
// (NaN -> 0x7F). `hi` lands in bits [8,16), `lo` in bits [0,8).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E4M3 codes (low byte -> low half) -> two exact halves (f16x2).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t codes16) {
  uint32_t r;
  uint16_t c = static_cast<uint16_t>(codes16);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(c));
  return r;
}

__device__ __forceinline__ float f16_lo_to_f32(uint32_t h2) {
  float f;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, lo;\n\t}"
      : "=f"(f)
      : "r"(h2));
  return f;
}

__device__ __forceinline__ float f16_hi_to_f32(uint32_t h2) {
  float f;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.f32.f16 %0, hi;\n\t}"
      : "=f"(f)
      : "r"(h2));
  return f;
}

// Two floats -> bf16x2 with round to nearest even (`hi` -> upper half).
__device__ __forceinline__ uint32_t cvt_bf16x2(float hi, float lo) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// The two FP32 lanes of a pair -> bf16x2 (low lane -> low half), RNE.
__device__ __forceinline__ uint32_t cvt_bf16x2_pair(uint64_t v) {
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
  return cvt_bf16x2(hi, lo);
}

// Two E4M3 codes -> their exact BF16 images (bf16x2, low byte -> low half).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t codes16) {
  const uint32_t h2 = e4m3x2_to_f16x2(codes16);
  return cvt_bf16x2(f16_hi_to_f32(h2), f16_lo_to_f32(h2));
}

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

// Output tile t of a persistent GEMM -> (token tile, weight tile). Tiles run
// in groups of gm token tiles: within a group the token tiles of one weight
// tile are neighbours (they share its slabs through L2), and a group sweeps
// every weight tile before the next group starts, so the group's activation
// rows stay in L2 while the weight streams past. The last group may be
// smaller.
__host__ __device__ __forceinline__ void tile_coords(int t, int mtiles, int ntiles_n, int gm,
                                                     int& mt, int& nt) {
  const int per = gm * ntiles_n;
  const int first = (t / per) * gm;
  const int r = t % per;
  const int gsz = mtiles - first < gm ? mtiles - first : gm;
  nt = r / gsz;
  mt = first + r % gsz;
}

}  // namespace fp8blk
