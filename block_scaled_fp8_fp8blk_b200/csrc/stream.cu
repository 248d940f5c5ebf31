// Layerwise FP8 weight streaming: linears whose E4M3 codes and block scales
// stay in host memory run through a ring of device weight slots, each slot
// refilled by the copy engine while the linears before it compute
// (FastVideo PR #1829, "Purpose": the FP8 checkpoint halves the bytes an
// offloaded encoder moves and what a resident one holds).
//
// Two streams and two events per slot: on `copy`, job i waits for the
// linear that last read its slot (event "free"), copies codes and scales in
// and records "full"; on `compute` it waits for "full", runs the linear and
// records "free". Everything is enqueued from the host in job order, so each
// wait sees the record it is meant to see. The copies are plain
// cudaMemcpyAsync calls, one per buffer.
#include <cuda_runtime.h>

#include "internal.cuh"

namespace fp8blk {
namespace {

constexpr size_t kSlotAlign = 256;

size_t round_up_sz(size_t a, size_t b) { return (a + b - 1) / b * b; }

size_t codes_bytes(int64_t N, int64_t ldq) {
  return static_cast<size_t>(N) * static_cast<size_t>(ldq);
}

size_t scale_bytes(int64_t N, int64_t K) {
  return static_cast<size_t>(cdiv(N, 128)) * static_cast<size_t>(cdiv(K, 128)) * sizeof(float);
}

}  // namespace
}  // namespace fp8blk

using namespace fp8blk;

extern "C" {

size_t fp8blk_stream_slot_bytes(int64_t N, int64_t K, int64_t ldq) {
  if (N < 0 || K < 0 || ldq < K) return 0;
  return round_up_sz(round_up_sz(codes_bytes(N, ldq), kSlotAlign) + scale_bytes(N, K), kSlotAlign);
}

fp8blk_status fp8blk_streamed_linears(const fp8blk_linear_job* jobs, int64_t njobs, void* slots,
                                      size_t slot_bytes, int32_t nslots, void* workspace,
                                      size_t workspace_bytes, fp8blk_stream compute,
                                      fp8blk_stream copy, fp8blk_event* events) {
  if (njobs < 0 || nslots < 1) return FP8BLK_ERR_INVALID_ARG;
  if (njobs == 0) return FP8BLK_OK;
  if (!jobs || !slots || !events || slot_bytes == 0) return FP8BLK_ERR_INVALID_ARG;
  if (slot_bytes % kSlotAlign || reinterpret_cast<uintptr_t>(slots) % kSlotAlign)
    return FP8BLK_ERR_ALIGNMENT;
  for (int32_t e = 0; e < 2 * nslots; ++e)
    if (!events[e]) return FP8BLK_ERR_INVALID_ARG;
  // Every job is checked, against the slot it will read its weights from,
  // before anything is enqueued.
  for (int64_t i = 0; i < njobs; ++i) {
    const fp8blk_linear_job& j = jobs[i];
    if (j.mode != 0 && j.mode != 1) return FP8BLK_ERR_INVALID_ARG;
    if (j.M < 0 || j.N < 0 || j.K < 0 || j.ldq < j.K) return FP8BLK_ERR_INVALID_ARG;
    if (j.M == 0 || j.N == 0) continue;
    if (j.K > 0 && (!j.q_host || !j.scale_host)) return FP8BLK_ERR_INVALID_ARG;
    if (fp8blk_stream_slot_bytes(j.N, j.K, j.ldq) > slot_bytes) return FP8BLK_ERR_INVALID_ARG;
    uint8_t* slot = static_cast<uint8_t*>(slots) + static_cast<size_t>(i % nslots) * slot_bytes;
    const float* s_dev = reinterpret_cast<const float*>(slot + round_up_sz(codes_bytes(j.N, j.ldq), kSlotAlign));
    const fp8blk_status st = validate_linear(j.x, j.ldx, slot, j.ldq, s_dev, j.y, j.ldy, j.M, j.N,
                                             j.K, workspace, workspace_bytes,
                                             required_workspace(j.mode, j.M, j.N, j.K));
    if (st != FP8BLK_OK) return st;
  }
  Launch L;
  fp8blk_status st = current_launch(compute, &L);  // device check
  if (st != FP8BLK_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(compute), ps = static_cast<cudaStream_t>(copy);
  // No copy of this call may start before the work already enqueued on
  // `compute` (an earlier call's linears may still read the slots).
  if (cudaEventRecord(static_cast<cudaEvent_t>(events[1]), cs) != cudaSuccess ||
      cudaStreamWaitEvent(ps, static_cast<cudaEvent_t>(events[1]), 0) != cudaSuccess)
    return FP8BLK_ERR_CUDA;
  for (int64_t i = 0; i < njobs; ++i) {
    const fp8blk_linear_job& j = jobs[i];
    const int32_t k = static_cast<int32_t>(i % nslots);
    cudaEvent_t full = static_cast<cudaEvent_t>(events[2 * k]);
    cudaEvent_t free_ev = static_cast<cudaEvent_t>(events[2 * k + 1]);
    uint8_t* slot = static_cast<uint8_t*>(slots) + static_cast<size_t>(k) * slot_bytes;
    float* s_dev = reinterpret_cast<float*>(slot + round_up_sz(codes_bytes(j.N, j.ldq), kSlotAlign));
    // The slot was last read by job i - nslots.
    if (i >= nslots && cudaStreamWaitEvent(ps, free_ev, 0) != cudaSuccess) return FP8BLK_ERR_CUDA;
    if (j.M > 0 && j.N > 0 && j.K > 0) {
      if (cudaMemcpyAsync(slot, j.q_host, codes_bytes(j.N, j.ldq), cudaMemcpyHostToDevice, ps) !=
              cudaSuccess ||
          cudaMemcpyAsync(s_dev, j.scale_host, scale_bytes(j.N, j.K), cudaMemcpyHostToDevice, ps) !=
              cudaSuccess)
        return FP8BLK_ERR_CUDA;
    }
    if (cudaEventRecord(full, ps) != cudaSuccess || cudaStreamWaitEvent(cs, full, 0) != cudaSuccess)
      return FP8BLK_ERR_CUDA;
    st = j.mode == 0
             ? fp8blk_linear_w8a16(j.x, j.ldx, slot, j.ldq, s_dev, j.y, j.ldy, j.M, j.N, j.K,
                                   workspace, workspace_bytes, compute)
             : fp8blk_linear_w8a8(j.x, j.ldx, slot, j.ldq, s_dev, j.y, j.ldy, j.M, j.N, j.K,
                                  workspace, workspace_bytes, compute);
    if (st != FP8BLK_OK) return st;
    if (cudaEventRecord(free_ev, cs) != cudaSuccess) return FP8BLK_ERR_CUDA;
  }
  return FP8BLK_OK;
}

}  // extern "C"
