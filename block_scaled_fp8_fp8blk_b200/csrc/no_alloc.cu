// fp8blk_linear_w8a8_noalloc: the W8A8 linear for callers that cannot hand
// the library a workspace.
//
// fp8blk_linear_w8a8 needs scratch device memory for the quantized
// activations (codes and per-group scales). Some callers cannot allocate it:
// an inference runtime that plans all device memory up front and forbids any
// allocation once it is serving, or host code that must not call cudaMalloc
// because that call can synchronize the whole device and stall other streams.
// This entry point takes the scratch from a fixed array compiled into the
// library instead, so the caller passes only x, the weight and y.
//
// The array is FP8BLK_NOALLOC_SCRATCH_BYTES (16 MiB) on every GPU that loads
// the library, held until the process exits. Its address is looked up once
// per device with cudaGetSymbolAddress, on the first call made while that
// device is current; that first call must not be made during stream capture
// (it is refused with FP8BLK_ERR_INVALID_ARG).
#include <cuda_runtime.h>

#include <mutex>

#include "fp8blk.h"
#include "internal.cuh"

// The shared scratch: quantized activation codes at offset 0, group scales
// after them (the same layout as the fp8blk_linear_w8a8 workspace). Nothing
// in it needs to start at zero: every byte a call reads is written earlier in
// that call, or lies in padding rows whose results are never stored.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FP8BLK_NOALLOC_SCRATCH_BYTES];

namespace fp8blk {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (host code may
// not use the symbol itself: on the host it is only a stand-in). The lookup
// is made once per device; a first call while `stream` is being captured is
// refused (INVALID_ARG), since the lookup may load the module.
fp8blk_status scratch_address(cudaStream_t stream, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8BLK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FP8BLK_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return FP8BLK_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return FP8BLK_ERR_INVALID_ARG;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FP8BLK_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return FP8BLK_OK;
}

}  // namespace
}  // namespace fp8blk

using namespace fp8blk;

extern "C" fp8blk_status fp8blk_linear_w8a8_noalloc(const void* x, int64_t ldx, const uint8_t* q,
                                                    int64_t ldq, const float* scale_inv, void* y,
                                                    int64_t ldy, int64_t M, int64_t N, int64_t K,
                                                    fp8blk_stream stream) {
  // The checks of fp8blk_linear_w8a8, without its workspace.
  fp8blk_status st = validate_linear(x, ldx, q, ldq, scale_inv, y, ldy, M, N, K, nullptr, 0, 0);
  if (st != FP8BLK_OK) return st;
  if (M == 0 || N == 0) return FP8BLK_OK;
  Launch L;
  st = current_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  if (K == 0)  // an empty sum: y = 0 (no scratch involved)
    return cudaMemset2DAsync(y, static_cast<size_t>(ldy) * 2, 0, static_cast<size_t>(N) * 2,
                             static_cast<size_t>(M), L.stream) == cudaSuccess
               ? FP8BLK_OK
               : FP8BLK_ERR_CUDA;
  // Same layout as the W8A8 workspace; refuse problems that do not fit.
  const size_t need = fp8blk_workspace_size(1, M, N, K);
  if (need > static_cast<size_t>(FP8BLK_NOALLOC_SCRATCH_BYTES)) return FP8BLK_ERR_WORKSPACE;
  void* scratch = nullptr;
  st = scratch_address(L.stream, &scratch);
  if (st != FP8BLK_OK) return st;

  uint8_t* qx = static_cast<uint8_t*>(scratch);
  const int64_t ldqx = round_up(K, 16), ldsx = round_up(M, 128);
  float* sx = reinterpret_cast<float*>(qx + round_up(M * ldqx, 256));
  if (launch_quantize_act(L, static_cast<const uint16_t*>(x), M, K, ldx, qx, ldqx, sx, ldsx) !=
      cudaSuccess)
    return FP8BLK_ERR_CUDA;
  return launch_w8a8_gemm(L, qx, ldqx, sx, ldsx, q, ldq, scale_inv, static_cast<uint16_t*>(y), ldy,
                          M, N, K, true) == cudaSuccess
             ? FP8BLK_OK
             : FP8BLK_ERR_CUDA;
}
