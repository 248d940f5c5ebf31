// The C ABI of include/fp8blk.h: argument validation (always before any CUDA
// call), the compute-capability gate, the device error word, tensor-map
// encoding, and the launches. No allocation, no synchronization (except in
// fp8blk_read_device_error, which says so).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <set>
#include <utility>

#include "fp8blk.h"
#include "internal.cuh"
#include "ptx.cuh"

namespace fp8blk {

// Bit flags set by kernels whose bounded waits ran out (see ptx.cuh).
__device__ unsigned g_device_error = 0;

// The failure-detection path on its own: one warp waits, with the kernels'
// bounded wait, on an mbarrier phase that nothing completes; the wait gives
// up after limit_cycles, sets kErrWaitSelfTest and the kernel returns.
__global__ void selftest_wait_kernel(unsigned* err, long long limit_cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none comes
    mbar_init_fence();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait_for(&bar, 0u, err, kErrWaitSelfTest, limit_cycles);
}

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool probed = false;
  bool supported = false;
  int num_sms = 0;
  unsigned* err = nullptr;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

// Probes the current device once: compute capability 10.x required (the
// kernels use tcgen05, TMEM and sm_100a TMA forms; there is no fallback).
fp8blk_status current_device(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP8BLK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FP8BLK_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FP8BLK_ERR_CUDA;
    d.supported = (major == 10);
    d.num_sms = sms;
    if (d.supported) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return FP8BLK_ERR_CUDA;
      d.err = static_cast<unsigned*>(p);
    }
    d.probed = true;
  }
  if (!d.supported) return FP8BLK_ERR_UNSUPPORTED_DEVICE;
  *out = d;
  return FP8BLK_OK;
}

fp8blk_status make_launch(fp8blk_stream stream, Launch* L) {
  DeviceInfo d;
  fp8blk_status st = current_device(&d);
  if (st != FP8BLK_OK) return st;
  L->stream = static_cast<cudaStream_t>(stream);
  L->err = d.err;
  L->num_sms = d.num_sms;
  return FP8BLK_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

fp8blk_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP8BLK_OK : FP8BLK_ERR_CUDA; }

constexpr int64_t kInt32Max = 0x7FFFFFFFLL;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int64_t w8a8_ldqx(int64_t K) { return round_up(K, 16); }
int64_t w8a8_ldsx(int64_t M) { return round_up(M, 128); }
int64_t w8a8_sx_offset(int64_t M, int64_t K) { return round_up(M * w8a8_ldqx(K), 256); }

}  // namespace

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t ensure_smem_limit(const void* kernel, size_t bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({kernel, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) done.insert({kernel, dev});
  return e;
}

// The argument checks of the linear calls, without any CUDA call (also used
// to check every job of a streamed sequence before anything is enqueued).
fp8blk_status validate_linear(const void* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                              const float* scale_inv, const void* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, const void* ws, size_t ws_bytes,
                              size_t ws_need) {
  if (M < 0 || N < 0 || K < 0) return FP8BLK_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FP8BLK_OK;
  if (!y || ldy < N) return FP8BLK_ERR_INVALID_ARG;
  if (ldy % 8 || !aligned(y, 16)) return FP8BLK_ERR_ALIGNMENT;
  if (K > 0) {
    if (!x || !q || !scale_inv || ldx < K || ldq < K) return FP8BLK_ERR_INVALID_ARG;
    if (M > kInt32Max || N > kInt32Max || K > kInt32Max) return FP8BLK_ERR_INVALID_ARG;
    if (ldx % 8 || ldq % 16 || !aligned(x, 16) || !aligned(q, 16) || !aligned(scale_inv, 4))
      return FP8BLK_ERR_ALIGNMENT;
    if (ws_need > 0 && (!ws || ws_bytes < ws_need || !aligned(ws, 256)))
      return FP8BLK_ERR_WORKSPACE;
  }
  return FP8BLK_OK;
}

// The workspace a linear call cannot run without (fp8blk_workspace_size
// gives the size that enables every path; for W8A16 above 128 tokens the
// stream-K tail it enables is optional).
size_t required_workspace(int mode, int64_t M, int64_t N, int64_t K) {
  if (mode == 0) return (M <= 0 || N <= 0 || K <= 0) ? 0 : w8a16_workspace_required(M, N, K);
  return fp8blk_workspace_size(mode, M, N, K);
}

// The launch context of the current device (stream, error word, SM count),
// for entry points defined in other files.
fp8blk_status current_launch(fp8blk_stream stream, Launch* L) { return make_launch(stream, L); }

}  // namespace fp8blk

using namespace fp8blk;

extern "C" {

fp8blk_status fp8blk_quantize_weight(const void* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q,
                                     int64_t ldq, float* scale_inv, fp8blk_stream stream) {
  if (N < 0 || K < 0) return FP8BLK_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return FP8BLK_OK;
  if (!w || !q || !scale_inv || ldw < K || ldq < K) return FP8BLK_ERR_INVALID_ARG;
  if (cdiv(N, 128) * cdiv(K, 128) > kInt32Max) return FP8BLK_ERR_INVALID_ARG;
  if (ldw % 8 || ldq % 16 || !aligned(w, 16) || !aligned(q, 16) || !aligned(scale_inv, 4))
    return FP8BLK_ERR_ALIGNMENT;
  Launch L;
  fp8blk_status st = make_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  return cuda_status(launch_quantize_weight(L, static_cast<const uint16_t*>(w), N, K, ldw, q, ldq,
                                            scale_inv));
}

fp8blk_status fp8blk_dequantize(const uint8_t* q, int64_t ldq, const float* scale_inv, int64_t N,
                                int64_t K, void* w, int64_t ldw, fp8blk_stream stream) {
  if (N < 0 || K < 0) return FP8BLK_ERR_INVALID_ARG;
  if (N == 0 || K == 0) return FP8BLK_OK;
  if (!w || !q || !scale_inv || ldw < K || ldq < K) return FP8BLK_ERR_INVALID_ARG;
  if (ldw % 8 || ldq % 16 || !aligned(w, 16) || !aligned(q, 16) || !aligned(scale_inv, 4))
    return FP8BLK_ERR_ALIGNMENT;
  Launch L;
  fp8blk_status st = make_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  return cuda_status(
      launch_dequantize(L, q, ldq, scale_inv, N, K, static_cast<uint16_t*>(w), ldw));
}

fp8blk_status fp8blk_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* qx,
                                  int64_t ldqx, float* sx, int64_t ldsx, fp8blk_stream stream) {
  if (M < 0 || K < 0) return FP8BLK_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return FP8BLK_OK;
  if (!x || !qx || !sx || ldx < K || ldqx < K || ldsx < M) return FP8BLK_ERR_INVALID_ARG;
  if (cdiv(K, 128) > kInt32Max) return FP8BLK_ERR_INVALID_ARG;
  if (ldx % 8 || ldqx % 16 || ldsx % 4 || !aligned(x, 16) || !aligned(qx, 16) || !aligned(sx, 16))
    return FP8BLK_ERR_ALIGNMENT;
  Launch L;
  fp8blk_status st = make_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  return cuda_status(
      launch_quantize_act(L, static_cast<const uint16_t*>(x), M, K, ldx, qx, ldqx, sx, ldsx));
}

namespace {

// Shared checks of the two linear calls. Returns FP8BLK_OK with *done set
// when there is nothing to compute (M or N is 0, or K is 0 and y was zeroed).
fp8blk_status check_linear(const void* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                           const float* scale_inv, void* y, int64_t ldy, int64_t M, int64_t N,
                           int64_t K, void* ws, size_t ws_bytes, size_t ws_need,
                           fp8blk_stream stream, Launch* L, bool* done) {
  *done = false;
  fp8blk_status st = validate_linear(x, ldx, q, ldq, scale_inv, y, ldy, M, N, K, ws, ws_bytes, ws_need);
  if (st != FP8BLK_OK) return st;
  if (M == 0 || N == 0) {
    *done = true;
    return FP8BLK_OK;
  }
  st = make_launch(stream, L);
  if (st != FP8BLK_OK) return st;
  if (K == 0) {  // empty sum: y = 0
    *done = true;
    return cuda_status(cudaMemset2DAsync(y, static_cast<size_t>(ldy) * 2, 0,
                                         static_cast<size_t>(N) * 2, static_cast<size_t>(M),
                                         L->stream));
  }
  return FP8BLK_OK;
}

}  // namespace

fp8blk_status fp8blk_linear_w8a16(const void* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                                  const float* scale_inv, void* y, int64_t ldy, int64_t M,
                                  int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                                  fp8blk_stream stream) {
  Launch L;
  bool done = false;
  fp8blk_status st = check_linear(x, ldx, q, ldq, scale_inv, y, ldy, M, N, K, workspace,
                                  workspace_bytes, required_workspace(0, M, N, K), stream, &L,
                                  &done);
  if (st != FP8BLK_OK || done) return st;
  return cuda_status(launch_w8a16_gemm(L, static_cast<const uint16_t*>(x), ldx, q, ldq, scale_inv,
                                       static_cast<uint16_t*>(y), ldy, M, N, K, workspace,
                                       workspace_bytes));
}

fp8blk_status fp8blk_linear_w8a8(const void* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                                 const float* scale_inv, void* y, int64_t ldy, int64_t M,
                                 int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                                 fp8blk_stream stream) {
  Launch L;
  bool done = false;
  fp8blk_status st = check_linear(x, ldx, q, ldq, scale_inv, y, ldy, M, N, K, workspace,
                                  workspace_bytes, fp8blk_workspace_size(1, M, N, K), stream, &L,
                                  &done);
  if (st != FP8BLK_OK || done) return st;
  uint8_t* qx = static_cast<uint8_t*>(workspace);
  float* sx = reinterpret_cast<float*>(qx + w8a8_sx_offset(M, K));
  const int64_t ldqx = w8a8_ldqx(K), ldsx = w8a8_ldsx(M);
  cudaError_t e =
      launch_quantize_act(L, static_cast<const uint16_t*>(x), M, K, ldx, qx, ldqx, sx, ldsx);
  if (e != cudaSuccess) return FP8BLK_ERR_CUDA;
  return cuda_status(launch_w8a8_gemm(L, qx, ldqx, sx, ldsx, q, ldq, scale_inv,
                                      static_cast<uint16_t*>(y), ldy, M, N, K, true));
}

fp8blk_status fp8blk_linear_sequence(const fp8blk_linear_args* jobs, int64_t njobs,
                                     void* workspace, size_t workspace_bytes,
                                     fp8blk_stream stream) {
  if (njobs < 0) return FP8BLK_ERR_INVALID_ARG;
  if (njobs == 0) return FP8BLK_OK;
  if (!jobs) return FP8BLK_ERR_INVALID_ARG;
  for (int64_t i = 0; i < njobs; ++i) {
    const fp8blk_linear_args& j = jobs[i];
    if (j.mode != 0 && j.mode != 1) return FP8BLK_ERR_INVALID_ARG;
    const fp8blk_status st = validate_linear(j.x, j.ldx, j.q, j.ldq, j.scale_inv, j.y, j.ldy, j.M,
                                             j.N, j.K, workspace, workspace_bytes,
                                             required_workspace(j.mode, j.M, j.N, j.K));
    if (st != FP8BLK_OK) return st;
  }
  Launch L;
  fp8blk_status st = make_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  // The first kernel waits for everything before the call; after it, each
  // GEMM may read its (read-only) weights before the kernel before it ends.
  bool first = true;
  for (int64_t i = 0; i < njobs; ++i) {
    const fp8blk_linear_args& j = jobs[i];
    if (j.M == 0 || j.N == 0) continue;
    if (j.K == 0) {
      if (cudaMemset2DAsync(j.y, static_cast<size_t>(j.ldy) * 2, 0, static_cast<size_t>(j.N) * 2,
                            static_cast<size_t>(j.M), L.stream) != cudaSuccess)
        return FP8BLK_ERR_CUDA;
      continue;
    }
    cudaError_t e;
    if (j.mode == 0) {
      e = launch_w8a16_gemm(L, static_cast<const uint16_t*>(j.x), j.ldx, j.q, j.ldq, j.scale_inv,
                            static_cast<uint16_t*>(j.y), j.ldy, j.M, j.N, j.K, workspace,
                            workspace_bytes, !first);
    } else {
      uint8_t* qx = static_cast<uint8_t*>(workspace);
      float* sx = reinterpret_cast<float*>(qx + w8a8_sx_offset(j.M, j.K));
      const int64_t ldqx = w8a8_ldqx(j.K), ldsx = w8a8_ldsx(j.M);
      e = launch_quantize_act(L, static_cast<const uint16_t*>(j.x), j.M, j.K, j.ldx, qx, ldqx, sx,
                              ldsx, !first);
      if (e == cudaSuccess)
        e = launch_w8a8_gemm(L, qx, ldqx, sx, ldsx, j.q, j.ldq, j.scale_inv,
                             static_cast<uint16_t*>(j.y), j.ldy, j.M, j.N, j.K, true);
    }
    if (e != cudaSuccess) return FP8BLK_ERR_CUDA;
    first = false;
  }
  return FP8BLK_OK;
}

fp8blk_status fp8blk_linear_w8a8_quantized(const uint8_t* qx, int64_t ldqx, const float* sx,
                                           int64_t ldsx, const uint8_t* q, int64_t ldq,
                                           const float* scale_inv, void* y, int64_t ldy, int64_t M,
                                           int64_t N, int64_t K, fp8blk_stream stream) {
  if (M < 0 || N < 0 || K < 0) return FP8BLK_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return FP8BLK_OK;
  if (!y || ldy < N) return FP8BLK_ERR_INVALID_ARG;
  if (ldy % 8 || !aligned(y, 16)) return FP8BLK_ERR_ALIGNMENT;
  if (K > 0) {
    if (!qx || !sx || !q || !scale_inv || ldqx < K || ldsx < M || ldq < K)
      return FP8BLK_ERR_INVALID_ARG;
    if (M > kInt32Max || N > kInt32Max || K > kInt32Max) return FP8BLK_ERR_INVALID_ARG;
    if (ldqx % 16 || ldq % 16 || !aligned(qx, 16) || !aligned(q, 16) || !aligned(sx, 4) ||
        !aligned(scale_inv, 4))
      return FP8BLK_ERR_ALIGNMENT;
  }
  Launch L;
  fp8blk_status st = make_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  if (K == 0)  // empty sum: y = 0
    return cuda_status(cudaMemset2DAsync(y, static_cast<size_t>(ldy) * 2, 0,
                                         static_cast<size_t>(N) * 2, static_cast<size_t>(M),
                                         L.stream));
  return cuda_status(launch_w8a8_gemm(L, qx, ldqx, sx, ldsx, q, ldq, scale_inv,
                                      static_cast<uint16_t*>(y), ldy, M, N, K, false));
}

size_t fp8blk_workspace_size(int mode, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return 0;
  if (M == 0 || N == 0 || K == 0) return 0;
  if (mode == 0) return w8a16_workspace_bytes(M, N, K);
  if (mode == 1)
    return static_cast<size_t>(w8a8_sx_offset(M, K) + cdiv(K, 128) * w8a8_ldsx(M) * 4);
  return 0;
}

fp8blk_status fp8blk_encode_e4m3(const float* v, int64_t n, uint8_t* codes, fp8blk_stream stream) {
  if (n < 0) return FP8BLK_ERR_INVALID_ARG;
  if (n == 0) return FP8BLK_OK;
  if (!v || !codes) return FP8BLK_ERR_INVALID_ARG;
  if (!aligned(v, 16) || !aligned(codes, 16)) return FP8BLK_ERR_ALIGNMENT;
  Launch L;
  fp8blk_status st = make_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  return cuda_status(launch_encode_e4m3(L, v, n, codes));
}

fp8blk_status fp8blk_selftest_wait_timeout(int64_t limit_cycles, fp8blk_stream stream) {
  if (limit_cycles < 1000 || limit_cycles > kWaitLimitCycles) return FP8BLK_ERR_INVALID_ARG;
  Launch L;
  fp8blk_status st = make_launch(stream, &L);
  if (st != FP8BLK_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, L.stream>>>(L.err, limit_cycles);
  return cuda_status(cudaGetLastError());
}

fp8blk_status fp8blk_read_device_error(uint32_t* word) {
  if (!word) return FP8BLK_ERR_INVALID_ARG;
  DeviceInfo d;
  fp8blk_status st = current_device(&d);
  if (st != FP8BLK_OK) return st;
  unsigned v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return FP8BLK_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return FP8BLK_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
    return FP8BLK_ERR_CUDA;
  *word = v;
  return v ? FP8BLK_ERR_TIMEOUT : FP8BLK_OK;
}

const char* fp8blk_status_string(fp8blk_status s) {
  switch (s) {
    case FP8BLK_OK: return "ok";
    case FP8BLK_ERR_INVALID_ARG: return "invalid argument";
    case FP8BLK_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case FP8BLK_ERR_UNSUPPORTED_DEVICE: return "device is not compute capability 10.x";
    case FP8BLK_ERR_WORKSPACE: return "workspace missing or too small";
    case FP8BLK_ERR_CUDA: return "CUDA error";
    case FP8BLK_ERR_TIMEOUT: return "a kernel wait timed out";
  }
  return "unknown status";
}

int fp8blk_version(void) { return 100; }

}  // extern "C"
