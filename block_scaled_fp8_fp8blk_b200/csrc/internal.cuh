// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "fp8blk.h"

namespace fp8blk {

struct Launch {
  cudaStream_t stream;
  unsigned* err;  // device error word (bounded-wait time-outs)
  int num_sms;
};

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }

// Token tiles per raster group of a persistent GEMM (see tile_coords): as
// many as keep a group's activation rows within `budget` bytes, in groups of
// near-equal size. Measured on the large-token linears: W8A8 with 24 MB of
// activation codes per group; W8A16 with up to 48 MB of BF16 activations
// (M = 4096 stays one group: two groups of 21 MB ran slower there).
constexpr int64_t kRasterBytesW8A8 = 24ll << 20;
constexpr int64_t kRasterBytesW8A16 = 48ll << 20;
inline int raster_group(int64_t mtiles, int64_t bytes_per_mtile, int64_t budget) {
  const int64_t most = bytes_per_mtile > 0 ? budget / bytes_per_mtile : mtiles;
  const int64_t groups = cdiv(mtiles, most > 0 ? most : 1);
  return static_cast<int>(cdiv(mtiles, groups > 0 ? groups : 1));
}

cudaError_t launch_quantize_weight(const Launch& L, const uint16_t* w, int64_t N, int64_t K,
                                   int64_t ldw, uint8_t* q, int64_t ldq, float* scale_inv);
cudaError_t launch_dequantize(const Launch& L, const uint8_t* q, int64_t ldq,
                              const float* scale_inv, int64_t N, int64_t K, uint16_t* w,
                              int64_t ldw);
// pdl: launched as a programmatic dependent of the kernel before it (which
// may still be running; the kernel reads x only after griddepcontrol.wait).
cudaError_t launch_quantize_act(const Launch& L, const uint16_t* x, int64_t M, int64_t K,
                                int64_t ldx, uint8_t* qx, int64_t ldqx, float* sx, int64_t ldsx,
                                bool pdl = false);
cudaError_t launch_encode_e4m3(const Launch& L, const float* v, int64_t n, uint8_t* codes);

// after_act_quant: launched right after launch_quantize_act on the same
// stream, as its programmatic dependent (weight loads overlap that kernel).
cudaError_t launch_w8a8_gemm(const Launch& L, const uint8_t* qx, int64_t ldqx, const float* sx,
                             int64_t ldsx, const uint8_t* q, int64_t ldq, const float* scale_inv,
                             uint16_t* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                             bool after_act_quant);

// Workspace of the W8A16 call: the size that enables every stream-K path,
// and the part of it that is required (M <= 128; for M > 128 a smaller or
// missing workspace runs every tile whole).
size_t w8a16_workspace_bytes(int64_t M, int64_t N, int64_t K);
size_t w8a16_workspace_required(int64_t M, int64_t N, int64_t K);
// Always a programmatic dependent of the kernel before it; early_weights:
// that kernel does not write q or scale_inv, so the weight stream may start
// before it has completed (x, y and the workspace still wait for it).
cudaError_t launch_w8a16_gemm(const Launch& L, const uint16_t* x, int64_t ldx, const uint8_t* q,
                              int64_t ldq, const float* scale_inv, uint16_t* y, int64_t ldy,
                              int64_t M, int64_t N, int64_t K, void* ws, size_t ws_bytes,
                              bool early_weights = false);

// 2-D tiled tensor map (128-byte swizzling unless stated) over a row-major
// matrix [outer][inner] whose rows are row_bytes apart; out-of-bounds reads
// are zero-filled and out-of-bounds parts of a store are dropped. Returns
// false when the driver rejects the description.
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

// Sets the kernel's dynamic shared-memory limit once per device.
cudaError_t ensure_smem_limit(const void* kernel, size_t bytes);

// The workspace a linear call cannot run without (for W8A16 above 128 tokens
// 0: its stream-K tail runs only when the workspace given is large enough).
size_t required_workspace(int mode, int64_t M, int64_t N, int64_t K);

// The launch context of the current device (checks compute capability 10.x).
fp8blk_status current_launch(fp8blk_stream stream, Launch* L);

// Argument checks of a linear call (no CUDA call): FP8BLK_OK, INVALID_ARG,
// ALIGNMENT or WORKSPACE; ws_need is fp8blk_workspace_size of the call.
fp8blk_status validate_linear(const void* x, int64_t ldx, const uint8_t* q, int64_t ldq,
                              const float* scale_inv, const void* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, const void* ws, size_t ws_bytes,
                              size_t ws_need);

}  // namespace fp8blk
