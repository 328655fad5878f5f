// internal.h -- launchers shared between the library's translation units.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/w8a8.h"

namespace w8a8 {

// Tile configuration of the GEMM kernel (see w8a8_gemm_config in w8a8.h).
struct GemmConfig {
  int block_m;
  int block_n;
  int stages;
  int grid;
  int raster_group;
};

// kAcc32: the raw 32-bit accumulators (int32 for int8 operands, fp32 for
// E4M3 operands) instead of the dequantized bf16 output.
enum class GemmOut { kBf16Dequant = 0, kAcc32 = 1 };

// Operand format: int8 (tcgen05 kind::i8, int32 accumulators) or OCP E4M3
// (kind::f8f6f4, fp32 accumulators).
enum class GemmElem { kInt8 = 0, kE4M3 = 1 };

struct GemmArgs {
  const int8_t* xq;  // int8 or E4M3 codes (bytes)
  const int8_t* wq;
  const float* scale_a;
  const float* scale_w;
  const void* bias;  // bf16 [N] or nullptr
  void* out;         // bf16 [M, N] or int32 [M, N]
  int64_t M, N, K;
  GemmOut out_kind;
  GemmElem elem = GemmElem::kInt8;
  uint64_t timeout_ns;
  int64_t l2_bytes = 0;  // L2 size of the device (chooses the A operand's cache policy)
  // The fused linear layer: quantize x [M, K] (bf16, row stride ldx) into
  // xq / scale_a inside the GEMM kernel (xq and scale_a are then outputs);
  // sync is the zeroed row-block counter workspace (linear_sync_words(M)).
  bool fused = false;
  // Launch as a programmatic dependent of the previous kernel (only when
  // that kernel is this library's quantizer writing xq / scale_a and
  // nothing else: the GEMM reads wq, scale_w and bias before it waits).
  bool overlap_prologue = false;
  const void* x = nullptr;
  int64_t ldx = 0;
  uint32_t* sync = nullptr;
};

// 32-bit words of the counter workspace of the fused linear layer.
inline int64_t linear_sync_words(int64_t M) { return (M + 127) / 128 + 1; }

cudaError_t launch_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq,
                                float* scale, cudaStream_t stream);
cudaError_t launch_quantize_weight(const float* w, int64_t N, int64_t K, int64_t ldw, int8_t* q, int64_t ldq,
                                   float* scale, cudaStream_t stream);
cudaError_t launch_quantize_act_e4m3(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                                     float* scale, cudaStream_t stream);
cudaError_t launch_quantize_weight_e4m3(const float* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q, int64_t ldq,
                                        float* scale, cudaStream_t stream);

// GELU before a linear layer: the per-token quantizer applied to
// bf16_rne(GELU(h)) in one pass, and the bf16 GELU alone.
cudaError_t launch_quantize_act_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, int8_t* q, int64_t ldq,
                                     float* scale, cudaStream_t stream);
cudaError_t launch_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, void* g, int64_t ldg, int sms,
                        cudaStream_t stream);
// Kernel setup for launch_quantize_act_gelu on rows of K, made before a
// stream capture that will record it.
cudaError_t prepare_quantize_act_gelu(int64_t K, cudaStream_t stream);

// Largest stage count the shared memory holds for a tile shape (0 if none).
// block_m 128: one CTA per tile; block_m 256: a CTA pair (cluster of 2).
int gemm_max_stages(int block_m, int block_n);

// Returns cudaSuccess or the launch error; tensor-map encoding failures are
// reported as cudaErrorInvalidValue.
cudaError_t launch_gemm(const GemmArgs& args, const GemmConfig& cfg, cudaStream_t stream);

cudaError_t launch_selftest_wait(uint64_t timeout_ns, cudaStream_t stream);

// Argument checks of w8a8_linear on its shapes, inputs and output (not the
// workspaces), made before any CUDA call; and the current device's support.
w8a8_status check_linear_io(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                            const void* out, int64_t M, int64_t N, int64_t K);
w8a8_status check_current_device();
// check_linear_io plus the non-null, 16-byte aligned workspaces ws_xq and ws_scale_a.
w8a8_status check_linear_call(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                              const void* out, const void* ws_xq, const float* ws_scale_a, int64_t M, int64_t N,
                              int64_t K);

// Synchronizes the current device and reads (optionally clears) the device
// error word written by timed-out waits.
cudaError_t read_device_error(int* value, bool clear);

}  // namespace w8a8
