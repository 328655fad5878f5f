// linear_noalloc.cu -- the W8A8 linear layer for callers that cannot
// allocate device memory.
//
// Some callers of a linear layer cannot hand it a workspace and must not
// make it allocate one: a runtime whose device memory is entirely
// pre-reserved by another framework's pool (cudaMalloc would fail), code on
// a latency-critical path where cudaMalloc / cudaFree would synchronize the
// device, or a plugin interface that offers inputs and outputs but no
// scratch.  w8a8_linear needs scratch for the quantized activations (M*K
// int8) and their per-token scales (M floats); this entry point takes that
// scratch from one fixed array compiled into the library instead.
//
// The array is a file-scope __device__ variable of kScratchBytes bytes:
// every GPU that loads the library holds it until the process exits.  Host
// code cannot use the array's name as a device address (it names a host-side
// stand-in), so the address is looked up with cudaGetSymbolAddress, once
// per device, with that device current, on the first call on that device.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/w8a8.h"
#include "internal.h"

namespace w8a8 {
namespace {

// 32 MiB: the codes and scales of up to 32 Mi activation elements, e.g.
// 9216 tokens x 3072 features, or 4096 x 8192.
constexpr int64_t kScratchBytes = 32LL << 20;

static __device__ __align__(256) uint8_t g_linear_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_linear_scratch on the current device (set up on the
// first call on each device).
cudaError_t scratch_address(uint8_t** out) {
  static uint8_t* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_linear_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace w8a8

extern "C" w8a8_status w8a8_linear_noalloc(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                                           void* out, int64_t M, int64_t N, int64_t K, w8a8_stream_t stream) {
  using namespace w8a8;
  // The same checks as w8a8_linear, in the same order, before any CUDA
  // call; then the device; only then the scratch capacity and its address.
  w8a8_status st = check_linear_io(x, wq, scale_w, bias, out, M, N, K);
  if (st != W8A8_OK) return st;
  if (M == 0 || N == 0) return W8A8_OK;
  if ((st = check_current_device()) != W8A8_OK) return st;
  const int64_t code_bytes = (M * K + 255) / 256 * 256;  // scales start 256-byte aligned
  if (code_bytes + 4 * M > kScratchBytes) return W8A8_ERR_SCRATCH_LIMIT;
  uint8_t* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return W8A8_ERR_CUDA;
  int8_t* xq = reinterpret_cast<int8_t*>(base);
  float* scale_a = reinterpret_cast<float*>(base + code_bytes);
  // The quantizer rewrites every code and scale the GEMM then reads, so
  // nothing in the scratch has to start at zero.
  return w8a8_linear(x, wq, scale_w, bias, out, xq, scale_a, M, N, K, stream);
}
