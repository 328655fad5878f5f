// api.cu -- the C ABI declared in include/w8a8.h: argument validation,
// per-shape configuration, and the launches.
//
// Every argument check happens before any CUDA call, so a rejected call
// touches no device state and launches nothing.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/w8a8.h"
#include "internal.h"

namespace w8a8 {
namespace {

constexpr int64_t kMaxK = 133144;  // K * 127^2 < 2^31 (int8); the E4M3 path takes the same range
constexpr int64_t kMaxMN = 2147483647;
std::atomic<int64_t> g_timeout_ns{2000000000LL};

struct DeviceInfo {
  bool valid = false;
  bool supported = false;
  int sms = 0;
  int64_t l2_bytes = 0;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;

// Properties of the current device (cached).
w8a8_status current_device(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return W8A8_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceInfo& d = g_devices[dev];
  if (!d.valid) {
    int major = 0, minor = 0, sms = 0, l2 = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess) {
      return W8A8_ERR_CUDA;
    }
    d.supported = (major == 10 && minor == 0);
    d.sms = sms;
    d.l2_bytes = l2;
    d.valid = true;
  }
  *out = d;
  return d.supported ? W8A8_OK : W8A8_ERR_UNSUPPORTED_DEVICE;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

w8a8_status check_gemm_shape(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || M > kMaxMN || N > kMaxMN) return W8A8_ERR_INVALID_ARG;
  if (K < 16 || K > kMaxK || K % 16 != 0) return W8A8_ERR_INVALID_ARG;
  if (N % 8 != 0) return W8A8_ERR_INVALID_ARG;
  return W8A8_OK;
}

w8a8_status check_config(const w8a8_gemm_config& c) {
  if (c.block_m != 128 && c.block_m != 256) return W8A8_ERR_INVALID_ARG;
  if (c.block_n != 128 && c.block_n != 256) return W8A8_ERR_INVALID_ARG;
  if (c.stages < 2 || c.stages > gemm_max_stages(c.block_m, c.block_n)) return W8A8_ERR_INVALID_ARG;
  if (c.grid < (c.block_m == 256 ? 2 : 1) || c.raster_group < 1) return W8A8_ERR_INVALID_ARG;
  return W8A8_OK;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Per-shape choice of the output tile (the paper autotunes its kernel per
// GEMM shape; here a cost model over measured per-tile efficiencies).
// Candidates: 128 x 256 tiles on single CTAs, 256 x 256 tiles on CTA pairs
// (cta_group::2), and the narrower 128 x 128 / 256 x 128 tiles, which keep
// more CTAs busy on small problems but need about twice the operand bytes
// per multiply-add and measured ~1.7-1.9x slower per operation on B200.
// The pair tile is the fastest where K % 128 == 0: it then loads boxes of
// two K-chunks, which the memory system delivers at ~100 B/clk per SM
// against the 64 it needs (0.88 of the single-CTA tile's time, measured);
// otherwise it is on a par with the single-CTA tile.  Each persistent CTA
// (pair) does ceil(tiles / units) tiles, the last round in half-width items
// when that leaves at least half the units idle; a tile costs its
// multiply-adds times its relative cost, plus a fixed fill / drain overhead
// of two K blocks.
w8a8_gemm_config select(int64_t M, int64_t N, int64_t K, int sms, bool allow_pair = true) {
  struct Cand { int bm, bn; double rel_cost; int raster; };
  const double pair_cost = K % 128 == 0 ? 0.88 : 1.02;
  const Cand cands[4] = {{128, 256, 1.00, 1}, {256, 256, pair_cost, 1}, {128, 128, 1.75, 1}, {256, 128, 1.90, 8}};
  double best = 1e300;
  w8a8_gemm_config cfg{};
  const double kblocks = static_cast<double>(ceil_div(K, 128));
  for (const Cand& c : cands) {
    if (c.bm == 256 && !allow_pair) continue;
    const int units = c.bm == 256 ? sms / 2 : sms;
    const int64_t tiles = ceil_div(M, c.bm) * ceil_div(N, c.bn);
    // rounds of tiles per unit; a short last round of 256-column tiles runs
    // as half-width items (half a round)
    const int64_t tail = tiles % units;
    const double per_unit = (c.bn == 256 && tail > 0 && 2 * tail <= units && tiles > units)
                                ? static_cast<double>(tiles / units) + 0.5
                                : static_cast<double>(ceil_div(tiles, units));
    const double macs_per_sm = static_cast<double>(c.bm / (c.bm == 256 ? 2 : 1)) * c.bn;
    const double cost = per_unit * macs_per_sm * (kblocks + 2.0) * c.rel_cost;
    if (cost < best * 0.999) {
      best = cost;
      cfg.block_m = c.bm;
      cfg.block_n = c.bn;
      cfg.stages = gemm_max_stages(c.bm, c.bn);
      const int64_t used = tiles < units ? tiles : units;
      cfg.grid = static_cast<int>(used * (c.bm == 256 ? 2 : 1));
      cfg.raster_group = c.raster;
    }
  }
  return cfg;
}

w8a8_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return W8A8_OK;
  if (e == cudaErrorInvalidValue) return W8A8_ERR_INVALID_ARG;
  return W8A8_ERR_LAUNCH;
}

w8a8_status gemm_common(const int8_t* xq, const int8_t* wq, const float* scale_a, const float* scale_w,
                        const void* bias, void* out, int64_t M, int64_t N, int64_t K,
                        const w8a8_gemm_config* user_cfg, GemmOut kind, cudaStream_t stream,
                        bool overlap_prologue = false, GemmElem elem = GemmElem::kInt8) {
  w8a8_status st = check_gemm_shape(M, N, K);
  if (st != W8A8_OK) return st;
  if (user_cfg != nullptr && (st = check_config(*user_cfg)) != W8A8_OK) return st;
  if (M == 0 || N == 0) return W8A8_OK;
  if (xq == nullptr || wq == nullptr || out == nullptr) return W8A8_ERR_INVALID_ARG;
  if (kind == GemmOut::kBf16Dequant && (scale_a == nullptr || scale_w == nullptr)) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(wq) || !aligned16(out) || !aligned16(scale_a) || !aligned16(scale_w) ||
      !aligned16(bias)) {
    return W8A8_ERR_ALIGNMENT;
  }
  DeviceInfo dev;
  if ((st = current_device(&dev)) != W8A8_OK) return st;
  const w8a8_gemm_config cfg = user_cfg ? *user_cfg : select(M, N, K, dev.sms);
  GemmArgs a;
  a.xq = xq;
  a.wq = wq;
  a.scale_a = scale_a;
  a.scale_w = scale_w;
  a.bias = bias;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.out_kind = kind;
  a.elem = elem;
  a.timeout_ns = static_cast<uint64_t>(g_timeout_ns.load());
  a.l2_bytes = dev.l2_bytes;
  a.overlap_prologue = overlap_prologue;
  GemmConfig c{cfg.block_m, cfg.block_n, cfg.stages, cfg.grid, cfg.raster_group};
  return from_cuda(launch_gemm(a, c, stream));
}

w8a8_status quantize_common(bool act, const void* x, int64_t M, int64_t K, int64_t ldx, int8_t* xq, int64_t ldxq,
                            float* scale, cudaStream_t stream, bool e4m3 = false, bool gelu = false) {
  if (M < 0 || M > kMaxMN || K < 16 || K > kMaxK || K % 16 != 0) return W8A8_ERR_INVALID_ARG;
  if (ldx < K || ldxq < K) return W8A8_ERR_INVALID_ARG;
  if (M == 0) return W8A8_OK;
  if (x == nullptr || xq == nullptr || scale == nullptr) return W8A8_ERR_INVALID_ARG;
  const int64_t elem = act ? 2 : 4;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(scale)) return W8A8_ERR_ALIGNMENT;
  if ((ldx * elem) % 16 != 0 || ldxq % 16 != 0) return W8A8_ERR_ALIGNMENT;
  DeviceInfo dev;
  w8a8_status st = current_device(&dev);
  if (st != W8A8_OK) return st;
  const float* w = static_cast<const float*>(x);
  uint8_t* codes = reinterpret_cast<uint8_t*>(xq);
  cudaError_t e;
  if (gelu) {
    e = launch_quantize_act_gelu(x, M, K, ldx, xq, ldxq, scale, stream);
  } else if (e4m3) {
    e = act ? launch_quantize_act_e4m3(x, M, K, ldx, codes, ldxq, scale, stream)
            : launch_quantize_weight_e4m3(w, M, K, ldx, codes, ldxq, scale, stream);
  } else {
    e = act ? launch_quantize_act(x, M, K, ldx, xq, ldxq, scale, stream)
            : launch_quantize_weight(w, M, K, ldx, xq, ldxq, scale, stream);
  }
  return from_cuda(e);
}

}  // namespace

// The checks w8a8_linear makes on its shapes and on its caller-owned inputs
// and output before any CUDA call (workspaces aside): shape, non-null
// pointers, 16-byte alignment.  W8A8_OK for an empty problem too.
w8a8_status check_linear_io(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                            const void* out, int64_t M, int64_t N, int64_t K) {
  w8a8_status st = check_gemm_shape(M, N, K);
  if (st != W8A8_OK) return st;
  if (M == 0 || N == 0) return W8A8_OK;
  if (x == nullptr || wq == nullptr || scale_w == nullptr || out == nullptr) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(wq) || !aligned16(scale_w) || !aligned16(bias) || !aligned16(out)) {
    return W8A8_ERR_ALIGNMENT;
  }
  return W8A8_OK;
}

// check_linear_io plus the caller's workspaces (non-null, 16-byte aligned):
// every check of a w8a8_linear-style call, before any CUDA call.
w8a8_status check_linear_call(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                              const void* out, const void* ws_xq, const float* ws_scale_a, int64_t M, int64_t N,
                              int64_t K) {
  w8a8_status st = check_linear_io(x, wq, scale_w, bias, out, M, N, K);
  if (st != W8A8_OK || M == 0 || N == 0) return st;
  if (ws_xq == nullptr || ws_scale_a == nullptr) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(ws_xq) || !aligned16(ws_scale_a)) return W8A8_ERR_ALIGNMENT;
  return W8A8_OK;
}

// W8A8_OK if the current device is supported (sm_100), from the cached
// device properties.
w8a8_status check_current_device() {
  DeviceInfo dev;
  return current_device(&dev);
}

}  // namespace w8a8

using namespace w8a8;

extern "C" {

const char* w8a8_status_string(int status) {
  switch (status) {
    case W8A8_OK: return "ok";
    case W8A8_ERR_INVALID_ARG: return "invalid argument";
    case W8A8_ERR_ALIGNMENT: return "pointer or stride not 16-byte aligned";
    case W8A8_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    case W8A8_ERR_LAUNCH: return "kernel launch failed";
    case W8A8_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case W8A8_ERR_CUDA: return "CUDA runtime error";
    case W8A8_ERR_SCRATCH_LIMIT: return "problem exceeds the fixed scratch of w8a8_linear_noalloc (32 MiB)";
    default: return "unknown status";
  }
}

int w8a8_abi_version(void) { return 101; }

w8a8_status w8a8_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, int8_t* xq, int64_t ldxq,
                              float* scale_a, w8a8_stream_t stream) {
  return quantize_common(true, x, M, K, ldx, xq, ldxq, scale_a, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_quantize_weight(const float* w, int64_t N, int64_t K, int64_t ldw, int8_t* wq, int64_t ldwq,
                                 float* scale_w, w8a8_stream_t stream) {
  return quantize_common(false, w, N, K, ldw, wq, ldwq, scale_w, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_gemm(const int8_t* xq, const int8_t* wq, const float* scale_a, const float* scale_w,
                      const void* bias, void* out, int64_t M, int64_t N, int64_t K, w8a8_stream_t stream) {
  return gemm_common(xq, wq, scale_a, scale_w, bias, out, M, N, K, nullptr, GemmOut::kBf16Dequant,
                     reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_gemm_ex(const int8_t* xq, const int8_t* wq, const float* scale_a, const float* scale_w,
                         const void* bias, void* out, int64_t M, int64_t N, int64_t K,
                         const w8a8_gemm_config* cfg, w8a8_stream_t stream) {
  return gemm_common(xq, wq, scale_a, scale_w, bias, out, M, N, K, cfg, GemmOut::kBf16Dequant,
                     reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_gemm_i32(const int8_t* xq, const int8_t* wq, int32_t* acc, int64_t M, int64_t N, int64_t K,
                          w8a8_stream_t stream) {
  return gemm_common(xq, wq, nullptr, nullptr, nullptr, acc, M, N, K, nullptr, GemmOut::kAcc32,
                     reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_gemm_i32_ex(const int8_t* xq, const int8_t* wq, int32_t* acc, int64_t M, int64_t N, int64_t K,
                             const w8a8_gemm_config* cfg, w8a8_stream_t stream) {
  return gemm_common(xq, wq, nullptr, nullptr, nullptr, acc, M, N, K, cfg, GemmOut::kAcc32,
                     reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_linear(const void* x, const int8_t* wq, const float* scale_w, const void* bias, void* out,
                        int8_t* ws_xq, float* ws_scale_a, int64_t M, int64_t N, int64_t K, w8a8_stream_t stream) {
  // Validate the whole call before launching its first kernel.
  w8a8_status st = check_linear_call(x, wq, scale_w, bias, out, ws_xq, ws_scale_a, M, N, K);
  if (st != W8A8_OK || M == 0 || N == 0) return st;
  st = w8a8_quantize_act(x, M, K, K, ws_xq, K, ws_scale_a, stream);
  if (st != W8A8_OK) return st;
  return gemm_common(ws_xq, wq, ws_scale_a, scale_w, bias, out, M, N, K, nullptr, GemmOut::kBf16Dequant,
                     reinterpret_cast<cudaStream_t>(stream), /*overlap_prologue=*/true);
}

w8a8_status w8a8_linear_fused(const void* x, const int8_t* wq, const float* scale_w, const void* bias, void* out,
                              int8_t* ws_xq, float* ws_scale_a, uint32_t* ws_sync, int64_t M, int64_t N, int64_t K,
                              w8a8_stream_t stream) {
  w8a8_status st = check_linear_call(x, wq, scale_w, bias, out, ws_xq, ws_scale_a, M, N, K);
  if (st != W8A8_OK || M == 0 || N == 0) return st;
  if (ws_sync == nullptr) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(ws_sync)) return W8A8_ERR_ALIGNMENT;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != W8A8_OK) return st;
  const w8a8_gemm_config cfg = select(M, N, K, dev.sms, /*allow_pair=*/false);
  GemmArgs a;
  a.xq = ws_xq;
  a.wq = wq;
  a.scale_a = ws_scale_a;
  a.scale_w = scale_w;
  a.bias = bias;
  a.out = out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.out_kind = GemmOut::kBf16Dequant;
  a.timeout_ns = static_cast<uint64_t>(g_timeout_ns.load());
  a.l2_bytes = dev.l2_bytes;
  a.fused = true;
  a.x = x;
  a.ldx = K;
  a.sync = ws_sync;
  GemmConfig c{cfg.block_m, cfg.block_n, cfg.stages, cfg.grid, cfg.raster_group};
  return from_cuda(launch_gemm(a, c, reinterpret_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ E4M3 variant

w8a8_status w8a8_quantize_act_fp8(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* xq, int64_t ldxq,
                                  float* scale_a, w8a8_stream_t stream) {
  return quantize_common(true, x, M, K, ldx, reinterpret_cast<int8_t*>(xq), ldxq, scale_a,
                         reinterpret_cast<cudaStream_t>(stream), /*e4m3=*/true);
}

w8a8_status w8a8_quantize_weight_fp8(const float* w, int64_t N, int64_t K, int64_t ldw, uint8_t* wq, int64_t ldwq,
                                     float* scale_w, w8a8_stream_t stream) {
  return quantize_common(false, w, N, K, ldw, reinterpret_cast<int8_t*>(wq), ldwq, scale_w,
                         reinterpret_cast<cudaStream_t>(stream), /*e4m3=*/true);
}

w8a8_status w8a8_gemm_fp8_ex(const uint8_t* xq, const uint8_t* wq, const float* scale_a, const float* scale_w,
                             const void* bias, void* out, int64_t M, int64_t N, int64_t K,
                             const w8a8_gemm_config* cfg, w8a8_stream_t stream) {
  return gemm_common(reinterpret_cast<const int8_t*>(xq), reinterpret_cast<const int8_t*>(wq), scale_a, scale_w,
                     bias, out, M, N, K, cfg, GemmOut::kBf16Dequant, reinterpret_cast<cudaStream_t>(stream),
                     /*overlap_prologue=*/false, GemmElem::kE4M3);
}

w8a8_status w8a8_gemm_fp8(const uint8_t* xq, const uint8_t* wq, const float* scale_a, const float* scale_w,
                          const void* bias, void* out, int64_t M, int64_t N, int64_t K, w8a8_stream_t stream) {
  return w8a8_gemm_fp8_ex(xq, wq, scale_a, scale_w, bias, out, M, N, K, nullptr, stream);
}

w8a8_status w8a8_gemm_fp8_f32_ex(const uint8_t* xq, const uint8_t* wq, float* acc, int64_t M, int64_t N, int64_t K,
                                 const w8a8_gemm_config* cfg, w8a8_stream_t stream) {
  return gemm_common(reinterpret_cast<const int8_t*>(xq), reinterpret_cast<const int8_t*>(wq), nullptr, nullptr,
                     nullptr, acc, M, N, K, cfg, GemmOut::kAcc32, reinterpret_cast<cudaStream_t>(stream),
                     /*overlap_prologue=*/false, GemmElem::kE4M3);
}

w8a8_status w8a8_gemm_fp8_f32(const uint8_t* xq, const uint8_t* wq, float* acc, int64_t M, int64_t N, int64_t K,
                              w8a8_stream_t stream) {
  return w8a8_gemm_fp8_f32_ex(xq, wq, acc, M, N, K, nullptr, stream);
}

w8a8_status w8a8_linear_fp8(const void* x, const uint8_t* wq, const float* scale_w, const void* bias, void* out,
                            uint8_t* ws_xq, float* ws_scale_a, int64_t M, int64_t N, int64_t K,
                            w8a8_stream_t stream) {
  w8a8_status st = check_linear_call(x, reinterpret_cast<const int8_t*>(wq), scale_w, bias, out, ws_xq, ws_scale_a,
                                     M, N, K);
  if (st != W8A8_OK || M == 0 || N == 0) return st;
  st = w8a8_quantize_act_fp8(x, M, K, K, ws_xq, K, ws_scale_a, stream);
  if (st != W8A8_OK) return st;
  return gemm_common(reinterpret_cast<const int8_t*>(ws_xq), reinterpret_cast<const int8_t*>(wq), ws_scale_a,
                     scale_w, bias, out, M, N, K, nullptr, GemmOut::kBf16Dequant,
                     reinterpret_cast<cudaStream_t>(stream), /*overlap_prologue=*/true, GemmElem::kE4M3);
}

// ------------------------------------------------- GELU before a linear layer

w8a8_status w8a8_quantize_act_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, int8_t* xq, int64_t ldxq,
                                   float* scale_a, w8a8_stream_t stream) {
  return quantize_common(true, h, M, K, ldh, xq, ldxq, scale_a, reinterpret_cast<cudaStream_t>(stream),
                         /*e4m3=*/false, /*gelu=*/true);
}

w8a8_status w8a8_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, void* g, int64_t ldg, w8a8_stream_t stream) {
  if (M < 0 || M > kMaxMN || K < 8 || K > kMaxMN || K % 8 != 0 || ldh < K || ldg < K) return W8A8_ERR_INVALID_ARG;
  if (M == 0) return W8A8_OK;
  if (h == nullptr || g == nullptr) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(g) || ldh % 8 != 0 || ldg % 8 != 0) return W8A8_ERR_ALIGNMENT;
  DeviceInfo dev;
  w8a8_status st = current_device(&dev);
  if (st != W8A8_OK) return st;
  return from_cuda(launch_gelu(h, M, K, ldh, g, ldg, dev.sms, reinterpret_cast<cudaStream_t>(stream)));
}

w8a8_status w8a8_linear_gelu(const void* h, const int8_t* wq, const float* scale_w, const void* bias, void* out,
                             int8_t* ws_xq, float* ws_scale_a, int64_t M, int64_t N, int64_t K,
                             w8a8_stream_t stream) {
  w8a8_status st = check_linear_call(h, wq, scale_w, bias, out, ws_xq, ws_scale_a, M, N, K);
  if (st != W8A8_OK || M == 0 || N == 0) return st;
  st = w8a8_quantize_act_gelu(h, M, K, K, ws_xq, K, ws_scale_a, stream);
  if (st != W8A8_OK) return st;
  return gemm_common(ws_xq, wq, ws_scale_a, scale_w, bias, out, M, N, K, nullptr, GemmOut::kBf16Dequant,
                     reinterpret_cast<cudaStream_t>(stream), /*overlap_prologue=*/true);
}

int64_t w8a8_linear_sync_words(int64_t M) { return M < 0 ? 0 : linear_sync_words(M); }

w8a8_status w8a8_select_config(int64_t M, int64_t N, int64_t K, w8a8_gemm_config* cfg) {
  if (cfg == nullptr) return W8A8_ERR_INVALID_ARG;
  w8a8_status st = check_gemm_shape(M, N, K);
  if (st != W8A8_OK) return st;
  DeviceInfo dev;
  if ((st = current_device(&dev)) != W8A8_OK) return st;
  *cfg = select(M > 0 ? M : 1, N > 0 ? N : 8, K, dev.sms);
  return W8A8_OK;
}

w8a8_status w8a8_read_device_error(int32_t* code, int32_t clear) {
  if (code == nullptr) return W8A8_ERR_INVALID_ARG;
  int v = 0;
  if (read_device_error(&v, clear != 0) != cudaSuccess) return W8A8_ERR_CUDA;
  *code = v;
  return v != 0 ? W8A8_ERR_TIMEOUT : W8A8_OK;
}

w8a8_status w8a8_set_wait_timeout_ns(int64_t ns) {
  if (ns < 100000) ns = 100000;
  g_timeout_ns.store(ns);
  return W8A8_OK;
}

w8a8_status w8a8_selftest_wait_timeout(int64_t timeout_ns, w8a8_stream_t stream) {
  if (timeout_ns < 100000) return W8A8_ERR_INVALID_ARG;
  DeviceInfo dev;
  w8a8_status st = current_device(&dev);
  if (st != W8A8_OK) return st;
  return from_cuda(launch_selftest_wait(static_cast<uint64_t>(timeout_ns), reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
