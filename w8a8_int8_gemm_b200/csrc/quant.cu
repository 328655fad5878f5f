// quant.cu -- symmetric absmax row quantizer (per-token activations, bf16;
// per-output-channel weights, fp32).
//
// Paper: "Realizing Native INT8 Compute for Diffusion Transformers on
// Consumer GPUs" (arXiv 2606.14598), abstract -- W8A8 post-training
// quantization with per-token (activations) and per-channel (weights)
// scales.  For each row r:
//   scale[r] = fl32(max_k |x[r,k]| / 127)
//   q[r,k]   = clamp(rne(fl32(x[r,k] / scale[r])), -127, 127), 0 if scale[r] == 0
//
// Layout: one warp per row.  Lanes read 16-byte vectors (8 bf16 or 4 fp32),
// keep up to VPL of them in registers, reduce |x| with a butterfly shuffle,
// then write the packed int8 codes (8 or 4 bytes per lane per vector).  The
// kernel moves 3 bytes per bf16 element (2 in, 1 out) and is bound by HBM
// bandwidth.
//
// Exactness.  The code q is decided in binary32 exactly as the definition
// says.  Instead of one IEEE division per element, the kernel multiplies by
// the row's reciprocal r = fl32(1/scale) and only divides where that could
// change the rounded integer: with |x/scale| <= 127 (1 + 2^-23), the product
// x*r differs from the exact quotient by less than 127 * 2^-22.9 and
// fl32(x/scale) differs from it by at most 127 * 2^-24, so the two round to
// the same integer unless x*r lies within 2^-15 of a half-integer; there the
// kernel computes the IEEE quotient (__fdiv_rn) and rounds that.  Rows whose
// reciprocal is not a finite normal number (scale below 2^-126) take the
// division for every element.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace w8a8 {
namespace {

__device__ __forceinline__ uint4 ld_stream_16B(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename T>
struct Vec;

// 8 bf16 per 16 bytes.
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int kElems = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

// 4 fp32 per 16 bytes.
template <>
struct Vec<float> {
  static constexpr int kElems = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
};

template <typename T>
__device__ __forceinline__ float vec_absmax(const uint4& v) {
  float f[Vec<T>::kElems];
  Vec<T>::unpack(v, f);
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < Vec<T>::kElems; ++i) m = fmaxf(m, fabsf(f[i]));
  return m;
}

// One code, decided as rne(fl32(x / s)) clamped to +-127 (see file header).
__device__ __forceinline__ int quantize_one(float x, float s, float r, bool fast) {
  float t;
  if (fast) {
    t = __fmul_rn(x, r);
    const float d = fabsf(t - floorf(t) - 0.5f);
    if (d <= 3.0517578125e-05f) t = __fdiv_rn(x, s);  // within 2^-15 of a tie
  } else {
    t = __fdiv_rn(x, s);
  }
  int q = __float2int_rn(t);
  q = q > 127 ? 127 : q;
  q = q < -127 ? -127 : q;
  return q;
}

template <typename T>
__device__ __forceinline__ void quantize_vec(const uint4& v, float s, float r, bool fast, bool zero,
                                             int8_t* dst) {
  constexpr int E = Vec<T>::kElems;
  float f[E];
  Vec<T>::unpack(v, f);
  uint32_t packed[E / 4];
#pragma unroll
  for (int w = 0; w < E / 4; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = zero ? 0 : quantize_one(f[4 * w + i], s, r, fast);
      word |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * i);
    }
    packed[w] = word;
  }
  if constexpr (E == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = packed[0];
  }
}

template <typename T, int VPL>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ x, int64_t M, int64_t K,
                                                            int64_t ldx, int8_t* __restrict__ q, int64_t ldq,
                                                            float* __restrict__ scale) {
  constexpr int E = Vec<T>::kElems;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;

  const char* xr = reinterpret_cast<const char*>(x + row * ldx);
  int8_t* qr = q + row * ldq;
  const int64_t nvec = K / E;

  uint4 cache[VPL];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int64_t v = lane + 32 * i;
    if (v < nvec) {
      cache[i] = ld_stream_16B(xr + 16 * v);
      amax = fmaxf(amax, vec_absmax<T>(cache[i]));
    }
  }
  for (int64_t v = lane + 32 * VPL; v < nvec; v += 32) {
    amax = fmaxf(amax, vec_absmax<T>(__ldg(reinterpret_cast<const uint4*>(xr) + v)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));

  const float s = __fdiv_rn(amax, 127.0f);
  const bool zero = (s == 0.0f);
  const float r = zero ? 0.0f : __frcp_rn(s);
  // The product shortcut needs a normal scale and a finite reciprocal.
  const bool fast = !zero && s >= 1.17549435e-38f && isfinite(r);
  if (lane == 0) scale[row] = s;

#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int64_t v = lane + 32 * i;
    if (v < nvec) quantize_vec<T>(cache[i], s, r, fast, zero, qr + E * v);
  }
  for (int64_t v = lane + 32 * VPL; v < nvec; v += 32) {
    quantize_vec<T>(__ldg(reinterpret_cast<const uint4*>(xr) + v), s, r, fast, zero, qr + E * v);
  }
}

template <typename T>
cudaError_t launch_quantize(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* scale,
                            cudaStream_t stream) {
  constexpr int E = Vec<T>::kElems;
  const int64_t per_lane = (K / E + 31) / 32;
  const int threads = 256;
  const int64_t blocks = (M + (threads / 32) - 1) / (threads / 32);
  const dim3 grid(static_cast<unsigned>(blocks));
  if (per_lane <= 4) {
    quantize_rows_kernel<T, 4><<<grid, threads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
  } else if (per_lane <= 8) {
    quantize_rows_kernel<T, 8><<<grid, threads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
  } else if (per_lane <= 12) {
    quantize_rows_kernel<T, 12><<<grid, threads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
  } else {
    quantize_rows_kernel<T, 16><<<grid, threads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq,
                                float* scale, cudaStream_t stream) {
  return launch_quantize<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), M, K, ldx, q, ldq, scale, stream);
}

cudaError_t launch_quantize_weight(const float* w, int64_t N, int64_t K, int64_t ldw, int8_t* q, int64_t ldq,
                                   float* scale, cudaStream_t stream) {
  return launch_quantize<float>(w, N, K, ldw, q, ldq, scale, stream);
}

}  // namespace w8a8
