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
// Layout: one warp per row, all rows in flight at once (about 40 registers
// per thread, 48 warps per SM).  Pass 1 reads the row as 16-byte vectors
// (8 bf16 or 4 fp32), four per lane in flight, and reduces |x| with a
// butterfly shuffle; pass 2 reads the row again -- from L1, where pass 1
// left it -- and writes the packed int8 codes (8 or 4 bytes per lane per
// vector).  HBM sees 3 bytes per bf16 element (2 in, 1 out): the kernel is
// bound by HBM bandwidth.
//
// Exactness.  The code q is decided in binary32 exactly as the definition
// says.  Instead of one IEEE division per element, the kernel multiplies by
// the row's reciprocal r = fl32(1/scale) and only divides where that could
// change the rounded integer: with |x/scale| <= 127 (1 + 2^-23), the product
// x*r differs from the exact quotient by less than 2^-16 and fl32(x/scale)
// differs from it by at most 2^-18, so both round to the same integer unless
// x*r lies within 2^-15 of a half-integer; a vector holding such an element
// is redone with IEEE division (__fdiv_rn) in an out-of-line path.  Rows
// whose scale is not a normal number, or whose reciprocal is not finite,
// take the division for every element.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"

namespace w8a8 {
namespace {

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

__device__ __forceinline__ int clamp127(int q) { return max(-127, min(127, q)); }

template <int E>
__device__ __forceinline__ uint32_t pack4(const int (&q)[E], int w) {
  return (static_cast<uint32_t>(q[4 * w]) & 0xFFu) | ((static_cast<uint32_t>(q[4 * w + 1]) & 0xFFu) << 8) |
         ((static_cast<uint32_t>(q[4 * w + 2]) & 0xFFu) << 16) | (static_cast<uint32_t>(q[4 * w + 3]) << 24);
}

template <int E>
__device__ __forceinline__ void store_codes(const int (&q)[E], int8_t* dst) {
  if constexpr (E == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack4<E>(q, 0), pack4<E>(q, 1));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack4<E>(q, 0);
  }
}

// The exact path: every element as rne(fl32(x / s)) clamped to +-127.
template <typename T>
__device__ __noinline__ void quantize_vec_div(uint4 v, float s, int8_t* dst) {
  constexpr int E = Vec<T>::kElems;
  float f[E];
  Vec<T>::unpack(v, f);
  int q[E];
#pragma unroll
  for (int i = 0; i < E; ++i) q[i] = clamp127(__float2int_rn(__fdiv_rn(f[i], s)));
  store_codes<E>(q, dst);
}

// The product path with the tie check described in the file header.
template <typename T>
__device__ __forceinline__ void quantize_vec(const uint4& v, float s, float r, bool fast, int8_t* dst) {
  constexpr int E = Vec<T>::kElems;
  if (!fast) {
    quantize_vec_div<T>(v, s, dst);
    return;
  }
  float f[E];
  Vec<T>::unpack(v, f);
  int q[E];
  bool near_tie = false;
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const float t = __fmul_rn(f[i], r);
    const float n = rintf(t);
    near_tie |= fabsf(t - n) >= 0.499969482421875f;  // 0.5 - 2^-15
    q[i] = clamp127(__float2int_rn(n));
  }
  if (near_tie) {
    quantize_vec_div<T>(v, s, dst);
    return;
  }
  store_codes<E>(q, dst);
}

template <typename T>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ x, int64_t M, int64_t K,
                                                            int64_t ldx, int8_t* __restrict__ q, int64_t ldq,
                                                            float* __restrict__ scale) {
  constexpr int E = Vec<T>::kElems;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;

  const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
  int8_t* qr = q + row * ldq;
  const int nvec = static_cast<int>(K / E);

  // pass 1: absmax, four 16-byte loads per lane in flight
  float amax = 0.0f;
  int v = lane;
  for (; v + 96 < nvec; v += 128) {
    const uint4 a0 = __ldg(xr + v), a1 = __ldg(xr + v + 32), a2 = __ldg(xr + v + 64), a3 = __ldg(xr + v + 96);
    amax = fmaxf(amax, fmaxf(fmaxf(vec_absmax<T>(a0), vec_absmax<T>(a1)),
                             fmaxf(vec_absmax<T>(a2), vec_absmax<T>(a3))));
  }
  for (; v < nvec; v += 32) amax = fmaxf(amax, vec_absmax<T>(__ldg(xr + v)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));

  const float s = __fdiv_rn(amax, 127.0f);
  if (lane == 0) scale[row] = s;
  if (s == 0.0f) {  // all-zero row (or an fp32 row whose scale underflows): all codes 0
    for (v = lane; v < nvec; v += 32) {
      if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(qr + E * v) = make_uint2(0u, 0u);
      } else {
        *reinterpret_cast<uint32_t*>(qr + E * v) = 0u;
      }
    }
    return;
  }
  const float r = __frcp_rn(s);
  const bool fast = s >= 1.17549435e-38f && isfinite(r);

  // pass 2: codes (the row is read again, from L1)
  v = lane;
  for (; v + 32 < nvec; v += 64) {
    const uint4 a0 = __ldg(xr + v), a1 = __ldg(xr + v + 32);
    quantize_vec<T>(a0, s, r, fast, qr + E * v);
    quantize_vec<T>(a1, s, r, fast, qr + E * (v + 32));
  }
  for (; v < nvec; v += 32) quantize_vec<T>(__ldg(xr + v), s, r, fast, qr + E * v);
}

template <typename T>
cudaError_t launch_quantize(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* scale,
                            cudaStream_t stream) {
  const int threads = 256;
  const int64_t blocks = (M + (threads / 32) - 1) / (threads / 32);
  quantize_rows_kernel<T><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
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
