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
// Layout: one warp per row.  For rows of up to 32*16 vectors the warp
// issues every 16-byte load of the row at once and keeps the row in
// registers (blocks of 128 threads, so that all rows of a DiT-sized batch are
// resident together); longer rows take two passes, the second re-reading the
// row from L1/L2.  |x| is reduced with a butterfly shuffle; the int8 codes
// are written packed (8 or 4 bytes per lane per vector).  HBM sees 3 bytes
// per bf16 element (2 in, 1 out): the kernel is bound by HBM bandwidth.
//
// Exactness.  The code q is decided in binary32 exactly as the definition
// says.  Instead of one IEEE division per element, the kernel multiplies by
// the row's reciprocal r = fl32(1/scale) and only divides where that could
// change the rounded integer: with |x/scale| <= 127 (1 + 2^-23), the product
// t = x*r differs from the exact quotient by less than 2^-16 and
// fl32(x/scale) differs from it by at most 2^-18, so both round to the same
// integer unless t lies within 2^-15 of a half-integer; a vector holding
// such an element is redone with IEEE division (__fdiv_rn) in an
// out-of-line path.  On the product path t is rounded to an integer by
// adding 1.5 * 2^23 (binary32 addition rounds to nearest even); the low byte
// of the sum's bit pattern is then the two's-complement int8 code, and
// |t| <= 127.0001 keeps it inside [-127, 127] without a clamp.  Rows whose
// scale is not a normal number, or whose reciprocal is not finite, take the
// division for every element.
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

// max |x| over one 16-byte vector, as a float.
template <typename T>
__device__ __forceinline__ float vec_absmax(const uint4& v);

template <>
__device__ __forceinline__ float vec_absmax<__nv_bfloat16>(const uint4& v) {
  // |x| of bf16 pairs by clearing the sign bits, then packed bf16 maxima.
  const uint32_t w[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
  __nv_bfloat162 m01 = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[0]),
                               *reinterpret_cast<const __nv_bfloat162*>(&w[1]));
  __nv_bfloat162 m23 = __hmax2(*reinterpret_cast<const __nv_bfloat162*>(&w[2]),
                               *reinterpret_cast<const __nv_bfloat162*>(&w[3]));
  const __nv_bfloat162 m = __hmax2(m01, m23);
  const uint32_t mb = *reinterpret_cast<const uint32_t*>(&m);
  return fmaxf(__uint_as_float(mb << 16), __uint_as_float(mb & 0xFFFF0000u));
}

template <>
__device__ __forceinline__ float vec_absmax<float>(const uint4& v) {
  return fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
               fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
}

__device__ __forceinline__ int clamp127(int q) { return max(-127, min(127, q)); }

// Low bytes of four 32-bit words, packed into one word (word 0 lowest).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

template <int E>
__device__ __forceinline__ void store_words(const uint32_t (&w)[E], int8_t* dst) {
  if constexpr (E == 8) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack_low_bytes(w[0], w[1], w[2], w[3]), pack_low_bytes(w[4], w[5], w[6], w[7]));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_low_bytes(w[0], w[1], w[2], w[3]);
  }
}

// The exact path: every element as rne(fl32(x / s)) clamped to +-127.
template <typename T>
__device__ __noinline__ void quantize_vec_div(uint4 v, float s, int8_t* dst) {
  constexpr int E = Vec<T>::kElems;
  float f[E];
  Vec<T>::unpack(v, f);
  uint32_t q[E];
#pragma unroll
  for (int i = 0; i < E; ++i) q[i] = static_cast<uint32_t>(clamp127(__float2int_rn(__fdiv_rn(f[i], s))));
  store_words<E>(q, dst);
}

// The product path with the tie check described in the file header.
template <typename T>
__device__ __forceinline__ void quantize_vec(const uint4& v, float s, float r, bool fast, int8_t* dst) {
  constexpr int E = Vec<T>::kElems;
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  if (fast) {
    float f[E];
    Vec<T>::unpack(v, f);
    uint32_t q[E];
    bool near_tie = false;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float t = __fmul_rn(f[i], r);
      const float m = __fadd_rn(t, kRound);          // rne(t) + 1.5 * 2^23, exactly
      const float n = __fsub_rn(m, kRound);          // rne(t)
      near_tie |= fabsf(__fsub_rn(t, n)) >= 0.499969482421875f;  // 0.5 - 2^-15
      q[i] = __float_as_uint(m);                     // low byte = int8 code
    }
    if (!near_tie) {
      store_words<E>(q, dst);
      return;
    }
  }
  quantize_vec_div<T>(v, s, dst);
}

struct RowScale {
  float s, r;
  bool zero, fast;
};

__device__ __forceinline__ RowScale row_scale(float amax) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  RowScale rs;
  rs.s = __fdiv_rn(amax, 127.0f);
  rs.zero = (rs.s == 0.0f);  // all-zero row (or an fp32 row whose scale underflows): codes 0
  rs.r = rs.zero ? 0.0f : __frcp_rn(rs.s);
  rs.fast = !rs.zero && rs.s >= 1.17549435e-38f && isfinite(rs.r);
  return rs;
}

template <int E>
__device__ __forceinline__ void store_zero(int8_t* dst) {
  if constexpr (E == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(0u, 0u);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = 0u;
  }
}

// Rows of up to 32 * VPL vectors: the whole row in registers.  Seven
// 128-thread blocks per SM (at most 72 registers) keep 28 rows per SM in
// flight, so a 4096-token batch is resident in one wave on 148 SMs.
template <typename T, int VPL>
__global__ void __launch_bounds__(128, (VPL <= 12 ? 7 : 5)) quantize_rows_regs_kernel(const T* __restrict__ x, int64_t M, int64_t K,
                                                                 int64_t ldx, int8_t* __restrict__ q, int64_t ldq,
                                                                 float* __restrict__ scale) {
  constexpr int E = Vec<T>::kElems;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
  int8_t* qr = q + row * ldq;
  const int nvec = static_cast<int>(K / E);

  uint4 c[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int v = lane + 32 * i;
    c[i] = v < nvec ? __ldg(xr + v) : make_uint4(0u, 0u, 0u, 0u);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) amax = fmaxf(amax, vec_absmax<T>(c[i]));
  const RowScale rs = row_scale(amax);
  if (lane == 0) scale[row] = rs.s;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int v = lane + 32 * i;
    if (v < nvec) {
      if (rs.zero) {
        store_zero<E>(qr + E * v);
      } else {
        quantize_vec<T>(c[i], rs.s, rs.r, rs.fast, qr + E * v);
      }
    }
  }
}

// Any row length: absmax pass, then a second pass that reads the row again.
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

  // pass 1: absmax, eight 16-byte loads per lane in flight
  float amax = 0.0f;
  int v = lane;
  for (; v + 224 < nvec; v += 256) {
    uint4 a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = __ldg(xr + v + 32 * i);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, vec_absmax<T>(a[i]));
  }
  for (; v < nvec; v += 32) amax = fmaxf(amax, vec_absmax<T>(__ldg(xr + v)));
  const RowScale rs = row_scale(amax);
  if (lane == 0) scale[row] = rs.s;

  // pass 2: codes
  v = lane;
  for (; v + 96 < nvec; v += 128) {
    uint4 a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = __ldg(xr + v + 32 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (rs.zero) {
        store_zero<E>(qr + E * (v + 32 * i));
      } else {
        quantize_vec<T>(a[i], rs.s, rs.r, rs.fast, qr + E * (v + 32 * i));
      }
    }
  }
  for (; v < nvec; v += 32) {
    if (rs.zero) {
      store_zero<E>(qr + E * v);
    } else {
      quantize_vec<T>(__ldg(xr + v), rs.s, rs.r, rs.fast, qr + E * v);
    }
  }
}

template <typename T, int VPL>
void launch_regs(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* scale,
                 cudaStream_t stream) {
  const int threads = 128;
  const int64_t blocks = (M + (threads / 32) - 1) / (threads / 32);
  quantize_rows_regs_kernel<T, VPL>
      <<<static_cast<unsigned>(blocks), threads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
}

template <typename T>
cudaError_t launch_quantize(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* scale,
                            cudaStream_t stream) {
  const int64_t per_lane = (K / Vec<T>::kElems + 31) / 32;
  if (per_lane <= 4) {
    launch_regs<T, 4>(x, M, K, ldx, q, ldq, scale, stream);
  } else if (per_lane <= 8) {
    launch_regs<T, 8>(x, M, K, ldx, q, ldq, scale, stream);
  } else if (per_lane <= 12) {
    launch_regs<T, 12>(x, M, K, ldx, q, ldq, scale, stream);
  } else if (per_lane <= 16) {
    launch_regs<T, 16>(x, M, K, ldx, q, ldq, scale, stream);
  } else {
    const int threads = 256;
    const int64_t blocks = (M + (threads / 32) - 1) / (threads / 32);
    quantize_rows_kernel<T><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(x, M, K, ldx, q, ldq, scale);
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
