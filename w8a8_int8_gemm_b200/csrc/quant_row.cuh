// quant_row.cuh -- one warp quantizes one row (symmetric absmax, int8 or
// OCP E4M3 codes).
//
// Shared by the standalone row quantizers (quant.cu) and the fused linear
// kernel (gemm_sm100.cu), which quantizes activation rows inside the GEMM.
// The rules, and why the int8 product shortcut decides the same codes as
// the IEEE division, are stated at the top of quant.cu.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace w8a8 {
namespace qrow {

// Code format: int8 (scale absmax / 127) or E4M3 (scale absmax / 448).
enum class Code { kInt8, kE4M3 };

// Element-wise step applied to a bf16 row before it is quantized (the
// producer of the linear layer's input, fused): none, or GELU.
enum class Pre { kNone, kGelu };

// Packed binary32 pairs (Blackwell f32x2 arithmetic): each lane of the
// pair is rounded exactly as the scalar operation would round it.
namespace f2 {
__device__ __forceinline__ uint64_t pack(float lo, float hi) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
  return v;
}
__device__ __forceinline__ void unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t splat(float x) { return pack(x, x); }
__device__ __forceinline__ uint64_t fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t neg(uint64_t a) { return a ^ 0x8000000080000000ull; }
}  // namespace f2

// GELU of one bf16 value (bit pattern in the low 16 bits of hb), as the
// library defines it: the tanh form (Hendrycks & Gimpel, "Gaussian Error
// Linear Units"), 0.5 h (1 + tanh(u)) with u = sqrt(2/pi) (h + 0.044715 h^3),
// rounded once to bf16 (nearest, ties to even).  It is evaluated in binary64
// through the equal form h / (1 + exp(-2u)), which does not cancel for
// negative h: every product and sum rounded on its own in the order
// written (no contraction into fused multiply-adds), CUDA's binary64 exp,
// an IEEE division, then one rounding from binary64 to bf16.  The binary64
// value is within far less than 2^-40 (relative) of the exact function, so
// the result is its correctly rounded bf16 value except where that lies
// nearer a rounding boundary than this error.
//
// Outside -11 < h < 4 and away from 0 the function is a closed form, taken
// without the binary64 evaluation (each equal to it for every bf16 input,
// which the exhaustive comparison with the CPU oracle checks):
//   h >= 4:        1 + exp(-2u) < 1 + 2^-15, so the result is h itself;
//   h <= -11:      |gelu(h)| is below half the least bf16 subnormal: -0;
//   |h| <= 2^-20:  gelu(h) = h/2 + 0.399 h^2 + ..., the h^2 term far below
//                  binary64's resolution of h/2, so the result is
//                  bf16_rne(h/2) (h/2 formed exactly in binary32).
// That leaves under 6000 of the 65536 bf16 inputs for the binary64 path.
__device__ __forceinline__ uint32_t gelu_bf16_bits(uint32_t hb) {
  const uint32_t m = hb & 0x7FFFu;
  if (m <= 0x3580u) {  // |h| <= 2^-20 (zeros included)
    return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__uint_as_float(hb << 16), 0.5f)));
  }
  if (m < 0x7F80u) {  // finite
    if (hb < 0x8000u && m >= 0x4080u) return hb;        // h >= 4
    if (hb >= 0x8000u && m >= 0x4130u) return 0x8000u;  // h <= -11
  }
  const double h = static_cast<double>(__uint_as_float(hb << 16));
  const double h3 = __dmul_rn(__dmul_rn(h, h), h);
  const double inner = __dadd_rn(h, __dmul_rn(0.044715, h3));
  const double u = __dmul_rn(0.79788456080286535587989211986876373695, inner);  // sqrt(2/pi)
  const double e = exp(__dmul_rn(-2.0, u));  // +inf for very negative h: h / inf = -0
  return __bfloat16_as_ushort(__double2bfloat16(__ddiv_rn(h, __dadd_rn(1.0, e))));
}

// Eight bf16 -> bf16_rne(GELU) of each (what a GELU kernel would store).
// One out-of-line copy: the row kernels apply it to every vector of a row.
static __device__ __noinline__ uint4 gelu_bf16x8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll 1
  for (int i = 0; i < 4; ++i) o[i] = gelu_bf16_bits(w[i] & 0xFFFFu) | (gelu_bf16_bits(w[i] >> 16) << 16);
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <typename T, Pre P>
__device__ __forceinline__ uint4 pre_vec(const uint4& v) {
  if constexpr (P == Pre::kGelu) {
    static_assert(sizeof(T) == 2, "GELU applies to bf16 activations");
    return gelu_bf16x8(v);
  } else {
    return v;
  }
}

template <Code C>
__device__ __forceinline__ constexpr float code_max() {
  return C == Code::kInt8 ? 127.0f : 448.0f;
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

struct RowScale {
  float s;  // the row's scale, fl32(amax / code_max)
  float r;  // fl32(1 / s)
  bool zero, fast;
};

// fl32(x / s) for a pair of elements without a division, by Markstein's
// correction (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990): with
// r = fl32(1/s) and q0 = fl32(x*r), which is within one ulp of x/s, the
// remainder x - q0*s is exact in one fused multiply-add, and
// q1 = fl32(q0 + (x - q0*s)*r) is the correctly rounded quotient.  Rows take
// this path when s >= 2^-100 (the remainder then never underflows for a
// quotient that decides a code) and r is finite; it was checked to equal
// IEEE division bit for bit for every pair of bf16 values |x| <= amax at
// both code ranges (quotients of magnitude below 2^-12, which give code 0,
// keep their sign and stay below 2^-11), and on 10^9 fp32 elements planted
// at and around the half-integer quotients.
__device__ __forceinline__ uint64_t quotient2(uint64_t x, uint64_t r2, uint64_t neg_s2) {
  const uint64_t q0 = f2::mul(x, r2);
  const uint64_t rem = f2::fma(q0, neg_s2, x);  // x - q0*s, exact
  return f2::fma(rem, r2, q0);
}

// int8 codes of one vector: rne(fl32(x / s)), the quotient from quotient2
// (or IEEE division on the rows that do not qualify).  q = fl32(x/s) + 1.5*2^23
// rounds the quotient to an integer n (ties to even; 1.5*2^23 is even) and
// the low byte of its bit pattern is n's two's-complement int8 code; |x/s|
// <= 127.0001 keeps n inside [-127, 127] without a clamp.
// fp32 rows (weights, quantized once at load time) always divide: the
// shortcut's equality with the division was checked exhaustively on bf16
// inputs only.
template <typename T>
__device__ __forceinline__ void quantize_vec(const uint4& v, const RowScale& rs, int8_t* dst) {
  constexpr int E = Vec<T>::kElems;
  if (sizeof(T) == 2 && rs.fast) {
    float f[E];
    Vec<T>::unpack(v, f);
    const uint64_t r2 = f2::splat(rs.r), neg_s2 = f2::splat(-rs.s), round2 = f2::splat(12582912.0f);
    uint32_t q[E];
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      float m0, m1;
      f2::unpack(f2::add(quotient2(f2::pack(f[i], f[i + 1]), r2, neg_s2), round2), m0, m1);
      q[i] = __float_as_uint(m0);
      q[i + 1] = __float_as_uint(m1);
    }
    store_words<E>(q, dst);
    return;
  }
  quantize_vec_div<T>(v, rs.s, dst);
}

// E4M3 codes of one vector: e4m3_rne(clamp(fl32(x / s), -448, 448)), the
// quotient from quotient2 with x's sign (a zero quotient of a negative x is
// -0, code 0x80) or IEEE division, then one rounding to E4M3 (the clamp is
// explicit although the conversion saturates: the definition clamps).
template <typename T>
__device__ __forceinline__ void quantize_vec_e4m3(const uint4& v, const RowScale& rs, int8_t* dst) {
  constexpr int E = Vec<T>::kElems;
  float f[E];
  Vec<T>::unpack(v, f);
  float d[E];
  if (sizeof(T) == 2 && rs.fast) {  // fp32 rows (weights) divide, as for int8 codes
    const uint64_t r2 = f2::splat(rs.r), neg_s2 = f2::splat(-rs.s);
#pragma unroll
    for (int i = 0; i < E; i += 2) {
      f2::unpack(quotient2(f2::pack(f[i], f[i + 1]), r2, neg_s2), d[i], d[i + 1]);
      d[i] = copysignf(d[i], f[i]);
      d[i + 1] = copysignf(d[i + 1], f[i + 1]);
    }
  } else {
#pragma unroll
    for (int i = 0; i < E; ++i) d[i] = __fdiv_rn(f[i], rs.s);
  }
  uint32_t h[E / 2];
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    h[i] = cvt_e4m3x2(fminf(fmaxf(d[2 * i], -448.0f), 448.0f), fminf(fmaxf(d[2 * i + 1], -448.0f), 448.0f));
  }
  if constexpr (E == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = h[0] | (h[1] << 16);
  }
}

template <Code C = Code::kInt8>
__device__ __forceinline__ RowScale row_scale(float amax) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  RowScale rs;
  rs.s = __fdiv_rn(amax, code_max<C>());
  rs.zero = (rs.s == 0.0f);  // all-zero row (or an fp32 row whose scale underflows): codes 0
  rs.r = rs.zero ? 0.0f : __frcp_rn(rs.s);
  rs.fast = !rs.zero && rs.s >= 0x1p-100f && isfinite(rs.r);
  return rs;
}

// Codes of one vector of a row whose scale is nonzero.
template <typename T, Code C>
__device__ __forceinline__ void encode_vec(const uint4& v, const RowScale& rs, int8_t* dst) {
  if constexpr (C == Code::kInt8) {
    quantize_vec<T>(v, rs, dst);
  } else {
    quantize_vec_e4m3<T>(v, rs, dst);
  }
}

template <int E>
__device__ __forceinline__ void store_zero(int8_t* dst) {
  if constexpr (E == 8) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(0u, 0u);
  } else {
    *reinterpret_cast<uint32_t*>(dst) = 0u;
  }
}

// One warp quantizes row `xr` (nvec 16-byte vectors) into `qr` and returns
// the row's scale in every lane.  VPL > 0: rows of up to 32 * VPL vectors,
// all loads issued at once and the row kept in registers; VPL == 0: any
// length, an absmax pass and a second pass that reads the row again.
template <typename T, int VPL, Code C = Code::kInt8, Pre P = Pre::kNone>
__device__ __forceinline__ float quantize_row(const uint4* __restrict__ xr, int nvec, int8_t* __restrict__ qr,
                                              int lane) {
  constexpr int E = Vec<T>::kElems;
  if constexpr (VPL > 0) {
    uint4 c[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = lane + 32 * i;
      c[i] = v < nvec ? pre_vec<T, P>(__ldg(xr + v)) : make_uint4(0u, 0u, 0u, 0u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) amax = fmaxf(amax, vec_absmax<T>(c[i]));
    const RowScale rs = row_scale<C>(amax);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = lane + 32 * i;
      if (v < nvec) {
        if (rs.zero) {
          store_zero<E>(qr + E * v);
        } else {
          encode_vec<T, C>(c[i], rs, qr + E * v);
        }
      }
    }
    return rs.s;
  } else {
    // pass 1: absmax, eight 16-byte loads per lane in flight
    float amax = 0.0f;
    int v = lane;
    for (; v + 224 < nvec; v += 256) {
      uint4 a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = pre_vec<T, P>(__ldg(xr + v + 32 * i));
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, vec_absmax<T>(a[i]));
    }
    for (; v < nvec; v += 32) amax = fmaxf(amax, vec_absmax<T>(pre_vec<T, P>(__ldg(xr + v))));
    const RowScale rs = row_scale<C>(amax);
    // pass 2: codes
    v = lane;
    for (; v + 96 < nvec; v += 128) {
      uint4 a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = pre_vec<T, P>(__ldg(xr + v + 32 * i));
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (rs.zero) {
          store_zero<E>(qr + E * (v + 32 * i));
        } else {
          encode_vec<T, C>(a[i], rs, qr + E * (v + 32 * i));
        }
      }
    }
    for (; v < nvec; v += 32) {
      if (rs.zero) {
        store_zero<E>(qr + E * v);
      } else {
        encode_vec<T, C>(pre_vec<T, P>(__ldg(xr + v)), rs, qr + E * v);
      }
    }
    return rs.s;
  }
}

// Two rows by one warp, both rows' loads in flight together (rows of up to
// 32 * VPL vectors, kept in registers): twice the memory parallelism of
// quantize_row for a warp that has several rows to do.  Scales are returned
// in s0 / s1 (every lane).
template <typename T, int VPL>
__device__ __forceinline__ void quantize_two_rows(const uint4* __restrict__ x0, const uint4* __restrict__ x1,
                                                  int nvec, int8_t* __restrict__ q0, int8_t* __restrict__ q1,
                                                  int lane, float& s0, float& s1) {
  constexpr int E = Vec<T>::kElems;
  uint4 c0[VPL], c1[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int v = lane + 32 * i;
    c0[i] = v < nvec ? __ldg(x0 + v) : make_uint4(0u, 0u, 0u, 0u);
    c1[i] = v < nvec ? __ldg(x1 + v) : make_uint4(0u, 0u, 0u, 0u);
  }
  float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    a0 = fmaxf(a0, vec_absmax<T>(c0[i]));
    a1 = fmaxf(a1, vec_absmax<T>(c1[i]));
  }
  const RowScale r0 = row_scale(a0);
  const RowScale r1 = row_scale(a1);
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int v = lane + 32 * i;
    if (v < nvec) {
      if (r0.zero) {
        store_zero<E>(q0 + E * v);
      } else {
        quantize_vec<T>(c0[i], r0, q0 + E * v);
      }
      if (r1.zero) {
        store_zero<E>(q1 + E * v);
      } else {
        quantize_vec<T>(c1[i], r1, q1 + E * v);
      }
    }
  }
  s0 = r0.s;
  s1 = r1.s;
}

}  // namespace qrow
}  // namespace w8a8
