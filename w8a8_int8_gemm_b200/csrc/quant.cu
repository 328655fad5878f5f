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
// Layout.  Rows of up to 32 * 16 vectors (K <= 4096 bf16): one warp per
// row, every 16-byte load of the row issued at once and the row kept in
// registers (blocks of 128 threads, so that all rows of a DiT-sized batch are
// resident together: the bytes in flight, not the instruction count, set
// the speed of this kernel).  Longer rows, up to 16 vectors per thread of a
// 256-thread block (K <= 32768 bf16, 16384 fp32): one block per row, the row
// in the block's registers, |x| reduced across its warps through shared
// memory, one pass over HBM.  Longer still: a two-pass register kernel that
// reads the row twice.  |x| is reduced with butterfly shuffles; the codes are
// written packed (8 or 4 bytes per lane per vector).  HBM sees 3 bytes per
// bf16 element (2 in, 1 out): the kernels are bound by HBM bandwidth.
//
// Exactness.  The code q is decided in binary32 exactly as the definition
// says, without one IEEE division per element: the quotient fl32(x/scale) is
// formed from the row's reciprocal r = fl32(1/scale) by Markstein's
// correction (q0 = fl32(x*r); the remainder x - q0*scale is exact in one
// fused multiply-add; fl32(q0 + remainder*r) is the correctly rounded
// quotient), three packed f32x2 operations per element pair, and rounded to
// an integer by adding 1.5*2^23 (ties to even), whose bit pattern's low byte
// is the int8 code.  An earlier scheme rounded the bare product x*r and
// redid near-half-integer elements by division; bf16 rows defeat it: with
// both x and amax bf16, 127*x/amax is an exact half-integer for about 0.3%
// of the elements of N(0,1) rows, one warp step in four, and the redo cost
// a third of the kernel's time.  The correction was checked against IEEE
// division for every pair of bf16 values |x| <= amax and on 10^9 planted
// fp32 elements.  Rows whose scale is below 2^-100 (where the remainder can
// underflow), or whose reciprocal is not finite, take IEEE division
// (__fdiv_rn) for every element.
//
// FP8 variant (OCP E4M3 codes; B200's native FP8 path, the comparison
// baseline of the same paper): the same scheme with 448, the largest finite
// E4M3 value, in place of 127:
//   scale[r] = fl32(max_k |x[r,k]| / 448)
//   q[r,k]   = e4m3_rne(clamp(fl32(x[r,k] / scale[r]), -448, 448)), 0 if scale[r] == 0
// Each element's quotient is the same correctly rounded fl32(x/scale) (with
// x's sign, so that a negative quotient that rounds to zero keeps it: code
// 0x80), then one hardware conversion (cvt.rn.satfinite.e4m3x2.f32: round to
// nearest even, saturating), which is the definition term by term.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "internal.h"
#include "quant_row.cuh"
#include "sm100_ptx.cuh"

namespace w8a8 {
namespace {

// Rows of up to 32 * VPL vectors: the whole row in registers.  Seven
// 128-thread blocks per SM (at most 72 registers) keep 28 rows per SM in
// flight, so a 4096-token batch is resident in one wave on 148 SMs.
template <typename T, int VPL, qrow::Code C, qrow::Pre P>
__global__ void __launch_bounds__(128, (VPL <= 12 ? 7 : 5))
    quantize_rows_regs_kernel(const T* __restrict__ x, int64_t M, int64_t K, int64_t ldx, int8_t* __restrict__ q,
                              int64_t ldq, float* __restrict__ scale) {
  // Launched as a programmatic dependent of the kernel before it (whose
  // output may be x): wait for that kernel first, then let this kernel's own
  // dependent (the GEMM, which reads its weight operand before it waits) be
  // scheduled.
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;
  const float s = qrow::quantize_row<T, VPL, C, P>(reinterpret_cast<const uint4*>(x + row * ldx),
                                                static_cast<int>(K / qrow::Vec<T>::kElems), q + row * ldq, lane);
  if (lane == 0) scale[row] = s;
}

// Any row length: absmax pass, then a second pass that reads the row again.
template <typename T, qrow::Code C, qrow::Pre P>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ x, int64_t M, int64_t K,
                                                            int64_t ldx, int8_t* __restrict__ q, int64_t ldq,
                                                            float* __restrict__ scale) {
  // Launched as a programmatic dependent of the kernel before it (whose
  // output may be x): wait for that kernel first, then let this kernel's own
  // dependent (the GEMM, which reads its weight operand before it waits) be
  // scheduled.
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= M) return;
  const float s = qrow::quantize_row<T, 0, C, P>(reinterpret_cast<const uint4*>(x + row * ldx),
                                              static_cast<int>(K / qrow::Vec<T>::kElems), q + row * ldq, lane);
  if (lane == 0) scale[row] = s;
}

// One 256-thread block per row of up to 256 * VPL vectors: the row in the
// block's registers, |x| reduced over the block through shared memory.
template <typename T, int VPL, qrow::Code C, qrow::Pre P>
__global__ void __launch_bounds__(256) quantize_rows_block_kernel(const T* __restrict__ x, int64_t K, int64_t ldx,
                                                                  int8_t* __restrict__ q, int64_t ldq,
                                                                  float* __restrict__ scale) {
  // Launched as a programmatic dependent of the kernel before it (whose
  // output may be x): wait for that kernel first, then let this kernel's own
  // dependent (the GEMM, which reads its weight operand before it waits) be
  // scheduled.
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  constexpr int E = qrow::Vec<T>::kElems;
  constexpr int kWarps = 8;
  __shared__ float wmax[kWarps];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int64_t row = blockIdx.x;
  const int nvec = static_cast<int>(K / E);
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * ldx);
  uint4 c[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int v = tid + 256 * i;
    c[i] = v < nvec ? qrow::pre_vec<T, P>(__ldg(xr + v)) : make_uint4(0u, 0u, 0u, 0u);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) amax = fmaxf(amax, qrow::vec_absmax<T>(c[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) wmax[tid >> 5] = amax;
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) amax = fmaxf(amax, wmax[w]);
  const qrow::RowScale rs = qrow::row_scale<C>(amax);  // every lane holds the row's max
  int8_t* qr = q + row * ldq;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int v = tid + 256 * i;
    if (v < nvec) {
      if (rs.zero) {
        qrow::store_zero<E>(qr + E * v);
      } else {
        qrow::encode_vec<T, C>(c[i], rs, qr + E * v);
      }
    }
  }
  if (tid == 0) scale[row] = rs.s;
}

// Launch as a programmatic dependent of the previous kernel in the stream:
// the launch overlaps that kernel's tail, and the kernel's first act is to
// wait for it (griddepcontrol.wait).
template <typename... Params, typename... Args>
void launch_after_prev(void (*kernel)(Params...), unsigned blocks, unsigned threads, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(blocks);
  lc.blockDim = dim3(threads);
  lc.dynamicSmemBytes = 0;
  lc.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  cudaLaunchKernelEx(&lc, kernel, static_cast<Params>(args)...);
}

template <typename T, int VPL, qrow::Code C, qrow::Pre P>
void launch_regs(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* scale,
                 cudaStream_t stream) {
  const int threads = 128;
  const int64_t blocks = (M + (threads / 32) - 1) / (threads / 32);
  launch_after_prev(quantize_rows_regs_kernel<T, VPL, C, P>, static_cast<unsigned>(blocks), threads, stream, x, M,
                    K, ldx, q, ldq, scale);
}

template <typename T, int VPL, qrow::Code C, qrow::Pre P>
void launch_block(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* scale,
                  cudaStream_t stream) {
  launch_after_prev(quantize_rows_block_kernel<T, VPL, C, P>, static_cast<unsigned>(M), 256, stream, x, K, ldx,
                    q, ldq, scale);
}

template <typename T, qrow::Code C, qrow::Pre P = qrow::Pre::kNone>
cudaError_t launch_quantize(const T* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq, float* scale,
                            cudaStream_t stream) {
  const int64_t nvec = K / qrow::Vec<T>::kElems;
  const int64_t per_lane = (nvec + 31) / 32;
  if (per_lane <= 4) {
    launch_regs<T, 4, C, P>(x, M, K, ldx, q, ldq, scale, stream);
    return cudaGetLastError();
  }
  if (per_lane <= 8) {
    launch_regs<T, 8, C, P>(x, M, K, ldx, q, ldq, scale, stream);
    return cudaGetLastError();
  }
  if (per_lane <= 12) {
    launch_regs<T, 12, C, P>(x, M, K, ldx, q, ldq, scale, stream);
    return cudaGetLastError();
  }
  if (per_lane <= 16) {
    launch_regs<T, 16, C, P>(x, M, K, ldx, q, ldq, scale, stream);
    return cudaGetLastError();
  }
  const int64_t per_thread = (nvec + 255) / 256;  // one 256-thread block per row
  if (per_thread <= 8) {
    launch_block<T, 8, C, P>(x, M, K, ldx, q, ldq, scale, stream);
  } else if (per_thread <= 12) {
    launch_block<T, 12, C, P>(x, M, K, ldx, q, ldq, scale, stream);
  } else if (per_thread <= 16) {
    launch_block<T, 16, C, P>(x, M, K, ldx, q, ldq, scale, stream);
  } else {
    const int threads = 256;
    const int64_t blocks = (M + (threads / 32) - 1) / (threads / 32);
    launch_after_prev(quantize_rows_kernel<T, C, P>, static_cast<unsigned>(blocks), threads, stream, x, M, K, ldx,
                      q, ldq, scale);
  }
  return cudaGetLastError();
}

// bf16 GELU of rows h [M, K] into g: 16-byte vectors, grid-stride.
__global__ void __launch_bounds__(256) gelu_rows_kernel(const __nv_bfloat16* __restrict__ h, int64_t M,
                                                        int64_t K, int64_t ldh, __nv_bfloat16* __restrict__ g,
                                                        int64_t ldg) {
  const int64_t vpr = K / 8;  // vectors per row
  const int64_t total = M * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vpr;
    const int64_t v = i - r * vpr;
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(h + r * ldh) + v);
    reinterpret_cast<uint4*>(g + r * ldg)[v] = qrow::gelu_bf16x8(x);
  }
}

}  // namespace

cudaError_t launch_quantize_act_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, int8_t* q, int64_t ldq,
                                     float* scale, cudaStream_t stream) {
  return launch_quantize<__nv_bfloat16, qrow::Code::kInt8, qrow::Pre::kGelu>(
      static_cast<const __nv_bfloat16*>(h), M, K, ldh, q, ldq, scale, stream);
}

cudaError_t launch_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, void* g, int64_t ldg, int sms,
                        cudaStream_t stream) {
  const int64_t total = M * (K / 8);
  const int64_t max_blocks = static_cast<int64_t>(sms > 0 ? sms : 148) * 8;
  const int64_t blocks = std::min<int64_t>(max_blocks, (total + 255) / 256);
  gelu_rows_kernel<<<static_cast<unsigned>(blocks > 0 ? blocks : 1), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(h), M, K, ldh, static_cast<__nv_bfloat16*>(g), ldg);
  return cudaGetLastError();
}

cudaError_t launch_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq,
                                float* scale, cudaStream_t stream) {
  return launch_quantize<__nv_bfloat16, qrow::Code::kInt8>(static_cast<const __nv_bfloat16*>(x), M, K, ldx, q, ldq,
                                                           scale, stream);
}

cudaError_t launch_quantize_weight(const float* w, int64_t N, int64_t K, int64_t ldw, int8_t* q, int64_t ldq,
                                   float* scale, cudaStream_t stream) {
  return launch_quantize<float, qrow::Code::kInt8>(w, N, K, ldw, q, ldq, scale, stream);
}

cudaError_t launch_quantize_act_e4m3(const void* x, int64_t M, int64_t K, int64_t ldx, uint8_t* q, int64_t ldq,
                                     float* scale, cudaStream_t stream) {
  return launch_quantize<__nv_bfloat16, qrow::Code::kE4M3>(static_cast<const __nv_bfloat16*>(x), M, K, ldx,
                                                           reinterpret_cast<int8_t*>(q), ldq, scale, stream);
}

cudaError_t launch_quantize_weight_e4m3(const float* w, int64_t N, int64_t K, int64_t ldw, uint8_t* q, int64_t ldq,
                                        float* scale, cudaStream_t stream) {
  return launch_quantize<float, qrow::Code::kE4M3>(w, N, K, ldw, reinterpret_cast<int8_t*>(q), ldq, scale, 
                                                   stream);
}

}  // namespace w8a8
