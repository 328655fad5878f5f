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
// reads the row twice.  GELU before the quantizer (and the bf16 GELU alone)
// goes through a table of GELU over all 65536 bf16 inputs in shared memory
// for rows of up to 16384 (see the table kernels below).  |x| is reduced with butterfly shuffles; the codes are
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
// (__fdiv_rn) for every element, and so do all fp32 rows (weights): they are
// quantized once at load time, where the division costs nothing that
// matters, and the shortcut's check covers bf16 inputs exhaustively only.
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
#include <mutex>

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

// ---------------------------------------------------------------------------
// GELU fused into the per-token quantizer, by table.  GELU's input is bf16,
// so it takes one of 65536 values, and what the quantizer consumes,
// bf16_rne(GELU(h)), is a function of the 16 input bits alone.  The kernel
// evaluates that function for every bit pattern with the binary64
// arithmetic the long-row kernels apply element by element (gelu_bf16x8),
// into a 128 KB table in shared memory, and then replaces GELU per element
// (a binary64 exp and division) by one shared-memory load.  The table is built by a
// cluster of CTAs: each computes 65536 / cluster entries and stores them into
// the shared memory of every CTA of the cluster (distributed shared memory),
// then the cluster synchronises once.  This happens before the kernel waits
// for its producer, so it overlaps the tail of the kernel that writes h.
//
// Rows: a persistent grid of one CTA per SM (the table leaves room for no
// second); each 256-thread group of the CTA quantizes one row at a time,
// VPL 16-byte vectors per thread held in registers, |GELU(h)| reduced over
// the group's eight warps through shared memory and a named barrier.  While
// a group looks its row up and encodes it, the loads of its next row are
// already in flight (a second register copy of the row): a group that only
// waited for its row and then worked on it left HBM and the shared-memory
// pipe each less than half busy.
constexpr int kLutMaxGroups = 4;
constexpr int kLutThreads = 1024;  // the standalone GELU kernel
constexpr int kLutTableBytes = 65536 * 2;
constexpr int kLutSmemBytes = kLutTableBytes + 2 * kLutMaxGroups * 8 * 4;

__device__ __forceinline__ void st_cluster_v4(uint32_t cluster_addr, const uint4& v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

// Two bf16 of a word -> their table entries, packed the same way.  The pack
// is an opaque prmt so that the row stays four registers per vector (seen
// through, the compiler keeps every entry in a register of its own and the
// row no longer fits the 64 registers a thread has at 1024 threads).
__device__ __forceinline__ uint32_t lut_pair(const uint16_t* table, uint32_t w) {
  const uint32_t lo = table[w & 0xFFFFu];
  const uint32_t hi = table[w >> 16];
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, 0x5410;" : "=r"(r) : "r"(lo), "r"(hi));
  return r;
}

__device__ __forceinline__ void st_cluster_u16(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u16 [%0], %1;" ::"r"(cluster_addr), "h"(static_cast<unsigned short>(v))
               : "memory");
}

// The bf16 inputs whose GELU has no closed form and takes the binary64
// evaluation (see qrow::gelu_bf16_bits): 0x3580..0x407F (2^-20 < h < 4),
// 0xB580..0xC12F (-11 < h < -2^-20), and the infinities and NaNs
// 0x7F80..0x7FFF, 0xFF80..0xFFFF -- 6064 patterns, all runs of 8 aligned.
constexpr int kGeluSlowPatterns = (0x4080 - 0x3580) + (0xC130 - 0xB580) + 128 + 128;

__device__ __forceinline__ uint32_t gelu_slow_pattern(int f) {
  if (f < 0x4080 - 0x3580) return 0x3580u + static_cast<uint32_t>(f);
  f -= 0x4080 - 0x3580;
  if (f < 0xC130 - 0xB580) return 0xB580u + static_cast<uint32_t>(f);
  f -= 0xC130 - 0xB580;
  return (f < 128 ? 0x7F80u : 0xFF80u - 128u) + static_cast<uint32_t>(f);
}

__device__ __forceinline__ bool gelu_slow_run(uint32_t u) {
  return (u >= 0x3580u && u < 0x4080u) || (u >= 0xB580u && u < 0xC130u) || (u >= 0x7F80u && u < 0x8000u) ||
         u >= 0xFF80u;
}

// The table of bf16_rne(GELU(h)) for every bf16 bit pattern h, built by a
// cluster and stored into the shared memory of every CTA of it.  The 59472
// entries with a closed form go first, this CTA taking 65536 / cluster
// consecutive patterns as 16-byte runs of 8 (one call of gelu_bf16x8 each);
// the 6064 binary64 evaluations are then dealt one per thread across the
// whole cluster (they lie in a few contiguous ranges, which whole runs would
// leave to one or two CTAs) and stored entry by entry.  The caller
// synchronises the cluster before any lookup.
__device__ __forceinline__ void build_gelu_table(uint16_t* table, int cluster) {
  const uint32_t rank = cluster_ctarank();
  const int per_cta = 65536 / cluster;
  const uint32_t table_addr = smem_u32(table);
  for (int e = static_cast<int>(rank) * per_cta + static_cast<int>(threadIdx.x) * 8;
       e < static_cast<int>(rank + 1) * per_cta; e += static_cast<int>(blockDim.x) * 8) {
    const uint32_t u = static_cast<uint32_t>(e);
    if (gelu_slow_run(u)) continue;
    const uint4 pats = make_uint4(u | ((u + 1) << 16), (u + 2) | ((u + 3) << 16), (u + 4) | ((u + 5) << 16),
                                  (u + 6) | ((u + 7) << 16));
    const uint4 g = qrow::gelu_bf16x8(pats);
    for (int r = 0; r < cluster; ++r) st_cluster_v4(map_to_cta(table_addr + 2u * u, static_cast<uint32_t>(r)), g);
  }
  const int stride = cluster * static_cast<int>(blockDim.x);
  for (int f = static_cast<int>(rank) + cluster * static_cast<int>(threadIdx.x); f < kGeluSlowPatterns; f += stride) {
    const uint32_t u = gelu_slow_pattern(f);
    const uint32_t g = qrow::gelu_bf16_bits(u);
    for (int r = 0; r < cluster; ++r) st_cluster_u16(map_to_cta(table_addr + 2u * u, static_cast<uint32_t>(r)), g);
  }
}

template <int VPL, int GROUPS>
__global__ void __launch_bounds__(256 * GROUPS, 1)
    quantize_rows_gelu_lut_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t K, int64_t ldx,
                                  int8_t* __restrict__ q, int64_t ldq, float* __restrict__ scale, int cluster) {
  static_assert(GROUPS >= 1 && GROUPS <= kLutMaxGroups, "row groups per CTA");
  extern __shared__ __align__(16) uint8_t lut_smem[];
  uint16_t* table = reinterpret_cast<uint16_t*>(lut_smem);
  float* wmax = reinterpret_cast<float*>(lut_smem + kLutTableBytes);  // [2][GROUPS][8]
  const int tid = threadIdx.x;
  build_gelu_table(table, cluster);
  // h is the previous kernel's output: wait for it only now.
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  cluster_sync_all();  // every table entry written and visible; no remote access after this

  const int grp = tid >> 8;
  const int t = tid & 255;
  const int lane = tid & 31;
  const int warp = t >> 5;
  const int nvec = static_cast<int>(K / 8);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * GROUPS;
  uint4 next[VPL];
  auto load_row = [&](int64_t r) {
    const uint4* xr = reinterpret_cast<const uint4*>(x + r * ldx);
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = t + 256 * i;
      next[i] = v < nvec ? __ldg(xr + v) : make_uint4(0u, 0u, 0u, 0u);  // GELU(+0) = +0
    }
  };
  int64_t row = static_cast<int64_t>(blockIdx.x) * GROUPS + grp;
  if (row < M) load_row(row);
  int parity = 0;
  for (; row < M; row += stride, parity ^= 1) {
    uint4 c[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) c[i] = next[i];
    if (row + stride < M) load_row(row + stride);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      c[i] = make_uint4(lut_pair(table, c[i].x), lut_pair(table, c[i].y), lut_pair(table, c[i].z),
                        lut_pair(table, c[i].w));
      amax = fmaxf(amax, qrow::vec_absmax<__nv_bfloat16>(c[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float* slot = wmax + (parity * GROUPS + grp) * 8;
    if (lane == 0) slot[warp] = amax;
    named_barrier_sync(1 + grp, 256);
#pragma unroll
    for (int w = 0; w < 8; ++w) amax = fmaxf(amax, slot[w]);
    const qrow::RowScale rs = qrow::row_scale<qrow::Code::kInt8>(amax);
    int8_t* qr = q + row * ldq;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int v = t + 256 * i;
      if (v < nvec) {
        if (rs.zero) {
          qrow::store_zero<8>(qr + 8 * v);
        } else {
          qrow::encode_vec<__nv_bfloat16, qrow::Code::kInt8>(c[i], rs, qr + 8 * v);
        }
      }
    }
    if (t == 0) scale[row] = rs.s;
  }
}

// bf16 GELU of rows h [M, K] into g by the same table: a persistent grid
// over the rows' 16-byte vectors, four vectors per thread in flight, eight
// lookups per vector.
__global__ void __launch_bounds__(kLutThreads, 1)
    gelu_rows_lut_kernel(const __nv_bfloat16* __restrict__ h, int64_t M, int64_t K, int64_t ldh,
                         __nv_bfloat16* __restrict__ g, int64_t ldg, int cluster) {
  extern __shared__ __align__(16) uint8_t lut_smem[];
  uint16_t* table = reinterpret_cast<uint16_t*>(lut_smem);
  build_gelu_table(table, cluster);
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  cluster_sync_all();
  constexpr int kUnroll = 4;
  const int64_t vpr = K / 8;  // vectors per row
  const int64_t total = M * vpr;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
       base += kUnroll * stride) {
    uint4 x[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * stride;
      if (i < total) {
        const int64_t r = i / vpr;
        x[u] = __ldg(reinterpret_cast<const uint4*>(h + r * ldh) + (i - r * vpr));
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = base + u * stride;
      if (i < total) {
        const int64_t r = i / vpr;
        reinterpret_cast<uint4*>(g + r * ldg)[i - r * vpr] = make_uint4(
            lut_pair(table, x[u].x), lut_pair(table, x[u].y), lut_pair(table, x[u].z), lut_pair(table, x[u].w));
      }
    }
  }
}

// Launch geometry of the table kernels on one device: cluster size and the
// number of clusters that are resident at once (one CTA per SM).
struct LutGeometry {
  int cluster = 0;
  int clusters = 0;
};

template <auto kernel, int kThreads>
LutGeometry lut_geometry(cudaStream_t stream) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static LutGeometry cache[kMaxDev];  // one per kernel (template argument) and device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return {};
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev].cluster != 0) return cache[dev];
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kLutSmemBytes) != cudaSuccess) {
    return {};
  }
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2) return {};
  // Clusters of 2 always fit side by side (SMs come in pairs).  A larger
  // cluster splits the table's construction over more CTAs; it is taken when
  // the clusters of that size that are resident at once leave at most
  // kSpareSms of the SMs idle (per the occupancy query).  The query is not
  // made while the stream is being captured.
  constexpr int kSpareSms = 8;
  LutGeometry g{2, sms / 2};
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusNone) {
    for (int c : {8, 4}) {
      cudaLaunchConfig_t lc = {};
      lc.gridDim = dim3(c * (sms / c));
      lc.blockDim = dim3(kThreads);
      lc.dynamicSmemBytes = kLutSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = c;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      lc.attrs = attr;
      lc.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kernel, &lc) != cudaSuccess) {
        (void)cudaGetLastError();  // the query's own error: fall back to a smaller cluster
        continue;
      }
      if (n * c >= 2 * (sms / 2) - kSpareSms) {
        g = LutGeometry{c, n};
        break;
      }
    }
    cache[dev] = g;
  }
  return g;
}

// Launches a table kernel: `units` work items (rows or vectors), `per_cta`
// of them per CTA per pass, on at most the clusters that are resident at once
// (the grid is persistent), as a programmatic dependent of the previous
// kernel in the stream.  The kernel's last argument is the cluster size.
template <auto kernel, int kThreads, typename... Args>
cudaError_t launch_lut(int64_t units, int64_t per_cta, cudaStream_t stream, Args... args) {
  const LutGeometry geo = lut_geometry<kernel, kThreads>(stream);
  if (geo.cluster == 0) return cudaErrorInvalidConfiguration;
  const int64_t per_cluster = per_cta * geo.cluster;
  const int64_t clusters = std::max<int64_t>(1, std::min<int64_t>(geo.clusters, (units + per_cluster - 1) / per_cluster));
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(static_cast<unsigned>(clusters * geo.cluster));
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = kLutSmemBytes;
  lc.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(geo.cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 2;
  return cudaLaunchKernelEx(&lc, kernel, args..., geo.cluster);
}

// Row groups per CTA for VPL vectors per thread: as many as the registers of
// two copies of the row allow (a CTA of 256 * G threads has 65536 / (256 * G)
// registers per thread).  At VPL 6 (rows of 12288) three groups would fit
// with a small spill but measured slower than two: 89.5 against 82.7 us on
// 9216 x 12288.
template <int VPL>
constexpr int lut_groups() {
  return VPL <= 2 ? 4 : (VPL <= 4 ? 3 : 2);
}

template <int VPL>
cudaError_t launch_gelu_lut(const __nv_bfloat16* x, int64_t M, int64_t K, int64_t ldx, int8_t* q, int64_t ldq,
                            float* scale, cudaStream_t stream) {
  constexpr int G = lut_groups<VPL>();
  return launch_lut<quantize_rows_gelu_lut_kernel<VPL, G>, 256 * G>(M, G, stream, x, M, K, ldx, q, ldq, scale);
}

}  // namespace

// Sets up the table kernel that launch_quantize_act_gelu uses for rows of K
// (its shared-memory size and cluster geometry) outside of any stream
// capture, so that a captured launch gets the geometry chosen by the
// occupancy query rather than the fallback.
cudaError_t prepare_quantize_act_gelu(int64_t K, cudaStream_t stream) {
  const int64_t per_thread = (K / 8 + 255) / 256;
  LutGeometry g;
  if (per_thread <= 2) {
    g = lut_geometry<quantize_rows_gelu_lut_kernel<2, lut_groups<2>()>, 256 * lut_groups<2>()>(stream);
  } else if (per_thread <= 4) {
    g = lut_geometry<quantize_rows_gelu_lut_kernel<4, lut_groups<4>()>, 256 * lut_groups<4>()>(stream);
  } else if (per_thread <= 6) {
    g = lut_geometry<quantize_rows_gelu_lut_kernel<6, lut_groups<6>()>, 256 * lut_groups<6>()>(stream);
  } else if (per_thread <= 8) {
    g = lut_geometry<quantize_rows_gelu_lut_kernel<8, lut_groups<8>()>, 256 * lut_groups<8>()>(stream);
  } else {
    return cudaSuccess;  // longer rows use the row kernels, which need no setup
  }
  return g.cluster != 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

// GELU then per-token int8 codes: rows of up to 16384 bf16 through the table
// kernel, longer rows through the row kernels with GELU evaluated per
// element (both give the same bits).
cudaError_t launch_quantize_act_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, int8_t* q, int64_t ldq,
                                     float* scale, cudaStream_t stream) {
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(h);
  const int64_t per_thread = (K / 8 + 255) / 256;
  if (per_thread <= 2) return launch_gelu_lut<2>(x, M, K, ldh, q, ldq, scale, stream);
  if (per_thread <= 4) return launch_gelu_lut<4>(x, M, K, ldh, q, ldq, scale, stream);
  if (per_thread <= 6) return launch_gelu_lut<6>(x, M, K, ldh, q, ldq, scale, stream);
  if (per_thread <= 8) return launch_gelu_lut<8>(x, M, K, ldh, q, ldq, scale, stream);
  return launch_quantize<__nv_bfloat16, qrow::Code::kInt8, qrow::Pre::kGelu>(x, M, K, ldh, q, ldq, scale, stream);
}

cudaError_t launch_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, void* g, int64_t ldg, int sms,
                        cudaStream_t stream) {
  (void)sms;  // the grid is sized from the cluster occupancy instead
  return launch_lut<gelu_rows_lut_kernel, kLutThreads>(M * (K / 8), kLutThreads, stream,
                                                      static_cast<const __nv_bfloat16*>(h), M, K, ldh,
                                                      static_cast<__nv_bfloat16*>(g), ldg);
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
