// gemm_sm100.cu -- fused W8A8 GEMM for B200 (sm_100a).
//
// Paper: "Realizing Native INT8 Compute for Diffusion Transformers on
// Consumer GPUs" (arXiv 2606.14598), abstract -- an int8 x int8 -> int32
// GEMM on the tensor cores with the per-token x per-channel dequantization
// and the bias folded into the epilogue:
//   out[m,n] = bf16_rne((fl32(acc[m,n]) * scale_a[m]) * scale_w[n] + bias[n]),
//   acc[m,n] = sum_k xq[m,k] * wq[n,k]  (exact in int32).
// The paper's kernel is Triton on Ampere mma.sync; this one is written for
// the 5th-generation tensor cores:
//
//   * persistent: one CTA (or CTA pair) per SM (pair of SMs) walks output
//     tiles of BLOCK_M x BLOCK_N in a grouped raster order; when the last
//     round would leave at least half of them idle, its tiles run as two
//     half-width items each;
//   * tiles: 128 x 256 or 128 x 128 on one CTA, or 256 x 256 / 256 x 128 on
//     a CTA pair (tcgen05 cta_group::2: each CTA loads its 128 rows of A and
//     half of B, the leader issues M=256 MMAs over both CTAs' shared memory,
//     each CTA's tensor memory holds its 128 rows of the accumulator);
//   * warp 0 (one elected lane) streams K-chunks of 128 bytes of both
//     operands with TMA into a ring of shared-memory stages (128-byte
//     swizzle), signalling "full" mbarriers with transaction counts; a
//     pair's stage holds two K-chunks loaded as one box each through 3-D
//     tensor maps when K allows (larger requests: the per-SM TMA delivery
//     rate depends on them);
//   * warp 1 allocates tensor memory and (one elected lane) issues
//     tcgen05.mma.kind::i8, K=32 per instruction, into int32 accumulators
//     held in tensor memory; tcgen05.commit frees each ring stage when its
//     MMAs retire and marks the accumulator full after the last K-chunk;
//   * warps 2-9 (the epilogue) work two per 32-lane quarter of tensor
//     memory (= 32 output rows), each on half of the tile's columns: they
//     load the int32 accumulators, apply the dequantization and bias in
//     binary32 in the order above, round to bf16, stage 32 x 64 bf16 blocks
//     in swizzled shared memory and write them with TMA stores;
//   * the accumulator is double-buffered in tensor memory (2 x BLOCK_N
//     columns), so the epilogue of one tile overlaps the MMAs of the next.

// The same kernel runs the FP8 variant (OCP E4M3 operands, the paper's
// comparison baseline): tcgen05.mma.kind::f8f6f4, also K=32 bytes per
// instruction, so the tiles, the ring and the swizzle are unchanged; the
// accumulators are fp32 and the epilogue uses them as they are.
//
// Every mbarrier wait is bounded in time (see sm100_ptx.cuh); on timeout the
// kernel records the site in the device error word, lets its in-flight
// copies and MMAs finish (again bounded), frees tensor memory and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "internal.h"
#include "quant_row.cuh"
#include "sm100_ptx.cuh"

namespace w8a8 {

// Device-side error word of this library's kernels (see WaitSite).
__device__ int g_device_error = 0;

namespace {

constexpr int kBlockM = 128;
constexpr int kBlockK = 128;            // bytes of K per stage = one 128-byte swizzle row
constexpr int kMmaK = 32;               // K per tcgen05.mma .kind::i8
constexpr int kEpiWarps = 8;            // two per 32-lane quarter of tensor memory
constexpr int kThreads = 64 + 32 * kEpiWarps;  // producer, MMA, epilogue warps
constexpr int kEpiBufBytes = 32 * 128;  // one staging block per epilogue warp: 32 rows x 128 bytes
constexpr int kSmemLimit = 232448;      // dynamic shared memory per block on sm_100
constexpr int kBarrierBytes = 256;

struct Params {
  int M, N, K;
  int m_tiles, n_tiles, k_blocks, num_tiles;
  // Work items: tiles [0, full_tiles) whole; when the last round of tiles
  // would leave CTAs idle, each remaining tile is done as two half-width
  // items (block_n / 2 columns each), so work_items = full_tiles + 2 * tail.
  int full_tiles, work_items;
  int raster_group;
  int stages;
  const float* scale_a;
  const float* scale_w;
  const __nv_bfloat16* bias;
  uint64_t timeout_ns;
  int* err;  // device error word
  // L2 policy of the A operand (the activations): evict_last, like B, while
  // A is small enough to stay in L2 beside B; evict_first when A alone is
  // more than half of L2 (long-K layers: A is then streamed once per tile
  // row and would push B out, which every tile row reads again).
  int a_evict_first;
  // Fused linear layer only: the bf16 activations, the workspace the kernel
  // quantizes them into (xq is also the A operand of tm_a), and the
  // row-block counters ([m_tiles] blocks + 1 CTA counter, zero on entry).
  const __nv_bfloat16* x;
  int64_t ldx;
  int8_t* xq_out;
  float* scale_out;
  uint32_t* sync;
};

__host__ __device__ constexpr int a_stage_bytes() { return kBlockM * kBlockK; }

// Per-tile epilogue constants in shared memory: scale_w (fp32) and bias
// (bf16) of the tile's block_n columns.
__host__ __device__ constexpr int params_bytes(int bn) { return bn * 6; }

// Dynamic shared memory of one CTA: alignment slack, the operand ring (A:
// 128 rows, B: block_n rows, or block_n / 2 for a CTA pair; `chunks` K-chunks
// of 128 bytes in all), the epilogue's staging blocks and per-tile
// constants, and the barriers.
int smem_bytes(bool pair, int bn, int chunks) {
  const int b_rows = pair ? bn / 2 : bn;
  return 1024 + chunks * (a_stage_bytes() + b_rows * kBlockK) + kEpiWarps * kEpiBufBytes + params_bytes(bn) +
         kBarrierBytes;
}

__device__ __forceinline__ void tile_coords(int tile, const Params& p, int& mb, int& nb);

// Work item -> output tile (mb, nb) and half (-1: the whole tile, 0 / 1:
// the left / right block_n / 2 columns of a tail tile).
__device__ __forceinline__ void item_coords(int item, const Params& p, int& mb, int& nb, int& hb) {
  if (item < p.full_tiles) {
    tile_coords(item, p, mb, nb);
    hb = -1;
  } else {
    const int r = item - p.full_tiles;
    tile_coords(p.full_tiles + (r >> 1), p, mb, nb);
    hb = r & 1;
  }
}

__device__ __forceinline__ void tile_coords(int tile, const Params& p, int& mb, int& nb) {
  const int per_group = p.raster_group * p.n_tiles;
  const int g = tile / per_group;
  const int first_m = g * p.raster_group;
  const int gsz = min(p.raster_group, p.m_tiles - first_m);
  const int r = tile - g * per_group;
  mb = first_m + r % gsz;
  nb = r / gsz;
}

// Dequantize 32 accumulators of one row into 16 packed bf16 pairs:
// y = (fl32(acc) * sa) * sw[n] + bias[n], each op rounded, with sw / bias
// (32 columns) read from shared memory.  kF32Acc: the accumulators are
// already fp32 (E4M3 operands); otherwise int32, converted with rounding.
template <bool kF32Acc>
__device__ __forceinline__ void dequant_32(const uint32_t (&v)[32], float sa, const float* sw_s,
                                           const uint16_t* bias_s, uint32_t* packed) {
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const float4 s0 = *reinterpret_cast<const float4*>(sw_s + 8 * g);
    const float4 s1 = *reinterpret_cast<const float4*>(sw_s + 8 * g + 4);
    const uint4 bw = *reinterpret_cast<const uint4*>(bias_s + 8 * g);
    const float sw[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    const uint32_t w[4] = {bw.x, bw.y, bw.z, bw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float y[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float b = __uint_as_float(j ? (w[i] & 0xFFFF0000u) : (w[i] << 16));
        const uint32_t a = v[8 * g + 2 * i + j];
        float t = kF32Acc ? __uint_as_float(a) : __int2float_rn(static_cast<int>(a));
        t = __fmul_rn(t, sa);
        t = __fmul_rn(t, sw[2 * i + j]);
        y[j] = __fadd_rn(t, b);
      }
      const __nv_bfloat162 h = __floats2bfloat162_rn(y[0], y[1]);
      packed[4 * g + i] = *reinterpret_cast<const uint32_t*>(&h);
    }
  }
}

// One kernel for both tile shapes.  PAIR = false: one CTA computes a
// 128 x BN tile.  PAIR = true: a cluster of two CTAs computes a 256 x BN tile
// with tcgen05 cta_group::2 -- each CTA loads its own 128 rows of A and half
// (BN/2 rows) of B, the pair's leader (cluster rank 0) issues M=256 MMAs that
// read both CTAs' shared memory, and each CTA's tensor memory receives its
// own 128 rows of the accumulator.  Barriers of the pair: the leader's "full"
// stages count both CTAs' TMA bytes; the leader's commits arrive on the
// "empty" and "accumulator full" barriers of both CTAs; both CTAs' epilogue
// warps arrive on the leader's "accumulator empty" barrier.
// FUSE (single CTAs only): the whole W8A8 linear layer in one kernel.  The
// epilogue warps, idle until the first accumulator is ready, first quantize
// the activation rows (one warp per row, rows dealt round-robin over all
// CTAs so that low row blocks finish first) into the workspace and count
// each finished row on its 128-row block's counter (release); the TMA
// producer acquires a block's counter before loading that block's rows of
// A, and the epilogue before reading its scales.  All CTAs are co-resident
// (cooperative launch), so these waits cannot deadlock; they are bounded
// all the same.  The last CTA to finish resets the counters to zero.
template <int BN, GemmOut OUT, bool PAIR, bool FUSE, GemmElem EL, int KCH>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_w8a8_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_b_half, const __grid_constant__ CUtensorMap tm_d,
                     const Params p) {
  constexpr int kTileM = PAIR ? 2 * kBlockM : kBlockM;  // rows of the output tile
  constexpr int kBRows = PAIR ? BN / 2 : BN;             // rows of B this CTA loads
  // A ring stage holds KCH K-chunks of 128 bytes of both operands, each
  // chunk [rows][128 B] (KCH = 2: CTA pairs, loaded as boxes spanning two
  // chunks through 3-D tensor maps).
  static_assert(KCH == 1 || (KCH == 2 && PAIR && !FUSE), "double-chunk stages are for CTA pairs");
  constexpr uint32_t kA = KCH * a_stage_bytes();
  constexpr uint32_t kB = KCH * kBRows * kBlockK;
  constexpr uint32_t kTxBytes = (PAIR ? 2 : 1) * (kA + kB);
  constexpr uint32_t kTmemCols = 2 * BN;  // two accumulator buffers; 256 or 512 (power of two)
  constexpr bool kE4M3 = EL == GemmElem::kE4M3;
  constexpr uint32_t kIdesc = kE4M3 ? make_idesc_e4m3(kTileM, BN) : make_idesc_i8(kTileM, BN);
  // half-width tail items
  constexpr uint32_t kIdescHalf = kE4M3 ? make_idesc_e4m3(kTileM, BN / 2) : make_idesc_i8(kTileM, BN / 2);
  constexpr int kEpiArrivals = (PAIR ? 2 : 1) * kEpiWarps;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stages = p.stages;
  uint8_t* sA = smem;
  uint8_t* sB = sA + stages * kA;
  uint8_t* sEpi = sB + stages * kB;
  float* ps_w = reinterpret_cast<float*>(sEpi + kEpiWarps * kEpiBufBytes);
  uint16_t* ps_b = reinterpret_cast<uint16_t*>(ps_w + BN);
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + kEpiWarps * kEpiBufBytes + params_bytes(BN));
  uint64_t* empty = full + stages;
  uint64_t* tfull = empty + stages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  // Tiles are walked per CTA (single) or per CTA pair.
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int num_units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiArrivals);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    if (p.work_items != p.num_tiles) prefetch_tensormap(&tm_b_half);
    prefetch_tensormap(&tm_d);
  }
  if constexpr (PAIR) {
    cluster_sync_all();  // the peer's barriers exist before anyone signals them
  } else {
    __syncthreads();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_alloc_permit_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish_alloc_permit();
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t peer_abort = PAIR ? map_to_cta(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u) : 0u;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    int64_t fills = 0;
    bool ok = true;
    int ready_mb = -1;  // fused layer: the last row block known to be quantized
    // Both operands are read again by other tiles: keep them in L2 ahead of
    // the streamed output -- B always; A unless it is too large to stay.
    const uint64_t keep = l2_policy_evict_last();
    const uint64_t a_pol = p.a_evict_first ? l2_policy_evict_first() : keep;
    for (int item = unit; ok && item < p.work_items; item += num_units) {
      int mb, nb, hb;
      item_coords(item, p, mb, nb, hb);
      const int a_row = mb * kTileM + static_cast<int>(rank) * kBlockM;
      // this CTA's rows of B: all BN (single CTA) or its half (pair); a
      // half-width item covers BN / 2 columns, of which a pair's CTA loads half
      const int b_row = nb * BN + (hb < 0 ? static_cast<int>(rank) * kBRows
                                          : hb * (BN / 2) + static_cast<int>(rank) * (kBRows / 2));
      // a half-width item loads half of B's rows, through the tensor map with half-height boxes
      const CUtensorMap* map_b = hb < 0 ? &tm_b : &tm_b_half;
      const uint32_t tx_bytes = hb < 0 ? kTxBytes : (PAIR ? 2u : 1u) * (kA + kB / 2);
      for (int kb = 0; kb < p.k_blocks; ++kb) {
        ok = warp_wait(&empty[stage], phase ^ 1u, abort_flag, p.timeout_ns, p.err, kSiteProducerEmpty);
        if (!ok) break;
        if (lane == 0) {
          if constexpr (PAIR && KCH == 2) {
            // 3-D maps {128 B, rows, K-chunk}: one box = this CTA's rows x two chunks
            const uint32_t bar = map_to_cta(smem_u32(&full[stage]), 0u);
            if (leader) mbar_arrive_expect_tx(&full[stage], tx_bytes);
            tma_load_3d_pair_hint(sB + stage * kB, map_b, bar, 0, b_row, 2 * kb, keep);
            if (fills == 0) pdl_wait_prerequisites();  // A may be written by the kernel before this one
            tma_load_3d_pair_hint(sA + stage * kA, &tm_a, bar, 0, a_row, 2 * kb, a_pol);
          } else if constexpr (PAIR) {
            const uint32_t bar = map_to_cta(smem_u32(&full[stage]), 0u);
            if (leader) mbar_arrive_expect_tx(&full[stage], tx_bytes);
            tma_load_2d_pair_hint(sB + stage * kB, map_b, bar, kb * kBlockK, b_row, keep);
            if (fills == 0) pdl_wait_prerequisites();  // A may be written by the kernel before this one
            tma_load_2d_pair_hint(sA + stage * kA, &tm_a, bar, kb * kBlockK, a_row, a_pol);
          } else {
            mbar_arrive_expect_tx(&full[stage], tx_bytes);
            tma_load_2d_hint(sB + stage * kB, map_b, &full[stage], kb * kBlockK, b_row, keep);
            if constexpr (!FUSE) {
              if (fills == 0) pdl_wait_prerequisites();  // A may be written by the kernel before this one
              tma_load_2d_hint(sA + stage * kA, &tm_a, &full[stage], kb * kBlockK, a_row, a_pol);
            }
          }
        }
        if constexpr (FUSE) {
          if (mb != ready_mb) {
            // This block's activation rows must be quantized before TMA reads them.
            bool rok = true;
            if (lane == 0) {
              rok = counter_wait_bounded(&p.sync[mb], static_cast<uint32_t>(min(kBlockM, p.M - mb * kBlockM)),
                                         abort_flag, p.timeout_ns, p.err, kSiteRowsReady);
              fence_proxy_async_global();
            }
            ok = __shfl_sync(0xffffffffu, rok ? 1 : 0, 0) != 0;
            if (ok) ready_mb = mb;
          }
          // After a failed wait the load is still issued (its data is
          // discarded): the stage's barrier completes and teardown drains it.
          if (lane == 0) tma_load_2d_hint(sA + stage * kA, &tm_a, &full[stage], kb * kBlockK, a_row, a_pol);
          if (!ok) {
            __syncwarp();
            ++fills;
            break;
          }
        }
        __syncwarp();
        ++fills;
        if (++stage == stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Every operand load of this CTA is issued: a kernel launched as this
    // one's programmatic dependent may be scheduled (it waits for this
    // grid's completion before reading anything it writes).
    pdl_launch_dependents();
    if (!ok && PAIR && lane == 0) st_cluster_u32(peer_abort, 1u);
    // Teardown: the last fill of each stage must have landed before the CTA
    // exits (on the normal path the MMA warp already waited for all of
    // them).  A pair's loads complete on the leader's barriers, which the
    // leader drains for both CTAs.
    if (leader && lane == 0) {
      const int64_t first = fills > stages ? fills - stages : 0;
      for (int64_t f = first; f < fills; ++f) {
        mbar_wait_drain(&full[f % stages], static_cast<uint32_t>((f / stages) & 1), p.timeout_ns, p.err);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int item = unit; ok && item < p.work_items; item += num_units, ++local) {
        const uint32_t idesc = item < p.full_tiles ? kIdesc : kIdescHalf;
        // bytes between the K-chunks of a stage's B block (half-width items hold half the rows)
        const uint32_t b_chunk = (item < p.full_tiles ? kBRows : kBRows / 2) * kBlockK;
        const int buf = local & 1;
        const uint32_t tphase = static_cast<uint32_t>(local >> 1) & 1u;
        ok = warp_wait(&tempty[buf], tphase ^ 1u, abort_flag, p.timeout_ns, p.err, kSiteMmaTmemEmpty);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; kb < p.k_blocks; ++kb) {
          ok = warp_wait(&full[stage], phase, abort_flag, p.timeout_ns, p.err, kSiteMmaFull);
          if (!ok) break;
          tc_fence_after_sync();
          if (lane == 0) {
#pragma unroll
            for (int kk = 0; kk < KCH * (kBlockK / kMmaK); ++kk) {
              // Chunk c of the stage, then K=32 slice k inside its 128-byte
              // swizzled rows: the start address advances by 32 bytes (2 in
              // units of 16 B) per slice.
              const int c = kk / (kBlockK / kMmaK);
              const int k = kk % (kBlockK / kMmaK);
              const uint64_t a_desc =
                  make_smem_desc_k_sw128(smem_u32(sA + stage * kA + c * a_stage_bytes()));
              const uint64_t b_desc = make_smem_desc_k_sw128(smem_u32(sB + stage * kB + c * b_chunk));
              const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
              if constexpr (PAIR && kE4M3) {
                mma_e4m3_pair(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, acc);
              } else if constexpr (PAIR) {
                mma_i8_pair(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, acc);
              } else if constexpr (kE4M3) {
                mma_e4m3(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, acc);
              } else {
                mma_i8(d_tmem, a_desc + 2 * k, b_desc + 2 * k, idesc, acc);
              }
            }
            if constexpr (PAIR) {
              mma_commit_pair(smem_u32(&empty[stage]));
              mma_commit_pair(map_to_cta(smem_u32(&empty[stage]), 1u));
            } else {
              mma_commit(&empty[stage]);
            }
          }
          __syncwarp();
          if (++stage == stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) {
          if constexpr (PAIR) {
            mma_commit_pair(smem_u32(&tfull[buf]));
            mma_commit_pair(map_to_cta(smem_u32(&tfull[buf]), 1u));
          } else {
            mma_commit(&tfull[buf]);
          }
        }
        __syncwarp();
      }
      if (!ok && PAIR && lane == 0) st_cluster_u32(peer_abort, 1u);
      // Teardown: no MMA may still write tensor memory when it is freed.
      if (lane == 0) {
        if constexpr (PAIR) {
          mma_commit_pair(smem_u32(drain));
        } else {
          mma_commit(drain);
        }
        mbar_wait_drain(drain, 0, p.timeout_ns, p.err);
      }
      __syncwarp();
    }
  } else {
    // --------------------------------------------------------- epilogue
    // Warp e = warp - 2 reads tensor-memory lanes 32 * (warp % 4) .. +31 (the
    // quarter a warp may address) and columns half * BN/2 .. +BN/2 of the
    // accumulator, 32 columns at a time, loading the next 32 while it
    // converts the current ones.
    constexpr int kSub = BN / 2 / 32;  // 32-column loads per warp for a whole tile (half-width items: kSub / 2)
    constexpr int kSubPerStore = (OUT == GemmOut::kBf16Dequant) ? 2 : 1;    // loads per 128-byte row block
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int half = e >> 2;
    uint8_t* sbuf = sEpi + e * kEpiBufBytes;
    const uint64_t stream_out = l2_policy_evict_first();  // the output is not read again here
    if constexpr (!FUSE) pdl_wait_prerequisites();  // scale_a may come from the kernel before this one
    int local = 0;
    bool ok = true;
    if constexpr (FUSE) {
      // Per-token quantization of the activations.  Warp w of the grid's
      // nq epilogue warps takes the row pairs (2w, 2w+1), (2(w+nq), ...),
      // both rows' loads in flight together, so the low row blocks the
      // first tiles need are finished first.
      const int nvec = p.K / 8;
      const int nq = static_cast<int>(gridDim.x) * kEpiWarps;
      auto publish = [&](int r, float srow) {
        if (lane == 0) p.scale_out[r] = srow;
        // Publish the row: its codes are read by other CTAs' TMA (async proxy).
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_gpu_add(&p.sync[r / kBlockM], 1u);
      };
      auto xrow = [&](int r) { return reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(r) * p.ldx); };
      auto qrow_ptr = [&](int r) { return p.xq_out + static_cast<int64_t>(r) * p.K; };
      for (int pr = static_cast<int>(blockIdx.x) * kEpiWarps + e; 2 * pr < p.M; pr += nq) {
        const int r = 2 * pr;
        const int r2 = r + 1;
        if (nvec <= 32 * 12) {
          if (r2 < p.M) {
            float s0, s1;
            qrow::quantize_two_rows<__nv_bfloat16, 12>(xrow(r), xrow(r2), nvec, qrow_ptr(r), qrow_ptr(r2), lane, s0,
                                                        s1);
            publish(r, s0);
            publish(r2, s1);
          } else {
            publish(r, qrow::quantize_row<__nv_bfloat16, 12>(xrow(r), nvec, qrow_ptr(r), lane));
          }
        } else {
          publish(r, qrow::quantize_row<__nv_bfloat16, 0>(xrow(r), nvec, qrow_ptr(r), lane));
          if (r2 < p.M) publish(r2, qrow::quantize_row<__nv_bfloat16, 0>(xrow(r2), nvec, qrow_ptr(r2), lane));
        }
      }
    }
    for (int item = unit; ok && item < p.work_items; item += num_units, ++local) {
      int mb, nb, hb;
      item_coords(item, p, mb, nb, hb);
      const int tile_n = hb < 0 ? BN : BN / 2;           // columns of this item
      const int col_base = nb * BN + (hb < 0 ? 0 : hb * (BN / 2));
      const int nsub = tile_n / 64;                       // this warp's 32-column loads
      const int buf = local & 1;
      const uint32_t tphase = static_cast<uint32_t>(local >> 1) & 1u;
      ok = warp_wait(&tfull[buf], tphase, abort_flag, p.timeout_ns, p.err, kSiteEpiTmemFull);
      if (!ok) break;
      tc_fence_after_sync();

      const int row0 = mb * kTileM + static_cast<int>(rank) * kBlockM + quarter * 32;
      const int row = row0 + lane;
      float sa = 0.0f;
      if constexpr (FUSE) {
        // The scales of this row block were written by other warps of the grid.
        ok = counter_wait_bounded(&p.sync[mb], static_cast<uint32_t>(min(kBlockM, p.M - mb * kBlockM)), abort_flag,
                                  p.timeout_ns, p.err, kSiteRowsReady);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      if constexpr (OUT == GemmOut::kBf16Dequant) {
        if (row < p.M) sa = FUSE ? p.scale_out[row] : __ldg(p.scale_a + row);
        // This tile's scale_w and bias, staged once for all epilogue warps
        // (the first barrier: every warp is done with the previous tile's).
        named_barrier_sync(1, 32 * kEpiWarps);
        for (int i = e * 32 + lane; i < tile_n; i += 32 * kEpiWarps) {
          const int n = col_base + i;
          ps_w[i] = n < p.N ? __ldg(p.scale_w + n) : 0.0f;
          ps_b[i] = (n < p.N && p.bias != nullptr) ? __bfloat16_as_ushort(p.bias[n]) : static_cast<uint16_t>(0);
        }
        named_barrier_sync(1, 32 * kEpiWarps);
      }
      const uint32_t t_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                              static_cast<uint32_t>(buf * BN + half * (tile_n / 2));

      uint32_t va[32], vb[32];
      tmem_load_32cols_async(t_base, va);
      tmem_wait_load(va);
#pragma unroll
      for (int sc = 0; sc < kSub; ++sc) {
        if (sc >= nsub) break;  // half-width item
        uint32_t(&cur)[32] = (sc & 1) ? vb : va;
        uint32_t(&nxt)[32] = (sc & 1) ? va : vb;
        if (sc + 1 < nsub) tmem_load_32cols_async(t_base + 32 * (sc + 1), nxt);
        if (sc + 1 == nsub) {
          // The last load of this accumulator buffer has completed.
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) {
            if (PAIR && !leader) {
              mbar_arrive_cluster(map_to_cta(smem_u32(&tempty[buf]), 0u));
            } else {
              mbar_arrive(&tempty[buf]);
            }
          }
        }
        const int cl = half * (tile_n / 2) + 32 * sc;  // column inside the item
        const int col0 = col_base + cl - 32 * (sc % kSubPerStore);  // first column of the 128-byte block
        const bool in_range = row0 < p.M && col0 < p.N;
        if (in_range && sc % kSubPerStore == 0) {
          // The previous store from this block must have finished reading it.
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
        }
        if constexpr (OUT == GemmOut::kBf16Dequant) {
          uint32_t pk[16];
          dequant_32<kE4M3>(cur, sa, ps_w + cl, ps_b + cl, pk);
          if (in_range) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int chunk = 4 * (sc % 2) + j;  // 16-byte chunk of the 128-byte row
              const int pos = chunk ^ (lane & 7);  // 128-byte swizzle
              *reinterpret_cast<uint4*>(sbuf + lane * 128 + pos * 16) =
                  make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
          }
        } else {
          if (in_range) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int pos = j ^ (lane & 7);
              *reinterpret_cast<uint4*>(sbuf + lane * 128 + pos * 16) =
                  make_uint4(cur[4 * j], cur[4 * j + 1], cur[4 * j + 2], cur[4 * j + 3]);
            }
          }
        }
        if (in_range && (sc + 1) % kSubPerStore == 0) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d_hint(&tm_d, sbuf, col0, row0, stream_out);
            bulk_commit_group();
          }
          __syncwarp();
        }
        if (sc + 1 < nsub) tmem_wait_load(nxt);
      }
    }
    if (!ok && PAIR && lane == 0) st_cluster_u32(peer_abort, 1u);
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (*abort_flag) {
    // A wait ran out somewhere: give copies already issued (by this CTA or
    // its peer, whose loads signal the leader) time to land before the
    // shared memory they target is released.
    if (threadIdx.x == 0) {
      const uint64_t t0 = global_timer_ns();
      while (global_timer_ns() - t0 < 200000ull) {
      }
    }
    __syncthreads();
  }
  if constexpr (FUSE) {
    // Every CTA is done with the row-block counters: the last one out
    // returns them to zero for the next call.
    if (threadIdx.x == 0) {
      __threadfence();
      const uint32_t prev = atomicAdd(&p.sync[p.m_tiles], 1u);
      if (prev == gridDim.x - 1) {
        for (int i = 0; i <= p.m_tiles; ++i) p.sync[i] = 0u;
        __threadfence();
      }
    }
  }
  if constexpr (PAIR) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after_sync();
    if constexpr (PAIR) {
      tmem_dealloc_pair(tmem_base, kTmemCols);
    } else {
      tmem_dealloc(tmem_base, kTmemCols);
    }
  }
}

// ------------------------------------------------------------------ host

// Device address of g_device_error on the current device (looked up once
// per device; host code must not take the symbol's address directly).
cudaError_t error_word_address(int** out) {
  constexpr int kMaxDev = 64;
  static int* addr[kMaxDev] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<int*>(p);
  }
  *out = addr[dev];
  return cudaSuccess;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] of `elem` bytes, box [box_rows, box_cols],
// 128-byte swizzle, zero fill outside the tensor.
bool encode_2d(CUtensorMap* map, CUtensorMapDataType dtype, int elem, const void* base, int64_t rows,
               int64_t cols, int box_rows, int box_cols) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * static_cast<cuuint64_t>(elem)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view {128 bytes, rows, K / 128} of a K-contiguous byte matrix (K a
// multiple of 128), boxes of box_rows rows x two K-chunks: one load lands
// as two [box_rows][128 B] blocks, 128-byte swizzled.
bool encode_chunks(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr || K % 128 != 0) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 128)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K), 128};
  const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, GemmOut OUT, bool PAIR, bool FUSE, GemmElem EL = GemmElem::kInt8, int KCH = 1>
cudaError_t launch_typed(const GemmArgs& a, const GemmConfig& cfg, cudaStream_t stream) {
  static_assert(!(FUSE && PAIR), "the fused linear layer runs on single CTAs");
  static_assert(!(FUSE && EL == GemmElem::kE4M3), "the fused linear layer is int8 only");
  constexpr int kTileM = PAIR ? 2 * kBlockM : kBlockM;
  constexpr int kBRows = PAIR ? BN / 2 : BN;
  CUtensorMap tm_a, tm_b, tm_b_half, tm_d;
  std::memset(&tm_a, 0, sizeof tm_a);
  std::memset(&tm_b, 0, sizeof tm_b);
  std::memset(&tm_b_half, 0, sizeof tm_b_half);
  std::memset(&tm_d, 0, sizeof tm_d);
  bool ok;
  if constexpr (KCH == 2) {
    ok = encode_chunks(&tm_a, a.xq, a.M, a.K, kBlockM) && encode_chunks(&tm_b, a.wq, a.N, a.K, kBRows) &&
         encode_chunks(&tm_b_half, a.wq, a.N, a.K, kBRows / 2);
  } else {
    ok = encode_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.xq, a.M, a.K, kBlockM, kBlockK) &&
         encode_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.wq, a.N, a.K, kBRows, kBlockK) &&
         encode_2d(&tm_b_half, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.wq, a.N, a.K, kBRows / 2, kBlockK);
  }
  if constexpr (OUT == GemmOut::kBf16Dequant) {
    ok = ok && encode_2d(&tm_d, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.out, a.M, a.N, 32, 64);
  } else {
    ok = ok && encode_2d(&tm_d, EL == GemmElem::kE4M3 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_INT32,
                         4, a.out, a.M, a.N, 32, 32);
  }
  if (!ok) return cudaErrorInvalidValue;

  Params p;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.m_tiles = static_cast<int>((a.M + kTileM - 1) / kTileM);
  p.n_tiles = static_cast<int>((a.N + BN - 1) / BN);
  p.k_blocks = static_cast<int>((a.K + KCH * kBlockK - 1) / (KCH * kBlockK));
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.full_tiles = p.num_tiles;
  p.work_items = p.num_tiles;
  p.raster_group = cfg.raster_group;
  p.stages = cfg.stages / KCH;  // cfg.stages counts K-chunks of ring depth
  p.scale_a = a.scale_a;
  p.scale_w = a.scale_w;
  p.bias = static_cast<const __nv_bfloat16*>(a.bias);
  p.timeout_ns = a.timeout_ns;
  p.err = nullptr;
  p.a_evict_first = a.M * a.K > a.l2_bytes / 2 ? 1 : 0;
  p.x = static_cast<const __nv_bfloat16*>(a.x);
  p.ldx = a.ldx;
  p.xq_out = const_cast<int8_t*>(a.xq);
  p.scale_out = const_cast<float*>(a.scale_a);
  p.sync = a.sync;
  cudaError_t e = error_word_address(&p.err);
  if (e != cudaSuccess) return e;

  const int smem = smem_bytes(PAIR, BN, p.stages * KCH);
  auto kernel = gemm_w8a8_kernel<BN, OUT, PAIR, FUSE, EL, KCH>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // Persistent grid: one CTA (or CTA pair) per tile at most.
  int units = (PAIR ? cfg.grid / 2 : cfg.grid);
  if (units < 1) units = 1;
  if (units > p.num_tiles) units = p.num_tiles;
  // Last round: if at most half the CTAs (pairs) would get a tile, give each
  // of the remaining tiles to two CTAs (pairs) as half-width items instead.
  const int tail = p.num_tiles % units;
  if (BN == 256 && tail > 0 && 2 * tail <= units) {
    p.full_tiles = p.num_tiles - tail;
    p.work_items = p.full_tiles + 2 * tail;
  }
  cudaLaunchConfig_t lc;
  std::memset(&lc, 0, sizeof lc);
  lc.gridDim = dim3(static_cast<unsigned>(units * (PAIR ? 2 : 1)));
  lc.blockDim = dim3(kThreads);
  lc.dynamicSmemBytes = static_cast<size_t>(smem);
  lc.stream = stream;
  cudaLaunchAttribute attr[2];
  if constexpr (FUSE) {
    // CTAs wait on rows quantized by other CTAs: all must be resident at
    // once, which a cooperative launch guarantees (or refuses to launch).
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
  } else {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = PAIR ? 2 : 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
  }
  lc.attrs = attr;
  lc.numAttrs = 1;
  if (!FUSE && a.overlap_prologue) {
    // Programmatic dependent launch: the kernel may start while the previous
    // kernel of the stream (the activation quantizer) finishes; it reads the
    // weight operand, scale_w and bias early and waits (griddepcontrol.wait)
    // before the first read of the quantized activations or their scales.
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.numAttrs = 2;
  }
  e = cudaLaunchKernelEx(&lc, kernel, tm_a, tm_b, tm_b_half, tm_d, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

__global__ void selftest_wait_kernel(uint64_t timeout_ns, int* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait runs out by construction.
  warp_wait(&bar, 0, &abort_flag, timeout_ns, err, kSiteSelfTest);
}

}  // namespace

int gemm_max_stages(int block_m, int block_n) {
  const bool pair = block_m == 2 * kBlockM;
  int s = 0;
  while (smem_bytes(pair, block_n, s + 1) <= kSmemLimit) ++s;
  return s;
}

// Non-fused launches of one operand format.
template <GemmElem EL>
cudaError_t launch_plain(const GemmArgs& a, const GemmConfig& cfg, cudaStream_t stream) {
  using O = GemmOut;
  const bool bf16 = a.out_kind == O::kBf16Dequant;
  if (cfg.block_m == 256) {
    // CTA pairs load two K-chunks per box when K allows it and the ring
    // holds at least two such stages.
    const bool chunks2 = a.K % 128 == 0 && cfg.stages >= 4;
    if (cfg.block_n == 256) {
      if (chunks2) {
        return bf16 ? launch_typed<256, O::kBf16Dequant, true, false, EL, 2>(a, cfg, stream)
                    : launch_typed<256, O::kAcc32, true, false, EL, 2>(a, cfg, stream);
      }
      return bf16 ? launch_typed<256, O::kBf16Dequant, true, false, EL>(a, cfg, stream)
                  : launch_typed<256, O::kAcc32, true, false, EL>(a, cfg, stream);
    }
    if (cfg.block_n == 128) {
      if (chunks2) {
        return bf16 ? launch_typed<128, O::kBf16Dequant, true, false, EL, 2>(a, cfg, stream)
                    : launch_typed<128, O::kAcc32, true, false, EL, 2>(a, cfg, stream);
      }
      return bf16 ? launch_typed<128, O::kBf16Dequant, true, false, EL>(a, cfg, stream)
                  : launch_typed<128, O::kAcc32, true, false, EL>(a, cfg, stream);
    }
  } else if (cfg.block_m == 128) {
    if (cfg.block_n == 256) {
      return bf16 ? launch_typed<256, O::kBf16Dequant, false, false, EL>(a, cfg, stream)
                  : launch_typed<256, O::kAcc32, false, false, EL>(a, cfg, stream);
    }
    if (cfg.block_n == 128) {
      return bf16 ? launch_typed<128, O::kBf16Dequant, false, false, EL>(a, cfg, stream)
                  : launch_typed<128, O::kAcc32, false, false, EL>(a, cfg, stream);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm(const GemmArgs& a, const GemmConfig& cfg, cudaStream_t stream) {
  using O = GemmOut;
  if (a.fused) {
    if (a.out_kind != O::kBf16Dequant || a.elem != GemmElem::kInt8 || cfg.block_m != 128) {
      return cudaErrorInvalidValue;
    }
    if (cfg.block_n == 256) return launch_typed<256, O::kBf16Dequant, false, true>(a, cfg, stream);
    if (cfg.block_n == 128) return launch_typed<128, O::kBf16Dequant, false, true>(a, cfg, stream);
    return cudaErrorInvalidValue;
  }
  return a.elem == GemmElem::kE4M3 ? launch_plain<GemmElem::kE4M3>(a, cfg, stream)
                                   : launch_plain<GemmElem::kInt8>(a, cfg, stream);
}

cudaError_t launch_selftest_wait(uint64_t timeout_ns, cudaStream_t stream) {
  int* err = nullptr;
  cudaError_t e = error_word_address(&err);
  if (e != cudaSuccess) return e;
  selftest_wait_kernel<<<1, 32, 0, stream>>>(timeout_ns, err);
  return cudaGetLastError();
}

cudaError_t read_device_error(int* value, bool clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(int));
  if (e != cudaSuccess) return e;
  if (clear && *value != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
  }
  return e;
}

}  // namespace w8a8
