/*
 * w8a8.h -- C ABI of the B200 (sm_100a) W8A8 linear layer.
 *
 * The operation is the one described in "Realizing Native INT8 Compute for
 * Diffusion Transformers on Consumer GPUs: A Fused INT8 GEMM Kernel for
 * Ideogram 4.0" (arXiv 2606.14598), abstract: post-training W8A8
 * quantization of a diffusion transformer's linear layers, computed as an
 * int8 x int8 -> int32 GEMM on the tensor cores with the per-token x
 * per-channel dequantization and the bias folded into the GEMM's epilogue,
 * in place of a dequantize-to-bf16-then-bf16-GEMM forward.  A linear layer
 * here is y = x W^T + b (the nn.Linear convention):
 *
 *   scale_a[m] = fl32(max_k |x[m,k]| / 127)                       per token
 *   xq[m,k]    = clamp(rne(fl32(x[m,k] / scale_a[m])), -127, 127)
 *   acc[m,n]   = sum_k xq[m,k] * wq[n,k]                    exact, int32
 *   out[m,n]   = bf16_rne((fl32(acc[m,n]) * scale_a[m]) * scale_w[n] + bias[n])
 *
 * The abstract gives no formulas; the readings above (symmetric absmax/127
 * scales, round to nearest even, clamp to +-127, a zero scale giving all-zero
 * codes, this epilogue order with no fused multiply-add) are the library's
 * definition.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every array argument is DEVICE memory on the current CUDA device,
 *           allocated and owned by the caller; the library never allocates
 *           device memory and never frees caller memory.  (It keeps a small
 *           host-side cache of device properties.)
 * Layout.   Row-major.  x: bf16 [M, K]; xq: int8 [M, K]; wq: int8 [N, K]
 *           (the nn.Linear weight layout, so both GEMM operands are
 *           K-contiguous); out: bf16 [M, N]; scale_a: fp32 [M]; scale_w:
 *           fp32 [N]; bias: bf16 [N].  bf16 is passed as void* (raw 16-bit
 *           IEEE bfloat16 values).
 * Async.    Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *           default stream) and the call returns without synchronizing.
 *           Errors found before the launch are returned; a wait inside a
 *           kernel that runs out of time (see w8a8_read_device_error) is
 *           reported later.
 * Shapes.   M >= 0 and N >= 0 (M == 0 or N == 0 is a valid empty call that
 *           launches nothing and returns W8A8_OK); 16 <= K <= 133144 and
 *           K % 16 == 0 (16-byte rows for the tensor-memory-access engine;
 *           K * 127^2 < 2^31 keeps the int32 accumulator exact);
 *           N % 8 == 0 (16-byte output rows); M, N < 2^31.
 * Alignment. Every pointer is 16-byte aligned; otherwise W8A8_ERR_ALIGNMENT.
 * Device.   Compute capability 10.0 (B200, sm_100a); otherwise
 *           W8A8_ERR_UNSUPPORTED_DEVICE.
 * Errors.   Argument errors are detected before any device work and launch
 *           nothing.  A CUDA launch error is returned as W8A8_ERR_LAUNCH.
 */
#ifndef W8A8_H
#define W8A8_H

#include <stdint.h>

#if defined(__GNUC__)
#define W8A8_API __attribute__((visibility("default")))
#else
#define W8A8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* w8a8_stream_t;

typedef enum {
    W8A8_OK = 0,
    W8A8_ERR_INVALID_ARG = 1,         /* bad shape, stride, or NULL pointer */
    W8A8_ERR_ALIGNMENT = 2,           /* a pointer or row stride is not 16-byte aligned */
    W8A8_ERR_UNSUPPORTED_DEVICE = 3,  /* current device is not sm_100 */
    W8A8_ERR_LAUNCH = 4,              /* CUDA refused the launch */
    W8A8_ERR_TIMEOUT = 5,             /* a kernel's bounded wait ran out (see w8a8_read_device_error) */
    W8A8_ERR_CUDA = 6,                /* another CUDA runtime error */
    W8A8_ERR_SCRATCH_LIMIT = 7        /* w8a8_linear_noalloc: the problem needs more than its fixed scratch */
} w8a8_status;

/* Human-readable name of a status code (static string, never NULL). */
W8A8_API const char* w8a8_status_string(int status);

/* ABI version of this header: 100 * major + minor (101: w8a8_linear_desc
 * has input_act). */
W8A8_API int w8a8_abi_version(void);

/*
 * Per-token activation quantization (the paper's per-token activation
 * quantizer; abstract: "per-token" dequantization of the W8A8 GEMM).
 *   x       bf16 [M, K], row stride ldx elements (ldx >= K, ldx % 8 == 0)
 *   xq      int8 [M, K] out, row stride ldxq bytes (ldxq >= K, ldxq % 16 == 0)
 *   scale_a fp32 [M] out
 * One warp per token row, 16-byte loads, a shuffle max-reduction, packed
 * int8 stores.  Results are bit-exact to the definition in the header.
 */
W8A8_API w8a8_status w8a8_quantize_act(const void* x, int64_t M, int64_t K, int64_t ldx,
                              int8_t* xq, int64_t ldxq, float* scale_a, w8a8_stream_t stream);

/*
 * Per-output-channel weight quantization (abstract: post-training W8A8
 * quantization, dequantized per channel in the epilogue).  Same rule as the
 * activation quantizer applied to each row of an fp32 weight:
 *   w       fp32 [N, K], row stride ldw elements (ldw >= K, ldw % 4 == 0)
 *   wq      int8 [N, K] out, row stride ldwq bytes (ldwq >= K, ldwq % 16 == 0)
 *   scale_w fp32 [N] out
 * Used once per weight at load time, not per forward.
 */
W8A8_API w8a8_status w8a8_quantize_weight(const float* w, int64_t N, int64_t K, int64_t ldw,
                                 int8_t* wq, int64_t ldwq, float* scale_w, w8a8_stream_t stream);

/*
 * Fused W8A8 GEMM (abstract: "int8xint8->int32 ... with per-token x
 * per-channel dequantization and bias folded into the epilogue"):
 *   out[m,n] = bf16_rne((fl32(sum_k xq[m,k]*wq[n,k]) * scale_a[m]) * scale_w[n] + bias[n])
 *   xq [M, K] int8, wq [N, K] int8 (row strides K), scale_a [M], scale_w [N]
 *   fp32, bias [N] bf16 or NULL (zero bias), out [M, N] bf16 (row stride N).
 * tcgen05 int8 tensor-core kernel with int32 accumulators in tensor memory;
 * the tile configuration is chosen per shape (w8a8_select_config).
 */
W8A8_API w8a8_status w8a8_gemm(const int8_t* xq, const int8_t* wq, const float* scale_a,
                      const float* scale_w, const void* bias, void* out,
                      int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/*
 * The whole W8A8 linear layer (abstract: the fused kernel "dropped into the
 * ... linear layers in place of the dequantize-to-bf16 path"):
 * w8a8_quantize_act of x into the caller's workspace, then w8a8_gemm.
 *   x [M, K] bf16 (row stride K); wq, scale_w, bias, out as in w8a8_gemm;
 *   ws_xq int8 [M, K] and ws_scale_a fp32 [M]: caller-owned workspace that
 *   receives the quantized activations and their scales (readable after the
 *   call completes).
 */
W8A8_API w8a8_status w8a8_linear(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                        void* out, int8_t* ws_xq, float* ws_scale_a,
                        int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/*
 * The same layer as ONE kernel (the paper's "single fused" kernel, abstract,
 * extended to the quantizer): the GEMM kernel's epilogue warps quantize the
 * activation rows into the workspace first, and the tensor-core pipeline
 * starts on each 128-row block as soon as that block is quantized, so the
 * quantizer's memory traffic overlaps the GEMM instead of preceding it.
 *   Arguments as in w8a8_linear, plus
 *   ws_sync  uint32 [w8a8_linear_sync_words(M)]: row-block counters.  The
 *            caller zeroes it ONCE (e.g. cudaMemset) before the first call;
 *            every call that completes leaves it zeroed again.  After a call
 *            that reported W8A8_ERR_TIMEOUT it must be zeroed again.
 * Calls sharing one ws_sync (or one ws_xq / ws_scale_a) must not overlap on
 * the GPU.  Needs every CTA of the grid resident at once (a cooperative
 * launch); if the device cannot guarantee that, the call fails with
 * W8A8_ERR_LAUNCH and nothing runs.  Results are bit-identical to
 * w8a8_linear.
 * Performance: SLOWER than w8a8_linear on every DiT shape measured on B200
 * (back to back, e.g. 4096 x 12288 x 3072: 132 us against 114 us; the long-K
 * 9216 x 3072 x 12288: 313 against 289): only the GEMM's 8 epilogue warps
 * per CTA can quantize, where the standalone quantizer runs 28 warps per
 * SM.  Kept as the measured alternative placement of the quantizer; use
 * w8a8_linear.
 */
W8A8_API w8a8_status w8a8_linear_fused(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                                       void* out, int8_t* ws_xq, float* ws_scale_a, uint32_t* ws_sync,
                                       int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/* Number of uint32 words of ws_sync for M tokens (M >= 0): ceil(M/128) + 1. */
W8A8_API int64_t w8a8_linear_sync_words(int64_t M);

/*
 * w8a8_linear for callers that cannot allocate device memory (the paper
 * has no counterpart: this is a deployment variant).  Some callers cannot
 * give the layer a workspace and must not make it allocate one: a runtime
 * whose device memory is all pre-reserved by another framework's pool, a
 * latency-critical path where cudaMalloc / cudaFree would synchronize the
 * device, or a plugin interface that passes only inputs and outputs.
 *   Arguments as in w8a8_linear, without ws_xq / ws_scale_a: the quantized
 *   activations and their scales go to one fixed 32 MiB array compiled into
 *   the library (held by every GPU that loads the library until exit).
 * Limit: the int8 codes (M*K bytes, rounded up to 256) plus 4*M bytes of
 * scales must fit in 32 MiB (e.g. 9216 x 3072, 4096 x 8192); larger
 * problems return W8A8_ERR_SCRATCH_LIMIT and launch nothing.  The call
 * allocates nothing (no cudaMalloc / cudaFree).  Its first call on a device
 * looks up the array's device address (cudaGetSymbolAddress, with that
 * device current); make that first call before any stream capture.  All
 * calls share the one array, which keeps the last call's contents: calls
 * that overlap on the GPU (other streams, other host threads) race on it.
 * Nothing in it needs to start at zero.  Results are bit-identical to
 * w8a8_linear.
 */
W8A8_API w8a8_status w8a8_linear_noalloc(const void* x, const int8_t* wq, const float* scale_w, const void* bias,
                                         void* out, int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/*
 * The GEMM without the epilogue: raw int32 accumulators
 *   acc[m,n] = sum_k xq[m,k]*wq[n,k], acc int32 [M, N] (row stride N).
 * The abstract states the int32 accumulation is bit-exact against a library
 * integer matmul; this entry point exposes it for that check.
 */
W8A8_API w8a8_status w8a8_gemm_i32(const int8_t* xq, const int8_t* wq, int32_t* acc,
                          int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/*
 * Per-shape GEMM configuration (abstract: the kernel is "autotuned per GEMM
 * shape"; here a static cost model over a measured table of tile shapes).
 */
typedef struct {
    int32_t block_m;       /* rows of the output tile: 128 (one CTA) or 256 (a CTA pair
                              sharing each MMA through tcgen05 cta_group::2) */
    int32_t block_n;       /* columns of the output tile: 128 or 256 */
    int32_t stages;        /* depth of the shared-memory operand ring */
    int32_t grid;          /* persistent CTAs launched (<= number of SMs; even for pairs) */
    int32_t raster_group;  /* M tiles walked together before moving along N */
    int32_t reserved[3];   /* zero */
} w8a8_gemm_config;

/* The configuration w8a8_gemm would use for this shape on the current
 * device.  Shapes are validated as for w8a8_gemm. */
W8A8_API w8a8_status w8a8_select_config(int64_t M, int64_t N, int64_t K, w8a8_gemm_config* cfg);

/* w8a8_gemm / w8a8_gemm_i32 with an explicit configuration (cfg NULL means
 * the selected one).  block_m 128 or 256, block_n 128 or 256, stages from 2
 * to what shared memory holds (4 at 128 x 256, 6 at 128 x 128 and 256 x 256,
 * 8 at 256 x 128), grid >= 1 (>= 2 for block_m 256), raster_group >= 1;
 * anything else is W8A8_ERR_INVALID_ARG.  For sweeps and tests: every valid
 * configuration computes the same result. */
W8A8_API w8a8_status w8a8_gemm_ex(const int8_t* xq, const int8_t* wq, const float* scale_a,
                         const float* scale_w, const void* bias, void* out,
                         int64_t M, int64_t N, int64_t K, const w8a8_gemm_config* cfg,
                         w8a8_stream_t stream);
W8A8_API w8a8_status w8a8_gemm_i32_ex(const int8_t* xq, const int8_t* wq, int32_t* acc,
                             int64_t M, int64_t N, int64_t K, const w8a8_gemm_config* cfg,
                             w8a8_stream_t stream);

/*
 * FP8 variant: OCP E4M3 codes in place of int8.  The paper measures its
 * int8 kernel against FP8 (abstract: the native FP8 path of datacenter
 * Blackwell is the comparison baseline); this is that path, with the same
 * per-token x per-channel scheme and 448 (the largest finite E4M3 value) in
 * place of 127:
 *
 *   scale_a[m] = fl32(max_k |x[m,k]| / 448)
 *   xq[m,k]    = e4m3_rne(clamp(fl32(x[m,k] / scale_a[m]), -448, 448))
 *                (0 for a row whose scale is 0; -0 keeps its sign, code 0x80)
 *   acc[m,n]   = sum_k e4m3(xq[m,k]) * e4m3(wq[n,k])    fp32, tensor cores
 *   out[m,n]   = bf16_rne((acc[m,n] * scale_a[m]) * scale_w[n] + bias[n])
 *
 * (the pages give no FP8 recipe: this reading is the library's definition).
 * Codes are bytes (uint8_t) in the E4M3 encoding: 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits, no infinities, 0x7F / 0xFF NaN (never
 * produced).  Quantized codes and scales are bit-exact to the definition.
 * The accumulator: each product of two E4M3 values is exact; the tensor
 * cores add them in fp32 in an order of their own, so acc differs from the
 * exact sum by rounding only (the library's tests bound the difference by
 * K * 2^-23 * sum_k |products|; exact when every partial sum is an fp32
 * value).  Shapes, strides, alignment and errors as for the int8 calls
 * (including 16 <= K <= 133144, K % 16 == 0, N % 8 == 0).
 */
W8A8_API w8a8_status w8a8_quantize_act_fp8(const void* x, int64_t M, int64_t K, int64_t ldx,
                                           uint8_t* xq, int64_t ldxq, float* scale_a, w8a8_stream_t stream);
W8A8_API w8a8_status w8a8_quantize_weight_fp8(const float* w, int64_t N, int64_t K, int64_t ldw,
                                              uint8_t* wq, int64_t ldwq, float* scale_w, w8a8_stream_t stream);

/* The FP8 GEMM with the dequantization + bias epilogue (tcgen05.mma
 * kind::f8f6f4): arguments as in w8a8_gemm, with E4M3 codes. */
W8A8_API w8a8_status w8a8_gemm_fp8(const uint8_t* xq, const uint8_t* wq, const float* scale_a,
                                   const float* scale_w, const void* bias, void* out,
                                   int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/* The FP8 GEMM without the epilogue: fp32 accumulators acc [M, N] (row
 * stride N), for checking the accumulation against an exact sum. */
W8A8_API w8a8_status w8a8_gemm_fp8_f32(const uint8_t* xq, const uint8_t* wq, float* acc,
                                       int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/* The two FP8 GEMMs with an explicit configuration (as w8a8_gemm_ex). */
W8A8_API w8a8_status w8a8_gemm_fp8_ex(const uint8_t* xq, const uint8_t* wq, const float* scale_a,
                                      const float* scale_w, const void* bias, void* out,
                                      int64_t M, int64_t N, int64_t K, const w8a8_gemm_config* cfg,
                                      w8a8_stream_t stream);
W8A8_API w8a8_status w8a8_gemm_fp8_f32_ex(const uint8_t* xq, const uint8_t* wq, float* acc,
                                          int64_t M, int64_t N, int64_t K, const w8a8_gemm_config* cfg,
                                          w8a8_stream_t stream);

/* The whole FP8 linear layer: w8a8_quantize_act_fp8 into the caller's
 * workspace (ws_xq uint8 [M, K], ws_scale_a fp32 [M]), then w8a8_gemm_fp8.
 * Arguments as in w8a8_linear. */
W8A8_API w8a8_status w8a8_linear_fp8(const void* x, const uint8_t* wq, const float* scale_w, const void* bias,
                                     void* out, uint8_t* ws_xq, float* ws_scale_a,
                                     int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/*
 * GELU before a linear layer, fused with its quantizer (the per-token
 * quantizer moved into the producer of X: a DiT MLP's GELU sits between the
 * up- and down-projections).  Unfused, a GELU kernel writes bf16 G =
 * GELU(H) to HBM and the quantizer reads it back; fused, one pass reads H and
 * writes the codes, saving a write and a read of G.  GELU is the tanh form
 * (Hendrycks & Gimpel, "Gaussian Error Linear Units"),
 *   gelu(h) = 0.5 h (1 + tanh(u)),  u = sqrt(2/pi) * (h + 0.044715 h^3),
 * evaluated in binary64 as h / (1 + exp(-2u)) (the same function, without
 * the cancellation of 1 + tanh(u) for negative h) and rounded once to bf16:
 * exactly what w8a8_gelu stores.  That is the correctly rounded bf16 value
 * of gelu(h) for every bf16 input except the 256 of magnitude below 2^-125
 * with an odd last bit, where gelu(h) = h/2 + O(h^2) lies within 1e-40
 * (relative) of a bf16 midpoint: there the result is bf16_rne(h/2).  The
 * pages name no activation; this is the library's definition.
 *
 * w8a8_quantize_act_gelu: codes and scales of bf16_rne(gelu(h)); arguments
 *   as w8a8_quantize_act (h in place of x).  Bit-identical to w8a8_gelu
 *   followed by w8a8_quantize_act.
 * w8a8_gelu: g = bf16_rne(gelu(h)), h and g bf16 [M, K] with row strides
 *   ldh, ldg (multiples of 8 elements), K % 8 == 0.
 * w8a8_linear_gelu: out = GELU(h) W^T + b through w8a8_quantize_act_gelu
 *   and w8a8_gemm; arguments as w8a8_linear.
 *
 * Resources.  w8a8_gelu, and w8a8_quantize_act_gelu on rows of up to 16384
 * elements, look GELU up in a table of all 65536 bf16 inputs that each
 * launch builds in shared memory (128 KB per CTA, one CTA per SM) with the
 * same binary64 arithmetic; they launch as thread-block clusters of 2 to 8
 * CTAs, which share the work of building the table.  The cluster size comes from
 * an occupancy query, made once per device by the first call whose stream
 * is not being captured and kept for the process; calls recorded in a stream
 * capture before that use clusters of 2 and do not keep them (same
 * results).  Longer rows evaluate GELU per element.  A failed cluster
 * launch returns W8A8_ERR_LAUNCH.
 */
W8A8_API w8a8_status w8a8_quantize_act_gelu(const void* h, int64_t M, int64_t K, int64_t ldh,
                                            int8_t* xq, int64_t ldxq, float* scale_a, w8a8_stream_t stream);
W8A8_API w8a8_status w8a8_gelu(const void* h, int64_t M, int64_t K, int64_t ldh, void* g, int64_t ldg,
                               w8a8_stream_t stream);
W8A8_API w8a8_status w8a8_linear_gelu(const void* h, const int8_t* wq, const float* scale_w, const void* bias,
                                      void* out, int8_t* ws_xq, float* ws_scale_a,
                                      int64_t M, int64_t N, int64_t K, w8a8_stream_t stream);

/*
 * A chain of W8A8 linear layers as one CUDA graph (the paper drops its
 * kernel into every linear layer of the DiT, abstract; a DiT block runs
 * four: attention QKV, attention output, MLP up, MLP down).  Each layer is
 * the w8a8_linear call (activation quantizer, then the GEMM as its
 * programmatic dependent); w8a8_chain_create records all of them once, in
 * order, into a CUDA graph, and w8a8_chain_launch replays it with one graph
 * launch instead of two kernel launches per layer.
 *
 * A layer's x may be an earlier layer's out (the same buffer, [M, K] with K
 * the earlier layer's N): the graph keeps the call order, so the later
 * quantizer reads the finished output.  All pointers are the caller's
 * device memory, as for w8a8_linear, and must stay valid, with the same
 * shapes, for the chain's lifetime: the graph holds the addresses, not
 * copies.  The chain holds no device memory.  Calls that launch the same
 * chain (or chains sharing buffers) must not overlap on the GPU.
 */
/* Element-wise step a chain layer applies to its input before quantizing
 * it (see w8a8_linear_gelu). */
enum { W8A8_ACT_NONE = 0, W8A8_ACT_GELU = 1 };

typedef struct {
    const void* x;            /* bf16 [M, K] input (row stride K) */
    const int8_t* wq;         /* int8 [N, K] weight codes */
    const float* scale_w;     /* fp32 [N] */
    const void* bias;         /* bf16 [N] or NULL */
    void* out;                /* bf16 [M, N] output (row stride N) */
    int8_t* ws_xq;            /* int8 [M, K] workspace */
    float* ws_scale_a;        /* fp32 [M] workspace */
    int64_t M, N, K;
    int32_t input_act;        /* W8A8_ACT_NONE, or W8A8_ACT_GELU: the layer computes GELU(x) W^T + b */
    int32_t reserved;         /* zero */
} w8a8_linear_desc;

typedef struct w8a8_chain_st* w8a8_chain_t;

/* Validates every layer as w8a8_linear does (errors as for w8a8_linear,
 * returned before any CUDA call; count must be 1..4096), then records the
 * chain on the current device (layers with input_act = W8A8_ACT_GELU have
 * their table kernel's cluster geometry set up first, outside the capture).
 * On success *chain is the new chain; on failure *chain is NULL and nothing
 * stays allocated. */
W8A8_API w8a8_status w8a8_chain_create(const w8a8_linear_desc* layers, int32_t count, w8a8_chain_t* chain);

/* Enqueues the whole chain on `stream` (asynchronous, one graph launch).
 * The current device must be the one the chain was created on. */
W8A8_API w8a8_status w8a8_chain_launch(w8a8_chain_t chain, w8a8_stream_t stream);

/* Number of layers of the chain (0 for NULL). */
W8A8_API int32_t w8a8_chain_layers(w8a8_chain_t chain);

/* Frees the chain's graph (NULL is a no-op).  No launch of it may still be
 * running on the GPU. */
W8A8_API w8a8_status w8a8_chain_destroy(w8a8_chain_t chain);

/*
 * Every wait inside the library's kernels is bounded in time.  When one
 * runs out the kernel records a nonzero code in a device-side error word,
 * finishes its own in-flight copies, frees its tensor memory and exits, so
 * the CUDA context stays usable and the output is incomplete.
 * w8a8_read_device_error synchronizes the current device, stores the word
 * in *code (0 = no timeout since the last clear), clears it if `clear` is
 * nonzero, and returns W8A8_ERR_TIMEOUT if the word was nonzero.
 */
W8A8_API w8a8_status w8a8_read_device_error(int32_t* code, int32_t clear);

/* Time limit of every bounded wait, in nanoseconds (default 2e9; values
 * below 1e5 are raised to 1e5).  Applies to launches made after the call. */
W8A8_API w8a8_status w8a8_set_wait_timeout_ns(int64_t ns);

/*
 * Self-test of the timeout path: launches one small kernel that waits on a
 * barrier nothing ever completes, with the given limit (>= 1e5 ns), so that
 * the wait runs out by construction and the error word is set.  No other
 * state is touched.  Used to check failure detection without any fault.
 */
W8A8_API w8a8_status w8a8_selftest_wait_timeout(int64_t timeout_ns, w8a8_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H */
