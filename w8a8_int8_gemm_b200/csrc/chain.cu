// chain.cu -- a sequence of W8A8 linear layers as one CUDA graph.
//
// The paper ("Realizing Native INT8 Compute for Diffusion Transformers on
// Consumer GPUs", abstract) drops its kernel into every linear layer of the
// DiT and reports whole-image times at 768px and 1024px.  A DiT block runs
// four linear layers per token batch (attention QKV, attention output, MLP
// up, MLP down), each one activation quantizer and one GEMM here: eight
// kernel launches per block, short enough (the smallest, the quantizer, is
// ~10 us) that host launch cost shows.  This runner records the layers once
// into a CUDA graph (stream capture of w8a8_linear, so each GEMM keeps its
// programmatic overlap with its quantizer) and replays it with one launch.
//
// A layer's input may be an earlier layer's output (same buffer): the
// graph keeps the stream order of the calls, so the later quantizer reads
// the finished output.  A layer may apply GELU to its input on the way into
// its quantizer (the producer of the input fused with the quantizer).  The
// runner owns no device memory: every buffer is the caller's and must
// outlive the chain.
#include <cuda_runtime.h>

#include <cstdint>
#include <new>

#include "../../include/w8a8.h"
#include "internal.h"

struct w8a8_chain_st {
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  int device = -1;
  int32_t layers = 0;
};

namespace {

// The checks w8a8_linear makes, before any CUDA call, and the layer's input step.
w8a8_status check_layer(const w8a8_linear_desc& l) {
  if (l.input_act != W8A8_ACT_NONE && l.input_act != W8A8_ACT_GELU) return W8A8_ERR_INVALID_ARG;
  return w8a8::check_linear_call(l.x, l.wq, l.scale_w, l.bias, l.out, l.ws_xq, l.ws_scale_a, l.M, l.N, l.K);
}

}  // namespace

extern "C" {

w8a8_status w8a8_chain_create(const w8a8_linear_desc* layers, int32_t count, w8a8_chain_t* chain) {
  if (chain == nullptr) return W8A8_ERR_INVALID_ARG;
  *chain = nullptr;
  if (layers == nullptr || count < 1 || count > 4096) return W8A8_ERR_INVALID_ARG;
  for (int32_t i = 0; i < count; ++i) {
    const w8a8_status st = check_layer(layers[i]);
    if (st != W8A8_OK) return st;
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    return W8A8_ERR_CUDA;
  }
  if (major != 10 || minor != 0) return W8A8_ERR_UNSUPPORTED_DEVICE;

  cudaStream_t s = nullptr;
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return W8A8_ERR_CUDA;
  for (int32_t i = 0; i < count; ++i) {
    if (layers[i].input_act == W8A8_ACT_GELU && layers[i].M > 0 && layers[i].N > 0 &&
        w8a8::prepare_quantize_act_gelu(layers[i].K, s) != cudaSuccess) {
      cudaStreamDestroy(s);
      return W8A8_ERR_CUDA;
    }
  }
  w8a8_status st = W8A8_OK;
  cudaGraph_t graph = nullptr;
  if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaStreamDestroy(s);
    return W8A8_ERR_CUDA;
  }
  for (int32_t i = 0; i < count && st == W8A8_OK; ++i) {
    const w8a8_linear_desc& l = layers[i];
    auto linear = l.input_act == W8A8_ACT_GELU ? w8a8_linear_gelu : w8a8_linear;
    st = linear(l.x, l.wq, l.scale_w, l.bias, l.out, l.ws_xq, l.ws_scale_a, l.M, l.N, l.K,
                reinterpret_cast<w8a8_stream_t>(s));
  }
  // Capture always ends, also after a failed layer (the partial graph is dropped).
  const cudaError_t ec = cudaStreamEndCapture(s, &graph);
  cudaStreamDestroy(s);
  if (st == W8A8_OK && (ec != cudaSuccess || graph == nullptr)) st = W8A8_ERR_CUDA;
  if (st != W8A8_OK) {
    if (graph != nullptr) cudaGraphDestroy(graph);
    return st;
  }
  cudaGraphExec_t exec = nullptr;
  if (cudaGraphInstantiateWithFlags(&exec, graph, 0) != cudaSuccess) {
    cudaGraphDestroy(graph);
    return W8A8_ERR_CUDA;
  }
  w8a8_chain_st* c = new (std::nothrow) w8a8_chain_st;
  if (c == nullptr) {
    cudaGraphExecDestroy(exec);
    cudaGraphDestroy(graph);
    return W8A8_ERR_CUDA;
  }
  c->graph = graph;
  c->exec = exec;
  c->device = dev;
  c->layers = count;
  *chain = c;
  return W8A8_OK;
}

w8a8_status w8a8_chain_launch(w8a8_chain_t chain, w8a8_stream_t stream) {
  if (chain == nullptr || chain->exec == nullptr) return W8A8_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_CUDA;
  if (dev != chain->device) return W8A8_ERR_INVALID_ARG;
  return cudaGraphLaunch(chain->exec, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? W8A8_OK
                                                                                              : W8A8_ERR_LAUNCH;
}

int32_t w8a8_chain_layers(w8a8_chain_t chain) { return chain == nullptr ? 0 : chain->layers; }

w8a8_status w8a8_chain_destroy(w8a8_chain_t chain) {
  if (chain == nullptr) return W8A8_OK;
  w8a8_status st = W8A8_OK;
  if (chain->exec != nullptr && cudaGraphExecDestroy(chain->exec) != cudaSuccess) st = W8A8_ERR_CUDA;
  if (chain->graph != nullptr && cudaGraphDestroy(chain->graph) != cudaSuccess) st = W8A8_ERR_CUDA;
  delete chain;
  return st;
}

}  // extern "C"
