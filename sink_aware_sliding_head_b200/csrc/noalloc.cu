// noalloc.cu - flint_attn_bwd_preprocess_static: the backward preprocess
// (D = rowsum(dO * O) and the sink-logit gradient) without any workspace from
// the caller and without allocating.
//
// Who needs it: code that must not allocate device memory at the point where
// it runs - a step inside a serving loop that has a fixed memory budget and no
// allocator of its own, a plugin interface that hands over tensors but no
// workspace, or a latency-critical path where cudaMalloc/cudaFree would
// synchronise the device. Such callers pass only their inputs and outputs.
//
// The only scratch the preprocess needs is one row of per-head partial sums per
// block of the launch. Here it lives in a file-scope __device__ array of fixed
// size, which every GPU that loads this library keeps until the process exits:
// kStaticPartRows x kStaticMaxHeads floats (1184 x 128 x 4 B = 592 KiB).
//
// Rules for callers:
//  * num_q_heads must not exceed FLINT_STATIC_MAX_HEADS (128); larger calls
//    return FLINT_ERR_WORKSPACE before any launch.
//  * All calls on a device share the one array. Every call writes each partial
//    row it later reads (nothing has to start at zero), but two calls whose
//    kernels overlap on the GPU (different streams, no ordering between them)
//    race on it. Order such calls on one stream or with events.
//  * The first call on a device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current and caches it. Make that
//    first call before any stream capture begins on that device. The cached
//    address belongs to the device's primary context: after cudaDeviceReset
//    (or any reset of that context) this library must not be called again on
//    that device in the same process.
#include "common.cuh"

namespace flint {

namespace {

constexpr int kStaticMaxHeads = FLINT_STATIC_MAX_HEADS;
constexpr int kStaticPartRows = kPartBlocks;   // the preprocess launch never uses more rows

// In host code this name is only a stand-in for the symbol, not a device
// address: the address is obtained with cudaGetSymbolAddress below.
static __device__ __align__(256) float g_bwd_pre_partials[kStaticPartRows * kStaticMaxHeads];

PerDeviceOnce g_lookup;
float* g_addr[kMaxDevices] = {};   // written once per device under g_lookup

// Device address of g_bwd_pre_partials on the current device (looked up once).
cudaError_t scratch_on_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  e = static_cast<cudaError_t>(g_lookup.run(dev, [&] {
    void* p = nullptr;
    const cudaError_t r = cudaGetSymbolAddress(&p, g_bwd_pre_partials);
    if (r == cudaSuccess) g_addr[dev] = static_cast<float*>(p);
    return r;
  }));
  if (e != cudaSuccess) return e;
  *out = g_addr[dev];
  return cudaSuccess;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace flint

using namespace flint;

extern "C" flint_status_t flint_attn_bwd_preprocess_static(const flint_attn_params_t* params,
                                                           const void* out, const void* dout,
                                                           const float* lse, const float* sink,
                                                           float* d_rowsum, float* dsink,
                                                           void* stream) {
  if (!params) return FLINT_ERR_INVALID_ARG;
  if (params->dtype != FLINT_BF16 && params->dtype != FLINT_FP32) return FLINT_ERR_INVALID_ARG;
  if (params->compute_f16 && params->dtype != FLINT_FP32) return FLINT_ERR_INVALID_ARG;
  if (params->total_tokens < 0 || params->num_q_heads < 1 || params->head_dim != kHeadDim)
    return params->head_dim != kHeadDim ? FLINT_ERR_UNSUPPORTED : FLINT_ERR_INVALID_ARG;
  if ((long long)params->total_tokens * params->num_q_heads * kHeadDim > 0x7fffffffLL)
    return FLINT_ERR_INVALID_ARG;
  if (params->num_q_heads > kStaticMaxHeads) return FLINT_ERR_WORKSPACE;
  // With no tokens the [T, ...] tensors (out, dout, lse, d_rowsum) are empty and may be null.
  const bool no_tokens = params->total_tokens == 0;
  if ((!no_tokens && (!out || !dout || !lse || !d_rowsum)) || !aligned16(out) ||
      !aligned16(dout) || !aligned4(lse) || !aligned4(d_rowsum))
    return FLINT_ERR_INVALID_ARG;
  if (!sink || !dsink || !aligned4(sink) || !aligned4(dsink)) return FLINT_ERR_INVALID_ARG;
  // The same type rules as flint_attn_bwd: out is float32 with fp32_out (always
  // for FP32 inputs), IEEE fp16 for FP32 inputs with compute_f16 and without
  // fp32_out, else the input type.
  Resolved p{};
  p.T = params->total_tokens;
  p.N = params->num_docs > 0 ? params->num_docs : 1;
  p.H = params->num_q_heads;
  p.Hk = params->num_kv_heads > 0 ? params->num_kv_heads : 1;
  p.D = kHeadDim;
  p.dtype = params->dtype;
  p.fp32_out = (params->fp32_out != 0 || params->dtype == FLINT_FP32) ? 1 : 0;
  p.tc = (params->dtype == FLINT_BF16 || params->compute_f16) ? 1 : 0;
  p.out_f16 = (params->compute_f16 && !params->fp32_out) ? 1 : 0;
  float* scratch = nullptr;
  if (scratch_on_current_device(&scratch) != cudaSuccess) return FLINT_ERR_CUDA;
  cudaError_t e = launch_bwd_preprocess(p, out, dout, lse, sink, d_rowsum, scratch, dsink,
                                        nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FLINT_OK : FLINT_ERR_CUDA;
}
