// padding.cu - rows of trailing padding, for flint_attn_fwd_padded /
// flint_attn_bwd_padded.
//
// Padded queries and keys are excluded while the sink stays valid (attention
// utils page, nemo_automodel.components.attention.utils: the BSHD
// attention_mask, with trailing padding as TE takes it; Flint layers page,
// FlintAttention.forward: the sink is a softmax category with a zero value
// vector, so it stays in every row). A padded query sees no
// key, so its row is the sink alone: O = 0, LSE = sink_h. Nothing downstream
// depends on a padded token, so its gradients are zero. The work lists give
// padded tokens no item, so the attention kernels never write these rows; the
// kernels here do, one block per token.
#include "common.cuh"

namespace flint {

namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ bool is_padding(const int32_t* cu, const int32_t* valid, int N,
                                           int t) {
  const int d = doc_of(cu, N, t);
  const int start = __ldg(cu + d), len = __ldg(cu + d + 1) - start;
  return t - start >= max(0, min(__ldg(valid + d), len));
}

__global__ void __launch_bounds__(kThreads)
pad_fill_fwd_kernel(int T, int N, int H, const int32_t* __restrict__ cu,
                    const int32_t* __restrict__ valid, const float* __restrict__ sink,
                    void* __restrict__ out, int out_f32, float* __restrict__ lse) {
  const int t = blockIdx.x;
  if (!is_padding(cu, valid, N, t)) return;
  const size_t row = (size_t)t * H * kHeadDim;
  if (out_f32) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + row);
    for (int e = threadIdx.x; e < H * kHeadDim / 4; e += kThreads) o[e] = make_float4(0, 0, 0, 0);
  } else {
    uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + row);
    for (int e = threadIdx.x; e < H * kHeadDim / 8; e += kThreads) o[e] = make_uint4(0, 0, 0, 0);
  }
  for (int h = threadIdx.x; h < H; h += kThreads) lse[(size_t)h * T + t] = __ldg(sink + h);
}

__global__ void __launch_bounds__(kThreads)
pad_fill_bwd_kernel(int N, int H, int Hk, const int32_t* __restrict__ cu,
                    const int32_t* __restrict__ valid, float* __restrict__ dq_acc,
                    float* __restrict__ dk_acc, void* __restrict__ dv, int dv_f32) {
  const int t = blockIdx.x;
  if (!is_padding(cu, valid, N, t)) return;
  const float4 z = make_float4(0, 0, 0, 0);
  float4* q = reinterpret_cast<float4*>(dq_acc + (size_t)t * H * kHeadDim);
  for (int e = threadIdx.x; e < H * kHeadDim / 4; e += kThreads) q[e] = z;
  float4* k = reinterpret_cast<float4*>(dk_acc + (size_t)t * Hk * kHeadDim);
  for (int e = threadIdx.x; e < Hk * kHeadDim / 4; e += kThreads) k[e] = z;
  const size_t vrow = (size_t)t * Hk * kHeadDim;
  if (dv_f32) {
    float4* v = reinterpret_cast<float4*>(static_cast<float*>(dv) + vrow);
    for (int e = threadIdx.x; e < Hk * kHeadDim / 4; e += kThreads) v[e] = z;
  } else {
    uint4* v = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dv) + vrow);
    for (int e = threadIdx.x; e < Hk * kHeadDim / 8; e += kThreads) v[e] = make_uint4(0, 0, 0, 0);
  }
}

}  // namespace

cudaError_t launch_pad_fill_fwd(const Resolved& p, const int32_t* cu, const int32_t* valid,
                                const float* sink, void* out, float* lse, cudaStream_t st) {
  if (p.T == 0) return cudaSuccess;
  ProfScope prof(kKPadFill, st);
  const int out_f32 = p.fp32_out && !p.out_f16;   // else a 2-byte type (zeros alike)
  pad_fill_fwd_kernel<<<p.T, kThreads, 0, st>>>(p.T, p.N, p.H, cu, valid, sink, out, out_f32,
                                                lse);
  return cudaGetLastError();
}

cudaError_t launch_pad_fill_bwd(const Resolved& p, const int32_t* cu, const int32_t* valid,
                                float* dq_acc, float* dk_acc, void* dv, int dv_f32,
                                cudaStream_t st) {
  if (p.T == 0) return cudaSuccess;
  ProfScope prof(kKPadFill, st);
  pad_fill_bwd_kernel<<<p.T, kThreads, 0, st>>>(p.N, p.H, p.Hk, cu, valid, dq_acc, dk_acc, dv,
                                                dv_f32);
  return cudaGetLastError();
}

}  // namespace flint
