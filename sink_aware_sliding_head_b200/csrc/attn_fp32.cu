// attn_fp32.cu - sink-aware attention in FP32 on CUDA cores, for FP32 inputs
// whose group size G has no tensor-core tile (G not 1, 2, 4, 8 or 16; the others
// take the split tensor-core path of attn_x3_sm100.cu): plain FP32 FMA with
// online softmax.
//
// Definition (Flint layers page, nemo_automodel.components.models.flint.layers,
// FlintAttention.forward and _FlintSinkParameters.forward): for query row
// (t, h) of document [d0, d1), visible keys j satisfy d0 <= j <= t and
// (W <= 0 or t - j < W) (window counting the current token, FlintConfig
// docstring); z_tj = scale * q_hat . k_hat; the sink logit s_h, not scaled, joins
// the softmax denominator with a zero value.
//   forward : running max starts at s_h and the running sum at 1 (the sink's
//             own weight), then O = acc / l, LSE = m + ln l.
//   backward: p = exp(z - LSE), dp = dO . v, ds = p (dp - D) with
//             D = rowsum(dO * O); dq_hat += scale ds k_hat, dk_hat += scale ds
//             q_hat, dv += p dO.
// Each block works on 32 rows (query rows of one head, or key rows of one KV
// head) with 4 threads per row, each owning 32 of the 128 channels; the other
// operand streams through shared memory in chunks of 32 rows.
#include "common.cuh"

namespace flint {

namespace {

constexpr int kRows = 32;
constexpr int kThreads = kRows * 4;
constexpr int kChunk = 32;
constexpr int kSub = kHeadDim / 4;   // channels per thread
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// grid: (ceil(T / 32), H)
__global__ void __launch_bounds__(kThreads)
fwd_fp32_kernel(const float* __restrict__ qh, const float* __restrict__ kh,
                const float* __restrict__ v, const float* __restrict__ sink,
                const int32_t* __restrict__ cu, int N, int T, int H, int Hk, int W, float scale,
                float* __restrict__ out, float* __restrict__ lse) {
  __shared__ float ks[kChunk][kHeadDim];
  __shared__ float vs[kChunk][kHeadDim];
  const int h = blockIdx.y, g = h / (H / Hk);
  const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int tb = blockIdx.x * kRows;
  const int t = tb + row;
  const bool valid = t < T;
  const int tt = valid ? t : T - 1;
  const int d0 = __ldg(cu + doc_of(cu, N, tt));
  const int lo = W > 0 ? max(d0, tt - W + 1) : d0;
  // block key range: the first row has the smallest lo, the last row the largest t
  const int tb_c = min(tb, T - 1);
  const int d0b = __ldg(cu + doc_of(cu, N, tb_c));
  const int kmin = W > 0 ? max(d0b, tb_c - W + 1) : d0b;
  const int kmax = min(tb + kRows, T) - 1;

  float q[kSub], acc[kSub];
  const float* qrow = qh + ((size_t)tt * H + h) * kHeadDim + part * kSub;
#pragma unroll
  for (int c = 0; c < kSub; ++c) { q[c] = qrow[c]; acc[c] = 0.f; }
  const float sc2 = scale * kLog2e;
  float m = sink[h] * kLog2e;       // running max (log2 units) starts at the sink
  float l = 1.f;                    // the sink's own weight 2^(m - m)
  if (m == -INFINITY) l = 0.f;

  for (int kc = kmin; kc <= kmax; kc += kChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kHeadDim / 4; e += kThreads) {
      const int r = e / (kHeadDim / 4), c4 = (e % (kHeadDim / 4)) * 4;
      const int j = kc + r;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (j < T) {
        a = *reinterpret_cast<const float4*>(kh + ((size_t)j * Hk + g) * kHeadDim + c4);
        b = *reinterpret_cast<const float4*>(v + ((size_t)j * Hk + g) * kHeadDim + c4);
      }
      *reinterpret_cast<float4*>(&ks[r][c4]) = a;
      *reinterpret_cast<float4*>(&vs[r][c4]) = b;
    }
    __syncthreads();
    const int nk = min(kChunk, kmax - kc + 1);
    for (int r = 0; r < nk; ++r) {
      const int j = kc + r;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < kSub; ++c) dot = fmaf(q[c], ks[r][part * kSub + c], dot);
      dot = quad_sum(dot);
      if (j < lo || j > tt) continue;        // uniform within the quad
      const float z = dot * sc2;
      if (z > m) {
        const float alpha = exp2f(m - z);
        l = l * alpha + 1.f;
#pragma unroll
        for (int c = 0; c < kSub; ++c) acc[c] = fmaf(acc[c], alpha, vs[r][part * kSub + c]);
        m = z;
      } else {
        const float p = exp2f(z - m);
        l += p;
#pragma unroll
        for (int c = 0; c < kSub; ++c) acc[c] = fmaf(p, vs[r][part * kSub + c], acc[c]);
      }
    }
  }
  if (valid) {
    const float inv = 1.f / l;
    float* orow = out + ((size_t)t * H + h) * kHeadDim + part * kSub;
#pragma unroll
    for (int c = 0; c < kSub; ++c) orow[c] = acc[c] * inv;
    if (part == 0) lse[(size_t)h * T + t] = (m + log2f(l)) * kLn2;
  }
}

// dq_hat for query rows. grid: (ceil(T / 32), H)
__global__ void __launch_bounds__(kThreads)
bwd_dq_fp32_kernel(const float* __restrict__ qh, const float* __restrict__ kh,
                   const float* __restrict__ v, const float* __restrict__ dout,
                   const float* __restrict__ lse, const float* __restrict__ dvec,
                   const int32_t* __restrict__ cu, int N, int T, int H, int Hk, int W,
                   float scale, float* __restrict__ dq_acc) {
  __shared__ float ks[kChunk][kHeadDim];
  __shared__ float vs[kChunk][kHeadDim];
  const int h = blockIdx.y, g = h / (H / Hk);
  const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int tb = blockIdx.x * kRows;
  const int t = tb + row;
  const bool valid = t < T;
  const int tt = valid ? t : T - 1;
  const int d0 = __ldg(cu + doc_of(cu, N, tt));
  const int lo = W > 0 ? max(d0, tt - W + 1) : d0;
  const int tb_c = min(tb, T - 1);
  const int d0b = __ldg(cu + doc_of(cu, N, tb_c));
  const int kmin = W > 0 ? max(d0b, tb_c - W + 1) : d0b;
  const int kmax = min(tb + kRows, T) - 1;

  float q[kSub], go[kSub], dq[kSub];
  const size_t rb = ((size_t)tt * H + h) * kHeadDim + part * kSub;
#pragma unroll
  for (int c = 0; c < kSub; ++c) { q[c] = qh[rb + c]; go[c] = dout[rb + c]; dq[c] = 0.f; }
  const float sc2 = scale * kLog2e;
  const float lse2 = lse[(size_t)h * T + tt] * kLog2e;
  const float Di = dvec[(size_t)h * T + tt];

  for (int kc = kmin; kc <= kmax; kc += kChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kHeadDim / 4; e += kThreads) {
      const int r = e / (kHeadDim / 4), c4 = (e % (kHeadDim / 4)) * 4;
      const int j = kc + r;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (j < T) {
        a = *reinterpret_cast<const float4*>(kh + ((size_t)j * Hk + g) * kHeadDim + c4);
        b = *reinterpret_cast<const float4*>(v + ((size_t)j * Hk + g) * kHeadDim + c4);
      }
      *reinterpret_cast<float4*>(&ks[r][c4]) = a;
      *reinterpret_cast<float4*>(&vs[r][c4]) = b;
    }
    __syncthreads();
    const int nk = min(kChunk, kmax - kc + 1);
    for (int r = 0; r < nk; ++r) {
      const int j = kc + r;
      float dot = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < kSub; ++c) {
        dot = fmaf(q[c], ks[r][part * kSub + c], dot);
        dp = fmaf(go[c], vs[r][part * kSub + c], dp);
      }
      dot = quad_sum(dot);
      dp = quad_sum(dp);
      if (j < lo || j > tt) continue;
      const float p = exp2f(dot * sc2 - lse2);
      const float ds = p * (dp - Di) * scale;
#pragma unroll
      for (int c = 0; c < kSub; ++c) dq[c] = fmaf(ds, ks[r][part * kSub + c], dq[c]);
    }
  }
  if (valid) {
#pragma unroll
    for (int c = 0; c < kSub; ++c) dq_acc[rb + c] = dq[c];
  }
}

// dk_hat and dv for key rows of one KV head, summed over the G query heads.
// grid: (ceil(T / 32), Hk). Query rows stream through shared memory in chunks
// of kChunk (token, head) pairs.
__global__ void __launch_bounds__(kThreads)
bwd_dkv_fp32_kernel(const float* __restrict__ qh, const float* __restrict__ kh,
                    const float* __restrict__ v, const float* __restrict__ dout,
                    const float* __restrict__ lse, const float* __restrict__ dvec,
                    const int32_t* __restrict__ cu, int N, int T, int H, int Hk, int W,
                    float scale, float* __restrict__ dk_acc, float* __restrict__ dv_out) {
  __shared__ float qs[kChunk][kHeadDim];
  __shared__ float os[kChunk][kHeadDim];
  __shared__ float ls[kChunk], dsv[kChunk];
  __shared__ int qend_s[kRows];
  const int g = blockIdx.y, G = H / Hk;
  const int row = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int jb = blockIdx.x * kRows;
  const int j = jb + row;
  const bool valid = j < T;
  const int jj = valid ? j : T - 1;
  const int d1 = __ldg(cu + doc_of(cu, N, jj) + 1);
  // queries that see key j: j <= i < qend
  const int qend = W > 0 ? min(d1, jj + W) : d1;
  if (part == 0) qend_s[row] = valid ? qend : 0;
  __syncthreads();
  int qmax = 0;
  for (int r = 0; r < kRows; ++r) qmax = max(qmax, qend_s[r]);
  const int qmin = min(jb, T - 1);

  float k[kSub], vv[kSub], dk[kSub], dv[kSub];
  const size_t rb = ((size_t)jj * Hk + g) * kHeadDim + part * kSub;
#pragma unroll
  for (int c = 0; c < kSub; ++c) { k[c] = kh[rb + c]; vv[c] = v[rb + c]; dk[c] = 0.f; dv[c] = 0.f; }
  const float sc2 = scale * kLog2e;
  const int rows_total = (qmax - qmin) * G;   // (token, head) pairs, token-major

  for (int qc = 0; qc < rows_total; qc += kChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * kHeadDim / 4; e += kThreads) {
      const int r = e / (kHeadDim / 4), c4 = (e % (kHeadDim / 4)) * 4;
      const int f = qc + r;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (f < rows_total) {
        const int i = qmin + f / G, h = g * G + f % G;
        a = *reinterpret_cast<const float4*>(qh + ((size_t)i * H + h) * kHeadDim + c4);
        b = *reinterpret_cast<const float4*>(dout + ((size_t)i * H + h) * kHeadDim + c4);
      }
      *reinterpret_cast<float4*>(&qs[r][c4]) = a;
      *reinterpret_cast<float4*>(&os[r][c4]) = b;
    }
    if (threadIdx.x < kChunk) {
      const int f = qc + threadIdx.x;
      float a = 0.f, b = 0.f;
      if (f < rows_total) {
        const int i = qmin + f / G, h = g * G + f % G;
        a = lse[(size_t)h * T + i] * kLog2e;
        b = dvec[(size_t)h * T + i];
      }
      ls[threadIdx.x] = a;
      dsv[threadIdx.x] = b;
    }
    __syncthreads();
    const int nr = min(kChunk, rows_total - qc);
    for (int r = 0; r < nr; ++r) {
      const int i = qmin + (qc + r) / G;
      float dot = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < kSub; ++c) {
        dot = fmaf(qs[r][part * kSub + c], k[c], dot);
        dp = fmaf(os[r][part * kSub + c], vv[c], dp);
      }
      dot = quad_sum(dot);
      dp = quad_sum(dp);
      if (!valid || i < jj || i >= qend) continue;
      const float p = exp2f(dot * sc2 - ls[r]);
      const float ds = p * (dp - dsv[r]) * scale;
#pragma unroll
      for (int c = 0; c < kSub; ++c) {
        dv[c] = fmaf(p, os[r][part * kSub + c], dv[c]);
        dk[c] = fmaf(ds, qs[r][part * kSub + c], dk[c]);
      }
    }
  }
  if (valid) {
#pragma unroll
    for (int c = 0; c < kSub; ++c) { dk_acc[rb + c] = dk[c]; dv_out[rb + c] = dv[c]; }
  }
}

}  // namespace

cudaError_t launch_attn_fwd_fp32(const Resolved& p, const float* qh, const float* kh,
                                 const float* v, const float* sink, const int32_t* cu, float* out,
                                 float* lse, cudaStream_t st) {
  if (p.T == 0) return cudaSuccess;
  dim3 grid((p.T + kRows - 1) / kRows, p.H);
  ProfScope prof(kKFwdFp32, st);
  fwd_fp32_kernel<<<grid, kThreads, 0, st>>>(qh, kh, v, sink, cu, p.N, p.T, p.H, p.Hk, p.W,
                                             p.scale, out, lse);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_fp32(const Resolved& p, const float* qh, const float* kh,
                                 const float* v, const float* dout, const float* lse,
                                 const float* dvec, const int32_t* cu, float* dq_acc,
                                 float* dk_acc, float* dv, cudaStream_t st) {
  if (p.T == 0) return cudaSuccess;
  dim3 gq((p.T + kRows - 1) / kRows, p.H);
  {
    ProfScope prof(kKBwdDqFp32, st);
    bwd_dq_fp32_kernel<<<gq, kThreads, 0, st>>>(qh, kh, v, dout, lse, dvec, cu, p.N, p.T, p.H,
                                                p.Hk, p.W, p.scale, dq_acc);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 gk((p.T + kRows - 1) / kRows, p.Hk);
  ProfScope prof(kKBwdDkvFp32, st);
  bwd_dkv_fp32_kernel<<<gk, kThreads, 0, st>>>(qh, kh, v, dout, lse, dvec, cu, p.N, p.T, p.H,
                                               p.Hk, p.W, p.scale, dk_acc, dv);
  return cudaGetLastError();
}

}  // namespace flint
