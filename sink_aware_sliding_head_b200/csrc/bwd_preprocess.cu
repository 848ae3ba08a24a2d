// bwd_preprocess.cu - per-row D_i = dO_i . O_i and the sink-logit gradient.
//
// The sink is a softmax category with a zero value (Flint layers page,
// nemo_automodel.components.models.flint.layers, FlintAttention.forward and
// _FlintSinkParameters.forward), so with p_sink_i = e^{s_h - LSE_i}:
//   d s_h = sum_i p_sink_i (0 - dO_i . O_i) = -sum_i e^{s_h - LSE_i} D_i.
// One 16-lane half-warp reduces one (token, head) row with warp shuffles; the
// sink sum is kept per half-warp and per head in shared memory (no atomics),
// summed per block in a fixed order, and the per-block partials are summed in a
// fixed order by a second tiny launch, so the result is deterministic.
#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {

cudaError_t launch_reduce_rows(const float* part, int nrows, int width, float* out,
                               cudaStream_t st);

namespace {

constexpr int kThreads = 256;
constexpr int kGroups = kThreads / 16;
constexpr int kTok = 4;

// Also writes an fp16 copy of dO (dout16, when non-null): the tensor-core
// backward's operands are fp16.
// amax (nullable): [max|dout|, max|v|] slots; dout16 gets dout * s_dout and dvec
// D * s_dout * s_v, the scales of the fp16 operands (d_sink uses the plain D).
// split: dout16 is [T, 2H, D], hi = fp16(dout * s_dout) in row (t, h) and
// lo = fp16(dout * s_dout - hi) in row (t, H + h).
template <typename TO, typename T>
__global__ void __launch_bounds__(kThreads)
bwd_pre_kernel(const TO* __restrict__ out, const T* __restrict__ dout,
               const float* __restrict__ lse, const float* __restrict__ sink,
               float* __restrict__ dvec, float* __restrict__ part, __half* __restrict__ dout16,
               const unsigned* __restrict__ amax, int ntok, int H, int split) {
  extern __shared__ float acc[];   // [kGroups][H]
  const int lane16 = threadIdx.x & 15, grp = threadIdx.x >> 4;
  const int c0 = lane16 * 8;
  const float s_do = slot_scale(amax, false);
  const float s_d = s_do * slot_scale(amax ? amax + 1 : nullptr, false);
  for (int e = threadIdx.x; e < kGroups * H; e += kThreads) acc[e] = 0.f;
  __syncthreads();
  const int rows = kTok * H;
  const int iters = (rows + kGroups - 1) / kGroups;
  for (int t0 = blockIdx.x * kTok; t0 < ntok; t0 += gridDim.x * kTok) {
    for (int it = 0; it < iters; ++it) {
      const int rr = grp + it * kGroups;
      const int t = t0 + rr / H, h = rr % H;
      const bool valid = rr < rows && t < ntok;
      float a[8], b[8];
      if (valid) {
        const size_t base = ((size_t)t * H + h) * kHeadDim + c0;
        load8(out + base, a);
        load8(dout + base, b);
        if (dout16 && split) {
          float hi[8], lo[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float x = b[e] * s_do;   // |x| < 8: no saturation needed
            hi[e] = __half2float(__float2half_rn(x));
            lo[e] = x - hi[e];
          }
          const size_t hb = ((size_t)t * 2 * H + h) * kHeadDim + c0;
          store8(dout16 + hb, hi);
          store8(dout16 + hb + (size_t)H * kHeadDim, lo);
        } else if (dout16) {
          float s8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) s8[e] = sat_f16(b[e] * s_do);
          store8(dout16 + base, s8);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) { a[e] = 0.f; b[e] = 0.f; }
      }
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) d = fmaf(a[e], b[e], d);
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
      if (valid && lane16 == 0) {
        dvec[(size_t)h * ntok + t] = d * s_d;
        acc[grp * H + h] -= expf(sink[h] - lse[(size_t)h * ntok + t]) * d;
      }
    }
  }
  __syncthreads();
  for (int h = threadIdx.x; h < H; h += kThreads) {
    float s = 0.f;
    for (int g = 0; g < kGroups; ++g) s += acc[g * H + h];
    part[(size_t)blockIdx.x * H + h] = s;
  }
}

// dst[i] = fp16(src[i] * 2^e) for n elements (n a multiple of 8), e from the
// max |src| slot (nullptr: e = 0); saturating at +-65504.
template <typename T>
__global__ void convert_f16_kernel(const T* __restrict__ src, __half* __restrict__ dst,
                                   size_t n8, const unsigned* __restrict__ amax) {
  const float sc = slot_scale(amax, false);
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    float f[8];
    load8(src + 8 * i, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = sat_f16(f[e] * sc);
    store8(dst + 8 * i, f);
  }
}

// Split copy: x [T][heads][D] -> dst [T][2 heads][D], hi = fp16(x * 2^e) and
// lo = fp16(x * 2^e - hi); one thread per 8 consecutive channels.
__global__ void convert_split_kernel(const float* __restrict__ src, __half* __restrict__ dst,
                                     size_t n8, int heads, const unsigned* __restrict__ amax) {
  const float sc = slot_scale(amax, false);
  const int row8 = kHeadDim / 8;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8;
       i += (size_t)gridDim.x * blockDim.x) {
    const size_t row = i / row8;              // t * heads + h
    const int c = (int)(i % row8) * 8;
    const size_t t = row / heads;
    const int h = (int)(row % heads);
    float f[8], hi[8], lo[8];
    load8(src + 8 * i, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = f[e] * sc;
      hi[e] = __half2float(__float2half_rn(x));
      lo[e] = x - hi[e];
    }
    const size_t hb = (t * 2 * heads + h) * kHeadDim + c;
    store8(dst + hb, hi);
    store8(dst + hb + (size_t)heads * kHeadDim, lo);
  }
}

// Largest magnitude of two tensors (8 elements per thread and step), one
// atomicMax per block and tensor on the float bit patterns. With padding (valid
// non-null), rows of padding tokens are skipped: whatever a caller leaves there
// must not set the scale of the real rows. row8_0 / row8_1: 8-element groups
// per token of x0 / x1.
template <typename T>
__global__ void __launch_bounds__(256)
absmax_kernel(const T* __restrict__ x0, size_t n0_8, const T* __restrict__ x1, size_t n1_8,
              unsigned* __restrict__ amax, const int32_t* __restrict__ cu,
              const int32_t* __restrict__ valid, int N, int row8_0, int row8_1) {
  __shared__ float red[2][8];
  float m0 = 0.f, m1 = 0.f;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n0_8 + n1_8; i += stride) {
    float f[8];
    const bool first = i < n0_8;
    if (valid) {
      const int t = (int)(first ? i / row8_0 : (i - n0_8) / row8_1);
      const int d = doc_of(cu, N, t);
      if (t - __ldg(cu + d) >= __ldg(valid + d)) continue;   // a padding token
    }
    load8(first ? x0 + 8 * i : x1 + 8 * (i - n0_8), f);
    float m = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    if (first) m0 = fmaxf(m0, m); else m1 = fmaxf(m1, m);
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { red[0][warp] = m0; red[1][warp] = m1; }
  __syncthreads();
  if (threadIdx.x < 2) {
    float m = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[threadIdx.x][w]);
    if (m > 0.f) atomicMax(amax + threadIdx.x, __float_as_uint(m));
  }
}

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n2) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += gridDim.x * blockDim.x) {
    float p0, p1;
    exp2_fma2(x[2 * i], x[2 * i + 1], p0, p1);
    y[2 * i] = p0;
    y[2 * i + 1] = p1;
  }
}

}  // namespace

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  exp2_poly_kernel<<<(n / 2 + 255) / 256, 256, 0, st>>>(x, y, n / 2);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t convert_f16(const T* src, __half* dst, size_t n, const unsigned* amax,
                               cudaStream_t st) {
  const size_t n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  size_t blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  ProfScope prof(kKConvert, st);
  convert_f16_kernel<T><<<(unsigned)blocks, 256, 0, st>>>(src, dst, n8, amax);
  return cudaGetLastError();
}
cudaError_t launch_convert_f16(const __nv_bfloat16* src, __half* dst, size_t n,
                               const unsigned* amax, cudaStream_t st) {
  return convert_f16(src, dst, n, amax, st);
}
cudaError_t launch_convert_f16(const float* src, __half* dst, size_t n, const unsigned* amax,
                               cudaStream_t st) {
  return convert_f16(src, dst, n, amax, st);
}

cudaError_t launch_convert_split(const float* src, __half* dst, int T, int heads,
                                 const unsigned* amax, cudaStream_t st) {
  const size_t n8 = (size_t)T * heads * kHeadDim / 8;
  if (n8 == 0) return cudaSuccess;
  size_t blocks = (n8 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  ProfScope prof(kKConvert, st);
  convert_split_kernel<<<(unsigned)blocks, 256, 0, st>>>(src, dst, n8, heads, amax);
  return cudaGetLastError();
}

cudaError_t launch_absmax(int dtype, const void* x0, size_t n0, const void* x1, size_t n1,
                          unsigned* amax, const int32_t* cu, const int32_t* valid, int N,
                          int heads0, int heads1, cudaStream_t st) {
  const size_t n0_8 = x0 ? n0 / 8 : 0, n1_8 = x1 ? n1 / 8 : 0;
  if (n0_8 + n1_8 == 0) return cudaSuccess;
  size_t blocks = (n0_8 + n1_8 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  ProfScope prof(kKAbsmax, st);
  const int r0 = heads0 * kHeadDim / 8, r1 = heads1 * kHeadDim / 8;   // 8-groups per token
  if (dtype == FLINT_BF16)
    absmax_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x0), n0_8, static_cast<const __nv_bfloat16*>(x1),
        n1_8, amax, cu, valid, N, r0 > 0 ? r0 : 1, r1 > 0 ? r1 : 1);
  else
    absmax_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
        static_cast<const float*>(x0), n0_8, static_cast<const float*>(x1), n1_8, amax, cu,
        valid, N, r0 > 0 ? r0 : 1, r1 > 0 ? r1 : 1);
  return cudaGetLastError();
}

cudaError_t launch_bwd_preprocess(const Resolved& p, const void* out, const void* dout,
                                  const float* lse, const float* sink, float* dvec, float* part,
                                  float* dsink, __half* dout16, const unsigned* amax,
                                  cudaStream_t st, int split) {
  if (p.T == 0) {
    cudaMemsetAsync(dsink, 0, p.H * sizeof(float), st);
    return cudaGetLastError();
  }
  int blocks = (p.T + kTok - 1) / kTok;
  if (blocks > kPartBlocks) blocks = kPartBlocks;
  const size_t smem = (size_t)kGroups * p.H * sizeof(float);
  {
  ProfScope prof(kKBwdPre, st);
  typedef __nv_bfloat16 bf;
  if (p.dtype == FLINT_BF16 && p.fp32_out)
    bwd_pre_kernel<float, bf><<<blocks, kThreads, smem, st>>>(
        (const float*)out, (const bf*)dout, lse, sink, dvec, part, dout16, amax, p.T, p.H, 0);
  else if (p.dtype == FLINT_BF16)
    bwd_pre_kernel<bf, bf><<<blocks, kThreads, smem, st>>>(
        (const bf*)out, (const bf*)dout, lse, sink, dvec, part, dout16, amax, p.T, p.H, 0);
  else if (p.out_f16)   // FP32 inputs at the fp16 compute boundary: out is fp16
    bwd_pre_kernel<__half, float><<<blocks, kThreads, smem, st>>>(
        (const __half*)out, (const float*)dout, lse, sink, dvec, part, dout16, amax, p.T, p.H, 0);
  else
    bwd_pre_kernel<float, float><<<blocks, kThreads, smem, st>>>(
        (const float*)out, (const float*)dout, lse, sink, dvec, part,
        (p.tc || split) ? dout16 : nullptr, (p.tc || split) ? amax : nullptr, p.T, p.H, split);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_reduce_rows(part, blocks, p.H, dsink, st);
}

}  // namespace flint
