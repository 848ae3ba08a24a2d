// prologue.cu - per-head RMSNorm + NeoX RoPE on q and k (forward), and its
// transpose (RoPE^T then RMSNorm backward) for the gradients (backward).
//
// Flint layers page (nemo_automodel.components.models.flint.layers),
// FlintAttention: per-head RMSNorm (q_norm, k_norm, eps = rms_norm_eps) then
// selective NeoX RoPE (_apply_rope: channel j rotates with channel j + D/2);
// Flint config page: full layers have no RoPE, sliding layers rotate all head
// channels; positions are document-local for THD packing.
//
// Layout: one 16-lane half-warp owns one (token, head) row of 128 channels,
// 8 channels per lane (a 16-byte load for bf16). A block owns kTok tokens and
// first builds their cos/sin table in shared memory (angles are shared by all
// heads of a token), so the row work is one pass of 16-byte loads and stores.
// The RoPE partner channel (c +- 64) lives in lane +- 8 of the half-warp.
#include "common.cuh"

namespace flint {

namespace {

constexpr int kTok = 4;            // tokens per block (per chunk in the backward)
constexpr int kThreads = 256;      // 16 half-warps
constexpr int kHalf = kHeadDim / 2;

// cos/sin of pos * theta^(-2j/D) for the block's tokens, j < 64. The angle is
// formed and reduced modulo 2*pi in double, then rounded to float.
__device__ void build_rope_table(const int32_t* __restrict__ cu, int N, int T, int t0,
                                 float theta, float (*cs)[kHalf], float (*sn)[kHalf],
                                 int* pos_s) {
  if (threadIdx.x < kTok) {
    int t = t0 + threadIdx.x;
    pos_s[threadIdx.x] = (t < T) ? t - __ldg(cu + doc_of(cu, N, t)) : 0;
  }
  __shared__ double inv_freq[kHalf];
  if (threadIdx.x < kHalf)
    inv_freq[threadIdx.x] = exp2(-(2.0 * threadIdx.x / kHeadDim) * log2((double)theta));
  __syncthreads();
  for (int e = threadIdx.x; e < kTok * kHalf; e += blockDim.x) {
    int tok = e / kHalf, j = e % kHalf;
    double a = (double)pos_s[tok] * inv_freq[j];
    const double two_pi = 6.283185307179586476925286766559;
    a -= two_pi * rint(a / two_pi);
    float s, c;
    sincosf((float)a, &s, &c);
    cs[tok][j] = c;
    sn[tok][j] = s;
  }
  __syncthreads();
}

// q and k in one launch: the first nblk0 blocks normalise kTok tokens of x0
// (heads0 rows per token) each, the rest kTok tokens of x1 (heads1 rows).
// kSplit (TO = __half): y is [T, 2*heads, D]; row (t, h) gets hi = fp16(x) and
// row (t, heads + h) lo = fp16(x - hi), the two parts of the split path.
template <typename T, typename TO, bool kSplit = false>
__global__ void __launch_bounds__(kThreads)
prologue_kernel(const T* __restrict__ x0, const T* __restrict__ w0, TO* __restrict__ y0,
                int heads0, const T* __restrict__ x1, const T* __restrict__ w1,
                TO* __restrict__ y1, int heads1, int nblk0, int ntok,
                const int32_t* __restrict__ cu, int N, int rope, float theta, float eps) {
  __shared__ float cs[kTok][kHalf], sn[kTok][kHalf];
  __shared__ int pos_s[kTok];
  const bool second = (int)blockIdx.x >= nblk0;
  const T* __restrict__ x = second ? x1 : x0;
  const T* __restrict__ w = second ? w1 : w0;
  TO* __restrict__ y = second ? y1 : y0;
  const int heads = second ? heads1 : heads0;
  const int t0 = (second ? blockIdx.x - nblk0 : blockIdx.x) * kTok;
  if (rope) build_rope_table(cu, N, ntok, t0, theta, cs, sn, pos_s);
  const int lane16 = threadIdx.x & 15;
  const int grp = threadIdx.x >> 4;
  const int c0 = lane16 * 8;
  float wv[8];
  load8(w + c0, wv);
  const int rows = kTok * heads;
  // Every half-warp runs the same number of iterations so the full-warp
  // shuffles below always see both halves; invalid rows load zeros, store nothing.
  const int iters = (rows + kThreads / 16 - 1) / (kThreads / 16);
  for (int it = 0; it < iters; ++it) {
    const int rr = grp + it * (kThreads / 16);
    const int tok = rr / heads;
    const int t = t0 + tok;
    const bool valid = rr < rows && t < ntok;
    const size_t base = valid ? ((size_t)t * heads + (rr % heads)) * kHeadDim + c0 : 0;
    float v[8];
    if (valid) load8(x + base, v);
    else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) ss += v[e] * v[e];
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss * (1.0f / kHeadDim) + eps);
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = v[e] * r * wv[e];
    if (rope) {
      float o8[8];
      const bool lo_half = lane16 < 8;
      const int j0 = lo_half ? c0 : c0 - kHalf;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float partner = __shfl_xor_sync(0xffffffffu, v[e], 8);
        const int tk = valid ? tok : 0;
        const float c = cs[tk][j0 + e], s = sn[tk][j0 + e];
        o8[e] = lo_half ? (v[e] * c - partner * s) : (v[e] * c + partner * s);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = o8[e];
    }
    if (valid) {
      if constexpr (kSplit) {
        const size_t hb = ((size_t)t * 2 * heads + (rr % heads)) * kHeadDim + c0;
        float hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          hi[e] = __half2float(__float2half_rn(v[e]));
          lo[e] = v[e] - hi[e];   // exact in fp32; rounded once to fp16 by store8
        }
        store8(y + hb, hi);
        store8(y + hb + (size_t)heads * kHeadDim, lo);
      } else {
        store8(y + base, v);
      }
    }
  }
}

// Gradient of the prologue. g_hat: fp32 gradient w.r.t. the normalised (and
// rotated) rows. dx = r*u - x*r^3*(1/D)*sum(u*x) with u = RoPE^T(g_hat)*w and
// r = (mean x^2 + eps)^-1/2; partial d w = sum over rows of RoPE^T(g_hat)*x*r.
template <typename T, typename TD>
__global__ void __launch_bounds__(kThreads)
prologue_bwd_kernel(const T* __restrict__ x, const T* __restrict__ w,
                    const float* __restrict__ g_hat, TD* __restrict__ dx,
                    float* __restrict__ dw_part, int ntok, int heads,
                    const int32_t* __restrict__ cu, int N, int rope, float theta, float eps) {
  __shared__ float cs[kTok][kHalf], sn[kTok][kHalf];
  __shared__ int pos_s[kTok];
  __shared__ float red[kThreads / 16][kHeadDim];
  const int lane16 = threadIdx.x & 15;
  const int grp = threadIdx.x >> 4;
  const int c0 = lane16 * 8;
  float wv[8], dwacc[8];
  load8(w + c0, wv);
#pragma unroll
  for (int e = 0; e < 8; ++e) dwacc[e] = 0.f;
  for (int t0 = blockIdx.x * kTok; t0 < ntok; t0 += gridDim.x * kTok) {
    if (rope) build_rope_table(cu, N, ntok, t0, theta, cs, sn, pos_s);
    const int rows = kTok * heads;
    const int iters = (rows + kThreads / 16 - 1) / (kThreads / 16);
    for (int it = 0; it < iters; ++it) {
      const int rr = grp + it * (kThreads / 16);
      const int tok = rr / heads;
      const int t = t0 + tok;
      const bool valid = rr < rows && t < ntok;
      const size_t base = valid ? ((size_t)t * heads + (rr % heads)) * kHeadDim + c0 : 0;
      float xv[8], g[8];
      if (valid) {
        load8(x + base, xv);
        load8(g_hat + base, g);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) { xv[e] = 0.f; g[e] = 0.f; }
      }
      if (rope) {
        float o8[8];
        const bool lo_half = lane16 < 8;
        const int j0 = lo_half ? c0 : c0 - kHalf;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float partner = __shfl_xor_sync(0xffffffffu, g[e], 8);
          const int tk = valid ? tok : 0;
          const float c = cs[tk][j0 + e], s = sn[tk][j0 + e];
          o8[e] = lo_half ? (g[e] * c + partner * s) : (g[e] * c - partner * s);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) g[e] = o8[e];
      }
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += xv[e] * xv[e];
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float r = rsqrtf(ss * (1.0f / kHeadDim) + eps);
      float ux = 0.f, u[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        dwacc[e] += g[e] * xv[e] * r;
        u[e] = g[e] * wv[e];
        ux += u[e] * xv[e];
      }
#pragma unroll
      for (int o = 8; o >= 1; o >>= 1) ux += __shfl_xor_sync(0xffffffffu, ux, o);
      const float k3 = r * r * r * ux * (1.0f / kHeadDim);
      float out8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) out8[e] = r * u[e] - xv[e] * k3;
      if (valid) store8(dx + base, out8);
    }
    __syncthreads();   // the rope table is rebuilt for the next chunk
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[grp][c0 + e] = dwacc[e];
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    float s = 0.f;
    for (int gi = 0; gi < kThreads / 16; ++gi) s += red[gi][threadIdx.x];
    dw_part[(size_t)blockIdx.x * kHeadDim + threadIdx.x] = s;
  }
}

// out[c] = sum over rows b < nrows of part[b * width + c], in a fixed order: a
// block of 32 warps owns 32 columns (one per lane, so loads are coalesced), warp
// w adds rows w, w + 32, ... in turn, and one warp then adds the 32 warp sums in
// warp order. The result does not depend on timing (deterministic).
constexpr int kRedWarps = 32;
__global__ void __launch_bounds__(32 * kRedWarps)
reduce_rows_kernel(const float* __restrict__ part, int nrows, int width,
                   float* __restrict__ out) {
  __shared__ float red[kRedWarps][33];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int c = blockIdx.x * 32 + lane;
  float s = 0.f;
  if (c < width) {
#pragma unroll 4
    for (int b = w; b < nrows; b += kRedWarps) s += part[(size_t)b * width + c];
  }
  red[w][lane] = s;
  __syncthreads();
  if (w == 0 && c < width) {
    float t = 0.f;
    for (int i = 0; i < kRedWarps; ++i) t += red[i][lane];
    out[c] = t;
  }
}

}  // namespace

cudaError_t launch_prologue_qk(const Resolved& p, const void* q, const void* wq, void* qh,
                               const void* k, const void* wk, void* kh, const int32_t* cu,
                               cudaStream_t st, int hat_mode) {
  const bool out_f16 = hat_mode == kHatF16;
  if (p.T == 0) return cudaSuccess;
  const int nblk = (p.T + kTok - 1) / kTok;   // per tensor
  dim3 grid(2 * nblk);
  ProfScope prof(kKPrologue, st);
  typedef __nv_bfloat16 bf;
  if (p.dtype == FLINT_BF16 && out_f16)
    prologue_kernel<bf, __half><<<grid, kThreads, 0, st>>>(
        (const bf*)q, (const bf*)wq, (__half*)qh, p.H, (const bf*)k, (const bf*)wk, (__half*)kh,
        p.Hk, nblk, p.T, cu, p.N, p.rope, p.theta, p.eps);
  else if (p.dtype == FLINT_BF16)
    prologue_kernel<bf, bf><<<grid, kThreads, 0, st>>>(
        (const bf*)q, (const bf*)wq, (bf*)qh, p.H, (const bf*)k, (const bf*)wk, (bf*)kh, p.Hk,
        nblk, p.T, cu, p.N, p.rope, p.theta, p.eps);
  else if (hat_mode == kHatSplit)   // FP32 inputs on the split path
    prologue_kernel<float, __half, true><<<grid, kThreads, 0, st>>>(
        (const float*)q, (const float*)wq, (__half*)qh, p.H, (const float*)k, (const float*)wk,
        (__half*)kh, p.Hk, nblk, p.T, cu, p.N, p.rope, p.theta, p.eps);
  else if (out_f16)   // FP32 inputs at the fp16 compute boundary
    prologue_kernel<float, __half><<<grid, kThreads, 0, st>>>(
        (const float*)q, (const float*)wq, (__half*)qh, p.H, (const float*)k, (const float*)wk,
        (__half*)kh, p.Hk, nblk, p.T, cu, p.N, p.rope, p.theta, p.eps);
  else
    prologue_kernel<float, float><<<grid, kThreads, 0, st>>>(
        (const float*)q, (const float*)wq, (float*)qh, p.H, (const float*)k, (const float*)wk,
        (float*)kh, p.Hk, nblk, p.T, cu, p.N, p.rope, p.theta, p.eps);
  return cudaGetLastError();
}

cudaError_t launch_bwd_epilogue(const Resolved& p, const void* x, const void* w,
                                const float* g_hat, void* dx, float* dw, float* part, int heads,
                                const int32_t* cu, cudaStream_t st) {
  int blocks = (p.T + kTok - 1) / kTok;
  if (blocks > kPartBlocks) blocks = kPartBlocks;
  if (blocks < 1) blocks = 1;
  if (p.T == 0) {
    cudaMemsetAsync(dw, 0, kHeadDim * sizeof(float), st);
    return cudaGetLastError();
  }
  {
  ProfScope prof(kKPrologueBwd, st);
  typedef __nv_bfloat16 bf;
  if (p.dtype == FLINT_BF16 && p.fp32_out)
    prologue_bwd_kernel<bf, float><<<blocks, kThreads, 0, st>>>(
        (const bf*)x, (const bf*)w, g_hat, (float*)dx, part, p.T, heads, cu, p.N, p.rope, p.theta,
        p.eps);
  else if (p.dtype == FLINT_BF16)
    prologue_bwd_kernel<bf, bf><<<blocks, kThreads, 0, st>>>(
        (const bf*)x, (const bf*)w, g_hat, (bf*)dx, part, p.T, heads, cu, p.N, p.rope, p.theta,
        p.eps);
  else
    prologue_bwd_kernel<float, float><<<blocks, kThreads, 0, st>>>(
        (const float*)x, (const float*)w, g_hat, (float*)dx, part, p.T, heads, cu, p.N, p.rope,
        p.theta, p.eps);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  ProfScope prof(kKReduce, st);
  reduce_rows_kernel<<<(kHeadDim + 31) / 32, 32 * kRedWarps, 0, st>>>(part, blocks, kHeadDim, dw);
  return cudaGetLastError();
}

cudaError_t launch_reduce_rows(const float* part, int nrows, int width, float* out,
                               cudaStream_t st) {
  ProfScope prof(kKReduce, st);
  reduce_rows_kernel<<<(width + 31) / 32, 32 * kRedWarps, 0, st>>>(part, nrows, width, out);
  return cudaGetLastError();
}

}  // namespace flint
