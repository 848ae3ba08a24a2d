// common.cuh - internal definitions shared by the library's kernels and its
// C-ABI layer: resolved parameters, workspace layout, status bits, and small
// device helpers (document lookup, bf16/fp32 loads and stores).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/flint_attn.h"
#include "device_once.h"

namespace flint {

constexpr int kHeadDim = 128;
constexpr int kTileRows = 128;   // query rows per tensor-core tile (tokens x heads-of-group)
constexpr int kTileKeys = 128;   // keys per tensor-core tile

// Status bits written into the workspace's status word by bounded device waits.
enum : int {
  kStatusTimeoutFwd = 1,
  kStatusTimeoutBwdKV = 2,
  kStatusTimeoutBwdQ = 4,
  kStatusSmemAlign = 8,        // dynamic shared memory not 1024-byte aligned
  kStatusDecodeRange = 16,     // a decode cache_lens entry outside [0, cache_capacity)
  kStatusTimeoutSelftest = 32, // the bounded-wait self-test's wait ran out
};

// int slots of the workspace's status region (int[64], zeroed at the start of
// every call): [0] status bits, [1..3] work-list lengths, [4..5] dynamic item
// counters, [8] and [9] the bit patterns of max |dout| and max |v|.
enum : int { kSlotAmaxDout = 8, kSlotAmaxV = 9 };

// Operand range of the fp16 tensor-core copies of dout and v. Each copy is
// multiplied by a power of two 2^e chosen from the tensor's largest magnitude,
// so that it lands in [4, 8) - the range of the N(0,1) data the kernels are
// tuned and tested on - and can neither saturate at fp16's 65504 nor lose
// precision in fp16's subnormal range (below 6.1e-5). Multiplying by a power
// of two is exact, and the FP32 epilogues divide it out again. amax_bits is
// the bit pattern of max |x| (non-negative floats order like their bits); an
// all-zero tensor gets e = 0.
__host__ __device__ inline int pow2_scale_exp(unsigned amax_bits) {
  if (amax_bits == 0) return 0;
  const int E = (int)((amax_bits >> 23) & 0xff);   // floor(log2 max|x|) + 127 (normal)
  int e = 129 - E;                                  // max|x| * 2^e in [4, 8)
  return e < -126 ? -126 : (e > 126 ? 126 : e);
}
__host__ __device__ inline float exp2_int(int e) {   // 2^e for -126 <= e <= 127
  union { unsigned u; float f; } c;
  c.u = (unsigned)(e + 127) << 23;
  return c.f;
}
// 2^e read from a device slot written by launch_absmax (nullptr: 1).
__device__ __forceinline__ float slot_scale(const unsigned* amax, bool inverse) {
  if (!amax) return 1.f;
  const int e = pow2_scale_exp(*reinterpret_cast<const volatile unsigned*>(amax));
  return exp2_int(inverse ? -e : e);
}

// Parameters after validation and defaulting.
struct Resolved {
  int T, N, H, Hk, D, G, W, rope;
  float theta, eps, scale;
  int dtype;
  int fp32_out;     // out, dq, dk, dv are float32 (always for FP32 inputs)
  int tc;           // the tcgen05 path with fp16 operands: BF16 inputs, or FP32 + compute_f16
  int out_f16;      // out is IEEE fp16 (FP32 inputs with compute_f16, without fp32_out)
  int x3;           // the tcgen05 path for FP32 inputs: operands split into fp16 hi + lo
                    // parts, three MMAs per product (no compute_f16; G in {1,2,4,8,16})
  int R;            // tokens per 128-row tile = 128 / G
};

// Offsets (bytes) of every region of the workspace. All regions are 256-byte aligned.
struct WsLayout {
  size_t status;        // int[64]: [0] status bits, [1..3] work-list lengths
  size_t qhat, khat;    // normalised+rotated q [T,H,D], k [T,Hk,D] (dtype; for the
                        // split path fp16 [T,2H,D], [T,2Hk,D]: hi rows, then lo rows)
  size_t items_q;       // int4 work items, query-major (forward: pairs of tiles)
  size_t items_q1;      // int4 work items, query-major single tiles (backward dQ)
  size_t items_kv;      // int4 work items, key-major (backward dK/dV)
  size_t sched_tmp;     // int4 + int per item, scratch for the LPT sort
  size_t sched_tmp2;    // the same for the backward's second list (built concurrently)
  size_t dvec;          // [H,T] fp32 rowsum(dO * O)      (backward)
  size_t part;          // fp32 partial sums (d sink, d norm weights)
  size_t dq_acc;        // [T,H,D] fp32 gradient w.r.t. q_hat (backward)
  size_t dk_acc;        // [T,Hk,D] fp32 gradient w.r.t. k_hat (backward)
  size_t dout16;        // [T,H,D] fp16 copy of dO (backward, tensor-core path; [T,2H,D]
                        // hi and lo parts on the split path)
  size_t v16;           // [T,Hk,D] fp16 copy of v (tensor-core path; [T,2Hk,D] split)
  size_t total;
  int max_items_q, max_items_q1, max_items_kv, max_items_any;
  int part_blocks;      // number of partial-sum rows per reduced quantity
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

inline int elem_bytes(int dtype) { return dtype == FLINT_BF16 ? 2 : 4; }

constexpr int kPartBlocks = 1184;   // 148 SMs x 8: rows of partial sums for reductions

inline WsLayout make_layout(const Resolved& p, bool backward) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) { size_t o = off; off = align256(off + bytes); return o; };
  const size_t eb = elem_bytes(p.dtype);
  L.status = take(64 * sizeof(int));
  L.qhat = take((size_t)p.T * p.H * p.D * eb);
  L.khat = take((size_t)p.T * p.Hk * p.D * eb);
  const int span_fwd = p.x3 ? p.R : 2 * p.R;   // tokens per forward item
  L.max_items_q = p.Hk * ((p.T + span_fwd - 1) / span_fwd + p.N);
  L.max_items_q1 = p.Hk * ((p.T + p.R - 1) / p.R + p.N);
  L.max_items_kv = p.Hk * ((p.T + kTileKeys - 1) / kTileKeys + p.N);
  L.max_items_any = L.max_items_q1;
  if (L.max_items_q > L.max_items_any) L.max_items_any = L.max_items_q;
  if (L.max_items_kv > L.max_items_any) L.max_items_any = L.max_items_kv;
  L.items_q = take((size_t)L.max_items_q * 16);
  L.items_q1 = backward ? take((size_t)L.max_items_q1 * 16) : off;
  L.items_kv = backward ? take((size_t)L.max_items_kv * 16) : off;
  L.sched_tmp = take((size_t)L.max_items_any * 20);
  L.sched_tmp2 = backward ? take((size_t)L.max_items_any * 20) : off;
  L.part_blocks = kPartBlocks;
  const size_t parts = p.x3 ? 2 : 1;   // the split path keeps hi and lo fp16 parts
  if (p.tc || p.x3) L.v16 = take((size_t)p.T * p.Hk * p.D * 2 * parts);
  if (backward) {
    L.dvec = take((size_t)p.H * p.T * 4);
    L.part = take((size_t)kPartBlocks * (p.H + 2 * p.D) * 4);
    L.dq_acc = take((size_t)p.T * p.H * p.D * 4);
    L.dk_acc = take((size_t)p.T * p.Hk * p.D * 4);
    if (p.tc || p.x3) L.dout16 = take((size_t)p.T * p.H * p.D * 2 * parts);
  }
  L.total = off;
  return L;
}

// ------------------------------------------------------------------ device helpers

// Index of the document that holds token t (cu non-decreasing, cu[0] = 0,
// cu[N] = T, t < T). Empty documents are skipped.
__device__ __forceinline__ int doc_of(const int32_t* __restrict__ cu, int N, int t) {
  int lo = 0, hi = N;           // invariant: cu[lo] <= t < cu[hi]
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// 8 consecutive elements <-> 8 floats (16-byte loads for bf16, 2 x 16 bytes for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const __half* p, float (&f)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&f)[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void store8(__half* p, const float (&f)[8]) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
// fp16 range: values beyond +-65504 saturate instead of becoming infinite
__device__ __forceinline__ float sat_f16(float x) { return fminf(fmaxf(x, -65504.f), 65504.f); }
__device__ __forceinline__ void store8(float* p, const float (&f)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// ------------------------------------------------------------------ kernel timing
// Every kernel launch of the library sits inside a ProfScope: it counts the
// launch and, when profiling is enabled, records a CUDA event pair around it
// on the launching stream (see flint_attn_profile_* in the public header).
enum KernelId {
  kKPrologue = 0, kKWorklist, kKFwdSm100, kKFwdFp32, kKBwdPre, kKReduce, kKBwdDkvSm100,
  kKBwdDqSm100, kKBwdDqFp32, kKBwdDkvFp32, kKPrologueBwd, kKConvert, kKDecode, kKPadFill,
  kKAbsmax, kKFwdX3, kKBwdDkvX3, kKBwdDqX3,
  kNumKernelIds
};
struct ProfScope {
  int id;
  cudaStream_t st;
  int slot;
  ProfScope(int id, cudaStream_t st);
  ~ProfScope();
};

// ------------------------------------------------------------------ launchers
// (defined in the .cu files; all return cudaGetLastError() of their launch)
// valid: per-document count of real tokens (trailing padding), or nullptr
cudaError_t launch_build_worklist(const int32_t* cu, const int32_t* valid, const Resolved& p,
                                  int mode, int span, int4* items, int* count, void* tmp,
                                  int max_items, cudaStream_t st);
// Two lists in one launch (one block each); tmp0 and tmp1 must not overlap.
cudaError_t launch_build_worklists2(const int32_t* cu, const int32_t* valid, const Resolved& p,
                                    int mode0, int span0, int4* items0, int* count0, void* tmp0,
                                    int max0, int mode1, int span1, int4* items1, int* count1,
                                    void* tmp1, int max1, cudaStream_t st);
// Padding: padded rows get out = 0 and lse = sink (forward), and zero gradient
// rows dq_acc, dk_acc (fp32 workspace) and dv (backward).
cudaError_t launch_pad_fill_fwd(const Resolved& p, const int32_t* cu, const int32_t* valid,
                                const float* sink, void* out, float* lse, cudaStream_t st);
cudaError_t launch_pad_fill_bwd(const Resolved& p, const int32_t* cu, const int32_t* valid,
                                float* dq_acc, float* dk_acc, void* dv, int dv_f32,
                                cudaStream_t st);
// q_hat [T,H,D] and k_hat [T,Hk,D] in one launch, written as
enum { kHatInput = 0,    // the input type
       kHatF16 = 1,      // fp16 (the tensor-core operands)
       kHatSplit = 2 };  // fp16 hi and lo parts, [T,2H,D] and [T,2Hk,D] (FP32 inputs)
cudaError_t launch_prologue_qk(const Resolved& p, const void* q, const void* wq, void* qh,
                               const void* k, const void* wk, void* kh, const int32_t* cu,
                               cudaStream_t st, int hat_mode);
// Split copy of an FP32 tensor x [T,heads,D]: dst [T,2*heads,D] fp16 holds
// hi = fp16(x * 2^e) in rows [0,heads) of each token and lo = fp16(x * 2^e - hi)
// in rows [heads, 2*heads); e from the max |x| slot (nullptr: e = 0).
cudaError_t launch_convert_split(const float* src, __half* dst, int T, int heads,
                                 const unsigned* amax, cudaStream_t st);
// dst = fp16(src * 2^e), e from the max |src| in *amax (nullptr: e = 0).
cudaError_t launch_convert_f16(const __nv_bfloat16* src, __half* dst, size_t n,
                               const unsigned* amax, cudaStream_t st);
cudaError_t launch_convert_f16(const float* src, __half* dst, size_t n, const unsigned* amax,
                               cudaStream_t st);
// amax[0] = bits of max |x0| over n0 elements, amax[1] = bits of max |x1| over n1
// (both raised with atomicMax, so the slots must start at zero); x0 or x1 may be
// null (n = 0). n0, n1 multiples of 8. dtype: FLINT_BF16 or FLINT_FP32 for both.
// x0 is [T, heads0, D] and x1 [T, heads1, D]; with valid non-null (padding),
// the rows of padding tokens (documents per cu, N) are left out.
cudaError_t launch_absmax(int dtype, const void* x0, size_t n0, const void* x1, size_t n1,
                          unsigned* amax, const int32_t* cu, const int32_t* valid, int N,
                          int heads0, int heads1, cudaStream_t st);
// Bounded-wait self-test (selftest.cu): status[0] gets the timeout bit, status[1]
// 1 if the wait completed and 0 if it gave up.
cudaError_t launch_wait_selftest(long long limit, int arrive_first, int* status,
                                 cudaStream_t st);

// Decode over a KV cache (decode.cu). A (sequence, KV head) window is split into
// chunks of at least kMinChunkKeysDecode keys (a multiple of the 16-key step).
constexpr int kMinChunkKeysDecode = 256;
struct DecodeLaunch {
  int B, C, H, Hk, W, rope, out_f32, num_sms;
  float theta, eps, scale;
  const void *q, *k, *v, *wq, *wk;
  const float* sink;
  const int32_t* lens;
  void *kc, *vc;
  int* counters;                    // workspace: [B * Hk], zeroed per call
  float *part_o, *part_ml;          // workspace
  void* out;
  float* lse;
  int* status;
};
// Split CTAs per (sequence, KV head): the most any call with capacity C and window W
// launches (the workspace is sized for it).
int decode_splits_max(int C, int W);
cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t st);
cudaError_t launch_attn_fwd_fp32(const Resolved& p, const float* qh, const float* kh,
                                 const float* v, const float* sink, const int32_t* cu, float* out,
                                 float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_fp32(const Resolved& p, const float* qh, const float* kh,
                                 const float* v, const float* dout, const float* lse,
                                 const float* dvec, const int32_t* cu, float* dq_acc,
                                 float* dk_acc, float* dv, cudaStream_t st);
// D = rowsum(dout * out) into dvec, d_sink, and (dout16 non-null) the fp16 copy of
// dout. amax (nullable): the [max|dout|, max|v|] slots; when given, dout16 is
// dout * s_dout and dvec holds D * s_dout * s_v (the scales of the fp16
// operands), while d_sink is formed from the unscaled D. split: dout16 is
// [T,2H,D] with the hi and lo fp16 parts of dout * s_dout (FP32 inputs).
cudaError_t launch_bwd_preprocess(const Resolved& p, const void* out, const void* dout,
                                  const float* lse, const float* sink, float* dvec, float* part,
                                  float* dsink, __half* dout16, const unsigned* amax,
                                  cudaStream_t st, int split = 0);
cudaError_t launch_bwd_epilogue(const Resolved& p, const void* x, const void* w,
                                const float* g_hat, void* dx, float* dw, float* part, int heads,
                                const int32_t* cu, cudaStream_t st);
enum { kModeQuery = 0, kModeKey = 1 };

// Raises a kernel's dynamic shared-memory limit on the current device the
// first time its launcher runs there (per device; safe from several threads).
template <typename Kernel>
cudaError_t smem_limit_once(PerDeviceOnce& once, Kernel* kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return static_cast<cudaError_t>(once.run(dev, [&] {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  }));
}

}  // namespace flint
