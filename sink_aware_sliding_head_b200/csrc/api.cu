// api.cu - the C ABI declared in include/flint_attn.h: argument validation,
// workspace carving, TMA tensor-map encoding and the launch sequence of each
// call. Everything here is host code; it allocates nothing and launches only
// this library's kernels on the caller's stream.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {

cudaError_t launch_reduce_rows(const float* part, int nrows, int width, float* out,
                               cudaStream_t st);
cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t st);
int fwd_kv_box_tokens();
cudaError_t launch_attn_fwd_sm100_impl(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, const Resolved& p, const float* sink,
                                       const int4* items, const int* n_items, int max_items,
                                       const unsigned* amax_v, void* out, float* lse,
                                       int* status, int num_sms, cudaStream_t st);
cudaError_t launch_attn_bwd_sm100_impl(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, const CUtensorMap& tdo,
                                       const Resolved& p, const float* lse, const float* dvec,
                                       const unsigned* amax, const int4* items_kv,
                                       const int* n_kv, int max_kv,
                                       const int4* items_q, const int* n_q, int max_q,
                                       float* dq_acc, float* dk_acc, void* dv, int* status,
                                       int num_sms, cudaStream_t st);
int x3_kv_box_tokens_fwd();
int x3_q_box_rows_dkv();
int x3_kv_box_tokens_dq();
cudaError_t launch_attn_fwd_x3(const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const Resolved& p, const float* sink,
                               const int4* items, const int* n_items, int max_items,
                               const unsigned* amax, float* out, float* lse, int* status,
                               int num_sms, cudaStream_t st);
cudaError_t launch_attn_bwd_x3(const CUtensorMap& tq64, const CUtensorMap& tk128,
                               const CUtensorMap& tdo64, const CUtensorMap& tk64,
                               const CUtensorMap& tv64, const Resolved& p, const float* lse,
                               const float* dvec, const unsigned* amax, const __half* qs,
                               const __half* dos, const __half* vs, const int4* items_kv,
                               const int* n_kv, int max_kv, const int4* items_q, const int* n_q,
                               int max_q, float* dq_acc, float* dk_acc, float* dv, int* status,
                               int num_sms, cudaStream_t st);

// ------------------------------------------------------------------ kernel timing
namespace {
const char* const kKernelNames[kNumKernelIds] = {
    "prologue_rmsnorm_rope", "build_worklist", "attn_fwd_sm100", "attn_fwd_fp32",
    "bwd_preprocess", "reduce_rows", "attn_bwd_dkv_sm100", "attn_bwd_dq_sm100",
    "attn_bwd_dq_fp32", "attn_bwd_dkv_fp32", "prologue_bwd", "convert_f16",
    "decode", "pad_fill", "absmax", "attn_fwd_x3_sm100", "attn_bwd_dkv_x3_sm100",
    "attn_bwd_dq_x3_sm100"};
constexpr int kMaxSlots = 1 << 15;
struct Prof {
  std::mutex mu;
  bool enabled = false;
  long long launches_total = 0;
  std::vector<cudaEvent_t> ev0, ev1;
  std::vector<int> slot_id;
  int used = 0;
  double total_ms[kNumKernelIds] = {};
  long long launches[kNumKernelIds] = {};
};
Prof& prof() {
  static Prof p;
  return p;
}
}  // namespace

ProfScope::ProfScope(int id_, cudaStream_t st_) : id(id_), st(st_), slot(-1) {
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  ++P.launches_total;
  if (!P.enabled || P.used >= kMaxSlots) return;
  if (P.used == (int)P.ev0.size()) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess) return;
    if (cudaEventCreate(&b) != cudaSuccess) { cudaEventDestroy(a); return; }
    P.ev0.push_back(a);
    P.ev1.push_back(b);
    P.slot_id.push_back(0);
  }
  slot = P.used++;
  P.slot_id[slot] = id;
  cudaEventRecord(P.ev0[slot], st);
}
ProfScope::~ProfScope() {
  if (slot < 0) return;
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  cudaEventRecord(P.ev1[slot], st);
}

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

flint_status_t resolve(const flint_attn_params_t* in, Resolved* p) {
  if (!in) return FLINT_ERR_INVALID_ARG;
  if (in->dtype != FLINT_BF16 && in->dtype != FLINT_FP32) return FLINT_ERR_INVALID_ARG;
  if (in->total_tokens < 0 || in->num_docs < 1 || in->num_q_heads < 1 || in->num_kv_heads < 1)
    return FLINT_ERR_INVALID_ARG;
  if (in->num_q_heads % in->num_kv_heads != 0) return FLINT_ERR_INVALID_ARG;
  if (in->head_dim != kHeadDim) return FLINT_ERR_UNSUPPORTED;
  const int G = in->num_q_heads / in->num_kv_heads;
  if (in->compute_f16 && in->dtype != FLINT_FP32) return FLINT_ERR_INVALID_ARG;
  const bool tc = in->dtype == FLINT_BF16 || in->compute_f16;
  const bool g_tc = G == 1 || G == 2 || G == 4 || G == 8 || G == 16;
  if (tc && !g_tc) return FLINT_ERR_UNSUPPORTED;
  if ((long long)in->total_tokens * in->num_q_heads * in->head_dim > 0x7fffffffLL)
    return FLINT_ERR_INVALID_ARG;
  if (!(std::isfinite(in->rms_eps) && in->rms_eps >= 0.f)) return FLINT_ERR_INVALID_ARG;
  if (in->use_rope && !(std::isfinite(in->rope_theta) && in->rope_theta > 0.f))
    return FLINT_ERR_INVALID_ARG;
  if (!std::isfinite(in->softmax_scale) || in->softmax_scale < 0.f) return FLINT_ERR_INVALID_ARG;
  p->T = in->total_tokens;
  p->N = in->num_docs;
  p->H = in->num_q_heads;
  p->Hk = in->num_kv_heads;
  p->D = in->head_dim;
  p->G = G;
  p->W = in->window > 0 ? in->window : 0;
  p->rope = in->use_rope ? 1 : 0;
  p->theta = in->rope_theta;
  p->eps = in->rms_eps;
  p->scale = in->softmax_scale > 0.f ? in->softmax_scale : 1.0f / std::sqrt((float)kHeadDim);
  p->dtype = in->dtype;
  p->fp32_out = (in->fp32_out != 0 || in->dtype == FLINT_FP32) ? 1 : 0;
  p->tc = tc ? 1 : 0;
  // FP32 inputs take the split tensor-core path wherever its tiles fit the group
  // size; other group sizes run the CUDA-core kernels.
  p->x3 = (!tc && g_tc) ? 1 : 0;
  p->out_f16 = (in->compute_f16 && !in->fp32_out) ? 1 : 0;
  p->R = kTileRows / (G <= 128 ? G : 128);
  if (p->R < 1) p->R = 1;
  return FLINT_OK;
}

int sm_count() {
  static std::atomic<int> cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D 16-bit tensor [T][heads][128] (bf16 or fp16) with a (64, box_heads,
// box_tokens) box and 128-byte swizzle: one box fills one 128-row operand panel.
bool encode_3d(CUtensorMap* m, const void* base, int T, int heads, int box_heads, int box_tokens,
               CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)heads, (cuuint64_t)(T > 0 ? T : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)heads * kHeadDim * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_tokens};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, type, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

flint_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? FLINT_OK : FLINT_ERR_CUDA; }

#define FLINT_TRY(expr)                                    \
  do {                                                     \
    cudaError_t e_ = (expr);                               \
    if (e_ != cudaSuccess) return FLINT_ERR_CUDA;          \
  } while (0)

}  // namespace
}  // namespace flint

using namespace flint;

extern "C" size_t flint_attn_workspace_bytes(const flint_attn_params_t* params, int backward) {
  Resolved p;
  if (resolve(params, &p) != FLINT_OK) return 0;
  return make_layout(p, backward != 0).total;
}

namespace {
// fp16 copy of v, the B operand of the PV / P^T dO MMAs
// amax_v: the max |v| slot; the copy is v * 2^e (pow2_scale_exp).
cudaError_t convert_v(const Resolved& p, const void* v, __half* v16, const unsigned* amax_v,
                      cudaStream_t st) {
  const size_t n = (size_t)p.T * p.Hk * kHeadDim;
  if (p.dtype == FLINT_BF16)
    return launch_convert_f16(static_cast<const __nv_bfloat16*>(v), v16, n, amax_v, st);
  return launch_convert_f16(static_cast<const float*>(v), v16, n, amax_v, st);
}

// valid: per-document count of real tokens (trailing padding), or nullptr.
flint_status_t fwd_impl(const flint_attn_params_t* params, const void* q, const void* k,
                        const void* v, const void* q_norm_w, const void* k_norm_w,
                        const float* sink, const int32_t* cu_doc_lens, const int32_t* valid,
                        void* out, float* lse, void* workspace, size_t workspace_bytes,
                        void* stream) {
  Resolved p;
  flint_status_t s = resolve(params, &p);
  if (s != FLINT_OK) return s;
  // padding needs a tensor-core path (the CUDA-core FP32 kernels have none)
  if (valid && !p.tc && !p.x3) return FLINT_ERR_UNSUPPORTED;
  // With no tokens the [T, ...] tensors are empty and may be null.
  const bool no_tokens = p.T == 0;
  const void* tok16[] = {q, k, v, out};
  for (const void* ptr : tok16)
    if ((!ptr && !no_tokens) || !aligned(ptr, 16)) return FLINT_ERR_INVALID_ARG;
  const void* w16[] = {q_norm_w, k_norm_w};
  for (const void* ptr : w16)
    if (!ptr || !aligned(ptr, 16)) return FLINT_ERR_INVALID_ARG;
  if (!sink || !aligned(sink, 4) || !cu_doc_lens || !aligned(cu_doc_lens, 4) ||
      (!lse && !no_tokens) || !aligned(lse, 4))
    return FLINT_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p, false);
  if (!workspace || !aligned(workspace, 256)) return FLINT_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return FLINT_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, L.status);
  FLINT_TRY(cudaMemsetAsync(status, 0, 64 * sizeof(int), st));
  if (p.T == 0) return FLINT_OK;
  void* qh = at<void>(workspace, L.qhat);
  void* kh = at<void>(workspace, L.khat);
  unsigned* amax = reinterpret_cast<unsigned*>(status + kSlotAmaxDout);   // [dout, v]
  if (p.x3) {
    FLINT_TRY(launch_prologue_qk(p, q, q_norm_w, qh, k, k_norm_w, kh, cu_doc_lens, st,
                                 kHatSplit));
    int4* items = at<int4>(workspace, L.items_q);
    FLINT_TRY(launch_build_worklist(cu_doc_lens, valid, p, kModeQuery, p.R, items, status + 1,
                                    at<void>(workspace, L.sched_tmp), L.max_items_q, st));
    __half* vs = at<__half>(workspace, L.v16);
    FLINT_TRY(launch_absmax(p.dtype, nullptr, 0, v, (size_t)p.T * p.Hk * kHeadDim, amax,
                            cu_doc_lens, valid, p.N, p.H, p.Hk, st));
    FLINT_TRY(launch_convert_split(static_cast<const float*>(v), vs, p.T, p.Hk, amax + 1, st));
    const CUtensorMapDataType f16t = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tq, tk, tv;
    const int kv_box = x3_kv_box_tokens_fwd();
    if (!encode_3d(&tq, qh, p.T, 2 * p.H, p.G, p.R, f16t) ||
        !encode_3d(&tk, kh, p.T, 2 * p.Hk, 1, kv_box, f16t) ||
        !encode_3d(&tv, vs, p.T, 2 * p.Hk, 1, kv_box, f16t))
      return FLINT_ERR_CUDA;
    FLINT_TRY(launch_attn_fwd_x3(tq, tk, tv, p, sink, items, status + 1, L.max_items_q, amax,
                                 static_cast<float*>(out), lse, status, sm_count(), st));
    if (valid) FLINT_TRY(launch_pad_fill_fwd(p, cu_doc_lens, valid, sink, out, lse, st));
    return FLINT_OK;
  }
  FLINT_TRY(launch_prologue_qk(p, q, q_norm_w, qh, k, k_norm_w, kh, cu_doc_lens, st,
                               p.tc ? kHatF16 : kHatInput));
  if (!p.tc) {
    return cuda_status(launch_attn_fwd_fp32(p, (const float*)qh, (const float*)kh,
                                            (const float*)v, sink, cu_doc_lens, (float*)out, lse,
                                            st));
  }
  int4* items = at<int4>(workspace, L.items_q);
  FLINT_TRY(launch_build_worklist(cu_doc_lens, valid, p, kModeQuery, 2 * p.R, items, status + 1,
                                  at<void>(workspace, L.sched_tmp), L.max_items_q, st));
  __half* v16 = at<__half>(workspace, L.v16);
  FLINT_TRY(launch_absmax(p.dtype, nullptr, 0, v, (size_t)p.T * p.Hk * kHeadDim, amax,
                          cu_doc_lens, valid, p.N, p.H, p.Hk, st));
  FLINT_TRY(convert_v(p, v, v16, amax + 1, st));
  const CUtensorMapDataType f16t = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tq, tk, tv;
  const int kv_box = fwd_kv_box_tokens();
  if (!encode_3d(&tq, qh, p.T, p.H, p.G, p.R, f16t) ||
      !encode_3d(&tk, kh, p.T, p.Hk, 1, kv_box, f16t) ||
      !encode_3d(&tv, v16, p.T, p.Hk, 1, kv_box, f16t))
    return FLINT_ERR_CUDA;
  FLINT_TRY(launch_attn_fwd_sm100_impl(tq, tk, tv, p, sink, items, status + 1, L.max_items_q,
                                       amax + 1, out, lse, status, sm_count(), st));
  if (valid) FLINT_TRY(launch_pad_fill_fwd(p, cu_doc_lens, valid, sink, out, lse, st));
  return FLINT_OK;
}

flint_status_t bwd_impl(const flint_attn_params_t* params, const void* q, const void* k,
                        const void* v, const void* q_norm_w, const void* k_norm_w,
                        const float* sink, const int32_t* cu_doc_lens, const int32_t* valid,
                        const void* out, const float* lse, const void* dout, void* dq, void* dk,
                        void* dv, float* dq_norm_w, float* dk_norm_w, float* dsink,
                        void* workspace, size_t workspace_bytes, void* stream) {
  Resolved p;
  flint_status_t s = resolve(params, &p);
  if (s != FLINT_OK) return s;
  // padding needs a tensor-core path (the CUDA-core FP32 kernels have none)
  if (valid && !p.tc && !p.x3) return FLINT_ERR_UNSUPPORTED;
  // With no tokens the [T, ...] tensors are empty and may be null.
  const bool no_tokens = p.T == 0;
  const void* tok16[] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* ptr : tok16)
    if ((!ptr && !no_tokens) || !aligned(ptr, 16)) return FLINT_ERR_INVALID_ARG;
  const void* w16[] = {q_norm_w, k_norm_w};
  for (const void* ptr : w16)
    if (!ptr || !aligned(ptr, 16)) return FLINT_ERR_INVALID_ARG;
  if ((!lse && !no_tokens) || !aligned(lse, 4)) return FLINT_ERR_INVALID_ARG;
  const void* vec4[] = {sink, cu_doc_lens, dq_norm_w, dk_norm_w, dsink};
  for (const void* ptr : vec4)
    if (!ptr || !aligned(ptr, 4)) return FLINT_ERR_INVALID_ARG;
  const WsLayout L = make_layout(p, true);
  if (!workspace || !aligned(workspace, 256)) return FLINT_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return FLINT_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, L.status);
  FLINT_TRY(cudaMemsetAsync(status, 0, 64 * sizeof(int), st));
  if (p.T == 0) {
    FLINT_TRY(cudaMemsetAsync(dsink, 0, p.H * sizeof(float), st));
    FLINT_TRY(cudaMemsetAsync(dq_norm_w, 0, kHeadDim * sizeof(float), st));
    FLINT_TRY(cudaMemsetAsync(dk_norm_w, 0, kHeadDim * sizeof(float), st));
    return FLINT_OK;
  }
  void* qh = at<void>(workspace, L.qhat);
  void* kh = at<void>(workspace, L.khat);
  float* dvec = at<float>(workspace, L.dvec);
  float* part = at<float>(workspace, L.part);
  float* dq_acc = at<float>(workspace, L.dq_acc);
  float* dk_acc = at<float>(workspace, L.dk_acc);
  const bool f16 = p.tc || p.x3;   // tensor-core operands of the backward are fp16
  __half* dout16 = f16 ? at<__half>(workspace, L.dout16) : nullptr;
  __half* v16 = f16 ? at<__half>(workspace, L.v16) : nullptr;
  unsigned* amax = reinterpret_cast<unsigned*>(status + kSlotAmaxDout);   // [dout, v]
  if (f16)
    FLINT_TRY(launch_absmax(p.dtype, dout, (size_t)p.T * p.H * kHeadDim, v,
                            (size_t)p.T * p.Hk * kHeadDim, amax, cu_doc_lens, valid, p.N, p.H,
                            p.Hk, st));
  FLINT_TRY(launch_prologue_qk(p, q, q_norm_w, qh, k, k_norm_w, kh, cu_doc_lens, st,
                               p.x3 ? kHatSplit : (p.tc ? kHatF16 : kHatInput)));
  FLINT_TRY(launch_bwd_preprocess(p, out, dout, lse, sink, dvec, part, dsink, dout16,
                                  f16 ? amax : nullptr, st, p.x3));
  if (p.x3) {
    int4* items_kv = at<int4>(workspace, L.items_kv);
    int4* items_q1 = at<int4>(workspace, L.items_q1);
    FLINT_TRY(launch_build_worklists2(cu_doc_lens, valid, p, kModeKey, kTileKeys, items_kv,
                                      status + 2, at<void>(workspace, L.sched_tmp),
                                      L.max_items_kv, kModeQuery, p.R, items_q1, status + 3,
                                      at<void>(workspace, L.sched_tmp2), L.max_items_q1, st));
    FLINT_TRY(launch_convert_split(static_cast<const float*>(v), v16, p.T, p.Hk, amax + 1, st));
    const CUtensorMapDataType f16t = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const int rows64 = x3_q_box_rows_dkv(), keys_dq = x3_kv_box_tokens_dq();
    CUtensorMap tq64, tk128, tdo64, tk64, tv64;
    if (!encode_3d(&tq64, qh, p.T, 2 * p.H, p.G, rows64 / p.G, f16t) ||
        !encode_3d(&tk128, kh, p.T, 2 * p.Hk, 1, kTileKeys, f16t) ||
        !encode_3d(&tdo64, dout16, p.T, 2 * p.H, p.G, rows64 / p.G, f16t) ||
        !encode_3d(&tk64, kh, p.T, 2 * p.Hk, 1, keys_dq, f16t) ||
        !encode_3d(&tv64, v16, p.T, 2 * p.Hk, 1, keys_dq, f16t))
      return FLINT_ERR_CUDA;
    FLINT_TRY(launch_attn_bwd_x3(tq64, tk128, tdo64, tk64, tv64, p, lse, dvec, amax,
                                 static_cast<const __half*>(qh), dout16, v16, items_kv,
                                 status + 2, L.max_items_kv, items_q1, status + 3,
                                 L.max_items_q1, dq_acc, dk_acc, static_cast<float*>(dv), status,
                                 sm_count(), st));
    if (valid)
      FLINT_TRY(launch_pad_fill_bwd(p, cu_doc_lens, valid, dq_acc, dk_acc, dv, 1, st));
  } else if (!p.tc) {
    FLINT_TRY(launch_attn_bwd_fp32(p, (const float*)qh, (const float*)kh, (const float*)v,
                                   (const float*)dout, lse, dvec, cu_doc_lens, dq_acc, dk_acc,
                                   (float*)dv, st));
  } else {
    int4* items_kv = at<int4>(workspace, L.items_kv);
    int4* items_q1 = at<int4>(workspace, L.items_q1);
    FLINT_TRY(launch_build_worklists2(cu_doc_lens, valid, p, kModeKey, kTileKeys, items_kv,
                                      status + 2, at<void>(workspace, L.sched_tmp),
                                      L.max_items_kv, kModeQuery, p.R, items_q1, status + 3,
                                      at<void>(workspace, L.sched_tmp2), L.max_items_q1, st));
    FLINT_TRY(convert_v(p, v, v16, amax + 1, st));
    const CUtensorMapDataType f16t = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tq, tk, tv, tdo;
    if (!encode_3d(&tq, qh, p.T, p.H, p.G, p.R, f16t) ||
        !encode_3d(&tk, kh, p.T, p.Hk, 1, kTileKeys, f16t) ||
        !encode_3d(&tv, v16, p.T, p.Hk, 1, kTileKeys, f16t) ||
        !encode_3d(&tdo, dout16, p.T, p.H, p.G, p.R, f16t))
      return FLINT_ERR_CUDA;
    FLINT_TRY(launch_attn_bwd_sm100_impl(tq, tk, tv, tdo, p, lse, dvec, amax, items_kv,
                                         status + 2, L.max_items_kv, items_q1, status + 3,
                                         L.max_items_q1,
                                         dq_acc, dk_acc, dv, status, sm_count(), st));
    if (valid)
      FLINT_TRY(launch_pad_fill_bwd(p, cu_doc_lens, valid, dq_acc, dk_acc, dv, p.fp32_out, st));
  }
  float* part_q = part + (size_t)kPartBlocks * p.H;
  float* part_k = part_q + (size_t)kPartBlocks * kHeadDim;
  FLINT_TRY(launch_bwd_epilogue(p, q, q_norm_w, dq_acc, dq, dq_norm_w, part_q, p.H, cu_doc_lens,
                                st));
  FLINT_TRY(launch_bwd_epilogue(p, k, k_norm_w, dk_acc, dk, dk_norm_w, part_k, p.Hk, cu_doc_lens,
                                st));
  return FLINT_OK;
}

bool padded_args_ok(const flint_attn_params_t* params, const int32_t* valid_lens) {
  return params && valid_lens && aligned(valid_lens, 4);
}
}  // namespace

extern "C" flint_status_t flint_attn_fwd(const flint_attn_params_t* params, const void* q,
                                         const void* k, const void* v, const void* q_norm_w,
                                         const void* k_norm_w, const float* sink,
                                         const int32_t* cu_doc_lens, void* out, float* lse,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  return fwd_impl(params, q, k, v, q_norm_w, k_norm_w, sink, cu_doc_lens, nullptr, out, lse,
                  workspace, workspace_bytes, stream);
}

extern "C" flint_status_t flint_attn_bwd(const flint_attn_params_t* params, const void* q,
                                         const void* k, const void* v, const void* q_norm_w,
                                         const void* k_norm_w, const float* sink,
                                         const int32_t* cu_doc_lens, const void* out,
                                         const float* lse, const void* dout, void* dq, void* dk,
                                         void* dv, float* dq_norm_w, float* dk_norm_w,
                                         float* dsink, void* workspace, size_t workspace_bytes,
                                         void* stream) {
  return bwd_impl(params, q, k, v, q_norm_w, k_norm_w, sink, cu_doc_lens, nullptr, out, lse,
                  dout, dq, dk, dv, dq_norm_w, dk_norm_w, dsink, workspace, workspace_bytes,
                  stream);
}

extern "C" flint_status_t flint_attn_fwd_padded(const flint_attn_params_t* params, const void* q,
                                                const void* k, const void* v,
                                                const void* q_norm_w, const void* k_norm_w,
                                                const float* sink, const int32_t* cu_doc_lens,
                                                const int32_t* valid_lens, void* out, float* lse,
                                                void* workspace, size_t workspace_bytes,
                                                void* stream) {
  if (!padded_args_ok(params, valid_lens)) return FLINT_ERR_INVALID_ARG;
  return fwd_impl(params, q, k, v, q_norm_w, k_norm_w, sink, cu_doc_lens, valid_lens, out, lse,
                  workspace, workspace_bytes, stream);
}

extern "C" flint_status_t flint_attn_bwd_padded(
    const flint_attn_params_t* params, const void* q, const void* k, const void* v,
    const void* q_norm_w, const void* k_norm_w, const float* sink, const int32_t* cu_doc_lens,
    const int32_t* valid_lens, const void* out, const float* lse, const void* dout, void* dq,
    void* dk, void* dv, float* dq_norm_w, float* dk_norm_w, float* dsink, void* workspace,
    size_t workspace_bytes, void* stream) {
  if (!padded_args_ok(params, valid_lens)) return FLINT_ERR_INVALID_ARG;
  return bwd_impl(params, q, k, v, q_norm_w, k_norm_w, sink, cu_doc_lens, valid_lens, out, lse,
                  dout, dq, dk, dv, dq_norm_w, dk_norm_w, dsink, workspace, workspace_bytes,
                  stream);
}

// ------------------------------------------------------------------ decode
namespace {
struct DecodeLayout {
  size_t status, counters, part_o, part_ml, total;   // status and counters are contiguous
};
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

flint_status_t resolve_decode(const flint_decode_params_t* d, DecodeLayout* L) {
  if (!d) return FLINT_ERR_INVALID_ARG;
  if (d->dtype != FLINT_BF16) return d->dtype == FLINT_FP32 ? FLINT_ERR_UNSUPPORTED
                                                           : FLINT_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return FLINT_ERR_UNSUPPORTED;
  if (d->batch < 1 || d->cache_capacity < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 ||
      d->num_q_heads % d->num_kv_heads != 0)
    return FLINT_ERR_INVALID_ARG;
  if (d->num_q_heads / d->num_kv_heads > 16) return FLINT_ERR_UNSUPPORTED;
  if (!(d->rms_eps >= 0.f) || !(d->softmax_scale >= 0.f) ||
      (d->use_rope && !(d->rope_theta > 0.f)))
    return FLINT_ERR_INVALID_ARG;
  const size_t B = d->batch, H = d->num_q_heads;
  const size_t S = decode_splits_max(d->cache_capacity, d->window);
  L->status = 0;
  L->counters = 64 * sizeof(int);
  L->part_o = round256(L->counters + B * d->num_kv_heads * sizeof(int));
  L->part_ml = L->part_o + round256(B * H * S * kHeadDim * sizeof(float));
  L->total = L->part_ml + round256(B * H * S * 2 * sizeof(float));
  return FLINT_OK;
}
}  // namespace

extern "C" size_t flint_attn_decode_workspace_bytes(const flint_decode_params_t* params) {
  DecodeLayout L;
  return resolve_decode(params, &L) == FLINT_OK ? L.total : 0;
}

extern "C" flint_status_t flint_attn_decode(const flint_decode_params_t* params, const void* q,
                                            const void* k, const void* v, const void* q_norm_w,
                                            const void* k_norm_w, const float* sink,
                                            const int32_t* cache_lens, void* k_cache,
                                            void* v_cache, void* out, float* lse,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream) {
  DecodeLayout L;
  flint_status_t s = resolve_decode(params, &L);
  if (s != FLINT_OK) return s;
  const void* vec16[] = {q, k, v, q_norm_w, k_norm_w, k_cache, v_cache, out};
  for (const void* ptr : vec16)
    if (!ptr || !aligned(ptr, 16)) return FLINT_ERR_INVALID_ARG;
  if (!sink || !aligned(sink, 4) || !cache_lens || !aligned(cache_lens, 4) || !lse ||
      !aligned(lse, 4))
    return FLINT_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256)) return FLINT_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return FLINT_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int* status = at<int>(workspace, L.status);
  FLINT_TRY(cudaMemsetAsync(status, 0, L.part_o, st));    // status word and split counters
  DecodeLaunch D;
  D.B = params->batch; D.C = params->cache_capacity;
  D.H = params->num_q_heads; D.Hk = params->num_kv_heads;
  D.W = params->window; D.rope = params->use_rope ? 1 : 0; D.out_f32 = params->fp32_out ? 1 : 0;
  D.num_sms = sm_count();
  D.theta = params->rope_theta; D.eps = params->rms_eps;
  D.scale = params->softmax_scale > 0.f ? params->softmax_scale
                                        : 1.0f / sqrtf((float)kHeadDim);
  D.q = q; D.k = k; D.v = v; D.wq = q_norm_w; D.wk = k_norm_w;
  D.sink = sink; D.lens = cache_lens; D.kc = k_cache; D.vc = v_cache;
  D.counters = at<int>(workspace, L.counters);
  D.part_o = at<float>(workspace, L.part_o);
  D.part_ml = at<float>(workspace, L.part_ml);
  D.out = out; D.lse = lse; D.status = status;
  return cuda_status(launch_decode(D, st));
}

extern "C" flint_status_t flint_attn_check_status(void* workspace, void* stream) {
  if (!workspace || !aligned(workspace, 256)) return FLINT_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLINT_ERR_CUDA;
  int host = 0;
  if (cudaMemcpy(&host, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return FLINT_ERR_CUDA;
  if (host != 0) {
    const int zero = 0;
    if (cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return FLINT_ERR_CUDA;
    if (host & flint::kStatusSmemAlign) return FLINT_ERR_CUDA;
    if (host & flint::kStatusDecodeRange) return FLINT_ERR_INVALID_ARG;
    return FLINT_ERR_TIMEOUT;
  }
  return FLINT_OK;
}

extern "C" void flint_attn_profile_enable(int enable) {
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  P.enabled = enable != 0;
}

extern "C" int flint_attn_profile_collect(int max_kernels, const char** names, double* total_ms,
                                          long long* launches) {
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  for (int i = 0; i < P.used; ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(P.ev1[i]) == cudaSuccess &&
        cudaEventElapsedTime(&ms, P.ev0[i], P.ev1[i]) == cudaSuccess) {
      P.total_ms[P.slot_id[i]] += ms;
      P.launches[P.slot_id[i]] += 1;
    }
  }
  P.used = 0;
  for (int k = 0; k < kNumKernelIds && k < max_kernels; ++k) {
    if (names) names[k] = kKernelNames[k];
    if (total_ms) total_ms[k] = P.total_ms[k];
    if (launches) launches[k] = P.launches[k];
  }
  return kNumKernelIds;
}

extern "C" void flint_attn_profile_reset(void) {
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  for (int k = 0; k < kNumKernelIds; ++k) {
    P.total_ms[k] = 0.0;
    P.launches[k] = 0;
  }
}

extern "C" long long flint_attn_launch_count(void) {
  Prof& P = prof();
  std::lock_guard<std::mutex> g(P.mu);
  return P.launches_total;
}

extern "C" flint_status_t flint_attn_exp2_poly(const float* x, float* y, int32_t n, void* stream) {
  if (n < 0 || (n & 1) || (n > 0 && (!x || !y || !aligned(x, 4) || !aligned(y, 4))))
    return FLINT_ERR_INVALID_ARG;
  return cuda_status(launch_exp2_poly(x, y, n, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" flint_status_t flint_attn_selftest_wait(int64_t wait_cycles, int32_t arrive_first,
                                                   int32_t* status, void* stream) {
  if (!status || !aligned(status, 256) || wait_cycles < 1 || wait_cycles > FLINT_WAIT_CYCLES)
    return FLINT_ERR_INVALID_ARG;
  return cuda_status(launch_wait_selftest((long long)wait_cycles, arrive_first != 0 ? 1 : 0,
                                          status, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" const char* flint_status_string(flint_status_t s) {
  switch (s) {
    case FLINT_OK: return "ok";
    case FLINT_ERR_INVALID_ARG: return "invalid argument";
    case FLINT_ERR_UNSUPPORTED: return "unsupported configuration";
    case FLINT_ERR_WORKSPACE: return "workspace too small";
    case FLINT_ERR_CUDA: return "CUDA error";
    case FLINT_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

extern "C" const char* flint_attn_version(void) { return "flint_attn 0.1 sm_100a"; }
