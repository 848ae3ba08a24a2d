// decode.cu - flint_attn_decode: the forward of one new token per sequence
// over a KV cache (serving).
//
// What it computes is flint_attn_fwd's definition restricted to the last row
// of each sequence (Flint layers page, nemo_automodel.components.models.flint.
// layers: FlintAttention.forward, causal attention in which the sink is one
// more softmax category with a zero value vector; per-head RMSNorm then NeoX
// RoPE; Flint config page: the window includes the current token). Sequence b has p = cache_lens[b] tokens cached;
// the new token's normalised, rotated key and its value go into slot p, and
// the new query attends to slots max(0, p - W + 1) .. p plus the sink.
//
// Decode is bound by HBM: every key costs 512 bytes of K and V and feeds only
// the G query heads of its group. One kernel, grid (splits, Hk, B); each CTA
// covers one chunk of one (sequence, KV head) window (the splits divide the
// largest window evenly in multiples of 16 keys; about five CTAs per SM, or for
// batches with 1 to 1.5 times as many pairs as resident CTA slots two full
// waves of one- and two-split pairs, see decode_split_plan):
//   * it normalises and rotates the G query rows of its group itself (RMSNorm
//     + RoPE at position p, a warp per row, kept in fp32 and pre-scaled by
//     softmax_scale * log2(e)); the CTA whose chunk holds slot p also computes
//     k_hat and appends k_hat (rounded to bf16) and v to the caches before it
//     stages them. The raw rows are requested together with cache_lens[b], and
//     each warp's first K/V step is staged before the rows are normalised, so
//     a CTA's fixed start-up latency overlaps its first loads;
//   * its 4 warps take 16-key steps, each staging its own K and V rows into
//     shared memory with cp.async (double buffered, coalesced 16-byte copies
//     of the head-major cache). The two small contractions run on mma.sync
//     m16n8k16 (bf16 in, fp32 accumulate) with q_hat split into bf16 hi + lo
//     parts. For G <= 8, S = Q K^T takes the hi parts as rows 0-7 and the lo
//     parts as rows 8-15 of one A operand (each lane adds its two halves), and
//     the PV product runs transposed, O^T += V^T P^T, so the 8 heads are the
//     MMA's N and the P fragment a lane holds is already the B operand; for
//     9 <= G <= 16 the heads are the 16 rows of both products. Tensor
//     throughput is not the limit here, so the per-SM tcgen05/TMEM machinery
//     of the prefill kernels would add nothing; K fragments come from
//     ldmatrix, V fragments from ldmatrix.trans, and P is the S accumulator
//     re-packed in registers. Online softmax with a lazily rescaled running
//     max;
//   * the warps merge in shared memory and the CTA writes one unnormalised
//     partial (m, l, O); the last CTA of the (sequence, KV head) to finish (an
//     atomic counter per pair) folds the sink in once (m = sink, l = 1 before
//     the partials), normalises and writes out and LSE.
#include <cuda_bf16.h>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {

namespace {

constexpr int kDecWarps = 4;
constexpr int kDecThreads = 32 * kDecWarps;
constexpr int kStepKeys = 16;                  // keys per warp step
constexpr int kRowBytes = 2 * kHeadDim + 16;   // a key row + 16 B: ldmatrix rows hit distinct banks
constexpr int kStageBytes = 2 * kStepKeys * kRowBytes;              // K and V rows of one step
constexpr int kDecStages = 2;                                       // steps in flight per warp
constexpr int kWarpSmem = kDecStages * kStageBytes;
constexpr int kAttnSmem = kDecWarps * kWarpSmem;
constexpr int kMergeBytes = kDecWarps * 16 * (kHeadDim + 2) * 4;    // per-warp m, l, O for merging
static_assert(kMergeBytes <= kAttnSmem && 16 * kHeadDim * 4 <= kStageBytes,
              "merge area and q_hat rows must fit in the staging area");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;               // log2 units

struct DecArgs {
  int B, C, H, Hk, G, W, rope, splits, out_f32;   // splits: stride of the partials
  int chunk_a, chunk_b, pair_split;  // keys per chunk: pairs < pair_split chunk_a, the rest chunk_b
  float theta, eps, scale_log2;
  const __nv_bfloat16 *q, *k, *v, *wq, *wk;
  const float* sink;
  const int* lens;
  __nv_bfloat16 *kc, *vc;
  int* counters;     // [B * Hk], zero at the start of a call
  float* part_o;     // [B, H, splits, D]
  float* part_ml;    // [B, H, splits, 2]
  void* out;
  float* lse;        // [B, H]
  int* status;
};

__device__ __forceinline__ bool pos_ok(const DecArgs& a, int p) { return p >= 0 && p < a.C; }

__device__ __forceinline__ int window_lo(const DecArgs& a, int p) {
  return a.W > 0 ? max(0, p - a.W + 1) : 0;
}

// ---------------------------------------------------------------------------
// Prologue of one row: RMSNorm with weight w, then NeoX RoPE from the table.
// A warp owns the row, lane l channels 4l..4l+3; channel c's RoPE partner
// c +- 64 is in lane l ^ 16.
// ---------------------------------------------------------------------------
// xr, wr: the lane's 4 bf16 channels of the row and of the weight.
__device__ __forceinline__ void warp_row_prologue(uint2 xr, uint2 wr, const float* cs,
                                                  const float* sn, bool rope, float eps,
                                                  float (&y)[4]) {
  const int lane = threadIdx.x & 31;
  const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xr);
  const __nv_bfloat162* wh = reinterpret_cast<const __nv_bfloat162*>(&wr);
  float xv[4], wv[4];
  xv[0] = __low2float(xh[0]); xv[1] = __high2float(xh[0]);
  xv[2] = __low2float(xh[1]); xv[3] = __high2float(xh[1]);
  wv[0] = __low2float(wh[0]); wv[1] = __high2float(wh[0]);
  wv[2] = __low2float(wh[1]); wv[3] = __high2float(wh[1]);
  float ss = xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float r = rsqrtf(ss * (1.0f / kHeadDim) + eps);
#pragma unroll
  for (int e = 0; e < 4; ++e) y[e] = xv[e] * r * wv[e];
  if (rope) {
    const bool lo_half = lane < 16;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float partner = __shfl_xor_sync(0xffffffffu, y[e], 16);
      const int j = (4 * lane + e) & (kHeadDim / 2 - 1);
      y[e] = lo_half ? (y[e] * cs[j] - partner * sn[j]) : (y[e] * cs[j] + partner * sn[j]);
    }
  }
}

// ---------------------------------------------------------------------------
// Split attention
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// 16-byte global -> shared copy; src_bytes = 0 writes zeros (src still valid).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  return pack_bf16x2(lo, hi);
}
__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
// the two bf16 halves of a packed pair as floats
__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// kPack (G <= 8): the 16 rows of the S MMA's A operand hold q_hat's bf16 hi
// parts (rows 0-7) and lo parts (rows 8-15) of the same heads, so one MMA
// gives both partial products and a lane adds its own c0 + c2 (c1 + c3); the
// PV product then runs transposed (O^T += V^T P^T: the 8 heads are the MMA's
// N, and the P fragment a lane holds is already the B operand). This halves
// the MMAs, the exponentials and the O registers of the padded layout.
// Otherwise (9 <= G <= 16) the rows are the heads and the hi and lo parts take
// one MMA each.
template <bool kPack>
__global__ void __launch_bounds__(kDecThreads, 3) decode_attn_kernel(const DecArgs a) {
  extern __shared__ __align__(128) uint8_t dsmem[];
  // q_hat rows of the group (log2 units), only until they are in registers: in
  // warp 0's second staging buffer, which is first filled inside the step loop,
  // so each warp's first step can be staged while the rows are computed
  float (*qs)[kHeadDim] = reinterpret_cast<float (*)[kHeadDim]>(dsmem + kStageBytes);
  __shared__ float cs[kHeadDim / 2], sn[kHeadDim / 2];
  __shared__ int last_flag;
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  // The raw rows this CTA normalises (the warp's query rows, and the new key and
  // value for the CTA that appends them) are requested with cache_lens[b], so
  // the loads overlap instead of following one another.
  constexpr int kRowsPerWarp = 16 / kDecWarps;       // G <= 16
  const size_t src = ((size_t)b * a.Hk + g) * kHeadDim;
  uint2 xq[kRowsPerWarp], xk = make_uint2(0u, 0u), xv = make_uint2(0u, 0u);
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int r = warp + kDecWarps * i;
    xq[i] = make_uint2(0u, 0u);
    if (r < a.G)
      xq[i] = *reinterpret_cast<const uint2*>(a.q + ((size_t)b * a.H + g * a.G + r) * kHeadDim +
                                              4 * lane);
  }
  const uint2 wq = *reinterpret_cast<const uint2*>(a.wq + 4 * lane);
  uint2 wk = make_uint2(0u, 0u);
  if (warp == kDecWarps - 1) {
    xk = *reinterpret_cast<const uint2*>(a.k + src + 4 * lane);
    xv = *reinterpret_cast<const uint2*>(a.v + src + 4 * lane);
    wk = *reinterpret_cast<const uint2*>(a.wk + 4 * lane);
  }
  const int p = __ldg(a.lens + b);
  if (!pos_ok(a, p)) {
    if (s == 0 && g == 0 && threadIdx.x == 0) atomicOr(a.status, kStatusDecodeRange);
    return;
  }
  const int lo = window_lo(a, p);
  const int chunk = (b * a.Hk + g < a.pair_split) ? a.chunk_a : a.chunk_b;
  const int k0 = lo + s * chunk;
  if (k0 > p) return;                                // this split has no keys
  const int k1 = min(k0 + chunk, p + 1);             // keys [k0, k1)
  const int nsplit = (p - lo + chunk) / chunk;
  const bool owner = k1 == p + 1;                    // this CTA reads slot p
  const size_t row0 = ((size_t)b * a.Hk + g) * a.C;  // slot 0 of this (sequence, KV head)
  const __nv_bfloat16* kbase = a.kc + row0 * kHeadDim;
  const __nv_bfloat16* vbase = a.vc + row0 * kHeadDim;

  const uint32_t wsm = smem_u32(dsmem) + warp * kWarpSmem;
  const int nsteps = (k1 - k0 + kStepKeys - 1) / kStepKeys;
  auto issue = [&](int step, int buf) {              // stage K and V rows of a step
    const int kb = k0 + step * kStepKeys;
    const uint32_t ks = wsm + buf * kStageBytes, vs = ks + kStepKeys * kRowBytes;
#pragma unroll
    for (int i = 0; i < (kStepKeys * 16) / 32; ++i) {
      const int c = lane + 32 * i;                   // 16-byte chunk of the step
      const int key = c >> 4, part = c & 15;
      const int j = kb + key;
      const bool in = j < k1;
      const size_t off = (size_t)(in ? j : k0) * kHeadDim + part * 8;
      cp_async16(ks + key * kRowBytes + part * 16, kbase + off, in ? 16 : 0);
      cp_async16(vs + key * kRowBytes + part * 16, vbase + off, in ? 16 : 0);
    }
  };
  // Each warp's first step goes into its first buffer now, unless it holds slot
  // p, which is staged only after the new key and value are written there.
  static_assert(kDecStages == 2, "one step staged ahead");
  const bool first_early = warp < nsteps && !(owner && p < k0 + (warp + 1) * kStepKeys);
  if (first_early) issue(warp, 0);

  // ---- prologue: RoPE table, the group's q_hat rows, and (owner) the append
  if (a.rope && threadIdx.x < kHeadDim / 2) {
    const int j = threadIdx.x;
    double inv_freq = exp2(-(2.0 * j / kHeadDim) * log2((double)a.theta));
    double ang = (double)p * inv_freq;
    const double two_pi = 6.283185307179586476925286766559;
    ang -= two_pi * rint(ang / two_pi);
    float sv, cv;
    sincosf((float)ang, &sv, &cv);
    cs[j] = cv;
    sn[j] = sv;
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < kRowsPerWarp; ++i) {
    const int r = warp + kDecWarps * i;
    if (r < a.G) {
      float y[4];
      warp_row_prologue(xq[i], wq, cs, sn, a.rope, a.eps, y);
#pragma unroll
      for (int e = 0; e < 4; ++e) qs[r][4 * lane + e] = y[e] * a.scale_log2;
    }
  }
  if (owner && warp == kDecWarps - 1) {
    float y[4];
    warp_row_prologue(xk, wk, cs, sn, a.rope, a.eps, y);
    uint2 kb;
    kb.x = pack_bf16x2(y[0], y[1]);
    kb.y = pack_bf16x2(y[2], y[3]);
    const size_t dst = (row0 + p) * kHeadDim + 4 * lane;
    *reinterpret_cast<uint2*>(a.kc + dst) = kb;
    *reinterpret_cast<uint2*>(a.vc + dst) = xv;
  }
  __threadfence_block();
  __syncthreads();                                   // slot p written before it is staged

  // q_hat fragments, bf16 hi + lo parts (zero past G)
  constexpr int kQParts = kPack ? 1 : 2;
  uint32_t qa[kQParts][8][4];
  {
    const bool v0 = gid < a.G, v1 = gid + 8 < a.G;
    const float* q0 = qs[gid];
    const float* q1 = qs[gid + 8];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        // a0: (row gid, k 2tig..+1), a1: (row gid+8, same), a2: (row gid, k+8),
        // a3: (row gid+8, k+8)
        const int d = kk * 16 + 2 * tig + ((r & 2) ? 8 : 0);
        const bool hv = (kPack || !(r & 1)) ? v0 : v1;
        const float* qr = (kPack || !(r & 1)) ? q0 : q1;
        float x0 = 0.f, x1 = 0.f;
        if (hv) {
          const float2 t = *reinterpret_cast<const float2*>(qr + d);
          x0 = t.x;
          x1 = t.y;
        }
        const float h0f = bf16_round(x0), h1f = bf16_round(x1);
        if constexpr (kPack) {
          qa[0][kk][r] = (r & 1) ? bf16x2_bits(x0 - h0f, x1 - h1f) : bf16x2_bits(h0f, h1f);
        } else {
          qa[0][kk][r] = bf16x2_bits(h0f, h1f);
          qa[1][kk][r] = bf16x2_bits(x0 - h0f, x1 - h1f);
        }
      }
    }
  }

  __syncthreads();                                   // every warp holds its fragments

  // kPack: O^T, 8 m-tiles of 16 dims x the 8 heads (lane: dims mt*16 + gid and
  // + 8, heads 2tig, 2tig+1); otherwise O, 16 n-tiles of 8 dims x 16 head rows
  constexpr int kOTiles = kPack ? 8 : 16;
  float o[kOTiles][4];
#pragma unroll
  for (int n = 0; n < kOTiles; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // rows (heads) gid, gid + 8

  // Each iteration commits one group (empty past the last step), so the wait
  // count below is constant: the group of the step being computed is done. The
  // first group holds the warp's first step, staged early or now.
  if (warp < nsteps && !first_early) issue(warp, 0);
  cp_async_commit();
  int it = 0;
  for (int step = warp; step < nsteps; step += kDecWarps, ++it) {
    const int buf = it % kDecStages;
    const int ahead = step + kDecWarps * (kDecStages - 1);
    if (ahead < nsteps) issue(ahead, (it + kDecStages - 1) % kDecStages);
    cp_async_commit();
    cp_async_wait<kDecStages - 1>();
    __syncwarp();
    const uint32_t ks = wsm + buf * kStageBytes, vs = ks + kStepKeys * kRowBytes;
    const int kb = k0 + step * kStepKeys;

    // S = q_hat K^T for keys kb .. kb+15 (two 8-key n-tiles); sc[nt][0..1] row
    // gid, sc[nt][2..3] row gid + 8 (heads 8-15, !kPack only)
    float sc[2][4];
    if constexpr (kPack) {
      // even and odd k-steps accumulate apart: four independent chains of four
      float acc[2][2][4];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          acc[nt][h][0] = acc[nt][h][1] = acc[nt][h][2] = acc[nt][h][3] = 0.f;
#pragma unroll
      for (int kp = 0; kp < 4; ++kp) {               // pairs of 16-dim k-steps
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t bk[4];
          const int key = nt * 8 + (lane & 7);
          const int col = kp * 32 + (lane >> 3) * 8;   // dims
          ldsm_x4(ks + key * kRowBytes + col * 2, bk);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int kk = 2 * kp + h;
            mma_bf16_16816(acc[nt][h], qa[0][kk][0], qa[0][kk][1], qa[0][kk][2], qa[0][kk][3],
                           bk[2 * h], bk[2 * h + 1]);
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {               // hi part (row gid) + lo part (row gid + 8)
        sc[nt][0] = (acc[nt][0][0] + acc[nt][1][0]) + (acc[nt][0][2] + acc[nt][1][2]);
        sc[nt][1] = (acc[nt][0][1] + acc[nt][1][1]) + (acc[nt][0][3] + acc[nt][1][3]);
        sc[nt][2] = sc[nt][3] = -INFINITY;
      }
    } else {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {             // pairs of 16-dim k-steps
          uint32_t bk[4];
          const int key = nt * 8 + (lane & 7);
          const int col = kp * 32 + (lane >> 3) * 8; // dims
          ldsm_x4(ks + key * kRowBytes + col * 2, bk);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int kk = 2 * kp + h;
            mma_bf16_16816(sc[nt], qa[0][kk][0], qa[0][kk][1], qa[0][kk][2], qa[0][kk][3],
                           bk[2 * h], bk[2 * h + 1]);
            mma_bf16_16816(sc[nt], qa[1][kk][0], qa[1][kk][1], qa[1][kk][2], qa[1][kk][3],
                           bk[2 * h], bk[2 * h + 1]);
          }
        }
      }
    }
    // mask keys past the end of the range; c0,c1 = row gid, c2,c3 = row gid + 8
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int j = kb + nt * 8 + 2 * tig;
      if (j >= k1) sc[nt][0] = sc[nt][2] = -INFINITY;
      if (j + 1 >= k1) sc[nt][1] = sc[nt][3] = -INFINITY;
    }
    float mx0 = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    // lazy rescale: the running max moves only when it grows by more than 2^8
    if constexpr (kPack) {
      float alpha = 1.f;                             // head gid's factor (< 2^-8 when it moves)
      if (mx0 > m0 + kRescale || m0 == -INFINITY) {
        alpha = (m0 == -INFINITY) ? 0.f : exp2f(m0 - mx0);
        m0 = mx0;
        l0 *= alpha;
      }
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        // this lane's O^T columns are heads 2tig and 2tig+1, whose factors the
        // lanes gid = 2tig (lane 8tig) and gid = 2tig+1 (lane 8tig+4) hold
        const float a_lo = __shfl_sync(0xffffffffu, alpha, 8 * tig);
        const float a_hi = __shfl_sync(0xffffffffu, alpha, 8 * tig + 4);
#pragma unroll
        for (int n = 0; n < kOTiles; ++n) {
          o[n][0] *= a_lo; o[n][1] *= a_hi; o[n][2] *= a_lo; o[n][3] *= a_hi;
        }
      }
    } else {
      if (mx0 > m0 + kRescale || m0 == -INFINITY) {
        const float alpha = (m0 == -INFINITY) ? 0.f : exp2f(m0 - mx0);
        m0 = mx0;
        l0 *= alpha;
#pragma unroll
        for (int n = 0; n < kOTiles; ++n) { o[n][0] *= alpha; o[n][1] *= alpha; }
      }
      float mx1 = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      if (mx1 > m1 + kRescale || m1 == -INFINITY) {
        const float alpha = (m1 == -INFINITY) ? 0.f : exp2f(m1 - mx1);
        m1 = mx1;
        l1 *= alpha;
#pragma unroll
        for (int n = 0; n < kOTiles; ++n) { o[n][2] *= alpha; o[n][3] *= alpha; }
      }
    }
    const float mb0 = (m0 == -INFINITY) ? 0.f : m0, mb1 = (m1 == -INFINITY) ? 0.f : m1;
    // P in bf16: the A fragment of P V (rows gid / gid+8, keys 2tig.. / 8+2tig..)
    // or, kPack, pa0 / pa2 as the B fragment of V^T P^T; the row sums use the
    // same rounded values
    uint32_t pa0, pa1 = 0u, pa2, pa3 = 0u;
    {
      const float p00 = ex2_approx(sc[0][0] - mb0), p01 = ex2_approx(sc[0][1] - mb0);
      const float p10 = ex2_approx(sc[1][0] - mb0), p11 = ex2_approx(sc[1][1] - mb0);
      pa0 = bf16x2_bits(p00, p01);
      pa2 = bf16x2_bits(p10, p11);
      l0 += (bf16_lo(pa0) + bf16_hi(pa0)) + (bf16_lo(pa2) + bf16_hi(pa2));
    }
    if constexpr (!kPack) {
      const float p02 = ex2_approx(sc[0][2] - mb1), p03 = ex2_approx(sc[0][3] - mb1);
      const float p12 = ex2_approx(sc[1][2] - mb1), p13 = ex2_approx(sc[1][3] - mb1);
      pa1 = bf16x2_bits(p02, p03);
      pa3 = bf16x2_bits(p12, p13);
      l1 += (bf16_lo(pa1) + bf16_hi(pa1)) + (bf16_lo(pa3) + bf16_hi(pa3));
    }
    if constexpr (kPack) {
      // O^T += V^T P^T: V^T (16 dims x 16 keys) is the A operand by
      // ldmatrix.trans, and the B operand P^T (keys 2tig.., head gid) is the
      // lane's own pa0 / pa2
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        uint32_t av[4];
        const int key = (lane & 7) + ((lane >> 4) & 1) * 8;
        const int col = mt * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x4_t(vs + key * kRowBytes + col * 2, av);
        mma_bf16_16816(o[mt], av[0], av[1], av[2], av[3], pa0, pa2);
      }
    } else {
      // O += P V: 16 n-tiles of 8 dims, V fragments by ldmatrix.trans
#pragma unroll
      for (int np = 0; np < 8; ++np) {               // pairs of n-tiles
        uint32_t bv[4];
        const int key = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = np * 16 + (lane >> 4) * 8;
        ldsm_x4_t(vs + key * kRowBytes + col * 2, bv);
        mma_bf16_16816(o[2 * np], pa0, pa1, pa2, pa3, bv[0], bv[1]);
        mma_bf16_16816(o[2 * np + 1], pa0, pa1, pa2, pa3, bv[2], bv[3]);
      }
    }
    __syncwarp();                                    // buffer reusable by a later step
  }
  cp_async_wait<0>();                                // only empty groups remain
  // row sums over the quad
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  if (!kPack) {
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  }

  // merge the warps: per warp [16 rows][m, l, O(128)]
  __syncthreads();
  float* ms = reinterpret_cast<float*>(dsmem);
  float* wrow = ms + (size_t)warp * 16 * (kHeadDim + 2);
  {
    float* r0 = wrow + gid * (kHeadDim + 2);
    float* r1 = wrow + (gid + 8) * (kHeadDim + 2);
    if (tig == 0) {
      r0[0] = m0; r0[1] = l0;
      if (!kPack) { r1[0] = m1; r1[1] = l1; }
    }
    if constexpr (kPack) {
      float* h0 = wrow + (2 * tig) * (kHeadDim + 2) + 2;       // head 2tig
      float* h1 = h0 + (kHeadDim + 2);                         // head 2tig + 1
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int d = mt * 16 + gid;
        h0[d] = o[mt][0];
        h1[d] = o[mt][1];
        h0[d + 8] = o[mt][2];
        h1[d + 8] = o[mt][3];
      }
    } else {
#pragma unroll
      for (int n = 0; n < 16; ++n) {                 // C layout: cols 2tig, 2tig+1 of tile n
        r0[2 + n * 8 + 2 * tig] = o[n][0];
        r0[2 + n * 8 + 2 * tig + 1] = o[n][1];
        r1[2 + n * 8 + 2 * tig] = o[n][2];
        r1[2 + n * 8 + 2 * tig + 1] = o[n][3];
      }
    }
  }
  __syncthreads();
  const int nw = min(kDecWarps, nsteps);             // warps that saw keys
  for (int e = threadIdx.x; e < a.G * kHeadDim; e += kDecThreads) {
    const int r = e / kHeadDim, d = e % kHeadDim;
    float M = -INFINITY;
    for (int w = 0; w < nw; ++w) M = fmaxf(M, ms[((size_t)w * 16 + r) * (kHeadDim + 2)]);
    float L = 0.f, O = 0.f;
    for (int w = 0; w < nw; ++w) {
      const float* wr = ms + ((size_t)w * 16 + r) * (kHeadDim + 2);
      const float f = (wr[0] == -INFINITY) ? 0.f : exp2f(wr[0] - M);
      L += wr[1] * f;
      O += wr[2 + d] * f;
    }
    const int h = g * a.G + r;
    const size_t pi = ((size_t)b * a.H + h) * a.splits + s;
    a.part_o[pi * kHeadDim + d] = O;
    if (d == 0) {
      a.part_ml[2 * pi] = M;
      a.part_ml[2 * pi + 1] = L;
    }
  }

  // ---- the last CTA of this (sequence, KV head) combines the splits and the sink
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0)
    last_flag = atomicAdd(a.counters + (size_t)b * a.Hk + g, 1) == nsplit - 1;
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  for (int r = warp; r < a.G; r += kDecWarps) {
    const int h = g * a.G + r;
    const size_t pb = ((size_t)b * a.H + h) * a.splits;
    const float s2 = __ldg(a.sink + h) * kLog2e;      // the sink's logit, log2 units
    float M = s2;
    for (int i = 0; i < nsplit; ++i) M = fmaxf(M, __ldcg(a.part_ml + 2 * (pb + i)));
    float L = exp2f(s2 - M);                         // the sink's own weight
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < nsplit; ++i) {
      const float mi = __ldcg(a.part_ml + 2 * (pb + i));
      const float f = (mi == -INFINITY) ? 0.f : exp2f(mi - M);
      L += __ldcg(a.part_ml + 2 * (pb + i) + 1) * f;
      const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part_o + (pb + i) * kHeadDim) +
                              lane);
      acc[0] += v.x * f; acc[1] += v.y * f; acc[2] += v.z * f; acc[3] += v.w * f;
    }
    const float inv = 1.f / L;
    const size_t ob = ((size_t)b * a.H + h) * kHeadDim + lane * 4;
    if (a.out_f32) {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ob) =
          make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    } else {
      uint2 pk;
      pk.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      pk.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ob) = pk;
    }
    if (lane == 0) a.lse[(size_t)b * a.H + h] = (M + log2f(L)) * kLn2;
  }
  if (threadIdx.x == 0) a.counters[(size_t)b * a.Hk + g] = 0;   // ready for the next call
}

}  // namespace

namespace {
int max_window_keys(int C, int W) { return (W > 0) ? (W < C ? W : C) : C; }
// Keys per chunk when the largest window is divided into s splits: even shares,
// rounded up to the 16-key step.
int chunk_keys(int C, int W, int s) {
  const int per = (max_window_keys(C, W) + s - 1) / s;
  return (per + kStepKeys - 1) / kStepKeys * kStepKeys;
}
}  // namespace

int decode_splits_max(int C, int W) {
  return (max_window_keys(C, W) + kMinChunkKeysDecode - 1) / kMinChunkKeysDecode;
}

namespace {
constexpr int kDecResident = 3;   // CTAs per SM (shared memory and registers alike)

// The split plan: the first pair_split pairs take s splits, the rest grid_x.
//   * Fewer pairs than resident CTA slots: about five CTAs per SM, one split
//     count for all pairs (at three resident CTAs per SM two waves, the second
//     nearly full). Measured on the 64-sequence, window-4096 serving shape (256
//     pairs, 148 SMs): 3 splits of 1376 keys 4235 GB/s of K and V, 4 of 1024
//     4100, 5 of 832 4040, 2 of 2048 3690 with the padded kernel; a two-wave plan
//     as below 4503-4506 against 4623.
//   * Between one and one and a half times as many pairs as slots: exactly two
//     waves, the first pairs with one split and the rest with two (the larger
//     chunks all launch in the first wave). 148 sequences (592 pairs): 5613-5663
//     GB/s against 5181-5224 for one split each (1.33 waves); 120 sequences (480
//     pairs): 5400 against 5285 for two splits each (2.16 waves).
struct SplitPlan {
  int s, pair_split, grid_x;
};
SplitPlan decode_split_plan(int B, int Hk, int C, int W, int num_sms) {
  const long long P = (long long)B * Hk;
  const int smax = decode_splits_max(C, W);
  if (P <= 0) return {1, 0, 1};
  if (P < (long long)kDecResident * num_sms) {
    long long s = (5LL * num_sms + P / 2) / P;
    if (s < 1) s = 1;
    if (s > smax) s = smax;
    return {(int)s, (int)P, (int)s};
  }
  const long long S = (long long)kDecResident * num_sms, T = 2 * S;
  long long s = T / P, r = T % P;
  // only while the larger chunks all start in the first wave (P <= 1.5 slots);
  // beyond, one split each (800 pairs: 6020 GB/s against 5936 for the plan)
  if (s < 1 || P - r > S) { s = 1; r = 0; }
  if (s >= smax) { s = smax; r = 0; }
  return {(int)s, (int)(P - r), (int)(s + (r > 0 ? 1 : 0))};
}
}  // namespace

cudaError_t launch_decode(const DecodeLaunch& L, cudaStream_t st) {
  static PerDeviceOnce smem_once_pack, smem_once_full;
  const bool pack = L.H / L.Hk <= 8;
  cudaError_t e = pack ? smem_limit_once(smem_once_pack, decode_attn_kernel<true>, kAttnSmem)
                       : smem_limit_once(smem_once_full, decode_attn_kernel<false>, kAttnSmem);
  if (e != cudaSuccess) return e;
  DecArgs a;
  a.B = L.B; a.C = L.C; a.H = L.H; a.Hk = L.Hk; a.G = L.H / L.Hk; a.W = L.W;
  a.rope = L.rope; a.theta = L.theta; a.eps = L.eps;
  a.scale_log2 = L.scale * kLog2e;
  a.splits = decode_splits_max(L.C, L.W);            // stride of the partials
  const SplitPlan plan = decode_split_plan(L.B, L.Hk, L.C, L.W, L.num_sms);
  a.chunk_a = chunk_keys(L.C, L.W, plan.s);
  a.chunk_b = chunk_keys(L.C, L.W, plan.grid_x);
  a.pair_split = plan.pair_split;
  const int launched = plan.grid_x;
  a.out_f32 = L.out_f32;
  a.q = static_cast<const __nv_bfloat16*>(L.q);
  a.k = static_cast<const __nv_bfloat16*>(L.k);
  a.v = static_cast<const __nv_bfloat16*>(L.v);
  a.wq = static_cast<const __nv_bfloat16*>(L.wq);
  a.wk = static_cast<const __nv_bfloat16*>(L.wk);
  a.sink = L.sink;
  a.lens = L.lens;
  a.kc = static_cast<__nv_bfloat16*>(L.kc);
  a.vc = static_cast<__nv_bfloat16*>(L.vc);
  a.counters = L.counters; a.part_o = L.part_o; a.part_ml = L.part_ml;
  a.out = L.out; a.lse = L.lse; a.status = L.status;
  ProfScope prof(kKDecode, st);
  const dim3 grid(launched, a.Hk, a.B);
  if (pack)
    decode_attn_kernel<true><<<grid, kDecThreads, kAttnSmem, st>>>(a);
  else
    decode_attn_kernel<false><<<grid, kDecThreads, kAttnSmem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace flint
