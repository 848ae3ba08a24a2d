// attn_bwd_sm100.cu - backward of the sink-aware attention on Blackwell tensor
// cores (tcgen05 + TMEM + TMA), FP16 operands, FP32 accumulation.
//
// Gradients of sum(dO * O) (Flint layers page, nemo_automodel.components.
// models.flint.layers: the learned-sink training kernel named in the module
// docstring; FlintAttention.forward defines O). With P_ij = e^{z_ij - LSE_i}
// over visible keys (the sink's share needs no term: its value is zero) and
// D_i = dO_i . O_i (computed by the preprocess kernel):
//   dV_j   = sum_i P_ij dO_i
//   dS_ij  = P_ij (dO_i . v_j - D_i)
//   dK^_j  = scale sum_i dS_ij q^_i        dQ^_i = scale sum_j dS_ij k^_j
// The sink gradient itself comes from the preprocess kernel.
//
// Operands: q_hat, k_hat (recomputed by the prologue in fp16), fp16 copies of v
// and dO, and P, dS rounded to fp16 - fp16's 10-bit mantissa keeps the bf16
// rounding of these intermediates from dominating the gradient error.
//
// Two persistent kernels share one warp layout: warps 0-7 do the elementwise
// math as two warpgroups that split the 128 columns of each tile (there is no
// row reduction in the backward, so the halves are independent; thread = TMEM
// lane), warp 8 issues TMA, warp 9 issues MMAs (converged, one elected lane
// issues) and owns TMEM. Each warpgroup
// writes its fp16 P/dS half into the first 32 of the 64 TMEM columns it has
// just read itself (columns [64c, 64c+32) for warpgroup c), so the TMEM A
// operand of the following MMA skips from column 32 to 64 halfway through K.
//  * dkv: key-major. A CTA owns 128 keys of one KV head and streams the
//    128-row query tiles (R tokens x G heads) that see them, farthest first:
//    the tensor cores align each product to the FP32 accumulator's exponent
//    before adding it, so a small term added to a large sum keeps few bits, and
//    a causal key's largest terms come from the queries just after it (few
//    competing keys there). Near-to-far, the first keys of a 32768-token layer
//    had 2x the dk/dv error (4.4e-3 against 2.3e-3) at the same speed. Per tile:
//    S^T = K Q^T and dP^T = V dO^T (TMEM), then P^T and dS^T in fp16 are
//    written over S^T and feed dV += P^T dO and dK += dS^T Q as TMEM A
//    operands. The S^T and dP^T regions swap roles every tile: the next S^T
//    goes into this tile's dP^T region as soon as the math warps hold dP^T in
//    registers, so it runs during their dS step. dK and dV stay in TMEM for the
//    whole key tile, so the G heads of a group are summed without atomics.
//    TMEM: 2 x 128 rotating columns + dV + dK = 512 cols. Query tiles stream
//    through 3 shared-memory stages, dO tiles (with the per-row statistics)
//    through 2.
//  * dq: query-major. A CTA owns one 128-row query tile and streams its key
//    tiles: S = Q K^T, dP = dO V^T, dS (fp16) over S, dQ += dS K. TMEM: two S
//    buffers, dP, dQ = 512 cols; S of the next key tile is computed while the
//    math warps finish the current one. K and V stream through a 5-slot ring.
// In the P steps one exponential pair in four (dK/dV) or eight (dQ) is evaluated
// on the FMA pipe (exp2_fma2); the special-function unit alone would bound them.
// An MMA that overwrites a TMEM region a previous MMA reads as its A operand
// is issued right behind it without a completion wait: tcgen05.mma operations
// issued by one thread are performed in issue order.
#include <type_traits>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {

namespace {

constexpr int kThreads = 320;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kMathWarps = 8;
constexpr uint32_t kChunkBytes = 128 * 64 * 2;
constexpr uint32_t kTileBytes = 2 * kChunkBytes;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdArgs {
  int T, H, Hk, G, R, W, logG;
  float scale, scale_log2;
  const float* lse;
  const float* dvec;      // D * s_dout * s_v (the scales of the fp16 operand copies)
  const unsigned* amax;   // [max |dout|, max |v|] slots (pow2_scale_exp)
  const int4* items;
  const int* n_items;
  int max_items;
  int* next_item;    // zeroed before the launch: dynamic item counter
  float* dq_acc;
  float* dk_acc;
  void* dv;          // float or bf16, per dv_f32
  int dv_f32;
  int* status;
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_base, int kk) {
  return make_sdesc(tile_base + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_base, int kk) {
  return make_sdesc(tile_base + kk * 2048, kChunkBytes, 1024);
}
// TMEM column of the fp16 A-operand slice kk (16 K-elements = 8 columns) of a
// region whose two 64-element halves sit at columns [0,32) and [64,96).
__device__ __forceinline__ uint32_t split_a_col(int kk) {
  return kk < 4 ? kk * 8 : 64 + (kk - 4) * 8;
}

__device__ __forceinline__ float2 unpack_f16x2(uint32_t u) {
  __half2 h = *reinterpret_cast<__half2*>(&u);
  return __half22float2(h);
}

// ============================================================================
// dK / dV : key-major
// ============================================================================
constexpr int kQStages = 3;   // Q tiles in flight (its buffer is released last, by dK)
struct __align__(8) KvBars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[kQStages], q_empty[kQStages], do_full[2], do_empty[2];
  uint64_t s_full, dp_full, p_full, dp_free, ds_full, acc_full, acc_empty;
  uint64_t drain;
  ItemRing ring;
};
constexpr uint32_t kKvOffK = 0;
constexpr uint32_t kKvOffV = kTileBytes;
constexpr uint32_t kKvOffQ = 2 * kTileBytes;                        // kQStages stages
constexpr uint32_t kKvOffDO = kKvOffQ + kQStages * kTileBytes;      // 2 stages
constexpr uint32_t kKvOffStats = kKvOffDO + 2 * kTileBytes;         // [2][2][128] fp32
constexpr uint32_t kKvOffBar = kKvOffStats + 2 * 2 * 128 * 4;
constexpr uint32_t kKvOffTmem = kKvOffBar + sizeof(KvBars);
constexpr uint32_t kKvOffAbort = kKvOffTmem + 16;
// No alignment slack: the kernel checks that the dynamic shared memory starts
// on a 1024-byte boundary (the 128-byte swizzle needs it) and reports
// kStatusSmemAlign otherwise.
constexpr uint32_t kKvSmem = kKvOffAbort + 16;
static_assert(kKvSmem <= 227 * 1024, "exceeds the shared memory of one CTA");

struct KvItem {
  int k0, d0, d1, g, qend, nq;
};
__device__ __forceinline__ KvItem decode_kv(const BwdArgs& a, int idx) {
  const int4 it = a.items[idx];
  KvItem r;
  r.k0 = it.x; r.d0 = it.y; r.d1 = it.z; r.g = it.w;
  r.qend = a.W > 0 ? min(r.d1, r.k0 + kTileKeys - 1 + a.W) : r.d1;
  r.nq = (r.qend - r.k0 + a.R - 1) / a.R;
  return r;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_do, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  KvBars* bars = reinterpret_cast<KvBars*>(smem + kKvOffBar);
  float* stats = reinterpret_cast<float*>(smem + kKvOffStats);   // [buf][-lse2|D][128]
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kKvOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kKvOffAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, a.status, kStatusTimeoutBwdKV};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(smem_u32(&bars->kv_full), 1);
    mbar_init(smem_u32(&bars->kv_empty), 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(smem_u32(&bars->q_full[s]), 1);
      mbar_init(smem_u32(&bars->q_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->do_full[s]), 2);   // TMA bytes + per-row statistics
      mbar_init(smem_u32(&bars->do_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->p_full), kMathWarps);
    mbar_init(smem_u32(&bars->ds_full), kMathWarps);
    mbar_init(smem_u32(&bars->dp_free), kMathWarps);
    mbar_init(smem_u32(&bars->acc_full), 1);
    mbar_init(smem_u32(&bars->acc_empty), kMathWarps);
    mbar_init(smem_u32(&bars->drain), 1);
    ring_init(&bars->ring, kMathWarps + 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32((const void*)tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = min(*a.n_items, a.max_items);

  if (warp == kWarpTma) {
    // Lane 0 takes items from the global counter and issues TMA; the whole warp
    // stages each query tile's per-row -log2-LSE and D into shared memory and
    // completes do_full's second arrival.
    uint32_t item_count = 0, qd_iter = 0, kv_arm = 0, q_arm[kQStages] = {}, do_arm[2] = {};
    bool ok = true;
    while (ok) {
      int idx = -1;
      if (lane == 0) {
        idx = atomicAdd(a.next_item, 1);
        if (idx >= n_items) idx = -1;
        ok = ring_push(&bars->ring, item_count, idx, wc);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      idx = __shfl_sync(0xffffffffu, idx, 0);
      if (!ok || idx < 0) break;
      const KvItem it = decode_kv(a, idx);
      if (lane == 0) {
        if (item_count > 0) ok = mbar_wait(smem_u32(&bars->kv_empty), (item_count - 1) & 1, wc);
        if (ok) {
          const uint32_t kf = smem_u32(&bars->kv_full);
          mbar_arrive_expect_tx(kf, 2 * kTileBytes);
          ++kv_arm;
          for (int c = 0; c < 2; ++c) {
            tma_load_3d(sbase + kKvOffK + c * kChunkBytes, &tm_k, kf, c * 64, it.g, it.k0);
            tma_load_3d(sbase + kKvOffV + c * kChunkBytes, &tm_v, kf, c * 64, it.g, it.k0);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int m = 0; m < it.nq && ok; ++m, ++qd_iter) {
        const int qs = it.k0 + (it.nq - 1 - m) * a.R;   // far to near
        const uint32_t sq = qd_iter % kQStages, phq = (qd_iter / kQStages) & 1;
        const uint32_t s = qd_iter & 1, ph = (qd_iter >> 1) & 1;
        // The tile's statistics are read before waiting for its buffer, so the
        // global-load latency overlaps the wait.
        float lse2[4], dr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = lane + 32 * e;
          const int tok = qs + (r >> a.logG), h = it.g * a.G + (r & (a.G - 1));
          const bool vr = tok < it.d1;
          lse2[e] = vr ? -__ldg(a.lse + (size_t)h * a.T + tok) * kLog2e : 0.f;   // negated
          dr[e] = vr ? __ldg(a.dvec + (size_t)h * a.T + tok) : 0.f;
        }
        const uint32_t qf = smem_u32(&bars->q_full[sq]), df = smem_u32(&bars->do_full[s]);
        if (lane == 0) {
          if (qd_iter >= kQStages) ok = mbar_wait(smem_u32(&bars->q_empty[sq]), phq ^ 1, wc);
          if (ok) {
            mbar_arrive_expect_tx(qf, kTileBytes);
            ++q_arm[sq];
            for (int c = 0; c < 2; ++c)
              tma_load_3d(sbase + kKvOffQ + sq * kTileBytes + c * kChunkBytes, &tm_q, qf, c * 64,
                          it.g * a.G, qs);
          }
          if (ok && qd_iter >= 2) ok = mbar_wait(smem_u32(&bars->do_empty[s]), ph ^ 1, wc);
          if (ok) {
            mbar_arrive_expect_tx(df, kTileBytes);
            ++do_arm[s];
            for (int c = 0; c < 2; ++c)
              tma_load_3d(sbase + kKvOffDO + s * kTileBytes + c * kChunkBytes, &tm_do, df,
                          c * 64, it.g * a.G, qs);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        float* st = stats + s * 256;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          st[lane + 32 * e] = lse2[e];
          st[128 + lane + 32 * e] = dr[e];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(df);
      }
      ++item_count;
    }
    if (lane == 0) {
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutBwdKV};
      if (kv_arm) mbar_wait(smem_u32(&bars->kv_full), (kv_arm - 1) & 1, drain);
      for (int s = 0; s < kQStages; ++s)
        if (q_arm[s]) mbar_wait(smem_u32(&bars->q_full[s]), (q_arm[s] - 1) & 1, drain);
      for (int s = 0; s < 2; ++s)
        if (do_arm[s]) mbar_wait(smem_u32(&bars->do_full[s]), (do_arm[s] - 1) & 1, drain);
    }
  } else if (warp == kWarpMma) {
    // TMEM regions R0 = [0,128), R1 = [128,256) rotate between query tiles
    // (numbered t across items): S^T(t) goes to X_t = R(t&1), dP^T(t) to
    // Y_t = R(~t&1). The math warps write P^T(t) and dS^T(t) into X_t, so Y_t
    // is free once they have loaded dP^T(t) into registers (dp_free, early in
    // their dS step). Issue order per tile: dV(t), S^T(t+1) into Y_t (runs
    // while dS(t) is computed), dK(t), then dP^T(t+1) into X_t, right behind
    // the dK(t) that reads X_t (MMAs are performed in issue order).
    {
      const uint32_t leader = elect_one();   // the one lane that issues
      const uint32_t idesc_ss = make_idesc_f16(128, 128, 0, 0);
      const uint32_t idesc_ts = make_idesc_f16(128, 128, 0, 1);
      uint32_t item_count = 0, t = 0, p_cnt = 0, ds_cnt = 0, dpf_cnt = 0;
      bool ok = true;
      const uint32_t kt = sbase + kKvOffK, vt = sbase + kKvOffV;
      auto region = [&](uint32_t r) { return tmem + (r & 1) * 128; };
      auto issue_s = [&](uint32_t tt) {          // S^T(tt) into X_tt
        const uint32_t qt = sbase + kKvOffQ + (tt % kQStages) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_w(region(tt), kmajor_desc(kt, kk), kmajor_desc(qt, kk), idesc_ss, kk > 0, leader);
        mma_commit_w(smem_u32(&bars->s_full), leader);
      };
      auto issue_dp = [&](uint32_t tt) {         // dP^T(tt) into Y_tt
        const uint32_t dot = sbase + kKvOffDO + (tt & 1) * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_w(region(tt + 1), kmajor_desc(vt, kk), kmajor_desc(dot, kk), idesc_ss, kk > 0,
                   leader);
        mma_commit_w(smem_u32(&bars->dp_full), leader);
      };
      while (ok) {
        int idx = -1;
        ok = ring_pop(&bars->ring, item_count, &idx, wc);
        if (!ok || idx < 0) break;
        const KvItem it = decode_kv(a, idx);
        ok = mbar_wait_warp(smem_u32(&bars->kv_full), item_count & 1, wc);
        if (!ok) break;
        {  // S^T and dP^T of the item's first query tile
          ok = mbar_wait_warp(smem_u32(&bars->q_full[t % kQStages]), (t / kQStages) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          issue_s(t);                            // X_t = Y_{t-1}: free after ds_full(t-1)
          ok = mbar_wait_warp(smem_u32(&bars->do_full[t & 1]), (t >> 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          issue_dp(t);                           // Y_t = X_{t-1}: behind dK(t-1), its reader
        }
        for (int m = 0; m < it.nq && ok; ++m, ++t) {
          const uint32_t s = t & 1, sq = t % kQStages;
          const uint32_t qt = sbase + kKvOffQ + sq * kTileBytes;
          const uint32_t dot = sbase + kKvOffDO + s * kTileBytes;
          const uint32_t X = region(t);
          const bool has_next = m + 1 < it.nq;
          // dV(t) += P^T(t) dO(t)
          ok = mbar_wait_warp(smem_u32(&bars->p_full), p_cnt & 1, wc);
          ++p_cnt;
          if (ok && m == 0 && item_count > 0)
            ok = mbar_wait_warp(smem_u32(&bars->acc_empty), (item_count - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(tmem + 256, X + split_a_col(kk), mnmajor_desc(dot, kk), idesc_ts,
                     (m > 0 || kk > 0) ? 1u : 0u, leader);
          // dP^T(t) read by the math warps -> Y_t free for S^T(t+1)
          if (has_next) {
            ok = mbar_wait_warp(smem_u32(&bars->dp_free), dpf_cnt & 1, wc);
            if (ok) ok = mbar_wait_warp(smem_u32(&bars->q_full[(t + 1) % kQStages]),
                                        ((t + 1) / kQStages) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            issue_s(t + 1);
          }
          ++dpf_cnt;
          // dS^T(t) written
          ok = mbar_wait_warp(smem_u32(&bars->ds_full), ds_cnt & 1, wc);
          ++ds_cnt;
          if (!ok) break;
          tc_fence_after();
          // dO(t) and its statistics: dV(t) (issued) is their last reader on the
          // tensor cores, and the math warps are done with them (ds_full).
          mma_commit_w(smem_u32(&bars->do_empty[s]), leader);
          // dK(t) += dS^T(t) Q(t)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(tmem + 384, X + 32 + split_a_col(kk), mnmajor_desc(qt, kk), idesc_ts,
                     (m > 0 || kk > 0) ? 1u : 0u, leader);
          mma_commit_w(smem_u32(&bars->q_empty[sq]), leader);
          if (has_next) {
            ok = mbar_wait_warp(smem_u32(&bars->do_full[(t + 1) & 1]), ((t + 1) >> 1) & 1, wc);
            if (!ok) break;
            tc_fence_after();
            issue_dp(t + 1);
          }
        }
        if (!ok) break;
        mma_commit_w(smem_u32(&bars->kv_empty), leader);
        mma_commit_w(smem_u32(&bars->acc_full), leader);
        ++item_count;
      }
      mma_commit_w(smem_u32(&bars->drain), leader);
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutBwdKV};
      mbar_wait_warp(smem_u32(&bars->drain), 0, drain);
    }
  } else {
    // ---------------------------------------------------------------- math warps
    const int wg = warp >> 2;                      // column half: query rows [64wg, 64wg+64)
    const int kl = (warp & 3) * 32 + lane;         // key row of the tile = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t c0 = 64 * wg;                   // first column of this warpgroup
    // dV carries the scale of the fp16 dO copy, dK that of dO and v
    const float inv_sdo = slot_scale(a.amax, true);
    const float dk_mul = a.scale * inv_sdo * slot_scale(a.amax + 1, true);
    uint32_t item_count = 0, s_cnt = 0, dp_cnt = 0, tile_count = 0;
    bool ok = true;
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const KvItem it = decode_kv(a, idx);
      const int j = it.k0 + kl;
      const bool valid_key = j < it.d1;
      for (int m = 0; m < it.nq; ++m, ++tile_count) {
        const int qs = it.k0 + (it.nq - 1 - m) * a.R;   // far to near
        const uint32_t stg = tile_count & 1, ph = (tile_count >> 1) & 1;
        const float* st = stats + stg * 256;
        const bool needs_mask = (it.k0 + kTileKeys - 1 > qs) || (it.k0 + kTileKeys > it.d1) ||
                                (qs + a.R > it.d1) || (a.W > 0 && qs + a.R - 1 - it.k0 >= a.W);
        // the tile's statistics are in shared memory once do_full completes
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->do_full[stg]), ph, wc));
        if (!ok) break;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full), s_cnt & 1, wc));
        ++s_cnt;
        if (!ok) break;
        tc_fence_after();
        // TMEM regions of this tile: S^T in X, dP^T in Y (rotating per tile)
        const uint32_t X = (tile_count & 1) * 128, Y = 128 - X;
        const uint64_t sc2 = f2(a.scale_log2, a.scale_log2);
        // P^T for query rows [c0, c0+64): 2^(s*scale - lse2), masked, fp16.
        // Row c of the tile is token qs + c/G, so the rows that see key j form
        // one column range [cmin, cmax); masked and unmasked tiles run separate
        // code so the mask costs nothing on interior tiles.
        int cmin = 0, cmax = kTileRows;
        if (needs_mask) {
          const int qend_j = a.W > 0 ? min(it.d1, j + a.W) : it.d1;
          cmin = valid_key ? max(0, (j - qs) * a.G) : kTileRows;
          cmax = valid_key ? min(kTileRows, (qend_j - qs) * a.G) : 0;
        }
        uint32_t pk[32];
        {
          uint32_t u0[32], u1[32];
          tmem_ld32(t_row + X + c0, u0);
          tmem_ld32(t_row + X + c0 + 32, u1);
          tc_wait_ld_dep(u0);
          tc_wait_ld_dep(u1);
          auto p_half = [&](auto masked) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int c = c0 + 2 * e;
              const float s0 = __uint_as_float(e < 16 ? u0[2 * e] : u1[2 * e - 32]);
              const float s1 = __uint_as_float(e < 16 ? u0[2 * e + 1] : u1[2 * e - 31]);
              const uint64_t nl2 = *reinterpret_cast<const uint64_t*>(st + c);   // -lse2 pair
              float x0, x1;
              f2_split(ffma2(f2(s0, s1), sc2, nl2), x0, x1);
              // one pair in four on the FMA pipe (polynomial 2^x), the rest on
              // the special-function unit, which alone would bound this loop
              float p0, p1;
              if ((e & 3) == 3) exp2_fma2(x0, x1, p0, p1);
              else { p0 = ex2_approx(x0); p1 = ex2_approx(x1); }
              if (decltype(masked)::value) {
                p0 = (c >= cmin && c < cmax) ? p0 : 0.f;
                p1 = (c + 1 >= cmin && c + 1 < cmax) ? p1 : 0.f;
              }
              pk[e] = pack_f16x2(p0, p1);
            }
          };
          if (needs_mask) p_half(std::true_type{});
          else p_half(std::false_type{});
        }
        tmem_st32(t_row + X + c0, pk);             // P^T into X columns [c0, c0+32)
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full));
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->dp_full), dp_cnt & 1, wc));
        ++dp_cnt;
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t u0[32], u1[32], ds[32];
          tmem_ld32(t_row + Y + c0, u0);
          tmem_ld32(t_row + Y + c0 + 32, u1);
          tc_wait_ld_dep(u0);
          tc_wait_ld_dep(u1);
          // dP^T(t) is in registers: Y may take S^T(t+1)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->dp_free));
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = c0 + 2 * e;
            const float d0 = __uint_as_float(e < 16 ? u0[2 * e] : u1[2 * e - 32]);
            const float d1 = __uint_as_float(e < 16 ? u0[2 * e + 1] : u1[2 * e - 31]);
            const float2 p = unpack_f16x2(pk[e]);
            const float2 dd = *reinterpret_cast<const float2*>(st + 128 + c);
            ds[e] = pack_f16x2(p.x * (d0 - dd.x), p.y * (d1 - dd.y));
          }
          tmem_st32(t_row + X + c0 + 32, ds);       // dS^T into X columns [c0+32, c0+64)
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->acc_full), item_count & 1, wc));
      if (!ok) break;
      tc_fence_after();
      {
        // this warpgroup writes columns [c0, c0+64) of the key row's dV, then dK
        const size_t rb = ((size_t)j * a.Hk + it.g) * kHeadDim + c0;
        {
          uint32_t v0[32], v1[32];
          tmem_ld32(t_row + 256 + c0, v0);
          tmem_ld32(t_row + 256 + c0 + 32, v1);
          tc_wait_ld_dep(v0);
          tc_wait_ld_dep(v1);
          if (valid_key) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t* vv = hh ? v1 : v0;
              float f[32];
#pragma unroll
              for (int c = 0; c < 32; ++c) f[c] = __uint_as_float(vv[c]) * inv_sdo;
              if (a.dv_f32) {
                float* dvrow = reinterpret_cast<float*>(a.dv) + rb + hh * 32;
#pragma unroll
                for (int c = 0; c < 32; c += 4)
                  *reinterpret_cast<float4*>(dvrow + c) =
                      make_float4(f[c], f[c + 1], f[c + 2], f[c + 3]);
              } else {
                __nv_bfloat16* dvrow = reinterpret_cast<__nv_bfloat16*>(a.dv) + rb + hh * 32;
#pragma unroll
                for (int c = 0; c < 32; c += 8) {
                  uint4 pkv;
                  pkv.x = pack_bf16x2(f[c], f[c + 1]);
                  pkv.y = pack_bf16x2(f[c + 2], f[c + 3]);
                  pkv.z = pack_bf16x2(f[c + 4], f[c + 5]);
                  pkv.w = pack_bf16x2(f[c + 6], f[c + 7]);
                  *reinterpret_cast<uint4*>(dvrow + c) = pkv;
                }
              }
            }
          }
        }
        {
          uint32_t k0[32], k1[32];
          tmem_ld32(t_row + 384 + c0, k0);
          tmem_ld32(t_row + 384 + c0 + 32, k1);
          tc_wait_ld_dep(k0);
          tc_wait_ld_dep(k1);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty));
          if (valid_key) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t* kv = hh ? k1 : k0;
              float* dkrow = a.dk_acc + rb + hh * 32;
#pragma unroll
              for (int c = 0; c < 32; c += 4)
                *reinterpret_cast<float4*>(dkrow + c) = make_float4(
                    __uint_as_float(kv[c]) * dk_mul, __uint_as_float(kv[c + 1]) * dk_mul,
                    __uint_as_float(kv[c + 2]) * dk_mul, __uint_as_float(kv[c + 3]) * dk_mul);
            }
          }
        }
      }
      ++item_count;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

// ============================================================================
// dQ : query-major
// ============================================================================
// K and V tiles stream through one ring of kQSlots 32 KB slots in the order
// K(0), V(0), K(1), V(1), ...; V(t) is released by dP(t), K(t) by dQ(t).
constexpr int kQSlots = 5;
struct __align__(8) QBars {
  uint64_t qd_full, qd_empty;
  uint64_t kv_full[kQSlots], kv_empty[kQSlots];
  uint64_t s_full[2];                 // per S buffer
  uint64_t dp_full, ds_full, acc_full, acc_empty;
  uint64_t drain;
  ItemRing ring;
};
constexpr uint32_t kQOffQ = 0;
constexpr uint32_t kQOffDO = kTileBytes;
constexpr uint32_t kQOffKV = 2 * kTileBytes;                 // kQSlots slots
constexpr uint32_t kQOffBar = kQOffKV + kQSlots * kTileBytes;
constexpr uint32_t kQOffTmem = kQOffBar + sizeof(QBars);
constexpr uint32_t kQOffAbort = kQOffTmem + 16;
constexpr uint32_t kQSmem = kQOffAbort + 16;   // no slack: the base is checked instead
static_assert(kQSmem <= 227 * 1024, "exceeds the shared memory of one CTA");
// TMEM columns: S double-buffered, dP, dQ accumulator
constexpr uint32_t kQColS0 = 0, kQColDP = 256, kQColDQ = 384;

struct QItem {
  int q0, d0, d1, g, kend, kbeg, ntiles;
};
__device__ __forceinline__ QItem decode_q(const BwdArgs& a, int idx) {
  const int4 it = a.items[idx];
  QItem r;
  r.q0 = it.x; r.d0 = it.y; r.d1 = it.z; r.g = it.w;
  r.kend = min(r.q0 + a.R, r.d1);
  r.kbeg = a.W > 0 ? max(r.d0, r.q0 - a.W + 1) : r.d0;
  r.ntiles = (r.kend - r.kbeg + kTileKeys - 1) / kTileKeys;
  return r;
}

// Tiles are numbered per CTA across items (t = 0, 1, ...): tile t uses S
// buffer t % 2, and K(t), V(t) take ring positions 2t and 2t + 1. An item has
// at least one key tile (kbeg <= q0 < kend).
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_do, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  QBars* bars = reinterpret_cast<QBars*>(smem + kQOffBar);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kQOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kQOffAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, a.status, kStatusTimeoutBwdQ};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(smem_u32(&bars->qd_full), 1);
    mbar_init(smem_u32(&bars->qd_empty), 1);
    for (int s = 0; s < kQSlots; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->s_full[s]), 1);
    }
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->ds_full), kMathWarps);
    mbar_init(smem_u32(&bars->acc_full), 1);
    mbar_init(smem_u32(&bars->acc_empty), kMathWarps);
    mbar_init(smem_u32(&bars->drain), 1);
    ring_init(&bars->ring, kMathWarps + 1);
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32((const void*)tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = min(*a.n_items, a.max_items);

  if (warp == kWarpTma) {
    if (lane == 0) {
      uint32_t item_count = 0, kv_load = 0, qd_arm = 0, arm[kQSlots] = {};
      bool ok = true;
      while (ok) {
        int idx = atomicAdd(a.next_item, 1);
        if (idx >= n_items) idx = -1;
        ok = ring_push(&bars->ring, item_count, idx, wc);
        if (!ok || idx < 0) break;
        const QItem it = decode_q(a, idx);
        if (item_count > 0) ok = mbar_wait(smem_u32(&bars->qd_empty), (item_count - 1) & 1, wc);
        if (!ok) break;
        const uint32_t qf = smem_u32(&bars->qd_full);
        mbar_arrive_expect_tx(qf, 2 * kTileBytes);
        ++qd_arm;
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sbase + kQOffQ + c * kChunkBytes, &tm_q, qf, c * 64, it.g * a.G, it.q0);
          tma_load_3d(sbase + kQOffDO + c * kChunkBytes, &tm_do, qf, c * 64, it.g * a.G, it.q0);
        }
        for (int j = 0; j < 2 * it.ntiles && ok; ++j, ++kv_load) {
          const int ks = it.kend - kTileKeys * ((j >> 1) + 1);
          const uint32_t s = kv_load % kQSlots, ph = (kv_load / kQSlots) & 1;
          if (kv_load >= kQSlots) ok = mbar_wait(smem_u32(&bars->kv_empty[s]), ph ^ 1, wc);
          if (!ok) break;
          const uint32_t f = smem_u32(&bars->kv_full[s]);
          mbar_arrive_expect_tx(f, kTileBytes);
          ++arm[s];
          const CUtensorMap* m = (j & 1) ? &tm_v : &tm_k;
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sbase + kQOffKV + s * kTileBytes + c * kChunkBytes, m, f, c * 64, it.g,
                        ks);
        }
        ++item_count;
      }
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutBwdQ};
      if (qd_arm) mbar_wait(smem_u32(&bars->qd_full), (qd_arm - 1) & 1, drain);
      for (int s = 0; s < kQSlots; ++s)
        if (arm[s]) mbar_wait(smem_u32(&bars->kv_full[s]), (arm[s] - 1) & 1, drain);
    }
  } else if (warp == kWarpMma) {
    // Per tile t: dP(t), S(t+1) (into the other S buffer, right behind the dQ(t-1)
    // that reads it: MMAs are performed in issue order), dQ(t). P of tile t+1 is
    // then computed while dQ(t) and dP(t+1) run.
    {
      const uint32_t leader = elect_one();   // the one lane that issues
      const uint32_t idesc_ss = make_idesc_f16(128, 128, 0, 0);
      const uint32_t idesc_ts = make_idesc_f16(128, 128, 0, 1);
      uint32_t item_count = 0, t = 0, ds_cnt = 0;
      bool ok = true;
      const uint32_t qt = sbase + kQOffQ, dot = sbase + kQOffDO;
      // S(tt) = Q K(tt)^T into buffer tt % 2, issued after the dQ that last read it.
      auto issue_s = [&](uint32_t tt) -> bool {
        const uint32_t b = tt & 1, lk = 2 * tt;                 // K(tt) in the ring
        const uint32_t st = lk % kQSlots, ph = (lk / kQSlots) & 1;
        if (!mbar_wait_warp(smem_u32(&bars->kv_full[st]), ph, wc)) return false;
        tc_fence_after();
        const uint32_t kt = sbase + kQOffKV + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss_w(tmem + kQColS0 + b * 128, kmajor_desc(qt, kk), kmajor_desc(kt, kk), idesc_ss,
                 kk > 0, leader);
        mma_commit_w(smem_u32(&bars->s_full[b]), leader);
        return true;
      };
      while (ok) {
        int idx = -1;
        ok = ring_pop(&bars->ring, item_count, &idx, wc);
        if (!ok || idx < 0) break;
        const QItem it = decode_q(a, idx);
        ok = mbar_wait_warp(smem_u32(&bars->qd_full), item_count & 1, wc);
        if (!ok) break;
        tc_fence_after();
        ok = issue_s(t);
        for (int n = 0; n < it.ntiles && ok; ++n, ++t) {
          const uint32_t sk = (2 * t) % kQSlots, lv = 2 * t + 1;   // K(t), V(t) in the ring
          const uint32_t sv = lv % kQSlots;
          const uint32_t vt = sbase + kQOffKV + sv * kTileBytes;
          const uint32_t kt = sbase + kQOffKV + sk * kTileBytes;
          ok = mbar_wait_warp(smem_u32(&bars->kv_full[sv]), (lv / kQSlots) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          // dP(t) = dO V(t)^T; the math warps finished reading dP(t-1) before ds_full(t-1)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_w(tmem + kQColDP, kmajor_desc(dot, kk), kmajor_desc(vt, kk), idesc_ss, kk > 0,
                     leader);
          mma_commit_w(smem_u32(&bars->dp_full), leader);
          mma_commit_w(smem_u32(&bars->kv_empty[sv]), leader);   // V(t) done after dP(t)
          // Q and dO are read only by the S and dP MMAs, so the item's last dP frees
          // them: the next item's Q/dO loads overlap this tile's dS and dQ.
          if (n + 1 == it.ntiles) mma_commit_w(smem_u32(&bars->qd_empty), leader);
          if (n + 1 < it.ntiles) {
            ok = issue_s(t + 1);
            if (!ok) break;
          }
          ok = mbar_wait_warp(smem_u32(&bars->ds_full), ds_cnt & 1, wc);
          ++ds_cnt;
          if (ok && n == 0 && item_count > 0)
            ok = mbar_wait_warp(smem_u32(&bars->acc_empty), (item_count - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          const uint32_t b = t & 1;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_w(tmem + kQColDQ, tmem + kQColS0 + b * 128 + split_a_col(kk),
                     mnmajor_desc(kt, kk), idesc_ts, (n > 0 || kk > 0) ? 1u : 0u, leader);
          mma_commit_w(smem_u32(&bars->kv_empty[sk]), leader);   // K(t) done after dQ(t)
        }
        if (!ok) break;
        mma_commit_w(smem_u32(&bars->acc_full), leader);
        ++item_count;
      }
      mma_commit_w(smem_u32(&bars->drain), leader);
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutBwdQ};
      mbar_wait_warp(smem_u32(&bars->drain), 0, drain);
    }
  } else {
    // ---------------------------------------------------------------- math warps
    const int wg = warp >> 2;                      // column half: keys [64wg, 64wg+64)
    const int r = (warp & 3) * 32 + lane;          // query row of the tile = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int c0 = 64 * wg;
    // dQ carries the scales of the fp16 dO and v copies
    const float dq_mul = a.scale * slot_scale(a.amax, true) * slot_scale(a.amax + 1, true);
    uint32_t item_count = 0, t = 0;
    bool ok = true;
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const QItem it = decode_q(a, idx);
      const int tok = it.q0 + (r >> a.logG);
      const int h = it.g * a.G + (r & (a.G - 1));
      const bool valid = tok < it.d1;
      const int lo_r = a.W > 0 ? max(it.d0, tok - a.W + 1) : it.d0;
      const float lse2 = valid ? __ldg(a.lse + (size_t)h * a.T + tok) * kLog2e : 0.f;
      const float Di = valid ? __ldg(a.dvec + (size_t)h * a.T + tok) : 0.f;
      const uint64_t sc2 = f2(a.scale_log2, a.scale_log2);
      const uint64_t nl2 = f2(-lse2, -lse2);
      const uint64_t nd2 = f2(-Di, -Di);
      for (int n = 0; n < it.ntiles; ++n, ++t) {
        const uint32_t b = t & 1;
        const uint32_t s_col = kQColS0 + b * 128;
        const int ks = it.kend - kTileKeys * (n + 1);
        const bool needs_mask = (ks + kTileKeys - 1 > it.q0) || (ks < it.d0) ||
                                (a.W > 0 && ks < it.q0 + a.R - a.W);
        const int c_lo = lo_r - ks, c_hi = tok - ks;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[b]), (t >> 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        uint32_t pk[32];
        {
          uint32_t u0[32], u1[32];
          tmem_ld32(t_row + s_col + c0, u0);
          tmem_ld32(t_row + s_col + c0 + 32, u1);
          tc_wait_ld_dep(u0);
          tc_wait_ld_dep(u1);
          // masked and unmasked key tiles run separate code
          auto p_half = [&](auto masked) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint32_t a0 = e < 16 ? u0[2 * e] : u1[2 * e - 32];
              const uint32_t a1 = e < 16 ? u0[2 * e + 1] : u1[2 * e - 31];
              float x0, x1;
              f2_split(ffma2(f2(__uint_as_float(a0), __uint_as_float(a1)), sc2, nl2), x0, x1);
              // one pair in eight on the FMA pipe (polynomial 2^x), the rest on
              // the special-function unit (one in four, or two, measured slower
              // here; the dK/dV kernel prefers one in four)
              float p0, p1;
              if ((e & 7) == 7) exp2_fma2(x0, x1, p0, p1);
              else { p0 = ex2_approx(x0); p1 = ex2_approx(x1); }
              if (decltype(masked)::value) {
                const int c = c0 + 2 * e;
                p0 = (valid && c >= c_lo && c <= c_hi) ? p0 : 0.f;
                p1 = (valid && c + 1 >= c_lo && c + 1 <= c_hi) ? p1 : 0.f;
              }
              pk[e] = pack_f16x2(p0, p1);
            }
          };
          if (needs_mask) p_half(std::true_type{});
          else p_half(std::false_type{});
        }
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->dp_full), t & 1, wc));
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t u0[32], u1[32], ds[32];
          tmem_ld32(t_row + kQColDP + c0, u0);
          tmem_ld32(t_row + kQColDP + c0 + 32, u1);
          tc_wait_ld_dep(u0);
          tc_wait_ld_dep(u1);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const uint32_t a0 = e < 16 ? u0[2 * e] : u1[2 * e - 32];
            const uint32_t a1 = e < 16 ? u0[2 * e + 1] : u1[2 * e - 31];
            float y0, y1;
            const float2 pr = unpack_f16x2(pk[e]);          // dS = P * (dP - D)
            f2_split(fmul2(f2(pr.x, pr.y),
                           fadd2(f2(__uint_as_float(a0), __uint_as_float(a1)), nd2)), y0, y1);
            ds[e] = pack_f16x2(y0, y1);
          }
          // dS for keys [c0, c0+64) into S-buffer columns [c0, c0+32), read above
          tmem_st32(t_row + s_col + c0, ds);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->acc_full), item_count & 1, wc));
      if (!ok) break;
      tc_fence_after();
      {
        uint32_t u0[32], u1[32];
        tmem_ld32(t_row + kQColDQ + c0, u0);
        tmem_ld32(t_row + kQColDQ + c0 + 32, u1);
        tc_wait_ld_dep(u0);
        tc_wait_ld_dep(u1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty));
        if (valid) {
          float* row = a.dq_acc + ((size_t)tok * a.H + h) * kHeadDim + c0;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint32_t* uu = hh ? u1 : u0;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(row + hh * 32 + c) = make_float4(
                  __uint_as_float(uu[c]) * dq_mul, __uint_as_float(uu[c + 1]) * dq_mul,
                  __uint_as_float(uu[c + 2]) * dq_mul, __uint_as_float(uu[c + 3]) * dq_mul);
          }
        }
      }
      ++item_count;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_attn_bwd_sm100_impl(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, const CUtensorMap& tdo,
                                       const Resolved& p, const float* lse, const float* dvec,
                                       const unsigned* amax, const int4* items_kv,
                                       const int* n_kv, int max_kv,
                                       const int4* items_q, const int* n_q, int max_q,
                                       float* dq_acc, float* dk_acc, void* dv, int* status,
                                       int num_sms, cudaStream_t st) {
  static PerDeviceOnce smem_once_kv, smem_once_q;
  cudaError_t e0 = smem_limit_once(smem_once_kv, attn_bwd_dkv_kernel, kKvSmem);
  if (e0 != cudaSuccess) return e0;
  e0 = smem_limit_once(smem_once_q, attn_bwd_dq_kernel, kQSmem);
  if (e0 != cudaSuccess) return e0;
  BwdArgs a;
  a.T = p.T; a.H = p.H; a.Hk = p.Hk; a.G = p.G; a.R = p.R; a.W = p.W;
  a.logG = 0;
  while ((1 << a.logG) < p.G) ++a.logG;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.lse = lse; a.dvec = dvec; a.amax = amax;
  a.dq_acc = dq_acc; a.dk_acc = dk_acc;
  a.dv = dv;
  a.dv_f32 = p.fp32_out || p.dtype == FLINT_FP32;
  a.status = status;

  a.items = items_kv; a.n_items = n_kv; a.max_items = max_kv;
  a.next_item = status + 4;
  int grid = num_sms < max_kv ? num_sms : max_kv;
  {
    ProfScope prof(kKBwdDkvSm100, st);
    attn_bwd_dkv_kernel<<<grid > 0 ? grid : 1, kThreads, kKvSmem, st>>>(tq, tk, tv, tdo, a);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  a.items = items_q; a.n_items = n_q; a.max_items = max_q;
  a.next_item = status + 5;
  grid = num_sms < max_q ? num_sms : max_q;
  ProfScope prof(kKBwdDqSm100, st);
  attn_bwd_dq_kernel<<<grid > 0 ? grid : 1, kThreads, kQSmem, st>>>(tq, tk, tv, tdo, a);
  return cudaGetLastError();
}

}  // namespace flint
