// attn_x3_sm100.cu - the sink-aware attention forward and backward for FP32
// inputs on Blackwell tensor cores, at FP32 accuracy.
//
// What is computed is the same as in attn_fwd_sm100.cu / attn_bwd_sm100.cu
// (Flint layers page, nemo_automodel.components.models.flint.layers,
// FlintAttention.forward: the sink is one more softmax category with a zero
// value vector; _FlintSinkParameters.forward: FP32 sink logits, not scaled;
// the learned-sink training kernel of the module docstring for the
// gradients). FP32 is the native precision of the Flint config page's
// attention_compute_dtype, so here every tensor-core operand x is carried as
// two fp16 parts, hi = fp16(x) and lo = fp16(x - hi), and every product is
// formed by three MMAs:
//   A B ~ A_hi B_hi + A_hi B_lo + A_lo B_hi        (FP32 accumulation)
// The dropped A_lo B_lo term is below 2^-22 of |A||B|, and hi + lo carries 22
// bits of each operand, so the products keep FP32-level accuracy. Two fp16
// parts take the bytes of one FP32 value, half those of two TF32 parts, and run
// at the f16 tensor rate. fp16's range is handled as on the fp16 path: v and dO
// are multiplied by a power of two from their max |x| (max in [4, 8)), P by a
// fixed power of two (kPBias, kPBiasB) that keeps small probabilities out of
// fp16's subnormal range; the epilogues divide the powers out exactly.
//
// Kernels (persistent, items from LPT-sorted device work lists through a
// global counter, bounded mbarrier waits, one elected lane issues MMAs):
//  * fwd_x3: one 128-row query tile (R tokens x the G heads of a KV group) per
//    item; K and V tiles of 128 keys stream through a ring of five 32 KB slots
//    (one fp16 part per slot, K one tile ahead of V). TMEM: two S buffers (QK of the next key tile
//    runs while the softmax works on this one) and O. P' = 2^kPBias P is split
//    into hi/lo over the S buffer it came from and is the TMEM A operand of PV.
//  * dkv_x3: key-major, 128 keys of one KV head per item, streaming 64-row
//    query tiles (Q and dO parts in shared memory, 3 and 2 stages) from the
//    farthest to the nearest. The tensor cores add each product into the
//    FP32 accumulator after aligning it to the accumulator's exponent, so a
//    small term added to a large sum keeps few bits; a key's largest terms come
//    from the queries just after it (a causal key sees few competitors there),
//    so those tiles go last and the long tail of small terms accumulates while
//    the sum is still small (measured on a 4096-token layer: 16-18x smaller dK
//    and dV errors than near-to-far). V's parts
//    sit in TMEM as the A operand of dP^T = V dO^T, written there by the math
//    warps; K's parts stay in shared memory. TMEM: V_hi, V_lo, dV, dK, X
//    (S^T, then P^T's parts), Y (dP^T, then dS^T's parts).
//  * dq_x3: query-major, one 128-row query tile per item; Q's and dO's parts
//    sit in TMEM as A operands (written by the math warps), K and V tiles of 64
//    keys stream through a ring of 16 KB slots. Two 64-column regions rotate
//    between S/dS and dP as in the dK/dV kernel of the fp16 path.
// An MMA that overwrites a TMEM region an earlier MMA reads is issued right
// behind it without a completion wait: tcgen05.mma operations issued by one
// thread are performed in issue order.
#include <type_traits>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {

namespace {

constexpr uint32_t kChunk128 = 128 * 64 * 2;   // 128 rows x 64 fp16: one 128B-swizzle panel
constexpr uint32_t kPart128 = 2 * kChunk128;   // 128 rows x 128 fp16 (one part of a tile)
constexpr uint32_t kChunk64 = 64 * 64 * 2;     // 64 rows x 64 fp16
constexpr uint32_t kPart64 = 2 * kChunk64;     // 64 rows x 128 fp16
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;      // log2 units
// Forward: P' = 2^kPBias * 2^(s - m) <= 2^(8 + kPBias) = 2^15 < 65504 under the
// lazy rescale, and fp16's subnormal floor (2^-24) sits 2^-31 below the row max.
constexpr float kPBias = 7.0f;
// Backward: P <= 1, so P' = 2^kPBiasB P <= 2^14.
constexpr float kPBiasB = 16384.0f;
constexpr float kInvPBiasB = 1.0f / 16384.0f;

// K-major operand panels (rows of 128 bytes, 8-row groups 1024 bytes apart);
// kk selects the 16-element K slice (of 8) across the two 64-column panels.
__device__ __forceinline__ uint64_t kdesc128(uint32_t base, int kk) {
  return make_sdesc(base + (kk >> 2) * kChunk128 + (kk & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t kdesc64(uint32_t base, int kk) {
  return make_sdesc(base + (kk >> 2) * kChunk64 + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (rows x D, D contiguous) used with K = rows: the two
// 64-column panels are one chunk apart (LBO); kk selects rows [16kk, 16kk+16).
__device__ __forceinline__ uint64_t mndesc128(uint32_t base, int kk) {
  return make_sdesc(base + kk * 2048, kChunk128, 1024);
}
__device__ __forceinline__ uint64_t mndesc64(uint32_t base, int kk) {
  return make_sdesc(base + kk * 2048, kChunk64, 1024);
}

// *p += v, four floats, as a reduction performed in L2 (no value returned).
__device__ __forceinline__ void red_add_f32x4(float* p, float4 v) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
               "f"(v.z), "f"(v.w)
               : "memory");
}

// hi and lo fp16 parts of two values, packed two per 32-bit word.
__device__ __forceinline__ void split_pair(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = pack_f16x2(x0 - hf.x, x1 - hf.y);
}

// A-operand columns of a 64-column region whose two 32-column halves each
// hold the hi part (first 16 columns) and the lo part (next 16) of 32
// K-elements: K slice kk (16 elements) of the hi part, +16 for the lo part.
__device__ __forceinline__ uint32_t half_split_col(int kk) {
  return 32 * (kk >> 1) + 8 * (kk & 1);
}

// ============================================================================
// Forward
// ============================================================================
constexpr int kFThreads = 192;   // warps 0-3 softmax, 4 TMA, 5 MMA
constexpr int kFWarpTma = 4;
constexpr int kFWarpMma = 5;
constexpr int kFSlots = 5;
struct __align__(8) FBars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kFSlots], kv_empty[kFSlots];
  uint64_t s_full[2], p_half[2], p_full[2], pv_done[2];   // per S buffer
  uint64_t o_full, o_empty;
  uint64_t drain;
  ItemRing ring;
};
constexpr uint32_t kFOffQ = 0;                              // Q hi, Q lo
constexpr uint32_t kFOffKV = 2 * kPart128;
constexpr uint32_t kFOffBar = kFOffKV + kFSlots * kPart128;
constexpr uint32_t kFOffTmem = kFOffBar + sizeof(FBars);
constexpr uint32_t kFOffAbort = kFOffTmem + 16;
constexpr uint32_t kFSmem = kFOffAbort + 16;   // no slack: the base is checked instead
static_assert(kFSmem <= 227 * 1024, "exceeds the shared memory of one CTA");
constexpr uint32_t kFColO = 256;               // TMEM: S0 [0,128), S1 [128,256), O

struct X3Args {
  int T, H, Hk, G, R, W, logG;
  float scale, scale_log2;
  const float* sink;
  const float* lse;
  const float* dvec;        // D * s_dout * s_v
  const unsigned* amax;     // [max |dout|, max |v|] slots
  const __half* qs;         // q_hat parts [T, 2H, D]
  const __half* dos;        // dout parts [T, 2H, D]
  const __half* vs;         // v parts [T, 2Hk, D]
  const int4* items;
  const int* n_items;
  int max_items;
  int* next_item;
  float* out;
  float* lse_out;
  float* dq_acc;
  float* dk_acc;
  float* dv;
  int* status;
};

struct FItem {
  int q0, d0, d1, g, kend, ntiles;
};
__device__ __forceinline__ FItem decode_f(const X3Args& a, int idx) {
  const int4 it = a.items[idx];
  FItem r;
  r.q0 = it.x; r.d0 = it.y; r.d1 = it.z; r.g = it.w;
  r.kend = min(r.q0 + a.R, r.d1);
  const int kbeg = a.W > 0 ? max(r.d0, r.q0 - a.W + 1) : r.d0;
  r.ntiles = (r.kend - kbeg + kTileKeys - 1) / kTileKeys;
  return r;
}

// An item's K and V parts go through the ring with K one key tile ahead of V:
// K(0), then K(n+1), V(n) for n = 0, 1, ..., and V(nt-1) last (hi part, then
// lo part, each). K(n+2) then lands in slots that QK(n+1) and PV(n-1) free, so
// QK(n+2) never waits for a load, and V(n+1) loads while QK(n+2) runs. Load
// positions within the item (in single-part loads; the lo part follows):
__device__ __forceinline__ uint32_t fwd_pos_k(uint32_t n) { return n == 0 ? 0u : 4 * n - 2; }
__device__ __forceinline__ uint32_t fwd_pos_v(uint32_t n, uint32_t nt) {
  return n + 1 < nt ? 4 * n + 4 : 4 * n + 2;
}
// Which tile (and whether K or V) the item's pj-th part pair is.
__device__ __forceinline__ void fwd_pair(int pj, int nt, int& tile, bool& is_v) {
  if (pj == 0) { tile = 0; is_v = false; return; }
  const int r = pj - 1;
  if (r < 2 * (nt - 1)) { tile = (r >> 1) + ((r & 1) ? 0 : 1); is_v = (r & 1) != 0; }
  else { tile = nt - 1; is_v = true; }
}

// Tiles are numbered per CTA across items (t): tile t uses S buffer t & 1.
__global__ void __launch_bounds__(kFThreads, 1)
attn_fwd_x3_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const X3Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  FBars* bars = reinterpret_cast<FBars*>(smem + kFOffBar);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kFOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFOffAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, a.status, kStatusTimeoutFwd};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 1);
    for (int s = 0; s < kFSlots; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->s_full[b]), 1);
      mbar_init(smem_u32(&bars->p_half[b]), 4);
      mbar_init(smem_u32(&bars->p_full[b]), 4);
      mbar_init(smem_u32(&bars->pv_done[b]), 1);
    }
    mbar_init(smem_u32(&bars->o_full), 1);
    mbar_init(smem_u32(&bars->o_empty), 4);
    mbar_init(smem_u32(&bars->drain), 1);
    ring_init(&bars->ring, 5);   // the MMA warp and the 4 softmax warps consume
    fence_mbar_init();
  }
  if (warp == kFWarpMma) {
    tmem_alloc(smem_u32((const void*)tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = min(*a.n_items, a.max_items);

  if (warp == kFWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_load = 0, item_count = 0, q_arm = 0, arm[kFSlots] = {};
      bool ok = true;
      while (ok) {
        int idx = atomicAdd(a.next_item, 1);
        if (idx >= n_items) idx = -1;
        ok = ring_push(&bars->ring, item_count, idx, wc);
        if (!ok || idx < 0) break;
        const FItem it = decode_f(a, idx);
        if (item_count > 0) ok = mbar_wait(smem_u32(&bars->q_empty), (item_count - 1) & 1, wc);
        if (!ok) break;
        const uint32_t qf = smem_u32(&bars->q_full);
        mbar_arrive_expect_tx(qf, 2 * kPart128);
        ++q_arm;
        for (int part = 0; part < 2; ++part)
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sbase + kFOffQ + part * kPart128 + c * kChunk128, &tm_q, qf, c * 64,
                        part * a.H + it.g * a.G, it.q0);
        for (int j = 0; j < 4 * it.ntiles && ok; ++j, ++kv_load) {
          int tile;
          bool is_v;
          fwd_pair(j >> 1, it.ntiles, tile, is_v);
          const int ks = it.kend - kTileKeys * (tile + 1);
          const uint32_t s = kv_load % kFSlots, ph = (kv_load / kFSlots) & 1;
          if (kv_load >= kFSlots) ok = mbar_wait(smem_u32(&bars->kv_empty[s]), ph ^ 1, wc);
          if (!ok) break;
          const uint32_t f = smem_u32(&bars->kv_full[s]);
          mbar_arrive_expect_tx(f, kPart128);
          ++arm[s];
          const CUtensorMap* m = is_v ? &tm_v : &tm_k;
          const int y = (j & 1) ? a.Hk + it.g : it.g;   // lo part rows follow the hi rows
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sbase + kFOffKV + s * kPart128 + c * kChunk128, m, f, c * 64, y, ks);
        }
        ++item_count;
      }
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutFwd};
      if (q_arm) mbar_wait(smem_u32(&bars->q_full), (q_arm - 1) & 1, drain);
      for (int s = 0; s < kFSlots; ++s)
        if (arm[s]) mbar_wait(smem_u32(&bars->kv_full[s]), (arm[s] - 1) & 1, drain);
    }
  } else if (warp == kFWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Order: QK(t), QK(t+1); then per tile PV(t) and QK(t+2). QK(t+2) reuses
    // the S buffer whose P(t) PV(t) reads and is issued right behind it (MMAs
    // are performed in issue order); pv_done tells the softmax when PV(t) has
    // completed (it rescales O).
    const uint32_t leader = elect_one();
    const uint32_t idesc_qk = make_idesc_f16(128, 128, 0, 0);
    const uint32_t idesc_pv = make_idesc_f16(128, 128, 0, 1);
    const uint32_t qh = sbase + kFOffQ, ql = sbase + kFOffQ + kPart128;
    uint32_t item_count = 0, t = 0, kv_base = 0;
    bool ok = true;
    auto slot = [&](uint32_t pos) { return sbase + kFOffKV + (pos % kFSlots) * kPart128; };
    auto wait_full = [&](uint32_t pos) {
      return mbar_wait_warp(smem_u32(&bars->kv_full[pos % kFSlots]), (pos / kFSlots) & 1, wc);
    };
    // S(tt) = Q K(tt)^T for tile n of the item; last: the item's last QK frees Q.
    auto issue_qk = [&](uint32_t n, uint32_t tt, bool last) -> bool {
      const uint32_t b = tt & 1, pos = kv_base + fwd_pos_k(n);
      if (!wait_full(pos) || !wait_full(pos + 1)) return false;
      tc_fence_after();
      const uint32_t kh = slot(pos), kl = slot(pos + 1), d = tmem + b * 128;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(d, kdesc128(qh, kk), kdesc128(kl, kk), idesc_qk, kk > 0, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(d, kdesc128(ql, kk), kdesc128(kh, kk), idesc_qk, 1u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(d, kdesc128(qh, kk), kdesc128(kh, kk), idesc_qk, 1u, leader);
      mma_commit_w(smem_u32(&bars->s_full[b]), leader);
      mma_commit_w(smem_u32(&bars->kv_empty[pos % kFSlots]), leader);
      mma_commit_w(smem_u32(&bars->kv_empty[(pos + 1) % kFSlots]), leader);
      if (last) mma_commit_w(smem_u32(&bars->q_empty), leader);
      return true;
    };
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const FItem it = decode_f(a, idx);
      const uint32_t nt = (uint32_t)it.ntiles;
      ok = mbar_wait_warp(smem_u32(&bars->q_full), item_count & 1, wc);
      if (!ok) break;
      tc_fence_after();
      ok = issue_qk(0, t, nt == 1);
      if (ok && nt > 1) ok = issue_qk(1, t + 1, nt == 2);
      for (uint32_t n = 0; n < nt && ok; ++n) {
        const uint32_t tt = t + n, b = tt & 1, ph = (tt >> 1) & 1;
        const uint32_t pos = kv_base + fwd_pos_v(n, nt);        // V_hi, V_lo
        ok = wait_full(pos) && wait_full(pos + 1);
        if (ok) ok = mbar_wait_warp(smem_u32(&bars->p_half[b]), ph, wc);
        if (ok && n == 0 && item_count > 0)
          ok = mbar_wait_warp(smem_u32(&bars->o_empty), (item_count - 1) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        const uint32_t vh = slot(pos), vl = slot(pos + 1), sb = tmem + b * 128;
        const uint32_t o = tmem + kFColO;
        // keys 0-63: P' hi in columns [0,32), lo in [32,64) of the S buffer
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t ah = sb + kk * 8, al = ah + 32;
          mma_ts_w(o, ah, mndesc128(vl, kk), idesc_pv, (n > 0 || kk > 0) ? 1u : 0u, leader);
          mma_ts_w(o, al, mndesc128(vh, kk), idesc_pv, 1u, leader);
          mma_ts_w(o, ah, mndesc128(vh, kk), idesc_pv, 1u, leader);
        }
        ok = mbar_wait_warp(smem_u32(&bars->p_full[b]), ph, wc);
        if (!ok) break;
        tc_fence_after();
        // keys 64-127: hi in [64,96), lo in [96,128)
#pragma unroll
        for (int kk = 4; kk < 8; ++kk) {
          const uint32_t ah = sb + 64 + (kk - 4) * 8, al = ah + 32;
          mma_ts_w(o, ah, mndesc128(vl, kk), idesc_pv, 1u, leader);
          mma_ts_w(o, al, mndesc128(vh, kk), idesc_pv, 1u, leader);
          mma_ts_w(o, ah, mndesc128(vh, kk), idesc_pv, 1u, leader);
        }
        mma_commit_w(smem_u32(&bars->pv_done[b]), leader);
        mma_commit_w(smem_u32(&bars->kv_empty[pos % kFSlots]), leader);
        mma_commit_w(smem_u32(&bars->kv_empty[(pos + 1) % kFSlots]), leader);
        if (n + 1 == nt) mma_commit_w(smem_u32(&bars->o_full), leader);
        if (n + 2 < nt) ok = issue_qk(n + 2, tt + 2, n + 3 == nt);
      }
      if (!ok) break;
      kv_base += 4 * nt;
      t += nt;
      ++item_count;
    }
    mma_commit_w(smem_u32(&bars->drain), leader);
    volatile int no_abort = 0;
    const WaitCtx drain{&no_abort, a.status, kStatusTimeoutFwd};
    mbar_wait_warp(smem_u32(&bars->drain), 0, drain);
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int r = warp * 32 + lane;        // row of the tile = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);
    const float inv_sv = slot_scale(a.amax + 1, true);
    uint32_t t = 0, item_count = 0;
    bool ok = true;
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const FItem it = decode_f(a, idx);
      const int tok = it.q0 + (r >> a.logG);
      const int h = it.g * a.G + (r & (a.G - 1));
      const bool valid = tok < it.d1;
      const int lo_r = a.W > 0 ? max(it.d0, tok - a.W + 1) : it.d0;
      const float sink2 = __ldg(a.sink + h) * kLog2e;
      float m = sink2;                     // running max (log2 units)
      float l = exp2f(kPBias);             // running sum of P', the sink's included
      for (int n = 0; n < it.ntiles; ++n) {
        const uint32_t tt = t + n, b = tt & 1;
        const uint32_t s_col = b * 128;
        const int ks = it.kend - kTileKeys * (n + 1);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[b]), (tt >> 1) & 1, wc));
        if (!ok) break;
        tc_fence_after();
        const bool needs_mask = (ks + kTileKeys - 1 > it.q0) || (ks < it.d0) ||
                                (a.W > 0 && ks < it.q0 + a.R - a.W);
        const int c_lo = needs_mask ? lo_r - ks : 0;
        const int c_hi = needs_mask ? tok - ks : 127;
        uint32_t u0[32], u1[32], u2[32], u3[32];
        tmem_ld32(t_row + s_col, u0);
        tmem_ld32(t_row + s_col + 32, u1);
        tmem_ld32(t_row + s_col + 64, u2);
        tmem_ld32(t_row + s_col + 96, u3);
        tc_wait_ld_dep(u0);
        tc_wait_ld_dep(u1);
        tc_wait_ld_dep(u2);
        tc_wait_ld_dep(u3);
        float mx0 = -INFINITY, mx1 = -INFINITY;
        auto row_max = [&](auto masked) {
          auto one = [&](uint32_t (&u)[32], int c0) {
            if (decltype(masked)::value) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c0 + e < c_lo || c0 + e > c_hi) u[e] = 0xff800000u;   // -inf
            }
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              mx0 = fmax3(mx0, __uint_as_float(u[e]), __uint_as_float(u[e + 1]));
              mx1 = fmax3(mx1, __uint_as_float(u[e + 2]), __uint_as_float(u[e + 3]));
            }
          };
          one(u0, 0);
          one(u1, 32);
          one(u2, 64);
          one(u3, 96);
        };
        if (needs_mask) row_max(std::true_type{});
        else row_max(std::false_type{});
        const float m_tile = fmaxf(mx0, mx1) * a.scale_log2;
        float alpha = 1.f;
        bool rescale_o = false;
        if (n == 0) {
          if (m_tile > m) { alpha = ex2_approx(m - m_tile); m = m_tile; }
        } else if (m_tile > m + kRescaleThreshold) {
          alpha = ex2_approx(m - m_tile);
          m = m_tile;
          rescale_o = true;
        }
        l *= alpha;
        const float mb = (m == -INFINITY) ? 0.f : m;
        const uint64_t sc2 = f2(a.scale_log2, a.scale_log2);
        const uint64_t nm2 = f2(kPBias - mb, kPBias - mb);
        uint64_t rs2 = f2(0.f, 0.f);
        // P' = 2^(s*scale - m + kPBias) for 32 keys; hi and lo parts to TMEM.
        // Chunk c holds keys [32c, 32c+32): hi at columns 64(c>>1) + 16(c&1),
        // lo 32 columns further (S was read whole above).
        auto exp_chunk = [&](const uint32_t (&u)[32], int c) {
          uint32_t ph[16], pl[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2_split(ffma2(f2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])), sc2, nm2),
                     x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            rs2 = fadd2(rs2, f2(p0, p1));
            split_pair(p0, p1, ph[e], pl[e]);
          }
          const uint32_t col = s_col + 64 * (c >> 1) + 16 * (c & 1);
          tmem_st16(t_row + col, ph);
          tmem_st16(t_row + col + 32, pl);
        };
        exp_chunk(u0, 0);
        if (__any_sync(0xffffffffu, rescale_o)) {
          // O holds PV(tt - 1), which may still run: wait for it, then scale.
          const uint32_t pb = (tt - 1) & 1;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(smem_u32(&bars->pv_done[pb]), ((tt - 1) >> 1) & 1, wc));
          if (!ok) break;
          tc_fence_after();
          const uint64_t a2 = f2(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t u[32];
            tmem_ld32(t_row + kFColO + c * 32, u);
            tc_wait_ld_dep(u);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float x0, x1;
              f2_split(fmul2(f2(__uint_as_float(u[e]), __uint_as_float(u[e + 1])), a2), x0, x1);
              u[e] = __float_as_uint(x0);
              u[e + 1] = __float_as_uint(x1);
            }
            tmem_st32(t_row + kFColO + c * 32, u);
          }
        }
        exp_chunk(u1, 1);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_half[b]));
        exp_chunk(u2, 2);
        exp_chunk(u3, 3);
        float rs_lo, rs_hi;
        f2_split(rs2, rs_lo, rs_hi);
        l += rs_lo + rs_hi;
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[b]));
      }
      if (!ok) break;
      t += it.ntiles;
      // epilogue: O / l -> fp32 out, LSE
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->o_full), item_count & 1, wc));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = inv_sv / l;
      const uint64_t il2 = f2(inv_l, inv_l);
      float* orow = a.out + ((size_t)tok * a.H + h) * kHeadDim;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        tmem_ld32(t_row + kFColO + c * 32, u);
        tc_wait_ld_dep(u);
        if (c == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->o_empty));
        }
        if (valid) {
          float o[32];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            f2_split(fmul2(f2(__uint_as_float(u[e]), __uint_as_float(u[e + 1])), il2), o[e],
                     o[e + 1]);
#pragma unroll
          for (int v4 = 0; v4 < 8; ++v4)
            *reinterpret_cast<float4*>(orow + c * 32 + 4 * v4) =
                make_float4(o[4 * v4], o[4 * v4 + 1], o[4 * v4 + 2], o[4 * v4 + 3]);
        }
      }
      if (valid) a.lse_out[(size_t)h * a.T + tok] = (m - kPBias + log2f(l)) * kLn2;
      ++item_count;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kFWarpMma) tmem_dealloc(tmem, 512);
}

// ============================================================================
// dK / dV : key-major, 64-row query tiles
// ============================================================================
constexpr int kBThreads = 320;   // warps 0-7 math (two warpgroups), 8 TMA, 9 MMA
constexpr int kBWarpTma = 8;
constexpr int kBWarpMma = 9;
constexpr int kBMathWarps = 8;
constexpr int kKQStages = 3;
constexpr int kQRows = 64;       // query rows per tile of the dK/dV kernel
// dV and dK leave TMEM every kDrainTiles query tiles: the first drain of an item
// stores them, later ones add (FP32 reductions in L2, in program order), so no
// TMEM accumulation chain is longer than kDrainTiles * 12 MMAs.
constexpr int kDrainTiles = 16;
struct __align__(8) KBars {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[kKQStages], q_empty[kKQStages], do_full[2], do_empty[2];
  uint64_t v_full, s_full, dp_full, p_full, ds_full, acc_full, acc_empty;
  uint64_t drain;
  ItemRing ring;
};
constexpr uint32_t kKOffK = 0;                                   // K hi, K lo (128 keys)
constexpr uint32_t kKOffQ = 2 * kPart128;                        // kKQStages x (hi, lo)
constexpr uint32_t kKOffDO = kKOffQ + kKQStages * 2 * kPart64;   // 2 x (hi, lo)
constexpr uint32_t kKOffStats = kKOffDO + 2 * 2 * kPart64;       // [2][2][64] fp32
constexpr uint32_t kKOffBar = kKOffStats + 2 * 2 * kQRows * 4;
constexpr uint32_t kKOffTmem = kKOffBar + sizeof(KBars);
constexpr uint32_t kKOffAbort = kKOffTmem + 16;
constexpr uint32_t kKSmem = kKOffAbort + 16;
static_assert(kKSmem <= 227 * 1024, "exceeds the shared memory of one CTA");
// TMEM columns
constexpr uint32_t kKColVH = 0, kKColVL = 64, kKColDV = 128, kKColDK = 256, kKColX = 384,
                   kKColY = 448;

struct KItem {
  int k0, d0, d1, g, qend, nq, R64;
};
__device__ __forceinline__ KItem decode_k(const X3Args& a, int idx) {
  const int4 it = a.items[idx];
  KItem r;
  r.k0 = it.x; r.d0 = it.y; r.d1 = it.z; r.g = it.w;
  r.R64 = kQRows >> a.logG;
  r.qend = a.W > 0 ? min(r.d1, r.k0 + kTileKeys - 1 + a.W) : r.d1;
  r.nq = (r.qend - r.k0 + r.R64 - 1) / r.R64;
  return r;
}

__global__ void __launch_bounds__(kBThreads, 1)
attn_bwd_dkv_x3_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_do, const X3Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  KBars* bars = reinterpret_cast<KBars*>(smem + kKOffBar);
  float* stats = reinterpret_cast<float*>(smem + kKOffStats);   // [buf][-lse2|D][64]
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kKOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kKOffAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, a.status, kStatusTimeoutBwdKV};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(smem_u32(&bars->kv_full), 1);
    mbar_init(smem_u32(&bars->kv_empty), 1);
    for (int s = 0; s < kKQStages; ++s) {
      mbar_init(smem_u32(&bars->q_full[s]), 1);
      mbar_init(smem_u32(&bars->q_empty[s]), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->do_full[s]), 2);   // TMA bytes + per-row statistics
      mbar_init(smem_u32(&bars->do_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->v_full), kBMathWarps);
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->p_full), kBMathWarps);
    mbar_init(smem_u32(&bars->ds_full), kBMathWarps);
    mbar_init(smem_u32(&bars->acc_full), 1);
    mbar_init(smem_u32(&bars->acc_empty), kBMathWarps);
    mbar_init(smem_u32(&bars->drain), 1);
    ring_init(&bars->ring, kBMathWarps + 1);
    fence_mbar_init();
  }
  if (warp == kBWarpMma) {
    tmem_alloc(smem_u32((const void*)tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = min(*a.n_items, a.max_items);

  if (warp == kBWarpTma) {
    // Lane 0 takes items and issues TMA; the whole warp stages each query
    // tile's per-row -log2-LSE and D and completes do_full's second arrival.
    uint32_t item_count = 0, qd_iter = 0, kv_arm = 0, q_arm[kKQStages] = {}, do_arm[2] = {};
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
      const KItem it = decode_k(a, idx);
      if (lane == 0) {
        if (item_count > 0) ok = mbar_wait(smem_u32(&bars->kv_empty), (item_count - 1) & 1, wc);
        if (ok) {
          const uint32_t kf = smem_u32(&bars->kv_full);
          mbar_arrive_expect_tx(kf, 2 * kPart128);
          ++kv_arm;
          for (int part = 0; part < 2; ++part)
            for (int c = 0; c < 2; ++c)
              tma_load_3d(sbase + kKOffK + part * kPart128 + c * kChunk128, &tm_k, kf, c * 64,
                          part * a.Hk + it.g, it.k0);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int m = 0; m < it.nq && ok; ++m, ++qd_iter) {
        const int qs = it.k0 + (it.nq - 1 - m) * it.R64;   // far to near
        const uint32_t sq = qd_iter % kKQStages, phq = (qd_iter / kKQStages) & 1;
        const uint32_t s = qd_iter & 1, ph = (qd_iter >> 1) & 1;
        float lse2[2], dr[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int r = lane + 32 * e;
          const int tok = qs + (r >> a.logG), h = it.g * a.G + (r & (a.G - 1));
          const bool vr = tok < it.d1;
          lse2[e] = vr ? -__ldg(a.lse + (size_t)h * a.T + tok) * kLog2e : 0.f;   // negated
          dr[e] = vr ? __ldg(a.dvec + (size_t)h * a.T + tok) : 0.f;
        }
        const uint32_t qf = smem_u32(&bars->q_full[sq]), df = smem_u32(&bars->do_full[s]);
        if (lane == 0) {
          if (qd_iter >= kKQStages) ok = mbar_wait(smem_u32(&bars->q_empty[sq]), phq ^ 1, wc);
          if (ok) {
            mbar_arrive_expect_tx(qf, 2 * kPart64);
            ++q_arm[sq];
            for (int part = 0; part < 2; ++part)
              for (int c = 0; c < 2; ++c)
                tma_load_3d(sbase + kKOffQ + (2 * sq + part) * kPart64 + c * kChunk64, &tm_q, qf,
                            c * 64, part * a.H + it.g * a.G, qs);
          }
          if (ok && qd_iter >= 2) ok = mbar_wait(smem_u32(&bars->do_empty[s]), ph ^ 1, wc);
          if (ok) {
            mbar_arrive_expect_tx(df, 2 * kPart64);
            ++do_arm[s];
            for (int part = 0; part < 2; ++part)
              for (int c = 0; c < 2; ++c)
                tma_load_3d(sbase + kKOffDO + (2 * s + part) * kPart64 + c * kChunk64, &tm_do,
                            df, c * 64, part * a.H + it.g * a.G, qs);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        float* st = stats + s * 2 * kQRows;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          st[lane + 32 * e] = lse2[e];
          st[kQRows + lane + 32 * e] = dr[e];
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
      for (int s = 0; s < kKQStages; ++s)
        if (q_arm[s]) mbar_wait(smem_u32(&bars->q_full[s]), (q_arm[s] - 1) & 1, drain);
      for (int s = 0; s < 2; ++s)
        if (do_arm[s]) mbar_wait(smem_u32(&bars->do_full[s]), (do_arm[s] - 1) & 1, drain);
    }
  } else if (warp == kBWarpMma) {
    // Per query tile t: S^T(t) into X, dP^T(t) into Y; the math warps write
    // P'^T(t) over X and dS^T(t) over Y. Issue order: dV(t), S^T(t+1) (right
    // behind dV(t), which reads X), dK(t), dP^T(t+1) (behind dK(t): Y).
    const uint32_t leader = elect_one();
    const uint32_t idesc_s = make_idesc_f16(128, kQRows, 0, 0);
    const uint32_t idesc_acc = make_idesc_f16(128, 128, 0, 1);
    const uint32_t kh = sbase + kKOffK, kl = sbase + kKOffK + kPart128;
    const uint32_t X = tmem + kKColX, Y = tmem + kKColY;
    uint32_t item_count = 0, t = 0, p_cnt = 0, ds_cnt = 0, drains = 0;
    bool ok = true;
    auto qstage = [&](uint32_t tt) { return sbase + kKOffQ + (tt % kKQStages) * 2 * kPart64; };
    auto dostage = [&](uint32_t tt) { return sbase + kKOffDO + (tt & 1) * 2 * kPart64; };
    auto issue_s = [&](uint32_t tt) {          // S^T(tt) = K Q(tt)^T into X
      const uint32_t qh = qstage(tt), ql = qh + kPart64;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(X, kdesc128(kh, kk), kdesc64(ql, kk), idesc_s, kk > 0, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(X, kdesc128(kl, kk), kdesc64(qh, kk), idesc_s, 1u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss_w(X, kdesc128(kh, kk), kdesc64(qh, kk), idesc_s, 1u, leader);
      mma_commit_w(smem_u32(&bars->s_full), leader);
    };
    auto issue_dp = [&](uint32_t tt) {         // dP^T(tt) = V dO(tt)^T into Y, V from TMEM
      const uint32_t dh = dostage(tt), dl = dh + kPart64;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(Y, tmem + kKColVH + kk * 8, kdesc64(dl, kk), idesc_s, kk > 0, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(Y, tmem + kKColVL + kk * 8, kdesc64(dh, kk), idesc_s, 1u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(Y, tmem + kKColVH + kk * 8, kdesc64(dh, kk), idesc_s, 1u, leader);
      mma_commit_w(smem_u32(&bars->dp_full), leader);
    };
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const KItem it = decode_k(a, idx);
      ok = mbar_wait_warp(smem_u32(&bars->kv_full), item_count & 1, wc);
      if (ok) ok = mbar_wait_warp(smem_u32(&bars->q_full[t % kKQStages]),
                                  (t / kKQStages) & 1, wc);
      if (!ok) break;
      tc_fence_after();
      issue_s(t);
      ok = mbar_wait_warp(smem_u32(&bars->v_full), item_count & 1, wc);
      if (ok) ok = mbar_wait_warp(smem_u32(&bars->do_full[t & 1]), (t >> 1) & 1, wc);
      if (!ok) break;
      tc_fence_after();
      issue_dp(t);
      for (int m = 0; m < it.nq && ok; ++m, ++t) {
        const bool has_next = m + 1 < it.nq;
        const bool c_first = m % kDrainTiles == 0;                  // dV, dK start over
        const bool c_last = (m + 1) % kDrainTiles == 0 || !has_next;  // then drained
        const uint32_t dh = dostage(t), dl = dh + kPart64;
        const uint32_t qh = qstage(t), ql = qh + kPart64;
        // dV += P'^T(t) dO(t)
        ok = mbar_wait_warp(smem_u32(&bars->p_full), p_cnt & 1, wc);
        ++p_cnt;
        if (ok && c_first && drains > 0)
          ok = mbar_wait_warp(smem_u32(&bars->acc_empty), (drains - 1) & 1, wc);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t ah = X + half_split_col(kk), al = ah + 16;
          mma_ts_w(tmem + kKColDV, ah, mndesc64(dl, kk), idesc_acc,
                   (!c_first || kk > 0) ? 1u : 0u, leader);
          mma_ts_w(tmem + kKColDV, al, mndesc64(dh, kk), idesc_acc, 1u, leader);
          mma_ts_w(tmem + kKColDV, ah, mndesc64(dh, kk), idesc_acc, 1u, leader);
        }
        if (has_next) {
          ok = mbar_wait_warp(smem_u32(&bars->q_full[(t + 1) % kKQStages]),
                              ((t + 1) / kKQStages) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          issue_s(t + 1);
        }
        // dS^T(t) written; dO(t) and its statistics are no longer needed
        ok = mbar_wait_warp(smem_u32(&bars->ds_full), ds_cnt & 1, wc);
        ++ds_cnt;
        if (!ok) break;
        tc_fence_after();
        mma_commit_w(smem_u32(&bars->do_empty[t & 1]), leader);
        // dK += dS^T(t) Q(t)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t ah = Y + half_split_col(kk), al = ah + 16;
          mma_ts_w(tmem + kKColDK, ah, mndesc64(ql, kk), idesc_acc,
                   (!c_first || kk > 0) ? 1u : 0u, leader);
          mma_ts_w(tmem + kKColDK, al, mndesc64(qh, kk), idesc_acc, 1u, leader);
          mma_ts_w(tmem + kKColDK, ah, mndesc64(qh, kk), idesc_acc, 1u, leader);
        }
        mma_commit_w(smem_u32(&bars->q_empty[t % kKQStages]), leader);
        if (c_last) {
          mma_commit_w(smem_u32(&bars->acc_full), leader);
          ++drains;
        }
        if (has_next) {
          ok = mbar_wait_warp(smem_u32(&bars->do_full[(t + 1) & 1]), ((t + 1) >> 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
          issue_dp(t + 1);
        }
      }
      if (!ok) break;
      mma_commit_w(smem_u32(&bars->kv_empty), leader);
      ++item_count;
    }
    mma_commit_w(smem_u32(&bars->drain), leader);
    volatile int no_abort = 0;
    const WaitCtx drain{&no_abort, a.status, kStatusTimeoutBwdKV};
    mbar_wait_warp(smem_u32(&bars->drain), 0, drain);
  } else {
    // ---------------------------------------------------------------- math warps
    const int wg = warp >> 2;                      // query rows [32wg, 32wg+32) of a tile
    const int kl = (warp & 3) * 32 + lane;         // key row of the item = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int c0 = 32 * wg;
    // dV carries 2^kPBiasB and the scale of dO's parts; dK those of dO and v
    const float inv_sdo = slot_scale(a.amax, true);
    const float dv_mul = inv_sdo * kInvPBiasB;
    const float dk_mul = a.scale * inv_sdo * slot_scale(a.amax + 1, true);
    const uint64_t sc2 = f2(a.scale_log2, a.scale_log2);
    uint32_t item_count = 0, tile_count = 0, drains = 0;
    bool ok = true;
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const KItem it = decode_k(a, idx);
      const int j = it.k0 + kl;
      const bool valid_key = j < it.d1;
      {
        // V's parts into TMEM (warpgroup 0: hi, 1: lo): the A operand of dP^T.
        // Every MMA of the previous item has completed (the acc_full of its
        // last drain), so nothing reads these columns any more.
        const uint4* src = reinterpret_cast<const uint4*>(
            a.vs + ((size_t)j * 2 * a.Hk + wg * a.Hk + it.g) * kHeadDim);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint4 v4 = valid_key ? __ldg(src + hh * 8 + i) : make_uint4(0, 0, 0, 0);
            w[4 * i] = v4.x; w[4 * i + 1] = v4.y; w[4 * i + 2] = v4.z; w[4 * i + 3] = v4.w;
          }
          tmem_st32(t_row + kKColVH + wg * 64 + hh * 32, w);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->v_full));
      }
      for (int m = 0; m < it.nq; ++m, ++tile_count) {
        const int qs = it.k0 + (it.nq - 1 - m) * it.R64;   // far to near
        const uint32_t stg = tile_count & 1, ph = (tile_count >> 1) & 1;
        const float* st = stats + stg * 2 * kQRows;
        const bool needs_mask = (it.k0 + kTileKeys - 1 > qs) || (it.k0 + kTileKeys > it.d1) ||
                                (qs + it.R64 > it.d1) ||
                                (a.W > 0 && qs + it.R64 - 1 - it.k0 >= a.W);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->do_full[stg]), ph, wc));
        if (!ok) break;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full), tile_count & 1, wc));
        if (!ok) break;
        tc_fence_after();
        // Row c of the tile is token qs + c/G, so the rows that see key j form
        // one range [cmin, cmax).
        int cmin = 0, cmax = kQRows;
        if (needs_mask) {
          const int qend_j = a.W > 0 ? min(it.d1, j + a.W) : it.d1;
          cmin = valid_key ? max(0, (j - qs) * a.G) : kQRows;
          cmax = valid_key ? min(kQRows, (qend_j - qs) * a.G) : 0;
        }
        float p[32];
        {
          uint32_t u[32], ph16[16], pl16[16];
          tmem_ld32(t_row + kKColX + c0, u);
          tc_wait_ld_dep(u);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = c0 + 2 * e;
            const uint64_t nl2 = *reinterpret_cast<const uint64_t*>(st + c);   // -lse2 pair
            float x0, x1;
            f2_split(ffma2(f2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])), sc2,
                           nl2), x0, x1);
            float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            if (needs_mask) {
              p0 = (c >= cmin && c < cmax) ? p0 : 0.f;
              p1 = (c + 1 >= cmin && c + 1 < cmax) ? p1 : 0.f;
            }
            p[2 * e] = p0;
            p[2 * e + 1] = p1;
            split_pair(p0 * kPBiasB, p1 * kPBiasB, ph16[e], pl16[e]);
          }
          tmem_st16(t_row + kKColX + c0, ph16);        // P'^T hi, then lo, over S^T
          tmem_st16(t_row + kKColX + c0 + 16, pl16);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full));
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->dp_full), tile_count & 1, wc));
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t u[32], dh16[16], dl16[16];
          tmem_ld32(t_row + kKColY + c0, u);
          tc_wait_ld_dep(u);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = c0 + 2 * e;
            const float2 dd = *reinterpret_cast<const float2*>(st + kQRows + c);
            const float ds0 = p[2 * e] * (__uint_as_float(u[2 * e]) - dd.x);
            const float ds1 = p[2 * e + 1] * (__uint_as_float(u[2 * e + 1]) - dd.y);
            split_pair(ds0, ds1, dh16[e], dl16[e]);
          }
          tmem_st16(t_row + kKColY + c0, dh16);        // dS^T hi, then lo, over dP^T
          tmem_st16(t_row + kKColY + c0 + 16, dl16);
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->ds_full));
        if ((m + 1) % kDrainTiles == 0 || m + 1 == it.nq) {
          // drain: this warpgroup owns channels [64wg, 64wg+64) of the key row
          ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->acc_full), drains & 1, wc));
          if (!ok) break;
          tc_fence_after();
          uint32_t v0[32], v1[32], k0[32], k1[32];
          tmem_ld32(t_row + kKColDV + 64 * wg, v0);
          tmem_ld32(t_row + kKColDV + 64 * wg + 32, v1);
          tmem_ld32(t_row + kKColDK + 64 * wg, k0);
          tmem_ld32(t_row + kKColDK + 64 * wg + 32, k1);
          tc_wait_ld_dep(v0);
          tc_wait_ld_dep(v1);
          tc_wait_ld_dep(k0);
          tc_wait_ld_dep(k1);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty));
          ++drains;
          if (valid_key) {
            const bool first = m < kDrainTiles;    // the item's first drain stores
            const size_t rb = ((size_t)j * a.Hk + it.g) * kHeadDim + 64 * wg;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t* vv = hh ? v1 : v0;
              const uint32_t* kv = hh ? k1 : k0;
              float* dvrow = a.dv + rb + hh * 32;
              float* dkrow = a.dk_acc + rb + hh * 32;
#pragma unroll
              for (int c = 0; c < 32; c += 4) {
                const float4 fv = make_float4(
                    __uint_as_float(vv[c]) * dv_mul, __uint_as_float(vv[c + 1]) * dv_mul,
                    __uint_as_float(vv[c + 2]) * dv_mul, __uint_as_float(vv[c + 3]) * dv_mul);
                const float4 fk = make_float4(
                    __uint_as_float(kv[c]) * dk_mul, __uint_as_float(kv[c + 1]) * dk_mul,
                    __uint_as_float(kv[c + 2]) * dk_mul, __uint_as_float(kv[c + 3]) * dk_mul);
                if (first) {
                  *reinterpret_cast<float4*>(dvrow + c) = fv;
                  *reinterpret_cast<float4*>(dkrow + c) = fk;
                } else {
                  red_add_f32x4(dvrow + c, fv);
                  red_add_f32x4(dkrow + c, fk);
                }
              }
            }
          }
        }
      }
      if (!ok) break;
      ++item_count;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBWarpMma) tmem_dealloc(tmem, 512);
}

// ============================================================================
// dQ : query-major, 64-key tiles
// ============================================================================
// K and V parts stream through a ring of kDSlots 16 KB slots in the order
// K_hi(t), K_lo(t), V_hi(t), V_lo(t), ...; V(t) is released by dP(t), K(t) by dQ(t).
constexpr int kDSlots = 12;
constexpr int kDKeys = 64;       // keys per tile of the dQ kernel
struct __align__(8) DBars {
  uint64_t kv_full[kDSlots], kv_empty[kDSlots];
  uint64_t qd_full, s_full, dp_full, dp_free, ds_full, acc_full, acc_empty;
  uint64_t drain;
  ItemRing ring;
};
constexpr uint32_t kDOffKV = 0;
constexpr uint32_t kDOffBar = kDSlots * kPart64;
constexpr uint32_t kDOffTmem = kDOffBar + sizeof(DBars);
constexpr uint32_t kDOffAbort = kDOffTmem + 16;
constexpr uint32_t kDSmem = kDOffAbort + 16;
static_assert(kDSmem <= 227 * 1024, "exceeds the shared memory of one CTA");
// TMEM columns: the A operands Q_hi, Q_lo, dO_hi, dO_lo; two rotating 64-column
// regions; the dQ accumulator.
constexpr uint32_t kDColQH = 0, kDColQL = 64, kDColDOH = 128, kDColDOL = 192, kDColR = 256,
                   kDColDQ = 384;

struct DItem {
  int q0, d0, d1, g, kend, ntiles;
};
__device__ __forceinline__ DItem decode_d(const X3Args& a, int idx) {
  const int4 it = a.items[idx];
  DItem r;
  r.q0 = it.x; r.d0 = it.y; r.d1 = it.z; r.g = it.w;
  r.kend = min(r.q0 + a.R, r.d1);
  const int kbeg = a.W > 0 ? max(r.d0, r.q0 - a.W + 1) : r.d0;
  r.ntiles = (r.kend - kbeg + kDKeys - 1) / kDKeys;
  return r;
}

// Tiles are numbered per CTA across items (t). Region R(t & 1) holds S(t) and
// then dS(t)'s parts; R(~t & 1) holds dP(t). S(t+1) goes into dP(t)'s region
// once the math warps hold dP(t) in registers (dp_free), dP(t+1) into S(t)'s
// region right behind dQ(t), which reads dS(t) there (MMAs are performed in
// issue order).
__global__ void __launch_bounds__(kBThreads, 1)
attn_bwd_dq_x3_kernel(const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const X3Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(a.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  const uint32_t sbase = smem_u32(smem);
  DBars* bars = reinterpret_cast<DBars*>(smem + kDOffBar);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kDOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kDOffAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, a.status, kStatusTimeoutBwdQ};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < kDSlots; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->qd_full), kBMathWarps);
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->dp_full), 1);
    mbar_init(smem_u32(&bars->dp_free), kBMathWarps);
    mbar_init(smem_u32(&bars->ds_full), kBMathWarps);
    mbar_init(smem_u32(&bars->acc_full), 1);
    mbar_init(smem_u32(&bars->acc_empty), kBMathWarps);
    mbar_init(smem_u32(&bars->drain), 1);
    ring_init(&bars->ring, kBMathWarps + 1);
    fence_mbar_init();
  }
  if (warp == kBWarpMma) {
    tmem_alloc(smem_u32((const void*)tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = min(*a.n_items, a.max_items);

  if (warp == kBWarpTma) {
    if (lane == 0) {
      uint32_t item_count = 0, kv_load = 0, arm[kDSlots] = {};
      bool ok = true;
      while (ok) {
        int idx = atomicAdd(a.next_item, 1);
        if (idx >= n_items) idx = -1;
        ok = ring_push(&bars->ring, item_count, idx, wc);
        if (!ok || idx < 0) break;
        const DItem it = decode_d(a, idx);
        for (int j = 0; j < 4 * it.ntiles && ok; ++j, ++kv_load) {
          const int ks = it.kend - kDKeys * ((j >> 2) + 1);
          const uint32_t s = kv_load % kDSlots, ph = (kv_load / kDSlots) & 1;
          if (kv_load >= kDSlots) ok = mbar_wait(smem_u32(&bars->kv_empty[s]), ph ^ 1, wc);
          if (!ok) break;
          const uint32_t f = smem_u32(&bars->kv_full[s]);
          mbar_arrive_expect_tx(f, kPart64);
          ++arm[s];
          const CUtensorMap* m = (j & 2) ? &tm_v : &tm_k;
          const int y = (j & 1) ? a.Hk + it.g : it.g;
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sbase + kDOffKV + s * kPart64 + c * kChunk64, m, f, c * 64, y, ks);
        }
        ++item_count;
      }
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutBwdQ};
      for (int s = 0; s < kDSlots; ++s)
        if (arm[s]) mbar_wait(smem_u32(&bars->kv_full[s]), (arm[s] - 1) & 1, drain);
    }
  } else if (warp == kBWarpMma) {
    // Per tile t: S(t+1) (after dp_free(t)), dQ(t) (after ds_full(t)), then
    // dP(t+1) right behind dQ(t).
    const uint32_t leader = elect_one();
    const uint32_t idesc_s = make_idesc_f16(128, kDKeys, 0, 0);
    const uint32_t idesc_acc = make_idesc_f16(128, 128, 0, 1);
    uint32_t item_count = 0, t = 0, kv_base = 0, dpf_cnt = 0, ds_cnt = 0;
    bool ok = true;
    auto slot = [&](uint32_t pos) { return sbase + kDOffKV + (pos % kDSlots) * kPart64; };
    auto wait_full = [&](uint32_t pos) {
      return mbar_wait_warp(smem_u32(&bars->kv_full[pos % kDSlots]), (pos / kDSlots) & 1, wc);
    };
    auto region = [&](uint32_t r) { return tmem + kDColR + (r & 1) * 64; };
    // S(tt) = Q K(tt)^T into R(tt); tile n of the item (K parts at kv_base + 4n)
    auto issue_s = [&](uint32_t n, uint32_t tt) -> bool {
      const uint32_t pos = kv_base + 4 * n;
      if (!wait_full(pos) || !wait_full(pos + 1)) return false;
      tc_fence_after();
      const uint32_t kh = slot(pos), kl = slot(pos + 1), d = region(tt);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(d, tmem + kDColQH + kk * 8, kdesc64(kl, kk), idesc_s, kk > 0, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(d, tmem + kDColQL + kk * 8, kdesc64(kh, kk), idesc_s, 1u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(d, tmem + kDColQH + kk * 8, kdesc64(kh, kk), idesc_s, 1u, leader);
      mma_commit_w(smem_u32(&bars->s_full), leader);
      return true;
    };
    // dP(tt) = dO V(tt)^T into R(tt + 1); V parts at kv_base + 4n + 2, 3
    auto issue_dp = [&](uint32_t n, uint32_t tt) -> bool {
      const uint32_t pos = kv_base + 4 * n + 2;
      if (!wait_full(pos) || !wait_full(pos + 1)) return false;
      tc_fence_after();
      const uint32_t vh = slot(pos), vl = slot(pos + 1), d = region(tt + 1);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(d, tmem + kDColDOH + kk * 8, kdesc64(vl, kk), idesc_s, kk > 0, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(d, tmem + kDColDOL + kk * 8, kdesc64(vh, kk), idesc_s, 1u, leader);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts_w(d, tmem + kDColDOH + kk * 8, kdesc64(vh, kk), idesc_s, 1u, leader);
      mma_commit_w(smem_u32(&bars->dp_full), leader);
      mma_commit_w(smem_u32(&bars->kv_empty[pos % kDSlots]), leader);
      mma_commit_w(smem_u32(&bars->kv_empty[(pos + 1) % kDSlots]), leader);
      return true;
    };
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const DItem it = decode_d(a, idx);
      const uint32_t nt = (uint32_t)it.ntiles;
      // Q and dO of this item in TMEM (written after the previous item's MMAs
      // completed); R(t) held dP(t-1), which the math warps have read; R(t+1)
      // held dS(t-1), which dQ(t-1), issued before, reads.
      ok = mbar_wait_warp(smem_u32(&bars->qd_full), item_count & 1, wc);
      if (ok && t > 0) ok = mbar_wait_warp(smem_u32(&bars->dp_free), (dpf_cnt - 1) & 1, wc);
      if (ok) ok = issue_s(0, t);
      if (ok) ok = issue_dp(0, t);
      for (uint32_t n = 0; n < nt && ok; ++n) {
        const uint32_t tt = t + n;
        const bool has_next = n + 1 < nt;
        if (has_next) {
          ok = mbar_wait_warp(smem_u32(&bars->dp_free), dpf_cnt & 1, wc);
          if (ok) ok = issue_s(n + 1, tt + 1);
          if (!ok) break;
        }
        ++dpf_cnt;
        ok = mbar_wait_warp(smem_u32(&bars->ds_full), ds_cnt & 1, wc);
        ++ds_cnt;
        if (ok && n == 0 && item_count > 0)
          ok = mbar_wait_warp(smem_u32(&bars->acc_empty), (item_count - 1) & 1, wc);
        if (!ok) break;
        tc_fence_after();
        // dQ += dS(t) K(t): dS parts in R(t), K(t) parts MN-major
        const uint32_t pos = kv_base + 4 * n;
        const uint32_t kh = slot(pos), kl = slot(pos + 1), x = region(tt);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t ah = x + half_split_col(kk), al = ah + 16;
          mma_ts_w(tmem + kDColDQ, ah, mndesc64(kl, kk), idesc_acc,
                   (n > 0 || kk > 0) ? 1u : 0u, leader);
          mma_ts_w(tmem + kDColDQ, al, mndesc64(kh, kk), idesc_acc, 1u, leader);
          mma_ts_w(tmem + kDColDQ, ah, mndesc64(kh, kk), idesc_acc, 1u, leader);
        }
        mma_commit_w(smem_u32(&bars->kv_empty[pos % kDSlots]), leader);
        mma_commit_w(smem_u32(&bars->kv_empty[(pos + 1) % kDSlots]), leader);
        if (has_next) ok = issue_dp(n + 1, tt + 1);
      }
      if (!ok) break;
      mma_commit_w(smem_u32(&bars->acc_full), leader);
      kv_base += 4 * nt;
      t += nt;
      ++item_count;
    }
    mma_commit_w(smem_u32(&bars->drain), leader);
    volatile int no_abort = 0;
    const WaitCtx drain{&no_abort, a.status, kStatusTimeoutBwdQ};
    mbar_wait_warp(smem_u32(&bars->drain), 0, drain);
  } else {
    // ---------------------------------------------------------------- math warps
    const int wg = warp >> 2;                      // keys [32wg, 32wg+32) of a tile
    const int r = (warp & 3) * 32 + lane;          // query row of the tile = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int c0 = 32 * wg;
    // dQ carries the scales of dO's and v's parts
    const float dq_mul = a.scale * slot_scale(a.amax, true) * slot_scale(a.amax + 1, true);
    const uint64_t sc2 = f2(a.scale_log2, a.scale_log2);
    uint32_t item_count = 0, t = 0;
    bool ok = true;
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const DItem it = decode_d(a, idx);
      const int tok = it.q0 + (r >> a.logG);
      const int h = it.g * a.G + (r & (a.G - 1));
      const bool valid = tok < it.d1;
      {
        // Q's (warpgroup 0) or dO's (warpgroup 1) parts of this row into TMEM,
        // the A operands of S and dP. Every MMA of the previous item has
        // completed (acc_full, waited in its epilogue).
        const __half* base = wg ? a.dos : a.qs;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint4* src = reinterpret_cast<const uint4*>(
              base + ((size_t)tok * 2 * a.H + part * a.H + h) * kHeadDim);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint4 v4 = valid ? __ldg(src + hh * 8 + i) : make_uint4(0, 0, 0, 0);
              w[4 * i] = v4.x; w[4 * i + 1] = v4.y; w[4 * i + 2] = v4.z; w[4 * i + 3] = v4.w;
            }
            tmem_st32(t_row + kDColQH + wg * 128 + part * 64 + hh * 32, w);
          }
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->qd_full));
      }
      const int lo_r = a.W > 0 ? max(it.d0, tok - a.W + 1) : it.d0;
      const float lse2 = valid ? __ldg(a.lse + (size_t)h * a.T + tok) * kLog2e : 0.f;
      const float Di = valid ? __ldg(a.dvec + (size_t)h * a.T + tok) : 0.f;
      const uint64_t nl2 = f2(-lse2, -lse2);
      for (int n = 0; n < it.ntiles; ++n, ++t) {
        const uint32_t X = kDColR + (t & 1) * 64, Y = kDColR + ((t + 1) & 1) * 64;
        const int ks = it.kend - kDKeys * (n + 1);
        const bool needs_mask = (ks + kDKeys - 1 > it.q0) || (ks < it.d0) ||
                                (a.W > 0 && ks < it.q0 + a.R - a.W);
        const int c_lo = lo_r - ks, c_hi = tok - ks;
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full), t & 1, wc));
        if (!ok) break;
        tc_fence_after();
        float p[32];
        {
          uint32_t u[32];
          tmem_ld32(t_row + X + c0, u);
          tc_wait_ld_dep(u);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2_split(ffma2(f2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])), sc2,
                           nl2), x0, x1);
            float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            if (needs_mask) {
              const int c = c0 + 2 * e;
              p0 = (valid && c >= c_lo && c <= c_hi) ? p0 : 0.f;
              p1 = (valid && c + 1 >= c_lo && c + 1 <= c_hi) ? p1 : 0.f;
            }
            p[2 * e] = p0;
            p[2 * e + 1] = p1;
          }
        }
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->dp_full), t & 1, wc));
        if (!ok) break;
        tc_fence_after();
        {
          uint32_t u[32], dh16[16], dl16[16];
          tmem_ld32(t_row + Y + c0, u);
          tc_wait_ld_dep(u);
          // dP(t) is in registers: its region may take S(t+1)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->dp_free));
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float ds0 = p[2 * e] * (__uint_as_float(u[2 * e]) - Di);
            const float ds1 = p[2 * e + 1] * (__uint_as_float(u[2 * e + 1]) - Di);
            split_pair(ds0, ds1, dh16[e], dl16[e]);
          }
          tmem_st16(t_row + X + c0, dh16);       // dS hi, then lo, over S
          tmem_st16(t_row + X + c0 + 16, dl16);
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
        tmem_ld32(t_row + kDColDQ + 64 * wg, u0);
        tmem_ld32(t_row + kDColDQ + 64 * wg + 32, u1);
        tc_wait_ld_dep(u0);
        tc_wait_ld_dep(u1);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->acc_empty));
        if (valid) {
          float* row = a.dq_acc + ((size_t)tok * a.H + h) * kHeadDim + 64 * wg;
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
  if (warp == kBWarpMma) tmem_dealloc(tmem, 512);
}

}  // namespace

// ------------------------------------------------------------------ launchers
int x3_kv_box_tokens_fwd() { return kTileKeys; }
int x3_q_box_rows_dkv() { return kQRows; }
int x3_kv_box_tokens_dq() { return kDKeys; }

namespace {
X3Args make_args(const Resolved& p, const float* sink, const float* lse, const float* dvec,
                 const unsigned* amax, const __half* qs, const __half* dos, const __half* vs,
                 int* status) {
  X3Args a{};
  a.T = p.T; a.H = p.H; a.Hk = p.Hk; a.G = p.G; a.R = p.R; a.W = p.W;
  a.logG = 0;
  while ((1 << a.logG) < p.G) ++a.logG;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.sink = sink; a.lse = lse; a.dvec = dvec; a.amax = amax;
  a.qs = qs; a.dos = dos; a.vs = vs;
  a.status = status;
  return a;
}
}  // namespace

cudaError_t launch_attn_fwd_x3(const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const Resolved& p, const float* sink,
                               const int4* items, const int* n_items, int max_items,
                               const unsigned* amax, float* out, float* lse, int* status,
                               int num_sms, cudaStream_t st) {
  static PerDeviceOnce smem_once;
  cudaError_t e = smem_limit_once(smem_once, attn_fwd_x3_kernel, kFSmem);
  if (e != cudaSuccess) return e;
  X3Args a = make_args(p, sink, nullptr, nullptr, amax, nullptr, nullptr, nullptr, status);
  a.items = items; a.n_items = n_items; a.max_items = max_items;
  a.next_item = status + 4;
  a.out = out;
  a.lse_out = lse;
  int grid = num_sms < max_items ? num_sms : max_items;
  ProfScope prof(kKFwdX3, st);
  attn_fwd_x3_kernel<<<grid > 0 ? grid : 1, kFThreads, kFSmem, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_x3(const CUtensorMap& tq64, const CUtensorMap& tk128,
                               const CUtensorMap& tdo64, const CUtensorMap& tk64,
                               const CUtensorMap& tv64, const Resolved& p, const float* lse,
                               const float* dvec, const unsigned* amax, const __half* qs,
                               const __half* dos, const __half* vs, const int4* items_kv,
                               const int* n_kv, int max_kv, const int4* items_q, const int* n_q,
                               int max_q, float* dq_acc, float* dk_acc, float* dv, int* status,
                               int num_sms, cudaStream_t st) {
  static PerDeviceOnce smem_once_kv, smem_once_q;
  cudaError_t e = smem_limit_once(smem_once_kv, attn_bwd_dkv_x3_kernel, kKSmem);
  if (e != cudaSuccess) return e;
  e = smem_limit_once(smem_once_q, attn_bwd_dq_x3_kernel, kDSmem);
  if (e != cudaSuccess) return e;
  X3Args a = make_args(p, nullptr, lse, dvec, amax, qs, dos, vs, status);
  a.dq_acc = dq_acc; a.dk_acc = dk_acc; a.dv = dv;

  a.items = items_kv; a.n_items = n_kv; a.max_items = max_kv;
  a.next_item = status + 4;
  int grid = num_sms < max_kv ? num_sms : max_kv;
  {
    ProfScope prof(kKBwdDkvX3, st);
    attn_bwd_dkv_x3_kernel<<<grid > 0 ? grid : 1, kBThreads, kKSmem, st>>>(tq64, tk128, tdo64,
                                                                           a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  a.items = items_q; a.n_items = n_q; a.max_items = max_q;
  a.next_item = status + 5;
  grid = num_sms < max_q ? num_sms : max_q;
  ProfScope prof(kKBwdDqX3, st);
  attn_bwd_dq_x3_kernel<<<grid > 0 ? grid : 1, kBThreads, kDSmem, st>>>(tk64, tv64, a);
  return cudaGetLastError();
}

}  // namespace flint
