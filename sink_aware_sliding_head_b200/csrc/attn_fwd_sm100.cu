// attn_fwd_sm100.cu - sink-aware sliding/full GQA attention forward on
// Blackwell tensor cores (tcgen05 + TMEM + TMA): BF16 inputs, FP16 tensor-core
// operands (q_hat, k_hat from the prologue, an fp16 copy of v, P), FP32
// accumulation, output in bf16 or fp32.
//
// What it computes (Flint layers page, nemo_automodel.components.models.flint.
// layers, FlintAttention.forward: causal attention in which the sink is one
// more softmax category with a zero value vector; _FlintSinkParameters.forward:
// FP32 sink logits, not scaled; Flint config page: the window includes the
// current token):
//   O_i = sum_j e^{z_ij - LSE_i} v_j,  LSE_i = ln(e^{s_h} + sum_j e^{z_ij}),
//   over keys j of the same document with 0 <= i - j < W (W <= 0: unbounded).
//
// Design:
//   * A 128-row tile is R = 128/G tokens x the G query heads of one KV group,
//     so every K/V tile staged by TMA feeds all G heads of the group (GQA
//     sharing inside the CTA; no tile is broadcast across CTAs). A CTA works
//     on two such tiles at once ("tile 0" and "tile 1": 2R consecutive tokens)
//     that share every K/V tile, so each K/V byte brought on chip serves 256
//     query rows.
//   * Persistent grid (one CTA per SM) taking items from an LPT-sorted work
//     list built on the device through a global counter (greedy LPT: a CTA
//     asks for its next item when it is ready for it); only key tiles inside
//     the window and the document are visited, and only edge tiles are masked.
//   * Warp roles: warps 0-3 run the softmax of tile 0, warps 4-7 of tile 1
//     (thread = TMEM lane = query row), warp 8 issues TMA loads, warp 9 owns
//     the TMEM allocation and issues tcgen05.mma: the warp runs its loop
//     converged and one elected lane issues, so descriptors stay warp-uniform
//     (issued from a lane-0 branch instead, each MMA cost ~75 issue cycles).
//   * TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
//     P_i (fp16, two per column) overwrites the first 64 columns of S_i and is
//     the A operand of the PV MMA straight from TMEM. The softmax reads S_i
//     once into registers and releases P_i in two parts (keys 0-95, then
//     96-127); the PV MMAs of the first part run while the rest is
//     computed. The next QK MMA of tile i, which overwrites S_i, is issued
//     right behind the PV MMA that reads P_i from it: tcgen05.mma operations
//     issued by one thread are performed in issue order, so the PV has read
//     its operand before the QK writes (no completion wait on this chain; the
//     commit that signals the new S also covers the PV, so O and P_i are
//     settled when the softmax sees it).
//   * Sink folding: the running max starts at the sink logit and the running
//     sum at 1 (the sink's own weight), so there is no extra pass and a row is
//     never all -inf. The max is updated lazily: O and l are rescaled only when
//     the max grows by more than 2^8.
#include <type_traits>

#include "common.cuh"
#include "sm100_primitives.cuh"

namespace flint {

namespace {

// K and V tiles stream through one ring of kSlots 32 KB slots in the order
// K(0), V(0), K(1), V(1), ...; five slots let the producer run 2.5 key tiles
// ahead of the MMAs, which covers the load latency of a tile.
constexpr int kSlots = 5;
constexpr int kThreads = 320;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr uint32_t kChunkBytes = 128 * 64 * 2;     // 128 rows x 64 bf16 (one 128B-swizzle panel)
constexpr uint32_t kTileBytes = 2 * kChunkBytes;   // 128 rows x 128 bf16
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;          // log2 units

struct FwdArgs {
  int T, H, Hk, G, R, W;
  float scale_log2;
  const float* sink;
  const int4* items;
  const int* n_items;
  int max_items;
  int* next_item;   // zeroed before the launch: dynamic item counter
  const unsigned* amax_v;   // max |v| slot: the fp16 copy of v is v * 2^e
  void* out;        // bf16, float (out_f32) or fp16 (out_f16)
  int out_f32, out_f16;
  float* lse;
  int* status;
};

struct __align__(8) Barriers {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kSlots], kv_empty[kSlots];
  uint64_t s_full[2], p_half[2], p_full[2], o_full[2], o_empty[2];
  uint64_t drain;
  ItemRing ring;
};

// Dynamic shared memory: [Q0 | Q1 | K stages | V stages | barriers | tmem addr | abort flag]
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKV = 2 * kTileBytes;
constexpr uint32_t kOffBar = kOffKV + kSlots * kTileBytes;
constexpr uint32_t kOffTmem = kOffBar + sizeof(Barriers);
constexpr uint32_t kOffAbort = kOffTmem + 16;
constexpr uint32_t kSmemBytes = kOffAbort + 16 + 1024;   // + alignment slack
static_assert(kSmemBytes <= 227 * 1024, "exceeds the shared memory of one CTA");

struct Item {
  int q0, d0, d1, g, kend, kbeg, ntiles;
};

__device__ __forceinline__ Item decode(const FwdArgs& a, int idx) {
  const int4 it = a.items[idx];
  Item r;
  r.q0 = it.x; r.d0 = it.y; r.d1 = it.z; r.g = it.w;
  r.kend = min(r.q0 + 2 * a.R, r.d1);
  r.kbeg = a.W > 0 ? max(r.d0, r.q0 - a.W + 1) : r.d0;
  r.ntiles = (r.kend - r.kbeg + kTileKeys - 1) / kTileKeys;
  return r;
}

// K-major operand panel with 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart. kk selects the 16-element K slice (of 8) across two panels.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_base, int kk) {
  return make_sdesc(tile_base + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (V: keys x D with D contiguous), 128-byte swizzle: the two
// 64-column panels are kChunkBytes apart (LBO), 8-key groups 1024 bytes (SBO);
// kk selects keys [16kk, 16kk+16).
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_base, int kk) {
  return make_sdesc(tile_base + kk * 2048, kChunkBytes, 1024);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Barriers* bars = reinterpret_cast<Barriers*>(smem + kOffBar);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + kOffTmem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, a.status, kStatusTimeoutFwd};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->q_empty), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(smem_u32(&bars->kv_full[s]), 1);
      mbar_init(smem_u32(&bars->kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bars->s_full[i]), 1);
      mbar_init(smem_u32(&bars->p_half[i]), 4);
      mbar_init(smem_u32(&bars->p_full[i]), 4);
      mbar_init(smem_u32(&bars->o_full[i]), 1);
      mbar_init(smem_u32(&bars->o_empty[i]), 4);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    ring_init(&bars->ring, 9);   // the MMA warp and the 8 softmax warps consume
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32((const void*)tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = min(*a.n_items, a.max_items);

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kv_load = 0, item_count = 0, q_arm = 0, arm[kSlots] = {};
      bool ok = true;
      while (ok) {
        // greedy LPT over the heaviest-first list: the next item goes to the
        // CTA that asks first; -1 ends every role's loop
        int idx = atomicAdd(a.next_item, 1);
        if (idx >= n_items) idx = -1;
        ok = ring_push(&bars->ring, item_count, idx, wc);
        if (!ok || idx < 0) break;
        const Item it = decode(a, idx);
        if (item_count > 0) ok = mbar_wait(smem_u32(&bars->q_empty), (item_count - 1) & 1, wc);
        if (!ok) break;
        const uint32_t qf = smem_u32(&bars->q_full);
        mbar_arrive_expect_tx(qf, 2 * kTileBytes);
        ++q_arm;
        for (int i = 0; i < 2; ++i)
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sbase + kOffQ + i * kTileBytes + c * kChunkBytes, &tm_q, qf, c * 64,
                        it.g * a.G, it.q0 + i * a.R);
        for (int j = 0; j < 2 * it.ntiles && ok; ++j, ++kv_load) {
          const int ks = it.kend - kTileKeys * ((j >> 1) + 1);
          const uint32_t s = kv_load % kSlots, ph = (kv_load / kSlots) & 1;
          if (kv_load >= kSlots) ok = mbar_wait(smem_u32(&bars->kv_empty[s]), ph ^ 1, wc);
          if (!ok) break;
          const uint32_t f = smem_u32(&bars->kv_full[s]);
          mbar_arrive_expect_tx(f, kTileBytes);
          ++arm[s];
          const CUtensorMap* m = (j & 1) ? &tm_v : &tm_k;
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sbase + kOffKV + s * kTileBytes + c * kChunkBytes, m, f, c * 64, it.g, ks);
        }
        ++item_count;
      }
      // Every copy this thread started has landed before the CTA can exit
      // (immediate on the normal path: the consumer already saw each one).
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutFwd};
      if (q_arm) mbar_wait(smem_u32(&bars->q_full), (q_arm - 1) & 1, drain);
      for (int s = 0; s < kSlots; ++s)
        if (arm[s]) mbar_wait(smem_u32(&bars->kv_full[s]), (arm[s] - 1) & 1, drain);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order per key tile n: PV0(n), QK0(n+1), PV1(n), QK1(n+1). Tile 1
    // runs half a period behind tile 0, so each tile's softmax overlaps the
    // other tile's MMAs. QK_i(n+1) overwrites S_i, which holds P_i(n); it is
    // issued right behind PV_i(n), the MMAs being performed in issue order.
    {
      const uint32_t leader = elect_one();   // the one lane that issues
      const uint32_t idesc_qk = make_idesc_f16(128, 128, 0, 0);
      const uint32_t idesc_pv = make_idesc_f16(128, 128, 0, 1);
      uint32_t kv_load = 0, item_count = 0;   // K/V ring loads consumed before this item
      uint32_t pc0 = 0, pc1 = 0;                     // P arrivals seen, per tile
      bool ok = true;
      const uint32_t q0t = sbase + kOffQ, q1t = sbase + kOffQ + kTileBytes;
      while (ok) {
        int idx = -1;
        ok = ring_pop(&bars->ring, item_count, &idx, wc);
        if (!ok || idx < 0) break;
        const Item it = decode(a, idx);
        ok = mbar_wait_warp(smem_u32(&bars->q_full), item_count & 1, wc);
        if (!ok) break;
        tc_fence_after();
        {  // QK of the first key tile for both query tiles
          const uint32_t s = kv_load % kSlots, ph = (kv_load / kSlots) & 1;   // K(0)
          ok = mbar_wait_warp(smem_u32(&bars->kv_full[s]), ph, wc);
          if (!ok) break;
          const uint32_t kt = sbase + kOffKV + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_w(tmem + 0, kmajor_desc(q0t, kk), kmajor_desc(kt, kk), idesc_qk, kk > 0, leader);
          mma_commit_w(smem_u32(&bars->s_full[0]), leader);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_w(tmem + 128, kmajor_desc(q1t, kk), kmajor_desc(kt, kk),
                     idesc_qk, kk > 0, leader);
          mma_commit_w(smem_u32(&bars->s_full[1]), leader);
          mma_commit_w(smem_u32(&bars->kv_empty[s]), leader);
          if (it.ntiles == 1) mma_commit_w(smem_u32(&bars->q_empty), leader);
        }
        for (int n = 0; n < it.ntiles; ++n) {
          const uint32_t lv = kv_load + 2 * n + 1, lk = lv + 1;       // V(n), K(n+1)
          const uint32_t s = lv % kSlots, ph = (lv / kSlots) & 1;
          const uint32_t s2 = lk % kSlots, ph2 = (lk / kSlots) & 1;
          const bool has_next = n + 1 < it.ntiles;
          const uint32_t vt = sbase + kOffKV + s * kTileBytes;
          const uint32_t kt2 = sbase + kOffKV + s2 * kTileBytes;
          ok = mbar_wait_warp(smem_u32(&bars->kv_full[s]), ph, wc);
          // ---- tile 0
          // keys 0-95 of P as soon as the softmax has written them, then 96-127
          if (ok) ok = mbar_wait_warp(smem_u32(&bars->p_half[0]), pc0 & 1, wc);
          if (ok && n == 0 && item_count > 0)
            ok = mbar_wait_warp(smem_u32(&bars->o_empty[0]), (item_count - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 6; ++kk)
            mma_ts_w(tmem + 256, tmem + 0 + kk * 8, mnmajor_desc(vt, kk), idesc_pv,
                   (n > 0 || kk > 0) ? 1u : 0u, leader);
          ok = mbar_wait_warp(smem_u32(&bars->p_full[0]), pc0 & 1, wc);
          ++pc0;
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 6; kk < 8; ++kk)
            mma_ts_w(tmem + 256, tmem + 0 + kk * 8, mnmajor_desc(vt, kk), idesc_pv, 1u, leader);
          if (!has_next) mma_commit_w(smem_u32(&bars->o_full[0]), leader);
          if (has_next) {
            ok = mbar_wait_warp(smem_u32(&bars->kv_full[s2]), ph2, wc);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss_w(tmem + 0, kmajor_desc(q0t, kk), kmajor_desc(kt2, kk),
                       idesc_qk, kk > 0, leader);
            mma_commit_w(smem_u32(&bars->s_full[0]), leader);
          }
          // ---- tile 1
          // keys 0-95 of P as soon as the softmax has written them, then 96-127
          if (ok) ok = mbar_wait_warp(smem_u32(&bars->p_half[1]), pc1 & 1, wc);
          if (ok && n == 0 && item_count > 0)
            ok = mbar_wait_warp(smem_u32(&bars->o_empty[1]), (item_count - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 6; ++kk)
            mma_ts_w(tmem + 384, tmem + 128 + kk * 8, mnmajor_desc(vt, kk), idesc_pv,
                   (n > 0 || kk > 0) ? 1u : 0u, leader);
          ok = mbar_wait_warp(smem_u32(&bars->p_full[1]), pc1 & 1, wc);
          ++pc1;
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 6; kk < 8; ++kk)
            mma_ts_w(tmem + 384, tmem + 128 + kk * 8, mnmajor_desc(vt, kk), idesc_pv, 1u, leader);
          if (!has_next) mma_commit_w(smem_u32(&bars->o_full[1]), leader);
          mma_commit_w(smem_u32(&bars->kv_empty[s]), leader);
          if (has_next) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss_w(tmem + 128, kmajor_desc(q1t, kk), kmajor_desc(kt2, kk),
                       idesc_qk, kk > 0, leader);
            mma_commit_w(smem_u32(&bars->s_full[1]), leader);
            mma_commit_w(smem_u32(&bars->kv_empty[s2]), leader);
            if (n + 2 == it.ntiles) mma_commit_w(smem_u32(&bars->q_empty), leader);
          }
        }
        if (!ok) break;
        kv_load += 2 * it.ntiles;
        ++item_count;
      }
      // Every MMA this thread issued has finished before TMEM is released.
      mma_commit_w(smem_u32(&bars->drain), leader);
      volatile int no_abort = 0;
      const WaitCtx drain{&no_abort, a.status, kStatusTimeoutFwd};
      mbar_wait_warp(smem_u32(&bars->drain), 0, drain);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int i = warp >> 2;               // which query tile of the pair
    const int wq = warp & 3;               // TMEM lane quarter
    const int r = wq * 32 + lane;          // row of the tile = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t s_col = i * 128, o_col = 256 + i * 128;
    const float inv_sv = slot_scale(a.amax_v, true);
    uint32_t s_count = 0, item_count = 0;
    bool ok = true;
    while (ok) {
      int idx = -1;
      ok = ring_pop(&bars->ring, item_count, &idx, wc);
      if (!ok || idx < 0) break;
      const Item it = decode(a, idx);
      const int tok = it.q0 + i * a.R + r / a.G;
      const int h = it.g * a.G + r % a.G;
      const bool valid = tok < it.d1;
      const int lo_r = a.W > 0 ? max(it.d0, tok - a.W + 1) : it.d0;
      const float sink2 = __ldg(a.sink + h) * kLog2e;
      float m = sink2;                     // running max (log2 units)
      float l = 1.f;                       // running sum, sink included
      for (int n = 0; n < it.ntiles; ++n) {
        const int ks = it.kend - kTileKeys * (n + 1);
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->s_full[i]), s_count & 1, wc));
        ++s_count;
        if (!ok) break;
        tc_fence_after();
        const bool needs_mask = (ks + kTileKeys - 1 > it.q0) || (ks < it.d0) ||
                                (a.W > 0 && ks < it.q0 + 2 * a.R - a.W);
        const int c_lo = needs_mask ? lo_r - ks : 0;
        const int c_hi = needs_mask ? tok - ks : 127;
        // The whole row of S (128 columns) is loaded once. Masked and
        // unmasked key tiles run separate code; masked entries become -inf
        // in place, so the exponentials below need no mask.
        uint32_t u0[32], u1[32], u2[32], u3[32];
        tmem_ld32(t_row + s_col, u0);
        tmem_ld32(t_row + s_col + 32, u1);
        tmem_ld32(t_row + s_col + 64, u2);
        tmem_ld32(t_row + s_col + 96, u3);
        tc_wait_ld_dep(u0);
        tc_wait_ld_dep(u1);
        tc_wait_ld_dep(u2);
        tc_wait_ld_dep(u3);
        float mx0 = -INFINITY, mx1 = -INFINITY, mx2 = -INFINITY, mx3 = -INFINITY;
        auto row_max = [&](auto masked) {
          auto one = [&](uint32_t (&u)[32], int c0, float& mxa, float& mxb) {
            if (decltype(masked)::value) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c0 + e < c_lo || c0 + e > c_hi) u[e] = 0xff800000u;   // -inf
            }
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              mxa = fmax3(mxa, __uint_as_float(u[e]), __uint_as_float(u[e + 1]));
              mxb = fmax3(mxb, __uint_as_float(u[e + 2]), __uint_as_float(u[e + 3]));
            }
          };
          one(u0, 0, mx0, mx1);
          one(u1, 32, mx2, mx3);
          one(u2, 64, mx0, mx1);
          one(u3, 96, mx2, mx3);
        };
        if (needs_mask) row_max(std::true_type{});
        else row_max(std::false_type{});
        const float mx = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        const float m_tile = mx * a.scale_log2;
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
        const uint64_t nm2 = f2(-mb, -mb);
        uint64_t rs2 = f2(0.f, 0.f);
        // P = 2^(s*scale - m) in fp16, two keys per TMEM column, over the
        // first 64 columns of S (already read). Keys 0-95 are handed to the
        // PV MMAs before keys 96-127 are computed, so only two PV MMAs are left
        // on the tile's chain after the softmax.
        auto exp_chunk = [&](const uint32_t (&u)[32], int col) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2_split(ffma2(f2(__uint_as_float(u[2 * e]), __uint_as_float(u[2 * e + 1])), sc2, nm2),
                     x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            rs2 = fadd2(rs2, f2(p0, p1));
            pk[e] = pack_f16x2(p0, p1);
          }
          tmem_st16(t_row + s_col + col, pk);
        };
        exp_chunk(u0, 0);
        if (__any_sync(0xffffffffu, rescale_o)) {
          // PV of the previous tile has completed (the commit that signalled
          // this S was issued after it and covers it), so O is stable here.
          // Done once the first quarter of S is consumed, to stay within
          // registers.
          const uint64_t a2 = f2(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t u[32];
            tmem_ld32(t_row + o_col + c * 32, u);
            tc_wait_ld_dep(u);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float x0, x1;
              f2_split(fmul2(f2(__uint_as_float(u[e]), __uint_as_float(u[e + 1])), a2), x0, x1);
              u[e] = __float_as_uint(x0);
              u[e + 1] = __float_as_uint(x1);
            }
            tmem_st32(t_row + o_col + c * 32, u);
          }
        }
        exp_chunk(u1, 16);
        exp_chunk(u2, 32);
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_half[i]));
        exp_chunk(u3, 48);
        float rs_lo, rs_hi;
        f2_split(rs2, rs_lo, rs_hi);
        const float rs = rs_lo + rs_hi;
        l += rs;
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bars->p_full[i]));
      }
      if (!ok) break;
      // epilogue: O / l -> bf16, LSE
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars->o_full[i]), item_count & 1, wc));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = inv_sv / l;   // 1/l, and the scale of the fp16 copy of v
      const uint64_t il2 = f2(inv_l, inv_l);
      const size_t obase = ((size_t)tok * a.H + h) * kHeadDim;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        tmem_ld32(t_row + o_col + c * 32, u);
        tc_wait_ld_dep(u);
        if (c == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bars->o_empty[i]));
        }
        if (valid) {
          float o[32];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            f2_split(fmul2(f2(__uint_as_float(u[e]), __uint_as_float(u[e + 1])), il2), o[e],
                     o[e + 1]);
          if (a.out_f32) {
            float* orow = reinterpret_cast<float*>(a.out) + obase + c * 32;
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              *reinterpret_cast<float4*>(orow + 4 * v4) =
                  make_float4(o[4 * v4], o[4 * v4 + 1], o[4 * v4 + 2], o[4 * v4 + 3]);
          } else {
            // bf16, or IEEE fp16 for the fp16 compute boundary (both 2 bytes)
            uint16_t* orow = reinterpret_cast<uint16_t*>(a.out) + obase + c * 32;
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              uint4 pk;
              if (a.out_f16) {
                pk.x = pack_f16x2(o[v4 * 8 + 0], o[v4 * 8 + 1]);
                pk.y = pack_f16x2(o[v4 * 8 + 2], o[v4 * 8 + 3]);
                pk.z = pack_f16x2(o[v4 * 8 + 4], o[v4 * 8 + 5]);
                pk.w = pack_f16x2(o[v4 * 8 + 6], o[v4 * 8 + 7]);
              } else {
                pk.x = pack_bf16x2(o[v4 * 8 + 0], o[v4 * 8 + 1]);
                pk.y = pack_bf16x2(o[v4 * 8 + 2], o[v4 * 8 + 3]);
                pk.z = pack_bf16x2(o[v4 * 8 + 4], o[v4 * 8 + 5]);
                pk.w = pack_bf16x2(o[v4 * 8 + 6], o[v4 * 8 + 7]);
              }
              *reinterpret_cast<uint4*>(orow + v4 * 8) = pk;
            }
          }
        }
      }
      if (valid) a.lse[(size_t)h * a.T + tok] = (m + log2f(l)) * kLn2;
      ++item_count;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

}  // namespace

// Keys per K/V box of the forward's tensor maps (one key tile).
int fwd_kv_box_tokens() { return kTileKeys; }

cudaError_t launch_attn_fwd_sm100_impl(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, const Resolved& p, const float* sink,
                                       const int4* items, const int* n_items, int max_items,
                                       const unsigned* amax_v, void* out, float* lse,
                                       int* status, int num_sms, cudaStream_t st) {
  static PerDeviceOnce smem_once;
  cudaError_t e = smem_limit_once(smem_once, attn_fwd_sm100_kernel, kSmemBytes);
  if (e != cudaSuccess) return e;
  FwdArgs a;
  a.T = p.T; a.H = p.H; a.Hk = p.Hk; a.G = p.G; a.R = p.R; a.W = p.W;
  a.scale_log2 = p.scale * kLog2e;
  a.sink = sink; a.items = items; a.n_items = n_items; a.max_items = max_items;
  a.next_item = status + 4;
  a.amax_v = amax_v;
  a.out = out;
  a.out_f32 = p.fp32_out && !p.out_f16;
  a.out_f16 = p.out_f16;
  a.lse = lse;
  a.status = status;
  int grid = num_sms;
  if (grid > max_items) grid = max_items;
  if (grid < 1) grid = 1;
  ProfScope prof(kKFwdSm100, st);
  attn_fwd_sm100_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace flint
