// attn_win.cuh - GDLA attention forward for sliding windows of at most one
// K/V tile (0 < W <= 128), sm_100a.
//
// Operation ("Motif 3: Technical Report", paper.rainbus.top, step 2 "GDLA
// forward"), as in attn_fwd.cuh; the sliding-window layers of Motif 3 use
// W = 128 (same page and "Вышла новая модель Motif 3", pikabu.ru).
//
// A work item is (batch b, KV group k, query block q0 .. q0+127).  Query row
// r (token i = q0 + r) keeps the keys i-W+1 .. i, all inside two K/V tiles:
// the edge tile E = keys [q0-128, q0) and the diagonal tile G = keys
// [q0, q0+128).  On a shard of a sequence split across GPUs, the K/V tensors
// start kv_prefix (0 or 128) rows before the shard's first query (the halo
// of the previous shard), and query row i reads K/V row i + kv_prefix.
// Column c of a row's "union" row is key q0 + c when c <= r (from G) and key
// q0 - 128 + c when c > r (from E), so the 128 union
// columns of every row hold exactly its W <= 128 kept keys (plus masked
// ones when W < 128).  Per head:
//   S_E = Q K_E^T, S_G = Q K_G^T        two tcgen05.mma (A, B in smem)
//   union row max and P = exp2(S*c - m) one pass per head, one thread per row;
//                                       P_E = P where c > r, P_G where c <= r
//   O = P_E V_E + P_G V_G               two tcgen05.mma (A = P from TMEM)
// K_E, K_G, V_E, V_G stay in shared memory for the item's g+1 heads; query
// tiles stream through a two-deep ring.
//
// Softmax: two warpgroups share every row, each taking two of the four
// 32-column union chunks.  Warp quarter qw owns rows 32qw .. 32qw+31, so its
// chunk qw mixes both tiles and the other chunks each come whole from one
// tile (G left of it, E right of it).  A warp reads its two chunks in one
// TMEM round trip; the two halves of a row agree on the (integral) reference
// maximum through shared memory and an mbarrier per pair of warps, then each
// writes P for its columns in one pass, with no running-max rescale (a head
// is one tile).  Each half hands its partial row sum to the epilogue.
//
// Epilogue: the noise head's H_N = O / l stays in TMEM next to O.  For a
// signal head the epilogue combines O and H_N with lambda and the gate tile,
// which a dedicated TMA warp streams through a 128B-swizzled staging buffer
// (loaded as soon as the previous output tile's store has read the buffer),
// writes the output over the gate tile in place and releases O.
//
// Warp roles (512 threads, 128 registers each):
//   warps 0-3   softmax, union chunks 0-1 (TMEM lanes 0..127)
//   warps 4-7   softmax, union chunks 2-3
//   warps 8-11  epilogue
//   warp  12    TMA producer: query tiles, K/V
//   warp  13    TMEM allocator and MMA issuer
//   warp  14    TMA for the gate / output staging tile
//   warp  15    idle
// TMEM (512 columns): S_E [0,128) S_G [128,256) O [256,256+d) H_N [256+d,256+2d).
// P_E / P_G occupy the first 64 columns of S_E / S_G as packed bf16 pairs.
#pragma once

#include "attn_fwd.cuh"

namespace gdla {

constexpr int kWinThreads = 16 * 32;
constexpr int kWinEpiWarp0 = 8;
constexpr int kWinProducerWarp = 12;
constexpr int kWinMmaWarp = 13;
constexpr int kWinGateWarp = 14;
// Every role fits the 128 registers a thread of a 16-warp block gets (no
// register re-split).
constexpr uint32_t kNegInfBits = 0xff800000u;

template <int D>
struct WinSmemLayout {
  static constexpr uint32_t kTile = kBM * D * 2;  // one [128][D] bf16 tile
  static constexpr uint32_t kQOff = 0;             // query ring, 2 tiles
  static constexpr uint32_t kKOff = kQOff + 2 * kTile;  // K_E, K_G
  static constexpr uint32_t kVOff = kKOff + 2 * kTile;  // V_E, V_G
  static constexpr uint32_t kGOff = kVOff + 2 * kTile;  // gate / output staging
  static constexpr uint32_t kHalf = kBM * 128;          // one [128][64] swizzled half
  static constexpr uint32_t kStatOff = kGOff + kTile;   // float l[2 slot][2 half][kBM]
  static constexpr uint32_t kMxOff = kStatOff + 2 * 2 * kBM * 4;  // int16 [2 half][kBM]
  static constexpr uint32_t kBarOff = kMxOff + 2 * kBM * 2;
  static constexpr uint32_t kNumBars = 22;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
};

// One arrival per warp: every lane's earlier writes (ordered before this call
// by the lane's own fences) are made visible to the lane that arrives.
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31u) == 0) mbar_arrive(bar);
}

template <int D>
__global__ void __launch_bounds__(kWinThreads, 1)
    gdla_attn_win_kernel(const __grid_constant__ CUtensorMap tm_qs,
                         const __grid_constant__ CUtensorMap tm_qn,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_gate,
                         const __grid_constant__ CUtensorMap tm_out, const AttnParams p) {
  using L = WinSmemLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) write_status(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto q_full = [&](int s) { return bar0 + 8u * s; };
  auto q_empty = [&](int s) { return bar0 + 8u * (2 + s); };
  const uint32_t k_full = bar0 + 8u * 4;    // K_E, K_G of the item landed
  const uint32_t k_free = bar0 + 8u * 5;    // last S of the item done
  const uint32_t v_full = bar0 + 8u * 6;    // V_E, V_G landed
  const uint32_t v_free = bar0 + 8u * 7;    // last PV of the item done
  const uint32_t s_full = bar0 + 8u * 8;    // S_E, S_G of a head written
  const uint32_t p_full = bar0 + 8u * 9;    // P_E, P_G written (softmax warps)
  const uint32_t o_done = bar0 + 8u * 10;   // O of a head complete
  const uint32_t o_free = bar0 + 8u * 11;   // epilogue has read O (epilogue warps)
  const uint32_t g_full = bar0 + 8u * 12;   // gate tile landed
  const uint32_t g_done = bar0 + 8u * 13;   // output tile written (epilogue warps)
  // row sums handed over through two slots (softmax warps) / read (epilogue warps)
  auto epi_go = [&](uint32_t s) { return bar0 + 8u * (14 + s); };
  auto stat_free = [&](uint32_t s) { return bar0 + 8u * (16 + s); };
  // the two softmax halves of lane quarter wq meet here once per head
  auto mx_bar = [&](uint32_t wq) { return bar0 + 8u * (18 + wq); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  float *stat = reinterpret_cast<float *>(smem + L::kStatOff);  // [2 slot][2 half][kBM]
  int16_t *mxs = reinterpret_cast<int16_t *>(smem + L::kMxOff);   // [2 half][kBM]
  const int warp = threadIdx.x >> 5;
  const int n_heads = p.g + 1;  // noise head + g signal heads
  const int W = static_cast<int>(p.window);

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    mbar_init(k_full, 1);
    mbar_init(k_free, 1);
    mbar_init(v_full, 1);
    mbar_init(v_free, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);  // one arrival per softmax warp
    mbar_init(o_done, 1);
    mbar_init(o_free, 4);
    for (uint32_t s = 0; s < 2; ++s) {
      mbar_init(epi_go(s), 8);
      mbar_init(stat_free(s), 4);
    }
    mbar_init(g_full, 1);
    mbar_init(g_done, 4);
    for (uint32_t wq = 0; wq < 4; ++wq) mbar_init(mx_bar(wq), 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWinMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_se = tmem, t_sg = tmem + 128u, t_o = tmem + 256u, t_hn = tmem + 256u + D;
  auto p_col = [](int k) -> uint32_t { return 8u * k; };

  if (warp >= kWinProducerWarp) {
  // =============================== control warpgroup (warps 12-15)
  if (warp == kWinProducerWarp) {
    // =============================== TMA producer
    // Per item: K_E, K_G once the previous item's last S is done, the first
    // query tile, V_E, V_G once the previous item's last PV is done, then the
    // remaining query tiles through the two-deep ring.  The whole warp runs
    // the loop; one elected lane issues.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_qs);
      tma_prefetch_desc(&tm_qn);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    uint32_t hq = 0;       // query tiles loaded (ring position)
    uint32_t kv_uses = 0;  // items whose K/V were loaded
    uint32_t k_issued = 0, v_issued = 0;
    bool ok = true;
    auto load_tile = [&](uint32_t dst, const CUtensorMap *map, uint32_t bar, int col, int row,
                         int b) {
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_3d(dst + kb * L::kHalf, map, bar, col + kb * 64, row, b);
    };
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const bool has_edge = w.q0 + p.kv_prefix > 0;
      const int kv0 = w.q0 + p.kv_prefix;  // K/V row of query row q0
      const uint32_t n_kv = has_edge ? 2u : 1u;
      ok = __all_sync(0xffffffffu, mbar_wait(k_free, (kv_uses & 1u) ^ 1u, abort_flag));
      if (!ok) break;
      if (leader) {
        mbar_arrive_expect_tx(k_full, n_kv * L::kTile);
        if (has_edge) load_tile(sbase + L::kKOff, &tm_k, k_full, w.kvh * D, kv0 - kBN, w.b);
        load_tile(sbase + L::kKOff + L::kTile, &tm_k, k_full, w.kvh * D, kv0, w.b);
      }
      ++k_issued;
      for (int hh = 0; hh < n_heads && ok; ++hh) {
        const int buf = static_cast<int>(hq & 1u);
        ok = __all_sync(0xffffffffu, mbar_wait(q_empty(buf), ((hq >> 1) & 1u) ^ 1u, abort_flag));
        if (!ok) break;
        ++hq;
        const bool noise = hh == 0;
        const int head = noise ? w.kvh : p.g * w.kvh + (hh - 1);
        if (leader) {
          mbar_arrive_expect_tx(q_full(buf), L::kTile);
          load_tile(sbase + L::kQOff + buf * L::kTile, noise ? &tm_qn : &tm_qs, q_full(buf),
                    head * D, w.q0, w.b);
        }
        if (hh == 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(v_free, (kv_uses & 1u) ^ 1u, abort_flag));
          if (!ok) break;
          if (leader) {
            mbar_arrive_expect_tx(v_full, n_kv * L::kTile);
            if (has_edge) load_tile(sbase + L::kVOff, &tm_v, v_full, w.kvh * D, kv0 - kBN, w.b);
            load_tile(sbase + L::kVOff + L::kTile, &tm_v, v_full, w.kvh * D, kv0, w.b);
          }
          ++v_issued;
        }
      }
      ++kv_uses;
    }
    if (!ok && leader) {
      // unwinding: let the copies already issued land before the CTA exits
      if (k_issued) mbar_wait_for(k_full, (k_issued - 1) & 1u, 100000000ull);
      if (v_issued) mbar_wait_for(v_full, (v_issued - 1) & 1u, 100000000ull);
      for (uint32_t s = 0; s < 2; ++s) {
        const uint32_t issued = hq > s ? (hq - 1 - s) / 2 + 1 : 0;
        if (issued) mbar_wait_for(q_full(s), (issued - 1) & 1u, 100000000ull);
      }
    }
  } else if (warp == kWinMmaWarp) {
    // =============================== MMA issuer
    // Per head: S_E, S_G; after the softmax, PV_E, PV_G into O.  The next
    // head's S overwrites the columns this head's PV reads P from; both come
    // from this thread, and tcgen05.mma instructions of one thread execute in
    // issue order.  The first block of a sequence has no edge tile: its S_E
    // and PV_E are not issued.
    const bool leader = elect_one();
    constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, false, true);
    uint32_t hq = 0, kv_uses = 0, p_waits = 0, ofree_waits = 0, o_commits = 0;
    bool o_used = false;
    bool ok = true;
    auto issue_s = [&](uint32_t t_dst, uint32_t q_base, uint32_t k_base) {
      const uint64_t qd = sdesc_sw128(q_base, 16, 1024);
      const uint64_t kd = sdesc_sw128(k_base, 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t qoff = (k >> 2) * (kBM * 128) + (k & 3) * 32;
        const uint32_t koff = (k >> 2) * (kBN * 128) + (k & 3) * 32;
        umma_ss(t_dst, qd + (qoff >> 4), kd + (koff >> 4), kIdescS, k > 0 ? 1u : 0u);
      }
    };
    auto issue_pv = [&](uint32_t t_p, uint32_t v_base, bool first) {
      const uint64_t vd = sdesc_sw128(v_base, kBN * 128, 1024);
#pragma unroll
      for (int k = 0; k < kBN / 16; ++k)
        umma_ts(t_o, t_p + p_col(k), vd + ((k * (16 * 128)) >> 4), kIdescPV,
                (!first || k > 0) ? 1u : 0u);
    };
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const bool has_edge = w.q0 + p.kv_prefix > 0;
      ok = __all_sync(0xffffffffu, mbar_wait(k_full, kv_uses & 1u, abort_flag));
      if (!ok) break;
      for (int hh = 0; hh < n_heads && ok; ++hh) {
        const int buf = static_cast<int>(hq & 1u);
        ok = __all_sync(0xffffffffu, mbar_wait(q_full(buf), (hq >> 1) & 1u, abort_flag));
        ++hq;
        if (!ok) break;
        tc_fence_after();
        const uint32_t qb = sbase + L::kQOff + buf * L::kTile;
        if (leader) {
          if (has_edge) issue_s(t_se, qb, sbase + L::kKOff);
          issue_s(t_sg, qb, sbase + L::kKOff + L::kTile);
          umma_commit(s_full);
          umma_commit(q_empty(buf));
          if (hh == n_heads - 1) umma_commit(k_free);
        }
        ok = __all_sync(0xffffffffu, mbar_wait(p_full, p_waits & 1u, abort_flag));
        ++p_waits;
        if (ok && hh == 0) ok = __all_sync(0xffffffffu, mbar_wait(v_full, kv_uses & 1u, abort_flag));
        if (ok && o_used) {
          // the previous head's epilogue must have read O
          ok = __all_sync(0xffffffffu, mbar_wait(o_free, ofree_waits & 1u, abort_flag));
          ++ofree_waits;
        }
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          if (has_edge) issue_pv(t_se, sbase + L::kVOff, true);
          issue_pv(t_sg, sbase + L::kVOff + L::kTile, !has_edge);
          umma_commit(o_done);
          if (hh == n_heads - 1) umma_commit(v_free);
        }
        ++o_commits;
        o_used = true;
      }
      ++kv_uses;
    }
    // drain: every MMA issued above must finish before TMEM is released
    if (leader && o_commits) mbar_wait_for(o_done, (o_commits - 1) & 1u, 100000000ull);
  } else if (warp == kWinGateWarp) {
    // =============================== gate / output staging (TMA)
    // For every signal head in order: load its gate tile into the staging
    // buffer once the previous output tile's store has read it, wait until
    // the epilogue has overwritten the tile with the output, store it.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_gate);
      tma_prefetch_desc(&tm_out);
    }
    const uint32_t gbuf = sbase + L::kGOff;
    uint32_t g_issued = 0, g_stored = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      for (int hh = 1; hh < n_heads && ok; ++hh) {
        const int h = p.g * w.kvh + (hh - 1);
        if (leader) {
          if (g_stored) bulk_wait_group_read0();  // the previous store has read the buffer
          mbar_arrive_expect_tx(g_full, (D / 64) * L::kHalf);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_3d(gbuf + hf * L::kHalf, &tm_gate, g_full, h * D + hf * 64, w.q0, w.b);
        }
        ++g_issued;
        ok = __all_sync(0xffffffffu, mbar_wait(g_done, g_stored & 1u, abort_flag));
        if (!ok) break;
        if (leader) {
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_store_3d(&tm_out, gbuf + hf * L::kHalf, h * D + hf * 64, w.q0, w.b);
          bulk_commit_group();
        }
        ++g_stored;
      }
    }
    if (leader) {
      // a gate tile still in flight (after an abort) lands before the CTA
      // exits; every output tile store completes
      if (!ok && g_issued) mbar_wait_for(g_full, (g_issued - 1) & 1u, 100000000ull);
      bulk_wait_group0();
    }
  }
  } else if (warp < kWinEpiWarp0) {
    // =============================== softmax (warps 0-7, one thread per row)
    // Warpgroup `half` takes union chunks 2 half and 2 half + 1 of every row.
    // Warp quarter qw's own chunk qw mixes both tiles (G left of the
    // diagonal, E right of it); the other chunks come whole from one tile.
    // The two halves of a row agree on the integral reference maximum once
    // per head through shared memory and the pair's mbarrier.
    const int half = warp >> 2;
    const int qw = warp & 3;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(qw * 32) << 16;
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_make(sl2, sl2);
    const int dlo = r - W + 1;  // kept diagonal-tile columns: [dlo, r]
    const int ca = 2 * half, cb = 2 * half + 1;
    const bool has_mixed = qw == ca || qw == cb;
    const int other = qw == ca ? cb : ca;  // the whole chunk next to the mixed one
    uint32_t s_waits = 0, handoffs = 0;
    bool ok = true;
    const uint32_t zero16[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u,
                                 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const bool has_edge = w.q0 + p.kv_prefix > 0;
      // kept edge-tile columns: [elo, 127]
      const int elo = has_edge ? max(r + 1, r + 129 - W) : 128;
      // whole chunk cc (cc != qw): its tile and its lowest kept column
      auto whole_src = [&](int cc) { return (cc < qw ? t_sg : t_se) + lane_off + 32 * cc; };
      auto cut_whole = [&](uint32_t (&v)[32], int cc) {
        const int lo = cc < qw ? dlo : elo;
        const int c0 = 32 * cc;
        if (__any_sync(0xffffffffu, lo > c0)) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c0 + e < lo) v[e] = kNegInfBits;
        }
      };
      for (int hh = 0; hh < n_heads && ok; ++hh) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full, s_waits & 1u, abort_flag));
        const uint32_t par = s_waits & 1u;
        ++s_waits;
        if (!ok) break;
        tc_fence_after();
        // ---- this half's two chunks in one TMEM round trip: va holds the
        // first (the mixed chunk when the half has it), vb chunk kb
        uint32_t va[32], vb[32];
        const int kb = has_mixed ? other : cb;
        if (has_mixed) {
          uint32_t me[32];
          if (has_edge) {
            tmem_ld32x3_sync(t_sg + lane_off + 32 * qw, t_se + lane_off + 32 * qw,
                             whole_src(other), va, me, vb);
          } else {
            tmem_ld32x2_sync(t_sg + lane_off + 32 * qw, whole_src(other), va, vb);
#pragma unroll
            for (int e = 0; e < 32; ++e) me[e] = kNegInfBits;
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = 32 * qw + e;
            const bool diag = c <= r;
            const bool kept = diag ? c >= dlo : c >= elo;
            va[e] = kept ? (diag ? va[e] : me[e]) : kNegInfBits;
          }
        } else {
          tmem_ld32x2_sync(whole_src(ca), whole_src(cb), va, vb);
          cut_whole(va, ca);
        }
        cut_whole(vb, kb);
        // ---- this half's maximum, as the integral reference it implies
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          m0 = fmax3(m0, __uint_as_float(va[e]), __uint_as_float(va[e + 1]));
          m1 = fmax3(m1, __uint_as_float(vb[e]), __uint_as_float(vb[e + 1]));
        }
        const float mh = fmaxf(m0, m1) * sl2;
        // ceil is monotone, so the row's reference is the larger of the two
        // halves'; it travels as int16 (scaled logits beyond +-32767 saturate)
        const int mi = mh == -INFINITY ? -32768 : static_cast<int>(fminf(fmaxf(ceilf(mh), -32767.f), 32767.f));
        mxs[half * kBM + r] = static_cast<int16_t>(mi);
        warp_arrive(mx_bar(qw));
        ok = __all_sync(0xffffffffu, mbar_wait(mx_bar(qw), par, abort_flag));
        if (!ok) break;
        const int mref_i = max(static_cast<int>(mxs[r]), static_cast<int>(mxs[kBM + r]));
        // one tile per head: no running max, nothing to rescale; a row with
        // no kept key (padding rows) keeps reference 0
        const float m_ref = mref_i == -32768 ? 0.f : static_cast<float>(mref_i);
        const uint64_t negm2 = f2_make(-m_ref, -m_ref);
        uint64_t rs2 = f2_make(0.f, 0.f);
        // ---- P = exp2(S*c - m) as bf16 pairs; chunk cc lands in columns
        // [16cc, 16cc+16) of its tile's S (the other half has read its S:
        // it arrived at the pair's barrier above)
        if (has_mixed) {
          uint32_t pg[16], pe[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float t0v, t1v;
            f2_split(f2_fma(f2_from_bits(va[2 * e], va[2 * e + 1]), sl2x2, negm2), t0v, t1v);
            const float p0 = ex2_approx(t0v);
            const float p1 = ex2_approx(t1v);
            rs2 = f2_add(rs2, f2_make(p0, p1));
            const bool d0 = 32 * qw + 2 * e <= r, d1 = 32 * qw + 2 * e + 1 <= r;
            pg[e] = pack_bf16x2(d0 ? p0 : 0.f, d1 ? p1 : 0.f);
            pe[e] = pack_bf16x2(d0 ? 0.f : p0, d1 ? 0.f : p1);
          }
          tmem_st16(t_sg + lane_off + 16 * qw, pg);
          if (has_edge) tmem_st16(t_se + lane_off + 16 * qw, pe);
        }
        auto exp_whole = [&](const uint32_t (&v)[32], int cc) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float t0v, t1v;
            f2_split(f2_fma(f2_from_bits(v[2 * e], v[2 * e + 1]), sl2x2, negm2), t0v, t1v);
            const float p0 = ex2_approx(t0v);
            const float p1 = ex2_approx(t1v);
            rs2 = f2_add(rs2, f2_make(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          const uint32_t col = lane_off + 16 * cc;
          if (cc < qw) {
            tmem_st16(t_sg + col, pk);
            if (has_edge) tmem_st16(t_se + col, zero16);
          } else {
            tmem_st16(t_sg + col, zero16);
            if (has_edge) tmem_st16(t_se + col, pk);
          }
        };
        if (!has_mixed) exp_whole(va, ca);
        exp_whole(vb, kb);
        float rs0, rs1;
        f2_split(rs2, rs0, rs1);
        const float l = rs0 + rs1;
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(p_full);
        // hand this half's row sum to the epilogue through slot handoffs % 2,
        // once the epilogue has read what the slot held two heads ago
        const uint32_t slot = handoffs & 1u;
        if (handoffs >= 2) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(stat_free(slot), ((handoffs >> 1) - 1) & 1u, abort_flag));
          if (!ok) break;
        }
        ++handoffs;
        stat[(slot * 2 + half) * kBM + r] = l;
        warp_arrive(epi_go(slot));
      }
    }
  } else {
    // =============================== epilogue (warps 8-11)
    // Noise head: H_N = O / l into its TMEM columns.  Signal head:
    // D = O/l - lambda H_N into registers (O released at once), then
    // out = G (.) D over the row of the staged gate tile, in place.
    const int qw = warp & 3;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(qw * 32) << 16;
    const uint32_t gbuf = sbase + L::kGOff;
    uint32_t go_waits = 0, o_seen = 0, g_seen = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const int i = w.q0 + r;
      const bool row_ok = i < p.T;
      const int64_t row = static_cast<int64_t>(w.b) * p.T + i;
      for (int hh = 0; hh < n_heads && ok; ++hh) {
        const int h = p.g * w.kvh + (hh - 1);  // signal head (hh >= 1)
        // lambda of a signal head: loaded now, used after the waits
        const float lam = (hh != 0 && row_ok) ? __bfloat162float(p.lam[row * p.Hs + h]) : 0.f;
        const uint32_t slot = go_waits & 1u;
        bool okw = mbar_wait(epi_go(slot), (go_waits >> 1) & 1u, abort_flag);
        ++go_waits;
        if (okw) okw = mbar_wait(o_done, o_seen & 1u, abort_flag);
        ++o_seen;
        ok = __all_sync(0xffffffffu, okw);
        if (!ok) break;
        tc_fence_after();
        const float l = stat[(slot * 2 + 0) * kBM + r] + stat[(slot * 2 + 1) * kBM + r];
        warp_arrive(stat_free(slot));
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        if (hh == 0) {
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32_sync(t_o + lane_off + cc * 32, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * inv_l);
            tmem_st32(t_hn + lane_off + cc * 32, o);
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(o_free);
          continue;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(g_full, g_seen & 1u, abort_flag));
        ++g_seen;
        if (!ok) break;
        // out = G (.) (O/l - lambda H_N), 32 columns at a time, in place over
        // the staged gate tile: row r of a 128B-swizzled [128][64] half holds
        // 16-byte unit j at j ^ (r % 8)
        const uint32_t rbase = gbuf + static_cast<uint32_t>(r) * 128u;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32], hn[32];
          tmem_ld32x2_sync(t_o + lane_off + cc * 32, t_hn + lane_off + cc * 32, o, hn);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int j = (cc & 1) * 4 + q;
            const uint32_t addr = rbase + static_cast<uint32_t>(cc >> 1) * L::kHalf +
                                  (static_cast<uint32_t>(j ^ (r & 7)) << 4);
            const uint4 gv = lds128(addr);
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int k0 = q * 8 + 2 * e;
              const float d0 = __uint_as_float(o[k0]) * inv_l - lam * __uint_as_float(hn[k0]);
              const float d1 =
                  __uint_as_float(o[k0 + 1]) * inv_l - lam * __uint_as_float(hn[k0 + 1]);
              ow[e] = pack_bf16x2(bf16lo_to_f32(gw[e]) * d0, bf16hi_to_f32(gw[e]) * d1);
            }
            sts128(addr, make_uint4(ow[0], ow[1], ow[2], ow[3]));
          }
        }
        // every column of O has been read: the next head's PV may start
        tc_fence_before();
        warp_arrive(o_free);
        // every row written (generic proxy) before the TMA store reads the tile
        fence_proxy_async_smem();
        warp_arrive(g_done);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) write_status(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == kWinMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gdla
