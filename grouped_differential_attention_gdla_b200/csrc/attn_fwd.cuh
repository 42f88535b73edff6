// attn_fwd.cuh - fused GDLA attention forward for sm_100a.
//
// Operation ("Motif 3: Technical Report", paper.rainbus.top, step 2 "GDLA
// forward"): for KV group k the noise head n = k and the g signal heads
// h = g*k .. g*k+g-1 attend over the shared KV head k;
//   D[h] = H_S[h] - lambda[h] * H_N[h / g],   O[h] = G[h] * D[h].
//
// A work item is one (batch b, KV group k, block of 128 query tokens); a CTA
// runs the group's g+1 heads (noise first) in phases of two "slots" A and B.
// In a normal phase the slots hold two heads over the same query rows, so
// every K/V tile the TMA warp stages in shared memory serves both.  When the
// head count is odd the last head runs as a split phase: both slots take the
// same head, slot A the even and slot B the odd K/V tiles, and the two partial
// softmax states (m, l, O) are merged in the epilogue.  Per K/V tile:
//   S_X  = Q_X K^T          tcgen05.mma, A = Q (smem), B = K (smem), D = TMEM
//   P_X  = exp2(S_X*c - m)  softmax warpgroup X (one thread per row):
//                           tcgen05.ld, row max, bf16 P written over S_X
//   O_X += P_X V            tcgen05.mma, A = P (TMEM), B = V (smem)
// The running max m is kept integral (log2 units), so P's bf16 rounding does
// not depend on which tiles a slot has seen and the split merge is exact.
// The noise head's normalised output H_N stays in shared memory (fp32) and is
// subtracted in the epilogue of every signal head of the group; neither H_S
// nor H_N reaches global memory.  Full attention launches one CTA per item;
// sliding-window items are walked by one persistent CTA per SM.
//
// Warp roles (512 threads, registers re-split with setmaxnreg; full
// attention / sliding windows wider than one tile):
//   warps  0-3   softmax for slot A (TMEM lanes 0..127)        168 / 144 regs
//   warps  4-7   softmax for slot B                             168 / 144 regs
//   warps  8-11  epilogue for both slots: O / l, H_N, gate, output 88 / 112 regs
//   warp  12     TMA producer (Q tiles, K/V ring)               }  88 / 112 regs
//   warp  13     TMEM allocator, MMA issuer for slot A          }
//   warp  14     MMA issuer for slot B                          }
//   warp  15     idle (completes the fourth warpgroup)          }
// A softmax warpgroup hands each finished head to the epilogue warpgroup
// (row sums and maxima through shared memory) and goes straight on to the
// next phase; the next PV into the same O columns waits for the epilogue.
//
// TMEM (512 columns): S_A [0,128) S_B [128,256) O_A [256,256+d) O_B [256+d,256+2d).
// P_X occupies the first 64 columns of S_X as packed bf16 pairs.
#pragma once

#include "sm100.cuh"

namespace gdla {

constexpr int kBM = 128;      // query rows per slot
constexpr int kBN = 128;      // keys per K/V tile
constexpr int kKvStages = 3;  // K/V ring depth (tiles)
constexpr int kProducerWarp = 12;
constexpr int kMmaWarp = 13;
constexpr int kAttnThreads = 16 * 32;
// Register split.  The block launches with kLaunchRegs per thread (the
// compiler's cap for 16 warps, four per SM sub-partition); the control and
// epilogue warpgroups give registers back and the softmax warpgroups take
// them, within the launch pool.  The host refuses to launch a build whose
// per-thread register count differs from kLaunchRegs.
// Full attention's softmax reads a whole score row (128 registers) per
// tile; the sliding-window instantiation reads chunk by chunk and its
// epilogue stages tiles through shared memory, so it moves registers from
// the softmax to the epilogue and the control warps.
constexpr uint32_t kLaunchRegs = 128;
template <bool kWin>
struct RegSplit {
  static constexpr uint32_t kSoftmax = kWin ? 144 : 168;
  static constexpr uint32_t kEpilogue = kWin ? 112 : 88;
  static constexpr uint32_t kControl = kWin ? 112 : 88;
  static_assert(2 * 128 * kSoftmax + 128 * kEpilogue + 128 * kControl <=
                    kAttnThreads * kLaunchRegs,
                "register split must fit in the launch pool");
};
constexpr int kSlotThreads = 128;          // one warpgroup per slot
constexpr float kRescaleThreshold = 8.0f;  // log2 units: O is rescaled only if the max grows by > 2^8

struct AttnParams {
  const __nv_bfloat16 *lam;   // [B, T, Hs]
  const __nv_bfloat16 *gate;  // [B, T, Hs*d]
  __nv_bfloat16 *out;         // [B, T, Hs*d]
  int *status;                // optional device status word
  int B;
  int T;
  int Hs;
  int Hn;
  int g;
  int n_qblk;
  int n_items;     // B * Hn * n_qblk work items; CTA c runs c, c + grid, ...
  int band;        // full attention: KV groups ordered heaviest-first together
  int kv_prefix;   // K/V rows before query row 0 (sequence-parallel halo; 0 or 128)
  int64_t window;  // 0 = full
  int causal;
  float scale_log2;  // softmax scale * log2(e)
};

template <int D>
struct AttnSmemLayout {
  static constexpr uint32_t kQBytes = kBM * D * 2;
  static constexpr uint32_t kKvBytes = kBN * D * 2;
  static constexpr uint32_t kHnBytes = kBM * D * 4;  // H_N fp32
  // Sliding window: the ring keeps two stages and the third holds the
  // epilogue's gate/output tile, [D/64] 128B-swizzled halves of [kBM][64].
  static constexpr uint32_t kStageHalf = kBM * 128;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKvOff = kQOff + 2 * kQBytes;
  static constexpr uint32_t kHnOff = kKvOff + kKvStages * kKvBytes;
  static constexpr uint32_t kStatOff = kHnOff + kHnBytes;  // float stat[slot][l, m][row]
  static constexpr uint32_t kStatBytes = 2 * 2 * kBM * 4;
  static constexpr uint32_t kBarOff = kStatOff + kStatBytes;
  // q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_done[2]
  // o_free[2] epi_go[2] stat_free[2] g_full g_done
  static constexpr uint32_t kNumBars = 2 + 2 + 2 * kKvStages + 2 + 2 + 2 + 2 + 2 + 2 + 2;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
};

// Which heads the two slots run in phase `ph` (head index 0 = noise,
// i >= 1 = signal head i-1 of the group).
struct PhasePlan {
  int nslot;   // active slots
  bool split;  // both slots run head0 on alternating K/V tiles
  int head0, head1;
};

__device__ __forceinline__ PhasePlan phase_plan(int ph, int n_heads, int n_tiles) {
  PhasePlan pl;
  const int first = 2 * ph;
  if (first + 1 < n_heads) {
    pl.nslot = 2;
    pl.split = false;
    pl.head0 = first;
    pl.head1 = first + 1;
  } else if (n_tiles >= 2) {
    pl.nslot = 2;
    pl.split = true;
    pl.head0 = first;
    pl.head1 = first;
  } else {
    pl.nslot = 1;
    pl.split = false;
    pl.head0 = first;
    pl.head1 = -1;
  }
  return pl;
}

// How a 32-column chunk of a masked score tile (a sliding-window edge or the
// causal diagonal) looks to the 32 rows of one warp, warp-uniformly: every
// column kept, none kept, or mixed.  Per warp at most one chunk is mixed, so
// only it pays for per-column tests, and chunks no row keeps cost neither
// TMEM loads nor exponentials.
constexpr int kChunkFull = 0, kChunkEmpty = 1, kChunkMixed = 2;
__device__ __forceinline__ int chunk_class(int cc, int c_lo, int c_hi) {
  const int col0 = cc * 32, col1 = col0 + 31;
  if (__all_sync(0xffffffffu, c_lo <= col0 && col1 <= c_hi)) return kChunkFull;
  if (__all_sync(0xffffffffu, col1 < c_lo || col0 > c_hi)) return kChunkEmpty;
  return kChunkMixed;
}

// One work item: a KV group of one batch over a block of kBM query tokens,
// and the K/V tiles its causal (or sliding-window) mask can reach.
struct WorkItem {
  int b, kvh, q0, j_lo, n_tiles;
};

// Heaviest query blocks first.  Full attention: the KV groups are taken in
// bands of p.band groups, and within a band the query blocks run heaviest
// first across the band's groups: CTAs running at the same time stream the
// K/V tiles of a few groups, which stay in L2, while the light blocks of
// every band come last and fill the tail.  Sliding window: all groups of a
// query block together, so the block's query/gate/output rows are read and
// written as whole token rows.
__device__ __forceinline__ WorkItem work_item(const AttnParams &p, int item) {
  int grp, qblk;
  if (p.window == 0) {
    const int groups = p.B * p.Hn;
    const int per_band = p.band * p.n_qblk;
    const int bi = item / per_band;
    const int g0 = bi * p.band;
    const int gb = min(p.band, groups - g0);  // groups in this band
    const int rr = item - bi * per_band;
    grp = g0 + rr % gb;
    qblk = p.n_qblk - 1 - rr / gb;
  } else {
    const int groups = p.B * p.Hn;
    grp = item % groups;
    qblk = p.n_qblk - 1 - item / groups;
  }
  WorkItem w;
  w.b = grp / p.Hn;
  w.kvh = grp % p.Hn;
  w.q0 = qblk * kBM;
  int j_lo, j_hi;
  if (p.causal) {
    const int last = min(w.q0 + kBM - 1, p.T - 1);
    j_hi = last / kBN;
    j_lo = 0;
    if (p.window > 0) {
      const int64_t first = static_cast<int64_t>(w.q0) - p.window + 1;
      j_lo = first > 0 ? static_cast<int>(first / kBN) : 0;
    }
  } else {
    j_lo = 0;
    j_hi = (p.T - 1) / kBN;
  }
  w.j_lo = j_lo;
  w.n_tiles = j_hi - j_lo + 1;
  return w;
}

__device__ __forceinline__ void write_status(int *status, int code) {
  if (status) atomicExch(status, code);
}

// kWin: sliding-window instantiation (p.window > 0); otherwise full
// attention (causal or not).
template <int D, bool kWin>
__global__ void __launch_bounds__(kAttnThreads, 1)
    gdla_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_qs,
                         const __grid_constant__ CUtensorMap tm_qn,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_gate,
                         const __grid_constant__ CUtensorMap tm_out, const AttnParams p) {
  using L = AttnSmemLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  // swizzled TMA/UMMA tiles need a 1024-byte aligned base; refuse to run otherwise
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) write_status(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto q_full = [&](int x) { return bar0 + 8u * (0 + x); };
  auto q_empty = [&](int x) { return bar0 + 8u * (2 + x); };
  auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (4 + kKvStages + s); };
  auto s_full = [&](int x) { return bar0 + 8u * (4 + 2 * kKvStages + x); };
  auto p_full = [&](int x) { return bar0 + 8u * (6 + 2 * kKvStages + x); };
  auto o_done = [&](int x) { return bar0 + 8u * (8 + 2 * kKvStages + x); };
  auto o_free = [&](int x) { return bar0 + 8u * (10 + 2 * kKvStages + x); };
  auto epi_go = [&](int x) { return bar0 + 8u * (12 + 2 * kKvStages + x); };
  auto stat_free = [&](int x) { return bar0 + 8u * (14 + 2 * kKvStages + x); };
  const uint32_t g_full = bar0 + 8u * (16 + 2 * kKvStages);  // staged gate tile landed
  const uint32_t g_done = bar0 + 8u * (17 + 2 * kKvStages);  // staged output tile written
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  float *hn_smem = reinterpret_cast<float *>(smem + L::kHnOff);  // [D][kBM]
  float *stat = reinterpret_cast<float *>(smem + L::kStatOff);   // [2][2][kBM]

  const int warp = threadIdx.x >> 5;

  // K/V ring depth: two stages in sliding-window mode, whose third stage is
  // the epilogue's staging tile
  constexpr uint32_t n_stages = kWin ? 2u : static_cast<uint32_t>(kKvStages);
  const int n_heads = p.g + 1;  // noise head + g signal heads
  const int n_phases = (n_heads + 1) / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
      mbar_init(s_full(s), 1);
      mbar_init(p_full(s), kSlotThreads);
      mbar_init(o_done(s), 1);
      mbar_init(o_free(s), kSlotThreads);
    }
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(kv_full(s), 1);
      // released once per entry by the lockstep issuer, or by both per-slot issuers
      mbar_init(kv_empty(s), kWin ? 2 : 1);
    }
    mbar_init(epi_go(0), kSlotThreads);
    mbar_init(epi_go(1), kSlotThreads);
    mbar_init(stat_free(0), kSlotThreads);
    mbar_init(stat_free(1), kSlotThreads);
    mbar_init(g_full, 1);
    mbar_init(g_done, kSlotThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto t_s = [&](int x) { return tmem + 128u * static_cast<uint32_t>(x); };
  auto t_o = [&](int x) { return tmem + 256u + static_cast<uint32_t>(D * x); };
  // TMEM column (relative to S_X) of the packed P for keys 16k .. 16k+15
  auto p_col = [](int k) -> uint32_t { return 8u * k; };

  if (warp >= 12) {
  // =============================== control warpgroup (warps 12-15)
  regs_decrease<RegSplit<kWin>::kControl>();
  if (warp == kProducerWarp) {
    // =============================== TMA producer
    // The whole warp runs the loop (warp-uniform control and addresses); one
    // elected lane issues the copies.  Ring order per phase: K_0 .. K_{A-1},
    // then V_t, K_{t+A} for t = 0..n-1, where A = 1 (normal phase) or 2
    // (split phase) is how far ahead of the values the slots need keys.
    // Work items follow one another without a break: the next item's query
    // tiles and keys load while the current one finishes.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_qs);
      tma_prefetch_desc(&tm_qn);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    uint32_t q_uses[2] = {0, 0};
    uint32_t c = 0;  // K/V ring position
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      auto load_kv = [&](int t, bool is_v) {
        const int s = static_cast<int>(c % n_stages);
        ok = __all_sync(0xffffffffu,
                        mbar_wait(kv_empty(s), ((c / n_stages) & 1u) ^ 1u, abort_flag));
        if (!ok) return;
        const uint32_t dst = sbase + L::kKvOff + s * L::kKvBytes;
        if (leader) {
          mbar_arrive_expect_tx(kv_full(s), L::kKvBytes);
          const CUtensorMap *map = is_v ? &tm_v : &tm_k;
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(dst + kb * (kBN * 128), map, kv_full(s), w.kvh * D + kb * 64,
                        (w.j_lo + t) * kBN, w.b);
        }
        ++c;
      };
      for (int ph = 0; ph < n_phases && ok; ++ph) {
        const PhasePlan pl = phase_plan(ph, n_heads, w.n_tiles);
        // a split head's query tile goes to both slots' buffers
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (x >= pl.nslot || !ok) break;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(q_empty(x), (q_uses[x] & 1u) ^ 1u, abort_flag));
          if (!ok) break;
          ++q_uses[x];
          const int hi = x == 0 ? pl.head0 : pl.head1;
          const uint32_t dst = sbase + L::kQOff + x * L::kQBytes;
          const bool noise = hi == 0;
          const int head = noise ? w.kvh : p.g * w.kvh + (hi - 1);
          if (leader) {
            mbar_arrive_expect_tx(q_full(x), L::kQBytes);
            const CUtensorMap *map = noise ? &tm_qn : &tm_qs;
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(dst + kb * (kBM * 128), map, q_full(x), head * D + kb * 64, w.q0, w.b);
          }
        }
        const int ahead = pl.split ? 2 : 1;
        for (int t = 0; t < ahead && t < w.n_tiles && ok; ++t) load_kv(t, false);
        for (int t = 0; t < w.n_tiles && ok; ++t) {
          load_kv(t, true);
          if (ok && t + ahead < w.n_tiles) load_kv(t + ahead, false);
        }
      }
    }
    if (!ok && leader) {
      // unwinding: let the copies already issued land before the CTA exits
      for (uint32_t s = 0; s < n_stages; ++s) {
        const uint32_t issued = c > s ? (c - 1 - s) / n_stages + 1 : 0;
        if (issued) mbar_wait_for(kv_full(s), (issued - 1) & 1u, 100000000ull);
      }
      for (int x = 0; x < 2; ++x)
        if (q_uses[x]) mbar_wait_for(q_full(x), (q_uses[x] - 1) & 1u, 100000000ull);
    }
  } else if (!kWin && warp == kMmaWarp) {
    // =============================== MMA issuer for both slots, in lockstep
    // (full attention).  Per slot X the issue order is S_X(t) .. PV_X(t),
    // S_X(t+A), and slot A's pair goes first: slot B's MMAs run while slot
    // A's softmax works and the other way round, and the fixed order keeps
    // the two softmaxes half a tile apart instead of contending.  S_X(t+A)
    // overwrites the TMEM columns PV_X(t) reads P from; tcgen05.mma
    // instructions of one thread execute in issue order, so the read of P
    // precedes the overwrite.  The whole warp runs the loop so descriptors
    // stay warp-uniform; one elected lane issues.
    const bool leader = elect_one();
    constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, false, true);
    uint32_t q_uses[2] = {0, 0};
    uint32_t p_waits[2] = {0, 0};
    uint32_t ofree_waits[2] = {0, 0};
    uint32_t o_commits[2] = {0, 0};
    bool o_used[2] = {false, false};
    uint32_t c = 0;  // ring position of the next K/V entry
    bool ok = true;
    auto issue_s = [&](int x, uint32_t k_base) {
      const uint64_t qd = sdesc_sw128(sbase + L::kQOff + x * L::kQBytes, 16, 1024);
      const uint64_t kd = sdesc_sw128(k_base, 16, 1024);
      if (leader) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t qoff = (k >> 2) * (kBM * 128) + (k & 3) * 32;
          const uint32_t koff = (k >> 2) * (kBN * 128) + (k & 3) * 32;
          umma_ss(t_s(x), qd + (qoff >> 4), kd + (koff >> 4), kIdescS, k > 0 ? 1u : 0u);
        }
        umma_commit(s_full(x));
      }
    };
    // waits for the next ring entry; returns its stage and smem address
    auto next_stage = [&](uint32_t &base) -> int {
      const int s = static_cast<int>(c % n_stages);
      ok = __all_sync(0xffffffffu, mbar_wait(kv_full(s), (c / n_stages) & 1u, abort_flag));
      tc_fence_after();
      base = sbase + L::kKvOff + s * L::kKvBytes;
      ++c;
      return s;
    };
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const int n = w.n_tiles;
      for (int ph = 0; ph < n_phases && ok; ++ph) {
        const PhasePlan pl = phase_plan(ph, n_heads, n);
        // last tile of slot x in this phase: its last use of Q_X
        auto last_tile = [&](int x) { return pl.split ? x + 2 * ((n - 1 - x) / 2) : n - 1; };
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (x < pl.nslot && ok) {
            ok = __all_sync(0xffffffffu, mbar_wait(q_full(x), q_uses[x] & 1u, abort_flag));
            ++q_uses[x];
          }
        }
        if (!ok) break;
        const int ahead = pl.split ? 2 : 1;
        // prologue: the first S of every slot
        if (!pl.split) {
          uint32_t kb;
          const int s = next_stage(kb);
          if (!ok) break;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (x < pl.nslot) {
              issue_s(x, kb);
              if (n == 1 && leader) umma_commit(q_empty(x));
            }
          }
          if (leader) umma_commit(kv_empty(s));
        } else {
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            uint32_t kb;
            const int s = next_stage(kb);
            if (!ok) break;
            issue_s(x, kb);
            if (leader) {
              if (last_tile(x) == x) umma_commit(q_empty(x));
              umma_commit(kv_empty(s));
            }
          }
          if (!ok) break;
        }
        for (int t = 0; t < n && ok; ++t) {
          uint32_t vb;
          const int sv = next_stage(vb);
          if (!ok) break;
          const uint64_t vd = sdesc_sw128(vb, kBN * 128, 1024);
          int sk = -1;
          uint32_t kb = 0;
#pragma unroll
          for (int xx = 0; xx < 2; ++xx) {
            if (pl.split && xx == 1) break;
            const int x = pl.split ? (t & 1) : xx;
            if (x >= pl.nslot || !ok) break;
            const uint32_t pw = x == 0 ? p_waits[0] : p_waits[1];
            ok = __all_sync(0xffffffffu, mbar_wait(p_full(x), pw & 1u, abort_flag));
            if (!ok) break;
            if (x == 0) ++p_waits[0]; else ++p_waits[1];
            const bool first_pv = pl.split ? (t == x) : (t == 0);
            if (first_pv && (x == 0 ? o_used[0] : o_used[1])) {
              // the previous head's epilogue must have read O_X
              const uint32_t fw = x == 0 ? ofree_waits[0] : ofree_waits[1];
              ok = __all_sync(0xffffffffu, mbar_wait(o_free(x), fw & 1u, abort_flag));
              if (!ok) break;
              if (x == 0) ++ofree_waits[0]; else ++ofree_waits[1];
            }
            tc_fence_after();
            if (leader) {
#pragma unroll
              for (int k = 0; k < kBN / 16; ++k)
                umma_ts(t_o(x), t_s(x) + p_col(k), vd + ((k * (16 * 128)) >> 4), kIdescPV,
                        (!first_pv || k > 0) ? 1u : 0u);
              umma_commit(o_done(x));
            }
            if (x == 0) ++o_commits[0]; else ++o_commits[1];
            const int tn = t + ahead;
            if (tn < n) {
              if (sk < 0) {
                sk = next_stage(kb);
                if (!ok) break;
              }
              issue_s(x, kb);
              if (tn == last_tile(x) && leader) umma_commit(q_empty(x));
            }
          }
          if (!ok) break;
          if (leader) {
            umma_commit(kv_empty(sv));
            if (sk >= 0) umma_commit(kv_empty(sk));
          }
        }
        o_used[0] = true;
        if (pl.nslot == 2) o_used[1] = true;
      }
    }
    // drain: every MMA issued above must finish before TMEM is released
    if (leader) {
      if (o_commits[0]) mbar_wait_for(o_done(0), (o_commits[0] - 1) & 1u, 100000000ull);
      if (o_commits[1]) mbar_wait_for(o_done(1), (o_commits[1] - 1) & 1u, 100000000ull);
    }
  } else if (kWin && (warp == kMmaWarp || warp == kMmaWarp + 1)) {
    // =============================== MMA issuers, one warp per slot
    // (sliding window, where a CTA's few tiles per head make the phase
    // boundaries, not the steady state, the critical path)
    // Each warp walks the K/V ring in the producer's order and issues its
    // slot's MMAs: S_X(t) on K_t, and PV_X(t) on V_t once the softmax has
    // written P_X(t).  Entries the slot does not use (the other half of a
    // split head, or a phase without a head for this slot) are released
    // after they have landed, so every entry gets exactly two releases.  The
    // slots run apart from each other as far as the ring allows.  S_X(t+A)
    // overwrites the TMEM columns PV_X(t) reads P from; both come from this
    // warp and tcgen05.mma instructions of one thread execute in issue order,
    // so the read of P precedes the overwrite.  The whole warp runs the loop
    // so descriptors stay warp-uniform; one elected lane issues.
    const int x = warp - kMmaWarp;
    const bool leader = elect_one();
    constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, false, true);
    uint32_t q_uses = 0, p_waits = 0, ofree_waits = 0, o_commits = 0;
    uint32_t c = 0;       // ring position of the next K/V entry
    bool o_used = false;  // O_X holds a finished head the epilogue must read first
    bool ok = true;
    const uint64_t qd = sdesc_sw128(sbase + L::kQOff + x * L::kQBytes, 16, 1024);
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      for (int ph = 0; ph < n_phases && ok; ++ph) {
        const PhasePlan pl = phase_plan(ph, n_heads, w.n_tiles);
        const bool active = x < pl.nslot;
        if (active) {
          ok = __all_sync(0xffffffffu, mbar_wait(q_full(x), q_uses & 1u, abort_flag));
          ++q_uses;
          if (!ok) break;
        }
        const int ahead = pl.split ? 2 : 1;
        // this slot's last tile of the phase (its last use of Q_X)
        const int last_t = pl.split ? x + 2 * ((w.n_tiles - 1 - x) / 2) : w.n_tiles - 1;
        bool first_pv = true;
        auto entry = [&](int t, bool is_v) {
          const int s = static_cast<int>(c % n_stages);
          ok = __all_sync(0xffffffffu, mbar_wait(kv_full(s), (c / n_stages) & 1u, abort_flag));
          ++c;
          if (!ok) return;
          const bool mine = active && (!pl.split || (t & 1) == x);
          if (!mine) {
            if (leader) mbar_arrive(kv_empty(s));
            return;
          }
          tc_fence_after();
          const uint32_t base = sbase + L::kKvOff + s * L::kKvBytes;
          if (!is_v) {
            const uint64_t kd = sdesc_sw128(base, 16, 1024);
            if (leader) {
#pragma unroll
              for (int k = 0; k < D / 16; ++k) {
                const uint32_t qoff = (k >> 2) * (kBM * 128) + (k & 3) * 32;
                const uint32_t koff = (k >> 2) * (kBN * 128) + (k & 3) * 32;
                umma_ss(t_s(x), qd + (qoff >> 4), kd + (koff >> 4), kIdescS, k > 0 ? 1u : 0u);
              }
              umma_commit(s_full(x));
              if (t == last_t) umma_commit(q_empty(x));
              umma_commit(kv_empty(s));
            }
          } else {
            ok = __all_sync(0xffffffffu, mbar_wait(p_full(x), p_waits & 1u, abort_flag));
            ++p_waits;
            if (ok && first_pv && o_used) {
              // the previous head's epilogue must have read O_X
              ok = __all_sync(0xffffffffu, mbar_wait(o_free(x), ofree_waits & 1u, abort_flag));
              ++ofree_waits;
            }
            if (!ok) return;
            tc_fence_after();
            const uint64_t vd = sdesc_sw128(base, kBN * 128, 1024);
            if (leader) {
#pragma unroll
              for (int k = 0; k < kBN / 16; ++k)
                umma_ts(t_o(x), t_s(x) + p_col(k), vd + ((k * (16 * 128)) >> 4), kIdescPV,
                        (!first_pv || k > 0) ? 1u : 0u);
              umma_commit(o_done(x));
              umma_commit(kv_empty(s));
            }
            ++o_commits;
            first_pv = false;
          }
        };
        for (int t = 0; t < ahead && t < w.n_tiles && ok; ++t) entry(t, false);
        for (int t = 0; t < w.n_tiles && ok; ++t) {
          entry(t, true);
          if (ok && t + ahead < w.n_tiles) entry(t + ahead, false);
        }
        if (active) o_used = true;
      }
    }
    // drain: every MMA issued above must finish before TMEM is released
    if (leader && o_commits) mbar_wait_for(o_done(x), (o_commits - 1) & 1u, 100000000ull);
  }
  } else if (warp >= 8) {
    // =============================== epilogue warpgroup (warps 8-11)
    // Sliding window (staged): a signal head's gate tile [128 rows][d]
    // arrives by TMA in a 128B-swizzled staging buffer, each thread
    // overwrites its row with the output in place, and TMA stores the tile:
    // global traffic moves as whole tiles instead of 16-byte pieces of 128
    // rows.  Full attention, where the epilogue is off the critical path,
    // reads the gate and writes the output row by row.
    regs_decrease<RegSplit<kWin>::kEpilogue>();
    const int wq = warp & 3;          // TMEM lane quarter
    const int r = threadIdx.x & 127;  // row in the block = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    constexpr bool staged = kWin;
    const uint32_t gbuf = sbase + L::kKvOff + 2 * L::kKvBytes;  // staging (window mode)
    const bool issuer = kWin && warp == 8 ? elect_one() : false;
    // H_N: [d/4][kBM] float4 in the window kernel (one 16-byte load per 4
    // columns), [d][kBM] floats in the full kernel (fewer live registers)
    float4 *hn4 = reinterpret_cast<float4 *>(hn_smem);
    uint32_t go_waits[2] = {0, 0};
    uint32_t pv_seen[2] = {0, 0};  // PV commits per slot in finished phases
    uint32_t g_issued = 0, g_seen = 0;  // staged gate tiles loaded / consumed
    bool ok = true;
    // waits until slot x has handed over the head it ran in this phase and
    // its last PV (number `last` of the slot) has completed
    auto wait_slot = [&](int x, uint32_t last) -> bool {
      const uint32_t gw = x == 0 ? go_waits[0] : go_waits[1];
      bool w = mbar_wait(epi_go(x), gw & 1u, abort_flag);
      if (x == 0) ++go_waits[0]; else ++go_waits[1];
      if (w) w = mbar_wait(o_done(x), last & 1u, abort_flag);
      w = __all_sync(0xffffffffu, w);
      tc_fence_after();
      return w;
    };
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const int kvh = w.kvh, n_tiles = w.n_tiles;
      const int i = w.q0 + r;  // query token
      const bool row_ok = i < p.T;
      const int64_t row = static_cast<int64_t>(w.b) * p.T + i;
      for (int ph = 0; ph < n_phases && ok; ++ph) {
        const PhasePlan pl = phase_plan(ph, n_heads, n_tiles);
        const int tiles0 = pl.split ? (n_tiles + 1) / 2 : n_tiles;
        const int tiles1 = pl.split ? n_tiles / 2 : n_tiles;
        // one epilogue per slot, or one merged epilogue for a split head
        const int n_epi = pl.split ? 1 : pl.nslot;
        for (int e_i = 0; e_i < n_epi && ok; ++e_i) {
          const int x = e_i;
          const int hi = x == 0 ? pl.head0 : pl.head1;
          const int h = p.g * kvh + (hi - 1);  // signal head (hi >= 1)
          if (hi != 0) {
            if (staged) {
              if (issuer) {
                // the previous tile's stores must have read the buffer
                bulk_wait_group_read0();
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(g_full, (D / 64) * L::kStageHalf);
#pragma unroll
                for (int hf = 0; hf < D / 64; ++hf)
                  tma_load_3d(gbuf + hf * L::kStageHalf, &tm_gate, g_full, h * D + hf * 64, w.q0,
                              w.b);
              }
              ++g_issued;
            } else if (row_ok) {
              // the gate row heads for L2 while the slot still computes
              const __nv_bfloat16 *gr = p.gate + (row * p.Hs + h) * static_cast<int64_t>(D);
#pragma unroll
              for (int ln = 0; ln < D * 2 / 128; ++ln) prefetch_l2(gr + ln * 64);
            }
            if (row_ok) prefetch_l2(p.lam + row * p.Hs + h);
          }
          float fa = 1.f, fb = 0.f, l_tot;
          if (pl.split) {
            ok = wait_slot(0, pv_seen[0] + tiles0 - 1);
            if (ok) ok = wait_slot(1, pv_seen[1] + tiles1 - 1);
            if (!ok) break;
            // both maxima are integral, so the merge factors are exact powers of two
            const float l_a = stat[0 * 2 * kBM + r], m_a = stat[0 * 2 * kBM + kBM + r];
            const float l_b = stat[1 * 2 * kBM + r], m_b = stat[1 * 2 * kBM + kBM + r];
            const float m = fmaxf(m_a, m_b);
            fa = (m_a == -INFINITY) ? 0.f : exp2_int(m_a - m);
            fb = (m_b == -INFINITY) ? 0.f : exp2_int(m_b - m);
            l_tot = l_a * fa + l_b * fb;
            mbar_arrive(stat_free(0));
            mbar_arrive(stat_free(1));
          } else {
            ok = wait_slot(x, pv_seen[x == 0 ? 0 : 1] + (x == 0 ? tiles0 : tiles1) - 1);
            if (!ok) break;
            l_tot = stat[x * 2 * kBM + r];
            mbar_arrive(stat_free(x));
          }
          const float inv_l = l_tot > 0.f ? 1.f / l_tot : 0.f;
          // O of this head, chunk cc (32 columns), merged over a split head's slots
          auto load_o = [&](int cc, uint32_t (&o)[32]) {
            tmem_ld32_sync(t_o(x) + lane_off + cc * 32, o);
            if (pl.split) {
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                uint32_t ob[16];
                tmem_ld16_sync(t_o(1) + lane_off + cc * 32 + hh * 16, ob);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                  o[hh * 16 + e] = __float_as_uint(__uint_as_float(o[hh * 16 + e]) * fa +
                                                   __uint_as_float(ob[e]) * fb);
              }
            }
          };
          // out = G (.) (O/l - lambda H_N) for 8 columns from column c
          auto combine8 = [&](const uint32_t *o8, int c, uint4 gv, float lam) -> uint4 {
            float hn[8];
            if (kWin) {
              const float4 n0 = hn4[(c >> 2) * kBM + r];
              const float4 n1 = hn4[((c >> 2) + 1) * kBM + r];
              hn[0] = n0.x; hn[1] = n0.y; hn[2] = n0.z; hn[3] = n0.w;
              hn[4] = n1.x; hn[5] = n1.y; hn[6] = n1.z; hn[7] = n1.w;
            }
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (!kWin) {
                hn[2 * e] = hn_smem[(c + 2 * e) * kBM + r];
                hn[2 * e + 1] = hn_smem[(c + 2 * e + 1) * kBM + r];
              }
              const float d0 = __uint_as_float(o8[2 * e]) * inv_l - lam * hn[2 * e];
              const float d1 = __uint_as_float(o8[2 * e + 1]) * inv_l - lam * hn[2 * e + 1];
              ow[e] = pack_bf16x2(bf16lo_to_f32(gw[e]) * d0, bf16hi_to_f32(gw[e]) * d1);
            }
            return make_uint4(ow[0], ow[1], ow[2], ow[3]);
          };
          if (hi == 0) {
            // noise head (never split: it runs in phase 0 next to signal head 0):
            // H_N = O / l stays in shared memory for the group's signal heads;
            // this warpgroup is also the only reader, row by row
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld32_sync(t_o(x) + lane_off + cc * 32, o);
              if (kWin) {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                  hn4[(cc * 8 + q) * kBM + r] = make_float4(
                      __uint_as_float(o[4 * q]) * inv_l, __uint_as_float(o[4 * q + 1]) * inv_l,
                      __uint_as_float(o[4 * q + 2]) * inv_l, __uint_as_float(o[4 * q + 3]) * inv_l);
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                  hn_smem[(cc * 32 + e) * kBM + r] = __uint_as_float(o[e]) * inv_l;
              }
            }
          } else if (staged) {
            const float lam = row_ok ? __bfloat162float(p.lam[row * p.Hs + h]) : 0.f;
            ok = __all_sync(0xffffffffu, mbar_wait(g_full, g_seen & 1u, abort_flag));
            ++g_seen;
            if (!ok) break;
            // row r of a 128B-swizzled [128][64] half: 16-byte unit j sits at j ^ (r % 8)
            const uint32_t rbase = gbuf + static_cast<uint32_t>(r) * 128u;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              load_o(cc, o);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int j = (cc & 1) * 4 + q;
                const uint32_t addr = rbase + static_cast<uint32_t>(cc >> 1) * L::kStageHalf +
                                      (static_cast<uint32_t>(j ^ (r & 7)) << 4);
                sts128(addr, combine8(o + q * 8, cc * 32 + q * 8, lds128(addr), lam));
              }
            }
            // every row written (generic proxy) before the TMA store reads the tile
            fence_proxy_async_smem();
            mbar_arrive(g_done);
            if (issuer) {
              ok = mbar_wait(g_done, (g_seen - 1) & 1u, abort_flag);
              if (ok) {
#pragma unroll
                for (int hf = 0; hf < D / 64; ++hf)
                  tma_store_3d(&tm_out, gbuf + hf * L::kStageHalf, h * D + hf * 64, w.q0, w.b);
                bulk_commit_group();
              }
            }
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          } else {
            const int64_t goff = (row * p.Hs + h) * static_cast<int64_t>(D);
            float lam = 0.f;
            if (row_ok) lam = __bfloat162float(p.lam[row * p.Hs + h]);
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld32_sync(t_o(x) + lane_off + cc * 32, o);
              if (pl.split) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  uint32_t ob[16];
                  tmem_ld16_sync(t_o(1) + lane_off + cc * 32 + hh * 16, ob);
#pragma unroll
                  for (int e = 0; e < 16; ++e)
                    o[hh * 16 + e] = __float_as_uint(__uint_as_float(o[hh * 16 + e]) * fa +
                                                     __uint_as_float(ob[e]) * fb);
                }
              }
              if (row_ok) {
                const uint4 *gp = reinterpret_cast<const uint4 *>(p.gate + goff + cc * 32);
                uint4 *op = reinterpret_cast<uint4 *>(p.out + goff + cc * 32);
                uint4 gv[4];
#pragma unroll
                for (int v = 0; v < 4; ++v) gv[v] = __ldg(gp + v);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                  const uint32_t gw[4] = {gv[v].x, gv[v].y, gv[v].z, gv[v].w};
                  uint32_t ow[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const int c0 = cc * 32 + v * 8 + 2 * e;
                    const float d0 = __uint_as_float(o[v * 8 + 2 * e]) * inv_l -
                                     lam * hn_smem[c0 * kBM + r];
                    const float d1 = __uint_as_float(o[v * 8 + 2 * e + 1]) * inv_l -
                                     lam * hn_smem[(c0 + 1) * kBM + r];
                    ow[e] = pack_bf16x2(bf16lo_to_f32(gw[e]) * d0, bf16hi_to_f32(gw[e]) * d1);
                  }
                  op[v] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
              }
            }
          }
          tc_fence_before();
          mbar_arrive(o_free(x));
          if (pl.split) mbar_arrive(o_free(1));
        }
        pv_seen[0] += static_cast<uint32_t>(tiles0);
        if (pl.nslot == 2) pv_seen[1] += static_cast<uint32_t>(tiles1);
      }
    }
    if (kWin && issuer) {
      // a gate tile still in flight (after an abort) lands before the CTA exits;
      // every output tile store completes
      if (g_issued > g_seen) mbar_wait_for(g_full, (g_issued - 1) & 1u, 100000000ull);
      bulk_wait_group0();
    }
  } else {
    // =============================== softmax (one warpgroup per slot)
    regs_increase<RegSplit<kWin>::kSoftmax>();
    const int x = warp >> 2;          // slot
    const int wq = warp & 3;          // TMEM lane quarter
    const int r = threadIdx.x & 127;  // row in the block = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t s_waits = 0;
    uint32_t o_seen = 0;  // PV commits of this slot in finished phases
    uint32_t handoffs = 0;  // heads handed to the epilogue warpgroup
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const int j_lo = w.j_lo, q0 = w.q0, n_tiles = w.n_tiles;
      const int i = q0 + r;  // query token
      for (int ph = 0; ph < n_phases && ok; ++ph) {
        const PhasePlan pl = phase_plan(ph, n_heads, n_tiles);
        if (x >= pl.nslot) break;
        const int t0 = pl.split ? x : 0;
        const int step = pl.split ? 2 : 1;
        const int my_tiles = pl.split ? (n_tiles - x + 1) / 2 : n_tiles;
        float m_run = -INFINITY, l_run = 0.f;
        int k_idx = 0;
        for (int t = t0; t < n_tiles; t += step, ++k_idx) {
          ok = mbar_wait(s_full(x), s_waits & 1u, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          ++s_waits;
          tc_fence_after();
          const int kbase = (j_lo + t) * kBN;
          // kept key columns of this row in the tile
          int c_lo, c_hi;
          if (p.causal) {
            c_hi = i - kbase;
            c_lo = p.window > 0 ? static_cast<int>(static_cast<int64_t>(i) - p.window + 1 - kbase)
                                : -1;
          } else {
            c_hi = p.T - 1 - kbase;
            c_lo = -1;
          }
          // CTA-uniform: does any row of the block lose a key of this tile?
          bool masked;
          if (p.causal) {
            masked = (kbase + kBN - 1 > q0) ||
                     (p.window > 0 && static_cast<int64_t>(kbase) <= q0 + kBM - 1 - p.window);
          } else {
            masked = kbase + kBN > p.T;
          }
          // Full attention reads the whole score row of the tile in one TMEM
          // round trip for the row max; chunks 0 and 1 stay in registers for
          // the exponentials while chunks 2 and 3 are read again behind them.
          // Columns the mask drops become -inf (a warp classifies each chunk
          // warp-uniformly: every column kept, none kept, or mixed).  Sliding
          // windows wider than one tile go chunk by chunk and skip the chunks
          // no row of the warp keeps.
          auto mask_chunk = [&](uint32_t (&v)[32], int cc) {
            const int cls = chunk_class(cc, c_lo, c_hi);
            if (cls == kChunkFull) return;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int c = cc * 32 + e;
              if (cls == kChunkEmpty || c < c_lo || c > c_hi) v[e] = 0xff800000u;
            }
          };
          float mt_raw = -INFINITY;
          uint32_t s0[32], s1[32], s2[32], s3[32];
          if constexpr (!kWin) {
            tmem_ld32x4_sync(t_s(x) + lane_off, s0, s1, s2, s3);
            if (masked) {
              mask_chunk(s0, 0);
              mask_chunk(s1, 1);
              mask_chunk(s2, 2);
              mask_chunk(s3, 3);
            }
            float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              ma = fmax3(ma, __uint_as_float(s0[e]), __uint_as_float(s0[e + 1]));
              mb = fmax3(mb, __uint_as_float(s1[e]), __uint_as_float(s1[e + 1]));
              ma = fmax3(ma, __uint_as_float(s2[e]), __uint_as_float(s2[e + 1]));
              mb = fmax3(mb, __uint_as_float(s3[e]), __uint_as_float(s3[e + 1]));
            }
            // chunk 2 is read again while chunks 0 and 1 are exponentiated
            tmem_ld32(t_s(x) + lane_off + 64, s2);
            mt_raw = fmaxf(ma, mb);
          } else {
            // chunks no row of the warp keeps are not even read
#pragma unroll 1
            for (int cc = 0; cc < kBN / 32; ++cc) {
              const int cls = chunk_class(cc, c_lo, c_hi);
              if (cls == kChunkEmpty) continue;
              uint32_t raw[32];
              tmem_ld32_sync(t_s(x) + lane_off + cc * 32, raw);
              if (cls == kChunkFull) {
#pragma unroll
                for (int e = 0; e < 32; e += 2)
                  mt_raw = fmax3(mt_raw, __uint_as_float(raw[e]), __uint_as_float(raw[e + 1]));
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  const int c = cc * 32 + e;
                  if (c >= c_lo && c <= c_hi) mt_raw = fmaxf(mt_raw, __uint_as_float(raw[e]));
                }
              }
            }
          }
          const float mt = mt_raw * sl2;  // scale > 0 keeps the arg max
          const float m_new = fmaxf(m_run, mt);
          float alpha = 1.f;
          float m_use = m_run;
          if (m_new > m_run + kRescaleThreshold || m_run == -INFINITY) {
            m_use = ceilf(m_new);  // integral reference; -inf stays -inf
            alpha = (m_run == -INFINITY) ? 0.f : exp2_int(m_run - m_use);
          }
          const float m_safe = (m_use == -INFINITY) ? 0.f : m_use;
          const uint64_t sl2x2 = f2_make(sl2, sl2);
          const uint64_t negm2 = f2_make(-m_safe, -m_safe);
          uint64_t rs2 = f2_make(0.f, 0.f);
          if constexpr (!kWin) {
            // P = exp2(S*c - m) as bf16 pairs; chunk cc lands in columns
            // [16cc, 16cc+16), below the S columns still to be read
            auto exp_chunk = [&](const uint32_t (&v)[32], int cc) {
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
              tmem_st16(t_s(x) + lane_off + cc * 16, pk);
            };
            exp_chunk(s0, 0);
            exp_chunk(s1, 1);
            tmem_wait_ld_fence(s2);
            tmem_ld32(t_s(x) + lane_off + 96, s3);
            if (masked) mask_chunk(s2, 2);
            exp_chunk(s2, 2);
            tmem_wait_ld_fence(s3);
            if (masked) mask_chunk(s3, 3);
            exp_chunk(s3, 3);
          } else {
            // sliding window: chunks no row of the warp keeps are neither read
            // nor exponentiated (their P is zero)
#pragma unroll 1
            for (int cc = 0; cc < kBN / 32; ++cc) {
              const int cls = chunk_class(cc, c_lo, c_hi);
              uint32_t pk[16];
              if (cls == kChunkEmpty) {
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = 0u;
              } else {
                uint32_t raw[32];
                tmem_ld32_sync(t_s(x) + lane_off + cc * 32, raw);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                  float t0v, t1v;
                  f2_split(f2_fma(f2_from_bits(raw[2 * e], raw[2 * e + 1]), sl2x2, negm2), t0v, t1v);
                  if (cls == kChunkMixed) {
                    const int c0 = cc * 32 + 2 * e;
                    if (!(c0 >= c_lo && c0 <= c_hi)) t0v = -INFINITY;
                    if (!(c0 + 1 >= c_lo && c0 + 1 <= c_hi)) t1v = -INFINITY;
                  }
                  const float p0 = ex2_approx(t0v);
                  const float p1 = ex2_approx(t1v);
                  rs2 = f2_add(rs2, f2_make(p0, p1));
                  pk[e] = pack_bf16x2(p0, p1);
                }
              }
              tmem_st16(t_s(x) + lane_off + cc * 16, pk);
            }
          }
          float rs0, rs1;
          f2_split(rs2, rs0, rs1);
          l_run = l_run * alpha + (rs0 + rs1);
          m_run = m_use;
          // O holds the sum over earlier tiles; rescale it when the max moved
          const bool need = (alpha != 1.f) && (k_idx > 0);
          if (__any_sync(0xffffffffu, need)) {
            const uint32_t prev = o_seen + static_cast<uint32_t>(k_idx - 1);
            ok = mbar_wait(o_done(x), prev & 1u, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[32];
              tmem_ld32_sync(t_o(x) + lane_off + cc * 32, o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(t_o(x) + lane_off + cc * 32, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(p_full(x));
        }
        if (!ok) break;
        // ---- hand the head to the epilogue warpgroup: row sum and reference
        // max.  The epilogue must have read the previous hand-off first (a
        // phase with one tile per slot waits on nothing else from it).
        if (handoffs > 0) {
          ok = mbar_wait(stat_free(x), (handoffs - 1) & 1u, abort_flag);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        ++handoffs;
        stat[x * 2 * kBM + r] = l_run;
        stat[x * 2 * kBM + kBM + r] = m_run;
        o_seen += static_cast<uint32_t>(my_tiles);
        mbar_arrive(epi_go(x));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) write_status(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gdla
