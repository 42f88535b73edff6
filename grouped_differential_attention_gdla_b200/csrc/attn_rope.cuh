// attn_rope.cuh - GDLA attention forward with the decoupled rotary term,
// sm_100a.
//
// Operation ("Motif 3: Technical Report", paper.rainbus.top: step 2 "GDLA
// forward", and the "technical novelty" paragraph: both query paths share the
// up-projected KV and one broadcast decoupled rotary key):
//   s_ij = scale * (q_i . k_j + q_r,i . k_r,j)
// where every head of both paths has its own rotary query q_r (kRope = 64
// wide) and every token one rotary key k_r shared by all heads, then softmax,
// P V, D = H_S - lambda Repeat_g(H_N), O = G (.) D as in attn_fwd.cuh.
//
// The score contracts over d + 64 = 192 columns, so a query tile and a K
// ring entry are 48 KB each.  Two query tiles next to a three-deep ring of
// such entries would not fit in shared memory, so this kernel runs one head
// at a time and keeps the tensor core busy another way:
//   - the score S is double-buffered in TMEM: S(t+1) and S(t+2) are computed
//     while the softmax works on S(t);
//   - two softmax warpgroups share every score row, each taking 64 of the 128
//     key columns; the two halves of a row meet once per tile to agree on
//     the row maximum (an mbarrier per pair of warps, so a wait can give up);
//   - the noise head's output stays in TMEM (unnormalised, H_N region) for
//     the whole item, and the epilogue warpgroup combines it with each signal
//     head's output: D = O / l - lambda * O_N / l_N.
// A work item is (batch b, KV group k, block of 128 query tokens); its g+1
// heads run noise first, each over the K/V tiles its mask reaches.  Per tile
// t of a head:
//   S(t)  = [Q | Q_r] [K_t | K_r,t]^T   tcgen05.mma, 12 K-steps (A, B in smem)
//   P(t)  = exp2(S*c - m)               softmax warpgroups, P over S in TMEM
//   O    += P(t) V_t                    tcgen05.mma (A = P from TMEM)
// The K ring entry holds the group's K tile and the rotary key tile of the
// same tokens (one TMA load each); V entries use 32 KB of their 48.
//
// Warp roles (512 threads, 128 registers each):
//   warps 0-3   softmax, key columns 0..63 of every row (TMEM lanes 0..127)
//   warps 4-7   softmax, key columns 64..127
//   warps 8-11  epilogue: D, lambda, gate, output rows
//   warp  12    TMA producer (query tiles, K/V ring)
//   warp  13    TMEM allocator and MMA issuer
//   warps 14-15 idle
// TMEM (512 columns): S0 [0,128) S1 [128,256) O [256,256+d) O_N [256+d,256+2d).
// P occupies the first 64 columns of its S buffer as packed bf16 pairs.
#pragma once

#include "attn_win.cuh"

namespace gdla {

constexpr int kRope = 64;  // rotary width the kernel takes
constexpr int kRopeThreads = 16 * 32;
constexpr int kRopeProducerWarp = 12;
constexpr int kRopeMmaWarp = 13;
constexpr int kRopeStages = 3;

// Parameters of the save mode (the forward a backward pass starts from):
// every head's output H = O / l (fp32, [B, T, Hs + Hn, d], signal heads first)
// and its log-sum-exp in log2 units of the scaled scores, head-major with the
// token axis padded to tp (a multiple of 128): [B, Hs + Hn, tp].
struct AttnSaveParams : AttnParams {
  float *h;
  float *lse;
  int tp;
};

// R: rotary width (kRope, or 0 without the rotary term).
template <int D, int R = kRope>
struct RopeSmemLayout {
  static constexpr uint32_t kSub = kBM * 128;          // one [128][64] bf16 swizzled sub-tile
  static constexpr int kQkSubs = (D + R) / 64;         // sub-tiles of a query tile / K entry
  static constexpr uint32_t kQBytes = kQkSubs * kSub;  // [Q | Q_r]
  static constexpr uint32_t kEntry = kQkSubs * kSub;   // [K | K_r], or V in its first D/64
  static constexpr uint32_t kVBytes = (D / 64) * kSub;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kRingOff = kQOff + kQBytes;
  static constexpr uint32_t kMaxOff = kRingOff + kRopeStages * kEntry;  // float [2 buf][2 half][kBM]
  static constexpr uint32_t kStatOff = kMaxOff + 2 * 2 * kBM * 4;  // float [2 slot][l0, l1, m][kBM]
  static constexpr uint32_t kBarOff = kStatOff + 2 * 3 * kBM * 4;
  // q_full q_empty kv_full[S] kv_empty[S] s_full[2] p_full[2] mx_bar[2][4]
  // o_done[2] acc_free[2] epi_go[2] stat_free[2] head_done
  static constexpr uint32_t kNumBars = 2 + 2 * kRopeStages + 2 + 2 + 8 + 2 + 2 + 2 + 2 + 1;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
};

// kSave (with R = 0): the save mode.  Every head, the noise head included,
// accumulates in the O region, and the epilogue writes H and the log-sum-exp
// of every head instead of the gated differential.
template <int D, int R = kRope, bool kSave = false, typename Params = AttnParams>
__global__ void __launch_bounds__(kRopeThreads, 1)
    gdla_attn_rope_kernel(const __grid_constant__ CUtensorMap tm_qs,
                          const __grid_constant__ CUtensorMap tm_qn,
                          const __grid_constant__ CUtensorMap tm_qrs,
                          const __grid_constant__ CUtensorMap tm_qrn,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_kr,
                          const __grid_constant__ CUtensorMap tm_v, const Params p) {
  static_assert(!kSave || R == 0, "the save mode takes no rotary term");
  using L = RopeSmemLayout<D, R>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) write_status(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t q_full = bar0, q_empty = bar0 + 8u;
  auto kv_full = [&](uint32_t s) { return bar0 + 8u * (2 + s); };
  auto kv_empty = [&](uint32_t s) { return bar0 + 8u * (2 + kRopeStages + s); };
  auto s_full = [&](uint32_t b) { return bar0 + 8u * (2 + 2 * kRopeStages + b); };
  auto p_full = [&](uint32_t b) { return bar0 + 8u * (4 + 2 * kRopeStages + b); };
  auto mx_bar = [&](uint32_t b, uint32_t wq) { return bar0 + 8u * (6 + 2 * kRopeStages + 4 * b + wq); };
  auto o_done = [&](uint32_t a) { return bar0 + 8u * (14 + 2 * kRopeStages + a); };
  auto acc_free = [&](uint32_t a) { return bar0 + 8u * (16 + 2 * kRopeStages + a); };
  auto epi_go = [&](uint32_t s) { return bar0 + 8u * (18 + 2 * kRopeStages + s); };
  auto stat_free = [&](uint32_t s) { return bar0 + 8u * (20 + 2 * kRopeStages + s); };
  // one phase per signal head: its last PV (and every MMA before it) is done.
  // o_done has a phase per PV, and S runs two tiles ahead of PV, so a wait
  // for a head's last PV there could come two phases early and alias.
  const uint32_t head_done = bar0 + 8u * (22 + 2 * kRopeStages);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  float *mx = reinterpret_cast<float *>(smem + L::kMaxOff);    // [buf][half][row]
  float *stat = reinterpret_cast<float *>(smem + L::kStatOff);  // [slot][l0, l1, m][row]
  const int warp = threadIdx.x >> 5;
  const int n_heads = p.g + 1;  // noise head + g signal heads

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (uint32_t s = 0; s < kRopeStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (uint32_t b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(p_full(b), 8);  // one arrival per softmax warp
      for (uint32_t wq = 0; wq < 4; ++wq) mbar_init(mx_bar(b, wq), 2);  // the two halves of a row
      mbar_init(o_done(b), 1);
      mbar_init(acc_free(b), 4);  // epilogue warps
      mbar_init(epi_go(b), 8);    // softmax warps
      mbar_init(stat_free(b), 4);
    }
    mbar_init(head_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kRopeMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto t_s = [&](uint32_t b) { return tmem + 128u * b; };
  // accumulator region a: 0 = O of the current signal head, 1 = O_N of the noise head
  auto t_acc = [&](uint32_t a) { return tmem + 256u + static_cast<uint32_t>(D) * a; };

  if (warp == kRopeProducerWarp) {
    // =============================== TMA producer
    // Per head: its query tile [Q | Q_r] once the previous head's last S has
    // read the buffer, then the ring in the order the MMA warp consumes it:
    // K_0, K_1, then V_t, K_{t+2} for t = 0..n-1.  The whole warp runs the
    // loop (warp-uniform waits); one elected lane issues the copies.
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_qs);
      tma_prefetch_desc(&tm_qn);
      if (R > 0) {
        tma_prefetch_desc(&tm_qrs);
        tma_prefetch_desc(&tm_qrn);
        tma_prefetch_desc(&tm_kr);
      }
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    uint32_t c = 0, q_uses = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      auto load_kv = [&](int t, bool is_v) {
        const uint32_t s = c % kRopeStages;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(kv_empty(s), ((c / kRopeStages) & 1u) ^ 1u, abort_flag));
        if (!ok) return;
        const uint32_t dst = sbase + L::kRingOff + s * L::kEntry;
        const int row = (w.j_lo + t) * kBN;
        if (leader) {
          mbar_arrive_expect_tx(kv_full(s), is_v ? L::kVBytes : L::kEntry);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(dst + kb * L::kSub, is_v ? &tm_v : &tm_k, kv_full(s), w.kvh * D + kb * 64,
                        row, w.b);
          if (R > 0 && !is_v)
            tma_load_3d(dst + (D / 64) * L::kSub, &tm_kr, kv_full(s), 0, row, w.b);
        }
        ++c;
      };
      for (int hi = 0; hi < n_heads && ok; ++hi) {
        ok = __all_sync(0xffffffffu, mbar_wait(q_empty, (q_uses & 1u) ^ 1u, abort_flag));
        if (!ok) break;
        ++q_uses;
        const bool noise = hi == 0;
        const int head = noise ? w.kvh : p.g * w.kvh + (hi - 1);
        if (leader) {
          mbar_arrive_expect_tx(q_full, L::kQBytes);
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(sbase + L::kQOff + kb * L::kSub, noise ? &tm_qn : &tm_qs, q_full,
                        head * D + kb * 64, w.q0, w.b);
          if (R > 0)
            tma_load_3d(sbase + L::kQOff + (D / 64) * L::kSub, noise ? &tm_qrn : &tm_qrs, q_full,
                        head * R, w.q0, w.b);
        }
        const int n = w.n_tiles;
        load_kv(0, false);
        if (ok && n > 1) load_kv(1, false);
        for (int t = 0; t < n && ok; ++t) {
          load_kv(t, true);
          if (ok && t + 2 < n) load_kv(t + 2, false);
        }
      }
    }
    if (!ok && leader) {
      // unwinding: let the copies already issued land before the CTA exits
      for (uint32_t s = 0; s < kRopeStages; ++s) {
        const uint32_t issued = c > s ? (c - 1 - s) / kRopeStages + 1 : 0;
        if (issued) mbar_wait_for(kv_full(s), (issued - 1) & 1u, 100000000ull);
      }
      if (q_uses) mbar_wait_for(q_full, (q_uses - 1) & 1u, 100000000ull);
    }
  } else if (warp == kRopeMmaWarp) {
    // =============================== MMA issuer
    // Per head: S(0), S(1), then for every tile PV(t) once the softmax has
    // written P(t), and S(t+2) into the buffer PV(t) reads P from.  The
    // tcgen05.mma instructions of one thread execute in issue order, so the
    // read of P precedes the overwrite.  A head's first PV waits until the
    // epilogue has read the accumulator region's previous contents.
    const bool leader = elect_one();
    constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, false, true);
    constexpr int kSSteps = (D + R) / 16;
    const uint64_t qd = sdesc_sw128(sbase + L::kQOff, 16, 1024);
    uint32_t c = 0, q_uses = 0, sc = 0;  // ring position, query tiles, S tiles issued
    // per S buffer / accumulator region (kept as scalars: runtime-indexed
    // arrays would live in local memory)
    uint32_t p_waits0 = 0, p_waits1 = 0;
    uint32_t acc_heads0 = 0, acc_heads1 = 0, acc_waits0 = 0, acc_waits1 = 0;
    bool ok = true;
    auto next_stage = [&](uint32_t &base) -> uint32_t {
      const uint32_t s = c % kRopeStages;
      ok = __all_sync(0xffffffffu, mbar_wait(kv_full(s), (c / kRopeStages) & 1u, abort_flag));
      tc_fence_after();
      base = sbase + L::kRingOff + s * L::kEntry;
      ++c;
      return s;
    };
    auto issue_s = [&](uint32_t k_base, uint32_t buf) {
      const uint64_t kd = sdesc_sw128(k_base, 16, 1024);
      if (leader) {
#pragma unroll
        for (int k = 0; k < kSSteps; ++k) {
          const uint32_t off = (k >> 2) * L::kSub + (k & 3) * 32;
          umma_ss(t_s(buf), qd + (off >> 4), kd + (off >> 4), kIdescS, k > 0 ? 1u : 0u);
        }
        umma_commit(s_full(buf));
      }
    };
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const int n = w.n_tiles;
      for (int hi = 0; hi < n_heads && ok; ++hi) {
        const uint32_t a = (hi == 0 && !kSave) ? 1u : 0u;
        ok = __all_sync(0xffffffffu, mbar_wait(q_full, q_uses & 1u, abort_flag));
        ++q_uses;
        if (!ok) break;
        const uint32_t sc0 = sc;
        for (int t = 0; t < 2 && t < n && ok; ++t) {
          uint32_t kb;
          const uint32_t s = next_stage(kb);
          if (!ok) break;
          issue_s(kb, (sc0 + t) & 1u);
          if (leader) {
            if (t == n - 1) umma_commit(q_empty);
            umma_commit(kv_empty(s));
          }
        }
        for (int t = 0; t < n && ok; ++t) {
          uint32_t vb;
          const uint32_t sv = next_stage(vb);
          if (!ok) break;
          const uint32_t buf = (sc0 + t) & 1u;
          const uint32_t pw = buf ? p_waits1++ : p_waits0++;
          ok = __all_sync(0xffffffffu, mbar_wait(p_full(buf), pw & 1u, abort_flag));
          if (!ok) break;
          if (t == 0 && (a ? acc_heads1 : acc_heads0) > 0) {
            const uint32_t aw = a ? acc_waits1++ : acc_waits0++;
            ok = __all_sync(0xffffffffu, mbar_wait(acc_free(a), aw & 1u, abort_flag));
            if (!ok) break;
          }
          tc_fence_after();
          const uint64_t vd = sdesc_sw128(vb, kBN * 128, 1024);
          if (leader) {
#pragma unroll
            for (int k = 0; k < kBN / 16; ++k)
              umma_ts(t_acc(a), t_s(buf) + 8u * k, vd + ((k * (16 * 128)) >> 4), kIdescPV,
                      (t > 0 || k > 0) ? 1u : 0u);
            umma_commit(o_done(a));
            umma_commit(kv_empty(sv));
            if (a == 0 && t == n - 1) umma_commit(head_done);
          }
          if (t + 2 < n) {
            uint32_t kb;
            const uint32_t sk = next_stage(kb);
            if (!ok) break;
            issue_s(kb, buf);
            if (leader) {
              if (t + 2 == n - 1) umma_commit(q_empty);
              umma_commit(kv_empty(sk));
            }
          }
        }
        sc = sc0 + static_cast<uint32_t>(n);
        if (a) ++acc_heads1; else ++acc_heads0;
      }
    }
    // drain: every MMA issued above must finish before TMEM is released.  On
    // the normal path the last one is the last signal head's last PV; the
    // head before it is complete (its epilogue released O for this one).
    if (leader && acc_heads0) mbar_wait_for(head_done, (acc_heads0 - 1) & 1u, 100000000ull);
  } else if (warp >= 8 && warp < 12) {
    // =============================== epilogue
    // Per signal head: D = O / l - lambda * O_N / l_N, times the gate, to the
    // output row (one thread per row).  O is released after its last read;
    // O_N after the item's last signal head.
    const int wq = warp & 3;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint32_t go = 0;       // heads handed over
    uint32_t heads = 0;    // signal heads finished
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const int i = w.q0 + r;
      const bool row_ok = i < p.T;
      const int64_t row = static_cast<int64_t>(w.b) * p.T + i;
      float inv_ln = 0.f;
      for (int hi = 0; hi < n_heads && ok; ++hi) {
        const int h = p.g * w.kvh + (hi - 1);  // signal head (hi >= 1)
        if (!kSave && hi > 0 && row_ok) {
          // the gate row heads for L2 while the head still computes
          const __nv_bfloat16 *gr = p.gate + (row * p.Hs + h) * static_cast<int64_t>(D);
#pragma unroll
          for (int ln = 0; ln < D * 2 / 128; ++ln) prefetch_l2(gr + ln * 64);
          prefetch_l2(p.lam + row * p.Hs + h);
        }
        const uint32_t slot = go & 1u;
        ok = __all_sync(0xffffffffu, mbar_wait(epi_go(slot), (go >> 1) & 1u, abort_flag));
        ++go;
        if (!ok) break;
        const float l = stat[(slot * 3 + 0) * kBM + r] + stat[(slot * 3 + 1) * kBM + r];
        const float m_ref = stat[(slot * 3 + 2) * kBM + r];
        warp_arrive(stat_free(slot));
        if constexpr (kSave) {
          // H = O / l and the log-sum-exp of the head (noise heads after the
          // signal heads in the [Hs + Hn] head index)
          ok = __all_sync(0xffffffffu, mbar_wait(head_done, heads & 1u, abort_flag));
          ++heads;
          if (!ok) break;
          tc_fence_after();
          const int hx = hi == 0 ? p.Hs + w.kvh : h;
          const int64_t hrow = row * (p.Hs + p.Hn) + hx;
          const float inv_l = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32_sync(t_acc(0) + lane_off + cc * 32, o);
            if (row_ok) {
              float4 *hp = reinterpret_cast<float4 *>(p.h + hrow * D + cc * 32);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                hp[v] = make_float4(__uint_as_float(o[4 * v]) * inv_l,
                                    __uint_as_float(o[4 * v + 1]) * inv_l,
                                    __uint_as_float(o[4 * v + 2]) * inv_l,
                                    __uint_as_float(o[4 * v + 3]) * inv_l);
            }
          }
          if (row_ok)
            p.lse[(static_cast<int64_t>(w.b) * (p.Hs + p.Hn) + hx) * p.tp + i] =
                l > 0.f ? m_ref + log2f(l) : -INFINITY;
          tc_fence_before();
          warp_arrive(acc_free(0));
          continue;
        }
        if (hi == 0) {
          inv_ln = l > 0.f ? 1.f / l : 0.f;
          continue;
        }
        // the head's last PV (and, issued before it, every PV of the noise head)
        ok = __all_sync(0xffffffffu, mbar_wait(head_done, heads & 1u, abort_flag));
        ++heads;
        if (!ok) break;
        tc_fence_after();
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        const float lam = row_ok ? __bfloat162float(p.lam[row * p.Hs + h]) : 0.f;
        const float lam_n = lam * inv_ln;
        const int64_t goff = (row * p.Hs + h) * static_cast<int64_t>(D);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32], on[32];
          tmem_ld32x2_sync(t_acc(0) + lane_off + cc * 32, t_acc(1) + lane_off + cc * 32, o, on);
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
                const int j = v * 8 + 2 * e;
                const float d0 =
                    __uint_as_float(o[j]) * inv_l - lam_n * __uint_as_float(on[j]);
                const float d1 =
                    __uint_as_float(o[j + 1]) * inv_l - lam_n * __uint_as_float(on[j + 1]);
                ow[e] = pack_bf16x2(bf16lo_to_f32(gw[e]) * d0, bf16hi_to_f32(gw[e]) * d1);
              }
              op[v] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
            }
          }
        }
        tc_fence_before();
        warp_arrive(acc_free(0));
        if (hi == n_heads - 1) warp_arrive(acc_free(1));
      }
    }
  } else if (warp < 8) {
    // =============================== softmax (two warpgroups, half a row each)
    const int half = warp >> 2;      // key columns [64 half, 64 half + 64)
    const int wq = warp & 3;         // TMEM lane quarter
    const int r = threadIdx.x & 127;  // row in the block = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int col0 = 64 * half;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0;                 // S tiles consumed
    uint32_t pv_base0 = 0, pv_base1 = 0;  // PV commits per region in finished heads
    uint32_t handoffs = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const WorkItem w = work_item(p, item);
      const int i = w.q0 + r;  // query token
      const int n = w.n_tiles;
      for (int hi = 0; hi < n_heads && ok; ++hi) {
        const uint32_t a = (hi == 0 && !kSave) ? 1u : 0u;
        float m_run = -INFINITY, l_run = 0.f;
        for (int t = 0; t < n; ++t) {
          const uint32_t b = sc & 1u, par = (sc >> 1) & 1u;
          ++sc;
          ok = __all_sync(0xffffffffu, mbar_wait(s_full(b), par, abort_flag));
          if (!ok) break;
          tc_fence_after();
          const int kbase = (w.j_lo + t) * kBN;
          int c_lo, c_hi;  // kept key columns of this row in the tile
          if (p.causal) {
            c_hi = i - kbase;
            c_lo = p.window > 0 ? static_cast<int>(static_cast<int64_t>(i) - p.window + 1 - kbase)
                                : -1;
          } else {
            c_hi = p.T - 1 - kbase;
            c_lo = -1;
          }
          bool masked;  // CTA-uniform: does any row of the block lose a key of this tile?
          if (p.causal) {
            masked = (kbase + kBN - 1 > w.q0) ||
                     (p.window > 0 && static_cast<int64_t>(kbase) <= w.q0 + kBM - 1 - p.window);
          } else {
            masked = kbase + kBN > p.T;
          }
          uint32_t s0[32], s1[32];
          tmem_ld32x2_sync(t_s(b) + lane_off + col0, t_s(b) + lane_off + col0 + 32, s0, s1);
          if (masked) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int ca = col0 + e, cb = col0 + 32 + e;
              if (ca < c_lo || ca > c_hi) s0[e] = kNegInfBits;
              if (cb < c_lo || cb > c_hi) s1[e] = kNegInfBits;
            }
          }
          float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            ma = fmax3(ma, __uint_as_float(s0[e]), __uint_as_float(s0[e + 1]));
            mb = fmax3(mb, __uint_as_float(s1[e]), __uint_as_float(s1[e + 1]));
          }
          // the two halves of the row meet: each publishes its maximum
          mx[(b * 2 + half) * kBM + r] = fmaxf(ma, mb);
          warp_arrive(mx_bar(b, wq));
          ok = __all_sync(0xffffffffu, mbar_wait(mx_bar(b, wq), par, abort_flag));
          if (!ok) break;
          const float mt_raw = fmaxf(mx[(b * 2 + 0) * kBM + r], mx[(b * 2 + 1) * kBM + r]);
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
          // P = exp2(S*c - m) as bf16 pairs over the S columns this half read
          // (the other half has read its S columns: it arrived above)
          auto exp_chunk = [&](const uint32_t (&v)[32], int cc) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float t0v, t1v;
              f2_split(f2_fma(f2_from_bits(v[2 * e], v[2 * e + 1]), sl2x2, negm2), t0v, t1v);
              const float p0 = ex2_approx(t0v);
              const float p1 = ex2_approx(t1v);
              pk[e] = pack_bf16x2(p0, p1);
              // the save mode sums the bf16 P the PV MMA reads, so that the
              // saved H and log-sum-exp describe the same weights (a row
              // with one key gets H = V exactly)
              if constexpr (kSave)
                rs2 = f2_add(rs2, f2_make(bf16lo_to_f32(pk[e]), bf16hi_to_f32(pk[e])));
              else
                rs2 = f2_add(rs2, f2_make(p0, p1));
            }
            tmem_st16(t_s(b) + lane_off + cc * 16, pk);
          };
          exp_chunk(s0, 2 * half);
          exp_chunk(s1, 2 * half + 1);
          float rs0, rs1;
          f2_split(rs2, rs0, rs1);
          l_run = l_run * alpha + (rs0 + rs1);
          m_run = m_use;
          // the accumulator holds earlier tiles; rescale this half's columns
          // of it when the max moved (both halves take the same decision)
          const bool need = (alpha != 1.f) && (t > 0);
          if (__any_sync(0xffffffffu, need)) {
            const uint32_t prev = (a ? pv_base1 : pv_base0) + static_cast<uint32_t>(t - 1);
            ok = __all_sync(0xffffffffu, mbar_wait(o_done(a), prev & 1u, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
              const uint32_t col = static_cast<uint32_t>(half * (D / 2) + cc * 32);
              uint32_t o[32];
              tmem_ld32_sync(t_acc(a) + lane_off + col, o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(t_acc(a) + lane_off + col, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(p_full(b));
        }
        if (!ok) break;
        // ---- hand the head's partial row sum to the epilogue
        const uint32_t slot = handoffs & 1u;
        if (handoffs >= 2) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(stat_free(slot), ((handoffs >> 1) - 1) & 1u, abort_flag));
          if (!ok) break;
        }
        ++handoffs;
        stat[(slot * 3 + half) * kBM + r] = l_run;
        if (half == 0) stat[(slot * 3 + 2) * kBM + r] = m_run;
        warp_arrive(epi_go(slot));
        if (a) pv_base1 += static_cast<uint32_t>(n); else pv_base0 += static_cast<uint32_t>(n);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) write_status(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == kRopeMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gdla
