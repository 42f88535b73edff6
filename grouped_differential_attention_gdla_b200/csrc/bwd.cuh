// bwd.cuh - GDLA attention backward, sm_100a.
//
// The model is trained with GDLA ("Вышла новая модель Motif 3", pikabu.ru);
// the backward is the gradient of the forward of "Motif 3: Technical Report"
// (paper.rainbus.top), step 2, for an upstream gradient dO of the output:
//   dG[h] = dO[h] (.) D[h],    dD[h] = dO[h] (.) G[h]
//   dlambda[h] = -sum_c dD[h][c] H_N[h/g][c]
//   dH_S[h] = dD[h],           dH_N[n] = -sum_{h/g = n} lambda[h] dD[h]
// and per head x (upstream dH_x): P = softmax(scale Q K^T + mask),
//   dP = dH_x V^T,  Delta_i = sum_j P_ij dP_ij = dH_x[i] . H_x[i],
//   dS = P (.) (dP - Delta),  dQ_x = scale dS K,
//   dK += scale dS^T Q_x,     dV += P^T dH_x       (every head of the group)
//
// Four launches (host: gdla_bwd.cu):
//   1. the forward in save mode (attn_rope.cuh): H of every head (fp32) and
//      its log-sum-exp (log2 units of the scaled scores);
//   2. gdla_bwd_prep_kernel (CUDA cores): dG, dlambda, dH of every head
//      (bf16, the MMA operand) and Delta;
//   3. gdla_bwd_dq_kernel (tcgen05, persistent): per (head, query block),
//      over the key tiles: S = Q K^T and dP = dH V^T in TMEM, P and dS by two
//      warpgroups (half the key columns each), dQ += dS K with dS read from
//      TMEM; the next tile's S and dP overlap the current tile's dS;
//   4. gdla_bwd_dkdv_kernel (tcgen05): per (KV group, key block), over the
//      group's g+1 heads and their query blocks: S^T = K Q^T and
//      dP^T = V dH^T in TMEM, P^T and dS^T per key row, dV += P^T dH and
//      dK += dS^T Q with both A operands read from TMEM; the next tile's
//      dP^T overlaps the current tile's P^T and dS^T.
// The softmax statistics come from step 1, so neither kernel needs a running
// maximum, and the two warpgroups that share a row never wait on each other:
// each writes its packed bf16 operands into TMEM columns of its own half of
// the tile, over columns it has already read.
#pragma once

#include "attn_rope.cuh"

namespace gdla {

constexpr int kBwdThreads = 16 * 32;
constexpr int kBwdProducerWarp = 12;
constexpr int kBwdMmaWarp = 13;
constexpr int kBwdMaxGroup = 8;  // signal heads per KV group the prep kernel takes

struct BwdParams {
  const __nv_bfloat16 *lam;   // [B, T, Hs]
  const __nv_bfloat16 *gate;  // [B, T, Hs*d]
  const __nv_bfloat16 *dout;  // [B, T, Hs*d]
  __nv_bfloat16 *dq_sig;      // [B, T, Hs, d]
  __nv_bfloat16 *dq_noise;    // [B, T, Hn, d]
  __nv_bfloat16 *dk;          // [B, T, Hkv, d]
  __nv_bfloat16 *dv;          // [B, T, Hkv, d]
  __nv_bfloat16 *dlam;        // [B, T, Hs]
  __nv_bfloat16 *dgate;       // [B, T, Hs*d]
  const float *h;             // workspace: H [B, T, Hs+Hn, d]
  const float *lse;           // workspace: [B, Hs+Hn, tp]
  float *delta;               // workspace: [B, Hs+Hn, tp]
  __nv_bfloat16 *dox;         // workspace: dH [B, T, Hs+Hn, d]
  int *status;
  int B, T, tp, Hs, Hn, g, n_qblk, n_kblk;
  int64_t window;  // 0 = full
  int causal;
  float scale, scale_log2;
};

// Non-tensor bulk copy global -> shared, completion on `bar` (no multicast).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// TMEM column (relative to the packed tile's base) of the bf16 pairs for
// keys (or queries) 16k .. 16k+15: the two warpgroups pack their halves at
// columns 0..31 and 64..95.
__device__ __forceinline__ uint32_t split_col(int k) { return 8u * k + (k >= 4 ? 32u : 0u); }

// ---------------------------------------------------------------- prep
// One warp per (token row, KV group k), four per CTA; lane l owns columns
// [CPL l, CPL l + CPL) with CPL = D / 32.  Per signal head h of the group:
// dG, dD (bf16, the dQ/dK/dV operand), dlambda and Delta_h = dD . H_S; then
// dH_N = -sum lambda dD and Delta_N = dH_N . H_N.  Delta uses the
// bf16-rounded dH the MMAs will read, so that sum_j dS_ij stays zero for the
// gradients the kernels form.
template <int D>
__device__ __forceinline__ void load_f32(const float *src, float (&v)[D / 32]) {
  if constexpr (D / 32 == 4) {
    const float4 t = *reinterpret_cast<const float4 *>(src);
    v[0] = t.x, v[1] = t.y, v[2] = t.z, v[3] = t.w;
  } else {
    const float2 t = *reinterpret_cast<const float2 *>(src);
    v[0] = t.x, v[1] = t.y;
  }
}
template <int D>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16 *src, float (&v)[D / 32]) {
  if constexpr (D / 32 == 4) {
    const uint2 t = *reinterpret_cast<const uint2 *>(src);
    v[0] = bf16lo_to_f32(t.x), v[1] = bf16hi_to_f32(t.x);
    v[2] = bf16lo_to_f32(t.y), v[3] = bf16hi_to_f32(t.y);
  } else {
    const uint32_t t = *reinterpret_cast<const uint32_t *>(src);
    v[0] = bf16lo_to_f32(t), v[1] = bf16hi_to_f32(t);
  }
}
// Rounds v to bf16, stores it, and returns the rounded values in v.
template <int D>
__device__ __forceinline__ void store_bf16(__nv_bfloat16 *dst, float (&v)[D / 32]) {
  if constexpr (D / 32 == 4) {
    const uint2 t = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    *reinterpret_cast<uint2 *>(dst) = t;
    v[0] = bf16lo_to_f32(t.x), v[1] = bf16hi_to_f32(t.x);
    v[2] = bf16lo_to_f32(t.y), v[3] = bf16hi_to_f32(t.y);
  } else {
    const uint32_t t = pack_bf16x2(v[0], v[1]);
    *reinterpret_cast<uint32_t *>(dst) = t;
    v[0] = bf16lo_to_f32(t), v[1] = bf16hi_to_f32(t);
  }
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kPrepWarps = 4;  // (token, group) pairs per CTA of the prep kernel

template <int D>
__global__ void __launch_bounds__(32 * kPrepWarps) gdla_bwd_prep_kernel(const BwdParams p) {
  constexpr int CPL = D / 32;
  const int64_t pair = static_cast<int64_t>(blockIdx.x) * kPrepWarps + (threadIdx.x >> 5);
  if (pair >= static_cast<int64_t>(p.B) * p.T * p.Hn) return;
  const int64_t row = pair / p.Hn;
  const int k = static_cast<int>(pair % p.Hn);
  const int lane = threadIdx.x & 31, c = CPL * lane;
  const int g = p.g, H80 = p.Hs + p.Hn;
  const int64_t b = row / p.T, i = row % p.T;
  float hn[CPL], dhn[CPL];
  load_f32<D>(p.h + (row * H80 + p.Hs + k) * D + c, hn);
#pragma unroll
  for (int e = 0; e < CPL; ++e) dhn[e] = 0.f;
  for (int j = 0; j < g; ++j) {
    const int h = g * k + j;
    const int64_t oc = (row * p.Hs + h) * D + c;
    const float lam = __bfloat162float(p.lam[row * p.Hs + h]);
    float hs[CPL], go[CPL], gt[CPL], dg[CPL], dd[CPL];
    load_f32<D>(p.h + (row * H80 + h) * D + c, hs);
    load_bf16<D>(p.dout + oc, go);
    load_bf16<D>(p.gate + oc, gt);
    float dlam = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) {
      dd[e] = go[e] * gt[e];
      dg[e] = go[e] * (hs[e] - lam * hn[e]);
      dhn[e] -= lam * dd[e];
      dlam -= dd[e] * hn[e];
    }
    store_bf16<D>(p.dgate + oc, dg);
    store_bf16<D>(p.dox + (row * H80 + h) * D + c, dd);  // dd now holds the rounded dD
    float delta = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) delta += dd[e] * hs[e];
    dlam = warp_sum(dlam);
    delta = warp_sum(delta);
    if (lane == 0) {
      p.dlam[row * p.Hs + h] = __float2bfloat16(dlam);
      p.delta[(b * H80 + h) * p.tp + i] = delta;
    }
  }
  store_bf16<D>(p.dox + (row * H80 + p.Hs + k) * D + c, dhn);
  float dn = 0.f;
#pragma unroll
  for (int e = 0; e < CPL; ++e) dn += dhn[e] * hn[e];
  dn = warp_sum(dn);
  if (lane == 0) p.delta[(b * H80 + p.Hs + k) * p.tp + i] = dn;
}

// ---------------------------------------------------------------- dQ
template <int D>
struct DqSmemLayout {
  static constexpr uint32_t kSub = kBM * 128;        // [128][64] bf16 swizzled
  static constexpr uint32_t kTile = (D / 64) * kSub;  // [128][D]
  // K/V ring (K_t, V_t alternate); K_t is held until dQ(t), so five stages
  // let K_{t+2} load while K_t and both tiles of t+1 are resident
  static constexpr uint32_t kStages = 5;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kDoOff = kQOff + kTile;
  static constexpr uint32_t kRingOff = kDoOff + kTile;
  static constexpr uint32_t kBarOff = kRingOff + kStages * kTile;
  // qd_full kv_full[S] kv_empty[S] s_full p_full[2] dp_free dq_done qd_free dq_free
  static constexpr uint32_t kNumBars = 1 + 2 * kStages + 7;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
};

// A dQ item: (batch b, head x of Hs + Hn, query block), heaviest blocks
// first in item order; its key tiles j_lo .. j_lo + n - 1.
struct DqItem {
  int b, x, kvh, q0, j_lo, n;
  bool noise;
};

__device__ __forceinline__ DqItem dq_item(const BwdParams &p, int item) {
  const int H80 = p.Hs + p.Hn;
  DqItem it;
  const int qb = p.n_qblk - 1 - item / (p.B * H80);
  const int rest = item % (p.B * H80);
  it.b = rest / H80;
  it.x = rest % H80;
  it.noise = it.x >= p.Hs;
  it.kvh = it.noise ? it.x - p.Hs : it.x / p.g;
  it.q0 = qb * kBM;
  int j_hi;
  it.j_lo = 0;
  if (p.causal) {
    j_hi = min(it.q0 + kBM - 1, p.T - 1) / kBN;
    if (p.window > 0) {
      const int64_t first = static_cast<int64_t>(it.q0) - p.window + 1;
      it.j_lo = first > 0 ? static_cast<int>(first / kBN) : 0;
    }
  } else {
    j_hi = (p.T - 1) / kBN;
  }
  it.n = j_hi - it.j_lo + 1;
  return it;
}

// Persistent: CTA c takes items c, c + gridDim.x, ...; the tile pipeline
// (ring positions, S buffers, barrier phases) runs on across items.
// Warps 0-7: P and dS (warpgroup `half` takes key columns [64 half,
// 64 half + 64)); 8-11: dQ epilogue; 12: TMA; 13: TMEM and MMA.
// TMEM: S of even tiles [0,128) and of odd tiles [384,512) (dS packed over
// each), dP [128,256), dQ [256, 256+D).  The MMA warp computes S(t+1) while
// the elementwise warps work on tile t, and dP(t+1) as soon as they have
// read dP(t) (half-way through the tile); the next tile may be the first of
// the next item, whose Q and dH load as soon as the last S and dP MMAs of
// the current item have read theirs.  An item's first dQ MMA waits for the
// epilogue to have read the previous item's dQ.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    gdla_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_qs,
                       const __grid_constant__ CUtensorMap tm_qn,
                       const __grid_constant__ CUtensorMap tm_dox,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const BwdParams p) {
  using L = DqSmemLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) write_status(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t qd_full = bar0;
  auto kv_full = [&](uint32_t s) { return bar0 + 8u * (1 + s); };
  auto kv_empty = [&](uint32_t s) { return bar0 + 8u * (1 + L::kStages + s); };
  const uint32_t s_full = bar0 + 8u * (1 + 2 * L::kStages);
  auto p_full = [&](uint32_t t) { return s_full + 8u * (1 + (t & 1u)); };  // dS(t) packed
  const uint32_t dp_free = s_full + 24u;  // dP(t) read out by every elementwise warp
  const uint32_t dq_done = s_full + 32u;  // an item's dQ complete
  const uint32_t qd_free = s_full + 40u;  // an item's last S and dP have read Q and dH
  const uint32_t dq_free = s_full + 48u;  // the epilogue has read an item's dQ
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  const int warp = threadIdx.x >> 5;
  const int H80 = p.Hs + p.Hn;
  const int n_items = p.n_qblk * p.B * H80;
  const int G = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (uint32_t s = 0; s < L::kStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full(0), 8);
    mbar_init(p_full(1), 8);
    mbar_init(dp_free, 8);
    mbar_init(dq_done, 1);
    mbar_init(qd_free, 1);
    mbar_init(dq_free, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_dp = tmem + 128u, t_dq = tmem + 256u;
  auto t_s = [&](uint32_t t) { return tmem + ((t & 1u) ? 384u : 0u); };

  if (warp == kBwdProducerWarp) {
    // =============================== TMA: per item Q_x and dH_x, then K_t, V_t per tile
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    uint32_t c = 0, ik = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += G, ++ik) {
      const DqItem it = dq_item(p, item);
      if (ik > 0) {  // the previous item's last S and dP have read Q and dH
        ok = __all_sync(0xffffffffu, mbar_wait(qd_free, (ik - 1) & 1u, abort_flag));
        if (!ok) break;
      }
      if (leader) {
        mbar_arrive_expect_tx(qd_full, 2 * L::kTile);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          const int head = it.noise ? it.kvh : it.x;
          tma_load_3d(sbase + L::kQOff + kb * L::kSub, it.noise ? &tm_qn : &tm_qs, qd_full,
                      head * D + kb * 64, it.q0, it.b);
          tma_load_3d(sbase + L::kDoOff + kb * L::kSub, &tm_dox, qd_full, it.x * D + kb * 64,
                      it.q0, it.b);
        }
      }
      for (int t = 0; t < it.n && ok; ++t) {
        for (int kv = 0; kv < 2 && ok; ++kv) {
          const uint32_t s = c % L::kStages;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(kv_empty(s), ((c / L::kStages) & 1u) ^ 1u, abort_flag));
          if (!ok) break;
          if (leader) {
            mbar_arrive_expect_tx(kv_full(s), L::kTile);
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(sbase + L::kRingOff + s * L::kTile + kb * L::kSub, kv ? &tm_v : &tm_k,
                          kv_full(s), it.kvh * D + kb * 64, (it.j_lo + t) * kBN, it.b);
          }
          ++c;
        }
      }
    }
    if (!ok && leader) {
      for (uint32_t s = 0; s < L::kStages; ++s) {
        const uint32_t issued = c > s ? (c - 1 - s) / L::kStages + 1 : 0;
        if (issued) mbar_wait_for(kv_full(s), (issued - 1) & 1u, 100000000ull);
      }
      // the Q and dH of the last item this warp armed
      if (ik > 0 || blockIdx.x < static_cast<unsigned>(n_items))
        mbar_wait_for(qd_full, ik & 1u, 100000000ull);
    }
  } else if (warp == kBwdMmaWarp) {
    // =============================== MMA: S(T+1) and dP(T+1) ahead of dQ += dS(T) K_T
    // (T counts this CTA's tiles; the ring holds K_T, V_T at positions 2T, 2T+1)
    const bool leader = elect_one();
    constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t kIdescQ = idesc_bf16_f32(kBM, D, false, true);
    const uint64_t qd = sdesc_sw128(sbase + L::kQOff, 16, 1024);
    const uint64_t dod = sdesc_sw128(sbase + L::kDoOff, 16, 1024);
    auto slot = [&](uint32_t pos) { return pos % L::kStages; };
    auto wait_full = [&](uint32_t pos) {
      return __all_sync(0xffffffffu,
                        mbar_wait(kv_full(slot(pos)), (pos / L::kStages) & 1u, abort_flag));
    };
    auto tile = [&](uint32_t pos) { return sbase + L::kRingOff + slot(pos) * L::kTile; };
    // S(T) = Q K_T^T into T's S buffer (K-major operands, D/16 K-steps)
    auto issue_s = [&](uint32_t T) {
      if (!leader) return;
      const uint64_t kd = sdesc_sw128(tile(2u * T), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * L::kSub + (k & 3) * 32;
        umma_ss(t_s(T), qd + (off >> 4), kd + (off >> 4), kIdescS, k > 0 ? 1u : 0u);
      }
    };
    // dP(T) = dH V_T^T, then S(T) and dP(T) are announced and V_T released;
    // after an item's last tile its Q and dH are released too
    auto issue_dp = [&](uint32_t T, bool last_of_item) {
      if (!leader) return;
      const uint64_t vd = sdesc_sw128(tile(2u * T + 1u), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * L::kSub + (k & 3) * 32;
        umma_ss(t_dp, dod + (off >> 4), vd + (off >> 4), kIdescS, k > 0 ? 1u : 0u);
      }
      umma_commit(s_full);
      umma_commit(kv_empty(slot(2u * T + 1u)));
      if (last_of_item) umma_commit(qd_free);
    };
    bool ok = true;
    uint32_t T = 0, dq_commits = 0;
    int item = blockIdx.x, t = 0;
    uint32_t ik = 0;
    DqItem it{};
    if (item < n_items) {
      it = dq_item(p, item);
      ok = __all_sync(0xffffffffu, mbar_wait(qd_full, 0, abort_flag)) && wait_full(0) &&
           wait_full(1);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0, it.n == 1);
      }
    } else {
      ok = false;
    }
    while (ok) {
      // the next tile: t + 1 of this item, or the first of the next item
      int n_item = item, n_t = t + 1;
      uint32_t n_ik = ik;
      DqItem nit = it;
      if (n_t >= it.n) {
        n_item = item + G;
        n_t = 0;
        n_ik = ik + 1;
        if (n_item < n_items) nit = dq_item(p, n_item);
      }
      const bool has_next = n_item < n_items;
      if (has_next) {
        if (n_t == 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(qd_full, n_ik & 1u, abort_flag));
          if (!ok) break;
        }
        ok = wait_full(2u * (T + 1)) && wait_full(2u * (T + 1) + 1u);
        if (!ok) break;
        tc_fence_after();
        issue_s(T + 1);  // its buffer last held dS(T-1), read by the dQ MMA issued before
        ok = __all_sync(0xffffffffu, mbar_wait(dp_free, T & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        issue_dp(T + 1, n_t == nit.n - 1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(p_full(T), (T >> 1) & 1u, abort_flag));
      if (!ok) break;
      if (t == 0 && ik > 0) {  // the epilogue has read the previous item's dQ
        ok = __all_sync(0xffffffffu, mbar_wait(dq_free, (ik - 1) & 1u, abort_flag));
        if (!ok) break;
      }
      tc_fence_after();
      // dQ += dS K_T: A = dS (TMEM, packed halves), B = K_T MN-major over d
      if (leader) {
        const uint64_t kmn = sdesc_sw128(tile(2u * T), kBN * 128, 1024);
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k)
          umma_ts(t_dq, t_s(T) + split_col(k), kmn + ((k * (16 * 128)) >> 4), kIdescQ,
                  (t > 0 || k > 0) ? 1u : 0u);
        umma_commit(kv_empty(slot(2u * T)));
        if (t == it.n - 1) umma_commit(dq_done);
      }
      if (t == it.n - 1) ++dq_commits;
      if (!has_next) break;
      item = n_item;
      t = n_t;
      ik = n_ik;
      it = nit;
      ++T;
    }
    if (leader && dq_commits) mbar_wait_for(dq_done, (dq_commits - 1) & 1u, 100000000ull);
  } else if (warp >= 8 && warp < 12) {
    // =============================== epilogue: dQ_x = scale * (dS K), bf16 rows, per item
    const int wq = warp & 3;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    bool ok = true;
    uint32_t ik = 0;
    for (int item = blockIdx.x; item < n_items && ok; item += G, ++ik) {
      const DqItem it = dq_item(p, item);
      ok = __all_sync(0xffffffffu, mbar_wait(dq_done, ik & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const int i = it.q0 + r;
      __nv_bfloat16 *dst =
          it.noise ? p.dq_noise + ((static_cast<int64_t>(it.b) * p.T + i) * p.Hn + it.kvh) * D
                   : p.dq_sig + ((static_cast<int64_t>(it.b) * p.T + i) * p.Hs + it.x) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32_sync(t_dq + lane_off + cc * 32, v);
        if (i < p.T) {
          uint4 *op = reinterpret_cast<uint4 *>(dst + cc * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            op[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]) * p.scale,
                                           __uint_as_float(v[8 * q + 1]) * p.scale),
                               pack_bf16x2(__uint_as_float(v[8 * q + 2]) * p.scale,
                                           __uint_as_float(v[8 * q + 3]) * p.scale),
                               pack_bf16x2(__uint_as_float(v[8 * q + 4]) * p.scale,
                                           __uint_as_float(v[8 * q + 5]) * p.scale),
                               pack_bf16x2(__uint_as_float(v[8 * q + 6]) * p.scale,
                                           __uint_as_float(v[8 * q + 7]) * p.scale));
        }
      }
      tc_fence_before();
      warp_arrive(dq_free);
    }
  } else if (warp < 8) {
    // =============================== P and dS, half a row per warpgroup
    const int half = warp >> 2, wq = warp & 3;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    uint32_t T = 0;
    for (int item = blockIdx.x; item < n_items && ok; item += G) {
      const DqItem it = dq_item(p, item);
      const int i = it.q0 + r;
      const bool row_ok = i < p.T;
      const int64_t srow = (static_cast<int64_t>(it.b) * H80 + it.x) * p.tp + i;
      const float lse = row_ok ? p.lse[srow] : 0.f;
      const float dl = row_ok ? p.delta[srow] : 0.f;
      for (int t = 0; t < it.n && ok; ++t, ++T) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full, T & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t ts = t_s(T);
        const int kbase = (it.j_lo + t) * kBN;
        int c_lo, c_hi;  // kept key columns of this row in the tile
        if (p.causal) {
          c_hi = i - kbase;
          c_lo = p.window > 0 ? static_cast<int>(static_cast<int64_t>(i) - p.window + 1 - kbase)
                              : -1;
        } else {
          c_hi = p.T - 1 - kbase;
          c_lo = -1;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cc = 2 * half + u;  // 32-column chunk of the tile
          uint32_t sv[32], dpv[32];
          tmem_ld32x2_sync(ts + lane_off + 32 * cc, t_dp + lane_off + 32 * cc, sv, dpv);
          if (u == 1) {  // this warp has read its whole dP(T): dP(T+1) may overwrite it
            tc_fence_before();
            warp_arrive(dp_free);
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = 32 * cc + 2 * e;
            const bool k0 = row_ok && c0 >= c_lo && c0 <= c_hi;
            const bool k1 = row_ok && c0 + 1 >= c_lo && c0 + 1 <= c_hi;
            const float p0 = k0 ? ex2_approx(__uint_as_float(sv[2 * e]) * sl2 - lse) : 0.f;
            const float p1 = k1 ? ex2_approx(__uint_as_float(sv[2 * e + 1]) * sl2 - lse) : 0.f;
            pk[e] = pack_bf16x2(p0 * (__uint_as_float(dpv[2 * e]) - dl),
                                p1 * (__uint_as_float(dpv[2 * e + 1]) - dl));
          }
          // dS of this chunk, packed into this half's own S columns
          tmem_st16(ts + lane_off + 64 * half + 16 * u, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        warp_arrive(p_full(T));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) write_status(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK, dV
template <int D>
struct DkdvSmemLayout {
  static constexpr uint32_t kSub = kBM * 128;
  static constexpr uint32_t kTile = (D / 64) * kSub;
  static constexpr uint32_t kQStages = 2;   // Q_x of a query block, then its lse[128], Delta[128]
  static constexpr uint32_t kDhStages = 3;  // dH_x of a query block
  static constexpr uint32_t kStatBytes = 2 * kBM * 4;
  static constexpr uint32_t kQEntry = kTile + 1024;
  static constexpr uint32_t kKOff = 0;
  static constexpr uint32_t kVOff = kKOff + kTile;
  static constexpr uint32_t kQOff = kVOff + kTile;
  static constexpr uint32_t kDhOff = kQOff + kQStages * kQEntry;
  static constexpr uint32_t kBarOff = kDhOff + kDhStages * kTile;
  // kv_full q_full[2] q_empty[2] dh_full[3] dh_empty[3] s_full p_full dp_free acc_done
  static constexpr uint32_t kNumBars = 1 + 2 * kQStages + 2 * kDhStages + 4;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
};

// The query blocks that reach key block kb (tokens kb*128 .. kb*128+127).
__device__ __forceinline__ void dkdv_qrange(const BwdParams &p, int kb, int &qlo, int &qhi) {
  if (!p.causal) {
    qlo = 0;
    qhi = p.n_qblk - 1;
    return;
  }
  qlo = kb;  // queries at or after the key
  qhi = p.n_qblk - 1;
  if (p.window > 0) {
    // the last query that keeps key kb*128 + 127 is kb*128 + 127 + W - 1
    const int64_t last = static_cast<int64_t>(kb) * kBN + kBN - 1 + p.window - 1;
    const int64_t lb = last / kBM;
    if (lb < qhi) qhi = static_cast<int>(lb);
  }
}

// One CTA per (batch b, KV group k, key block kb), heaviest (earliest) key
// blocks first.  Warps 0-7: P^T and dS^T (warpgroup `half` takes query
// columns [64 half, 64 half + 64)); 8-11: dK, dV epilogue; 12: TMA;
// 13: TMEM and MMA.  TMEM: S^T [0,128), dP^T [128,256), dV [256, 256+D),
// dK [256+D, 256+2D).  Each 32-column chunk of S^T is overwritten by its own
// P^T (16 columns of bf16 pairs) and dS^T (the next 16), so dP^T is free as
// soon as the elementwise warps have read it and the MMA warp computes the
// next tile's dP^T while they work.  K and V stay in shared memory; Q (with
// the block's lse and Delta rows) and dH stream through rings of two and
// three entries.
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    gdla_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_qs,
                         const __grid_constant__ CUtensorMap tm_qn,
                         const __grid_constant__ CUtensorMap tm_dox,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const BwdParams p) {
  using L = DkdvSmemLayout<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) write_status(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t kv_full = bar0;
  auto q_full = [&](uint32_t s) { return bar0 + 8u * (1 + s); };
  auto q_empty = [&](uint32_t s) { return bar0 + 8u * (1 + L::kQStages + s); };
  auto dh_full = [&](uint32_t s) { return bar0 + 8u * (1 + 2 * L::kQStages + s); };
  auto dh_empty = [&](uint32_t s) { return bar0 + 8u * (1 + 2 * L::kQStages + L::kDhStages + s); };
  const uint32_t s_full = bar0 + 8u * (1 + 2 * L::kQStages + 2 * L::kDhStages);
  const uint32_t p_full = s_full + 8u;
  const uint32_t dp_free = s_full + 16u;
  const uint32_t acc_done = s_full + 24u;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  const int warp = threadIdx.x >> 5;
  const int H80 = p.Hs + p.Hn;
  const int n_heads = p.g + 1;

  const int item = blockIdx.x;
  const int kb = item / (p.B * p.Hn);
  const int rest = item % (p.B * p.Hn);
  const int b = rest / p.Hn, kvh = rest % p.Hn;
  const int k0 = kb * kBN;
  int qlo, qhi;
  dkdv_qrange(p, kb, qlo, qhi);
  const int nq = qhi - qlo + 1;
  const int n_tiles = n_heads * nq;
  // head of tile number tt (noise head first, then the group's signal heads)
  auto tile_head = [&](int tt) {
    const int hh = tt / nq;
    return hh == 0 ? p.Hs + kvh : p.g * kvh + (hh - 1);
  };
  auto q_slot = [](int tt) { return static_cast<uint32_t>(tt) % L::kQStages; };
  auto q_par = [](int tt) { return (static_cast<uint32_t>(tt) / L::kQStages) & 1u; };
  auto dh_slot = [](int tt) { return static_cast<uint32_t>(tt) % L::kDhStages; };
  auto dh_par = [](int tt) { return (static_cast<uint32_t>(tt) / L::kDhStages) & 1u; };
  auto q_base = [&](int tt) { return sbase + L::kQOff + q_slot(tt) * L::kQEntry; };
  auto dh_base = [&](int tt) { return sbase + L::kDhOff + dh_slot(tt) * L::kTile; };

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (uint32_t s = 0; s < L::kQStages; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    for (uint32_t s = 0; s < L::kDhStages; ++s) {
      mbar_init(dh_full(s), 1);
      mbar_init(dh_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    mbar_init(dp_free, 8);
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kBwdMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem, t_dp = tmem + 128u;
  const uint32_t t_dv = tmem + 256u, t_dk = tmem + 256u + D;
  // TMEM column (from t_s) of the bf16 pairs of query K-step k (16 queries):
  // chunk 32 * (k / 2) of S^T, P^T in its first 16 columns, dS^T in the next
  auto pt_col = [](int k) -> uint32_t { return 32u * (k >> 1) + 8u * (k & 1); };

  if (warp == kBwdProducerWarp) {
    // =============================== TMA: K, V once; then per tile the
    // head's dH block, and its Q block with the lse and Delta rows
    const bool leader = elect_one();
    if (leader) {
      mbar_arrive_expect_tx(kv_full, 2 * L::kTile);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(sbase + L::kKOff + c * L::kSub, &tm_k, kv_full, kvh * D + c * 64, k0, b);
        tma_load_3d(sbase + L::kVOff + c * L::kSub, &tm_v, kv_full, kvh * D + c * 64, k0, b);
      }
    }
    bool ok = true;
    uint32_t q_issued = 0, dh_issued = 0;
    for (int tt = 0; tt < n_tiles && ok; ++tt) {
      const int xh = tile_head(tt);
      const int q0 = (qlo + tt % nq) * kBM;
      // dH first: its slot frees one tile earlier than Q's
      ok = __all_sync(0xffffffffu, mbar_wait(dh_empty(dh_slot(tt)), dh_par(tt) ^ 1u, abort_flag));
      if (!ok) break;
      if (leader) {
        mbar_arrive_expect_tx(dh_full(dh_slot(tt)), L::kTile);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(dh_base(tt) + c * L::kSub, &tm_dox, dh_full(dh_slot(tt)), xh * D + c * 64,
                      q0, b);
      }
      ++dh_issued;
      ok = __all_sync(0xffffffffu, mbar_wait(q_empty(q_slot(tt)), q_par(tt) ^ 1u, abort_flag));
      if (!ok) break;
      if (leader) {
        const uint32_t dst = q_base(tt);
        mbar_arrive_expect_tx(q_full(q_slot(tt)), L::kTile + L::kStatBytes);
        const bool noise = xh >= p.Hs;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(dst + c * L::kSub, noise ? &tm_qn : &tm_qs, q_full(q_slot(tt)),
                      (noise ? xh - p.Hs : xh) * D + c * 64, q0, b);
        const int64_t so = (static_cast<int64_t>(b) * H80 + xh) * p.tp + q0;
        bulk_load(dst + L::kTile, p.lse + so, kBM * 4, q_full(q_slot(tt)));
        bulk_load(dst + L::kTile + kBM * 4, p.delta + so, kBM * 4, q_full(q_slot(tt)));
      }
      ++q_issued;
    }
    if (!ok && leader) {
      for (uint32_t s = 0; s < L::kQStages; ++s) {
        const uint32_t n_s = q_issued > s ? (q_issued - 1 - s) / L::kQStages + 1 : 0;
        if (n_s) mbar_wait_for(q_full(s), (n_s - 1) & 1u, 100000000ull);
      }
      for (uint32_t s = 0; s < L::kDhStages; ++s) {
        const uint32_t n_s = dh_issued > s ? (dh_issued - 1 - s) / L::kDhStages + 1 : 0;
        if (n_s) mbar_wait_for(dh_full(s), (n_s - 1) & 1u, 100000000ull);
      }
      mbar_wait_for(kv_full, 0, 100000000ull);
    }
  } else if (warp == kBwdMmaWarp) {
    // =============================== MMA: S^T(t), dP^T(t); dP^T(t+1) once
    // dP^T(t) is read; dV += P^T dH, dK += dS^T Q; then S^T(t+1)
    const bool leader = elect_one();
    constexpr uint32_t kIdescS = idesc_bf16_f32(kBN, kBM, false, false);
    constexpr uint32_t kIdescA = idesc_bf16_f32(kBN, D, false, true);
    const uint64_t kd = sdesc_sw128(sbase + L::kKOff, 16, 1024);
    const uint64_t vd = sdesc_sw128(sbase + L::kVOff, 16, 1024);
    auto issue_st = [&](int tt) {  // S^T = K Q^T
      if (!leader) return;
      const uint64_t qdk = sdesc_sw128(q_base(tt), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * L::kSub + (k & 3) * 32;
        umma_ss(t_s, kd + (off >> 4), qdk + (off >> 4), kIdescS, k > 0 ? 1u : 0u);
      }
    };
    auto issue_dpt = [&](int tt) {  // dP^T = V dH^T
      if (!leader) return;
      const uint64_t dodk = sdesc_sw128(dh_base(tt), 16, 1024);
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = (k >> 2) * L::kSub + (k & 3) * 32;
        umma_ss(t_dp, vd + (off >> 4), dodk + (off >> 4), kIdescS, k > 0 ? 1u : 0u);
      }
    };
    auto wait_q = [&](int tt) {
      return __all_sync(0xffffffffu, mbar_wait(q_full(q_slot(tt)), q_par(tt), abort_flag));
    };
    auto wait_dh = [&](int tt) {
      return __all_sync(0xffffffffu, mbar_wait(dh_full(dh_slot(tt)), dh_par(tt), abort_flag));
    };
    bool ok = __all_sync(0xffffffffu, mbar_wait(kv_full, 0, abort_flag));
    bool done = false;
    if (ok && n_tiles > 0) ok = wait_q(0) && wait_dh(0);
    if (ok && n_tiles > 0) {
      tc_fence_after();
      issue_st(0);
      issue_dpt(0);
      if (leader) umma_commit(s_full);
    }
    for (int tt = 0; tt < n_tiles && ok; ++tt) {
      if (tt + 1 < n_tiles) {
        ok = wait_dh(tt + 1);
        if (!ok) break;
        ok = __all_sync(0xffffffffu, mbar_wait(dp_free, static_cast<uint32_t>(tt) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        issue_dpt(tt + 1);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(p_full, static_cast<uint32_t>(tt) & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        // B operands MN-major over d: dH_x and Q_x, 16 query rows per K-step
        const uint64_t domn = sdesc_sw128(dh_base(tt), kBM * 128, 1024);
        const uint64_t qmn = sdesc_sw128(q_base(tt), kBM * 128, 1024);
#pragma unroll
        for (int k = 0; k < kBM / 16; ++k)
          umma_ts(t_dv, t_s + pt_col(k), domn + ((k * (16 * 128)) >> 4), kIdescA,
                  (tt > 0 || k > 0) ? 1u : 0u);
        umma_commit(dh_empty(dh_slot(tt)));
#pragma unroll
        for (int k = 0; k < kBM / 16; ++k)
          umma_ts(t_dk, t_s + pt_col(k) + 16u, qmn + ((k * (16 * 128)) >> 4), kIdescA,
                  (tt > 0 || k > 0) ? 1u : 0u);
        umma_commit(q_empty(q_slot(tt)));
        if (tt == n_tiles - 1) umma_commit(acc_done);
      }
      if (tt == n_tiles - 1) done = true;
      if (tt + 1 < n_tiles) {
        ok = wait_q(tt + 1);
        if (!ok) break;
        tc_fence_after();
        issue_st(tt + 1);  // over the P^T, dS^T columns the MMAs above read (issue order)
        if (leader) umma_commit(s_full);
      }
    }
    if (leader && done) mbar_wait_for(acc_done, 0, 100000000ull);
  } else if (warp >= 8 && warp < 12) {
    // =============================== epilogue: dK = scale * sum dS^T Q, dV
    const int wq = warp & 3;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int j = k0 + r;
    bool ok = __all_sync(0xffffffffu, mbar_wait(acc_done, 0, abort_flag));
    if (ok) {
      tc_fence_after();
      const int64_t off = ((static_cast<int64_t>(b) * p.T + j) * p.Hn + kvh) * D;
#pragma unroll
      for (int w2 = 0; w2 < 2; ++w2) {
        const uint32_t src = w2 == 0 ? t_dk : t_dv;
        const float f = w2 == 0 ? p.scale : 1.f;
        __nv_bfloat16 *dst = (w2 == 0 ? p.dk : p.dv) + off;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32_sync(src + lane_off + cc * 32, v);
          if (j < p.T) {
            uint4 *op = reinterpret_cast<uint4 *>(dst + cc * 32);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              op[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]) * f,
                                             __uint_as_float(v[8 * q + 1]) * f),
                                 pack_bf16x2(__uint_as_float(v[8 * q + 2]) * f,
                                             __uint_as_float(v[8 * q + 3]) * f),
                                 pack_bf16x2(__uint_as_float(v[8 * q + 4]) * f,
                                             __uint_as_float(v[8 * q + 5]) * f),
                                 pack_bf16x2(__uint_as_float(v[8 * q + 6]) * f,
                                             __uint_as_float(v[8 * q + 7]) * f));
          }
        }
      }
    }
  } else if (warp < 8) {
    // =============================== P^T and dS^T, half the query columns each
    const int half = warp >> 2, wq = warp & 3;
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int j = k0 + r;  // key token of this row
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int tt = 0; tt < n_tiles && ok; ++tt) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, static_cast<uint32_t>(tt) & 1u, abort_flag));
      // the block's lse and Delta rows came by bulk copy with Q: observe that
      // barrier too (complete already; the entry is not reloaded before this
      // tile's dK MMA, which waits for these warps)
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(q_full(q_slot(tt)), q_par(tt), abort_flag));
      if (!ok) break;
      tc_fence_after();
      const float *lse = reinterpret_cast<const float *>(smem + L::kQOff + q_slot(tt) * L::kQEntry +
                                                         L::kTile);
      const float *dlt = lse + kBM;
      const int q0 = (qlo + tt % nq) * kBM;
      // query columns c of this tile that keep key j
      int c_lo, c_hi;
      if (p.causal) {
        c_lo = j - q0;  // queries at or after the key
        c_hi = p.window > 0 ? static_cast<int>(static_cast<int64_t>(j) + p.window - 1 - q0) : kBM;
        c_hi = min(c_hi, p.T - 1 - q0);
      } else {
        c_lo = 0;
        c_hi = p.T - 1 - q0;
      }
      if (j >= p.T) c_hi = -1;  // padding key rows keep nothing
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int cc = 2 * half + u;
        uint32_t sv[32], dpv[32];
        tmem_ld32x2_sync(t_s + lane_off + 32 * cc, t_dp + lane_off + 32 * cc, sv, dpv);
        if (u == 1) {  // this warp has read its whole dP^T: the next tile's may land
          tc_fence_before();
          warp_arrive(dp_free);
        }
        uint32_t pk[16], dk[16];
        // the chunk's lse and Delta values, four columns per shared-memory read
        const float4 *lse4 = reinterpret_cast<const float4 *>(lse + 32 * cc);
        const float4 *dlt4 = reinterpret_cast<const float4 *>(dlt + 32 * cc);
#pragma unroll
        for (int e2 = 0; e2 < 8; ++e2) {
          const float4 l4 = lse4[e2], d4 = dlt4[e2];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
          const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = 2 * e2 + h2;
            const int c0 = 32 * cc + 2 * e;
            const bool a0 = c0 >= c_lo && c0 <= c_hi;
            const bool a1 = c0 + 1 >= c_lo && c0 + 1 <= c_hi;
            const float p0 = a0 ? ex2_approx(__uint_as_float(sv[2 * e]) * sl2 - lv[2 * h2]) : 0.f;
            const float p1 =
                a1 ? ex2_approx(__uint_as_float(sv[2 * e + 1]) * sl2 - lv[2 * h2 + 1]) : 0.f;
            pk[e] = pack_bf16x2(p0, p1);
            // selected, not multiplied: a masked column's lse and Delta may be
            // the unwritten padding past T
            dk[e] = pack_bf16x2(a0 ? p0 * (__uint_as_float(dpv[2 * e]) - dv[2 * h2]) : 0.f,
                                a1 ? p1 * (__uint_as_float(dpv[2 * e + 1]) - dv[2 * h2 + 1]) : 0.f);
          }
        }
        // P^T and dS^T over this chunk's own S^T columns (already read)
        tmem_st16(t_s + lane_off + 32 * cc, pk);
        tmem_st16(t_s + lane_off + 32 * cc + 16, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      warp_arrive(p_full);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) write_status(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gdla
