// attn_fwd.cuh - fused GDLA attention forward for sm_100a.
//
// Operation ("Motif 3: Technical Report", paper.rainbus.top, step 2 "GDLA
// forward"): for KV group k the noise head n = k and the g signal heads
// h = g*k .. g*k+g-1 attend over the shared KV head k;
//   D[h] = H_S[h] - lambda[h] * H_N[h / g],   O[h] = G[h] * D[h].
//
// One CTA owns one (batch b, KV group k, block of 128 query tokens).  It runs
// the g+1 heads of the group in phases of two "slots" (A, B): phase 0 is
// (noise, signal 0), then (signal 1, signal 2), ...  Both slots of a phase
// share the same query rows and therefore every K/V tile the TMA warp brings
// into shared memory.  Per KV tile of 128 keys:
//   S_X  = Q_X K^T          tcgen05.mma, A = Q (smem), B = K (smem), D = TMEM
//   P_X  = exp2(S_X*c - m)  softmax warpgroup X: tcgen05.ld, online max/sum,
//                           bf16 P written back over S_X with tcgen05.st
//   O_X += P_X V            tcgen05.mma, A = P (TMEM), B = V (smem)
// The noise head's normalised output H_N goes to shared memory (fp32) and is
// subtracted in the epilogue of every signal head of the group; neither H_S
// nor H_N is written to global memory.
//
// Warp roles (320 threads):
//   warps 0-3  softmax + epilogue for slot A (TMEM lanes 0..127)
//   warps 4-7  softmax + epilogue for slot B
//   warp  8    TMA producer (Q tiles, K/V ring)
//   warp  9    TMEM allocator and single-thread MMA issuer
//
// TMEM (512 columns): S_A [0,128) S_B [128,256) O_A [256,256+d) O_B [256+d, 256+2d).
// P_X occupies the first 64 columns of S_X as packed bf16 pairs.
#pragma once

#include "sm100.cuh"

namespace gdla {

constexpr int kBM = 128;          // query rows per slot
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kKvStages = 3;      // K/V ring depth (tiles)
constexpr int kAttnThreads = 320;
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
  int64_t window;  // 0 = full
  int causal;
  float scale_log2;  // softmax scale * log2(e)
};

template <int D>
struct AttnSmemLayout {
  static constexpr uint32_t kQBytes = kBM * D * 2;
  static constexpr uint32_t kKvBytes = kBN * D * 2;
  static constexpr uint32_t kHnBytes = kBM * D * 4;
  static constexpr uint32_t kQOff = 0;
  static constexpr uint32_t kKvOff = kQOff + 2 * kQBytes;
  static constexpr uint32_t kHnOff = kKvOff + kKvStages * kKvBytes;
  static constexpr uint32_t kBarOff = kHnOff + kHnBytes;
  // barriers: q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] p_full[2]
  //           o_done[2] o_free[2] hn_ready
  static constexpr uint32_t kNumBars = 2 + 2 + 2 * kKvStages + 2 + 2 + 2 + 2 + 1;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

// Key window of query row i inside tile j: columns [c_lo, c_hi] are kept.
struct RowMask {
  int c_lo, c_hi;
};

__device__ __forceinline__ void write_status(int *status, int code) {
  if (status) atomicExch(status, code);
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    gdla_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_qs,
                         const __grid_constant__ CUtensorMap tm_qn,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using L = AttnSmemLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
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
  const uint32_t hn_ready = bar0 + 8u * (12 + 2 * kKvStages);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  float *hn_smem = reinterpret_cast<float *>(smem + L::kHnOff);  // [D][kBM]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work item: heaviest query blocks first (causal), KV groups interleaved
  const int groups = p.B * p.Hn;
  const int qblk = p.n_qblk - 1 - static_cast<int>(blockIdx.x / groups);
  const int grp = static_cast<int>(blockIdx.x % groups);
  const int b = grp / p.Hn;
  const int kvh = grp % p.Hn;
  const int q0 = qblk * kBM;
  int j_lo, j_hi;
  if (p.causal) {
    const int last = min(q0 + kBM - 1, p.T - 1);
    j_hi = last / kBN;
    j_lo = 0;
    if (p.window > 0) {
      const int64_t first = static_cast<int64_t>(q0) - p.window + 1;
      j_lo = first > 0 ? static_cast<int>(first / kBN) : 0;
    }
  } else {
    j_lo = 0;
    j_hi = (p.T - 1) / kBN;
  }
  const int n_tiles = j_hi - j_lo + 1;
  const int n_heads = p.g + 1;               // noise head + g signal heads
  const int n_phases = (n_heads + 1) / 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_empty(i), 1);
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), kBM);
      mbar_init(o_done(i), 1);
      mbar_init(o_free(i), kBM);
    }
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(hn_ready, kBM);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto t_s = [&](int x) { return tmem + 128u * static_cast<uint32_t>(x); };
  auto t_o = [&](int x) { return tmem + 256u + static_cast<uint32_t>(D * x); };

  if (warp == 8) {
    // =============================== TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_qs);
      tma_prefetch_desc(&tm_qn);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t q_uses[2] = {0, 0};
      uint32_t c = 0;  // K/V ring position
      bool ok = true;
      for (int ph = 0; ph < n_phases && ok; ++ph) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int hi = 2 * ph + x;
          if (hi >= n_heads || !ok) break;
          ok = mbar_wait(q_empty(x), (q_uses[x] & 1u) ^ 1u, abort_flag);
          if (!ok) break;
          ++q_uses[x];
          const uint32_t dst = sbase + L::kQOff + x * L::kQBytes;
          mbar_arrive_expect_tx(q_full(x), L::kQBytes);
          const bool noise = (hi == 0);
          const int head = noise ? kvh : p.g * kvh + (hi - 1);
          const CUtensorMap *map = noise ? &tm_qn : &tm_qs;
#pragma unroll
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(dst + kb * (kBM * 128), map, q_full(x), head * D + kb * 64, q0, b);
        }
        for (int j = j_lo; j <= j_hi && ok; ++j) {
          for (int kv = 0; kv < 2 && ok; ++kv) {
            const int s = static_cast<int>(c % kKvStages);
            ok = mbar_wait(kv_empty(s), ((c / kKvStages) & 1u) ^ 1u, abort_flag);
            if (!ok) break;
            const uint32_t dst = sbase + L::kKvOff + s * L::kKvBytes;
            mbar_arrive_expect_tx(kv_full(s), L::kKvBytes);
            const CUtensorMap *map = kv == 0 ? &tm_k : &tm_v;
#pragma unroll
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(dst + kb * (kBN * 128), map, kv_full(s), kvh * D + kb * 64, j * kBN, b);
            ++c;
          }
        }
      }
      if (!ok) {
        // unwinding: let the copies already issued land before the CTA exits
        for (int s = 0; s < kKvStages; ++s) {
          const uint32_t issued = c > static_cast<uint32_t>(s) ? (c - 1 - s) / kKvStages + 1 : 0;
          if (issued) mbar_wait_for(kv_full(s), (issued - 1) & 1u, 100000000ull);
        }
        for (int x = 0; x < 2; ++x)
          if (q_uses[x]) mbar_wait_for(q_full(x), (q_uses[x] - 1) & 1u, 100000000ull);
      }
    }
  } else if (warp == 9) {
    // =============================== MMA issuer
    // Per slot X the issue order is S_X(j) .. PV_X(j), S_X(j+1), so that slot
    // B's MMAs run while slot A's softmax works and vice versa.  S_X(j+1)
    // overwrites the TMEM columns PV_X(j) reads P from; tcgen05.mma
    // instructions from one thread execute in issue order, so the read of P
    // precedes the overwrite.
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, false, true);
      uint32_t q_uses[2] = {0, 0};
      uint32_t o_commits[2] = {0, 0};
      uint32_t p_waits[2] = {0, 0};
      uint32_t ofree_waits[2] = {0, 0};
      uint32_t c = 0;  // ring position of the next K/V tile to consume
      bool ok = true;
      auto issue_s = [&](int x, uint32_t k_base) {
        const uint32_t q_base = sbase + L::kQOff + x * L::kQBytes;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t qoff = (k >> 2) * (kBM * 128) + (k & 3) * 32;
          const uint32_t koff = (k >> 2) * (kBN * 128) + (k & 3) * 32;
          umma_ss(t_s(x), sdesc_sw128(q_base + qoff, 16, 1024),
                  sdesc_sw128(k_base + koff, 16, 1024), kIdescS, k > 0 ? 1u : 0u);
        }
        umma_commit(s_full(x));
      };
      for (int ph = 0; ph < n_phases && ok; ++ph) {
        const int nslot = min(2, n_heads - 2 * ph);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (x < nslot && ok) {
            ok = mbar_wait(q_full(x), q_uses[x] & 1u, abort_flag);
            ++q_uses[x];
          }
        }
        if (!ok) break;
        // prologue: S_X(j_lo)
        {
          const int sk = static_cast<int>(c % kKvStages);
          ok = mbar_wait(kv_full(sk), (c / kKvStages) & 1u, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k_base = sbase + L::kKvOff + sk * L::kKvBytes;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (x < nslot) {
              issue_s(x, k_base);
              if (j_lo == j_hi) umma_commit(q_empty(x));
            }
          }
          umma_commit(kv_empty(sk));
          ++c;
        }
        for (int j = j_lo; j <= j_hi && ok; ++j) {
          const int sv = static_cast<int>(c % kKvStages);
          ok = mbar_wait(kv_full(sv), (c / kKvStages) & 1u, abort_flag);
          if (!ok) break;
          tc_fence_after();
          ++c;
          const uint32_t v_base = sbase + L::kKvOff + sv * L::kKvBytes;
          int sk = 0;
          uint32_t k_base = 0;
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            if (x >= nslot || !ok) break;
            ok = mbar_wait(p_full(x), p_waits[x] & 1u, abort_flag);
            if (!ok) break;
            ++p_waits[x];
            if (j == j_lo && ph > 0) {
              // the previous phase's epilogue must have read O_X
              ok = mbar_wait(o_free(x), ofree_waits[x] & 1u, abort_flag);
              if (!ok) break;
              ++ofree_waits[x];
            }
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < kBN / 16; ++k) {
              umma_ts(t_o(x), t_s(x) + 8u * k,
                      sdesc_sw128(v_base + k * (16 * 128), kBN * 128, 1024), kIdescPV,
                      (j > j_lo || k > 0) ? 1u : 0u);
            }
            umma_commit(o_done(x));
            ++o_commits[x];
            if (j < j_hi) {
              if (x == 0) {
                sk = static_cast<int>(c % kKvStages);
                ok = mbar_wait(kv_full(sk), (c / kKvStages) & 1u, abort_flag);
                if (!ok) break;
                tc_fence_after();
                k_base = sbase + L::kKvOff + sk * L::kKvBytes;
              }
              issue_s(x, k_base);
              if (j + 1 == j_hi) umma_commit(q_empty(x));
            }
          }
          if (!ok) break;
          umma_commit(kv_empty(sv));
          if (j < j_hi) {
            umma_commit(kv_empty(sk));
            ++c;
          }
        }
      }
      // drain: every MMA issued above must finish before TMEM is released
#pragma unroll
      for (int x = 0; x < 2; ++x)
        if (o_commits[x]) mbar_wait_for(o_done(x), (o_commits[x] - 1) & 1u, 100000000ull);
    }
  } else {
    // =============================== softmax + epilogue (slot = warpgroup)
    const int x = warp >> 2;        // slot
    const int wq = warp & 3;        // TMEM lane quarter
    const int r = threadIdx.x & 127;  // row in the block = TMEM lane
    const int i = q0 + r;           // query token
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t s_waits = 0;
    uint32_t o_seen = 0;  // PV commits of this slot in finished phases
    bool hn_waited = false;
    bool ok = true;
    for (int ph = 0; ph < n_phases && ok; ++ph) {
      const int hi = 2 * ph + x;
      if (hi >= n_heads) break;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = j_lo; j <= j_hi; ++j) {
        ok = mbar_wait(s_full(x), s_waits & 1u, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ++s_waits;
        tc_fence_after();
        // kept columns of this row in tile j
        const int kbase = j * kBN;
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
        // pass 1: row max of the tile (32 columns live at a time)
        float mt;
        if (!masked) {
          float ma = -INFINITY, mb = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < kBN / 32; cc += 2) {
            uint32_t r0[32], r1[32];
            tmem_ld32x2_sync(t_s(x) + lane_off + cc * 32, t_s(x) + lane_off + cc * 32 + 32, r0, r1);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              ma = fmax3(ma, __uint_as_float(r0[e]), __uint_as_float(r0[e + 1]));
              mb = fmax3(mb, __uint_as_float(r1[e]), __uint_as_float(r1[e + 1]));
            }
          }
          mt = fmaxf(ma, mb);
        } else {
          mt = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < kBN / 32; ++cc) {
            uint32_t raw[32];
            tmem_ld32_sync(t_s(x) + lane_off + cc * 32, raw);
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int c = cc * 32 + e;
              if (c >= c_lo && c <= c_hi) mt = fmaxf(mt, __uint_as_float(raw[e]));
            }
          }
        }
        mt = mt * sl2;  // scale > 0 keeps the arg max
        const float m_new = fmaxf(m_run, mt);
        float alpha = 1.f;
        float m_use = m_run;
        if (m_new > m_run + kRescaleThreshold || m_run == -INFINITY) {
          m_use = m_new;
          alpha = (m_run == -INFINITY) ? 0.f : ex2_approx(m_run - m_new);
        }
        const float m_safe = (m_use == -INFINITY) ? 0.f : m_use;
        // pass 2: P = exp2(S*c - m) as bf16 pairs.  The P columns of chunk cc
        // ([16cc, 16cc+16)) lie below the S columns still to be read.
        const uint64_t sl2x2 = f2_make(sl2, sl2);
        const uint64_t negm2 = f2_make(-m_safe, -m_safe);
        uint64_t rs2 = f2_make(0.f, 0.f);
#pragma unroll
        for (int cc = 0; cc < kBN / 32; ++cc) {
          uint32_t raw[32];
          tmem_ld32_sync(t_s(x) + lane_off + cc * 32, raw);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float t0, t1;
            f2_split(f2_fma(f2_from_bits(raw[2 * e], raw[2 * e + 1]), sl2x2, negm2), t0, t1);
            if (masked) {
              const int c0 = cc * 32 + 2 * e;
              if (!(c0 >= c_lo && c0 <= c_hi)) t0 = -INFINITY;
              if (!(c0 + 1 >= c_lo && c0 + 1 <= c_hi)) t1 = -INFINITY;
            }
            const float p0 = ex2_approx(t0);
            const float p1 = ex2_approx(t1);
            rs2 = f2_add(rs2, f2_make(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(t_s(x) + lane_off + cc * 16, pk);
        }
        float rs0, rs1;
        f2_split(rs2, rs0, rs1);
        const float rs = rs0 + rs1;
        l_run = l_run * alpha + rs;
        m_run = m_use;
        // O holds the sum over earlier tiles; rescale it when the max moved
        const bool need = (alpha != 1.f) && (j > j_lo);
        if (__any_sync(0xffffffffu, need)) {
          const uint32_t prev = o_seen + static_cast<uint32_t>(j - 1 - j_lo);
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
      // ---- epilogue: wait for the last PV of this phase
      const uint32_t last = o_seen + static_cast<uint32_t>(n_tiles - 1);
      o_seen += static_cast<uint32_t>(n_tiles);
      ok = mbar_wait(o_done(x), last & 1u, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      if (hi == 0) {
        // noise head: keep H_N = O / l on chip for the group's signal heads
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32_sync(t_o(x) + lane_off + cc * 32, o);
#pragma unroll
          for (int e = 0; e < 32; ++e) hn_smem[(cc * 32 + e) * kBM + r] = __uint_as_float(o[e]) * inv_l;
        }
        tc_fence_before();
        mbar_arrive(o_free(x));
        mbar_arrive(hn_ready);
      } else {
        if (!hn_waited) {
          if (x != 0) {
            ok = mbar_wait(hn_ready, 0, abort_flag);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          hn_waited = true;
        }
        const int h = p.g * kvh + (hi - 1);
        const bool row_ok = i < p.T;
        const int64_t row = static_cast<int64_t>(b) * p.T + i;
        float lam = 0.f;
        if (row_ok) lam = __bfloat162float(p.lam[row * p.Hs + h]);
        const int64_t goff = (row * p.Hs + h) * static_cast<int64_t>(D);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32_sync(t_o(x) + lane_off + cc * 32, o);
          if (row_ok) {
            const uint4 *gp = reinterpret_cast<const uint4 *>(p.gate + goff + cc * 32);
            uint4 *op = reinterpret_cast<uint4 *>(p.out + goff + cc * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 gv = __ldg(gp + v);
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
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
        tc_fence_before();
        mbar_arrive(o_free(x));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) write_status(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace gdla
