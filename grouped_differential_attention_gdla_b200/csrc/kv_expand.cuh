// kv_expand.cuh - RMSNorm of the KV latent fused into the W^KV_b
// up-projection, sm_100a ("Motif 3: Technical Report", paper.rainbus.top,
// step 2: "RMSNorm, then W^KV_b expands 16 KV heads").
//
// One CTA owns 128 tokens.  The TMA warp loads their whole latent rows
// (128 x DL bf16) once; the norm warpgroup computes each row's fp32 sum of
// squares, rescales the row in place (c / sqrt(mean c^2 + eps) * w, rounded
// to bf16) and hands the tile to the MMA warp.  The CTA then walks the KV
// heads: for head h it multiplies the resident tile by the W^KV_b columns
// [h*2*dh, (h+1)*2*dh), streamed from global memory in 64-row chunks through a
// 3-deep ring, accumulating [128 x 2*dh] in TMEM (two buffers, so the
// epilogue of head h overlaps the MMAs of head h+1).  The epilogue splits the
// accumulator into K_h and V_h and stores bf16 rows.
//
// Warp roles (192 threads): warps 0-3 norm + epilogue, warp 4 TMA, warp 5 MMA.
#pragma once

#include "sm100.cuh"

namespace gdla {

constexpr int kExpBM = 128;
constexpr int kExpKC = 64;       // latent rows of W^KV_b per ring stage
constexpr int kExpStages = 3;
constexpr int kExpThreads = 192;

struct ExpandParams {
  const __nv_bfloat16 *rms_w;  // [DL] or null
  __nv_bfloat16 *k_out;        // [N, Hkv, DH]
  __nv_bfloat16 *v_out;        // [N, Hkv, DH]
  int *status;
  int64_t n_tokens;
  int d_latent;  // DL, multiple of 64, <= 512
  int n_kv_heads;
  float eps;
};

template <int DH>
struct ExpandSmemLayout {
  static constexpr int kNT = 2 * DH;                         // accumulator columns per head
  static constexpr uint32_t kABytesMax = kExpBM * 512 * 2;   // 128 KB for DL = 512
  static constexpr uint32_t kStageBytes = kExpKC * kNT * 2;  // 32 KB for DH = 128
  static constexpr uint32_t kAOff = 0;
  static constexpr uint32_t kWOff = kABytesMax;
  static constexpr uint32_t kBarOff = kWOff + kExpStages * kStageBytes;
  // a_full, a_ready, w_full[S], w_empty[S], acc_full[2], acc_empty[2]
  static constexpr uint32_t kNumBars = 2 + 2 * kExpStages + 4;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};

template <int DH>
__global__ void __launch_bounds__(kExpThreads, 1)
    gdla_kv_expand_kernel(const __grid_constant__ CUtensorMap tm_c,
                          const __grid_constant__ CUtensorMap tm_w, const ExpandParams p) {
  using L = ExpandSmemLayout<DH>;
  constexpr int NT = L::kNT;
  constexpr uint32_t kTmemCols = 2 * NT >= 32 ? 2 * NT : 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  const uint32_t a_full = bar0;
  const uint32_t a_ready = bar0 + 8;
  auto w_full = [&](int s) { return bar0 + 16u + 8u * s; };
  auto w_empty = [&](int s) { return bar0 + 16u + 8u * (kExpStages + s); };
  auto acc_full = [&](int b) { return bar0 + 16u + 8u * (2 * kExpStages + b); };
  auto acc_empty = [&](int b) { return bar0 + 16u + 8u * (2 * kExpStages + 2 + b); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kExpBM;
  const int DL = p.d_latent;
  const int n_kb = DL / 64;         // 64-wide column blocks of the latent tile
  const int n_chunks = DL / kExpKC; // ring stages per head
  const int H = p.n_kv_heads;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_ready, kExpBM);
    for (int s = 0; s < kExpStages; ++s) {
      mbar_init(w_full(s), 1);
      mbar_init(w_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full(b), 1);
      mbar_init(acc_empty(b), kExpBM);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // =============================== TMA producer (warp-uniform loop, one lane issues)
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_c);
      tma_prefetch_desc(&tm_w);
      mbar_arrive_expect_tx(a_full, static_cast<uint32_t>(kExpBM * DL * 2));
      for (int kb = 0; kb < n_kb; ++kb)
        tma_load_2d(sbase + L::kAOff + kb * (kExpBM * 128), &tm_c, a_full, kb * 64,
                    static_cast<int32_t>(m0));
    }
    uint32_t c = 0;
    bool ok = true;
    for (int h = 0; h < H && ok; ++h) {
      for (int kc = 0; kc < n_chunks; ++kc) {
        const int s = static_cast<int>(c % kExpStages);
        ok = __all_sync(0xffffffffu, mbar_wait(w_empty(s), ((c / kExpStages) & 1u) ^ 1u, abort_flag));
        if (!ok) break;
        const uint32_t dst = sbase + L::kWOff + s * L::kStageBytes;
        if (leader) {
          mbar_arrive_expect_tx(w_full(s), L::kStageBytes);
#pragma unroll
          for (int nb = 0; nb < NT / 64; ++nb)
            tma_load_2d(dst + nb * (kExpKC * 128), &tm_w, w_full(s), h * NT + nb * 64,
                        kc * kExpKC);
        }
        ++c;
      }
    }
    if (!ok && leader) {
      for (int s = 0; s < kExpStages; ++s) {
        const uint32_t issued = c > static_cast<uint32_t>(s) ? (c - 1 - s) / kExpStages + 1 : 0;
        if (issued) mbar_wait_for(w_full(s), (issued - 1) & 1u, 100000000ull);
      }
      mbar_wait_for(a_full, 0, 100000000ull);
    }
  } else if (warp == 5) {
    // =============================== MMA issuer (warp-uniform loop, one lane issues)
    const bool leader = elect_one();
    constexpr uint32_t kIdesc = idesc_bf16_f32(kExpBM, NT, false, true);
    bool ok = __all_sync(0xffffffffu, mbar_wait(a_ready, 0, abort_flag));
    tc_fence_after();
    const uint64_t ad = sdesc_sw128(sbase + L::kAOff, 16, 1024);
    uint32_t c = 0;
    uint32_t commits = 0;
    for (int h = 0; h < H && ok; ++h) {
      const int buf = h & 1;
      const uint32_t use = static_cast<uint32_t>(h >> 1);
      ok = __all_sync(0xffffffffu, mbar_wait(acc_empty(buf), (use & 1u) ^ 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem + static_cast<uint32_t>(buf * NT);
      for (int kc = 0; kc < n_chunks && ok; ++kc) {
        const int s = static_cast<int>(c % kExpStages);
        ok = __all_sync(0xffffffffu, mbar_wait(w_full(s), (c / kExpStages) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint64_t wd = sdesc_sw128(sbase + L::kWOff + s * L::kStageBytes, kExpKC * 128, 1024);
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < kExpKC / 16; ++kk) {
            const int ks = kc * (kExpKC / 16) + kk;  // 16-wide k step over the latent
            const uint32_t a_off = (ks >> 2) * (kExpBM * 128) + (ks & 3) * 32;
            umma_ss(d_tmem, ad + (a_off >> 4), wd + ((kk * (16 * 128)) >> 4), kIdesc,
                    (kc > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(w_empty(s));
        }
        ++c;
      }
      if (!ok) break;
      if (leader) umma_commit(acc_full(buf));
      ++commits;
    }
    if (commits && leader)
      mbar_wait_for(acc_full((commits - 1) & 1), ((commits - 1) >> 1) & 1u, 100000000ull);
  } else {
    // =============================== norm + epilogue (warps 0-3, one row per thread)
    const int r = threadIdx.x;  // row = TMEM lane
    const int64_t t = m0 + r;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    bool ok = mbar_wait(a_full, 0, abort_flag);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      // pass 1: fp32 sum of squares of the row (order inside the row is irrelevant)
      uint8_t *row_base = smem + L::kAOff + r * 128;
      const int sw = r & 7;
      float ss = 0.f;
      for (int kb = 0; kb < n_kb; ++kb) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = *reinterpret_cast<const uint4 *>(row_base + kb * (kExpBM * 128) + q * 16);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = bf16lo_to_f32(w4[e]), bb = bf16hi_to_f32(w4[e]);
            ss = fmaf(a, a, ss);
            ss = fmaf(bb, bb, ss);
          }
        }
      }
      const float rinv = rsqrtf(ss / static_cast<float>(DL) + p.eps);
      // pass 2: rescale in place; physical 16-byte chunk q holds logical
      // columns 8*(q ^ (row % 8)) .. +7 of this 64-column block
      for (int kb = 0; kb < n_kb; ++kb) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint4 *ptr = reinterpret_cast<uint4 *>(row_base + kb * (kExpBM * 128) + q * 16);
          const uint4 v = *ptr;
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
          const int col0 = kb * 64 + ((q ^ sw) * 8);
          uint32_t o4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float w0 = 1.f, w1 = 1.f;
            if (p.rms_w) {
              w0 = __bfloat162float(p.rms_w[col0 + 2 * e]);
              w1 = __bfloat162float(p.rms_w[col0 + 2 * e + 1]);
            }
            o4[e] = pack_bf16x2(bf16lo_to_f32(w4[e]) * rinv * w0, bf16hi_to_f32(w4[e]) * rinv * w1);
          }
          *ptr = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(a_ready);
      // epilogue per head
      for (int h = 0; h < H && ok; ++h) {
        const int buf = h & 1;
        const uint32_t use = static_cast<uint32_t>(h >> 1);
        ok = mbar_wait(acc_full(buf), use & 1u, abort_flag);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * NT) + lane_off;
#pragma unroll
        for (int cc = 0; cc < NT / 32; ++cc) {
          uint32_t a[32];
          tmem_ld32_sync(acc + cc * 32, a);
          if (t < p.n_tokens) {
            const bool is_v = cc * 32 >= DH;
            const int col = cc * 32 - (is_v ? DH : 0);
            __nv_bfloat16 *dst = (is_v ? p.v_out : p.k_out) + (t * H + h) * static_cast<int64_t>(DH) + col;
            uint4 *dp = reinterpret_cast<uint4 *>(dst);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              dp[v] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * v + 0]), __uint_as_float(a[8 * v + 1])),
                                 pack_bf16x2(__uint_as_float(a[8 * v + 2]), __uint_as_float(a[8 * v + 3])),
                                 pack_bf16x2(__uint_as_float(a[8 * v + 4]), __uint_as_float(a[8 * v + 5])),
                                 pack_bf16x2(__uint_as_float(a[8 * v + 6]), __uint_as_float(a[8 * v + 7])));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(acc_empty(buf));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && p.status) atomicExch(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace gdla
