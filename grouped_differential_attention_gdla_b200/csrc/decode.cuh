// decode.cuh - GDLA decode over the KV latent cache, sm_100a.
//
// Operation ("Motif 3: Technical Report", paper.rainbus.top, step 2 "GDLA
// forward" and the "technical novelty" paragraph: the two query paths share
// one up-projected KV, so the inference cache holds only the 512-d KV latent
// per token, the size of MLA's).  Sequence b has cache_len[b] cached tokens
// whose RMSNorm'd latents c_hat are in the cache; its newest token is the
// query.  Per head h of KV group k, with W_K = W^KV_b[:, k*2d : k*2d+d] and
// W_V = W^KV_b[:, k*2d+d : (k+1)*2d]:
//   s_j = q_h . (c_hat_j W_K) = (W_K q_h) . c_hat_j      absorbed query q~_h
//   H_h = sum_j p_j (c_hat_j W_V) = (sum_j p_j c_hat_j) W_V
// so attention runs in the latent space and reads 1 KB per cached token for
// all 80 heads at once.  Four kernels:
//   absorb   q~ = (scale log2 e) W_K q for every head, bf16, into workspace
//            (tcgen05 GEMM tiles);
//   attn     split-KV attention over the cache (tcgen05): per chunk of 128
//            cached tokens, S^T = c_hat q~^T (M = 128 tokens, N = heads,
//            K = latent), a per-head online softmax across tokens, and
//            z^T += c_hat^T P (M = latent, N = heads, K = tokens); each CTA
//            leaves (max, sum, z) of its chunks in workspace;
//   merge    folds the splits per head into z / l (bf16);
//   out      H = z W_V (tcgen05 GEMM per KV group and block of sequences),
//            then out = G (.) (H_S - lambda Repeat_g(H_N)).
#pragma once

#include "sm100.cuh"

namespace gdla {

constexpr int kDecTok = 128;    // cached tokens per chunk (MMA M of S^T)
constexpr int kDecUnit = 128;   // latent columns per ring unit (MMA M of z^T)
constexpr int kDecRing = 3;     // ring depth (units of [128 tokens][128 latent])
constexpr int kDecThreads = 320;  // warps 0-7 softmax / partials (two halves of the heads), 8 TMA, 9 MMA
constexpr int kDecTmaWarp = 8;
constexpr int kDecMmaWarp = 9;
constexpr int kDecMaxLatent = 512;
constexpr int kDecMaxGroup = 8;   // signal heads per KV group in the decode kernels
constexpr int kDecMaxSplit = 256;  // splits per sequence (the host plan stays below)
constexpr float kDecRescale = 8.0f;  // log2 units: a head's reference moves only past 2^8

struct DecodeParams {
  const __nv_bfloat16 *q_sig;    // [B, Hs, d]
  const __nv_bfloat16 *q_noise;  // [B, Hn, d]
  const __nv_bfloat16 *w_kvb;    // [dl, Hn * 2d]
  const __nv_bfloat16 *lam;      // [B, Hs]
  const __nv_bfloat16 *gate;     // [B, Hs * d]
  __nv_bfloat16 *out;            // [B, Hs * d]
  const int32_t *cache_len;      // [B], device
  __nv_bfloat16 *qt;             // workspace: absorbed queries [B, Np, dl]
  float *part;                   // workspace: per (b, split): m[Np], l[Np], z[Np][dl]
  int *status;
  int B, Hs, Hn, d, dl, Np, n_split, cps;
  int64_t L_max, window;
  float qscale;  // softmax scale * log2(e)
};

// The cached tokens sequence b's query keeps, and the chunks split s covers.
struct DecodeRange {
  int64_t len, t_lo;     // keys [t_lo, len)
  int64_t c_begin, c_end;  // chunks [c_begin, c_end) of this split
  bool bad_len;
};

__device__ __forceinline__ DecodeRange decode_range(const DecodeParams &p, int b, int s) {
  DecodeRange r;
  int64_t L = p.cache_len[b];
  r.bad_len = L < 1 || L > p.L_max;
  if (r.bad_len) L = L < 1 ? 1 : p.L_max;
  r.len = L;
  r.t_lo = (p.window > 0 && L > p.window) ? L - p.window : 0;
  const int64_t c_first = r.t_lo / kDecTok, c_last = (L - 1) / kDecTok;
  r.c_begin = c_first + static_cast<int64_t>(s) * p.cps;
  const int64_t e = r.c_begin + p.cps;
  r.c_end = e < c_last + 1 ? e : c_last + 1;
  if (r.c_end < r.c_begin) r.c_end = r.c_begin;
  return r;
}

__device__ __forceinline__ float *decode_part(const DecodeParams &p, int b, int s) {
  return p.part + (static_cast<size_t>(b) * p.n_split + s) * p.Np * (p.dl + 2);
}

// ---------------------------------------------------------------- absorb
// q~ = (scale log2 e) W_K q for every head (signal head h -> row h, noise
// head k -> row Hs + k; rows Hs + Hn .. Np - 1 are zero padding), as one
// tcgen05 GEMM tile per (KV group k, tile of query rows, 128 latent columns):
//   D[r][x] = sum_c Q[r][c] W_K[x][c],   A = Q rows, B = W_K rows (both K-major)
// A signal tile holds the group's g signal heads of 128 / g sequences (one
// TMA box of [sequences][heads][64]); a noise tile holds the noise head of
// 128 sequences.  Warp 0 loads and issues; the four warps write the rows.
constexpr int kAbsThreads = 128;

struct AbsorbSmem {
  static constexpr uint32_t kSub = 128 * 128;  // [128 rows][64] bf16, 128B swizzle
  static constexpr uint32_t kAOff = 0;
  static constexpr uint32_t kBOff = 2 * kSub;  // up to d = 128
  static constexpr uint32_t kBarOff = kBOff + 2 * kSub;
  static constexpr uint32_t kBytes = kBarOff + 16 + 16;
};

template <int D>
__global__ void __launch_bounds__(kAbsThreads, 1)
    gdla_decode_absorb_kernel(const __grid_constant__ CUtensorMap tm_qs,
                              const __grid_constant__ CUtensorMap tm_qn,
                              const __grid_constant__ CUtensorMap tm_w, const DecodeParams p,
                              int n_sig_tiles) {
  using L = AbsorbSmem;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const int x0 = blockIdx.x * 128;  // latent columns
  const int k = blockIdx.y;         // KV group
  const int g = p.Hs / p.Hn;
  const int nb = 128 / g;           // sequences per signal tile
  const bool noise = static_cast<int>(blockIdx.z) >= n_sig_tiles;
  const int b0 = noise ? (blockIdx.z - n_sig_tiles) * 128 : blockIdx.z * nb;
  const int rows = noise ? 128 : nb * g;  // A rows the box fills
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full = sbase + L::kBarOff, done = full + 8u;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBarOff + 16);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int abort_local = 0;
  bool ok = true;
  if (warp == 0) {
    const bool leader = elect_one();
    if (leader) {
      mbar_arrive_expect_tx(full, static_cast<uint32_t>((D / 64) * (rows + 128) * 128));
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb) {
        if (noise)
          tma_load_3d(sbase + L::kAOff + kb * L::kSub, &tm_qn, full, kb * 64, k, b0);
        else
          tma_load_3d(sbase + L::kAOff + kb * L::kSub, &tm_qs, full, kb * 64, g * k, b0);
        tma_load_2d(sbase + L::kBOff + kb * L::kSub, &tm_w, full, k * 2 * D + kb * 64, x0);
      }
    }
    ok = __all_sync(0xffffffffu, mbar_wait(full, 0, &abort_local));
    tc_fence_after();
    if (ok && leader) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, false, false);
      const uint64_t ad = sdesc_sw128(sbase + L::kAOff, 16, 1024);
      const uint64_t bd = sdesc_sw128(sbase + L::kBOff, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * L::kSub + (kk & 3) * 32;
        umma_ss(tmem, ad + (off >> 4), bd + (off >> 4), kIdesc, kk > 0 ? 1u : 0u);
      }
      umma_commit(done);
    }
    if (!ok && leader) mbar_wait_for(full, 0, 100000000ull);
  }
  ok = __all_sync(0xffffffffu, ok && mbar_wait(done, 0, &abort_local));
  if (ok) {
    tc_fence_after();
    // row r of the tile: (sequence b0 + r / g, signal head g k + r % g), or
    // (sequence b0 + r, noise head k)
    const int r = threadIdx.x;
    const int b = noise ? b0 + r : b0 + r / g;
    const int row = noise ? p.Hs + k : g * k + r % g;
    const bool valid = r < rows && b < p.B;
    __nv_bfloat16 *qt = p.qt + (static_cast<int64_t>(b) * p.Np + row) * p.dl + x0;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t v[32];
      tmem_ld32_sync(tmem + lane_off + cc * 32, v);
      if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(qt + cc * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]) * p.qscale,
                                         __uint_as_float(v[8 * q + 1]) * p.qscale),
                              pack_bf16x2(__uint_as_float(v[8 * q + 2]) * p.qscale,
                                          __uint_as_float(v[8 * q + 3]) * p.qscale),
                              pack_bf16x2(__uint_as_float(v[8 * q + 4]) * p.qscale,
                                          __uint_as_float(v[8 * q + 5]) * p.qscale),
                              pack_bf16x2(__uint_as_float(v[8 * q + 6]) * p.qscale,
                                          __uint_as_float(v[8 * q + 7]) * p.qscale));
      }
    }
    // the padding rows of these sequences, once (group 0's noise tiles)
    if (noise && k == 0 && b < p.B) {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      for (int pr = p.Hs + p.Hn; pr < p.Np; ++pr) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.qt + (static_cast<int64_t>(b) * p.Np + pr) * p.dl + x0);
#pragma unroll
        for (int q = 0; q < 16; ++q) dst[q] = z;
      }
    }
  }
  if (!ok && threadIdx.x == 0 && p.status) atomicExch(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------- attention
template <int NP>
struct DecSmem {
  static constexpr uint32_t kUnitBytes = kDecTok * kDecUnit * 2;  // 32 KB
  static constexpr uint32_t kQtOff = 0;  // q~: [dl/64 blocks][NP rows][128 B], K-major
  static constexpr uint32_t kQtBytes = NP * kDecMaxLatent * 2;
  static constexpr uint32_t kRingOff = kQtOff + kQtBytes;
  static constexpr uint32_t kPOff = kRingOff + kDecRing * kUnitBytes;  // P: [2][NP][128 B]
  static constexpr uint32_t kPBytes = 2 * NP * 128;
  static constexpr uint32_t kRedOff = kPOff + kPBytes;     // int red[2][4][NP]; float lred[4][NP]
  static constexpr uint32_t kRedBytes = 2 * 4 * NP * 4 + 4 * NP * 4;
  static constexpr uint32_t kRefOff = kRedOff + kRedBytes;  // int ref[2][4][NP] (per warp, per chunk parity)
  static constexpr uint32_t kBarOff = kRefOff + 2 * 4 * NP * 4;
  static constexpr int kZStride = (NP + 31) / 32 * 32;        // TMEM columns per z^T block
  static constexpr uint32_t kNumBars = 2 * kDecRing + 9;
  static constexpr uint32_t kMiscOff = kBarOff + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscOff + 16;
  static_assert(kQtBytes % 1024 == 0 && kRingOff % 1024 == 0 && kPOff % 1024 == 0,
                "swizzled operands need 1024-byte alignment");
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  static_assert(NP % 16 == 0 && NP <= 80, "head rows: a multiple of 16, at most 80");
};

// Warp-collective load / store of 8 consecutive 32-bit TMEM columns of the
// warp's 32 lanes (thread i: lane addr.lane + i).
__device__ __forceinline__ void tmem_ld8_sync(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// One arrival per warp after the lanes' own writes.
__device__ __forceinline__ void dec_warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31u) == 0) mbar_arrive(bar);
}

// One CTA per (split s, sequence b); NP = head rows (Hs + Hn padded to 16).
// Warps 0-7: softmax (thread t = token t of the chunk = TMEM lane t) and the
// partial results, warps 0-3 for heads 0 .. NP/2-1 and warps 4-7 for the
// rest (the heads are independent, so the halves never wait on each other);
// warp 8: TMA; warp 9: TMEM allocation and MMA issue.
// TMEM: S^T [0, NP), z^T block u (latent rows 128u..128u+127) at
// [Z (1 + u), Z (1 + u) + NP) with Z = NP rounded up to 32 columns.
template <int NP>
__global__ void __launch_bounds__(kDecThreads, 1)
    gdla_decode_attn_kernel(const __grid_constant__ CUtensorMap tm_qt,
                            const __grid_constant__ CUtensorMap tm_c, const DecodeParams p) {
  using L = DecSmem<NP>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int s = blockIdx.x, b = blockIdx.y;
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const DecodeRange rg = decode_range(p, b, s);
  if (rg.bad_len && s == 0 && threadIdx.x == 0 && p.status)
    atomicExch(p.status, -1 /* GDLA_ERR_INVALID_ARG: cache_len out of 1..L_max */);
  const int n_chunks = static_cast<int>(rg.c_end - rg.c_begin);
  float *part = decode_part(p, b, s);
  if (n_chunks == 0) {  // nothing for this split: a partial that weighs nothing
    for (int h = threadIdx.x; h < NP; h += blockDim.x) {
      part[h] = -INFINITY;
      part[NP + h] = 0.f;
    }
    return;
  }
  const int U = p.dl / kDecUnit;  // ring units per chunk
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto ring_full = [&](int i) { return bar0 + 8u * i; };
  auto ring_empty = [&](int i) { return bar0 + 8u * (kDecRing + i); };
  const uint32_t qt_full = bar0 + 8u * (2 * kDecRing);
  const uint32_t s_full = bar0 + 8u * (2 * kDecRing + 1);   // S^T of a chunk written
  const uint32_t p_full = bar0 + 8u * (2 * kDecRing + 2);   // P written, z^T rescaled
  const uint32_t z_done = bar0 + 8u * (2 * kDecRing + 3);   // z^T MMAs of a chunk done
  // maxima exchanged among the four warps of one half of the heads
  auto red_full = [&](int half, int i) { return bar0 + 8u * (2 * kDecRing + 4 + 2 * half + i); };
  const uint32_t s_free = bar0 + 8u * (2 * kDecRing + 8);   // S^T of a chunk read out
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  int *red = reinterpret_cast<int *>(smem + L::kRedOff);                  // [2][4][NP]
  float *lred = reinterpret_cast<float *>(smem + L::kRedOff + 2 * 4 * NP * 4);  // [4][NP]
  int *refw = reinterpret_cast<int *>(smem + L::kRefOff);                 // [2][4][NP]
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecRing; ++i) {
      mbar_init(ring_full(i), 1);
      mbar_init(ring_empty(i), 1);
    }
    mbar_init(qt_full, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    mbar_init(z_done, 1);
    mbar_init(s_free, 8);
    for (int hf = 0; hf < 2; ++hf) {
      mbar_init(red_full(hf, 0), 4);
      mbar_init(red_full(hf, 1), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kDecMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_s = tmem;
  auto t_z = [&](int u) { return tmem + static_cast<uint32_t>(L::kZStride * (1 + u)); };
  const uint32_t sP = sbase + L::kPOff;

  if (warp == kDecTmaWarp) {
    // =============================== TMA: q~ once, then per chunk the units
    // of pass 1 (scores) and of pass 2 (z^T; the same rows again, from L2)
    const bool leader = elect_one();
    if (leader) {
      tma_prefetch_desc(&tm_qt);
      tma_prefetch_desc(&tm_c);
      mbar_arrive_expect_tx(qt_full, static_cast<uint32_t>(NP * p.dl * 2));
      for (int kb = 0; kb < p.dl / 64; ++kb)
        tma_load_2d(sbase + L::kQtOff + kb * (NP * 128), &tm_qt, qt_full, kb * 64, b * NP);
    }
    // chunk order of the loads: 0, then per chunk ch the scores pass of ch + 1
    // ahead of the z^T pass of ch (0, 1, 0, 2, 1, ..., n-1, n-2, n-1), so the
    // cache streams from HBM while the softmax of ch runs
    uint32_t c = 0;
    bool ok = true;
    for (int q = 0; q < 2 * n_chunks && ok; ++q) {
      const int chx = q == 0                  ? 0
                      : q == 2 * n_chunks - 1 ? n_chunks - 1
                      : (q & 1)               ? (q + 1) / 2
                                              : q / 2 - 1;
      const int32_t tok0 = static_cast<int32_t>((rg.c_begin + chx) * kDecTok);
      for (int u = 0; u < U; ++u) {
        const int slot = static_cast<int>(c % kDecRing);
        ok = __all_sync(0xffffffffu,
                        mbar_wait(ring_empty(slot), ((c / kDecRing) & 1u) ^ 1u, abort_flag));
        if (!ok) break;
        if (leader) {
          const uint32_t dst = sbase + L::kRingOff + slot * L::kUnitBytes;
          mbar_arrive_expect_tx(ring_full(slot), L::kUnitBytes);
          tma_load_3d(dst, &tm_c, ring_full(slot), u * kDecUnit, tok0, b);
          tma_load_3d(dst + kDecTok * 128, &tm_c, ring_full(slot), u * kDecUnit + 64, tok0, b);
        }
        ++c;
      }
    }
    if (!ok && leader) {
      for (int i = 0; i < kDecRing; ++i) {
        const uint32_t issued = c > static_cast<uint32_t>(i) ? (c - 1 - i) / kDecRing + 1 : 0;
        if (issued) mbar_wait_for(ring_full(i), (issued - 1) & 1u, 100000000ull);
      }
      mbar_wait_for(qt_full, 0, 100000000ull);
    }
  } else if (warp == kDecMmaWarp) {
    // =============================== MMA issue (one elected lane)
    const bool leader = elect_one();
    const uint32_t idesc_s = idesc_bf16_f32(kDecTok, NP, false, false);
    const uint32_t idesc_z = idesc_bf16_f32(kDecUnit, NP, true, false);
    bool ok = __all_sync(0xffffffffu, mbar_wait(qt_full, 0, abort_flag));
    uint32_t c = 0, commits = 0;
    // pass 1: S^T = c_hat q~^T over the latent, one unit (two K-blocks) at a time
    auto score_pass = [&]() {
      for (int u = 0; u < U && ok; ++u) {
        const int slot = static_cast<int>(c % kDecRing);
        ok = __all_sync(0xffffffffu, mbar_wait(ring_full(slot), (c / kDecRing) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint32_t a0 = sbase + L::kRingOff + slot * L::kUnitBytes;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint64_t ad = sdesc_sw128(a0 + half * (kDecTok * 128), 16, 1024);
            const uint64_t bd =
                sdesc_sw128(sbase + L::kQtOff + (2 * u + half) * (NP * 128), 16, 1024);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_ss(t_s, ad + ((k * 32) >> 4), bd + ((k * 32) >> 4), idesc_s,
                      (u > 0 || half > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(ring_empty(slot));
        }
        ++c;
      }
      if (ok && leader) umma_commit(s_full);
    };
    if (ok) score_pass();
    for (int ch = 0; ch < n_chunks && ok; ++ch) {
      // the scores of chunk ch + 1 as soon as the softmax has read those of ch
      if (ch + 1 < n_chunks) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_free, ch & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        score_pass();
        if (!ok) break;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(p_full, ch & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // pass 2: z^T[u] += c_hat_u^T P (A: the unit, MN-major over the latent;
      // B: P, K-major over the tokens)
      for (int u = 0; u < U && ok; ++u) {
        const int slot = static_cast<int>(c % kDecRing);
        ok = __all_sync(0xffffffffu, mbar_wait(ring_full(slot), (c / kDecRing) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
        if (leader) {
          const uint64_t ad =
              sdesc_sw128(sbase + L::kRingOff + slot * L::kUnitBytes, kDecTok * 128, 1024);
#pragma unroll
          for (int k = 0; k < kDecTok / 16; ++k) {
            const uint64_t bd = sdesc_sw128(sP + (k >> 2) * (NP * 128), 16, 1024);
            umma_ss(t_z(u), ad + ((k * 16 * 128) >> 4), bd + (((k & 3) * 32) >> 4), idesc_z,
                    (ch > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(ring_empty(slot));
        }
        ++c;
      }
      if (!ok) break;
      if (leader) umma_commit(z_done);
      ++commits;
    }
    if (leader && commits) mbar_wait_for(z_done, (commits - 1) & 1u, 100000000ull);
  } else {
    // =============================== softmax over the chunk's tokens, per head
    // (this half's heads hb .. hb + NH - 1)
    constexpr int NH = NP / 2;
    const int half = warp >> 2;
    const int w = warp & 3;
    const int hb = half * NH;
    const int lane = threadIdx.x & 31;
    const int t = threadIdx.x & 127;  // token row of the chunk = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(w * 32) << 16;
    float lsum[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) lsum[h] = 0.f;
    for (int i = hb + lane; i < hb + NH; i += 32) refw[w * NP + i] = refw[(4 + w) * NP + i] = INT_MIN;
    __syncwarp();
    bool ok = true;
    for (int ch = 0; ch < n_chunks && ok; ++ch) {
      ok = __all_sync(0xffffffffu, mbar_wait(s_full, ch & 1u, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float sv[NH];
#pragma unroll
      for (int i = 0; i < NH / 8; ++i) {
        uint32_t r8[8];
        tmem_ld8_sync(t_s + lane_off + hb + 8 * i, r8);
#pragma unroll
        for (int e = 0; e < 8; ++e) sv[8 * i + e] = __uint_as_float(r8[e]);
      }
      // S^T is in registers: the next chunk's scores may overwrite it
      tc_fence_before();
      dec_warp_arrive(s_free);
      const int64_t tok = (rg.c_begin + ch) * kDecTok + t;
      const bool valid = tok >= rg.t_lo && tok < rg.len;
      // per head: the chunk's largest score rounded up to an integer, over the
      // warp (one redux each), then over the half's four warps through shared memory
      int *rb = red + (ch & 1) * 4 * NP;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const int mi = valid ? static_cast<int>(ceilf(sv[h])) : INT_MIN;
        const int wm = __reduce_max_sync(0xffffffffu, mi);
        if (lane == 0) rb[w * NP + hb + h] = wm;
      }
      dec_warp_arrive(red_full(half, ch & 1));
      ok = __all_sync(0xffffffffu, mbar_wait(red_full(half, ch & 1), (ch >> 1) & 1u, abort_flag));
      if (!ok) break;
      // the previous chunk's z^T MMAs must be done before P is overwritten or
      // z^T rescaled
      if (ch > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(z_done, (ch - 1) & 1u, abort_flag));
        if (!ok) break;
        tc_fence_after();
      }
      // new integral reference per head: the lanes compute it for heads
      // hb + lane, hb + lane + 32, ... into this warp's copy for the chunk
      // (every warp of the half computes the same values); a head's reference
      // moves only when its maximum passes it by more than 2^8
      const int *ref_old = refw + ((ch & 1) * 4 + w) * NP;
      int *ref_new = refw + (((ch & 1) ^ 1) * 4 + w) * NP;
      bool moved = false;
      for (int h = hb + lane; h < hb + NH; h += 32) {
        const int cm = max(max(rb[h], rb[NP + h]), max(rb[2 * NP + h], rb[3 * NP + h]));
        const int old = ref_old[h];
        const bool move =
            old == INT_MIN || static_cast<float>(cm) > static_cast<float>(old) + kDecRescale;
        ref_new[h] = move ? cm : old;
        moved = moved || (move && old != INT_MIN);
      }
      __syncwarp();
      if (__any_sync(0xffffffffu, moved) && ch > 0) {
        // z^T and the row sums hold earlier chunks at the old references
#pragma unroll
        for (int h = 0; h < NH; ++h)
          lsum[h] *= exp2_int(static_cast<float>(ref_old[hb + h] - ref_new[hb + h]));
        for (int u = 0; u < U; ++u) {
#pragma unroll
          for (int i = 0; i < NH / 8; ++i) {
            uint32_t r8[8];
            tmem_ld8_sync(t_z(u) + lane_off + hb + 8 * i, r8);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int h = hb + 8 * i + e;
              const float a = exp2_int(static_cast<float>(ref_old[h] - ref_new[h]));
              r8[e] = __float_as_uint(__uint_as_float(r8[e]) * a);
            }
            tmem_st8(t_z(u) + lane_off + hb + 8 * i, r8);
          }
        }
        tmem_wait_st();
      }
      // P[h][t] = 2^(s - ref) (bf16), K-major over the tokens: block t / 64,
      // row h, 16-byte unit ((t % 64) / 8) ^ (h % 8)
      const uint32_t pb = sP + static_cast<uint32_t>(t >> 6) * (NP * 128) +
                          static_cast<uint32_t>((t & 7) * 2);
      const uint32_t unit = static_cast<uint32_t>((t & 63) >> 3);
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const int hh = hb + h;
        const float pv = valid ? ex2_approx(sv[h] - static_cast<float>(ref_new[hh])) : 0.f;
        lsum[h] += pv;
        const uint32_t addr = pb + static_cast<uint32_t>(hh) * 128u +
                              ((unit ^ static_cast<uint32_t>(hh & 7)) << 4);
        const unsigned short bits = __bfloat16_as_ushort(__float2bfloat16(pv));
        asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(bits) : "memory");
      }
      fence_proxy_async_smem();
      tc_fence_before();
      dec_warp_arrive(p_full);
    }
    // ---- partial results of this split for this half's heads: reference,
    // row sums, z^T
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(z_done, (n_chunks - 1) & 1u, abort_flag));
    if (ok) {
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float v = lsum[h];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) lred[w * NP + hb + h] = v;
      }
      dec_warp_arrive(red_full(half, n_chunks & 1));
      ok = __all_sync(0xffffffffu,
                      mbar_wait(red_full(half, n_chunks & 1), (n_chunks >> 1) & 1u, abort_flag));
    }
    if (ok) {
      const int *ref_last = refw + ((n_chunks & 1) * 4 + w) * NP;
      for (int h = hb + t; h < hb + NH; h += kDecTok) {
        part[h] = static_cast<float>(ref_last[h]);  // this warp's copy; all copies agree
        part[NP + h] = lred[h] + lred[NP + h] + lred[2 * NP + h] + lred[3 * NP + h];
      }
      float *zp = part + 2 * NP;
      for (int u = 0; u < U; ++u) {
#pragma unroll
        for (int i = 0; i < NH / 8; ++i) {
          uint32_t r8[8];
          tmem_ld8_sync(t_z(u) + lane_off + hb + 8 * i, r8);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            zp[static_cast<size_t>(hb + 8 * i + e) * p.dl + u * kDecUnit + t] = __uint_as_float(r8[e]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && p.status) atomicExch(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  if (warp == kDecMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- merge and output
// Two kernels.  merge: one CTA per (KV group k, sequence b, head j of the
// group; j < g: signal head g k + j, j = g: noise head k), thread = 4 latent
// columns: over the splits, M = max_s m_s, l = sum_s 2^(m_s - M) l_s and
// z = sum_s 2^(m_s - M) z_s / l (online over batches of 8 splits, so the loads
// of a batch are in flight together; a split that saw no key weighs nothing),
// written as bf16 row (k B + b) NH + j of Z (over the absorbed queries, which
// the attention kernel no longer needs).  out: one CTA per (k, block of SB
// sequences), one tcgen05 GEMM H^T = W_V^T Z^T (M = 128 value columns, N = the
// block's NH SB rows padded to 16, K = latent; W_V MN-major and Z K-major, both
// by TMA), then out = G (.) (H_S - lambda H_N) for the group's signal heads.
// Merge of one Z row item (row, 4 latent columns) over the splits.
struct MergeItem {
  const float *pm, *pz;  // split 0's m of the head row, and its z at the item's columns
  float M, l;
  float4 acc;
};

// item < Hn B NH dl / 4 <= 80 * 65535 * 128 < 2^31 (the host limits B and the heads)
template <int NH>
__device__ __forceinline__ void merge_item_init(const DecodeParams &p, uint32_t item, MergeItem &it,
                                                __nv_bfloat16 *&dst) {
  constexpr int g = NH - 1;
  const uint32_t tpr = static_cast<uint32_t>(p.dl) / 4;
  const uint32_t row = item / tpr;  // Z row (k B + b) NH + j
  const int x = 4 * static_cast<int>(item - row * tpr);
  const uint32_t kb = row / NH;
  const int j = static_cast<int>(row - kb * NH);
  const uint32_t k = kb / static_cast<uint32_t>(p.B);
  const int b = static_cast<int>(kb - k * static_cast<uint32_t>(p.B));
  const int prow = j < g ? g * static_cast<int>(k) + j : p.Hs + static_cast<int>(k);
  const int64_t ss = static_cast<int64_t>(p.Np) * (p.dl + 2);
  const float *pb = p.part + static_cast<int64_t>(b) * p.n_split * ss;
  it.pm = pb + prow;
  it.pz = pb + 2 * p.Np + static_cast<int64_t>(prow) * p.dl + x;
  it.M = -INFINITY;
  it.l = 0.f;
  it.acc = make_float4(0.f, 0.f, 0.f, 0.f);
  dst = p.qt + static_cast<int64_t>(row) * p.dl + x;
}

// Folds the splits [s0, s0 + SPB) whose values are in m, lv, v into the item.
template <int SPB>
__device__ __forceinline__ void merge_fold(MergeItem &it, const float *m, const float *lv,
                                           const float4 *v) {
  float mn = it.M;
#pragma unroll
  for (int i = 0; i < SPB; ++i) mn = fmaxf(mn, m[i]);
  if (mn == -INFINITY) return;  // no key so far
  const float a = exp2f(it.M - mn);  // 0 while M is -inf
  it.l *= a;
  it.acc.x *= a, it.acc.y *= a, it.acc.z *= a, it.acc.w *= a;
#pragma unroll
  for (int i = 0; i < SPB; ++i) {
    if (m[i] == -INFINITY) continue;  // a split that saw no key: its z was never written
    const float w = exp2f(m[i] - mn);
    it.l = fmaf(w, lv[i], it.l);
    it.acc.x = fmaf(w, v[i].x, it.acc.x);
    it.acc.y = fmaf(w, v[i].y, it.acc.y);
    it.acc.z = fmaf(w, v[i].z, it.acc.z);
    it.acc.w = fmaf(w, v[i].w, it.acc.w);
  }
  it.M = mn;
}

template <int SPB>
__device__ __forceinline__ void merge_load(const DecodeParams &p, const MergeItem &it, bool live,
                                           int s0, float *m, float *lv, float4 *v) {
  const int64_t ss = static_cast<int64_t>(p.Np) * (p.dl + 2);
#pragma unroll
  for (int i = 0; i < SPB; ++i) {
    const bool on = live && s0 + i < p.n_split;
    const int64_t so = on ? (s0 + i) * ss : 0;
    m[i] = on ? it.pm[so] : -INFINITY;
    lv[i] = on ? it.pm[so + p.Np] : 0.f;
    v[i] = on ? *reinterpret_cast<const float4 *>(it.pz + so) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

__device__ __forceinline__ void merge_store(const MergeItem &it, __nv_bfloat16 *dst) {
  const float il = it.l > 0.f ? 1.f / it.l : 0.f;
  uint2 o;
  o.x = pack_bf16x2(it.acc.x * il, it.acc.y * il);
  o.y = pack_bf16x2(it.acc.z * il, it.acc.w * il);
  *reinterpret_cast<uint2 *>(dst) = o;
}

// One thread per IPT items (Hn B NH rows x dl / 4 column groups; a CTA's
// threads take consecutive items, IPT blocks of 128), SPB splits of each per
// batch, all IPT x SPB loads of a batch in flight together (IPT = 1, SPB = 8
// for several splits; IPT = 4, SPB = 1 for one).  Few registers, so many
// CTAs per SM keep many loads in flight.
template <int NH, int IPT, int SPB>
__global__ void __launch_bounds__(128) gdla_decode_merge_kernel(const DecodeParams p) {
  const uint32_t items = static_cast<uint32_t>(p.Hn * NH) * static_cast<uint32_t>(p.B) *
                         static_cast<uint32_t>(p.dl / 4);
  const uint32_t i0 = blockIdx.x * (128 * IPT) + threadIdx.x;
  MergeItem it[IPT];
  __nv_bfloat16 *dst[IPT];
  bool live[IPT];
#pragma unroll
  for (int u = 0; u < IPT; ++u) {
    live[u] = i0 + u * 128 < items;
    merge_item_init<NH>(p, live[u] ? i0 + u * 128 : 0, it[u], dst[u]);
  }
  for (int s0 = 0; s0 < p.n_split; s0 += SPB) {
    float m[IPT][SPB], lv[IPT][SPB];
    float4 v[IPT][SPB];
#pragma unroll
    for (int u = 0; u < IPT; ++u) merge_load<SPB>(p, it[u], live[u], s0, m[u], lv[u], v[u]);
#pragma unroll
    for (int u = 0; u < IPT; ++u) merge_fold<SPB>(it[u], m[u], lv[u], v[u]);
  }
#pragma unroll
  for (int u = 0; u < IPT; ++u)
    if (live[u]) merge_store(it[u], dst[u]);
}

constexpr int kCombThreads = 256;
constexpr int kCombMaxRows = 80;  // N of the GEMM at most
struct CombSmem {
  static constexpr uint32_t kWOff = 0;  // W_V: [dl / 128][2 halves of 64 columns][128 x][128 B]
  static constexpr uint32_t kWBytes = kDecMaxLatent / 128 * 32768;
  static constexpr uint32_t kZOff = kWOff + kWBytes;  // Z: [dl / 64][Npad rows][128 B]
  static constexpr uint32_t kZBytes = kCombMaxRows * kDecMaxLatent * 2;
  static constexpr uint32_t kBarOff = kZOff + kZBytes;
  static constexpr uint32_t kBytes = kBarOff + 32;
  static_assert(kZOff % 1024 == 0, "swizzled operands need 1024-byte alignment");
  static_assert(kBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  // H [rows][128] fp32 overlays W_V once the GEMM is done
  static_assert(kCombMaxRows * 128 * 4 <= kWBytes, "H must fit over W_V");
};

template <int NH>
__global__ void __launch_bounds__(kCombThreads, 1)
    gdla_decode_out_kernel(const __grid_constant__ CUtensorMap tm_w,
                           const __grid_constant__ CUtensorMap tm_z, const DecodeParams p, int SB) {
  using L = CombSmem;
  constexpr int g = NH - 1;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0 && p.status) atomicExch(p.status, -4 /* GDLA_ERR_CUDA */);
    return;
  }
  const int k = blockIdx.x, b0 = blockIdx.y * SB;
  const int d = p.d, dl = p.dl;
  const int Npad = (SB * NH + 15) / 16 * 16;  // N of the GEMM (host: SB NH <= kCombMaxRows)
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full = sbase + L::kBarOff, mma_done = full + 8u;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kBarOff + 16);
  volatile int abort_local = 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (warp == 0) {
    const bool leader = elect_one();
    if (leader) {
      // W_V of group k: value columns k 2d + d + [0, 128) (lanes past d unused);
      // the block's Z rows (rows past them belong to other blocks or lie
      // outside Z: their columns of H^T are not read)
      mbar_arrive_expect_tx(full, static_cast<uint32_t>(dl / 128 * 32768 + dl / 64 * Npad * 128));
      for (int kb = 0; kb < dl / 128; ++kb)
        for (int hf = 0; hf < 2; ++hf)
          tma_load_2d(sbase + L::kWOff + kb * 32768 + hf * 16384, &tm_w, full,
                      k * 2 * d + d + 64 * hf, kb * 128);
      const int row0 = (k * p.B + b0) * NH;
      for (int kb = 0; kb < dl / 64; ++kb)
        tma_load_2d(sbase + L::kZOff + kb * (Npad * 128), &tm_z, full, kb * 64, row0);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(full, 0, &abort_local));
    tc_fence_after();
    if (ok && leader) {
      const uint32_t idesc = idesc_bf16_f32(128, Npad, true, false);
      for (int kk = 0; kk < dl / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(sbase + L::kWOff + (kk >> 3) * 32768 + (kk & 7) * 2048,
                                        16384, 1024);
        const uint64_t bd =
            sdesc_sw128(sbase + L::kZOff + (kk >> 2) * (Npad * 128) + (kk & 3) * 32, 16, 1024);
        umma_ss(tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
      }
      umma_commit(mma_done);
    }
    if (!ok && leader) mbar_wait_for(full, 0, 100000000ull);
  }
  ok = __all_sync(0xffffffffu, ok && mbar_wait(mma_done, 0, &abort_local));
  tc_fence_after();
  // H^T in TMEM (lane = value column c, column = row r) -> H [r][c] in shared
  // memory over W_V (the GEMM has read it)
  __syncthreads();
  float *hs = reinterpret_cast<float *>(smem + L::kWOff);
  if (ok && warp < 4) {
    const int c = warp * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    for (int q = 0; q < Npad / 8; ++q) {
      uint32_t r8[8];
      tmem_ld8_sync(tmem + lane_off + 8 * q, r8);
#pragma unroll
      for (int e = 0; e < 8; ++e) hs[(8 * q + e) * 128 + c] = __uint_as_float(r8[e]);
    }
  }
  __syncthreads();
  if (ok) {
    // items of 8 value columns of one (sequence, signal head); per thread two
    // items, their gate and lambda loads issued before any store
    const int nb = min(SB, p.B - b0), nq = d / 8;
    const int items = nb * g * nq;
    for (int i0 = threadIdx.x; i0 < items; i0 += 2 * kCombThreads) {
      uint4 gv[2];
      float lamv[2];
      int64_t o[2];
      int hrow[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int i = i0 + u * kCombThreads;
        const bool on = i < items;
        const int ii = on ? i : i0;
        const int c8 = (ii % nq) * 8, j = (ii / nq) % g, bb = ii / (nq * g);
        const int b = b0 + bb, h = g * k + j;
        o[u] = (static_cast<int64_t>(b) * p.Hs + h) * d + c8;
        hrow[u] = (bb * NH + j) * 128 + c8;
        gv[u] = *reinterpret_cast<const uint4 *>(p.gate + o[u]);
        lamv[u] = __bfloat162float(p.lam[static_cast<int64_t>(b) * p.Hs + h]);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (i0 + u * kCombThreads >= items) break;
        const float *hsg = hs + hrow[u];
        const float *hno = hsg + (g - (hrow[u] / 128) % NH) * 128;  // the noise row of the sequence
        const uint32_t gw[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
        uint32_t ow[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float d0 = hsg[2 * e] - lamv[u] * hno[2 * e];
          const float d1 = hsg[2 * e + 1] - lamv[u] * hno[2 * e + 1];
          ow[e] = pack_bf16x2(bf16lo_to_f32(gw[e]) * d0, bf16hi_to_f32(gw[e]) * d1);
        }
        *reinterpret_cast<uint4 *>(p.out + o[u]) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      }
    }
  }
  if (!ok && threadIdx.x == 0 && p.status) atomicExch(p.status, -5 /* GDLA_ERR_TIMEOUT */);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ---------------------------------------------------------------- cache write
// RMSNorm of the KV latent of tokens entering the cache: one warp per token,
// fp32 sum of squares, c / sqrt(mean c^2 + eps) * w rounded to bf16.
__global__ void __launch_bounds__(256) gdla_latent_rmsnorm_kernel(
    const __nv_bfloat16 *c, const __nv_bfloat16 *w, float eps, __nv_bfloat16 *out,
    int64_t n_tokens, int dl) {
  const int64_t tkn = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tkn >= n_tokens) return;
  const __nv_bfloat16 *row = c + tkn * dl;
  float ss = 0.f;
  for (int x = lane * 8; x < dl; x += 32 * 8) {
    const uint4 v = *reinterpret_cast<const uint4 *>(row + x);
    const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = bf16lo_to_f32(q[e]), bb = bf16hi_to_f32(q[e]);
      ss = fmaf(a, a, ss);
      ss = fmaf(bb, bb, ss);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rinv = rsqrtf(ss / static_cast<float>(dl) + eps);
  __nv_bfloat16 *orow = out + tkn * dl;
  for (int x = lane * 8; x < dl; x += 32 * 8) {
    const uint4 v = *reinterpret_cast<const uint4 *>(row + x);
    const uint32_t q[4] = {v.x, v.y, v.z, v.w};
    uint32_t o4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float w0 = 1.f, w1 = 1.f;
      if (w) {
        w0 = __bfloat162float(w[x + 2 * e]);
        w1 = __bfloat162float(w[x + 2 * e + 1]);
      }
      o4[e] = pack_bf16x2(bf16lo_to_f32(q[e]) * rinv * w0, bf16hi_to_f32(q[e]) * rinv * w1);
    }
    *reinterpret_cast<uint4 *>(orow + x) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
  }
}

}  // namespace gdla
