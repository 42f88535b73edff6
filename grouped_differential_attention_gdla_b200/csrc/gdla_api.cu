// gdla_api.cu - the C ABI of libgdla.so (declared in include/gdla.h).
//
// Host side only: argument validation, TMA tensor-map encoding (driver entry
// point fetched through the runtime, so the library links no libcuda), and
// kernel launches on the caller's stream.  The library never allocates,
// frees or synchronises.
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gdla.h"
#include "host_util.cuh"
#include "attn_fwd.cuh"
#include "attn_rope.cuh"
#include "attn_win.cuh"
#include "decode.cuh"
#include "kv_expand.cuh"
#include "selftest.cuh"

namespace {

using namespace gdla_host;

template <int D>
int launch_attn(const void *q_sig, const void *q_noise, const void *k, const void *v,
                const gdla::AttnParams &prm, int Hs, int Hn, cudaStream_t stream) {
  using L = gdla::AttnSmemLayout<D>;
  CUtensorMap tm_qs, tm_qn, tm_k, tm_v, tm_gate, tm_out;
  const uint64_t T = static_cast<uint64_t>(prm.T), B = static_cast<uint64_t>(prm.B);
  const uint64_t dqs[3] = {static_cast<uint64_t>(Hs) * D, T, B};
  const uint64_t dqn[3] = {static_cast<uint64_t>(Hn) * D, T, B};
  // K and V hold kv_prefix rows (a sequence shard's halo) before query row 0
  const uint64_t dkv[3] = {static_cast<uint64_t>(Hn) * D,
                           T + static_cast<uint64_t>(prm.kv_prefix), B};
  const uint32_t qbox[3] = {64, gdla::kBM, 1};
  const uint32_t kvbox[3] = {64, gdla::kBN, 1};
  if (!make_map(&tm_qs, q_sig, 3, dqs, qbox) || !make_map(&tm_qn, q_noise, 3, dqn, qbox) ||
      !make_map(&tm_k, k, 3, dkv, kvbox) || !make_map(&tm_v, v, 3, dkv, kvbox) ||
      !make_map(&tm_gate, prm.gate, 3, dqs, qbox) || !make_map(&tm_out, prm.out, 3, dqs, qbox))
    return GDLA_ERR_CUDA;
  const uint64_t items = static_cast<uint64_t>(prm.n_qblk) * B * static_cast<uint64_t>(Hn);
  if (items > 0x7fffffffull) return GDLA_ERR_UNSUPPORTED;
  gdla::AttnParams run = prm;
  run.n_items = static_cast<int>(items);
  // Sliding-window items are short and alike: one resident CTA per SM walks
  // them, so each CTA's next item loads while its current one finishes.  Full
  // attention items differ in length; one CTA each lets the hardware balance.
  uint64_t grid = items;
  if (prm.window > 0) {
    int sms = 0;
    if (sm_count(&sms) != GDLA_OK) return GDLA_ERR_CUDA;
    if (grid > static_cast<uint64_t>(sms)) grid = static_cast<uint64_t>(sms);
  }
  // every CTA allocates all 512 TMEM columns: at least 116 KB of shared
  // memory keeps a second CTA off the SM
  constexpr uint32_t kMinSmem = 118784u;
  if (prm.window > 0 && prm.window <= gdla::kBN) {
    // windows of at most one K/V tile: the union-row kernel
    using LW = gdla::WinSmemLayout<D>;
    const uint32_t smem = LW::kBytes > kMinSmem ? LW::kBytes : kMinSmem;
    constexpr auto kern = gdla::gdla_attn_win_kernel<D>;
    const int rc = prepare_kernel<kern>(smem, 0);
    if (rc != GDLA_OK) return rc;
    kern<<<static_cast<unsigned>(grid), gdla::kWinThreads, smem, stream>>>(
        tm_qs, tm_qn, tm_k, tm_v, tm_gate, tm_out, run);
    return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
  }
  const uint32_t smem = L::kBytes > kMinSmem ? L::kBytes : kMinSmem;
  // The kernel re-splits its register pool between warpgroups (setmaxnreg);
  // that is only sound for the per-thread count it was written for, so any
  // other build is refused rather than launched.
  const int rc = prm.window > 0
                     ? prepare_kernel<gdla::gdla_attn_fwd_kernel<D, true>>(
                           smem, static_cast<int>(gdla::kLaunchRegs))
                     : prepare_kernel<gdla::gdla_attn_fwd_kernel<D, false>>(
                           smem, static_cast<int>(gdla::kLaunchRegs));
  if (rc != GDLA_OK) return rc;
  auto kern = prm.window > 0 ? gdla::gdla_attn_fwd_kernel<D, true>
                              : gdla::gdla_attn_fwd_kernel<D, false>;
  kern<<<static_cast<unsigned>(grid), gdla::kAttnThreads, smem, stream>>>(
      tm_qs, tm_qn, tm_k, tm_v, tm_gate, tm_out, run);
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

// The decoupled rotary term: q_rope_* are [B, T, H, kRope], k_rope [B, T, kRope].
template <int D>
int launch_attn_rope(const void *q_sig, const void *q_noise, const void *q_rope_sig,
                     const void *q_rope_noise, const void *k, const void *v, const void *k_rope,
                     const gdla::AttnParams &prm, int Hs, int Hn, cudaStream_t stream) {
  using L = gdla::RopeSmemLayout<D>;
  CUtensorMap tm_qs, tm_qn, tm_qrs, tm_qrn, tm_k, tm_kr, tm_v;
  const uint64_t T = static_cast<uint64_t>(prm.T), B = static_cast<uint64_t>(prm.B);
  const uint64_t dqs[3] = {static_cast<uint64_t>(Hs) * D, T, B};
  const uint64_t dqn[3] = {static_cast<uint64_t>(Hn) * D, T, B};
  const uint64_t dqrs[3] = {static_cast<uint64_t>(Hs) * gdla::kRope, T, B};
  const uint64_t dqrn[3] = {static_cast<uint64_t>(Hn) * gdla::kRope, T, B};
  const uint64_t dkv[3] = {static_cast<uint64_t>(Hn) * D, T, B};
  const uint64_t dkr[3] = {static_cast<uint64_t>(gdla::kRope), T, B};
  const uint32_t box[3] = {64, gdla::kBM, 1};
  if (!make_map(&tm_qs, q_sig, 3, dqs, box) || !make_map(&tm_qn, q_noise, 3, dqn, box) ||
      !make_map(&tm_qrs, q_rope_sig, 3, dqrs, box) ||
      !make_map(&tm_qrn, q_rope_noise, 3, dqrn, box) || !make_map(&tm_k, k, 3, dkv, box) ||
      !make_map(&tm_kr, k_rope, 3, dkr, box) || !make_map(&tm_v, v, 3, dkv, box))
    return GDLA_ERR_CUDA;
  const uint64_t items = static_cast<uint64_t>(prm.n_qblk) * B * static_cast<uint64_t>(Hn);
  if (items > 0x7fffffffull) return GDLA_ERR_UNSUPPORTED;
  gdla::AttnParams run = prm;
  run.n_items = static_cast<int>(items);
  uint64_t grid = items;
  if (prm.window > 0) {
    int sms = 0;
    if (sm_count(&sms) != GDLA_OK) return GDLA_ERR_CUDA;
    if (grid > static_cast<uint64_t>(sms)) grid = static_cast<uint64_t>(sms);
  }
  constexpr auto kern = gdla::gdla_attn_rope_kernel<D>;
  const int rc = prepare_kernel<kern>(L::kBytes, 0);
  if (rc != GDLA_OK) return rc;
  kern<<<static_cast<unsigned>(grid), gdla::kRopeThreads, L::kBytes, stream>>>(
      tm_qs, tm_qn, tm_qrs, tm_qrn, tm_k, tm_kr, tm_v, run);
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

template <int DH>
int launch_expand(const void *c_kv, const void *w_kvb, const gdla::ExpandParams &prm,
                  cudaStream_t stream) {
  using L = gdla::ExpandSmemLayout<DH>;
  CUtensorMap tm_c, tm_w;
  const uint64_t dc[2] = {static_cast<uint64_t>(prm.d_latent), static_cast<uint64_t>(prm.n_tokens)};
  const uint32_t cbox[2] = {64, gdla::kExpBM};
  const uint64_t dw[2] = {static_cast<uint64_t>(prm.n_kv_heads) * 2 * DH,
                          static_cast<uint64_t>(prm.d_latent)};
  const uint32_t wbox[2] = {64, gdla::kExpKC};
  if (!make_map(&tm_c, c_kv, 2, dc, cbox) || !make_map(&tm_w, w_kvb, 2, dw, wbox))
    return GDLA_ERR_CUDA;
  constexpr auto kern = gdla::gdla_kv_expand_kernel<DH>;
  const int rc = prepare_kernel<kern>(L::kAlloc, 0);
  if (rc != GDLA_OK) return rc;
  const uint64_t blocks = (static_cast<uint64_t>(prm.n_tokens) + gdla::kExpBM - 1) / gdla::kExpBM;
  if (blocks > 0x7fffffffull) return GDLA_ERR_UNSUPPORTED;
  kern<<<static_cast<unsigned>(blocks), gdla::kExpThreads, L::kAlloc, stream>>>(tm_c, tm_w, prm);
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

// ---------------------------------------------------------------- decode
// Work split of the decode: each CTA of the attention kernel takes `cps`
// chunks of 128 cached tokens of one sequence.  One CTA fits an SM (it holds
// all of TMEM), so the grid runs in waves of 148 CTAs on a B200; the split
// minimises waves * (cps + kDecodeCtaOverhead), the second term standing for
// what every CTA pays besides its chunks (loading q~, filling the pipeline,
// writing its partial result of Np * (d_latent + 2) floats), in chunk units.
// The split depends on the shapes only, so the workspace size does too.
constexpr int64_t kDecodeSms = 148;
constexpr int64_t kDecodeMinChunks = 4;
constexpr int64_t kDecodeCtaOverhead = 3;

struct DecodePlan {
  int Np, cps, n_split;
  size_t qt_bytes, part_bytes;
};

bool decode_plan(int B, int64_t L_max, int Hs, int Hn, int d_latent, int64_t window,
                 DecodePlan *pl) {
  if (B <= 0 || L_max <= 0 || Hs <= 0 || Hn <= 0 || d_latent <= 0 || window < 0) return false;
  const int64_t np = (static_cast<int64_t>(Hs) + Hn + 15) / 16 * 16;
  int64_t chunks = (L_max + gdla::kDecTok - 1) / gdla::kDecTok;
  if (window > 0) {
    // the most 128-token chunks W consecutive keys can touch
    const int64_t w = (window + gdla::kDecTok - 2) / gdla::kDecTok + 1;
    if (w < chunks) chunks = w;
  }
  int64_t cps = chunks, best = -1;
  int64_t max_split = 8 * kDecodeSms / B + 1;
  if (max_split > gdla::kDecMaxSplit) max_split = gdla::kDecMaxSplit;
  for (int64_t ns = 1; ns <= chunks && ns <= max_split; ++ns) {
    int64_t c = (chunks + ns - 1) / ns;
    if (c < kDecodeMinChunks) c = kDecodeMinChunks;
    const int64_t ctas = static_cast<int64_t>(B) * ((chunks + c - 1) / c);
    const int64_t cost = (ctas + kDecodeSms - 1) / kDecodeSms * (c + kDecodeCtaOverhead);
    if (best < 0 || cost < best) {
      best = cost;
      cps = c;
    }
  }
  const int64_t n_split = (chunks + cps - 1) / cps;
  if (np > 256 || n_split > gdla::kDecMaxSplit || cps > 0x7fffffffll) return false;
  pl->Np = static_cast<int>(np);
  pl->cps = static_cast<int>(cps);
  pl->n_split = static_cast<int>(n_split);
  pl->qt_bytes = (static_cast<size_t>(B) * np * d_latent * 2 + 255) / 256 * 256;
  pl->part_bytes = static_cast<size_t>(B) * n_split * np * (d_latent + 2) * 4;
  return true;
}

// Tensor maps of one decode call, all encoded before its first launch so the
// four kernels go out back to back.
struct DecodeMaps {
  CUtensorMap qs, qn;  // queries [B, Hs | Hn, d]: absorb A tiles
  CUtensorMap w;       // W^KV_b [dl, Hn 2d], boxes {64, 128}: absorb B, W_V of the output GEMM
  CUtensorMap qt;      // absorbed queries [B Np, dl], boxes {64, Np}
  CUtensorMap c;       // latent cache [B, L_max, dl], boxes {64, 128 tokens}
  CUtensorMap z;       // merged z [Hn B NH, dl] over the absorbed queries, boxes {64, Npad}
  int sb;              // sequences per CTA of the output GEMM
};

bool decode_maps(const gdla::DecodeParams &prm, const void *c_hat, DecodeMaps *m) {
  const int g = prm.Hs / prm.Hn, nh = g + 1;
  const int nb = 128 / g;
  const uint64_t dqs[3] = {static_cast<uint64_t>(prm.d), static_cast<uint64_t>(prm.Hs),
                           static_cast<uint64_t>(prm.B)};
  const uint32_t bqs[3] = {64, static_cast<uint32_t>(g), static_cast<uint32_t>(nb)};
  const uint64_t dqn[3] = {static_cast<uint64_t>(prm.d), static_cast<uint64_t>(prm.Hn),
                           static_cast<uint64_t>(prm.B)};
  const uint32_t bqn[3] = {64, 1, 128};
  const uint64_t dw[2] = {static_cast<uint64_t>(prm.Hn) * 2 * prm.d, static_cast<uint64_t>(prm.dl)};
  const uint32_t bw[2] = {64, 128};
  const uint64_t dq[2] = {static_cast<uint64_t>(prm.dl), static_cast<uint64_t>(prm.B) * prm.Np};
  const uint32_t qbox[2] = {64, static_cast<uint32_t>(prm.Np)};
  const uint64_t dc[3] = {static_cast<uint64_t>(prm.dl), static_cast<uint64_t>(prm.L_max),
                          static_cast<uint64_t>(prm.B)};
  const uint32_t cbox[3] = {64, gdla::kDecTok, 1};
  // output GEMM: about one wave of CTAs over the groups, at most
  // kCombMaxRows head rows per CTA
  const int per_group = std::max(1, static_cast<int>(kDecodeSms) / prm.Hn);
  m->sb = std::min(std::max(1, (prm.B + per_group - 1) / per_group), gdla::kCombMaxRows / nh);
  const int npad = (m->sb * nh + 15) / 16 * 16;
  const uint64_t dz[2] = {static_cast<uint64_t>(prm.dl),
                          static_cast<uint64_t>(prm.Hn) * prm.B * nh};
  const uint32_t bz[2] = {64, static_cast<uint32_t>(npad)};
  return make_map(&m->qs, prm.q_sig, 3, dqs, bqs) && make_map(&m->qn, prm.q_noise, 3, dqn, bqn) &&
         make_map(&m->w, prm.w_kvb, 2, dw, bw) && make_map(&m->qt, prm.qt, 2, dq, qbox) &&
         make_map(&m->c, c_hat, 3, dc, cbox) && make_map(&m->z, prm.qt, 2, dz, bz);
}

// The absorb GEMM tiles: signal tiles of 128 / g sequences (all g signal
// heads of a group), noise tiles of 128 sequences, 128 latent columns each.
template <int D>
int launch_decode_absorb(const gdla::DecodeParams &prm, const DecodeMaps &m, cudaStream_t stream) {
  const int nb = 128 / (prm.Hs / prm.Hn);
  constexpr auto kern = gdla::gdla_decode_absorb_kernel<D>;
  const int rc = prepare_kernel<kern>(gdla::AbsorbSmem::kBytes, 0);
  if (rc != GDLA_OK) return rc;
  const int n_sig = (prm.B + nb - 1) / nb, n_noise = (prm.B + 127) / 128;
  kern<<<dim3(static_cast<unsigned>(prm.dl / 128), static_cast<unsigned>(prm.Hn),
              static_cast<unsigned>(n_sig + n_noise)),
         gdla::kAbsThreads, gdla::AbsorbSmem::kBytes, stream>>>(m.qs, m.qn, m.w, prm, n_sig);
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

template <int NP>
int launch_decode_attn(const gdla::DecodeParams &prm, const DecodeMaps &m, cudaStream_t stream) {
  using L = gdla::DecSmem<NP>;
  constexpr auto kern = gdla::gdla_decode_attn_kernel<NP>;
  const int rc = prepare_kernel<kern>(L::kBytes, 0);
  if (rc != GDLA_OK) return rc;
  kern<<<dim3(static_cast<unsigned>(prm.n_split), static_cast<unsigned>(prm.B)), gdla::kDecThreads,
         L::kBytes, stream>>>(m.qt, m.c, prm);
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

// merge of the splits into Z, then the output GEMM and gate
template <int NH>
int launch_decode_merge_out(const gdla::DecodeParams &prm, const DecodeMaps &m,
                          cudaStream_t stream) {
  constexpr auto kout = gdla::gdla_decode_out_kernel<NH>;
  const int rc = prepare_kernel<kout>(gdla::CombSmem::kBytes, 0);
  if (rc != GDLA_OK) return rc;
  const int64_t items = static_cast<int64_t>(prm.Hn) * prm.B * NH * (prm.dl / 4);
  if (prm.n_split > 1)
    gdla::gdla_decode_merge_kernel<NH, 1, 8>
        <<<static_cast<unsigned>((items + 127) / 128), 128, 0, stream>>>(prm);
  else
    gdla::gdla_decode_merge_kernel<NH, 4, 1>
        <<<static_cast<unsigned>((items + 511) / 512), 128, 0, stream>>>(prm);
  if (cudaGetLastError() != cudaSuccess) return GDLA_ERR_CUDA;
  kout<<<dim3(static_cast<unsigned>(prm.Hn), static_cast<unsigned>((prm.B + m.sb - 1) / m.sb)),
         gdla::kCombThreads, gdla::CombSmem::kBytes, stream>>>(m.w, m.z, prm, m.sb);
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

}  // namespace

extern "C" {

int gdla_version(void) { return 100; /* 0.1.0 */ }

const char *gdla_status_string(int code) {
  switch (code) {
    case GDLA_OK: return "ok";
    case GDLA_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or bad flag)";
    case GDLA_ERR_UNSUPPORTED: return "unsupported shape for the sm_100a kernels";
    case GDLA_ERR_ALIGNMENT:
      return "a pointer is misaligned (tensors need 16 bytes, the status word 4)";
    case GDLA_ERR_CUDA: return "a CUDA runtime or driver call failed";
    case GDLA_ERR_TIMEOUT: return "a device-side pipeline wait timed out";
    default: return "unknown status code";
  }
}

int gdla_kv_expand(const void *c_kv, const void *rms_w, const void *w_kvb, float eps,
                   void *k_out, void *v_out, int64_t n_tokens, int d_latent, int n_kv_heads,
                   int d_head, int *d_status, void *stream) {
  if (n_tokens < 0 || d_latent <= 0 || n_kv_heads <= 0 || d_head <= 0) return GDLA_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps < 0.f) return GDLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return GDLA_OK;
  if (!c_kv || !w_kvb || !k_out || !v_out) return GDLA_ERR_INVALID_ARG;
  if (d_latent % 64 != 0 || d_latent > 512) return GDLA_ERR_UNSUPPORTED;
  if (d_head != 64 && d_head != 128) return GDLA_ERR_UNSUPPORTED;
  if (n_tokens > 0x7fffffffll) return GDLA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(n_kv_heads) * 2 * d_head > 0x7fffffffll) return GDLA_ERR_UNSUPPORTED;
  if (!aligned16(c_kv) || !aligned16(w_kvb) || !aligned16(k_out) || !aligned16(v_out) ||
      (rms_w && !aligned16(rms_w)) || (d_status && !aligned4(d_status)))
    return GDLA_ERR_ALIGNMENT;
  gdla::ExpandParams prm;
  prm.rms_w = static_cast<const __nv_bfloat16 *>(rms_w);
  prm.k_out = static_cast<__nv_bfloat16 *>(k_out);
  prm.v_out = static_cast<__nv_bfloat16 *>(v_out);
  prm.status = d_status;
  prm.n_tokens = n_tokens;
  prm.d_latent = d_latent;
  prm.n_kv_heads = n_kv_heads;
  prm.eps = eps;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d_head == 128 ? launch_expand<128>(c_kv, w_kvb, prm, s)
                       : launch_expand<64>(c_kv, w_kvb, prm, s);
}

}  // extern "C"

namespace {

// q_rope_sig, q_rope_noise and k_rope are read only when d_rope > 0.
int attn_fwd_impl(const void *q_sig, const void *q_noise, const void *k, const void *v,
                  const void *lambda, const void *gate, void *out, int B, int64_t T,
                  int64_t kv_prefix, int Hs, int Hn, int Hkv, int d, int64_t window, int causal,
                  float scale, int *d_status, void *stream, const void *q_rope_sig = nullptr,
                  const void *q_rope_noise = nullptr, const void *k_rope = nullptr,
                  int d_rope = 0) {
  if (B < 0 || T < 0 || Hs <= 0 || Hn <= 0 || Hkv <= 0 || d <= 0) return GDLA_ERR_INVALID_ARG;
  if (d_rope < 0 || (d_rope > 0 && kv_prefix != 0)) return GDLA_ERR_INVALID_ARG;
  if (window < 0 || (causal != 0 && causal != 1) || (causal == 0 && window > 0))
    return GDLA_ERR_INVALID_ARG;
  // a shard's halo: one K/V tile, only for windows of at most one tile
  if (kv_prefix != 0 && kv_prefix != gdla::kBN) return GDLA_ERR_INVALID_ARG;
  if (kv_prefix != 0 && !(causal == 1 && window > 0 && window <= gdla::kBN))
    return GDLA_ERR_INVALID_ARG;
  if (std::isnan(scale) || std::isinf(scale)) return GDLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return GDLA_OK;
  if (!q_sig || !q_noise || !k || !v || !lambda || !gate || !out) return GDLA_ERR_INVALID_ARG;
  if (d_rope > 0 && (!q_rope_sig || !q_rope_noise || !k_rope)) return GDLA_ERR_INVALID_ARG;
  if (Hn != Hkv || Hs % Hn != 0) return GDLA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return GDLA_ERR_UNSUPPORTED;
  if (d_rope != 0 && d_rope != gdla::kRope) return GDLA_ERR_UNSUPPORTED;
  if (d_rope > 0 && (!aligned16(q_rope_sig) || !aligned16(q_rope_noise) || !aligned16(k_rope)))
    return GDLA_ERR_ALIGNMENT;
  if (T + kv_prefix > 0x7fffffffll - gdla::kBM) return GDLA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(Hs) * d > 0x7fffffffll) return GDLA_ERR_UNSUPPORTED;
  if (!aligned16(q_sig) || !aligned16(q_noise) || !aligned16(k) || !aligned16(v) ||
      !aligned16(lambda) || !aligned16(gate) || !aligned16(out) ||
      (d_status && !aligned4(d_status)))
    return GDLA_ERR_ALIGNMENT;
  gdla::AttnParams prm;
  prm.lam = static_cast<const __nv_bfloat16 *>(lambda);
  prm.gate = static_cast<const __nv_bfloat16 *>(gate);
  prm.out = static_cast<__nv_bfloat16 *>(out);
  prm.status = d_status;
  prm.B = B;
  prm.T = static_cast<int>(T);
  prm.Hs = Hs;
  prm.Hn = Hn;
  prm.g = Hs / Hn;
  prm.n_qblk = static_cast<int>((T + gdla::kBM - 1) / gdla::kBM);
  prm.kv_prefix = static_cast<int>(kv_prefix);
  // a window covering every key is full causal (not so on a shard: its
  // first rows still reach back into the halo)
  prm.window = (kv_prefix == 0 && window >= T) ? 0 : window;
  // Full attention orders its items heaviest-first within bands of KV groups
  // whose K and V together fill about 32 MB of L2.
  {
    const int64_t groups = static_cast<int64_t>(B) * Hn;
    const int64_t kv_group_bytes = T * static_cast<int64_t>(d) * 2 * 2;
    int64_t band = (32ll << 20) / (kv_group_bytes > 0 ? kv_group_bytes : 1);
    if (band < 1) band = 1;
    if (band > groups) band = groups;
    prm.band = static_cast<int>(band);
  }
  prm.causal = causal;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d + d_rope));
  prm.scale_log2 = sc * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d_rope > 0)
    return d == 128 ? launch_attn_rope<128>(q_sig, q_noise, q_rope_sig, q_rope_noise, k, v,
                                            k_rope, prm, Hs, Hn, s)
                    : launch_attn_rope<64>(q_sig, q_noise, q_rope_sig, q_rope_noise, k, v,
                                           k_rope, prm, Hs, Hn, s);
  return d == 128 ? launch_attn<128>(q_sig, q_noise, k, v, prm, Hs, Hn, s)
                  : launch_attn<64>(q_sig, q_noise, k, v, prm, Hs, Hn, s);
}

}  // namespace

extern "C" {

int gdla_attn_fwd(const void *q_sig, const void *q_noise, const void *k, const void *v,
                  const void *lambda, const void *gate, void *out, int B, int64_t T, int Hs,
                  int Hn, int Hkv, int d, int64_t window, int causal, float scale,
                  int *d_status, void *stream) {
  return attn_fwd_impl(q_sig, q_noise, k, v, lambda, gate, out, B, T, 0, Hs, Hn, Hkv, d, window,
                       causal, scale, d_status, stream);
}

int gdla_attn_fwd_sp(const void *q_sig, const void *q_noise, const void *k, const void *v,
                     const void *lambda, const void *gate, void *out, int B, int64_t T,
                     int64_t kv_prefix, int Hs, int Hn, int Hkv, int d, int64_t window,
                     float scale, int *d_status, void *stream) {
  if (window <= 0 || window > gdla::kBN) return GDLA_ERR_INVALID_ARG;
  return attn_fwd_impl(q_sig, q_noise, k, v, lambda, gate, out, B, T, kv_prefix, Hs, Hn, Hkv, d,
                       window, 1, scale, d_status, stream);
}

int gdla_attn_fwd_rope(const void *q_sig, const void *q_noise, const void *q_rope_sig,
                       const void *q_rope_noise, const void *k, const void *v,
                       const void *k_rope, const void *lambda, const void *gate, void *out, int B,
                       int64_t T, int Hs, int Hn, int Hkv, int d, int d_rope, int64_t window,
                       int causal, float scale, int *d_status, void *stream) {
  return attn_fwd_impl(q_sig, q_noise, k, v, lambda, gate, out, B, T, 0, Hs, Hn, Hkv, d, window,
                       causal, scale, d_status, stream, q_rope_sig, q_rope_noise, k_rope, d_rope);
}

size_t gdla_decode_workspace_bytes(int B, int64_t L_max, int Hs, int Hn, int d_latent,
                                   int64_t window) {
  DecodePlan pl;
  if (!decode_plan(B, L_max, Hs, Hn, d_latent, window, &pl)) return 0;
  return pl.qt_bytes + pl.part_bytes;
}

int gdla_decode_fwd(const void *q_sig, const void *q_noise, const void *c_hat,
                    const int32_t *cache_len, const void *w_kvb, const void *lambda,
                    const void *gate, void *out, int B, int64_t L_max, int Hs, int Hn, int Hkv,
                    int d, int d_latent, int64_t window, float scale, void *workspace,
                    size_t workspace_bytes, int *d_status, void *stream) {
  if (B < 0 || L_max <= 0 || Hs <= 0 || Hn <= 0 || Hkv <= 0 || d <= 0 || d_latent <= 0 ||
      window < 0)
    return GDLA_ERR_INVALID_ARG;
  if (std::isnan(scale) || std::isinf(scale)) return GDLA_ERR_INVALID_ARG;
  if (B == 0) return GDLA_OK;
  if (!q_sig || !q_noise || !c_hat || !cache_len || !w_kvb || !lambda || !gate || !out ||
      !workspace)
    return GDLA_ERR_INVALID_ARG;
  if (Hn != Hkv || Hs % Hn != 0 || Hs / Hn > gdla::kDecMaxGroup) return GDLA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return GDLA_ERR_UNSUPPORTED;
  if (d_latent % gdla::kDecUnit != 0 || d_latent > gdla::kDecMaxLatent) return GDLA_ERR_UNSUPPORTED;
  if (B > 65535 || L_max > 0x7fffffffll - gdla::kDecTok) return GDLA_ERR_UNSUPPORTED;
  DecodePlan pl;
  if (!decode_plan(B, L_max, Hs, Hn, d_latent, window, &pl)) return GDLA_ERR_UNSUPPORTED;
  if (pl.Np > 80) return GDLA_ERR_UNSUPPORTED;  // head rows: 16, 32, 48, 64 or 80
  if (workspace_bytes < pl.qt_bytes + pl.part_bytes) return GDLA_ERR_INVALID_ARG;
  if (!aligned16(q_sig) || !aligned16(q_noise) || !aligned16(c_hat) || !aligned16(w_kvb) ||
      !aligned16(lambda) || !aligned16(gate) || !aligned16(out) || !aligned16(workspace) ||
      !aligned4(cache_len) || (d_status && !aligned4(d_status)))
    return GDLA_ERR_ALIGNMENT;
  gdla::DecodeParams prm;
  prm.q_sig = static_cast<const __nv_bfloat16 *>(q_sig);
  prm.q_noise = static_cast<const __nv_bfloat16 *>(q_noise);
  prm.w_kvb = static_cast<const __nv_bfloat16 *>(w_kvb);
  prm.lam = static_cast<const __nv_bfloat16 *>(lambda);
  prm.gate = static_cast<const __nv_bfloat16 *>(gate);
  prm.out = static_cast<__nv_bfloat16 *>(out);
  prm.cache_len = cache_len;
  prm.qt = static_cast<__nv_bfloat16 *>(workspace);
  prm.part = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + pl.qt_bytes);
  prm.status = d_status;
  prm.B = B;
  prm.Hs = Hs;
  prm.Hn = Hn;
  prm.d = d;
  prm.dl = d_latent;
  prm.Np = pl.Np;
  prm.n_split = pl.n_split;
  prm.cps = pl.cps;
  prm.L_max = L_max;
  prm.window = window;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
  prm.qscale = sc * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DecodeMaps maps;
  if (!decode_maps(prm, c_hat, &maps)) return GDLA_ERR_CUDA;
  const int arc =
      d == 128 ? launch_decode_absorb<128>(prm, maps, s) : launch_decode_absorb<64>(prm, maps, s);
  if (arc != GDLA_OK) return arc;
  int rc;
  switch (pl.Np) {  // head rows of the attention tiles
    case 16: rc = launch_decode_attn<16>(prm, maps, s); break;
    case 32: rc = launch_decode_attn<32>(prm, maps, s); break;
    case 48: rc = launch_decode_attn<48>(prm, maps, s); break;
    case 64: rc = launch_decode_attn<64>(prm, maps, s); break;
    default: rc = launch_decode_attn<80>(prm, maps, s); break;
  }
  if (rc != GDLA_OK) return rc;
  switch (Hs / Hn) {  // merge and output are specialised for the heads of a group
    case 1: return launch_decode_merge_out<2>(prm, maps, s);
    case 2: return launch_decode_merge_out<3>(prm, maps, s);
    case 3: return launch_decode_merge_out<4>(prm, maps, s);
    case 4: return launch_decode_merge_out<5>(prm, maps, s);
    case 5: return launch_decode_merge_out<6>(prm, maps, s);
    case 6: return launch_decode_merge_out<7>(prm, maps, s);
    case 7: return launch_decode_merge_out<8>(prm, maps, s);
    default: return launch_decode_merge_out<9>(prm, maps, s);
  }
}

int gdla_latent_rmsnorm(const void *c_kv, const void *rms_w, float eps, void *out,
                        int64_t n_tokens, int d_latent, int *d_status, void *stream) {
  (void)d_status;
  if (n_tokens < 0 || d_latent <= 0) return GDLA_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps < 0.f) return GDLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return GDLA_OK;
  if (!c_kv || !out) return GDLA_ERR_INVALID_ARG;
  if (d_latent % 8 != 0 || d_latent > 8192) return GDLA_ERR_UNSUPPORTED;
  if (n_tokens > 0x7fffffffll * 8) return GDLA_ERR_UNSUPPORTED;
  if (!aligned16(c_kv) || !aligned16(out) || (rms_w && !aligned16(rms_w)) ||
      (d_status && !aligned4(d_status)))
    return GDLA_ERR_ALIGNMENT;
  const uint64_t blocks = (static_cast<uint64_t>(n_tokens) + 7) / 8;
  gdla::gdla_latent_rmsnorm_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                                     static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16 *>(c_kv), static_cast<const __nv_bfloat16 *>(rms_w), eps,
      static_cast<__nv_bfloat16 *>(out), n_tokens, d_latent);
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

int gdla_selftest_wait_timeout(int *d_status, int64_t limit_ns, void *stream) {
  if (!d_status || limit_ns <= 0 || limit_ns > 1000000000ll) return GDLA_ERR_INVALID_ARG;
  if (!aligned4(d_status)) return GDLA_ERR_ALIGNMENT;
  gdla::gdla_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      d_status, static_cast<uint64_t>(limit_ns));
  return cudaGetLastError() == cudaSuccess ? GDLA_OK : GDLA_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------- decode without allocation
// Scratch for gdla_decode_fwd_noalloc, compiled into the library so that
// callers which cannot allocate device memory still have a workspace.  Host
// code must not pass `g_decode_scratch` itself to a kernel: on the host the
// name stands for a host-side shadow, not the device address.  The device
// address is looked up once per device, with that device current.
static __device__ __align__(256) uint8_t g_decode_scratch[GDLA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

int decode_scratch_address(void **ptr) {
  static std::atomic<void *> cache[kCachedDevices];
  int dev = 0;
  if (current_device(&dev) != GDLA_OK) return GDLA_ERR_CUDA;
  if (dev >= 0 && dev < kCachedDevices) {
    void *c = cache[dev].load(std::memory_order_acquire);
    if (c) {
      *ptr = c;
      return GDLA_OK;
    }
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
    return GDLA_ERR_CUDA;
  if (dev >= 0 && dev < kCachedDevices) cache[dev].store(p, std::memory_order_release);
  *ptr = p;
  return GDLA_OK;
}

}  // namespace

extern "C" int gdla_decode_fwd_noalloc(const void *q_sig, const void *q_noise, const void *c_hat,
                                       const int32_t *cache_len, const void *w_kvb,
                                       const void *lambda, const void *gate, void *out, int B,
                                       int64_t L_max, int Hs, int Hn, int Hkv, int d,
                                       int d_latent, int64_t window, float scale, int *d_status,
                                       void *stream) {
  // the size check comes first, so an oversized request touches no device
  if (B > 0 && gdla_decode_workspace_bytes(B, L_max, Hs, Hn, d_latent, window) >
                   GDLA_DECODE_NOALLOC_SCRATCH_BYTES)
    return GDLA_ERR_UNSUPPORTED;
  void *scratch = nullptr;
  if (B > 0) {
    const int rc = decode_scratch_address(&scratch);
    if (rc != GDLA_OK) return rc;
  }
  return gdla_decode_fwd(q_sig, q_noise, c_hat, cache_len, w_kvb, lambda, gate, out, B, L_max,
                         Hs, Hn, Hkv, d, d_latent, window, scale, scratch,
                         GDLA_DECODE_NOALLOC_SCRATCH_BYTES, d_status, stream);
}
