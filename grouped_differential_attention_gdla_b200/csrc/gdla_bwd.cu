// gdla_bwd.cu - C ABI of the GDLA attention backward (declared in
// include/gdla.h): argument validation, workspace layout, tensor maps and
// the four launches of bwd.cuh on the caller's stream.  Like the forward
// entry points, nothing here allocates, frees or synchronises.
#include <cmath>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gdla.h"
#include "host_util.cuh"
#include "bwd.cuh"

namespace {

using namespace gdla_host;

// 3-D row-major bf16 tensor [d2][d1][d0] with [1][128][64] boxes, 128B swizzle.
bool map3(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2) {
  const uint64_t dims[3] = {d0, d1, d2};
  const uint32_t box[3] = {64, static_cast<uint32_t>(gdla::kBM), 1};
  return make_map(map, base, 3, dims, box);
}

// Workspace: H (fp32) of every head, its log-sum-exp and Delta (fp32,
// head-major, tokens padded to 128), dH (bf16) of every head.
struct BwdWorkspace {
  size_t h, lse, delta, dox, total;
  int64_t tp;
};

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

bool bwd_workspace(int B, int64_t T, int Hs, int Hn, int d, BwdWorkspace *w) {
  if (B <= 0 || T <= 0 || Hs <= 0 || Hn <= 0 || d <= 0) return false;
  const int64_t tp = (T + gdla::kBM - 1) / gdla::kBM * gdla::kBM;
  const size_t h80 = static_cast<size_t>(Hs) + Hn;
  const size_t rows = static_cast<size_t>(B) * static_cast<size_t>(T);
  w->tp = tp;
  w->h = 0;
  w->lse = up256(w->h + rows * h80 * d * 4);
  w->delta = up256(w->lse + static_cast<size_t>(B) * h80 * tp * 4);
  w->dox = up256(w->delta + static_cast<size_t>(B) * h80 * tp * 4);
  w->total = up256(w->dox + rows * h80 * d * 2);
  return true;
}

template <int D>
int launch_bwd(const void *q_sig, const void *q_noise, const void *k, const void *v,
               gdla::AttnSaveParams sp, gdla::BwdParams bp, cudaStream_t s) {
  const uint64_t T = static_cast<uint64_t>(bp.T), B = static_cast<uint64_t>(bp.B);
  const uint64_t H80 = static_cast<uint64_t>(bp.Hs) + bp.Hn;
  CUtensorMap tm_qs, tm_qn, tm_k, tm_v, tm_dox;
  if (!map3(&tm_qs, q_sig, static_cast<uint64_t>(bp.Hs) * D, T, B) ||
      !map3(&tm_qn, q_noise, static_cast<uint64_t>(bp.Hn) * D, T, B) ||
      !map3(&tm_k, k, static_cast<uint64_t>(bp.Hn) * D, T, B) ||
      !map3(&tm_v, v, static_cast<uint64_t>(bp.Hn) * D, T, B) ||
      !map3(&tm_dox, bp.dox, H80 * D, T, B))
    return GDLA_ERR_CUDA;
  int sms = 0;
  if (sm_count(&sms) != GDLA_OK) return GDLA_ERR_CUDA;

  // 1. the forward in save mode: H and the log-sum-exp of every head
  {
    using L = gdla::RopeSmemLayout<D, 0>;
    constexpr auto kern = gdla::gdla_attn_rope_kernel<D, 0, true, gdla::AttnSaveParams>;
    const int rc = prepare_kernel<kern>(L::kBytes, 0);
    if (rc != GDLA_OK) return rc;
    const uint64_t items = static_cast<uint64_t>(sp.n_qblk) * B * static_cast<uint64_t>(bp.Hn);
    if (items > 0x7fffffffull) return GDLA_ERR_UNSUPPORTED;
    sp.n_items = static_cast<int>(items);
    uint64_t grid = items;
    if (sp.window > 0 && grid > static_cast<uint64_t>(sms)) grid = static_cast<uint64_t>(sms);
    kern<<<static_cast<unsigned>(grid), gdla::kRopeThreads, L::kBytes, s>>>(
        tm_qs, tm_qn, tm_qs, tm_qn, tm_k, tm_k, tm_v, sp);
    if (cudaGetLastError() != cudaSuccess) return GDLA_ERR_CUDA;
  }
  // 2. dG, dlambda, dH of every head and Delta
  const uint64_t pairs = static_cast<uint64_t>(B) * static_cast<uint64_t>(T) * bp.Hn;
  if (B * T > 0x7fffffffull || (pairs + gdla::kPrepWarps - 1) / gdla::kPrepWarps > 0x7fffffffull)
    return GDLA_ERR_UNSUPPORTED;
  gdla::gdla_bwd_prep_kernel<D>
      <<<static_cast<unsigned>((pairs + gdla::kPrepWarps - 1) / gdla::kPrepWarps),
         32 * gdla::kPrepWarps, 0, s>>>(bp);
  if (cudaGetLastError() != cudaSuccess) return GDLA_ERR_CUDA;
  // 3. dQ of every head, heaviest query blocks first
  {
    using L = gdla::DqSmemLayout<D>;
    constexpr auto kern = gdla::gdla_bwd_dq_kernel<D>;
    const int rc = prepare_kernel<kern>(L::kBytes, 0);
    if (rc != GDLA_OK) return rc;
    const uint64_t items = static_cast<uint64_t>(bp.n_qblk) * B * H80;
    if (items > 0x7fffffffull) return GDLA_ERR_UNSUPPORTED;
    // persistent: one CTA per SM walks the items
    const uint64_t grid = items < static_cast<uint64_t>(sms) ? items : static_cast<uint64_t>(sms);
    kern<<<static_cast<unsigned>(grid), gdla::kBwdThreads, L::kBytes, s>>>(
        tm_qs, tm_qn, tm_dox, tm_k, tm_v, bp);
    if (cudaGetLastError() != cudaSuccess) return GDLA_ERR_CUDA;
  }
  // 4. dK, dV of every KV group, earliest key blocks first
  {
    using L = gdla::DkdvSmemLayout<D>;
    constexpr auto kern = gdla::gdla_bwd_dkdv_kernel<D>;
    const int rc = prepare_kernel<kern>(L::kBytes, 0);
    if (rc != GDLA_OK) return rc;
    const uint64_t items = static_cast<uint64_t>(bp.n_kblk) * B * static_cast<uint64_t>(bp.Hn);
    if (items > 0x7fffffffull) return GDLA_ERR_UNSUPPORTED;
    kern<<<static_cast<unsigned>(items), gdla::kBwdThreads, L::kBytes, s>>>(
        tm_qs, tm_qn, tm_dox, tm_k, tm_v, bp);
    if (cudaGetLastError() != cudaSuccess) return GDLA_ERR_CUDA;
  }
  return GDLA_OK;
}

}  // namespace

extern "C" {

size_t gdla_attn_bwd_workspace_bytes(int B, int64_t T, int Hs, int Hn, int d) {
  BwdWorkspace w;
  return bwd_workspace(B, T, Hs, Hn, d, &w) ? w.total : 0;
}

int gdla_attn_bwd(const void *q_sig, const void *q_noise, const void *k, const void *v,
                  const void *lambda, const void *gate, const void *d_out, void *dq_sig,
                  void *dq_noise, void *dk, void *dv, void *dlambda, void *dgate, int B,
                  int64_t T, int Hs, int Hn, int Hkv, int d, int64_t window, int causal,
                  float scale, void *workspace, size_t workspace_bytes, int *d_status,
                  void *stream) {
  if (B < 0 || T < 0 || Hs <= 0 || Hn <= 0 || Hkv <= 0 || d <= 0) return GDLA_ERR_INVALID_ARG;
  if (window < 0 || (causal != 0 && causal != 1) || (causal == 0 && window > 0))
    return GDLA_ERR_INVALID_ARG;
  if (std::isnan(scale) || std::isinf(scale)) return GDLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return GDLA_OK;
  if (!q_sig || !q_noise || !k || !v || !lambda || !gate || !d_out || !dq_sig || !dq_noise ||
      !dk || !dv || !dlambda || !dgate || !workspace)
    return GDLA_ERR_INVALID_ARG;
  if (Hn != Hkv || Hs % Hn != 0 || Hs / Hn > gdla::kBwdMaxGroup) return GDLA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return GDLA_ERR_UNSUPPORTED;
  if (T > 0x7fffffffll - gdla::kBM) return GDLA_ERR_UNSUPPORTED;
  BwdWorkspace ws;
  if (!bwd_workspace(B, T, Hs, Hn, d, &ws)) return GDLA_ERR_INVALID_ARG;
  if (workspace_bytes < ws.total) return GDLA_ERR_INVALID_ARG;
  const void *ptrs[] = {q_sig, q_noise, k, v, lambda, gate, d_out, dq_sig, dq_noise,
                        dk,    dv,      dlambda, dgate, workspace};
  for (const void *p : ptrs)
    if (!aligned16(p)) return GDLA_ERR_ALIGNMENT;
  if (d_status && (reinterpret_cast<uintptr_t>(d_status) & 3u) != 0) return GDLA_ERR_ALIGNMENT;

  uint8_t *wsb = static_cast<uint8_t *>(workspace);
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d));
  const int n_blk = static_cast<int>((T + gdla::kBM - 1) / gdla::kBM);
  const int64_t win = window >= T ? 0 : window;  // a window covering every key is full causal

  gdla::AttnSaveParams sp{};
  sp.lam = static_cast<const __nv_bfloat16 *>(lambda);
  sp.gate = static_cast<const __nv_bfloat16 *>(gate);
  sp.out = nullptr;
  sp.status = d_status;
  sp.B = B;
  sp.T = static_cast<int>(T);
  sp.Hs = Hs;
  sp.Hn = Hn;
  sp.g = Hs / Hn;
  sp.n_qblk = n_blk;
  sp.kv_prefix = 0;
  sp.window = win;
  sp.causal = causal;
  sp.scale_log2 = sc * 1.4426950408889634f;
  {
    const int64_t groups = static_cast<int64_t>(B) * Hn;
    const int64_t kv_group_bytes = T * static_cast<int64_t>(d) * 2 * 2;
    int64_t band = (32ll << 20) / (kv_group_bytes > 0 ? kv_group_bytes : 1);
    if (band < 1) band = 1;
    if (band > groups) band = groups;
    sp.band = static_cast<int>(band);
  }
  sp.h = reinterpret_cast<float *>(wsb + ws.h);
  sp.lse = reinterpret_cast<float *>(wsb + ws.lse);
  sp.tp = static_cast<int>(ws.tp);

  gdla::BwdParams bp{};
  bp.lam = sp.lam;
  bp.gate = sp.gate;
  bp.dout = static_cast<const __nv_bfloat16 *>(d_out);
  bp.dq_sig = static_cast<__nv_bfloat16 *>(dq_sig);
  bp.dq_noise = static_cast<__nv_bfloat16 *>(dq_noise);
  bp.dk = static_cast<__nv_bfloat16 *>(dk);
  bp.dv = static_cast<__nv_bfloat16 *>(dv);
  bp.dlam = static_cast<__nv_bfloat16 *>(dlambda);
  bp.dgate = static_cast<__nv_bfloat16 *>(dgate);
  bp.h = sp.h;
  bp.lse = sp.lse;
  bp.delta = reinterpret_cast<float *>(wsb + ws.delta);
  bp.dox = reinterpret_cast<__nv_bfloat16 *>(wsb + ws.dox);
  bp.status = d_status;
  bp.B = B;
  bp.T = static_cast<int>(T);
  bp.tp = sp.tp;
  bp.Hs = Hs;
  bp.Hn = Hn;
  bp.g = Hs / Hn;
  bp.n_qblk = n_blk;
  bp.n_kblk = n_blk;
  bp.window = win;
  bp.causal = causal;
  bp.scale = sc;
  bp.scale_log2 = sp.scale_log2;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return d == 128 ? launch_bwd<128>(q_sig, q_noise, k, v, sp, bp, s)
                  : launch_bwd<64>(q_sig, q_noise, k, v, sp, bp, s);
}

}  // extern "C"
