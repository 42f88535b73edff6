/*
 * gdla.h - C ABI of libgdla.so, the B200 (sm_100a) forward pass of Grouped
 * Differential Latent Attention (GDLA).
 *
 * The operation is the one the page "Motif 3: Technical Report"
 * (paper.rainbus.top digest), step 2 "GDLA forward", writes out:
 *
 *   c_KV,t --RMSNorm--> --W^KV_b--> K_t, V_t           (16 shared KV heads)
 *   H_S = softmax(Q_sig K^T * scale + mask) V           (signal query heads)
 *   H_N = softmax(Q_noise K^T * scale + mask) V         (noise query heads)
 *   D_t = H_S,t - lambda_t (.) Repeat_g(H_N,t)           (g = Hs / Hn)
 *   O_t = G_t (.) D_t                                    (sigmoid gate, given)
 *
 * Head counts 64 signal / 16 noise / 16 shared KV heads and the 1-full : 3
 * sliding (window 128) schedule come from the same page and from
 * "Вышла новая модель Motif 3" (pikabu.ru).  Readings of what the pages leave
 * open, fixed by this ABI:
 *   - signal head h pairs with noise head h / g and reads KV head h / g;
 *     noise head n reads KV head n (so Hn must equal Hkv);
 *   - lambda holds one value per (token, signal head) and, like the gate, is
 *     passed in after its sigmoid; the library only multiplies;
 *   - a window W > 0 keeps keys j with i - W < j <= i; W = 0 is full causal;
 *   - W^KV_b stores the columns of KV head h as [K_h (d_head) | V_h (d_head)].
 *
 * Conventions for every entry point:
 *   - Tensors are dense, row-major and contiguous, bfloat16 unless stated.
 *     Every pointer must be 16-byte aligned (the kernels move data with TMA
 *     and 16-byte vector accesses); otherwise GDLA_ERR_ALIGNMENT.
 *   - Device pointers only (cudaMalloc'd, or memory the GPU can address).
 *     The caller owns all memory.  The library never allocates, frees or
 *     synchronises: a call validates its arguments, enqueues its kernel on
 *     `stream` (a cudaStream_t; NULL is the legacy default stream) and
 *     returns.  Results are ready when that stream reaches the call.
 *   - Argument errors are reported before anything is enqueued; in that case
 *     the call has no effect.
 *   - d_status (optional, may be NULL): a device int, 4-byte aligned
 *     (otherwise GDLA_ERR_ALIGNMENT), that a kernel sets to GDLA_ERR_TIMEOUT
 *     if one of its internal pipeline waits gives up (after about two
 *     seconds); the kernel then stops early and its output is undefined.  The
 *     library never clears it; the caller zeroes it and reads it once the
 *     stream has passed the call.
 *   - The only state the library keeps is a per-device record that a
 *     kernel's launch attributes (its shared-memory limit) have been set and
 *     the device's SM count; calls from several host threads are safe.
 */
#ifndef GDLA_H_
#define GDLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every entry point (and written to d_status). */
#define GDLA_OK 0
#define GDLA_ERR_INVALID_ARG (-1) /* null pointer, negative size, bad flag  */
#define GDLA_ERR_UNSUPPORTED (-2) /* valid but not a shape the kernels take */
#define GDLA_ERR_ALIGNMENT (-3)   /* a pointer is misaligned (16 B; d_status 4 B) */
#define GDLA_ERR_CUDA (-4)        /* a CUDA runtime/driver call failed       */
#define GDLA_ERR_TIMEOUT (-5)     /* a device-side wait gave up (d_status)   */

/* Library version, major * 10000 + minor * 100 + patch. */
int gdla_version(void);

/* Static, human-readable text for a status code (never NULL). */
const char *gdla_status_string(int code);

/*
 * gdla_kv_expand - RMSNorm of the KV latent followed by the W^KV_b
 * up-projection ("Motif 3: Technical Report", paper.rainbus.top, step 2:
 * "RMSNorm, then W^KV_b expands 16 KV heads").
 *
 *   r_t        = sqrt(mean_k c_kv[t, k]^2 + eps)
 *   chat[t, k] = c_kv[t, k] / r_t * rms_w[k]          (fp32, rounded to bf16)
 *   KV[t, :]   = chat[t, :] @ w_kvb                   (fp32 accumulate)
 *   k_out[t, h, :] = KV[t, h*2*d_head + 0      : h*2*d_head + d_head]
 *   v_out[t, h, :] = KV[t, h*2*d_head + d_head : (h+1)*2*d_head]
 *
 * c_kv   [n_tokens, d_latent]                        bf16, read
 * rms_w  [d_latent] or NULL (weight of ones)         bf16, read
 * w_kvb  [d_latent, n_kv_heads * 2 * d_head]         bf16, read
 * k_out  [n_tokens, n_kv_heads, d_head]              bf16, written
 * v_out  [n_tokens, n_kv_heads, d_head]              bf16, written
 * eps    finite, >= 0
 * Supported: d_latent a multiple of 64 in [64, 512]; d_head 64 or 128;
 * n_kv_heads >= 1.  n_tokens == 0 is a no-op returning GDLA_OK.
 * k_out/v_out may not overlap any input.
 */
int gdla_kv_expand(const void *c_kv, const void *rms_w, const void *w_kvb,
                   float eps, void *k_out, void *v_out, int64_t n_tokens,
                   int d_latent, int n_kv_heads, int d_head, int *d_status,
                   void *stream);

/*
 * gdla_attn_fwd - fused GDLA attention forward ("Motif 3: Technical Report",
 * paper.rainbus.top, step 2): both query paths attend over the shared KV
 * heads, the noise output is repeated per group, subtracted with the
 * per-token lambda, and the result is multiplied by the gate.  H_S and H_N
 * stay on chip.
 *
 * q_sig   [B, T, Hs, d]      bf16, read
 * q_noise [B, T, Hn, d]      bf16, read
 * k, v    [B, T, Hkv, d]     bf16, read
 * lambda  [B, T, Hs]         bf16, read (values in [0, 1] expected)
 * gate    [B, T, Hs * d]     bf16, read
 * out     [B, T, Hs * d]     bf16, written; must not overlap any input
 * window  0 = full causal; W > 0 = sliding window (keys i-W < j <= i)
 * causal  1 = causal mask; 0 = no mask at all (window must then be 0)
 * scale   softmax scale on q.k; <= 0 selects 1/sqrt(d)
 *
 * Supported: Hn == Hkv, Hs % Hn == 0, d in {64, 128}, T < 2^31.
 * B == 0 or T == 0 is a no-op returning GDLA_OK.
 * Output rows are computed in fp32 and rounded to bf16 once.
 */
int gdla_attn_fwd(const void *q_sig, const void *q_noise, const void *k,
                  const void *v, const void *lambda, const void *gate,
                  void *out, int B, int64_t T, int Hs, int Hn, int Hkv, int d,
                  int64_t window, int causal, float scale, int *d_status,
                  void *stream);

/*
 * gdla_attn_fwd_rope - gdla_attn_fwd with the decoupled rotary term in the
 * score ("Motif 3: Technical Report", paper.rainbus.top, "technical novelty"
 * paragraph: both query paths share the up-projected KV and one broadcast
 * decoupled rotary key):
 *
 *   s_ij = scale * (q_i . k_j + q_rope_i . k_rope_j)
 *
 * Every head of both paths has its own rotary query; every token has one
 * rotary key that all heads share.  The rotation by position is applied
 * before this call (q_rope and k_rope arrive rotated), as lambda and the gate
 * arrive after their sigmoids.
 *
 * q_sig, q_noise, k, v, lambda, gate, out   as in gdla_attn_fwd
 * q_rope_sig    [B, T, Hs, d_rope]   bf16, read
 * q_rope_noise  [B, T, Hn, d_rope]   bf16, read
 * k_rope        [B, T, d_rope]       bf16, read
 * d_rope        64, or 0 (the rotary pointers are then ignored and the call is
 *               gdla_attn_fwd); other widths give GDLA_ERR_UNSUPPORTED
 * scale         <= 0 selects 1/sqrt(d + d_rope)
 * Same masks, shapes, alignment and errors as gdla_attn_fwd.
 */
int gdla_attn_fwd_rope(const void *q_sig, const void *q_noise,
                       const void *q_rope_sig, const void *q_rope_noise,
                       const void *k, const void *v, const void *k_rope,
                       const void *lambda, const void *gate, void *out, int B,
                       int64_t T, int Hs, int Hn, int Hkv, int d, int d_rope,
                       int64_t window, int causal, float scale, int *d_status,
                       void *stream);

/*
 * gdla_attn_fwd_sp - gdla_attn_fwd with a sliding window on one shard of a
 * sequence split across GPUs ("Motif 3: Technical Report", paper.rainbus.top:
 * its long-context training step and "technical novelty" paragraph describe
 * window-aware ring attention for the sliding-window layers, where one halo
 * exchange of the previous shard's last keys replaces the ring's rotations).
 *
 * The shard holds T consecutive query tokens.  K and V hold kv_prefix rows
 * before the shard's first token, the halo copied from the previous shard,
 * then the shard's own T rows: query row i reads K/V row i + kv_prefix and
 * keeps keys j with i + kv_prefix - window < j <= i + kv_prefix.  The first
 * shard of a sequence passes kv_prefix = 0 (no keys before it).
 *
 * q_sig, q_noise, lambda, gate, out   as in gdla_attn_fwd ([B, T, ...])
 * k, v       [B, kv_prefix + T, Hkv, d]  bf16, read
 * kv_prefix  0 or 128 (one K/V tile; 128 >= window - 1 covers any window)
 * window     1 .. 128, causal
 * Returns GDLA_ERR_INVALID_ARG for another kv_prefix or window; otherwise as
 * gdla_attn_fwd.  Each output row equals, bit for bit, the row the unsharded
 * call computes for the same token when the shard starts on a multiple of
 * 128 tokens (and the window is shorter than the whole sequence).
 */
int gdla_attn_fwd_sp(const void *q_sig, const void *q_noise, const void *k,
                     const void *v, const void *lambda, const void *gate,
                     void *out, int B, int64_t T, int64_t kv_prefix, int Hs,
                     int Hn, int Hkv, int d, int64_t window, float scale,
                     int *d_status, void *stream);

/*
 * gdla_latent_rmsnorm - RMSNorm of KV latents entering the decode cache
 * ("Motif 3: Technical Report", paper.rainbus.top, step 2: the KV latent
 * c_KV,t goes through RMSNorm before W^KV_b; the "technical novelty"
 * paragraph: the inference cache is this latent, the size of MLA's).
 *
 *   c_hat[t, k] = c_kv[t, k] / sqrt(mean_k c_kv[t, k]^2 + eps) * rms_w[k]
 *
 * c_kv   [n_tokens, d_latent]   bf16, read
 * rms_w  [d_latent] or NULL     bf16, read (NULL: weight of ones)
 * out    [n_tokens, d_latent]   bf16, written (may be a slice of the cache)
 * Supported: d_latent a multiple of 8, at most 8192.  n_tokens == 0 is a
 * no-op.  d_status is accepted for symmetry (this kernel has no waits).
 */
int gdla_latent_rmsnorm(const void *c_kv, const void *rms_w, float eps,
                        void *out, int64_t n_tokens, int d_latent,
                        int *d_status, void *stream);

/*
 * gdla_decode_workspace_bytes - bytes of device scratch gdla_decode_fwd needs
 * for these shapes (absorbed queries and per-split partial results); 0 for
 * shapes gdla_decode_fwd cannot take.  Depends on the shapes only.
 */
size_t gdla_decode_workspace_bytes(int B, int64_t L_max, int Hs, int Hn,
                                   int d_latent, int64_t window);

/*
 * gdla_decode_fwd - GDLA forward for the newest token of B sequences over
 * their cache of RMSNorm'd KV latents (same page, step 2 and the "technical
 * novelty" paragraph: both query paths share one up-projected KV, so the
 * cache holds only the latent).  For sequence b with L = cache_len[b]
 * cached tokens, the query token is token L - 1 and the result equals the
 * row gdla_kv_expand + gdla_attn_fwd would compute for it:
 *   K, V = c_hat[b, 0..L-1] W^KV_b,   keys j in (L-1-window, L-1] (0: all)
 *   out[b] = G (.) (H_S - lambda Repeat_g(H_N))
 * The kernels never expand K and V: W^KV_b's K columns are absorbed into the
 * queries and its V columns applied after the attention, which runs in the
 * d_latent-dimensional latent space and reads the cache once for all heads.
 *
 * q_sig      [B, Hs, d]                  bf16, read
 * q_noise    [B, Hn, d]                  bf16, read
 * c_hat      [B, L_max, d_latent]        bf16, read (gdla_latent_rmsnorm output)
 * cache_len  [B] int32, device           1 .. L_max (a value out of range sets
 *                                        d_status to GDLA_ERR_INVALID_ARG and
 *                                        is clamped)
 * w_kvb      [d_latent, Hkv * 2 * d]     bf16, read (per head [K_h | V_h])
 * lambda     [B, Hs], gate [B, Hs * d]   bf16, read
 * out        [B, Hs * d]                 bf16, written
 * workspace  device scratch of at least gdla_decode_workspace_bytes(...)
 *            bytes, 16-byte aligned, owned by the caller; its contents on
 *            entry do not matter, and calls that overlap on the GPU must not
 *            share it
 * window     0 = every cached token; W > 0 = the last W
 * scale      softmax scale on q.k; <= 0 selects 1/sqrt(d)
 * Cache rows the query does not keep (past cache_len, before the window)
 * are read and multiplied by zero weights: they must hold finite values.
 * Supported: Hn == Hkv, Hs / Hn <= 8, Hs + Hn <= 80 (the head rows are
 * padded to a multiple of 16), d in {64, 128}, d_latent in {128, 256, 384,
 * 512}, B <= 65535.
 */
int gdla_decode_fwd(const void *q_sig, const void *q_noise, const void *c_hat,
                    const int32_t *cache_len, const void *w_kvb,
                    const void *lambda, const void *gate, void *out, int B,
                    int64_t L_max, int Hs, int Hn, int Hkv, int d,
                    int d_latent, int64_t window, float scale,
                    void *workspace, size_t workspace_bytes, int *d_status,
                    void *stream);

/*
 * gdla_attn_bwd_workspace_bytes - bytes of device scratch gdla_attn_bwd needs
 * for these shapes: every head's output H (fp32), its log-sum-exp and the
 * softmax-gradient term Delta (fp32), and its upstream gradient (bf16);
 * about (Hs + Hn) * (6 d + 8) bytes per token.  0 for invalid shapes.
 */
size_t gdla_attn_bwd_workspace_bytes(int B, int64_t T, int Hs, int Hn, int d);

/*
 * gdla_attn_bwd - gradients of the GDLA attention forward (gdla_attn_fwd) for
 * an upstream gradient d_out of its output.  The pages give the forward only
 * ("Motif 3: Technical Report", paper.rainbus.top, step 2) and say the model
 * is trained with it ("Вышла новая модель Motif 3", pikabu.ru); these are the
 * chain-rule gradients of that forward:
 *   dgate    = d_out (.) D,           dD = d_out (.) G
 *   dlambda  = -sum_c dD (.) Repeat_g(H_N)        (per token and signal head)
 *   dq_sig, dq_noise, dk, dv: the softmax-attention gradients of both paths
 *   for upstream gradients dH_S = dD and dH_N = -sum_{group} lambda dD; dk and
 *   dv add up the g signal heads and the noise head of each KV group.
 * The forward is recomputed inside (H and the log-sum-exp of every head), so
 * only the forward's inputs are needed.
 *
 * q_sig, q_noise, k, v, lambda, gate   as in gdla_attn_fwd, read
 * d_out     [B, T, Hs * d]   bf16, read
 * dq_sig    [B, T, Hs, d], dq_noise [B, T, Hn, d], dk, dv [B, T, Hkv, d],
 * dlambda   [B, T, Hs], dgate [B, T, Hs * d]: bf16, written (fp32 accumulate,
 *           one rounding); none may overlap another argument
 * workspace device scratch of at least gdla_attn_bwd_workspace_bytes(...)
 *           bytes, 16-byte aligned, owned by the caller; contents on entry do
 *           not matter; calls that overlap on the GPU must not share it
 * window, causal, scale, d_status, stream   as in gdla_attn_fwd
 * Supported: Hn == Hkv, Hs / Hn <= 8, d in {64, 128}.  Four kernels are
 * enqueued on `stream`.
 */
int gdla_attn_bwd(const void *q_sig, const void *q_noise, const void *k,
                  const void *v, const void *lambda, const void *gate,
                  const void *d_out, void *dq_sig, void *dq_noise, void *dk,
                  void *dv, void *dlambda, void *dgate, int B, int64_t T,
                  int Hs, int Hn, int Hkv, int d, int64_t window, int causal,
                  float scale, void *workspace, size_t workspace_bytes,
                  int *d_status, void *stream);

/*
 * gdla_selftest_wait_timeout - device-side check of the failure path.
 *
 * Every pipeline wait inside the kernels above polls an mbarrier with a time
 * limit; when it passes, the kernel writes GDLA_ERR_TIMEOUT to d_status,
 * stops early and releases what it holds, instead of hanging the GPU.  This
 * entry point runs that same wait, in one warp, on a barrier that nothing
 * ever completes, and gives up after limit_ns nanoseconds.
 *
 * d_status  device int, required; receives GDLA_ERR_TIMEOUT when the kernel
 *           has run (the caller zeroes it beforehand)
 * limit_ns  1 .. 1e9
 * Returns GDLA_OK once the kernel is enqueued on `stream`; GDLA_ERR_INVALID_ARG
 * for a null status pointer or a limit out of range.  Nothing traps or
 * faults: the CUDA context stays usable afterwards.
 */
int gdla_selftest_wait_timeout(int *d_status, int64_t limit_ns, void *stream);

/*
 * gdla_decode_fwd_noalloc - gdla_decode_fwd for callers that cannot allocate
 * device memory.  The pages have no counterpart to this entry point: it
 * exists for the library's users, not for the method.
 *
 * gdla_decode_fwd needs a device workspace for the absorbed queries and the
 * per-split partial results.  Some callers have no way to obtain one: code
 * that runs where the process's allocator is owned by someone else (a host
 * framework that forbids cudaMalloc inside its callbacks, a plugin without
 * an allocator handle), or a serving loop that must not allocate between
 * requests.  This entry point takes the same arguments minus the workspace
 * and uses instead a scratch array compiled into the library: a file-scope
 * __device__ array of GDLA_DECODE_NOALLOC_SCRATCH_BYTES bytes (16 MiB), which
 * every GPU that loads the library holds until the process exits.
 *
 *   - It allocates nothing (no cudaMalloc, cudaFree or allocating library
 *     routine) and otherwise behaves exactly like gdla_decode_fwd.
 *   - Shapes whose workspace (gdla_decode_workspace_bytes) exceeds
 *     GDLA_DECODE_NOALLOC_SCRATCH_BYTES are refused with GDLA_ERR_UNSUPPORTED
 *     before anything else happens; use gdla_decode_fwd for them.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it; make that
 *     first call before any stream capture.  A failed look-up returns
 *     GDLA_ERR_CUDA.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents.  Nothing in it needs to start at zero: the kernels
 *     write each byte they read first.  Calls whose kernels overlap on the
 *     GPU (other streams, other host threads) race on the array and give
 *     undefined results: serialise them on one stream.
 */
#define GDLA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int gdla_decode_fwd_noalloc(const void *q_sig, const void *q_noise,
                            const void *c_hat, const int32_t *cache_len,
                            const void *w_kvb, const void *lambda,
                            const void *gate, void *out, int B, int64_t L_max,
                            int Hs, int Hn, int Hkv, int d, int d_latent,
                            int64_t window, float scale, int *d_status,
                            void *stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* GDLA_H_ */
