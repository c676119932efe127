/*
 * dg.h — C ABI of the canvas-step library (block-wise discrete diffusion, sm_100a).
 *
 * One denoising step of block-wise discrete-diffusion decoding, as the pages describe it:
 *   "DiffusionGemma Technical Report" (metalmedia.ai), Figure 4: a prompt is encoded
 *   causally into a KV cache; the decoder refines a canvas with bidirectional attention over
 *   the canvas and cross-attention to the cache; the finished canvas is re-encoded causally and
 *   appended to the cache.  Same page, explanatory visual ("Inference: block-wise diffusion
 *   decoding"): an entropy-bounded sampler with adaptive stopping finishes a 256-token block in
 *   a few steps.  Model card "diffusiongemma" (axforge.ai), "Model Overview" and
 *   "Mixture-of-Experts (MoE) Efficiency": encoder-decoder, 8 of 128 experts active.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library never allocates,
 *     frees or keeps them.  Structs (dg_config, dg_model, dg_layer_weights) are HOST memory
 *     read during the call only.
 *   - Scratch memory is a caller-provided device buffer `ws` of at least the size that
 *     dg_workspace_size() returns for the same (cfg, batch, n_tokens, cache_cap); 256-byte
 *     aligned.  Contents need not be initialised and are clobbered.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*) and does not
 *     synchronise.  The return value reports host-detectable problems (bad arguments, launch
 *     failure) before or at launch; nothing is launched when an argument is rejected.
 *   - Problems only the device can see (a non-finite entropy, a token id out of range, a full
 *     KV cache) are recorded in the caller's device word `dev_status` (int32, first error
 *     wins) and the affected work is skipped; read it with dg_read_status().  `dev_status`
 *     may be NULL, in which case such problems are not reported.
 *   - Layouts are row-major with the LAST index contiguous.  B = batch (independent canvases),
 *     C = cfg->canvas, d = cfg->d_model, Hq/Hkv = query/kv heads, hd = head_dim, E = experts,
 *     k = top_k, F = d_ff, V = vocab.  Activation element type = cfg->act_dtype (F32 or BF16);
 *     layer-weight element type = cfg->w_dtype (F32, BF16, or E4M3 with one fp32 scale per
 *     output channel).  The K/V cache of one layer is [B][Hkv][cache_cap][hd], the full cache
 *     [L][B][Hkv][cache_cap][hd], both in the activation type.
 *   - The residual stream (embedding rows, the hidden rows after the attention block and after
 *     the expert FFN) is fp32 for every activation type; the tensors that feed a matrix product
 *     or the attention (normalised rows, q, k, v, attention output, expert activations) are in
 *     the activation type.
 *   - Calls keep no state between them and may be made from several host threads on different
 *     streams, with two exceptions, documented at their declarations: dg_generate keeps the
 *     CUDA graphs it instantiates (a bounded cache), and dg_logits_entropy_static keeps its
 *     scratch in one fixed device array shared by all its calls.
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------------- */
enum {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,  /* bad pointer, size, or combination of arguments               */
  DG_ERR_UNSUPPORTED = 2,  /* a shape or dtype combination this build has no kernel for     */
  DG_ERR_CAPACITY = 3,     /* KV-cache rows would exceed cache_cap (device-detected)        */
  DG_ERR_CUDA = 4,         /* a CUDA call or launch failed; see dg_last_cuda_error()         */
  DG_ERR_NUMERIC = 5,      /* a non-finite logit or entropy was seen (device-detected)       */
  DG_ERR_TIMEOUT = 6,      /* a bounded device-side wait expired (device-detected)           */
  DG_ERR_WORKSPACE = 7     /* ws_bytes smaller than dg_workspace_size()                      */
};

enum { DG_F32 = 0, DG_BF16 = 1, DG_E4M3 = 2, DG_NVFP4 = 3 };

/* NVFP4 storage (the tied embedding / LM head only; the model card names an NVFP4 build of the
 * checkpoint, and the format is NVIDIA's: FP4 E2M1 elements, one FP8 E4M3 scale per 16
 * consecutive elements of a row, one fp32 tensor scale g; element = e2m1 * e4m3 * g).  For a
 * matrix of R rows and K columns (K a multiple of 256), Rp = R rounded up to a multiple of 256:
 *   codes  uint8 [K/64][Rp][32]: byte i of (k-block kb, row r) holds column kb*64 + 2i in its
 *          low nibble and column kb*64 + 2i + 1 in its high nibble;
 *   scales uint8 [K/64][Rp][4]:  scale j of (kb, r) covers columns kb*64 + 16j .. + 15.
 * Rows [R, Rp) are padding (read, never used).  Both arrays 16-byte aligned. */

/* Model shape.  The MASK token id is `vocab` (one extra embedding row); the LM head covers
 * ids [0, vocab), so argmax never returns MASK.  rope_theta: rotary base; rms_eps: RMSNorm eps. */
typedef struct dg_config {
  int32_t d_model, n_q_heads, n_kv_heads, head_dim;
  int32_t n_experts, top_k, d_ff;
  int32_t vocab, canvas, n_layers;
  double rope_theta, rms_eps;
  int32_t act_dtype; /* DG_F32 or DG_BF16 */
  int32_t w_dtype;   /* DG_F32 (with act F32), DG_BF16 or DG_E4M3 (with act BF16) */
  int32_t emb_dtype; /* the tied embedding / LM head: act_dtype, or DG_NVFP4 (with act BF16,
                        d_model a multiple of 256, at most 4096) */
  int32_t n_shared;  /* always-on shared experts S >= 0 (the model card's MoE "+1 shared"):
                        experts E .. E + S - 1 of the expert arrays take every live token with
                        gate 1, in the slots after its k routed ones; E + S <= 256, k + S <= 32 */
} dg_config;

/* One layer's weights (device pointers).  Every matrix is [out][in], `in` contiguous.
 *   w_qkv     [(Hq + 2 Hkv) hd][d]   rows: q heads, then k heads, then v heads
 *   w_o       [d][Hq hd]
 *   w_router  [E][d]                 BF16 (F32 when w_dtype is F32), never E4M3
 *   w_gate_up [E + S][2F][d]         rows [0,F) gate, [F,2F) up (S = n_shared: the shared
 *   w_down    [E + S][d][F]          experts after the E routed ones)
 * s_* : fp32 per-output-channel scales, required for E4M3 and ignored otherwise. */
typedef struct dg_layer_weights {
  const void *w_qkv;     const float *s_qkv;
  const void *w_o;       const float *s_o;
  const void *w_router;
  const void *w_gate_up; const float *s_gate_up;
  const void *w_down;    const float *s_down;
} dg_layer_weights;

/* A whole model: `layers` is a HOST array of n_layers structs; `emb` the tied embedding /
 * LM head [V + 1][d] in the activation type (row V = MASK; rows [0,V) = LM head).  With
 * emb_dtype DG_NVFP4, `emb` holds the NVFP4 codes of that [V + 1][d] matrix, emb_scale its
 * block scales and emb_scale_global its tensor scale (layout above); otherwise both are
 * ignored. */
typedef struct dg_model {
  const dg_layer_weights *layers;
  const void *emb;
  const uint8_t *emb_scale;
  float emb_scale_global;
} dg_model;

/* Sampler variants ("DiffusionGemma Technical Report": explanatory visual and Figure 3, a canvas
 * that starts as uniform noise; Figure 9, a temperature annealed over the step budget N, milder
 * for a larger N; Figure 10, tau_t = 1 with annealing off; ainewsonline.de article: the model
 * corrects its own mistakes while denoising, before the output is final).  The pages give no
 * formulas; the library's readings:
 *   tau_s = tau_start + (tau_end - tau_start) * min(s, N - 1) / max(N - 1, 1)  (fp64; s = the
 *           canvas's step index, N = max_steps).  tau_s > 0: each masked position's token is
 *           drawn from softmax(z / tau_s) as argmax_v (z_v * (1/tau_s) + G_v), G = -ln(-ln U)
 *           (Gumbel-max; 1/tau_s rounded to fp32), and the EB rule ranks the entropies of
 *           softmax(z / tau_s).  tau_s <= 0: greedy argmax, entropy at tau = 1.
 *   U = ((w >> 9) + 1/2) * 2^-23, w a word of Philox4x32-10 (Salmon et al., SC 2011) keyed by
 *           (seed low word, seed high word) at counter (v >> 2, i, s, (1 << 24) | b), word v & 3,
 *           for vocabulary entry v of position i of canvas b at step s.
 *   revise: positions that are not final (masked = 1) hold revisable draft tokens: they are
 *           embedded by their token instead of MASK, and every such position the EB rule does not
 *           commit takes this step's drawn token as its new draft (committed positions are final,
 *           as before).  Used with dg_noise_canvas. */
typedef struct dg_sampler {
  double tau_start, tau_end; /* temperature at step 0 and at step max_steps - 1 (finite) */
  uint64_t seed;             /* generator key */
  int32_t revise;            /* 1: revisable drafts (noise canvas); 0: absorbing MASK positions */
} dg_sampler;

/* ---- sizes and status ------------------------------------------------------------------ */

/* Bytes of scratch the calls below need for `batch` canvases of `n_tokens` tokens each and a
 * cache of `cache_cap` rows per (layer, batch, kv head), on the current device (the attention's
 * key-split plan depends on its SM count).  0 on an invalid config. */
size_t dg_workspace_size(const dg_config *cfg, int batch, int n_tokens, int cache_cap);

/* Synchronises `stream`, copies *dev_status to the host and returns it (DG_ERR_CUDA if the
 * copy fails).  Does not clear it; dg_clear_status() zeroes it asynchronously. */
int dg_read_status(const int32_t *dev_status, void *stream);
int dg_clear_status(int32_t *dev_status, void *stream);

/* Last CUDA error string seen by this thread's calls (static storage, never NULL). */
const char *dg_last_cuda_error(void);

/* Number of kernels this process has launched through the library (monotone counter). */
uint64_t dg_launch_count(void);

/* Profiling aid (host side, per calling thread): after dg_profile_begin(max_records) every
 * kernel launch of the library first records a CUDA timing event on its stream (up to
 * max_records).  dg_profile_mark(stream) records a closing event labelled "(mark)".
 * dg_profile_end synchronises on the last event, writes ms[i] = time from record i to record
 * i + 1 (i < *n_out <= max_out) and stops recording; dg_profile_name(i) is record i's kernel
 * name ("" when out of range).  Events are created once and reused; no device memory is
 * allocated.  Under stream capture the records become external event-record nodes, so the
 * times are those of the graph's replay (call dg_profile_end after the replay). */
int dg_profile_begin(int max_records);
int dg_profile_mark(void *stream);
int dg_profile_end(float *ms, int max_out, int *n_out);
const char *dg_profile_name(int i);

/* Diagnostic of the bounded device-side wait (not a step of the method).  Every wait inside the
 * library's tensor-core kernels gives up after about 2 s (4e9 SM cycles): the kernel then records
 * DG_ERR_TIMEOUT in *dev_status, waits (again bounded) for what it has issued, frees its tensor
 * memory and returns, so a stalled kernel never hangs the device.  This probe runs that wait
 * primitive alone: one CTA allocates tensor memory and waits at most limit_cycles (1 .. 4e9) on
 * an mbarrier phase that completes only if `arrive` != 0 (the probe arrives on it itself); no
 * copy or MMA is issued.  On expiry *dev_status gets DG_ERR_TIMEOUT (first error wins); either
 * way the tensor memory is freed and the context stays usable. */
int dg_debug_wait_probe(long long limit_cycles, int arrive, int32_t *dev_status, void *stream);

/* ---- the hot-path operations ------------------------------------------------------------ */

/* Canvas attention, "DiffusionGemma Technical Report", Figure 4 (bidirectional attention
 * across the canvas, cross-attention to the KV cache) and the model card's "Model Overview".
 * For canvas b, query token i, query head h (kv head g = h / (Hq/Hkv)):
 *   o = softmax(q K^T / sqrt(hd)) V over keys = cache rows [0, cache_len[b]) followed by the
 *   n_tokens new rows; causal = 0: every new key visible (decoder); causal = 1: new key j
 *   visible iff j <= i (causal encoder, used by the append).  Cache rows are all visible.
 *   q      [B][n_tokens][Hq][hd]        k_cache, v_cache [B][Hkv][cache_cap][hd] (one layer)
 *   k_new, v_new [B][Hkv][n_tokens][hd] out [B][n_tokens][Hq][hd]
 *   cache_len: device int32[B], each <= cache_cap.  done: device int32[B] or NULL; canvases
 *   with done[b] != 0 are skipped (their `out` rows are left as they were).
 * Range: with bf16 activations the tensor-core kernels (head_dim 64 and 128) convert V to fp16
 *   for the P V product; every bf16 value of magnitude below 65520 is exact there, larger ones
 *   become +-inf and make the affected outputs non-finite.  Keep |v| < 65520 (K and q have no
 *   such limit). */
int dg_canvas_attn(const dg_config *cfg, int batch, int n_tokens, const void *q,
                   const void *k_cache, const void *v_cache, const int32_t *cache_len,
                   int cache_cap, const void *k_new, const void *v_new, int causal,
                   const int32_t *done, void *out, void *ws, size_t ws_bytes,
                   int32_t *dev_status, void *stream);

/* Router top-k and token permutation, model card "diffusiongemma", "Mixture-of-Experts (MoE)
 * Efficiency" (8 active of 128) and "DiffusionGemma Technical Report", Table 1.
 * z = y W_r^T (fp32), p = softmax(z) over all E, the k largest p (lower expert index first on
 * equal values), renormalised to sum 1.  Then assignments (t, j) are grouped by expert,
 * stable in (t, j) order:
 *   y [T][d]; topk_idx int32 [T][k + S]; topk_w fp32 [T][k + S] (S = n_shared: slots
 *   k .. k + S - 1 hold the shared experts E .. E + S - 1 with weight 1); expert_off int32
 *   [E + S + 1] (exclusive prefix of per-expert counts); perm int32 [T (k + S)]: perm[p] =
 *   t (k + S) + j of the assignment at permuted position p; inv_perm: the inverse.
 *   token_live: device uint8 [T] or NULL; a token with token_live[t] == 0 gets no experts
 *   (topk_idx = -1, weight 0) and no assignments. */
int dg_moe_route(const dg_config *cfg, int n_tokens, const void *y, const void *w_router,
                 const uint8_t *token_live, int32_t *topk_idx, float *topk_w,
                 int32_t *expert_off, int32_t *perm, int32_t *inv_perm, void *ws,
                 size_t ws_bytes, int32_t *dev_status, void *stream);

/* Expert FFN with combine and residual (same passages).  For assignment (t, j) with expert e:
 *   [g; u] = y_t W_gu,e^T ; a = gelu_tanh(g) * u (stored in the activation type) ;
 *   Y = a W_d,e^T (fp32) ;
 *   out_t = residual_t + sum_j topk_w[t][j] Y_(t,j), summed in fp32 in slot order
 *   j = 0 .. k + S - 1 (the shared experts' slots last, weight 1).
 * Routing arrays as produced by dg_moe_route.  y [T][d] in the activation type; residual and
 * out [T][d] fp32 (out may not alias y; it may alias residual). */
int dg_moe_ffn(const dg_config *cfg, int n_tokens, const void *y, const int32_t *topk_idx,
               const float *topk_w, const int32_t *expert_off, const int32_t *perm,
               const int32_t *inv_perm, const dg_layer_weights *lw, const void *residual,
               void *out, void *ws, size_t ws_bytes, int32_t *dev_status, void *stream);

/* Final RMSNorm, LM head and fused softmax entropy / greedy argmax, per masked position
 * ("DiffusionGemma Technical Report", explanatory visual: the entropy-bounded sampler consumes
 * per-position confidence; Table 1: vocabulary 262k; model card, Benchmark Results: EB sampler).
 * For r < n_rows (or < *n_rows_dev when that pointer is non-NULL), with source row
 * s = row_idx ? row_idx[r] : r:
 *   f = RMSNorm(h_s) (stored in the activation type);  z = f W_lm^T over ids [0, V) (fp32);
 *   entropy[s] = -sum_v p_v ln p_v with p = softmax(z);  argmax[s] = first index of max z.
 *   h [*][d] fp32 (residual stream); w_lm = the embedding [V + 1][d] in the activation type
 *   (rows [0, V) used); entropy fp32, argmax int32
 *   indexed by source row; logits_dbg fp32 [n_rows][V] or NULL (written when non-NULL).
 * A non-finite logit sets DG_ERR_NUMERIC. */
int dg_logits_entropy(const dg_config *cfg, int n_rows, const int32_t *n_rows_dev,
                      const void *h, const int32_t *row_idx, const void *w_lm, float *entropy,
                      int32_t *argmax, float *logits_dbg, void *ws, size_t ws_bytes,
                      int32_t *dev_status, void *stream);

/* dg_logits_entropy with the LM head in NVFP4 (cfg->emb_dtype DG_NVFP4): w_codes, w_scale and
 * w_scale_global hold the [V + 1][d] embedding in the NVFP4 layout above; the logits are
 * z = f (e2m1 * e4m3)^T, accumulated in fp32 from the normalised rows f stored in fp16 and the
 * exact fp16 products e2m1 * e4m3, then times w_scale_global.  (The same holds for the final
 * RMSNorm rows of dg_canvas_step with an NVFP4 model.)  Other arguments, outputs and errors as
 * dg_logits_entropy; DG_ERR_INVALID_ARG if cfg->emb_dtype is not DG_NVFP4. */
int dg_logits_entropy_nvfp4(const dg_config *cfg, int n_rows, const int32_t *n_rows_dev,
                            const void *h, const int32_t *row_idx, const uint8_t *w_codes,
                            const uint8_t *w_scale, float w_scale_global, float *entropy,
                            int32_t *argmax, float *logits_dbg, void *ws, size_t ws_bytes,
                            int32_t *dev_status, void *stream);

/* Entropy-bounded selection and commit (model card "diffusiongemma", Benchmark Results: the
 * EB sampler; "DiffusionGemma Technical Report", What they did: adaptive stopping).  The
 * pages name the sampler but print no formula; the rule is the published EB sampler
 * (Ben-Hamu et al., 2025): for each canvas b with done[b] == 0, order its masked positions by
 * entropy ascending (negative values and -0 as 0; lower position first on ties) and commit the
 * first k for the largest k >= 1 with  sum_{i<k} Q(H_(i)) <= Q(gamma), where
 * Q(H) = nearest integer to H * 2^32 (ties to even) and Q(gamma) = floor(gamma * 2^32)
 * (+inf: no bound).  When step[b] >= max_steps - 1 every masked position is committed.
 * Commit: tokens[b][i] = argmax[b][i], masked[b][i] = 0, selected[b][i] = 1.  Then
 * n_masked[b] -= k, step[b] += 1, done[b] = (n_masked[b] == 0).
 *   entropy fp32 [B][C] and argmax int32 [B][C] are read at masked positions only;
 *   tokens int32, masked uint8, selected uint8 (or NULL) [B][C]; n_masked, done, step int32 [B].
 * revise != 0 (the noise canvas's revisable drafts, see dg_sampler): every masked position that
 * is not committed also takes tokens[b][i] = argmax[b][i] and stays masked.
 * canvas <= 1024, gamma >= 0.  A non-finite entropy at a masked position sets DG_ERR_NUMERIC
 * and leaves that canvas unchanged. */
int dg_eb_select(int batch, int canvas, const float *entropy, const int32_t *argmax,
                 double gamma, int max_steps, int32_t *tokens, uint8_t *masked,
                 uint8_t *selected, int32_t *n_masked, int32_t *done, int32_t *step, int revise,
                 int32_t *dev_status, void *stream);

/* Encode & append ("DiffusionGemma Technical Report", Figure 4, stage 3; model card,
 * "Model Overview"): run the causal encoder (the decoder's weights, causal within the new
 * tokens, full visibility of the cache) over tokens [B][n_tokens] (device int32, ids in
 * [0, V]) at positions cache_len[b] + i, write every layer's K/V (after RoPE) into cache rows
 * [cache_len[b], cache_len[b] + n_tokens), then cache_len[b] += n_tokens.  Also used to
 * prefill a prompt in chunks.  k_cache, v_cache: [L][B][Hkv][cache_cap][hd].  A canvas whose
 * rows would pass cache_cap is left unchanged and sets DG_ERR_CAPACITY.  forced_topk: NULL, or
 * int32 [n_layers][B n_tokens][k] expert ids used instead of each layer's router top-k (see
 * dg_canvas_step). */
int dg_kv_append(const dg_config *cfg, const dg_model *model, int batch, const int32_t *tokens,
                 int n_tokens, void *k_cache, void *v_cache, int32_t *cache_len, int cache_cap,
                 const int32_t *forced_topk, void *ws, size_t ws_bytes, int32_t *dev_status,
                 void *stream);

/* Autoregressive mode ("DiffusionGemma Technical Report", What they did: the fine-tuned weights
 * still run as a standard autoregressive model, leaving room for hybrid diffusion-AR decoding;
 * "Limits and open work": routing requests between diffusion and AR decoding).  Reading: the
 * causal encoder is the AR model.  For each sequence b, tokens[b][0 .. n_tokens) (device int32,
 * ids in [0, V)) are appended to the cache exactly as by dg_kv_append, the last layer also runs
 * its attention and expert FFN, and the final RMSNorm + LM head of the last new row give the
 * next token: next_token[b] = argmax z (greedy), or with smp->tau_start > 0 a draw from
 * softmax(z / tau_start) by the Gumbel-max rule of dg_sampler on the stream of counter
 * (v >> 2, p, 0, (3 << 24) | b), p = cache_len[b] + n_tokens (the predicted token's position;
 * tau_end and revise are not used).  entropy[b] (or NULL): the entropy of that distribution.
 * logits_dbg (or NULL): fp32 [B][V] raw logits.  forced_topk (or NULL): int32
 * [n_layers][B n_tokens][k] expert ids (see dg_canvas_step).  Then cache_len[b] += n_tokens.
 * The next token is not appended: pass it as the next call's token.  A diffusion canvas and AR
 * tokens may follow one another on the same cache (hybrid decoding).  Workspace as
 * dg_workspace_size(cfg, batch, n_tokens, cache_cap).  Errors as dg_kv_append. */
int dg_ar_step(const dg_config *cfg, const dg_model *model, int batch, const int32_t *tokens,
               int n_tokens, void *k_cache, void *v_cache, int32_t *cache_len, int cache_cap,
               const dg_sampler *smp, int32_t *next_token, float *entropy, float *logits_dbg,
               const int32_t *forced_topk, void *ws, size_t ws_bytes, int32_t *dev_status,
               void *stream);

/* One denoising step of every live canvas ("DiffusionGemma Technical Report", Figure 4,
 * stage 2 and the explanatory visual): embed the canvas (masked positions as MASK = V), run
 * the n_layers decoder layers (pre-norm RMSNorm; GQA attention with RoPE at absolute positions
 * cache_len[b] + i over the cache plus the canvas, bidirectional; output projection + residual;
 * RMSNorm; top-k MoE FFN + residual), then for the masked positions the final RMSNorm, LM head
 * entropy / argmax and the EB select-and-commit of dg_eb_select.  Canvases with done[b] != 0
 * are left unchanged.  State arrays as in dg_eb_select.  k_cache, v_cache
 * [L][B][Hkv][cache_cap][hd] are read only (the canvas's own K/V live in `ws`).
 * entropy_out fp32 [B][C], argmax_out int32 [B][C] (or NULL): written at the positions that
 * were masked when the step began.  logits_dbg (or NULL): fp32 [B C][V], row b C + i written for
 * each such position (debug and parity only; costs a full logits write).  expert_load (or
 * NULL): int32 [n_layers][E + S], the number of (token, slot) assignments each expert received in
 * each layer this step (for load monitoring and byte accounting).  forced_topk (or NULL):
 * int32 [n_layers][B C][k] expert ids that replace each layer's router top-k choice (the gates
 * are still the softmax of this step's router logits over the given experts).  It lets a caller
 * reproduce another computation's expert choices exactly — e.g. to compare a deep stack with a
 * reference, where bf16 rounding legitimately flips near-tied routing decisions; bf16 models
 * with a tensor-core router only (DG_ERR_UNSUPPORTED otherwise). */
int dg_canvas_step(const dg_config *cfg, const dg_model *model, int batch, int32_t *tokens,
                   uint8_t *masked, int32_t *n_masked, int32_t *done, int32_t *step,
                   int max_steps, double gamma, const void *k_cache, const void *v_cache,
                   const int32_t *cache_len, int cache_cap, float *entropy_out,
                   int32_t *argmax_out, float *logits_dbg, int32_t *expert_load,
                   const int32_t *forced_topk, void *ws, size_t ws_bytes, int32_t *dev_status,
                   void *stream);

/* dg_canvas_step with a sampler variant (dg_sampler, non-NULL): the temperature-annealed
 * Gumbel-max draw of each masked position's token (tau_s of its canvas's step; argmax_out then
 * holds the drawn tokens and entropy_out the entropies at tau_s), and with smp->revise the
 * revisable drafts of a noise canvas.  logits_dbg stays the raw z.  Other arguments, outputs and
 * errors as dg_canvas_step (no expert_load).  DG_ERR_INVALID_ARG for a non-finite temperature. */
int dg_canvas_step_sampler(const dg_config *cfg, const dg_model *model, int batch,
                           int32_t *tokens, uint8_t *masked, int32_t *n_masked, int32_t *done,
                           int32_t *step, int max_steps, double gamma, const dg_sampler *smp,
                           const void *k_cache, const void *v_cache, const int32_t *cache_len,
                           int cache_cap, float *entropy_out, int32_t *argmax_out,
                           float *logits_dbg, const int32_t *forced_topk, void *ws,
                           size_t ws_bytes, int32_t *dev_status, void *stream);

/* Uniform-noise canvases (see dg_sampler): tokens[b][i] = (w0 * vocab) >> 32 for the first word
 * w0 of Philox4x32-10 at counter (i, 0, 0, (2 << 24) | b) keyed by the seed; masked = 1 (every
 * position a revisable draft), n_masked[b] = canvas, done[b] = 0, step[b] = 0.  Device arrays as
 * in dg_eb_select; canvas <= 1024. */
int dg_noise_canvas(int batch, int canvas, int vocab, uint64_t seed, int32_t *tokens,
                    uint8_t *masked, int32_t *n_masked, int32_t *done, int32_t *step,
                    void *stream);

/* Device-resident generation: dg_canvas_step repeated on the device until every canvas is done
 * ("DiffusionGemma Technical Report", explanatory visual: a canvas is refined over a number of
 * steps until confident and stable; Figure 4 stage 3: the finished canvas goes back through the
 * causal encoder), with no host round trip per step, then, if `append` is non-zero, dg_kv_append
 * of the canvases' final tokens (n_tokens = canvas; their cache_len grows by canvas).
 * The steps run as one CUDA graph: a while node whose body is one step and a one-thread kernel
 * that keeps the loop going while some done[b] is 0, *dev_status (if non-NULL) is DG_OK and fewer
 * than max_steps + 1 iterations have run.  Every canvas finishes within max_steps steps (D7), so
 * the bound only ends a loop that a device error (DG_ERR_NUMERIC, DG_ERR_TIMEOUT) has stalled;
 * the error is then in *dev_status.  Canvases already done are skipped, as in dg_canvas_step.
 * Arguments, layouts and errors as dg_canvas_step and dg_kv_append (k_cache and v_cache are
 * written only by the append; with append, cache_cap >= canvas).  The instantiated graph is
 * cached inside the library per argument set (device, config, weight pointers, state, cache and
 * scratch pointers, sizes, max_steps, gamma, sampler values; at most 8, least recent dropped), so
 * repeated calls with the same buffers launch one graph.  Not capturable into another graph;
 * profiling (dg_profile_begin) must be off while a new argument set is first used.
 * smp (or NULL: greedy): the sampler variant of every step, as dg_canvas_step_sampler. */
int dg_generate(const dg_config *cfg, const dg_model *model, int batch, int32_t *tokens,
                uint8_t *masked, int32_t *n_masked, int32_t *done, int32_t *step, int max_steps,
                double gamma, const dg_sampler *smp, void *k_cache, void *v_cache,
                int32_t *cache_len, int cache_cap, int append, void *ws, size_t ws_bytes,
                int32_t *dev_status, void *stream);

/* ---- fixed-scratch entry point ---------------------------------------------------------- */

/* dg_logits_entropy for callers that cannot provide device scratch memory.  The pages have no
 * counterpart: this is a library-integration variant, not a step of the method.  Some callers
 * cannot allocate device memory at all — an engine that has reserved the whole device for its
 * own pools, or a plugin whose host owns every allocation — so this call takes no `ws` and keeps
 * its scratch in a fixed array of DG_STATIC_SCRATCH_BYTES inside the library's device image,
 * which every GPU that loads the library holds until the process exits.  It allocates nothing.
 *   Same arguments and results as dg_logits_entropy, without logits_dbg and ws.
 *   Limits: bf16 activations and a bf16 LM head (DG_ERR_UNSUPPORTED otherwise; NVFP4 takes
 *   dg_logits_entropy_nvfp4), n_rows <= 256, d_model <= 2048,
 *   vocab <= 262144; larger requests return DG_ERR_WORKSPACE and launch nothing.
 *   The array's device address belongs to the CUDA context that loaded the library's module:
 *   every call made outside stream capture looks it up in the calling thread's current context
 *   (cudaGetSymbolAddress; it also sets up the device's primary context if none is current),
 *   and a call made while `stream` is being captured reuses the address found by an earlier
 *   call in the same context — so the first call in each context must come before any stream
 *   capture there (a first call inside a capture returns DG_ERR_CUDA).
 *   Config checks and errors as dg_logits_entropy (DG_ERR_INVALID_ARG on a malformed config).
 *   All calls share the one array and it keeps the last call's contents (nothing in it has to
 *   start at zero): calls whose work overlaps on the GPU — on different streams, or from
 *   different threads — race on it and must be serialised by the caller. */
#define DG_STATIC_SCRATCH_BYTES (6u * 1024u * 1024u + 4096u)
int dg_logits_entropy_static(const dg_config *cfg, int n_rows, const int32_t *n_rows_dev,
                             const void *h, const int32_t *row_idx, const void *w_lm,
                             float *entropy, int32_t *argmax, int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_H */
