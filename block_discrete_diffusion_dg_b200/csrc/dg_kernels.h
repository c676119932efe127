// Internal launchers of the canvas-step library (host functions, one per kernel family).
// Each returns DG_OK or DG_ERR_CUDA and never synchronises.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dg.h"

namespace dg {

// A tile of a grouped GEMM: rows [m0, m0 + tile) of group `g` (MoE expert).
struct GroupTile { int32_t g, m0; };

// ---- rows: embedding, RMSNorm, compaction (k_rows.cu) -----------------------------------
// x_out: fp32 residual stream rows; a_out: RMSNorm(x) in the activation type.
int launch_embed_norm(int act, const int32_t *tokens, const uint8_t *masked, const void *emb,
                      int rows, int d, int vocab, double eps, void *x_out, void *a_out,
                      int32_t *st, cudaStream_t s);
// Embedding + pre-norm of `rows` rows, the RoPE table, and (row_idx non-null) the compaction of
// the rows needing logits (row_idx, *n_rows, slot [rows]: index in row_idx or -1, token_live).
// drafts: masked rows are embedded by their token (a revisable draft) instead of MASK.
int launch_prologue(int act, const int32_t *tokens, const uint8_t *masked, const void *emb, int rows,
                    int d, int vocab, double eps, void *x_out, void *a_out, int32_t *st, int batch,
                    int n, int hd, double theta, const int32_t *cache_len, float *cs,
                    const int32_t *done, int32_t *row_idx, int32_t *n_rows, int32_t *slot,
                    uint8_t *token_live, cudaStream_t s, const uint8_t *emb_scale = nullptr,
                    float emb_g = 1.0f, int drafts = 0);
// Rows of an NVFP4 matrix of `rows` rows as stored (padded to a multiple of 256).
inline int nvfp4_rows_pad(int rows) { return (rows + 255) / 256 * 256; }
// e4m3 codes [n] -> bf16 [n] (n % 16 == 0), exact.
int launch_dequant_e4m3(const void *src, size_t n, void *dst, cudaStream_t s);
// in: fp32 rows (residual stream); out: activation type.
// h_out = res + sum of n_parts fp32 partials [n_parts][rows][d]; out = RMSNorm(h_out).
int launch_resid_norm(int act, const float *part, int n_parts, const float *res, int rows, int d,
                      double eps, float *h_out, void *out, cudaStream_t s);
// f16_out: out in fp16 instead (the rows an NVFP4 LM head multiplies).
int launch_rmsnorm(int act, const void *in, const int32_t *row_idx, const int32_t *n_rows_dev,
                   int max_rows, int d, double eps, void *out, cudaStream_t s, int f16_out = 0);
// live[b*C+i] = !done[b] && (masked == NULL || masked[b*C+i]); row_idx = positions with live
// set, in order; *n_rows = their count; token_live[t] = !done[b] (may be NULL).
int launch_compact_rows(int batch, int canvas, const uint8_t *masked, const int32_t *done,
                        int32_t *row_idx, int32_t *n_rows, uint8_t *token_live, cudaStream_t s);

// ---- GEMM on CUDA cores (k_gemm_simt.cu) --------------------------------------------------
// C[m][n] = sum_k A[arow(m)][k] * B[g][n][k] (* bscale[g][n]); fp32 accumulation in k order.
struct GemmDesc {
  int act, w;                  // element types of A and B (DG_F32 / DG_BF16 / DG_E4M3)
  const void *A; int lda;
  const void *B; int ldb; long long strideB;   // group stride of B in elements
  const float *bscale;         // [groups][N] or NULL
  int M, N, K;                 // M: rows (max rows if M_dev set)
  const int32_t *M_dev;        // device row count (<= M) or NULL
  const int32_t *a_rowmap;     // A row of output row m = a_rowmap[m] / a_rowdiv, or NULL
  int a_rowdiv;
  const GroupTile *tiles;      // grouped mode: tile list, count at *n_tiles, max_tiles
  const int32_t *n_tiles;
  const int32_t *group_off;    // grouped mode: row offsets [groups + 1]
  int max_tiles;
  const char *name;            // label for launch accounting / profiling
};
enum EpiKind { EPI_F32 = 0, EPI_ACT = 1, EPI_RESID = 2 };
// EPI_F32: out fp32 [M][ldo]; EPI_ACT: out act type; EPI_RESID: out = acc + res[m][n] (fp32).
int launch_gemm_simt(const GemmDesc &g, int epi, void *out, int ldo, const void *res,
                     cudaStream_t s);

// ---- RoPE and head split (k_rope.cu) -----------------------------------------------------
// Positions cache_len[b] + i; cos/sin of angle pos * theta^(-2j/hd) in fp64, stored fp32.
int launch_rope_table(int batch, int n, int hd, double theta, const int32_t *cache_len,
                      float *cs, cudaStream_t s);
// qkv fp32 [B*n][(Hq+2Hkv)hd] -> q [B*n][Hq][hd], k_new/v_new [B][Hkv][n][hd] (act type, RoPE
// on q and k).  If k_cache != NULL also writes k/v to cache rows cache_len[b] + i (< cap).
int launch_qkv_split(int act, int batch, int n, int Hq, int Hkv, int hd, const float *qkv,
                     int n_parts, const float *cs, void *q, void *k_new, void *v_new,
                     void *k_cache, void *v_cache, const int32_t *cache_len, int cap, int32_t *st,
                     cudaStream_t s);
int launch_add_cache_len(int batch, int n, int cap, int32_t *cache_len, cudaStream_t s);

// ---- attention (k_attn.cu) ----------------------------------------------------------------
int launch_attention(int act, int batch, int n, int Hq, int Hkv, int hd, const void *q,
                     const void *k_cache, const void *v_cache, const int32_t *cache_len,
                     int cap, const void *k_new, const void *v_new, int causal,
                     const int32_t *done, void *out, void *ws, int32_t *st, cudaStream_t s);
size_t attention_ws_bytes(int act, int batch, int n, int Hq, int Hkv, int hd, int cap);
// bf16 tensor-core path (k_attn_tc.cu): split-KV flash attention (tcgen05 for head_dim 128,
// mma.sync otherwise) + merge.  st: device status word (bounded-wait timeouts), may be NULL.
bool attention_tc_supported(int act, int Hq, int Hkv, int hd);
size_t attention_tc_ws_bytes(int batch, int n, int Hq, int Hkv, int hd, int cap);
int launch_attention_tc(int batch, int n, int Hq, int Hkv, int hd, const void *q,
                        const void *k_cache, const void *v_cache, const int32_t *cache_len, int cap,
                        const void *k_new, const void *v_new, int causal, const int32_t *done,
                        void *out, void *ws, int32_t *st, cudaStream_t s);

// ---- MoE (k_moe.cu) ---------------------------------------------------------------------------
// n_shared: shared experts E .. E + n_shared - 1 appended to every live token's slots (gate 1);
// the outputs are then [T][k + n_shared].
int launch_router(int act, int wr_type, int T, int d, int E, int k, const void *y,
                  const void *w_router, const uint8_t *token_live, int32_t *topk_idx,
                  float *topk_w, cudaStream_t s, int n_shared = 0);
// Top-k + gates from fp32 router logits z [T][E] (E <= 256, k <= 32), one warp per token.
int launch_router_topk(int T, int E, int k, const float *z, const uint8_t *token_live,
                       int32_t *topk_idx, float *topk_w, cudaStream_t s,
                       const int32_t *forced = nullptr,
                       int n_parts = 1, int n_shared = 0);
// Top-k + gates (router_topk, many blocks), then the stable permutation and the tile list in one
// block (permute_tiles).
int launch_route(int T, int E, int k, const float *z, const uint8_t *token_live, int32_t *topk_idx,
                 float *topk_w, int32_t *expert_off, int32_t *perm, int32_t *inv_perm, int tile_m,
                 GroupTile *tiles, int32_t *n_tiles, int max_tiles, int32_t *load_out,
                 cudaStream_t s, const int32_t *forced = nullptr,
                 int n_parts = 1, int n_shared = 0, int32_t *scratch = nullptr);
// The stable permutation and the tile list in one block (the second half of launch_route).
int launch_permute_tiles(int T, int E, int k, const int32_t *topk_idx, int32_t *expert_off,
                         int32_t *perm, int32_t *inv_perm, int tile_m, GroupTile *tiles,
                         int32_t *n_tiles, int max_tiles, int32_t *load_out, cudaStream_t s,
                         int n_shared = 0, int32_t *scratch = nullptr);
// Scratch the permutation needs beyond 2048 assignments (per-block counts); with scratch null
// there, one block does it all (slower).
size_t permute_scratch_bytes(int n_assign, int E);
// Builds expert_off [E+1] and perm/inv_perm [T k] (stable in flat order t k + j).
int launch_permute(int T, int k, int E, const int32_t *topk_idx, int32_t *expert_off,
                   int32_t *perm, int32_t *inv_perm, cudaStream_t s);
// Grouped-GEMM tile list from expert_off: tiles of tile_m rows, count at *n_tiles; the
// per-expert counts also go to load_out [E] when it is non-null.
int launch_build_tiles(int E, const int32_t *expert_off, int tile_m, GroupTile *tiles,
                       int32_t *n_tiles, int max_tiles, int32_t *load_out, cudaStream_t s);
// Scatter rows: dst[row_idx[r]][:] = src[r][:] for r < *n_rows.
int launch_scatter_rows(const float *src, int width, int max_rows, const int32_t *n_rows,
                        const int32_t *row_idx, float *dst, cudaStream_t s);
// X[p] = y[perm[p] / k] for p < expert_off[E]; bf16 rows of d elements (d % 8 == 0).
int launch_gather_rows(int rows_max, int d, int k, const int32_t *perm, const int32_t *expert_off,
                       int E, const void *y, void *X, cudaStream_t s);
// a = act(gelu_tanh(u[:, :F]) * u[:, F:]) for rows < expert_off[E].
int launch_gate(int act, int rows_max, int F, const float *u, const int32_t *expert_off, int E,
                void *a, cudaStream_t s);
// Combine and the following RMSNorm: out (fp32 residual stream) as launch_combine; then
// RMSNorm(out_t) in the activation type to a_out[t] (if non-null) and to f_out[slot[t]] (if
// slot non-null and slot[t] >= 0; in fp16 when f_out_f16, with bf16 activations).
int launch_combine_norm(int act, int T, int d, int k, double eps, const int32_t *topk_idx,
                        const float *topk_w, const int32_t *inv_perm, const void *Y,
                        const void *res, void *out, void *a_out, const int32_t *slot, void *f_out,
                        cudaStream_t s, int f_out_f16 = 0);
// out_t = res_t + sum_j w[t][j] Y[inv_perm[t k + j]]; res, Y and out fp32.
int launch_combine(int act, int T, int d, int k, const int32_t *topk_idx, const float *topk_w,
                   const int32_t *inv_perm, const void *Y, const void *res, void *out,
                   cudaStream_t s);

// ---- sampler variants (sampler.cuh) -----------------------------------------------------------
// How the LM-head kernels turn logits into a token: greedy (argmax, entropy at tau = 1), or the
// Gumbel-max draw at a per-row temperature (entropy of softmax(z / tau)) for canvas rows (source
// row b * canvas + i; tau annealed with step[b]) or autoregressive rows (source row b; tau0).
enum { SAMPLE_GREEDY = 0, SAMPLE_CANVAS = 1, SAMPLE_AR = 2 };
enum { SAMPLE_TAG_DENOISE = 1, SAMPLE_TAG_NOISE = 2, SAMPLE_TAG_AR = 3 };
struct SampleSpec {
  int mode;              // SAMPLE_*
  const int32_t *step;   // SAMPLE_CANVAS: per-canvas step counters (device)
  const int32_t *pos;    // SAMPLE_AR: per-sequence cache length before the append (device)
  int canvas, pos_add, max_steps;
  double tau0, tau1;     // temperature at step 0 and at step max_steps - 1
  uint32_t key0, key1;   // generator key: the seed's low and high words
};

// Uniform-noise canvases: tokens[b][i] = (w0 * vocab) >> 32 for the first word w0 of stream
// (TAG_NOISE, b, i, 0); masked = 1, n_masked = canvas, done = 0, step = 0.
int launch_noise_canvas(int batch, int canvas, int vocab, uint32_t key0, uint32_t key1,
                        int32_t *tokens, uint8_t *masked, int32_t *n_masked, int32_t *done,
                        int32_t *step, cudaStream_t s);
// slot[t] = b for the last of the n tokens of sequence b (t = b n + n - 1), -1 otherwise.
int launch_last_row_slots(int batch, int n, int32_t *slot, cudaStream_t s);

// Bounded-wait probe (k_debug.cu): one CTA holds TMEM and waits at most limit_cycles on an
// mbarrier phase that completes only if `arrive`; on expiry DG_ERR_TIMEOUT goes to *st.
int launch_wait_probe(long long limit_cycles, int arrive, int32_t *st, cudaStream_t s);

// ---- entropy / argmax (k_entropy.cu) -----------------------------------------------------------
// From materialised fp32 logits [rows][V]: per row r < *n_rows: H and argmax stored at
// out index row_idx ? row_idx[r] : r.
// smp (or null: greedy): the draw of each row's token (source row = row_idx ? row_idx[r] : r).
int launch_entropy_rows(const float *logits, int V, int max_rows, const int32_t *n_rows,
                        const int32_t *row_idx, float *entropy, int32_t *argmax, int32_t *st,
                        cudaStream_t s, const SampleSpec *smp = nullptr);

// ---- LM head on tensor cores with fused entropy (k_lmhead_tc.cu) ----------------------------
// F: normalised rows [roundup(max_rows, 128)][K] bf16 (rows >= *n_rows_dev ignored); w_lm [V][K].
// Entropy/argmax of row r stored at row_idx ? row_idx[r] : r.  logits (debug, may be null):
// row r written at logits_rows ? logits_rows[r] : r.  ws: lmhead_tc_ws_bytes(max_rows, V).
bool lmhead_tc_supported(int act, int d);
// The same with the weights in NVFP4 (codes and scales in the k-block-major layout of dg.h, rows
// padded to nvfp4_rows_pad(V + 1)) and F in fp16; logits = gscale * (F (e2m1 * e4m3)^T).
// K % 256 == 0.
int launch_lmhead_q4(const void *F, int max_rows, const int32_t *n_rows_dev, const uint8_t *codes,
                     const uint8_t *scales, float gscale, int V, int K, const int32_t *row_idx,
                     float *entropy, int32_t *argmax, float *logits, const int32_t *logits_rows,
                     void *ws, int32_t *st, cudaStream_t s, const SampleSpec *smp = nullptr);
size_t lmhead_tc_ws_bytes(int max_rows, int V);
// smp (or null: greedy): each row's token drawn as SampleSpec says (source row as the outputs);
// the debug logits stay the raw z.
int launch_lmhead_tc(const void *F, int max_rows, const int32_t *n_rows_dev, const void *w_lm,
                     int V, int K, const int32_t *row_idx, float *entropy, int32_t *argmax,
                     float *logits, const int32_t *logits_rows, void *ws, int32_t *st,
                     cudaStream_t s, const SampleSpec *smp = nullptr);

// ---- tensor-core GEMMs (k_gemm_tc.cu) -----------------------------------------------------------
bool gemm_tc_supported(int act, int w, int K);
// Swap-AB split-K projection for at most 256 tokens: part[s][t][n] (fp32) over K slices s.
// w_static: W is a model weight that no kernel of the stream writes (not a dequantised scratch
// copy), so the kernel may fetch it before waiting on the preceding kernel.
bool split_supported(int act, int w, int T, int N, int K);
int split_k_slices(int N, int K, int max_slices = 16);
int launch_gemm_tc_split(const void *W, int N, const void *X, int T, int T_alloc, int K,
                         int k_split, float *part, const char *name, int32_t *st, cudaStream_t s,
                         const float *scale, bool w_static);
// out[M][N] = A[M][K] W[N][K]^T (+ res[M][N]) in fp32; A has room for roundup(M, 128) rows.
// scale (or null): per output channel (W row), multiplies the fp32 accumulator.
int launch_gemm_tc_dense(const void *A, int M, const void *W, int N, int K, float *out,
                         const float *res, int ldo, const char *name, int32_t *st, cudaStream_t s,
                         const float *scale = nullptr);
// Swap-AB expert GEMM over token tiles of experts_tc_tile_tokens() rows.
int launch_gemm_tc_experts(int gate_up, const void *W, int E, int w_rows, int F, const void *X,
                           int n_assign_max, int K, const GroupTile *tiles,
                           const int32_t *n_tiles_dev, int max_tiles, const int32_t *expert_off,
                           void *out, int ld_out, const char *name, int32_t *st, cudaStream_t s,
                           const float *scale = nullptr);
int experts_tc_tile_tokens();

// ---- EB select (k_eb.cu) -------------------------------------------------------------------
// revise: masked positions that are not committed take argmax as their new draft token.
int launch_eb_select(int batch, int canvas, const float *entropy, const int32_t *argmax,
                     long long q_gamma, int max_steps, int32_t *tokens, uint8_t *masked,
                     uint8_t *selected, int32_t *n_masked, int32_t *done, int32_t *step,
                     int32_t *st, cudaStream_t s, int revise = 0);

}  // namespace dg
