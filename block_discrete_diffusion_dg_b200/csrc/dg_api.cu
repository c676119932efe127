// C ABI of the canvas-step library: argument checks, the scratch layout, and the chaining of the
// kernels into the operations declared in include/dg.h.  Nothing here allocates device memory or
// synchronises; every launch goes to the caller's stream.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

// NVTX range over one entry point's host work (its checks and launches); a profiler projects it
// onto the kernels it launched, so a timeline groups them under the call (and the layer) that
// issued them.  Without an attached tool the calls return at once.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  // a range named `name` carrying an integer payload (the layer index)
  NvtxRange(const char *name, int payload) {
    nvtxEventAttributes_t a{};
    a.version = NVTX_VERSION;
    a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    a.messageType = NVTX_MESSAGE_TYPE_ASCII;
    a.message.ascii = name;
    a.payloadType = NVTX_PAYLOAD_TYPE_INT32;
    a.payload.iValue = payload;
    nvtxRangePushEx(&a);
  }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

static std::atomic<unsigned long long> g_launches{0};
static thread_local char g_err[256] = "no error";

// Per-thread launch timeline for dg_profile_*: one event recorded before every launch.
struct Profile {
  std::vector<cudaEvent_t> ev;
  std::vector<const char *> name;
  int n = 0;
  bool on = false;
};
static thread_local Profile g_prof;

void note_launch(cudaStream_t s, const char *name) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_prof.on && g_prof.n < (int)g_prof.ev.size()) {
    // inside stream capture the record becomes a graph node whose timestamp is taken at replay
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cs);
    if (cs == cudaStreamCaptureStatusActive)
      cudaEventRecordWithFlags(g_prof.ev[g_prof.n], s, cudaEventRecordExternal);
    else
      cudaEventRecord(g_prof.ev[g_prof.n], s);
    g_prof.name[g_prof.n] = name;
    ++g_prof.n;
  }
}

bool &pdl_allowed() {
  static thread_local bool on = true;
  return on;
}

int check_launch(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return DG_OK;
  snprintf(g_err, sizeof(g_err), "%s: %s", what, cudaGetErrorString(e));
  return DG_ERR_CUDA;
}

namespace {

// Rows per grouped-GEMM tile: the tensor-core expert GEMM's token tile, or the CUDA-core GEMM's
// 64-row tile; the scratch tile list is sized for the smaller of the two.
constexpr int SIMT_TILE_M = 64;
inline int min_tile_m() {
  return experts_tc_tile_tokens() < SIMT_TILE_M ? experts_tc_tile_tokens() : SIMT_TILE_M;
}

inline size_t align_up(size_t v) { return (v + 255) & ~size_t(255); }
inline size_t esz(int dt) { return dt == DG_F32 ? 4 : (dt == DG_BF16 ? 2 : 1); }

enum Buf {
  B_X, B_A, B_QKV, B_CS, B_Q, B_KN, B_VN, B_O, B_H, B_Y, B_IDX, B_W, B_OFF, B_PERM, B_INV,
  B_TILES, B_NTILES, B_U, B_ACT, B_YE, B_XP, B_Z, B_WDQ, B_LIVE, B_ROWS, B_NROWS, B_SLOT, B_FIN, B_LOGITS, B_PART,
  B_ENT, B_AM, B_ATTN, B_HP, B_GEN, B_PCNT, B_COUNT
};

struct Layout {
  size_t off[B_COUNT];
  size_t total;
  int max_tiles;
};

// K slices of the split-K projections for T tokens (1: the projection runs unsplit).
int router_type(const dg_config *c);
int qkv_parts(const dg_config &c, int T) {
  const int N = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim, K = c.d_model;
  return split_supported(c.act_dtype, c.w_dtype, T, N, K) ? split_k_slices(N, K) : 1;
}
int o_parts(const dg_config &c, int T) {
  const int N = c.d_model, K = c.n_q_heads * c.head_dim;
  return split_supported(c.act_dtype, c.w_dtype, T, N, K) ? split_k_slices(N, K) : 1;
}
int router_parts(const dg_config &c, int T) {
  // few channel tiles: cap the slices, or the partials outweigh the router's weights
  return split_supported(c.act_dtype, router_type(&c), T, c.n_experts, c.d_model)
             ? split_k_slices(c.n_experts, c.d_model, 8)
             : 1;
}

Layout make_layout(const dg_config &c, int batch, int n, int cap) {
  const size_t T = (size_t)batch * n, a = esz(c.act_dtype);
  // routing slots and experts include the shared experts
  const size_t d = c.d_model, hd = c.head_dim, k = c.top_k + c.n_shared, F = c.d_ff;
  const size_t qkvw = (size_t)(c.n_q_heads + 2 * c.n_kv_heads) * hd;
  const size_t TK = T * k;
  Layout L;
  L.max_tiles = (int)((TK + min_tile_m() - 1) / min_tile_m()) + c.n_experts + c.n_shared;
  size_t sz[B_COUNT];
  const size_t T128 = (T + 127) / 128 * 128;  // tensor-core A operands read whole 128-row tiles
  sz[B_X] = T * d * 4;  // residual stream: fp32
  sz[B_A] = T128 * d * a;
  sz[B_QKV] = T * qkvw * 4 * qkv_parts(c, (int)T);
  sz[B_CS] = T * hd * 4;
  sz[B_Q] = T * c.n_q_heads * hd * a;
  sz[B_KN] = T * c.n_kv_heads * hd * a;
  sz[B_VN] = T * c.n_kv_heads * hd * a;
  sz[B_O] = T128 * c.n_q_heads * hd * a;
  sz[B_H] = T * d * 4;
  sz[B_Y] = T128 * d * a;
  sz[B_Z] = T * (size_t)c.n_experts * 4 * router_parts(c, (int)T);
  sz[B_IDX] = TK * 4;
  sz[B_W] = TK * 4;
  sz[B_OFF] = (size_t)(c.n_experts + c.n_shared + 1) * 4;
  sz[B_PERM] = TK * 4;
  sz[B_INV] = TK * 4;
  sz[B_TILES] = (size_t)L.max_tiles * sizeof(GroupTile);
  sz[B_NTILES] = 4;
  sz[B_U] = TK * 2 * F * 4;
  sz[B_ACT] = TK * F * a;
  sz[B_YE] = TK * d * 4;  // expert outputs: fp32
  sz[B_XP] = TK * d * a;
  // e4m3 weights on the tensor-core path: bf16 copies of one layer's matrices (the expert
  // matrices are the largest; QKV and the output projection reuse the front of the region)
  sz[B_WDQ] = c.w_dtype == DG_E4M3
                  ? ((size_t)(c.n_experts + c.n_shared) * 3 * F * d +
                     (size_t)(c.n_q_heads + 2 * c.n_kv_heads) * hd * d) * 2
                  : 0;
  sz[B_LIVE] = T;
  sz[B_ROWS] = T * 4;
  sz[B_NROWS] = 4;
  sz[B_SLOT] = T * 4;
  const bool tc_lm = lmhead_tc_supported(c.act_dtype, c.d_model);
  sz[B_FIN] = T128 * d * a;
  sz[B_LOGITS] = tc_lm ? 0 : T * (size_t)c.vocab * 4;
  sz[B_PART] = tc_lm ? lmhead_tc_ws_bytes((int)T, c.vocab) : 0;
  sz[B_ENT] = T * 4;
  sz[B_AM] = T * 4;
  { const int op = o_parts(c, (int)T); sz[B_HP] = op > 1 ? T * d * 4 * op : 0; }
  sz[B_GEN] = 16;  // dg_generate's loop counter
  sz[B_PCNT] = permute_scratch_bytes((int)TK, c.n_experts + c.n_shared);
  sz[B_ATTN] = attention_ws_bytes(c.act_dtype, batch, n, c.n_q_heads, c.n_kv_heads, c.head_dim,
                                  cap);
  size_t o = 0;
  for (int i = 0; i < B_COUNT; ++i) {
    L.off[i] = o;
    o += align_up(sz[i]);
  }
  L.total = o;
  return L;
}

struct Ws {
  char *base;
  const Layout *L;
  int32_t *st;  // the caller's device status word (may be null): bounded-wait timeouts land here
  template <typename P> P *at(Buf b) const { return reinterpret_cast<P *>(base + L->off[b]); }
};

}  // namespace

// Shape and dtype checks shared by every entry point (declared in dg_kernels.h).
bool cfg_ok(const dg_config *c) {
  if (!c) return false;
  if (c->d_model <= 0 || c->d_model % 8 || c->n_q_heads <= 0 || c->n_kv_heads <= 0) return false;
  if (c->n_q_heads % c->n_kv_heads) return false;
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) return false;
  if (c->n_experts <= 0 || c->n_experts > 256 || c->top_k <= 0 || c->top_k > c->n_experts ||
      c->top_k > 32)
    return false;
  if (c->n_shared < 0 || c->n_experts + c->n_shared > 256 || c->top_k + c->n_shared > 32)
    return false;
  if (c->d_ff <= 0 || c->d_ff % 8 || c->vocab < 2 || c->canvas <= 0 || c->canvas > 1024)
    return false;
  if (c->n_layers <= 0) return false;
  if (!(c->rope_theta > 0.0) || !(c->rms_eps >= 0.0)) return false;
  if (c->act_dtype == DG_F32) return c->w_dtype == DG_F32 && c->emb_dtype == DG_F32;
  if (c->act_dtype != DG_BF16 || (c->w_dtype != DG_BF16 && c->w_dtype != DG_E4M3)) return false;
  if (c->emb_dtype == DG_NVFP4) return c->d_model % 256 == 0 && c->d_model <= 4096;
  return c->emb_dtype == DG_BF16;
}

namespace {

// The tied embedding / LM head as the calls take it.
struct LmWeights {
  const void *w;             // bf16 / fp32 rows, or NVFP4 codes
  const uint8_t *scale;      // NVFP4 block scales (null otherwise)
  float g;                   // NVFP4 tensor scale
};

LmWeights lm_weights(const dg_config &c, const dg_model *m) {
  if (c.emb_dtype == DG_NVFP4) return LmWeights{m->emb, m->emb_scale, m->emb_scale_global};
  return LmWeights{m->emb, nullptr, 1.0f};
}

bool lm_weights_ok(const dg_config &c, const LmWeights &lw) {
  if (!lw.w) return false;
  if (c.emb_dtype != DG_NVFP4) return true;
  return lw.scale && std::isfinite(lw.g) && lw.g > 0.f && !((uintptr_t)lw.w & 15) &&
         !((uintptr_t)lw.scale & 15);
}

bool lw_ok(const dg_config *c, const dg_layer_weights *w) {
  if (!w || !w->w_qkv || !w->w_o || !w->w_router || !w->w_gate_up || !w->w_down) return false;
  if (c->w_dtype == DG_E4M3 && (!w->s_qkv || !w->s_o || !w->s_gate_up || !w->s_down))
    return false;
  return true;
}

int router_type(const dg_config *c) { return c->w_dtype == DG_F32 ? DG_F32 : DG_BF16; }
const float *scale_or_null(const dg_config *c, const float *s) {
  return c->w_dtype == DG_E4M3 ? s : nullptr;
}

#define DG_TRY(x)                 \
  do {                            \
    const int rc__ = (x);         \
    if (rc__ != DG_OK) return rc__; \
  } while (0)

// ---- one layer's pieces, shared by the step and the append --------------------------------

// The weights the tensor-core GEMMs read: bf16 weights as given; e4m3 weights dequantised into the
// B_WDQ scratch at element offset `off` (the per-channel scales are applied in the epilogues).
const void *tc_weight(const dg_config &c, const Ws &ws, const void *w, size_t n, size_t off,
                      cudaStream_t s, int *rc) {
  *rc = DG_OK;
  if (c.w_dtype != DG_E4M3) return w;
  bf16 *dst = ws.at<bf16>(B_WDQ) + off;
  *rc = launch_dequant_e4m3(w, n, dst, s);
  return dst;
}

int qkv_proj(const dg_config &c, const dg_layer_weights &w, const Ws &ws, int T, cudaStream_t s) {
  GemmDesc g{};
  g.act = c.act_dtype; g.w = c.w_dtype;
  g.A = ws.at<void>(B_A); g.lda = c.d_model;
  g.B = w.w_qkv; g.ldb = c.d_model; g.strideB = 0;
  g.bscale = scale_or_null(&c, w.s_qkv);
  g.M = T; g.N = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim; g.K = c.d_model;
  g.name = "gemm_qkv";
  if (gemm_tc_supported(c.act_dtype, c.w_dtype, c.d_model)) {
    int rc;
    const void *wq = tc_weight(c, ws, w.w_qkv, (size_t)g.N * c.d_model, 0, s, &rc);
    if (rc != DG_OK) return rc;
    const int parts = qkv_parts(c, T);
    if (parts > 1)
      return launch_gemm_tc_split(wq, g.N, ws.at<void>(B_A), T, (T + 127) / 128 * 128, c.d_model,
                                  parts, ws.at<float>(B_QKV), "gemm_qkv_tc", ws.st, s, g.bscale,
                                  wq == w.w_qkv);
    return launch_gemm_tc_dense(ws.at<void>(B_A), T, wq, g.N, c.d_model, ws.at<float>(B_QKV),
                                nullptr, g.N, "gemm_qkv_tc", ws.st, s, g.bscale);
  }
  return launch_gemm_simt(g, EPI_F32, ws.at<void>(B_QKV), g.N, nullptr, s);
}

bool experts_tc(const dg_config &c) {
  return gemm_tc_supported(c.act_dtype, c.w_dtype, c.d_model) && c.d_ff % 64 == 0 &&
         c.d_model % 128 == 0;
}
bool router_tc(const dg_config &c) {
  return gemm_tc_supported(c.act_dtype, router_type(&c), c.d_model) && c.n_experts % 16 == 0;
}

// o -> h = x + o W_o^T -> y = RMSNorm(h) -> router top-k -> stable permutation (+ tile list for the
// tensor-core experts, built here when the router runs on tensor cores: *tiles_ready).
int attn_out_and_route(const dg_config &c, const dg_layer_weights &w, const Ws &ws, int T,
                       const uint8_t *token_live, int32_t *load_out, bool *tiles_ready,
                       cudaStream_t s, const int32_t *forced = nullptr) {
  const int d = c.d_model, hq = c.n_q_heads * c.head_dim;
  GemmDesc g{};
  g.act = c.act_dtype; g.w = c.w_dtype;
  g.A = ws.at<void>(B_O); g.lda = hq;
  g.B = w.w_o; g.ldb = hq;
  g.bscale = scale_or_null(&c, w.s_o);
  g.M = T; g.N = d; g.K = hq;
  g.name = "gemm_o_resid";
  const int T128 = (T + 127) / 128 * 128;
  const int op = o_parts(c, T);
  if (op > 1) {  // split-K partials; the residual add happens in resid_norm
    int rc;
    const void *wo = tc_weight(c, ws, w.w_o, (size_t)d * hq, 0, s, &rc);
    if (rc != DG_OK) return rc;
    DG_TRY(launch_gemm_tc_split(wo, d, ws.at<void>(B_O), T, T128, hq, op, ws.at<float>(B_HP),
                                "gemm_o_resid_tc", ws.st, s, g.bscale, wo == w.w_o));
    DG_TRY(launch_resid_norm(c.act_dtype, ws.at<float>(B_HP), op, ws.at<float>(B_X), T, d,
                             c.rms_eps, ws.at<float>(B_H), ws.at<void>(B_Y), s));
  } else {
    if (gemm_tc_supported(c.act_dtype, c.w_dtype, hq)) {
      int rc;
      const void *wo = tc_weight(c, ws, w.w_o, (size_t)d * hq, 0, s, &rc);
      if (rc != DG_OK) return rc;
      DG_TRY(launch_gemm_tc_dense(ws.at<void>(B_O), T, wo, d, hq, ws.at<float>(B_H),
                                  ws.at<float>(B_X), d, "gemm_o_resid_tc", ws.st, s, g.bscale));
    } else
      DG_TRY(launch_gemm_simt(g, EPI_RESID, ws.at<void>(B_H), d, ws.at<void>(B_X), s));
    DG_TRY(launch_rmsnorm(c.act_dtype, ws.at<void>(B_H), nullptr, nullptr, T, d, c.rms_eps,
                          ws.at<void>(B_Y), s));
  }
  *tiles_ready = false;
  if (router_tc(c)) {
    const int rp = router_parts(c, T);
    if (rp > 1)
      DG_TRY(launch_gemm_tc_split(w.w_router, c.n_experts, ws.at<void>(B_Y), T, T128, d, rp,
                                  ws.at<float>(B_Z), "router_logits_tc", ws.st, s, nullptr,
                                  true));
    else
      DG_TRY(launch_gemm_tc_dense(ws.at<void>(B_Y), T, w.w_router, c.n_experts, d,
                                  ws.at<float>(B_Z), nullptr, c.n_experts, "router_logits_tc",
                                  ws.st, s));
    const bool tc = experts_tc(c);
    DG_TRY(launch_route(T, c.n_experts, c.top_k, ws.at<float>(B_Z), token_live,
                        ws.at<int32_t>(B_IDX), ws.at<float>(B_W), ws.at<int32_t>(B_OFF),
                        ws.at<int32_t>(B_PERM), ws.at<int32_t>(B_INV),
                        tc ? experts_tc_tile_tokens() : SIMT_TILE_M, ws.at<GroupTile>(B_TILES),
                        ws.at<int32_t>(B_NTILES), ws.L->max_tiles, load_out, s, forced, rp,
                        c.n_shared, ws.at<int32_t>(B_PCNT)));
    *tiles_ready = true;
    return DG_OK;
  }
  if (forced) return DG_ERR_UNSUPPORTED;  // forced routing needs the tensor-core router
  DG_TRY(launch_router(c.act_dtype, router_type(&c), T, d, c.n_experts, c.top_k,
                       ws.at<void>(B_Y), w.w_router, token_live, ws.at<int32_t>(B_IDX),
                       ws.at<float>(B_W), s, c.n_shared));
  return launch_permute(T, c.top_k + c.n_shared, c.n_experts + c.n_shared, ws.at<int32_t>(B_IDX),
                        ws.at<int32_t>(B_OFF), ws.at<int32_t>(B_PERM), ws.at<int32_t>(B_INV), s);
}

// The expert FFN, then combine + residual into `out`; the combine also writes RMSNorm(out) to
// a_out (next layer's input) and/or to f_out rows slot[t] (final-norm rows), when given.
int moe_experts(const dg_config &c, const dg_layer_weights &w, const Ws &ws, int T,
                const void *y, const int32_t *topk_idx, const float *topk_w,
                const int32_t *expert_off, const int32_t *perm, const int32_t *inv_perm,
                const void *residual, void *out, cudaStream_t s, bool tiles_ready = false,
                int32_t *load_out = nullptr, void *a_out = nullptr,
                const int32_t *slot = nullptr, void *f_out = nullptr) {
  // every slot, the shared experts' included (experts n_experts .. n_experts + n_shared - 1)
  const int d = c.d_model, F = c.d_ff, E = c.n_experts + c.n_shared, k = c.top_k + c.n_shared;
  const int TK = T * k;
  const bool tc = experts_tc(c);
  if (!tiles_ready)
    DG_TRY(launch_build_tiles(E, expert_off, tc ? experts_tc_tile_tokens() : SIMT_TILE_M,
                              ws.at<GroupTile>(B_TILES), ws.at<int32_t>(B_NTILES),
                              ws.L->max_tiles, load_out, s));
  if (tc) {
    int rc;
    const size_t n_gu = (size_t)E * 2 * F * d, n_dn = (size_t)E * d * F;
    const void *wgu = tc_weight(c, ws, w.w_gate_up, n_gu, 0, s, &rc);
    if (rc != DG_OK) return rc;
    const void *wdn = tc_weight(c, ws, w.w_down, n_dn, n_gu, s, &rc);
    if (rc != DG_OK) return rc;
    const bool e4 = c.w_dtype == DG_E4M3;
    DG_TRY(launch_gather_rows(TK, d, k, perm, expert_off, E, y, ws.at<void>(B_XP), s));
    DG_TRY(launch_gemm_tc_experts(1, wgu, E, 2 * F, F, ws.at<void>(B_XP), TK, d,
                                  ws.at<GroupTile>(B_TILES), ws.at<int32_t>(B_NTILES),
                                  ws.L->max_tiles, expert_off, ws.at<void>(B_ACT), F,
                                  "moe_gate_up_tc", ws.st, s, e4 ? w.s_gate_up : nullptr));
    DG_TRY(launch_gemm_tc_experts(0, wdn, E, d, F, ws.at<void>(B_ACT), TK, F,
                                  ws.at<GroupTile>(B_TILES), ws.at<int32_t>(B_NTILES),
                                  ws.L->max_tiles, expert_off, ws.at<void>(B_YE), d,
                                  "moe_down_tc", ws.st, s, e4 ? w.s_down : nullptr));
  } else {
    GemmDesc g1{};
    g1.act = c.act_dtype; g1.w = c.w_dtype;
    g1.A = y; g1.lda = d; g1.a_rowmap = perm; g1.a_rowdiv = k;
    g1.B = w.w_gate_up; g1.ldb = d; g1.strideB = (long long)2 * F * d;
    g1.bscale = scale_or_null(&c, w.s_gate_up);
    g1.M = TK; g1.N = 2 * F; g1.K = d;
    g1.tiles = ws.at<GroupTile>(B_TILES); g1.n_tiles = ws.at<int32_t>(B_NTILES);
    g1.group_off = expert_off; g1.max_tiles = ws.L->max_tiles;
    g1.name = "moe_gemm_gate_up";
    DG_TRY(launch_gemm_simt(g1, EPI_F32, ws.at<void>(B_U), 2 * F, nullptr, s));
    DG_TRY(launch_gate(c.act_dtype, TK, F, ws.at<float>(B_U), expert_off, E, ws.at<void>(B_ACT), s));
    GemmDesc g2{};
    g2.act = c.act_dtype; g2.w = c.w_dtype;
    g2.A = ws.at<void>(B_ACT); g2.lda = F;
    g2.B = w.w_down; g2.ldb = F; g2.strideB = (long long)d * F;
    g2.bscale = scale_or_null(&c, w.s_down);
    g2.M = TK; g2.N = d; g2.K = F;
    g2.tiles = g1.tiles; g2.n_tiles = g1.n_tiles; g2.group_off = expert_off;
    g2.max_tiles = ws.L->max_tiles;
    g2.name = "moe_gemm_down";
    DG_TRY(launch_gemm_simt(g2, EPI_F32, ws.at<void>(B_YE), d, nullptr, s));
  }
  return launch_combine_norm(c.act_dtype, T, d, k, c.rms_eps, topk_idx, topk_w, inv_perm,
                             ws.at<void>(B_YE), residual, out, a_out, slot, f_out, s,
                             f_out && c.emb_dtype == DG_NVFP4);
}

// Final RMSNorm of rows row_idx[r] (r < *n_rows) of h, LM head, entropy/argmax at source rows.
// (h == nullptr: the normalised rows are already in the B_FIN scratch rows.)
int lm_entropy(const dg_config &c, const Ws &ws, int max_rows, const int32_t *n_rows_dev,
               const void *h, const int32_t *row_idx, const LmWeights &lw, float *entropy,
               int32_t *argmax, float *logits_out, int scatter_logits, int32_t *st,
               cudaStream_t s, const SampleSpec *smp = nullptr) {
  const void *w_lm = lw.w;
  if (h)  // an NVFP4 LM head multiplies fp16 rows
    DG_TRY(launch_rmsnorm(c.act_dtype, h, row_idx, n_rows_dev, max_rows, c.d_model, c.rms_eps,
                          ws.at<void>(B_FIN), s, c.emb_dtype == DG_NVFP4));
  if (c.emb_dtype == DG_NVFP4)
    return launch_lmhead_q4(ws.at<void>(B_FIN), max_rows, n_rows_dev,
                            static_cast<const uint8_t *>(lw.w), lw.scale, lw.g, c.vocab,
                            c.d_model, row_idx, entropy, argmax, logits_out,
                            scatter_logits ? row_idx : nullptr, ws.at<void>(B_PART), st, s, smp);
  if (lmhead_tc_supported(c.act_dtype, c.d_model))
    return launch_lmhead_tc(ws.at<void>(B_FIN), max_rows, n_rows_dev, w_lm, c.vocab, c.d_model,
                            row_idx, entropy, argmax, logits_out,
                            scatter_logits ? row_idx : nullptr, ws.at<void>(B_PART), st, s, smp);
  float *logits = (logits_out && !scatter_logits) ? logits_out : ws.at<float>(B_LOGITS);
  GemmDesc g{};
  g.act = c.act_dtype; g.w = c.act_dtype;
  g.A = ws.at<void>(B_FIN); g.lda = c.d_model;
  g.B = w_lm; g.ldb = c.d_model;
  g.M = max_rows; g.M_dev = n_rows_dev; g.N = c.vocab; g.K = c.d_model;
  g.name = "lm_head_logits";
  DG_TRY(launch_gemm_simt(g, EPI_F32, logits, c.vocab, nullptr, s));
  DG_TRY(launch_entropy_rows(logits, c.vocab, max_rows, n_rows_dev, row_idx, entropy, argmax, st,
                             s, smp));
  if (logits_out && scatter_logits)
    DG_TRY(launch_scatter_rows(logits, c.vocab, max_rows, n_rows_dev, row_idx, logits_out, s));
  return DG_OK;
}

long long quant_gamma(double gamma) {
  if (std::isinf(gamma)) return INT64_MAX;
  const double v = std::floor(gamma * 4294967296.0);
  if (v >= 9.2233720368547758e18) return INT64_MAX;
  return (long long)v;
}

bool sampler_ok(const dg_sampler *smp) {
  return !smp || (std::isfinite(smp->tau_start) && std::isfinite(smp->tau_end));
}

// The LM head's draw for canvas rows: greedy unless the schedule has a positive temperature.
SampleSpec canvas_spec(const dg_sampler *smp, const int32_t *step, int canvas, int max_steps) {
  SampleSpec sp{};
  if (!smp || !(smp->tau_start > 0.0 || smp->tau_end > 0.0)) return sp;
  sp.mode = SAMPLE_CANVAS;
  sp.step = step;
  sp.canvas = canvas;
  sp.max_steps = max_steps;
  sp.tau0 = smp->tau_start;
  sp.tau1 = smp->tau_end;
  sp.key0 = (uint32_t)(smp->seed & 0xFFFFFFFFu);
  sp.key1 = (uint32_t)(smp->seed >> 32);
  return sp;
}

int check_ws(const dg_config *c, int batch, int n, int cap, const void *ws, size_t ws_bytes,
             Layout *L) {
  *L = make_layout(*c, batch, n, cap);
  if (!ws) return DG_ERR_INVALID_ARG;
  if (((uintptr_t)ws) & 255) return DG_ERR_INVALID_ARG;
  if (ws_bytes < L->total) return DG_ERR_WORKSPACE;
  return DG_OK;
}

}  // namespace
}  // namespace dg

namespace dg {
namespace {

// Condition of dg_generate's device loop (one thread, after the step's EB kernel): run the body
// again while some canvas is not done, no device error has been recorded, and fewer than `cap`
// iterations have run (the cap ends the loop even if an error keeps a canvas from finishing).
__global__ void gen_cond_kernel(cudaGraphConditionalHandle h, const int32_t *done, int batch,
                                int32_t *iter, int cap, const int32_t *st) {
  int running = 0;
  for (int b = 0; b < batch; ++b) running |= (done[b] == 0);
  const int it = *iter + 1;
  *iter = it;
  const bool ok = st == nullptr || *st == DG_OK;
  cudaGraphSetConditional(h, (running && ok && it < cap) ? 1u : 0u);
}

// A stream of this thread for capturing graph bodies (one per device).
cudaStream_t capture_stream() {
  static thread_local cudaStream_t streams[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!streams[dev]) cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking);
  return streams[dev];
}

// Records a failed CUDA call (dg_last_cuda_error) and returns DG_ERR_CUDA.
int cuda_fail(const char *what, cudaError_t e) {
  (void)cudaGetLastError();
  snprintf(g_err, sizeof(g_err), "%s: %s", what, cudaGetErrorString(e));
  return DG_ERR_CUDA;
}

// Instantiated device-loop graphs, keyed by every argument that is baked into them.
struct GenCache {
  std::mutex mu;
  std::vector<std::pair<std::string, cudaGraphExec_t>> entries;  // most recent last
};
GenCache &gen_cache() {
  static GenCache c;
  return c;
}
constexpr size_t GEN_CACHE_MAX = 8;

template <typename T> void key_add(std::string &k, const T &v) {
  k.append(reinterpret_cast<const char *>(&v), sizeof(T));
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" {

size_t dg_workspace_size(const dg_config *cfg, int batch, int n_tokens, int cache_cap) {
  if (!cfg_ok(cfg) || batch <= 0 || n_tokens <= 0 || cache_cap < 0) return 0;
  return make_layout(*cfg, batch, n_tokens, cache_cap).total;
}

int dg_read_status(const int32_t *dev_status, void *stream) {
  if (!dev_status) return DG_ERR_INVALID_ARG;
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, dev_status, 4, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) {
    snprintf(g_err, sizeof(g_err), "dg_read_status: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return h;
}

int dg_clear_status(int32_t *dev_status, void *stream) {
  if (!dev_status) return DG_ERR_INVALID_ARG;
  const cudaError_t e = cudaMemsetAsync(dev_status, 0, 4, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    snprintf(g_err, sizeof(g_err), "dg_clear_status: %s", cudaGetErrorString(e));
    return DG_ERR_CUDA;
  }
  return DG_OK;
}

const char *dg_last_cuda_error(void) { return g_err; }

uint64_t dg_launch_count(void) { return g_launches.load(); }

int dg_profile_begin(int max_records) {
  if (max_records <= 0) return DG_ERR_INVALID_ARG;
  while ((int)g_prof.ev.size() < max_records) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return check_launch("dg_profile_begin");
    g_prof.ev.push_back(e);
    g_prof.name.push_back(nullptr);
  }
  g_prof.n = 0;
  g_prof.on = true;
  return DG_OK;
}

int dg_profile_mark(void *stream) {
  if (!g_prof.on) return DG_ERR_INVALID_ARG;
  note_launch((cudaStream_t)stream, "(mark)");
  g_launches.fetch_sub(1, std::memory_order_relaxed);  // a mark is not a kernel
  return DG_OK;
}

int dg_profile_end(float *ms, int max_out, int *n_out) {
  if (!g_prof.on) return DG_ERR_INVALID_ARG;
  g_prof.on = false;
  const int n = g_prof.n;
  if (n > 0 && cudaEventSynchronize(g_prof.ev[n - 1]) != cudaSuccess)
    return check_launch("dg_profile_end");
  int k = 0;
  for (int i = 0; i + 1 < n && k < max_out; ++i, ++k) {
    float t = 0.f;
    cudaEventElapsedTime(&t, g_prof.ev[i], g_prof.ev[i + 1]);
    if (ms) ms[k] = t;
  }
  if (n_out) *n_out = k;
  return DG_OK;
}

const char *dg_profile_name(int i) {
  if (i < 0 || i >= g_prof.n || !g_prof.name[i]) return "";
  return g_prof.name[i];
}

int dg_debug_wait_probe(long long limit_cycles, int arrive, int32_t *dev_status, void *stream) {
  if (limit_cycles < 1 || limit_cycles > 4000000000LL || !dev_status) return DG_ERR_INVALID_ARG;
  return launch_wait_probe(limit_cycles, arrive ? 1 : 0, dev_status, (cudaStream_t)stream);
}

int dg_canvas_attn(const dg_config *cfg, int batch, int n_tokens, const void *q,
                   const void *k_cache, const void *v_cache, const int32_t *cache_len,
                   int cache_cap, const void *k_new, const void *v_new, int causal,
                   const int32_t *done, void *out, void *ws, size_t ws_bytes,
                   int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_canvas_attn");
  if (!cfg_ok(cfg) || batch <= 0 || n_tokens <= 0 || cache_cap < 0) return DG_ERR_INVALID_ARG;
  if (!q || !cache_len || !k_new || !v_new || !out) return DG_ERR_INVALID_ARG;
  if (cache_cap > 0 && (!k_cache || !v_cache)) return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, batch, n_tokens, cache_cap, ws, ws_bytes, &L));
  return launch_attention(cfg->act_dtype, batch, n_tokens, cfg->n_q_heads, cfg->n_kv_heads,
                          cfg->head_dim, q, k_cache, v_cache, cache_len, cache_cap, k_new, v_new,
                          causal ? 1 : 0, done, out, (char *)ws + L.off[B_ATTN], dev_status,
                          (cudaStream_t)stream);
}

int dg_moe_route(const dg_config *cfg, int n_tokens, const void *y, const void *w_router,
                 const uint8_t *token_live, int32_t *topk_idx, float *topk_w,
                 int32_t *expert_off, int32_t *perm, int32_t *inv_perm, void *ws,
                 size_t ws_bytes, int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_moe_route");
  if (!cfg_ok(cfg) || n_tokens <= 0) return DG_ERR_INVALID_ARG;
  if (!y || !w_router || !topk_idx || !topk_w || !expert_off || !perm || !inv_perm)
    return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, 1, n_tokens, 0, ws, ws_bytes, &L));
  const cudaStream_t s = (cudaStream_t)stream;
  Ws w{(char *)ws, &L, dev_status};
  const int d = cfg->d_model, E = cfg->n_experts;
  if (gemm_tc_supported(cfg->act_dtype, router_type(cfg), d) && E % 16 == 0) {
    // the tensor-core router reads whole 128-row tiles: stage y into the padded scratch rows
    const cudaError_t e = cudaMemcpyAsync(w.at<void>(B_Y), y, (size_t)n_tokens * d * esz(cfg->act_dtype),
                                          cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return check_launch("dg_moe_route copy");
    DG_TRY(launch_gemm_tc_dense(w.at<void>(B_Y), n_tokens, w_router, E, d, w.at<float>(B_Z), nullptr,
                                E, "router_logits_tc", w.st, s));
    DG_TRY(launch_router_topk(n_tokens, E, cfg->top_k, w.at<float>(B_Z), token_live, topk_idx,
                              topk_w, s, nullptr, 1, cfg->n_shared));
  } else {
    DG_TRY(launch_router(cfg->act_dtype, router_type(cfg), n_tokens, d, E, cfg->top_k, y,
                         w_router, token_live, topk_idx, topk_w, s, cfg->n_shared));
  }
  return launch_permute(n_tokens, cfg->top_k + cfg->n_shared, cfg->n_experts + cfg->n_shared,
                        topk_idx, expert_off, perm, inv_perm, s);
}

int dg_moe_ffn(const dg_config *cfg, int n_tokens, const void *y, const int32_t *topk_idx,
               const float *topk_w, const int32_t *expert_off, const int32_t *perm,
               const int32_t *inv_perm, const dg_layer_weights *lw, const void *residual,
               void *out, void *ws, size_t ws_bytes, int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_moe_ffn");
  if (!cfg_ok(cfg) || n_tokens <= 0 || !lw_ok(cfg, lw)) return DG_ERR_INVALID_ARG;
  if (!y || !topk_idx || !topk_w || !expert_off || !perm || !inv_perm || !residual || !out)
    return DG_ERR_INVALID_ARG;
  if (out == y) return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, 1, n_tokens, 0, ws, ws_bytes, &L));
  Ws w{(char *)ws, &L, dev_status};
  return moe_experts(*cfg, *lw, w, n_tokens, y, topk_idx, topk_w, expert_off, perm, inv_perm,
                     residual, out, (cudaStream_t)stream);
}

int dg_logits_entropy(const dg_config *cfg, int n_rows, const int32_t *n_rows_dev,
                      const void *h, const int32_t *row_idx, const void *w_lm, float *entropy,
                      int32_t *argmax, float *logits_dbg, void *ws, size_t ws_bytes,
                      int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_logits_entropy");
  if (!cfg_ok(cfg) || cfg->emb_dtype == DG_NVFP4 || n_rows <= 0 || !h || !w_lm || !entropy ||
      !argmax)
    return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, 1, n_rows, 0, ws, ws_bytes, &L));
  Ws w{(char *)ws, &L, dev_status};
  return lm_entropy(*cfg, w, n_rows, n_rows_dev, h, row_idx, LmWeights{w_lm, nullptr, 1.0f},
                    entropy, argmax, logits_dbg, 0, dev_status, (cudaStream_t)stream);
}

int dg_logits_entropy_nvfp4(const dg_config *cfg, int n_rows, const int32_t *n_rows_dev,
                            const void *h, const int32_t *row_idx, const uint8_t *w_codes,
                            const uint8_t *w_scale, float w_scale_global, float *entropy,
                            int32_t *argmax, float *logits_dbg, void *ws, size_t ws_bytes,
                            int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_logits_entropy_nvfp4");
  if (!cfg_ok(cfg) || cfg->emb_dtype != DG_NVFP4 || n_rows <= 0 || !h || !entropy || !argmax)
    return DG_ERR_INVALID_ARG;
  const LmWeights lw{w_codes, w_scale, w_scale_global};
  if (!lm_weights_ok(*cfg, lw)) return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, 1, n_rows, 0, ws, ws_bytes, &L));
  Ws w{(char *)ws, &L, dev_status};
  return lm_entropy(*cfg, w, n_rows, n_rows_dev, h, row_idx, lw, entropy, argmax, logits_dbg, 0,
                    dev_status, (cudaStream_t)stream);
}

int dg_eb_select(int batch, int canvas, const float *entropy, const int32_t *argmax,
                 double gamma, int max_steps, int32_t *tokens, uint8_t *masked,
                 uint8_t *selected, int32_t *n_masked, int32_t *done, int32_t *step, int revise,
                 int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_eb_select");
  if (batch <= 0 || canvas <= 0 || canvas > 1024 || max_steps <= 0) return DG_ERR_INVALID_ARG;
  if (!(gamma >= 0.0)) return DG_ERR_INVALID_ARG;
  if (!entropy || !argmax || !tokens || !masked || !n_masked || !done || !step)
    return DG_ERR_INVALID_ARG;
  return launch_eb_select(batch, canvas, entropy, argmax, quant_gamma(gamma), max_steps, tokens,
                          masked, selected, n_masked, done, step, dev_status,
                          (cudaStream_t)stream, revise ? 1 : 0);
}

int dg_kv_append(const dg_config *cfg, const dg_model *model, int batch, const int32_t *tokens,
                 int n_tokens, void *k_cache, void *v_cache, int32_t *cache_len, int cache_cap,
                 const int32_t *forced_topk, void *ws, size_t ws_bytes, int32_t *dev_status,
                 void *stream) {
  const NvtxRange nvtx_range("dg_kv_append");
  if (!cfg_ok(cfg) || !model || !model->layers || !model->emb || batch <= 0 || n_tokens <= 0)
    return DG_ERR_INVALID_ARG;
  if (!tokens || !k_cache || !v_cache || !cache_len || cache_cap <= 0) return DG_ERR_INVALID_ARG;
  if (n_tokens > cache_cap) return DG_ERR_CAPACITY;
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!lw_ok(cfg, &model->layers[l])) return DG_ERR_INVALID_ARG;
  const LmWeights emb = lm_weights(*cfg, model);
  if (!lm_weights_ok(*cfg, emb)) return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, batch, n_tokens, cache_cap, ws, ws_bytes, &L));
  Ws w{(char *)ws, &L, dev_status};
  const dg_config &c = *cfg;
  const cudaStream_t s = (cudaStream_t)stream;
  const int T = batch * n_tokens, d = c.d_model;
  const size_t layer_elems = (size_t)batch * c.n_kv_heads * cache_cap * c.head_dim;
  const size_t ae = esz(c.act_dtype);
  DG_TRY(launch_prologue(c.act_dtype, tokens, nullptr, model->emb, T, d, c.vocab, c.rms_eps,
                         w.at<void>(B_X), w.at<void>(B_A), dev_status, batch, n_tokens, c.head_dim,
                         c.rope_theta, cache_len, w.at<float>(B_CS), nullptr, nullptr, nullptr,
                         nullptr, nullptr, s, emb.scale, emb.g));
  for (int l = 0; l < c.n_layers; ++l) {
    const NvtxRange layer_range("layer", l);
    const dg_layer_weights &lw = model->layers[l];
    char *kc = (char *)k_cache + l * layer_elems * ae;
    char *vc = (char *)v_cache + l * layer_elems * ae;
    DG_TRY(qkv_proj(c, lw, w, T, s));
    DG_TRY(launch_qkv_split(c.act_dtype, batch, n_tokens, c.n_q_heads, c.n_kv_heads, c.head_dim,
                            w.at<float>(B_QKV), qkv_parts(c, T), w.at<float>(B_CS), w.at<void>(B_Q),
                            w.at<void>(B_KN), w.at<void>(B_VN), kc, vc, cache_len, cache_cap,
                            dev_status, s));
    if (l + 1 == c.n_layers) break;
    DG_TRY(launch_attention(c.act_dtype, batch, n_tokens, c.n_q_heads, c.n_kv_heads, c.head_dim,
                            w.at<void>(B_Q), kc, vc, cache_len, cache_cap, w.at<void>(B_KN),
                            w.at<void>(B_VN), 1, nullptr, w.at<void>(B_O),
                            w.at<void>(B_ATTN), dev_status, s));
    bool tiles_ready = false;
    DG_TRY(attn_out_and_route(c, lw, w, T, nullptr, nullptr, &tiles_ready, s,
                              forced_topk ? forced_topk + (size_t)l * T * c.top_k : nullptr));
    // the combine also forms the next layer's normalised input
    DG_TRY(moe_experts(c, lw, w, T, w.at<void>(B_Y), w.at<int32_t>(B_IDX), w.at<float>(B_W),
                       w.at<int32_t>(B_OFF), w.at<int32_t>(B_PERM), w.at<int32_t>(B_INV),
                       w.at<void>(B_H), w.at<void>(B_X), s, tiles_ready, nullptr,
                       w.at<void>(B_A)));
  }
  return launch_add_cache_len(batch, n_tokens, cache_cap, cache_len, s);
}

int dg_ar_step(const dg_config *cfg, const dg_model *model, int batch, const int32_t *tokens,
               int n_tokens, void *k_cache, void *v_cache, int32_t *cache_len, int cache_cap,
               const dg_sampler *smp, int32_t *next_token, float *entropy, float *logits_dbg,
               const int32_t *forced_topk, void *ws, size_t ws_bytes, int32_t *dev_status,
               void *stream) {
  const NvtxRange nvtx_range("dg_ar_step");
  if (!cfg_ok(cfg) || !model || !model->layers || !model->emb || batch <= 0 || n_tokens <= 0)
    return DG_ERR_INVALID_ARG;
  if (!tokens || !k_cache || !v_cache || !cache_len || cache_cap <= 0 || !next_token)
    return DG_ERR_INVALID_ARG;
  if (!sampler_ok(smp)) return DG_ERR_INVALID_ARG;
  if (n_tokens > cache_cap) return DG_ERR_CAPACITY;
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!lw_ok(cfg, &model->layers[l])) return DG_ERR_INVALID_ARG;
  const LmWeights emb = lm_weights(*cfg, model);
  if (!lm_weights_ok(*cfg, emb)) return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, batch, n_tokens, cache_cap, ws, ws_bytes, &L));
  Ws w{(char *)ws, &L, dev_status};
  const dg_config &c = *cfg;
  const cudaStream_t s = (cudaStream_t)stream;
  const int T = batch * n_tokens, d = c.d_model;
  const size_t layer_elems = (size_t)batch * c.n_kv_heads * cache_cap * c.head_dim;
  const size_t ae = esz(c.act_dtype);
  int32_t *slot = w.at<int32_t>(B_SLOT);
  DG_TRY(launch_prologue(c.act_dtype, tokens, nullptr, model->emb, T, d, c.vocab, c.rms_eps,
                         w.at<void>(B_X), w.at<void>(B_A), dev_status, batch, n_tokens, c.head_dim,
                         c.rope_theta, cache_len, w.at<float>(B_CS), nullptr, nullptr, nullptr,
                         nullptr, nullptr, s, emb.scale, emb.g));
  DG_TRY(launch_last_row_slots(batch, n_tokens, slot, s));
  for (int l = 0; l < c.n_layers; ++l) {
    const NvtxRange layer_range("layer", l);
    const dg_layer_weights &lw = model->layers[l];
    char *kc = (char *)k_cache + l * layer_elems * ae;
    char *vc = (char *)v_cache + l * layer_elems * ae;
    DG_TRY(qkv_proj(c, lw, w, T, s));
    DG_TRY(launch_qkv_split(c.act_dtype, batch, n_tokens, c.n_q_heads, c.n_kv_heads, c.head_dim,
                            w.at<float>(B_QKV), qkv_parts(c, T), w.at<float>(B_CS), w.at<void>(B_Q),
                            w.at<void>(B_KN), w.at<void>(B_VN), kc, vc, cache_len, cache_cap,
                            dev_status, s));
    DG_TRY(launch_attention(c.act_dtype, batch, n_tokens, c.n_q_heads, c.n_kv_heads, c.head_dim,
                            w.at<void>(B_Q), kc, vc, cache_len, cache_cap, w.at<void>(B_KN),
                            w.at<void>(B_VN), 1, nullptr, w.at<void>(B_O),
                            w.at<void>(B_ATTN), dev_status, s));
    bool tiles_ready = false;
    DG_TRY(attn_out_and_route(c, lw, w, T, nullptr, nullptr, &tiles_ready, s,
                              forced_topk ? forced_topk + (size_t)l * T * c.top_k : nullptr));
    // the last layer's combine writes the final-norm row of each sequence's last token
    const bool last = l + 1 == c.n_layers;
    DG_TRY(moe_experts(c, lw, w, T, w.at<void>(B_Y), w.at<int32_t>(B_IDX), w.at<float>(B_W),
                       w.at<int32_t>(B_OFF), w.at<int32_t>(B_PERM), w.at<int32_t>(B_INV),
                       w.at<void>(B_H), w.at<void>(B_X), s, tiles_ready, nullptr,
                       last ? nullptr : w.at<void>(B_A), last ? slot : nullptr,
                       last ? w.at<void>(B_FIN) : nullptr));
  }
  SampleSpec sp{};
  if (smp && smp->tau_start > 0.0) {
    sp.mode = SAMPLE_AR;
    sp.pos = cache_len;
    sp.pos_add = n_tokens;
    sp.tau0 = smp->tau_start;
    sp.key0 = (uint32_t)(smp->seed & 0xFFFFFFFFu);
    sp.key1 = (uint32_t)(smp->seed >> 32);
  }
  DG_TRY(lm_entropy(c, w, batch, nullptr, nullptr, nullptr, emb,
                    entropy ? entropy : w.at<float>(B_ENT), next_token, logits_dbg, 0, dev_status,
                    s, &sp));
  return launch_add_cache_len(batch, n_tokens, cache_cap, cache_len, s);
}

}  // extern "C"

namespace dg {
namespace {

// One denoising step (dg_canvas_step), with the sampler variant `smp` (null: greedy argmax,
// entropy at tau = 1, masked positions embedded as MASK).
int canvas_step_impl(const dg_config *cfg, const dg_model *model, int batch, int32_t *tokens,
                     uint8_t *masked, int32_t *n_masked, int32_t *done, int32_t *step,
                     int max_steps, double gamma, const void *k_cache, const void *v_cache,
                     const int32_t *cache_len, int cache_cap, float *entropy_out,
                     int32_t *argmax_out, float *logits_dbg, int32_t *expert_load,
                     const int32_t *forced_topk, const dg_sampler *smp, void *ws,
                     size_t ws_bytes, int32_t *dev_status, void *stream) {
  if (!cfg_ok(cfg) || !model || !model->layers || !model->emb || batch <= 0 || max_steps <= 0)
    return DG_ERR_INVALID_ARG;
  if (!sampler_ok(smp)) return DG_ERR_INVALID_ARG;
  if (!tokens || !masked || !n_masked || !done || !step || !cache_len) return DG_ERR_INVALID_ARG;
  if (cache_cap < 0 || (cache_cap > 0 && (!k_cache || !v_cache))) return DG_ERR_INVALID_ARG;
  if (!(gamma >= 0.0)) return DG_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!lw_ok(cfg, &model->layers[l])) return DG_ERR_INVALID_ARG;
  const LmWeights emb = lm_weights(*cfg, model);
  if (!lm_weights_ok(*cfg, emb)) return DG_ERR_INVALID_ARG;
  const dg_config &c = *cfg;
  const int C = c.canvas, T = batch * C, d = c.d_model;
  Layout L;
  DG_TRY(check_ws(cfg, batch, C, cache_cap, ws, ws_bytes, &L));
  Ws w{(char *)ws, &L, dev_status};
  const cudaStream_t s = (cudaStream_t)stream;
  const size_t layer_elems = (size_t)batch * c.n_kv_heads * cache_cap * c.head_dim;
  const size_t ae = esz(c.act_dtype);
  uint8_t *live = w.at<uint8_t>(B_LIVE);
  int32_t *rows = w.at<int32_t>(B_ROWS), *n_rows = w.at<int32_t>(B_NROWS);

  int32_t *slot = w.at<int32_t>(B_SLOT);
  const int revise = smp && smp->revise ? 1 : 0;
  DG_TRY(launch_prologue(c.act_dtype, tokens, masked, model->emb, T, d, c.vocab, c.rms_eps,
                         w.at<void>(B_X), w.at<void>(B_A), dev_status, batch, C, c.head_dim,
                         c.rope_theta, cache_len, w.at<float>(B_CS), done, rows, n_rows, slot, live,
                         s, emb.scale, emb.g, revise));
  for (int l = 0; l < c.n_layers; ++l) {
    const NvtxRange layer_range("layer", l);
    const dg_layer_weights &lw = model->layers[l];
    const char *kc = (const char *)k_cache + l * layer_elems * ae;
    const char *vc = (const char *)v_cache + l * layer_elems * ae;
    DG_TRY(qkv_proj(c, lw, w, T, s));
    DG_TRY(launch_qkv_split(c.act_dtype, batch, C, c.n_q_heads, c.n_kv_heads, c.head_dim,
                            w.at<float>(B_QKV), qkv_parts(c, T), w.at<float>(B_CS), w.at<void>(B_Q),
                            w.at<void>(B_KN), w.at<void>(B_VN), nullptr, nullptr, cache_len,
                            cache_cap, dev_status, s));
    DG_TRY(launch_attention(c.act_dtype, batch, C, c.n_q_heads, c.n_kv_heads, c.head_dim,
                            w.at<void>(B_Q), kc, vc, cache_len, cache_cap, w.at<void>(B_KN),
                            w.at<void>(B_VN), 0, done, w.at<void>(B_O), w.at<void>(B_ATTN),
                            dev_status, s));
    int32_t *load_l = expert_load ? expert_load + (size_t)l * (c.n_experts + c.n_shared) : nullptr;
    bool tiles_ready = false;
    DG_TRY(attn_out_and_route(c, lw, w, T, live, load_l, &tiles_ready, s,
                              forced_topk ? forced_topk + (size_t)l * T * c.top_k : nullptr));
    // the combine also forms the next layer's normalised input, or after the last layer the
    // final-norm rows of the masked positions (the LM head's input)
    const bool last = l + 1 == c.n_layers;
    DG_TRY(moe_experts(c, lw, w, T, w.at<void>(B_Y), w.at<int32_t>(B_IDX), w.at<float>(B_W),
                       w.at<int32_t>(B_OFF), w.at<int32_t>(B_PERM), w.at<int32_t>(B_INV),
                       w.at<void>(B_H), w.at<void>(B_X), s, tiles_ready, load_l,
                       last ? nullptr : w.at<void>(B_A), last ? slot : nullptr,
                       last ? w.at<void>(B_FIN) : nullptr));
  }
  float *ent = entropy_out ? entropy_out : w.at<float>(B_ENT);
  int32_t *am = argmax_out ? argmax_out : w.at<int32_t>(B_AM);
  const SampleSpec sp = canvas_spec(smp, step, C, max_steps);
  DG_TRY(lm_entropy(c, w, T, n_rows, nullptr, rows, emb, ent, am, logits_dbg, 1, dev_status,
                    s, &sp));
  return launch_eb_select(batch, C, ent, am, quant_gamma(gamma), max_steps, tokens, masked,
                          nullptr, n_masked, done, step, dev_status, s, revise);
}

}  // namespace
}  // namespace dg

extern "C" {

int dg_canvas_step(const dg_config *cfg, const dg_model *model, int batch, int32_t *tokens,
                   uint8_t *masked, int32_t *n_masked, int32_t *done, int32_t *step,
                   int max_steps, double gamma, const void *k_cache, const void *v_cache,
                   const int32_t *cache_len, int cache_cap, float *entropy_out,
                   int32_t *argmax_out, float *logits_dbg, int32_t *expert_load,
                   const int32_t *forced_topk, void *ws, size_t ws_bytes, int32_t *dev_status,
                   void *stream) {
  const NvtxRange nvtx_range("dg_canvas_step");
  return canvas_step_impl(cfg, model, batch, tokens, masked, n_masked, done, step, max_steps,
                          gamma, k_cache, v_cache, cache_len, cache_cap, entropy_out, argmax_out,
                          logits_dbg, expert_load, forced_topk, nullptr, ws, ws_bytes, dev_status,
                          stream);
}

int dg_canvas_step_sampler(const dg_config *cfg, const dg_model *model, int batch,
                           int32_t *tokens, uint8_t *masked, int32_t *n_masked, int32_t *done,
                           int32_t *step, int max_steps, double gamma, const dg_sampler *smp,
                           const void *k_cache, const void *v_cache, const int32_t *cache_len,
                           int cache_cap, float *entropy_out, int32_t *argmax_out,
                           float *logits_dbg, const int32_t *forced_topk, void *ws,
                           size_t ws_bytes, int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_canvas_step_sampler");
  if (!smp) return DG_ERR_INVALID_ARG;
  return canvas_step_impl(cfg, model, batch, tokens, masked, n_masked, done, step, max_steps,
                          gamma, k_cache, v_cache, cache_len, cache_cap, entropy_out, argmax_out,
                          logits_dbg, nullptr, forced_topk, smp, ws, ws_bytes, dev_status,
                          stream);
}

int dg_noise_canvas(int batch, int canvas, int vocab, uint64_t seed, int32_t *tokens,
                    uint8_t *masked, int32_t *n_masked, int32_t *done, int32_t *step,
                    void *stream) {
  const NvtxRange nvtx_range("dg_noise_canvas");
  if (batch <= 0 || canvas <= 0 || canvas > 1024 || vocab < 1) return DG_ERR_INVALID_ARG;
  if (!tokens || !masked || !n_masked || !done || !step) return DG_ERR_INVALID_ARG;
  return launch_noise_canvas(batch, canvas, vocab, (uint32_t)(seed & 0xFFFFFFFFu),
                             (uint32_t)(seed >> 32), tokens, masked, n_masked, done, step,
                             (cudaStream_t)stream);
}

int dg_generate(const dg_config *cfg, const dg_model *model, int batch, int32_t *tokens,
                uint8_t *masked, int32_t *n_masked, int32_t *done, int32_t *step, int max_steps,
                double gamma, const dg_sampler *smp, void *k_cache, void *v_cache,
                int32_t *cache_len, int cache_cap, int append, void *ws, size_t ws_bytes,
                int32_t *dev_status, void *stream) {
  const NvtxRange nvtx_range("dg_generate");
  if (!cfg_ok(cfg) || !model || !model->layers || !model->emb || batch <= 0 || max_steps <= 0)
    return DG_ERR_INVALID_ARG;
  if (!tokens || !masked || !n_masked || !done || !step || !cache_len) return DG_ERR_INVALID_ARG;
  if (cache_cap < 0 || (cache_cap > 0 && (!k_cache || !v_cache))) return DG_ERR_INVALID_ARG;
  if (append && (cache_cap <= 0 || cfg->canvas > cache_cap)) return DG_ERR_INVALID_ARG;
  if (!(gamma >= 0.0) || !sampler_ok(smp)) return DG_ERR_INVALID_ARG;
  for (int l = 0; l < cfg->n_layers; ++l)
    if (!lw_ok(cfg, &model->layers[l])) return DG_ERR_INVALID_ARG;
  if (!lm_weights_ok(*cfg, lm_weights(*cfg, model))) return DG_ERR_INVALID_ARG;
  Layout L;
  DG_TRY(check_ws(cfg, batch, cfg->canvas, cache_cap, ws, ws_bytes, &L));
  Ws w{(char *)ws, &L, dev_status};
  int32_t *iter = w.at<int32_t>(B_GEN);
  const cudaStream_t s = (cudaStream_t)stream;

  std::string key;
  int dev = 0;
  cudaGetDevice(&dev);
  key_add(key, dev);
  key_add(key, *cfg);
  key_add(key, model->emb);
  key_add(key, model->emb_scale);
  key_add(key, model->emb_scale_global);
  for (int l = 0; l < cfg->n_layers; ++l) key_add(key, model->layers[l]);
  const void *ptrs[] = {tokens, masked, n_masked, done, step, k_cache, v_cache, cache_len, ws,
                        dev_status};
  key.append(reinterpret_cast<const char *>(ptrs), sizeof(ptrs));
  key_add(key, batch);
  key_add(key, max_steps);
  key_add(key, gamma);
  const dg_sampler no_smp{0.0, 0.0, 0, 0};
  key_add(key, smp ? smp->tau_start : no_smp.tau_start);
  key_add(key, smp ? smp->tau_end : no_smp.tau_end);
  key_add(key, smp ? smp->seed : no_smp.seed);
  key_add(key, smp ? smp->revise : no_smp.revise);
  key_add(key, smp != nullptr);
  key_add(key, cache_cap);
  key_add(key, ws_bytes);

  // A cached graph is launched under the cache lock, so another thread cannot evict (destroy) it
  // between the lookup and the launch; a destroyed graph that is already launched finishes.
  cudaGraphExec_t exec = nullptr;
  cudaError_t launched = cudaErrorUnknown;
  {
    GenCache &gc = gen_cache();
    std::lock_guard<std::mutex> lock(gc.mu);
    for (auto &e : gc.entries)
      if (e.first == key) exec = e.second;
    if (exec) launched = cudaGraphLaunch(exec, s);
  }
  if (!exec) {
    // parent graph: reset the loop counter, then a while node whose body is one captured step
    // and the condition kernel.  Programmatic edges are tried first; without them if the body
    // does not take them.
    int rc = DG_ERR_CUDA;
    for (int attempt = 0; attempt < 2 && rc != DG_OK; ++attempt) {
      cudaGraph_t g = nullptr;
      cudaError_t e = cudaGraphCreate(&g, 0);
      if (e != cudaSuccess) return cuda_fail("cudaGraphCreate", e);
      cudaMemsetParams mp{};
      mp.dst = iter;
      mp.value = 0;
      mp.elementSize = 4;
      mp.width = 1;
      mp.height = 1;
      cudaGraphNode_t reset = nullptr, loop = nullptr;
      cudaGraphConditionalHandle h{};
      cudaGraphNodeParams cp{};
      e = cudaGraphAddMemsetNode(&reset, g, nullptr, 0, &mp);
      if (e == cudaSuccess) e = cudaGraphConditionalHandleCreate(&h, g, 1, cudaGraphCondAssignDefault);
      if (e == cudaSuccess) {
        cp.type = cudaGraphNodeTypeConditional;
        cp.conditional.handle = h;
        cp.conditional.type = cudaGraphCondTypeWhile;
        cp.conditional.size = 1;
        e = cudaGraphAddNode(&loop, g, &reset, 1, &cp);
      }
      cudaStream_t cs = capture_stream();
      if (e == cudaSuccess && !cs) e = cudaErrorInvalidDevice;
      if (e == cudaSuccess)
        e = cudaStreamBeginCaptureToGraph(cs, cp.conditional.phGraph_out[0], nullptr, nullptr, 0,
                                          cudaStreamCaptureModeThreadLocal);
      if (e != cudaSuccess) {
        cudaGraphDestroy(g);
        return cuda_fail("dg_generate graph", e);
      }
      pdl_allowed() = attempt == 0;
      int src = canvas_step_impl(cfg, model, batch, tokens, masked, n_masked, done, step,
                                 max_steps, gamma, k_cache, v_cache, cache_len, cache_cap, nullptr,
                                 nullptr, nullptr, nullptr, nullptr, smp, ws, ws_bytes, dev_status,
                                 cs);
      if (src == DG_OK) {
        gen_cond_kernel<<<1, 1, 0, cs>>>(h, done, batch, iter, max_steps + 1, dev_status);
        src = check_launch("gen_cond");
      }
      pdl_allowed() = true;
      cudaGraph_t body = nullptr;
      e = cudaStreamEndCapture(cs, &body);
      if (src == DG_OK && e == cudaSuccess) e = cudaGraphInstantiate(&exec, g, 0);
      cudaGraphDestroy(g);
      if (src != DG_OK && src != DG_ERR_CUDA) {
        (void)cudaGetLastError();
        return src;  // the step refused its arguments (checked above, so not expected)
      }
      if (src == DG_OK && e == cudaSuccess) {
        rc = DG_OK;
      } else {  // a launch or the graph was refused: once more without programmatic edges
        exec = nullptr;
        rc = src != DG_OK ? DG_ERR_CUDA : cuda_fail("dg_generate graph", e);
        (void)cudaGetLastError();
      }
    }
    if (rc != DG_OK) return rc;
    GenCache &gc = gen_cache();
    std::lock_guard<std::mutex> lock(gc.mu);
    if (gc.entries.size() >= GEN_CACHE_MAX) {
      cudaGraphExecDestroy(gc.entries.front().second);  // freed when its launches complete
      gc.entries.erase(gc.entries.begin());
    }
    gc.entries.emplace_back(key, exec);
    launched = cudaGraphLaunch(exec, s);
  }
  if (launched != cudaSuccess) return cuda_fail("dg_generate launch", launched);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!append) return DG_OK;
  return dg_kv_append(cfg, model, batch, tokens, cfg->canvas, k_cache, v_cache, cache_len,
                      cache_cap, nullptr, ws, ws_bytes, dev_status, stream);
}

}  // extern "C"
