// Mixture-of-experts routing and the element-wise parts of the expert FFN.
// Model card "diffusiongemma", "Mixture-of-Experts (MoE) Efficiency": 8 of 128 experts active per
// token; "DiffusionGemma Technical Report", Table 1: 8 / 128 experts.
//
// Router: z = y W_r^T in fp32 (fixed k order), p = softmax(z) over all E; the k largest p with the
// lower expert index first among equal values; gates renormalised to sum 1 — computed as a softmax
// over the selected logits, which is the same quantity.
// Permutation: assignments (t, j) grouped by expert, stable in flat order t k + j; expert_off is the
// exclusive prefix of the per-expert counts; the grouped GEMMs read a tile list built here.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int ROUTER_TPB = 4;  // tokens per router block

template <typename T, typename WT>
__global__ void router_kernel(int T_, int d, int E, int k, int S, const T *__restrict__ y,
                              const WT *__restrict__ wr, const uint8_t *__restrict__ token_live,
                              int32_t *topk_idx, float *topk_w) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float sm[];
  float *ys = sm;                        // [TPB][d]
  float *zs = sm + ROUTER_TPB * d;       // [TPB][E]
  const int t0 = blockIdx.x * ROUTER_TPB;
  for (int e = threadIdx.x; e < ROUTER_TPB * d; e += blockDim.x) {
    const int tt = e / d, c = e % d;
    ys[e] = (t0 + tt < T_) ? to_f(y[(size_t)(t0 + tt) * d + c]) : 0.f;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const WT *w = wr + (size_t)e * d;
    float acc[ROUTER_TPB];
#pragma unroll
    for (int tt = 0; tt < ROUTER_TPB; ++tt) acc[tt] = 0.f;
    for (int c = 0; c < d; ++c) {
      const float wv = to_f(w[c]);
#pragma unroll
      for (int tt = 0; tt < ROUTER_TPB; ++tt) acc[tt] = fmaf(ys[tt * d + c], wv, acc[tt]);
    }
#pragma unroll
    for (int tt = 0; tt < ROUTER_TPB; ++tt) zs[tt * E + e] = acc[tt];
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int tt = warp; tt < ROUTER_TPB; tt += blockDim.x >> 5) {
    const int t = t0 + tt;
    if (t >= T_) continue;
    const bool live = token_live == nullptr || token_live[t] != 0;
    const float *z = zs + tt * E;
    float zsel0 = 0.f, denom = 0.f;
    // selected set as a bitmask over the lane's experts e = lane + 32 i (E <= 256)
    unsigned taken = 0u;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
      for (int i = 0, e = lane; e < E; ++i, e += 32) {
        if (taken & (1u << i)) continue;
        const float v = z[e];
        if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (j == 0) zsel0 = bv;
      const float p = expf(bv - zsel0);
      denom += p;
      if (lane == 0) {
        topk_idx[(size_t)t * (k + S) + j] = live ? bi : -1;
        topk_w[(size_t)t * (k + S) + j] = p;  // normalised below
      }
    }
    __syncwarp();
    if (lane < k)
      topk_w[(size_t)t * (k + S) + lane] = live ? topk_w[(size_t)t * (k + S) + lane] / denom : 0.f;
    if (lane < S) {  // shared experts: every live token, gate 1, after the routed slots
      topk_idx[(size_t)t * (k + S) + k + lane] = live ? E + lane : -1;
      topk_w[(size_t)t * (k + S) + k + lane] = live ? 1.f : 0.f;
    }
  }
}

// Top-k and gates of one token by one warp, from its router logits held as zv[i] = z[lane + 32 i]
// (-inf past E): the k largest logits (lower expert index first on equal values), gates = softmax
// over the selected logits.  With `forced_row` non-null the k experts are forced_row[0..k-1] (in
// that order) instead; the gates are still the softmax over the selected logits.  Writes slots
// [0, k) and the S shared-expert slots after them (gate 1); a token that is not live gets -1 / 0.
__device__ __forceinline__ void route_warp(const float (&zv)[8], int E, int k, int S, bool live,
                                           const int32_t *__restrict__ forced_row,
                                           int32_t *idx_row, float *w_row) {
  const int lane = threadIdx.x & 31;
  if (forced_row) {
    const int e = lane < k ? forced_row[lane] : -1;
    const bool ok = e >= 0 && e < E;
    float mine_z = -INFINITY;
    const int src_lane = ok ? (e & 31) : 0, src_i = ok ? (e >> 5) : 0;
    // every lane fetches the logit its forced expert's owner holds (one shuffle per register)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = __shfl_sync(0xffffffffu, zv[i], src_lane);
      if (i == src_i) mine_z = v;
    }
    const float ze = ok ? mine_z : -INFINITY;
    const float z0 = __shfl_sync(0xffffffffu, ze, 0);
    const float p = (lane < k && ok) ? expf(ze - z0) : 0.f;
    float denom = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, o);
    if (lane < k) {
      idx_row[lane] = (live && ok) ? e : -1;
      w_row[lane] = (live && ok) ? p / denom : 0.f;
    }
  } else {
    unsigned taken = 0u;
    float z0 = 0.f, denom = 0.f, mine = 0.f;
    int my_idx = -1;
    for (int j = 0; j < k; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !(taken & (1u << i)) && (zv[i] > bv || (zv[i] == bv && e < bi))) {
          bv = zv[i];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
      if (j == 0) z0 = bv;
      const float p = expf(bv - z0);
      denom += p;
      if (lane == j) { mine = p; my_idx = bi; }
    }
    if (lane < k) {
      idx_row[lane] = live ? my_idx : -1;
      w_row[lane] = live ? mine / denom : 0.f;
    }
  }
  if (lane < S) {  // shared experts: every live token, gate 1, after the routed slots
    idx_row[k + lane] = live ? E + lane : -1;
    w_row[k + lane] = live ? 1.f : 0.f;
  }
}

// Top-k and gates from router logits z [T][E] (fp32), one warp per token (route_warp).
// z may hold n_parts fp32 partial sums [n_parts][T][E] (split-K router logits), added in order.
__global__ void router_topk_kernel(int T_, int E, int k, int S, const float *__restrict__ z,
                                   int n_parts, const uint8_t *__restrict__ token_live,
                                   const int32_t *__restrict__ forced, int32_t *topk_idx,
                                   float *topk_w) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T_) return;
  const bool live = token_live == nullptr || token_live[t] != 0;
  float zv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) zv[i] = 0.f;
  sum_parts8(z + (size_t)t * E, n_parts, (size_t)T_ * E, lane, 32, E, zv);
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (lane + 32 * i >= E) zv[i] = -INFINITY;
  route_warp(zv, E, k, S, live, forced ? forced + (size_t)t * k : nullptr,
             topk_idx + (size_t)t * (k + S), topk_w + (size_t)t * (k + S));
}

// Permutation and tile list in one block of 1024 threads (T k <= 65536, E <= 256): from the top-k
// expert ids (router_topk_kernel's output) the per-expert counts, expert_off, the stable grouping
// of the assignments by expert (as permute_kernel) and the grouped-GEMM tile list (as
// build_tiles_kernel), with the per-expert counts in load_out when it is non-null.
__global__ void __launch_bounds__(1024) permute_tiles_kernel(int n_assign, int E,
                                                             const int32_t *__restrict__ topk_idx,
                                                             int32_t *expert_off, int32_t *perm,
                                                             int32_t *inv_perm, int tile_m,
                                                             GroupTile *tiles, int32_t *n_tiles,
                                                             int max_tiles, int32_t *load_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt[256], off[257], running[256], toff[257];
  __shared__ int wc[32][256];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int e = tid; e < E; e += blockDim.x) { cnt[e] = 0; running[e] = 0; }
  __syncthreads();
  for (int a = tid; a < n_assign; a += blockDim.x) {
    const int e = topk_idx[a];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0, tacc = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = acc;
      toff[e] = tacc;
      acc += cnt[e];
      tacc += (cnt[e] + tile_m - 1) / tile_m;
    }
    off[E] = acc;
    toff[E] = tacc;
    *n_tiles = min(tacc, max_tiles);
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) expert_off[e] = off[e];
  for (int e = tid; e < E; e += blockDim.x) {
    if (load_out) load_out[e] = cnt[e];
    const int nt = toff[e + 1] - toff[e];
    for (int i = 0; i < nt; ++i) {
      const int slot = toff[e] + i;
      if (slot < max_tiles) tiles[slot] = GroupTile{e, i * tile_m};
    }
  }
  for (int c0 = 0; c0 < n_assign; c0 += blockDim.x) {
    for (int i = tid; i < 32 * E; i += blockDim.x) wc[i / E][i % E] = 0;
    __syncthreads();
    const int a = c0 + tid;
    int e = -1;
    if (a < n_assign) {
      e = topk_idx[a];
      if (e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank == 0) wc[w][e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int ww = 0; ww < w; ++ww) before += wc[ww][e];
      const int pos = off[e] + running[e] + before + rank;
      perm[pos] = a;
      inv_perm[a] = pos;
    } else if (a < n_assign) {
      inv_perm[a] = -1;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += blockDim.x) {
      int t = 0;
      for (int ww = 0; ww < 32; ++ww) t += wc[ww][ee];
      running[ee] += t;
    }
    __syncthreads();
  }
}

// The permutation and tile list for many assignments (more than 2048), in three launches over
// blocks of 2048 consecutive assignments, with the same outputs as permute_tiles_kernel:
//   perm_count: per block, the number of its assignments routed to each expert -> bcnt[blk][e];
//   perm_offsets (one block): expert offsets (exclusive scan of the totals), expert_off, counts,
//     the tile list, and each block's first position within each expert -> bcnt[blk][e];
//   perm_scatter: per block, the rank of each assignment among the same-expert ones of its block
//     (warp match + per-(expert, warp) counts, first half of a warp before the second, as in
//     permute_tiles_small_kernel) plus its block's first position.
// Assignments a0 = 64 w + lane and a1 = a0 + 32 of warp w, in increasing index order, so the
// grouping is stable in assignment order.
constexpr int PERM_CHUNK = 2048;

__global__ void __launch_bounds__(1024) perm_count_kernel(int n_assign, int E,
                                                          const int32_t *__restrict__ topk_idx,
                                                          int32_t *bcnt) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt[256];
  const int tid = threadIdx.x, blk = blockIdx.x;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int j = tid; j < PERM_CHUNK; j += blockDim.x) {
    const int a = blk * PERM_CHUNK + j;
    if (a < n_assign) {
      const int e = topk_idx[a];
      if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) bcnt[(size_t)blk * E + e] = cnt[e];
}

__global__ void __launch_bounds__(1024) perm_offsets_kernel(int n_blocks, int E, int32_t *bcnt,
                                                            int32_t *expert_off, int tile_m,
                                                            GroupTile *tiles, int32_t *n_tiles,
                                                            int max_tiles, int32_t *load_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ int tot[256], off[257], toff[257];
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += blockDim.x) {
    int t = 0;
    for (int b = 0; b < n_blocks; ++b) t += bcnt[(size_t)b * E + e];
    tot[e] = t;
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0, tacc = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = acc;
      toff[e] = tacc;
      acc += tot[e];
      tacc += (tot[e] + tile_m - 1) / tile_m;
    }
    off[E] = acc;
    toff[E] = tacc;
    *n_tiles = min(tacc, max_tiles);
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) expert_off[e] = off[e];
  for (int e = tid; e < E; e += blockDim.x) {
    if (load_out) load_out[e] = tot[e];
    int run = off[e];
    for (int b = 0; b < n_blocks; ++b) {  // block b's first position within expert e
      const int c = bcnt[(size_t)b * E + e];
      bcnt[(size_t)b * E + e] = run;
      run += c;
    }
    const int nt = toff[e + 1] - toff[e];
    for (int i = 0; i < nt; ++i) {
      const int slot = toff[e] + i;
      if (slot < max_tiles) tiles[slot] = GroupTile{e, i * tile_m};
    }
  }
}

__global__ void __launch_bounds__(1024) perm_scatter_kernel(int n_assign, int E,
                                                            const int32_t *__restrict__ topk_idx,
                                                            const int32_t *__restrict__ bbase,
                                                            int32_t *perm, int32_t *inv_perm) {
  pdl_wait();
  pdl_trigger();
  __shared__ int hist[256 * 32];  // [expert][warp] counts, then exclusive prefixes over the warps
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, blk = blockIdx.x;
  for (int i = tid; i < 32 * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int a0 = blk * PERM_CHUNK + w * 64 + lane, a1 = a0 + 32;
  int e0 = a0 < n_assign ? topk_idx[a0] : -1;
  int e1 = a1 < n_assign ? topk_idx[a1] : -1;
  if (e0 >= E) e0 = -1;
  if (e1 >= E) e1 = -1;
  const unsigned lt = (1u << lane) - 1u;
  const unsigned m0 = __match_any_sync(0xffffffffu, e0), m1 = __match_any_sync(0xffffffffu, e1);
  const int r0 = __popc(m0 & lt), r1 = __popc(m1 & lt);
  if (e0 >= 0 && r0 == 0) hist[e0 * 32 + w] = __popc(m0);
  __syncwarp();
  const int base1 = e1 >= 0 ? hist[e1 * 32 + w] : 0;  // e1's count in the warp's first half
  __syncwarp();
  if (e1 >= 0 && r1 == 0) hist[e1 * 32 + w] = base1 + __popc(m1);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {  // exclusive prefix over the warps, per expert
    int run = 0;
    for (int ww = 0; ww < 32; ++ww) {
      const int c = hist[e * 32 + ww];
      hist[e * 32 + ww] = run;
      run += c;
    }
  }
  __syncthreads();
  if (e0 >= 0) {
    const int pos = bbase[(size_t)blk * E + e0] + hist[e0 * 32 + w] + r0;
    perm[pos] = a0;
    inv_perm[a0] = pos;
  } else if (a0 < n_assign) {
    inv_perm[a0] = -1;
  }
  if (e1 >= 0) {
    const int pos = bbase[(size_t)blk * E + e1] + hist[e1 * 32 + w] + base1 + r1;
    perm[pos] = a1;
    inv_perm[a1] = pos;
  } else if (a1 < n_assign) {
    inv_perm[a1] = -1;
  }
}

// permute_tiles_kernel for at most 2048 assignments in one pass (one block of 1024 threads, two
// assignments per thread: a0 = 64 w + lane and a1 = a0 + 32 for warp w).  Counting sort: the rank
// of an assignment among the same-expert ones of its warp half comes from __match_any_sync, the
// warp leaders write a per-(expert, warp) histogram, and one block-wide exclusive scan of that
// histogram in expert-major order gives every expert's offset and every warp's first position
// within it, so the grouping is stable in assignment order.  Same outputs as
// permute_tiles_kernel.
__global__ void __launch_bounds__(1024) permute_tiles_small_kernel(
    int n_assign, int E, const int32_t *__restrict__ topk_idx, int32_t *expert_off, int32_t *perm,
    int32_t *inv_perm, int tile_m, GroupTile *tiles, int32_t *n_tiles, int max_tiles,
    int32_t *load_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ int hist[256 * 32];  // [expert][warp], then its exclusive scan
  __shared__ int wtot[32], s_total;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int H = 32 * E;
  for (int i = tid; i < H; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int a0 = w * 64 + lane, a1 = a0 + 32;
  int e0 = a0 < n_assign ? topk_idx[a0] : -1;
  int e1 = a1 < n_assign ? topk_idx[a1] : -1;
  if (e0 >= E) e0 = -1;
  if (e1 >= E) e1 = -1;
  const unsigned lt = (1u << lane) - 1u;
  const unsigned m0 = __match_any_sync(0xffffffffu, e0), m1 = __match_any_sync(0xffffffffu, e1);
  const int r0 = __popc(m0 & lt), r1 = __popc(m1 & lt);
  if (e0 >= 0 && r0 == 0) hist[e0 * 32 + w] = __popc(m0);
  __syncwarp();
  const int base1 = e1 >= 0 ? hist[e1 * 32 + w] : 0;  // e1's count in the warp's first half
  __syncwarp();
  if (e1 >= 0 && r1 == 0) hist[e1 * 32 + w] = base1 + __popc(m1);
  __syncthreads();
  // exclusive scan of hist[0, H): thread t owns the run [t P, t P + P)
  const int P = (H + blockDim.x - 1) / blockDim.x;
  int run = 0;
  for (int j = 0; j < P; ++j) {
    const int i = tid * P + j;
    if (i < H) run += hist[i];
  }
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wtot[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int v = wtot[lane];
    int iv = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, iv, o);
      if (lane >= o) iv += u;
    }
    wtot[lane] = iv - v;  // exclusive over warps
    if (lane == 31) s_total = iv;
  }
  __syncthreads();
  int acc = wtot[w] + incl - run;  // exclusive prefix of this thread's run
  for (int j = 0; j < P; ++j) {
    const int i = tid * P + j;
    if (i < H) {
      const int v = hist[i];
      hist[i] = acc;
      acc += v;
    }
  }
  __syncthreads();
  if (e0 >= 0) {
    const int pos = hist[e0 * 32 + w] + r0;
    perm[pos] = a0;
    inv_perm[a0] = pos;
  } else if (a0 < n_assign) {
    inv_perm[a0] = -1;
  }
  if (e1 >= 0) {
    const int pos = hist[e1 * 32 + w] + base1 + r1;
    perm[pos] = a1;
    inv_perm[a1] = pos;
  } else if (a1 < n_assign) {
    inv_perm[a1] = -1;
  }
  // expert offsets (hist[32 e] = the first position of expert e), counts and the tile list:
  // warp 0, eight experts per lane (E <= 256)
  if (w == 0) {
    int cnt[8], nt[8], tsum = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      cnt[j] = 0;
      nt[j] = 0;
      if (e < E) {
        const int hi = e + 1 < E ? hist[(e + 1) * 32] : s_total;
        cnt[j] = hi - hist[e * 32];
        nt[j] = (cnt[j] + tile_m - 1) / tile_m;
        tsum += nt[j];
      }
    }
    int tinc = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, tinc, o);
      if (lane >= o) tinc += v;
    }
    int tbase = tinc - tsum;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane * 8 + j;
      if (e >= E) continue;
      expert_off[e] = hist[e * 32];
      if (load_out) load_out[e] = cnt[j];
      for (int i = 0; i < nt[j]; ++i) {
        const int slot = tbase + i;
        if (slot < max_tiles) tiles[slot] = GroupTile{e, i * tile_m};
      }
      tbase += nt[j];
    }
    if (lane == 31) {
      expert_off[E] = s_total;
      *n_tiles = min(tinc, max_tiles);
    }
  }
}

// Single block of 1024 threads; E <= 256.
__global__ void __launch_bounds__(1024) permute_kernel(int n_assign, int E,
                                                       const int32_t *__restrict__ topk_idx,
                                                       int32_t *expert_off, int32_t *perm,
                                                       int32_t *inv_perm) {
  pdl_wait();
  pdl_trigger();
  __shared__ int cnt[256], off[257], running[256];
  __shared__ int wc[32][256];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int e = tid; e < E; e += blockDim.x) { cnt[e] = 0; running[e] = 0; }
  __syncthreads();
  for (int a = tid; a < n_assign; a += blockDim.x) {
    const int e = topk_idx[a];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) { off[e] = acc; acc += cnt[e]; }
    off[E] = acc;
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) expert_off[e] = off[e];
  for (int c0 = 0; c0 < n_assign; c0 += blockDim.x) {
    for (int i = tid; i < 32 * E; i += blockDim.x) wc[i / E][i % E] = 0;
    __syncthreads();
    const int a = c0 + tid;
    int e = -1;
    if (a < n_assign) {
      e = topk_idx[a];
      if (e >= E) e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rank == 0) wc[w][e] = __popc(peers);
    __syncthreads();
    if (e >= 0) {
      int before = 0;
      for (int ww = 0; ww < w; ++ww) before += wc[ww][e];
      const int pos = off[e] + running[e] + before + rank;
      perm[pos] = a;
      inv_perm[a] = pos;
    } else if (a < n_assign) {
      inv_perm[a] = -1;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += blockDim.x) {
      int t = 0;
      for (int ww = 0; ww < 32; ++ww) t += wc[ww][ee];
      running[ee] += t;
    }
    __syncthreads();
  }
}

// Tile list of the grouped expert GEMMs: for each expert with rows, tiles of tile_m rows.
// Optionally also stores the per-expert assignment counts (expert load) in load_out [E].
__global__ void build_tiles_kernel(int E, const int32_t *__restrict__ expert_off, int tile_m,
                                   GroupTile *tiles, int32_t *n_tiles, int max_tiles,
                                   int32_t *load_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ int toff[257];
  const int tid = threadIdx.x;
  if (load_out)
    for (int e = tid; e < E; e += blockDim.x) load_out[e] = expert_off[e + 1] - expert_off[e];
  if (tid == 0) {
    int acc = 0;
    for (int e = 0; e < E; ++e) {
      toff[e] = acc;
      acc += (expert_off[e + 1] - expert_off[e] + tile_m - 1) / tile_m;
    }
    toff[E] = acc;
    *n_tiles = min(acc, max_tiles);
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int nt = toff[e + 1] - toff[e];
    for (int i = 0; i < nt; ++i) {
      const int slot = toff[e] + i;
      if (slot < max_tiles) tiles[slot] = GroupTile{e, i * tile_m};
    }
  }
}

// X[p] = y[perm[p] / k] for the routed assignments p < expert_off[E] (bf16 rows, 16-byte copies).
__global__ void gather_rows_kernel(int d, int k, const int32_t *__restrict__ perm,
                                   const int32_t *__restrict__ expert_off, int E,
                                   const uint4 *__restrict__ y, uint4 *X) {
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  if (p >= expert_off[E]) return;
  const int t = perm[p] / k;
  const int n16 = d / 8;
  for (int i = threadIdx.x; i < n16; i += blockDim.x) X[(size_t)p * n16 + i] = y[(size_t)t * n16 + i];
}

template <typename T>
__global__ void gate_kernel(int F, const float *__restrict__ u, const int32_t *__restrict__ expert_off,
                            int E, T *a) {
  pdl_wait();
  pdl_trigger();
  const int p = blockIdx.x;
  if (p >= expert_off[E]) return;
  const float *ur = u + (size_t)p * 2 * F;
  T *ar = a + (size_t)p * F;
  for (int f = threadIdx.x; f < F; f += blockDim.x) {
    const float g = ur[f], up = ur[F + f];
    const float gl = 0.5f * g * (1.0f + tanhf(0.7978845608028654f * (g + 0.044715f * g * g * g)));
    ar[f] = from_f<T>(gl * up);
  }
}

// out_t = res_t + sum_j w[t][j] Y[inv_perm[t k + j]] in fp32, slot order j = 0..k-1 (the
// residual stream and the expert outputs are fp32).
__global__ void combine_kernel(int d, int k, const int32_t *__restrict__ topk_idx,
                               const float *__restrict__ topk_w, const int32_t *__restrict__ inv_perm,
                               const float *__restrict__ Y, const float *__restrict__ res,
                               float *out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float acc = res[(size_t)t * d + c];
    for (int j = 0; j < k; ++j) {
      const int a = t * k + j;
      if (topk_idx[a] < 0) continue;
      acc = fmaf(topk_w[a], Y[(size_t)inv_perm[a] * d + c], acc);
    }
    out[(size_t)t * d + c] = acc;
  }
}

// Combine + the next RMSNorm, one block per token: x_t = res_t + sum_j w[t][j] Y[inv_perm[t k + j]]
// (fp32, slot order), stored; then RMSNorm(x_t) rounded to the activation type, stored in a_out
// (the next layer's QKV input) and/or in f_out row slot[t] (the final-norm rows of the masked
// positions that the LM head reads).  d <= 256 * 16.
template <typename T>
__global__ void __launch_bounds__(256) combine_norm_kernel(int d, int k, float eps,
                                                           const int32_t *__restrict__ topk_idx,
                                                           const float *__restrict__ topk_w,
                                                           const int32_t *__restrict__ inv_perm,
                                                           const float *__restrict__ Y,
                                                           const float *__restrict__ res, float *out,
                                                           T *a_out, const int32_t *__restrict__ slot,
                                                           T *f_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  __shared__ int idx[32];
  __shared__ float wt[32];
  const int t = blockIdx.x;
  float xv[16];
  float ss = 0.f;
  if (threadIdx.x < k) {
    idx[threadIdx.x] = topk_idx[t * k + threadIdx.x] >= 0 ? inv_perm[t * k + threadIdx.x] : -1;
    wt[threadIdx.x] = topk_w[t * k + threadIdx.x];
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int c = threadIdx.x + u * 256;
    if (c < d) {
      float acc = res[(size_t)t * d + c];
      for (int j0 = 0; j0 < k; j0 += 8) {  // eight expert rows in flight, added in slot order
        float yv[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = j0 + jj;
          yv[jj] = (j < k && idx[j] >= 0) ? Y[(size_t)idx[j] * d + c] : 0.f;
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = j0 + jj;
          if (j < k && idx[j] >= 0) acc = fmaf(wt[j], yv[jj], acc);
        }
      }
      out[(size_t)t * d + c] = acc;
      xv[u] = acc;
      ss += acc * acc;
    }
  }
  const int sl = slot ? slot[t] : -1;
  if (!a_out && sl < 0) return;  // uniform in the block
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int c = threadIdx.x + u * 256;
    if (c < d) {
      const T v = from_f<T>(xv[u] * inv);
      if (a_out) a_out[(size_t)t * d + c] = v;
      if (sl >= 0) f_out[(size_t)sl * d + c] = v;
    }
  }
}

// combine_norm_kernel with one float4 per thread (blockDim = d / 4 <= 1024); same arithmetic in
// the same order, with the eight expert rows of a thread loaded ahead of the FMAs.
template <typename T, typename TF = T>
__global__ void __launch_bounds__(1024) combine_norm4_kernel(
    int d4, int k, float eps, const int32_t *__restrict__ topk_idx,
    const float *__restrict__ topk_w, const int32_t *__restrict__ inv_perm,
    const float4 *__restrict__ Y, const float4 *__restrict__ res, float4 *out, T *a_out,
    const int32_t *__restrict__ slot, TF *f_out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  __shared__ int idx[32];
  __shared__ float wt[32];
  const int t = blockIdx.x, c = threadIdx.x;
  if (threadIdx.x < k) {
    idx[threadIdx.x] = topk_idx[t * k + threadIdx.x] >= 0 ? inv_perm[t * k + threadIdx.x] : -1;
    wt[threadIdx.x] = topk_w[t * k + threadIdx.x];
  }
  __syncthreads();
  float4 acc = res[(size_t)t * d4 + c];
  for (int j0 = 0; j0 < k; j0 += 8) {
    float4 yv[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = j0 + jj;
      if (j < k && idx[j] >= 0) yv[jj] = Y[(size_t)idx[j] * d4 + c];
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = j0 + jj;
      if (j < k && idx[j] >= 0) {
        const float w = wt[j];
        acc.x = fmaf(w, yv[jj].x, acc.x);
        acc.y = fmaf(w, yv[jj].y, acc.y);
        acc.z = fmaf(w, yv[jj].z, acc.z);
        acc.w = fmaf(w, yv[jj].w, acc.w);
      }
    }
  }
  out[(size_t)t * d4 + c] = acc;
  const int sl = slot ? slot[t] : -1;
  if (!a_out && sl < 0) return;  // uniform in the block
  float ss = acc.x * acc.x;
  ss += acc.y * acc.y;
  ss += acc.z * acc.z;
  ss += acc.w * acc.w;
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)(4 * d4) + eps);
  if (a_out) store4<T>(a_out + ((size_t)t * d4 + c) * 4, acc.x * inv, acc.y * inv, acc.z * inv,
                       acc.w * inv);
  if (sl >= 0) store4<TF>(f_out + ((size_t)sl * d4 + c) * 4, acc.x * inv, acc.y * inv, acc.z * inv,
                          acc.w * inv);
}

}  // namespace

int launch_combine_norm(int act, int T_, int d, int k, double eps, const int32_t *topk_idx,
                        const float *topk_w, const int32_t *inv_perm, const void *Y,
                        const void *res, void *out, void *a_out, const int32_t *slot, void *f_out,
                        cudaStream_t s, int f_out_f16) {
  if (T_ <= 0) return DG_OK;
  if (d > 256 * 16 || k > 32) return DG_ERR_UNSUPPORTED;
  const bool vec4 = d % 4 == 0 && d / 4 <= 1024 && d / 4 >= 32;
  if (f_out_f16 && (act != DG_BF16 || !vec4)) return DG_ERR_UNSUPPORTED;
  note_launch(s, "combine_norm");
  if (vec4) {
    if (f_out_f16)
      launch_pdl(combine_norm4_kernel<bf16, __half>, T_, d / 4, 0, s, d / 4, k, (float)eps,
                 topk_idx, topk_w, inv_perm, (const float4 *)Y, (const float4 *)res,
                 (float4 *)out, (bf16 *)a_out, slot, (__half *)f_out);
    else if (act == DG_F32)
      launch_pdl(combine_norm4_kernel<float>, T_, d / 4, 0, s, d / 4, k, (float)eps, topk_idx,
                 topk_w, inv_perm, (const float4 *)Y, (const float4 *)res, (float4 *)out,
                 (float *)a_out, slot, (float *)f_out);
    else
      launch_pdl(combine_norm4_kernel<bf16>, T_, d / 4, 0, s, d / 4, k, (float)eps, topk_idx,
                 topk_w, inv_perm, (const float4 *)Y, (const float4 *)res, (float4 *)out,
                 (bf16 *)a_out, slot, (bf16 *)f_out);
    return check_launch("combine_norm");
  }
  if (act == DG_F32)
    launch_pdl(combine_norm_kernel<float>, T_, 256, 0, s, d, k, (float)eps, topk_idx, topk_w, inv_perm,
                                                  (const float *)Y, (const float *)res, (float *)out,
                                                  (float *)a_out, slot, (float *)f_out);
  else
    launch_pdl(combine_norm_kernel<bf16>, T_, 256, 0, s, d, k, (float)eps, topk_idx, topk_w, inv_perm,
                                                 (const float *)Y, (const float *)res, (float *)out,
                                                 (bf16 *)a_out, slot, (bf16 *)f_out);
  return check_launch("combine_norm");
}

int launch_router(int act, int wr_type, int T_, int d, int E, int k, const void *y,
                  const void *w_router, const uint8_t *token_live, int32_t *topk_idx,
                  float *topk_w, cudaStream_t s, int n_shared) {
  if (T_ <= 0) return DG_OK;
  if (n_shared < 0 || k + n_shared > 32) return DG_ERR_UNSUPPORTED;
  const int threads = E < 32 ? 32 : (E > 256 ? 256 : ((E + 31) / 32) * 32);
  const size_t smem = sizeof(float) * ROUTER_TPB * (size_t)(d + E);
  const int grid = (T_ + ROUTER_TPB - 1) / ROUTER_TPB;
  if (act == DG_F32 && wr_type == DG_F32) {
    auto kf = router_kernel<float, float>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    note_launch(s, "router");
    launch_pdl(kf, grid, threads, smem, s, T_, d, E, k, n_shared, (const float *)y, (const float *)w_router,
                                   token_live, topk_idx, topk_w);
  } else if (act == DG_BF16 && wr_type == DG_BF16) {
    auto kb = router_kernel<bf16, bf16>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    note_launch(s, "router");
    launch_pdl(kb, grid, threads, smem, s, T_, d, E, k, n_shared, (const bf16 *)y, (const bf16 *)w_router,
                                   token_live, topk_idx, topk_w);
  } else {
    return DG_ERR_UNSUPPORTED;
  }
  return check_launch("router");
}

int launch_router_topk(int T_, int E, int k, const float *z, const uint8_t *token_live,
                       int32_t *topk_idx, float *topk_w, cudaStream_t s, const int32_t *forced,
                       int n_parts, int n_shared) {
  if (T_ <= 0) return DG_OK;
  if (E > 256 || n_shared < 0 || k + n_shared > 32) return DG_ERR_UNSUPPORTED;
  note_launch(s, "router_topk");
  launch_pdl(router_topk_kernel, (T_ + 7) / 8, 256, 0, s, T_, E, k, n_shared, z, n_parts,
             token_live, forced, topk_idx, topk_w);
  return check_launch("router_topk");
}

size_t permute_scratch_bytes(int n_assign, int E) {
  return (size_t)((n_assign + PERM_CHUNK - 1) / PERM_CHUNK) * E * sizeof(int32_t);
}

int launch_permute_tiles(int T_, int E, int k, const int32_t *topk_idx, int32_t *expert_off,
                         int32_t *perm, int32_t *inv_perm, int tile_m, GroupTile *tiles,
                         int32_t *n_tiles, int max_tiles, int32_t *load_out, cudaStream_t s,
                         int n_shared, int32_t *scratch) {
  if (T_ <= 0) return DG_OK;
  const int ka = k + n_shared, Ea = E + n_shared;
  if (Ea > 256 || n_shared < 0 || ka > 32) return DG_ERR_UNSUPPORTED;
  const int n_assign = T_ * ka;
  if (n_assign <= PERM_CHUNK) {
    note_launch(s, "permute_tiles");
    launch_pdl(permute_tiles_small_kernel, 1, 1024, 0, s, n_assign, Ea, topk_idx, expert_off,
               perm, inv_perm, tile_m, tiles, n_tiles, max_tiles, load_out);
    return check_launch("permute_tiles");
  }
  if (!scratch) {
    note_launch(s, "permute_tiles");
    launch_pdl(permute_tiles_kernel, 1, 1024, 0, s, n_assign, Ea, topk_idx, expert_off, perm,
               inv_perm, tile_m, tiles, n_tiles, max_tiles, load_out);
    return check_launch("permute_tiles");
  }
  const int nb = (n_assign + PERM_CHUNK - 1) / PERM_CHUNK;
  note_launch(s, "perm_count");
  launch_pdl(perm_count_kernel, nb, 1024, 0, s, n_assign, Ea, topk_idx, scratch);
  int rc = check_launch("perm_count");
  if (rc != DG_OK) return rc;
  note_launch(s, "perm_offsets");
  launch_pdl(perm_offsets_kernel, 1, 1024, 0, s, nb, Ea, scratch, expert_off, tile_m, tiles,
             n_tiles, max_tiles, load_out);
  rc = check_launch("perm_offsets");
  if (rc != DG_OK) return rc;
  note_launch(s, "perm_scatter");
  launch_pdl(perm_scatter_kernel, nb, 1024, 0, s, n_assign, Ea, topk_idx, scratch, perm,
             inv_perm);
  return check_launch("perm_scatter");
}

int launch_route(int T_, int E, int k, const float *z, const uint8_t *token_live, int32_t *topk_idx,
                 float *topk_w, int32_t *expert_off, int32_t *perm, int32_t *inv_perm, int tile_m,
                 GroupTile *tiles, int32_t *n_tiles, int max_tiles, int32_t *load_out,
                 cudaStream_t s, const int32_t *forced, int n_parts, int n_shared,
                 int32_t *scratch) {
  if (T_ <= 0) return DG_OK;
  const int ka = k + n_shared, Ea = E + n_shared;  // slots and experts with the shared ones
  if (Ea > 256 || n_shared < 0 || ka > 32) return DG_ERR_UNSUPPORTED;
  const int rc = launch_router_topk(T_, E, k, z, token_live, topk_idx, topk_w, s, forced, n_parts,
                                    n_shared);
  if (rc != DG_OK) return rc;
  return launch_permute_tiles(T_, E, k, topk_idx, expert_off, perm, inv_perm, tile_m, tiles,
                              n_tiles, max_tiles, load_out, s, n_shared, scratch);
}

int launch_permute(int T_, int k, int E, const int32_t *topk_idx, int32_t *expert_off,
                   int32_t *perm, int32_t *inv_perm, cudaStream_t s) {
  if (E > 256) return DG_ERR_UNSUPPORTED;
  note_launch(s, "permute");
  launch_pdl(permute_kernel, 1, 1024, 0, s, T_ * k, E, topk_idx, expert_off, perm, inv_perm);
  return check_launch("permute");
}

int launch_build_tiles(int E, const int32_t *expert_off, int tile_m, GroupTile *tiles,
                       int32_t *n_tiles, int max_tiles, int32_t *load_out, cudaStream_t s) {
  if (E > 256) return DG_ERR_UNSUPPORTED;
  note_launch(s, "build_tiles");
  launch_pdl(build_tiles_kernel, 1, 256, 0, s, E, expert_off, tile_m, tiles, n_tiles, max_tiles, load_out);
  return check_launch("build_tiles");
}

int launch_gather_rows(int rows_max, int d, int k, const int32_t *perm, const int32_t *expert_off,
                       int E, const void *y, void *X, cudaStream_t s) {
  if (rows_max <= 0) return DG_OK;
  note_launch(s, "gather_rows");
  launch_pdl(gather_rows_kernel, rows_max, 128, 0, s, d, k, perm, expert_off, E, (const uint4 *)y, (uint4 *)X);
  return check_launch("gather_rows");
}

int launch_gate(int act, int rows_max, int F, const float *u, const int32_t *expert_off, int E,
                void *a, cudaStream_t s) {
  if (rows_max <= 0) return DG_OK;
  note_launch(s, "gate");
  if (act == DG_F32)
    launch_pdl(gate_kernel<float>, rows_max, 128, 0, s, F, u, expert_off, E, (float *)a);
  else
    launch_pdl(gate_kernel<bf16>, rows_max, 128, 0, s, F, u, expert_off, E, (bf16 *)a);
  return check_launch("gate");
}

int launch_combine(int act, int T_, int d, int k, const int32_t *topk_idx, const float *topk_w,
                   const int32_t *inv_perm, const void *Y, const void *res, void *out,
                   cudaStream_t s) {
  if (T_ <= 0) return DG_OK;
  (void)act;
  note_launch(s, "combine");
  launch_pdl(combine_kernel, T_, 256, 0, s, d, k, topk_idx, topk_w, inv_perm, (const float *)Y,
                                    (const float *)res, (float *)out);
  return check_launch("combine");
}

}  // namespace dg
