// LM head with fused softmax entropy and greedy argmax on the 5th-generation tensor cores.
// "DiffusionGemma Technical Report", explanatory visual and What they did: the entropy-bounded
// sampler ranks canvas positions by the entropy of their predictive distribution; Table 1:
// vocabulary 262k.  The logits z = f W_lm^T of the masked rows are never stored (except for
// debugging); each (row, vocabulary tile) leaves a partial softmax state that a second kernel
// merges exactly.
//
// Persistent, warp-specialised kernel, one CTA per SM:
//   warp 0      TMA producer: A = 128 normalised rows x 64 k, B = 256 vocabulary rows x 64 k,
//               4-stage ring in shared memory (48 KB per stage, 128-byte swizzle);
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma (M 128, N 256, K 16) into one
//               of two 256-column fp32 accumulators, so the epilogue of one tile overlaps the
//               MMAs of the next;
//   warps 2-5   epilogue: each thread owns one row and reads its 256 logits from TMEM in chunks
//               of 32, keeping m = max, s = sum e^(z-m), u = sum e^(z-m)(z-m) and the first
//               argmax (see entropy_state.cuh).
// Work units are (row tile, vocabulary tile) with the row tile varying fastest, so the CTAs
// working on the same vocabulary tile run together and share it through L2.
// Every wait is bounded (tc::WAIT_LIMIT_CYCLES); on expiry the kernel records DG_ERR_TIMEOUT,
// drains what it issued, frees TMEM and returns.
// Sampler variants (SAMPLE = true instantiations): each row's logits are multiplied by its 1/tau
// and its token is the argmax of z/tau + Gumbel noise drawn from the row's counter stream (the
// report's annealed-temperature sampler, Figures 9 and 10; see sampler.cuh); the entropy is that
// of softmax(z/tau).  A greedy row (tau <= 0) in such a launch keeps tau = 1 and no noise.
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "entropy_state.cuh"
#include "sampler.cuh"
#include "tc_common.cuh"
#include "tc_host.h"

namespace dg {

namespace {

using namespace tc;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + 256;

struct Params {
  const int32_t *n_rows_dev;
  int max_rows, V, K, n_vtiles;
  float4 *part;             // [max_rows][n_vtiles]: (m, s, u, max value)
  int32_t *part_am;         // [max_rows][n_vtiles]: first argmax in the tile
  float *logits;            // debug: [*][V] or null
  const int32_t *logits_rows;  // debug: output row of row r (null: r)
  int only_one_tile;        // the single-CTA kernel leaves more than 128 rows to the pair kernel
  int32_t *status;
  // NVFP4 weights (lmhead_q4_kernel): k-block-major codes and scales, rows padded to rows_pad
  const uint8_t *q_codes, *q_scales;
  int rows_pad;
  float gscale;
  // sampler variants: the draw of each row's token (source row = row_src ? row_src[r] : r)
  SampleSpec smp;
  const int32_t *row_src;
};

__device__ __forceinline__ void fail(int32_t *st, volatile int *abort_flag) {
  set_status(st, DG_ERR_TIMEOUT);
  *abort_flag = 1;
}

// Online update of one row's softmax state with 32 consecutive logits r (columns col0 ..
// col0 + nvalid - 1 valid): m = running max, s = sum e^(z - m), u = sum e^(z - m)(z - m), and
// av / am = the maximum and the first column holding it.  A full chunk takes the branch-free
// path: tree maximum, first argmax from the bit mask of the columns equal to it, and four
// partial sums, so the exponentials of different columns overlap (a per-column test inside the
// unrolled loop made every column its own dependent block, and the epilogue took ~14 us per
// 256-column tile instead of ~5).  A ragged chunk (the end of the vocabulary) tests each column.
// SCALED: the logits are the accumulator values times gs (the NVFP4 tensor scale).
// SAMPLE: the logits are further multiplied by the row's 1/tau (rd), the softmax state is that of
// the scaled logits, and av / am track the maximum of the keys z/tau + G (G = 0 for a greedy row)
// instead of the logits.
template <bool SCALED = false, bool SAMPLE = false>
__device__ __forceinline__ void ent_chunk(const uint32_t (&r)[32], int nvalid, int col0, float &m,
                                          float &s, float &u, float &av, int &am, float gs = 1.f,
                                          const RowDraw *rd = nullptr, uint32_t k0 = 0u,
                                          uint32_t k1 = 0u) {
  float cm, cs, cu;
  float mn;
  const float mul = SAMPLE ? rd->inv_tau : 1.f;
  if (nvalid == 32) {
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      v[j] = SCALED ? __uint_as_float(r[j]) * gs : __uint_as_float(r[j]);
      if (SAMPLE) v[j] *= mul;
    }
    float t[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) t[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
    for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
      for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
    cm = t[0];
    if (!SAMPLE && cm > av) {
      uint32_t bits = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) bits |= (v[j] == cm) ? (1u << j) : 0u;
      av = cm;
      am = col0 + __ffs(bits) - 1;
    }
    mn = fmaxf(m, cm);
    float ps[4] = {0.f, 0.f, 0.f, 0.f}, pu[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float d = v[j] - mn;
      const float e = __expf(d);
      ps[j & 3] += e;
      pu[j & 3] = fmaf(e, d, pu[j & 3]);
    }
    cs = (ps[0] + ps[1]) + (ps[2] + ps[3]);
    cu = (pu[0] + pu[1]) + (pu[2] + pu[3]);
    if (SAMPLE) {  // keys = scaled logits + Gumbel draws; first maximum
      if (rd->on) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 g = gumbel4(*rd, (uint32_t)(col0 >> 2) + q, k0, k1);
          v[4 * q] += g.x;
          v[4 * q + 1] += g.y;
          v[4 * q + 2] += g.z;
          v[4 * q + 3] += g.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) t[j] = fmaxf(v[j], v[j + 16]);
#pragma unroll
      for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
        for (int j = 0; j < w; ++j) t[j] = fmaxf(t[j], t[j + w]);
      const float ck = t[0];
      if (ck > av) {
        uint32_t bits = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) bits |= (v[j] == ck) ? (1u << j) : 0u;
        av = ck;
        am = col0 + __ffs(bits) - 1;
      }
    }
  } else {
    cm = -INFINITY;
    int ci = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float v = SCALED ? __uint_as_float(r[j]) * gs : __uint_as_float(r[j]);
      if (SAMPLE) v *= mul;
      if (j < nvalid && v > cm) { cm = v; ci = j; }
    }
    if (!SAMPLE && cm > av) { av = cm; am = col0 + ci; }
    mn = fmaxf(m, cm);
    cs = 0.f;
    cu = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < nvalid) {
        float v = SCALED ? __uint_as_float(r[j]) * gs : __uint_as_float(r[j]);
        if (SAMPLE) v *= mul;
        const float d = v - mn;
        const float e = __expf(d);
        cs += e;
        cu = fmaf(e, d, cu);
      }
    }
    if (SAMPLE) {
      float ck = -INFINITY;
      int ck_i = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (4 * q < nvalid) {
          const float4 g = rd->on ? gumbel4(*rd, (uint32_t)(col0 >> 2) + q, k0, k1)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
          const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 4 * q + e;
            if (j < nvalid) {
              float v = SCALED ? __uint_as_float(r[j]) * gs : __uint_as_float(r[j]);
              v = v * mul + gg[e];
              if (v > ck) { ck = v; ck_i = j; }
            }
          }
        }
      }
      if (ck > av) { av = ck; am = col0 + ck_i; }
    }
  }
  if (s > 0.f) {
    const float sc = __expf(m - mn);
    u = sc * fmaf(s, m - mn, u);
    s *= sc;
  }
  s += cs;
  u += cu;
  m = mn;
}

template <bool SAMPLE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    lmhead_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, Params p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * A_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(sB + STAGES * B_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_rows = p.max_rows;
  if (p.n_rows_dev) n_rows = min(*p.n_rows_dev, p.max_rows);
  const int m_tiles = (n_rows + BM - 1) / BM;
  const int units = m_tiles * p.n_vtiles;
  if ((int)blockIdx.x >= units) return;  // uniform across the block
  if (p.only_one_tile && m_tiles > 1) return;  // the pair kernel handles these rows
  const int kblocks = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int armed[STAGES];
      uint32_t armed_ph[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) { armed[s] = 0; armed_ph[s] = 0; }
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int mt = u % m_tiles, nt = u / m_tiles;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) { fail(p.status, abort_flag); break; }
          mbar_expect_tx(&full[stage], A_BYTES + B_BYTES);
          tma_load_2d(sA + stage * A_BYTES, &tmA, &full[stage], kb * BK, mt * BM);
          tma_load_2d(sB + stage * B_BYTES, &tmB, &full[stage], kb * BK, nt * BN);
          armed[stage] = 1;
          armed_ph[stage] = ph;
          if (++stage == STAGES) { stage = 0; ph ^= 1; }
        }
      }
      if (*abort_flag) {  // let every issued copy land before the CTA's shared memory goes away
        for (int s = 0; s < STAGES; ++s)
          if (armed[s]) (void)mbar_wait(&full[s], armed_ph[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(BM, BN);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      int last_stage = -1;
      uint32_t last_ph = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        if (!mbar_wait(&tempty[acc], aph ^ 1)) { fail(p.status, abort_flag); break; }
        fence_after();
        const uint32_t d = tmem + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], ph)) { fail(p.status, abort_flag); ok = false; break; }
          fence_after();
          const uint64_t ad = sdesc_sw128(sA + stage * A_BYTES);
          const uint64_t bd = sdesc_sw128(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          commit(&empty[stage]);
          last_stage = stage;
          last_ph = ph;
          if (++stage == STAGES) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      if (*abort_flag && last_stage >= 0)  // the MMAs issued so far finish before TMEM is freed
        (void)mbar_wait(&empty[last_stage], last_ph);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    int acc = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      const int mt = u % m_tiles, nt = u / m_tiles;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph))) {
        fail(p.status, abort_flag);
        break;
      }
      fence_after();
      const int row = mt * BM + q * 32 + lane;
      const bool row_ok = row < n_rows;
      RowDraw rd{1.f, 0, 0u, 0u, 0u};
      if (SAMPLE && row_ok) rd = row_draw(p.smp, p.row_src ? p.row_src[row] : row);
      float m = -INFINITY, s = 0.f, uu = 0.f, av = -INFINITY;
      int am = 0x7fffffff;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      float *lrow = nullptr;
      if (p.logits && row_ok)
        lrow = p.logits + (size_t)(p.logits_rows ? p.logits_rows[row] : row) * p.V;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = nt * BN + c * 32;
        if (col0 >= p.V) break;  // uniform in the warp
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_ld_wait(r);
        const int nvalid = min(32, p.V - col0);
        ent_chunk<false, SAMPLE>(r, nvalid, col0, m, s, uu, av, am, 1.f, &rd, p.smp.key0,
                                 p.smp.key1);
        if (lrow) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nvalid) lrow[col0 + j] = __uint_as_float(r[j]);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (row_ok) {
        const size_t o = (size_t)row * p.n_vtiles + nt;
        p.part[o] = make_float4(m, s, uu, av);
        p.part_am[o] = am;
      }
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// The same LM head on CTA pairs (clusters of 2) with the 2-SM MMA form, for more than 128 rows.
// A unit is (256 rows, 256 vocabulary rows): CTA r of the pair holds rows 128 r .. 128 r + 127
// and vocabulary rows 128 r .. 128 r + 127 of the unit, so each SM streams half the weight tile
// and its stage is 32 KB (7 stages, 224 KB); the tensor cores of both SMs compute
// the 256 x 256 product, each into its own TMEM (its 128 rows, all 256 vocabulary columns).
//   warp 0 of both CTAs: TMA into its own shared memory, completion counted on the leading
//     CTA's full barrier (the leader arms it with both CTAs' bytes);
//   warp 1 of the leading CTA: the 2-SM MMAs; commits arrive on the stage-empty and
//     accumulator-full barriers of both CTAs;
//   warps 2-5 of both CTAs: the entropy epilogue of its own rows, then an arrival on the
//     leading CTA's accumulator-empty barrier (8 arrivals per use).
// Every wait is bounded.  On expiry a CTA records DG_ERR_TIMEOUT and unwinds; its peer then
// times out on the barrier the aborted CTA no longer feeds.  Both reach the final cluster
// barrier, so neither frees TMEM or leaves while the other may still use its shared memory.
// The copies a producer issued before a stall land within microseconds, long before the ~2 s
// limit ends the wait.
constexpr int P_STAGES = 7;  // 7 x 32 KB + barriers: within the 227 KB of one CTA
constexpr int PA_BYTES = BM * BK * 2;        // this CTA's 128 rows x 64 k
constexpr int PB_BYTES = (BN / 2) * BK * 2;  // this CTA's 128 of the unit's 256 vocabulary rows
constexpr size_t P_SMEM_BYTES = 1024 + (size_t)P_STAGES * (PA_BYTES + PB_BYTES) + 256;
static_assert(P_SMEM_BYTES <= 232448, "more shared memory than one CTA may have");

template <bool SAMPLE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    lmhead_tc2_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmB, Params p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sA = smem;
  uint8_t *sB = smem + P_STAGES * PA_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(sB + P_STAGES * PB_BYTES);
  uint64_t *empty = full + P_STAGES;
  uint64_t *tfull = empty + P_STAGES;
  uint64_t *tempty = tfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  int n_rows = p.max_rows;
  if (p.n_rows_dev) n_rows = min(*p.n_rows_dev, p.max_rows);
  const int m_pairs = (n_rows + 2 * BM - 1) / (2 * BM);
  const int units = m_pairs * p.n_vtiles;
  if (pair >= units || n_rows <= BM) return;  // uniform across the pair; <= 128 rows: 1-CTA kernel
  const int kblocks = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
  fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t full_lead = mapa_shared(smem_u32(&full[0]), 0);
  const uint32_t tempty_lead = mapa_shared(smem_u32(&tempty[0]), 0);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      int armed[P_STAGES];
      uint32_t armed_ph[P_STAGES];
#pragma unroll
      for (int s = 0; s < P_STAGES; ++s) { armed[s] = 0; armed_ph[s] = 0; }
      for (int u = pair; u < units && !*abort_flag; u += npairs) {
        const int mp = u % m_pairs, nt = u / m_pairs;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) { fail(p.status, abort_flag); break; }
          if (rank == 0) mbar_expect_tx(&full[stage], 2 * (PA_BYTES + PB_BYTES));
          const uint32_t fb = full_lead + 8u * stage;
          tma_load_2d_pair(sA + stage * PA_BYTES, &tmA, fb, kb * BK, mp * 2 * BM + rank * BM);
          tma_load_2d_pair(sB + stage * PB_BYTES, &tmB, fb, kb * BK, nt * BN + rank * (BN / 2));
          armed[stage] = 1;
          armed_ph[stage] = ph;
          if (++stage == P_STAGES) { stage = 0; ph ^= 1; }
        }
      }
      if (*abort_flag && rank == 0) {  // the leader's full barriers count both CTAs' copies
        for (int s = 0; s < P_STAGES; ++s)
          if (armed[s]) (void)mbar_wait(&full[s], armed_ph[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16(2 * BM, BN);
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      int last_stage = -1;
      uint32_t last_ph = 0;
      for (int u = pair; u < units && !*abort_flag; u += npairs) {
        if (!mbar_wait(&tempty[acc], aph ^ 1)) { fail(p.status, abort_flag); break; }
        fence_after();
        const uint32_t d = tmem + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], ph)) { fail(p.status, abort_flag); ok = false; break; }
          fence_after();
          const uint64_t ad = sdesc_sw128(sA + stage * PA_BYTES);
          const uint64_t bd = sdesc_sw128(sB + stage * PB_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16_pair(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          commit_pair(&empty[stage]);
          last_stage = stage;
          last_ph = ph;
          if (++stage == P_STAGES) { stage = 0; ph ^= 1; }
        }
        if (!ok) break;
        commit_pair(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      if (*abort_flag && last_stage >= 0)  // the MMAs issued so far finish before TMEM is freed
        (void)mbar_wait(&empty[last_stage], last_ph);
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    int acc = 0;
    uint32_t aph = 0;
    for (int u = pair; u < units; u += npairs) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      const int mp = u % m_pairs, nt = u / m_pairs;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph))) {
        fail(p.status, abort_flag);
        break;
      }
      fence_after();
      const int row = mp * 2 * BM + (int)rank * BM + q * 32 + lane;
      const bool row_ok = row < n_rows;
      RowDraw rd{1.f, 0, 0u, 0u, 0u};
      if (SAMPLE && row_ok) rd = row_draw(p.smp, p.row_src ? p.row_src[row] : row);
      float m = -INFINITY, s = 0.f, uu = 0.f, av = -INFINITY;
      int am = 0x7fffffff;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      float *lrow = nullptr;
      if (p.logits && row_ok)
        lrow = p.logits + (size_t)(p.logits_rows ? p.logits_rows[row] : row) * p.V;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = nt * BN + c * 32;
        if (col0 >= p.V) break;  // uniform in the warp
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_ld_wait(r);
        const int nvalid = min(32, p.V - col0);
        ent_chunk<false, SAMPLE>(r, nvalid, col0, m, s, uu, av, am, 1.f, &rd, p.smp.key0,
                                 p.smp.key1);
        if (lrow) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nvalid) lrow[col0 + j] = __uint_as_float(r[j]);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(&tempty[acc]);
        else mbar_arrive_cluster(tempty_lead + 8u * acc);
      }
      if (row_ok) {
        const size_t o = (size_t)row * p.n_vtiles + nt;
        p.part[o] = make_float4(m, s, uu, av);
        p.part_am[o] = am;
      }
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }
  fence_before();
  cluster_sync();  // no CTA frees TMEM or exits while its peer may still use its shared memory
  if (warp == 1) {
    fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// The LM head with NVFP4 weights, one CTA per SM, for any number of rows (units (row tile,
// vocabulary tile), the row tile varying fastest).  The weight tile of a k-block arrives as 8 KB
// of FP4 codes and 1 KB of E4M3 block scales (two 1-D bulk copies from the k-block-major
// layout); converter warps expand it in shared memory into the fp16 tile the MMA reads, in the
// 128-byte-swizzled K-major layout TMA would have written: one hardware e2m1x2 -> f16x2
// conversion and one f16x2 multiply by the block scale per pair of weights (e2m1 * e4m3 is exact
// in fp16).  The MMA is kind::f16 with fp16 operands, so the normalised rows come in fp16 too;
// the tensor scale is applied to the fp32 logits in the epilogue.  (A bf16 tile would need two
// more conversions per pair, and those run at a quarter of the FP32 rate.)
// Three rings.  A k-block carries only 9 KB of weight bytes from DRAM, so the codes and scales
// get a ring of their own (8 stages, 72 KB in flight per SM), filled by one producer warp; the
// normalised rows (L2-resident) get a 5-stage TMA ring filled by another (5 rows stages and 8
// weight stages measured ~3% faster than 3 and 12); the expanded tiles a 2-stage ring between
// converters and MMA.
// With one ring for all three, a stage's 9 KB could not be refilled before its MMA completed,
// and four stages kept ~36 KB in flight: the loop ran at DRAM latency / 4 per k-block.
//   warp 0      producer of the codes and scales ring;
//   warp 1      TMEM owner and MMA issuer (M 128, N 256, K 16), two 256-column accumulators;
//   warps 2-5   entropy epilogue (as lmhead_tc_kernel, logits times the tensor scale);
//   warps 6-13  converters: thread i expands vocabulary row i of the tile, then fences its stores
//               for the tensor cores' (async) proxy;
//   warp 14     producer of the normalised-rows ring (TMA).
// Every wait is bounded.
constexpr int Q_QSTAGES = 8, Q_ASTAGES = 5, Q_CSTAGES = 2, Q_CONV_WARPS = 8;
constexpr int Q_A_BYTES = BM * BK * 2;   // 16 KB normalised rows (fp16)
constexpr int Q_C_BYTES = BN * BK / 2;   // 8 KB FP4 codes
constexpr int Q_S_BYTES = BN * BK / 16;  // 1 KB E4M3 scales
constexpr int Q_R_BYTES = Q_C_BYTES + Q_S_BYTES;
constexpr int Q_B_BYTES = BN * BK * 2;   // 32 KB expanded fp16 tile
constexpr int Q_THREADS = 32 * (6 + Q_CONV_WARPS + 1);
constexpr int Q_APROD_WARP = 6 + Q_CONV_WARPS;
constexpr size_t Q_SMEM = 1024 + (size_t)Q_CSTAGES * Q_B_BYTES + (size_t)Q_ASTAGES * Q_A_BYTES +
                          (size_t)Q_QSTAGES * Q_R_BYTES + 512;
static_assert(Q_SMEM <= 232448, "more shared memory than one CTA may have");
static_assert(Q_CONV_WARPS * 32 == BN, "one converter thread per vocabulary row of a tile");

template <bool SAMPLE>
__global__ void __launch_bounds__(Q_THREADS, 1)
    lmhead_q4_kernel(const __grid_constant__ CUtensorMap tmA, Params p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sB = smem;                               // [Q_CSTAGES][32 KB], 1024-aligned
  uint8_t *sA = sB + Q_CSTAGES * Q_B_BYTES;         // [Q_ASTAGES][16 KB], 1024-aligned
  uint8_t *sR = sA + Q_ASTAGES * Q_A_BYTES;         // [Q_QSTAGES][8 KB codes + 1 KB scales]
  uint64_t *qfull = reinterpret_cast<uint64_t *>(sR + Q_QSTAGES * Q_R_BYTES);
  uint64_t *qempty = qfull + Q_QSTAGES;
  uint64_t *afull = qempty + Q_QSTAGES;
  uint64_t *aempty = afull + Q_ASTAGES;
  uint64_t *cfull = aempty + Q_ASTAGES;
  uint64_t *cempty = cfull + Q_CSTAGES;
  uint64_t *tfull = cempty + Q_CSTAGES;
  uint64_t *tempty = tfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int n_rows = p.max_rows;
  if (p.n_rows_dev) n_rows = min(*p.n_rows_dev, p.max_rows);
  const int m_tiles = (n_rows + BM - 1) / BM;
  const int units = m_tiles * p.n_vtiles;
  if ((int)blockIdx.x >= units) return;  // uniform across the block
  const int kblocks = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Q_QSTAGES; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], Q_CONV_WARPS);
    }
    for (int s = 0; s < Q_ASTAGES; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int c = 0; c < Q_CSTAGES; ++c) {
      mbar_init(&cfull[c], Q_CONV_WARPS);
      mbar_init(&cempty[c], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == Q_APROD_WARP && lane == 0) tma_prefetch_desc(&tmA);
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // codes and scales
      int stage = 0;
      uint32_t ph = 0;
      int armed[Q_QSTAGES];
      uint32_t armed_ph[Q_QSTAGES];
#pragma unroll
      for (int s = 0; s < Q_QSTAGES; ++s) { armed[s] = 0; armed_ph[s] = 0; }
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int nt = u / m_tiles;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&qempty[stage], ph ^ 1)) { fail(p.status, abort_flag); break; }
          mbar_expect_tx(&qfull[stage], Q_R_BYTES);
          const size_t slab = (size_t)kb * p.rows_pad + (size_t)nt * BN;
          uint8_t *dst = sR + stage * Q_R_BYTES;
          bulk_load(dst, p.q_codes + slab * (BK / 2), Q_C_BYTES, &qfull[stage]);
          bulk_load(dst + Q_C_BYTES, p.q_scales + slab * (BK / 16), Q_S_BYTES, &qfull[stage]);
          armed[stage] = 1;
          armed_ph[stage] = ph;
          if (++stage == Q_QSTAGES) { stage = 0; ph ^= 1; }
        }
      }
      if (*abort_flag) {  // let every issued copy land before the CTA's shared memory goes away
        for (int s = 0; s < Q_QSTAGES; ++s)
          if (armed[s]) (void)mbar_wait(&qfull[s], armed_ph[s]);
      }
    }
  } else if (warp == Q_APROD_WARP) {
    if (lane == 0) {  // normalised rows
      int stage = 0;
      uint32_t ph = 0;
      int armed[Q_ASTAGES];
      uint32_t armed_ph[Q_ASTAGES];
#pragma unroll
      for (int s = 0; s < Q_ASTAGES; ++s) { armed[s] = 0; armed_ph[s] = 0; }
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int mt = u % m_tiles;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&aempty[stage], ph ^ 1)) { fail(p.status, abort_flag); break; }
          mbar_expect_tx(&afull[stage], Q_A_BYTES);
          tma_load_2d(sA + stage * Q_A_BYTES, &tmA, &afull[stage], kb * BK, mt * BM);
          armed[stage] = 1;
          armed_ph[stage] = ph;
          if (++stage == Q_ASTAGES) { stage = 0; ph ^= 1; }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < Q_ASTAGES; ++s)
          if (armed[s]) (void)mbar_wait(&afull[s], armed_ph[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(BM, BN);
      int ast = 0, cst = 0, acc = 0;
      uint32_t aph = 0, cph = 0, tph = 0;
      int last_ast = -1;
      uint32_t last_aph = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        if (!mbar_wait(&tempty[acc], tph ^ 1)) { fail(p.status, abort_flag); break; }
        fence_after();
        const uint32_t d = tmem + acc * BN;
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&afull[ast], aph) || !mbar_wait(&cfull[cst], cph)) {
            fail(p.status, abort_flag);
            ok = false;
            break;
          }
          fence_after();
          const uint64_t ad = sdesc_sw128(sA + ast * Q_A_BYTES);
          const uint64_t bd = sdesc_sw128(sB + cst * Q_B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          commit(&aempty[ast]);
          commit(&cempty[cst]);
          last_ast = ast;
          last_aph = aph;
          if (++ast == Q_ASTAGES) { ast = 0; aph ^= 1; }
          if (++cst == Q_CSTAGES) { cst = 0; cph ^= 1; }
        }
        if (!ok) break;
        commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) tph ^= 1;
      }
      if (*abort_flag && last_ast >= 0)  // the MMAs issued so far finish before TMEM is freed
        (void)mbar_wait(&aempty[last_ast], last_aph);
    }
  } else if (warp < 6) {
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    int acc = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      const int mt = u % m_tiles, nt = u / m_tiles;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph))) {
        fail(p.status, abort_flag);
        break;
      }
      fence_after();
      const int row = mt * BM + q * 32 + lane;
      const bool row_ok = row < n_rows;
      RowDraw rd{1.f, 0, 0u, 0u, 0u};
      if (SAMPLE && row_ok) rd = row_draw(p.smp, p.row_src ? p.row_src[row] : row);
      float m = -INFINITY, s = 0.f, uu = 0.f, av = -INFINITY;
      int am = 0x7fffffff;
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      float *lrow = nullptr;
      if (p.logits && row_ok)
        lrow = p.logits + (size_t)(p.logits_rows ? p.logits_rows[row] : row) * p.V;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int col0 = nt * BN + c * 32;
        if (col0 >= p.V) break;  // uniform in the warp
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_ld_wait(r);
        const int nvalid = min(32, p.V - col0);
        ent_chunk<true, SAMPLE>(r, nvalid, col0, m, s, uu, av, am, p.gscale, &rd, p.smp.key0,
                                p.smp.key1);
        if (lrow) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nvalid) lrow[col0 + j] = __uint_as_float(r[j]) * p.gscale;
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (row_ok) {
        const size_t o = (size_t)row * p.n_vtiles + nt;
        p.part[o] = make_float4(m, s, uu, av);
        p.part_am[o] = am;
      }
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  } else {
    // converter: thread i of warps 6-13 owns vocabulary row i of the tile.  Codes word w (8
    // codes, columns 8w .. 8w + 7 of the k-block) becomes 16-byte chunk w of the row's 128 bytes,
    // stored at chunk position w ^ (row % 8) (the 128-byte swizzle).
    const int row = (warp - 6) * 32 + lane;
    uint32_t chunk_off[8];  // byte offset of 16-byte chunk c of this row in a tile (swizzled)
#pragma unroll
    for (int c = 0; c < 8; ++c) chunk_off[c] = (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4));
    int qst = 0, cst = 0;
    uint32_t qph = 0, cph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&qfull[qst], qph)) ||
            !__all_sync(0xffffffffu, mbar_wait(&cempty[cst], cph ^ 1))) {
          fail(p.status, abort_flag);
          ok = false;
          break;
        }
        const uint8_t *raw = sR + qst * Q_R_BYTES;
        const uint4 *src = reinterpret_cast<const uint4 *>(raw + row * 32);
        const uint4 q0 = src[0], q1 = src[1];
        const uint32_t sc4 = *reinterpret_cast<const uint32_t *>(raw + Q_C_BYTES + row * 4);
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[qst]);  // the raw stage is in registers now
        const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        __half2 sc[4];  // scale j covers words 2j and 2j + 1
        e4m3_scales_f16x2(sc4, sc[0], sc[1]);
        e4m3_scales_f16x2(sc4 >> 16, sc[2], sc[3]);
        uint8_t *tile = sB + cst * Q_B_BYTES;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t o[4];
          nvfp4_word_f16(w[c], sc[c >> 1], o);
          *reinterpret_cast<uint4 *>(tile + chunk_off[c]) = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();  // the tensor cores read these stores through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&cfull[cst]);
        if (++qst == Q_QSTAGES) { qst = 0; qph ^= 1; }
        if (++cst == Q_CSTAGES) { cst = 0; cph ^= 1; }
      }
      if (!ok) break;
    }
  }
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Merge the partial states of one row over all vocabulary tiles (fixed order) and store the
// entropy and argmax at the row's source index.
__global__ void __launch_bounds__(256) lm_combine_kernel(const float4 *__restrict__ part,
                                                         const int32_t *__restrict__ part_am,
                                                         int n_vtiles,
                                                         const int32_t *__restrict__ n_rows_dev,
                                                         const int32_t *__restrict__ row_idx,
                                                         float *entropy, int32_t *argmax,
                                                         int32_t *st) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  if (n_rows_dev && r >= *n_rows_dev) return;
  EntState es;
  es.init();
  for (int t0 = threadIdx.x; t0 < n_vtiles; t0 += 4 * blockDim.x) {  // four tiles in flight
    float4 v[4];
    int a[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + j * blockDim.x;
      if (t < n_vtiles) {
        v[j] = part[(size_t)r * n_vtiles + t];
        a[j] = part_am[(size_t)r * n_vtiles + t];
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (t0 + j * (int)blockDim.x >= n_vtiles) continue;
      EntState o;
      o.m = v[j].x; o.s = v[j].y; o.u = v[j].z; o.av = v[j].w;
      o.am = a[j];
      es.merge(o);
    }
  }
  __shared__ EntState red[8];
  es = es.warp_reduce();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = es;
  __syncthreads();
  if (threadIdx.x == 0) {
    EntState t = red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) t.merge(red[i]);
    const float H = t.entropy();
    if (!isfinite(H)) set_status(st, DG_ERR_NUMERIC);
    const int out = row_idx ? row_idx[r] : r;
    entropy[out] = H;
    argmax[out] = t.am;
  }
}

}  // namespace

int launch_lmhead_q4(const void *F, int max_rows, const int32_t *n_rows_dev, const uint8_t *codes,
                     const uint8_t *scales, float gscale, int V, int K, const int32_t *row_idx,
                     float *entropy, int32_t *argmax, float *logits, const int32_t *logits_rows,
                     void *ws, int32_t *st, cudaStream_t s, const SampleSpec *smp) {
  if (max_rows <= 0) return DG_OK;
  if (K % 256 != 0 || ((uintptr_t)codes & 15) || ((uintptr_t)scales & 15)) return DG_ERR_UNSUPPORTED;
  const int n_vtiles = (V + BN - 1) / BN;
  CUtensorMap tmA;
  const int rows_alloc = (max_rows + BM - 1) / BM * BM;
  int rc = make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, F, (uint64_t)K,
                        (uint64_t)rows_alloc, (uint64_t)K * 2, BK, BM);
  if (rc != DG_OK) return rc;
  Params p{};
  p.n_rows_dev = n_rows_dev;
  p.max_rows = max_rows;
  p.V = V;
  p.K = K;
  p.n_vtiles = n_vtiles;
  p.part = reinterpret_cast<float4 *>(ws);
  p.part_am = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(ws) +
                                          (size_t)max_rows * n_vtiles * sizeof(float4));
  p.logits = logits;
  p.logits_rows = logits_rows;
  p.status = st;
  p.q_codes = codes;
  p.q_scales = scales;
  p.rows_pad = nvfp4_rows_pad(V + 1);
  p.gscale = gscale;
  const bool sample = smp && smp->mode != SAMPLE_GREEDY;
  if (sample) {
    p.smp = *smp;
    p.row_src = row_idx;
  }
  auto kq = sample ? lmhead_q4_kernel<true> : lmhead_q4_kernel<false>;
  cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Q_SMEM);
  const int units_all = ((max_rows + BM - 1) / BM) * n_vtiles;
  const int grid = units_all < num_sms() ? units_all : num_sms();
  note_launch(s, "lm_head_q4");
  launch_pdl(kq, grid, Q_THREADS, Q_SMEM, s, tmA, p);
  rc = check_launch("lm_head_q4");
  if (rc != DG_OK) return rc;
  note_launch(s, "lm_combine");
  launch_pdl(lm_combine_kernel, max_rows, 256, 0, s, p.part, p.part_am, n_vtiles, n_rows_dev,
             row_idx, entropy, argmax, st);
  return check_launch("lm_combine");
}

size_t lmhead_tc_ws_bytes(int max_rows, int V) {
  const size_t nvt = (size_t)(V + BN - 1) / BN;
  return (size_t)max_rows * nvt * (sizeof(float4) + sizeof(int32_t)) + 256;
}

bool lmhead_tc_supported(int act, int d) { return act == DG_BF16 && d % BK == 0 && d >= BK; }

int launch_lmhead_tc(const void *F, int max_rows, const int32_t *n_rows_dev, const void *w_lm,
                     int V, int K, const int32_t *row_idx, float *entropy, int32_t *argmax,
                     float *logits, const int32_t *logits_rows, void *ws, int32_t *st,
                     cudaStream_t s, const SampleSpec *smp) {
  if (max_rows <= 0) return DG_OK;
  const int n_vtiles = (V + BN - 1) / BN;
  CUtensorMap tmA, tmB;
  // F has room for whole 128-row tiles (rows past max_rows are never stored)
  const int rows_alloc = (max_rows + BM - 1) / BM * BM;
  int rc = make_tmap_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, F, (uint64_t)K,
                        (uint64_t)rows_alloc, (uint64_t)K * 2, BK, BM);
  if (rc != DG_OK) return rc;
  rc = make_tmap_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_lm, (uint64_t)K, (uint64_t)V,
                    (uint64_t)K * 2, BK, BN);
  if (rc != DG_OK) return rc;
  Params p{};
  p.n_rows_dev = n_rows_dev;
  p.max_rows = max_rows;
  p.V = V;
  p.K = K;
  p.n_vtiles = n_vtiles;
  p.part = reinterpret_cast<float4 *>(ws);
  p.part_am = reinterpret_cast<int32_t *>(reinterpret_cast<char *>(ws) +
                                          (size_t)max_rows * n_vtiles * sizeof(float4));
  p.logits = logits;
  p.logits_rows = logits_rows;
  p.status = st;
  const bool sample = smp && smp->mode != SAMPLE_GREEDY;
  if (sample) {
    p.smp = *smp;
    p.row_src = row_idx;
  }
  auto k1 = sample ? lmhead_tc_kernel<true> : lmhead_tc_kernel<false>;
  auto k2 = sample ? lmhead_tc2_kernel<true> : lmhead_tc2_kernel<false>;
  // The number of rows is known on the device only.  Up to 128 rows the single-CTA kernel runs;
  // beyond, CTA pairs with the 2-SM MMA (each SM streams half of every weight tile).  When both
  // are possible both are launched and the one that does not apply returns at once.
  p.only_one_tile = max_rows > BM;
  if (max_rows > BM) {
    CUtensorMap tmB2;
    rc = make_tmap_2d(&tmB2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_lm, (uint64_t)K, (uint64_t)V,
                      (uint64_t)K * 2, BK, BN / 2);  // each CTA loads 128 of the 256 rows
    if (rc != DG_OK) return rc;
    cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P_SMEM_BYTES);
    const int pairs_max = ((max_rows + 2 * BM - 1) / (2 * BM)) * n_vtiles;
    const int pairs = pairs_max < num_sms() / 2 ? pairs_max : num_sms() / 2;
    note_launch(s, "lm_head_tc2");
    launch_pdl_cluster(k2, 2 * pairs, NUM_THREADS, P_SMEM_BYTES, s, 2, tmA, tmB2, p);
    rc = check_launch("lm_head_tc2");
    if (rc != DG_OK) return rc;
  }
  cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
  {
    const int units_max = n_vtiles;  // one row tile: the single-CTA kernel's only case here
    const int units_all = ((max_rows + BM - 1) / BM) * n_vtiles;
    const int um = p.only_one_tile ? units_max : units_all;
    const int grid = um < num_sms() ? um : num_sms();
    note_launch(s, "lm_head_tc");
    launch_pdl(k1, grid, NUM_THREADS, SMEM_BYTES, s, tmA, tmB, p);
  }
  rc = check_launch("lm_head_tc");
  if (rc != DG_OK) return rc;
  note_launch(s, "lm_combine");
  launch_pdl(lm_combine_kernel, max_rows, 256, 0, s, p.part, p.part_am, n_vtiles, n_rows_dev, row_idx,
                                             entropy, argmax, st);
  return check_launch("lm_combine");
}

}  // namespace dg
