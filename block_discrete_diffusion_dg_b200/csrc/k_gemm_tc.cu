// Tensor-core GEMMs of the layer: the dense projections (QKV, output projection + residual) and
// the grouped expert GEMMs of the MoE FFN (model card "diffusiongemma", Mixture-of-Experts
// bullet: 8 of 128 experts per token).
//
// D[128 x n] = A[128 x K] * B[n x K]^T on tcgen05 (kind::f16, bf16 operands, fp32 accumulator in
// TMEM), K-major operands staged by TMA with the 128-byte swizzle.  Persistent and
// warp-specialised like the LM-head kernel: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer,
// warps 2-5 epilogue over a double-buffered accumulator.
//
// Dense:  A = activation rows (M = tokens), B = weight rows (N = output channels).
// Split (swap-AB, split-K; at most 256 tokens): A = 128 weight rows (output channels), B = all
// the token rows; a unit is (channel tile, K slice) and leaves an fp32 partial
// part[slice][token][channel] that the consumer sums over the slices in order.  Each unit runs
// K / slices of the reduction, so ~128 CTAs stream the weights in a few k-steps each, and the
// activation rows are read once per channel tile instead of once per 64 channels.
// Experts (swap-AB): A = expert weight rows (M = 128 output channels), B = the tokens routed to
// the expert (N = their count rounded up to 16, at most BN_MAX per unit), so the weights stream
// through the tensor cores once at the small per-expert token counts of batch 1.  For the
// gate/up GEMM the 128 A rows are 64 gate rows and the matching 64 up rows, and the epilogue
// forms a = gelu_tanh(gate) * up; the down GEMM stores Y.
// Waits are bounded (tc::WAIT_LIMIT_CYCLES) and record DG_ERR_TIMEOUT on expiry.
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace dg {

namespace {

using namespace tc;

constexpr int BM = 128, BK = 64;
constexpr int NUM_THREADS = 192;

enum Kind { K_DENSE_F32 = 0, K_DENSE_RESID = 1, K_MOE_GATE = 2, K_MOE_DOWN = 3, K_SPLIT = 4 };

struct Params {
  int kind, K;
  // dense: M rows (tokens), N columns (channels), tile width bn
  // split: M tokens, N channels, m_tiles = N / 128 channel tiles, k_split K slices
  int M, N, m_tiles, bn, k_split;
  float *out_f32;        // dense output (fp32)
  const float *res;      // dense residual (fp32) or null
  int ldo;
  // experts: token tiles (expert, first token) and per-expert row offsets
  const GroupTile *tiles;
  const int32_t *n_tiles_dev;
  const int32_t *expert_off;
  int w_rows;       // weight rows per expert (2F for gate/up, d for down)
  int F;            // expert FFN width (gate/up half)
  int ld_out;       // row stride of the expert output (F for a, d for Y)
  void *out;        // gate/up: a [assignments][F] (bf16); down: Y [assignments][d] (fp32)
  const float *scale;  // per output channel (dense: [N]; experts: [E][w_rows]) or null
  int smem_epi;        // split with one unit per CTA: stage the tile in the (then idle) pipeline
                       // buffers and write it with one TMA store through tmC
  int a_static;        // split: A is a weight no kernel of the stream writes, so its first stages
                       // are fetched before the wait on the preceding kernel
  int32_t *status;
};

struct Unit {
  int a_row0, a_row1;  // A box rows (a_row1 < 0: one 128-row box)
  int b_row0, n_mma;   // first B row, MMA N (multiple of 16)
  int n_valid;         // valid columns
  int row0, col0;      // dense: first token row / first channel; experts: first channel, pos0
};

__device__ __forceinline__ int n_units(const Params &p) {
  if (p.kind <= K_DENSE_RESID) return p.m_tiles * ((p.N + p.bn - 1) / p.bn);
  if (p.kind == K_SPLIT) return p.m_tiles * p.k_split;
  return *p.n_tiles_dev * p.m_tiles;
}

template <int BN_MAX>
__device__ __forceinline__ Unit decode(const Params &p, int u) {
  Unit x;
  const int mt = u % p.m_tiles, t = u / p.m_tiles;
  if (p.kind == K_SPLIT) {
    x.a_row0 = mt * BM;
    x.a_row1 = -1;
    x.b_row0 = 0;
    x.n_valid = p.M;
    x.n_mma = (p.M + 15) & ~15;
    x.row0 = mt * BM;  // first channel
    x.col0 = t;        // K slice
  } else if (p.kind <= K_DENSE_RESID) {
    x.a_row0 = mt * BM;
    x.a_row1 = -1;
    x.b_row0 = t * p.bn;
    x.n_valid = min(p.bn, p.N - x.b_row0);
    x.n_mma = (x.n_valid + 15) & ~15;
    x.row0 = mt * BM;
    x.col0 = x.b_row0;
  } else {
    const GroupTile g = p.tiles[t];
    const int off = p.expert_off[g.g];
    const int cnt = p.expert_off[g.g + 1] - off;
    x.n_valid = min(BN_MAX, cnt - g.m0);
    x.n_mma = (x.n_valid + 15) & ~15;
    x.b_row0 = off + g.m0;
    x.col0 = off + g.m0;  // first output row (assignment position)
    if (p.kind == K_MOE_GATE) {
      x.a_row0 = g.g * p.w_rows + mt * 64;
      x.a_row1 = g.g * p.w_rows + p.F + mt * 64;
      x.row0 = mt * 64;  // first gate channel
    } else {
      x.a_row0 = g.g * p.w_rows + mt * BM;
      x.a_row1 = -1;
      x.row0 = mt * BM;  // first output channel
    }
  }
  return x;
}

__device__ __forceinline__ void fail(int32_t *st, volatile int *abort_flag) {
  set_status(st, DG_ERR_TIMEOUT);
  *abort_flag = 1;
}

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int BN_MAX, int STAGES>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN_MAX * BK * 2;
  // accumulators are read in chunks of 32 columns, so each buffer spans at least 32
  static constexpr int ACC_STRIDE = BN_MAX < 32 ? 32 : BN_MAX;
  static constexpr uint32_t TMEM_COLS = 2 * ACC_STRIDE;
  static constexpr int XCH_BYTES = 64 * 33 * 4;  // gate/up exchange: 64 rows x 32 columns
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES) + XCH_BYTES + 256;
};

template <int BN_MAX, int STAGES, int B_BOX>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, Params p) {
  // Programmatic dependent launch: with a static A the weight stream starts before the wait on the
  // preceding kernel (whose output only B and the stores depend on); every role that reads that
  // output or writes this kernel's output waits first.
  const bool early = p.kind == K_SPLIT && p.a_static;
  if (!early) pdl_wait();
  pdl_trigger();
  using C = Cfg<BN_MAX, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * C::A_BYTES;
  float *xch = reinterpret_cast<float *>(sB + STAGES * C::B_BYTES);
  uint64_t *full = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(xch) + C::XCH_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = n_units(p);
  if ((int)blockIdx.x >= units) return;
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
    if (p.smem_epi) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
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
      // early: the A boxes of the first unit's first k-blocks go out before the dependency wait
      // (the ring is empty, so stages 0 .. pre-1 in phase 0 are free); the loop below then adds
      // only their B boxes, which the same full barrier counts
      int pre = 0;
      if (early) {
        const Unit x = decode<BN_MAX>(p, blockIdx.x);
        const int nb = (x.n_mma + B_BOX - 1) / B_BOX;
        const int kpb = kblocks / p.k_split, kb0 = x.col0 * kpb;
        pre = kpb < STAGES ? kpb : STAGES;
        for (int j = 0; j < pre; ++j) {
          mbar_expect_tx(&full[j], C::A_BYTES + (uint32_t)nb * B_BOX * BK * 2);
          tma_load_2d(sA + j * C::A_BYTES, &tmA, &full[j], (kb0 + j) * BK, x.a_row0);
          armed[j] = 1;
        }
        pdl_wait();
      }
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const Unit x = decode<BN_MAX>(p, u);
        const int nb = (x.n_mma + B_BOX - 1) / B_BOX;
        const uint32_t bytes = C::A_BYTES + (uint32_t)nb * B_BOX * BK * 2;
        const int kpb = p.kind == K_SPLIT ? kblocks / p.k_split : kblocks;
        const int kb0 = p.kind == K_SPLIT ? x.col0 * kpb : 0;
        for (int kb = kb0; kb < kb0 + kpb; ++kb) {
          if (!mbar_wait(&empty[stage], ph ^ 1)) { fail(p.status, abort_flag); break; }
          uint8_t *a = sA + stage * C::A_BYTES;
          if (u == (int)blockIdx.x && kb - kb0 < pre) {
            // A already in flight, bytes already expected
          } else if (x.a_row1 < 0) {
            mbar_expect_tx(&full[stage], bytes);
            tma_load_2d(a, &tmA, &full[stage], kb * BK, x.a_row0);
          } else {
            mbar_expect_tx(&full[stage], bytes);
            tma_load_2d(a, &tmA, &full[stage], kb * BK, x.a_row0);
            tma_load_2d(a + 64 * BK * 2, &tmA, &full[stage], kb * BK, x.a_row1);
          }
          uint8_t *b = sB + stage * C::B_BYTES;
          for (int i = 0; i < nb; ++i)
            tma_load_2d(b + i * B_BOX * BK * 2, &tmB, &full[stage], kb * BK, x.b_row0 + i * B_BOX);
          armed[stage] = 1;
          armed_ph[stage] = ph;
          if (++stage == STAGES) { stage = 0; ph ^= 1; }
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < STAGES; ++s)
          if (armed[s]) (void)mbar_wait(&full[s], armed_ph[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      int last_stage = -1;
      uint32_t last_ph = 0;
      // stage descriptors = base descriptor + byte offset / 16 (the start-address field holds the
      // shared-memory address / 16), so the issue loop does not rebuild them per k-block
      const uint64_t dA = sdesc_sw128(sA), dB = sdesc_sw128(sB);
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const Unit x = decode<BN_MAX>(p, u);
        const uint32_t idesc = idesc_bf16(BM, x.n_mma);
        if (!mbar_wait(&tempty[acc], aph ^ 1)) { fail(p.status, abort_flag); break; }
        fence_after();
        const uint32_t d = tmem + acc * C::ACC_STRIDE;
        bool ok = true;
        const int kpb = p.kind == K_SPLIT ? kblocks / p.k_split : kblocks;
        const int kb0 = p.kind == K_SPLIT ? x.col0 * kpb : 0;
        for (int kb = kb0; kb < kb0 + kpb; ++kb) {
          if (!mbar_wait(&full[stage], ph)) { fail(p.status, abort_flag); ok = false; break; }
          fence_after();
          const uint64_t ad = dA + (uint64_t)((stage * C::A_BYTES) >> 4);
          const uint64_t bd = dB + (uint64_t)((stage * C::B_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            mma_bf16(d, ad + 2 * k, bd + 2 * k, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
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
      if (*abort_flag && last_stage >= 0) (void)mbar_wait(&empty[last_stage], last_ph);
    }
  } else {
    if (early) pdl_wait();  // before the first read of the tiles or store of this kernel's output
    const int q = warp & 3;
    int acc = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;  // warp-uniform exit
      const Unit x = decode<BN_MAX>(p, u);
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph))) {
        fail(p.status, abort_flag);
        break;
      }
      fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_STRIDE);
      const int r = q * 32 + lane;  // accumulator row of this thread
#pragma unroll 1
      for (int c = 0; c * 32 < x.n_valid; ++c) {
        uint32_t v[32];
        tmem_ld32(tbase + c * 32, v);
        tmem_ld_wait(v);
        const int nv = min(32, x.n_valid - c * 32);
        if (p.scale) {  // e4m3 weights: the fp32 accumulator times the output channel's scale
          if (p.kind == K_SPLIT) {
            const float sc = p.scale[x.row0 + r];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * sc);
          } else if (p.kind == K_DENSE_F32 || p.kind == K_DENSE_RESID) {
            const float *sc = p.scale + x.col0 + c * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nv) v[j] = __float_as_uint(__uint_as_float(v[j]) * sc[j]);
          } else {
            const GroupTile g = p.tiles[u / p.m_tiles];
            const int arow = (p.kind == K_MOE_GATE)
                                 ? (q < 2 ? x.row0 + r : p.F + x.row0 + (r - 64))
                                 : x.row0 + r;
            const float sc = p.scale[(size_t)g.g * p.w_rows + arow];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * sc);
          }
        }
        if (p.kind == K_SPLIT && p.smem_epi) {
          // staged as [token][128 channels] over the pipeline buffers (all MMAs of the CTA's only
          // unit have completed, so nothing reads or fills them any more)
          float *stg = reinterpret_cast<float *>(sA);
#pragma unroll
          for (int j = 0; j < 32; ++j) stg[(c * 32 + j) * BM + r] = __uint_as_float(v[j]);
        } else if (p.kind == K_SPLIT) {
          // part[slice][token][channel]: for each token the 32 lanes store 32 consecutive channels
          const int ch = x.row0 + r;
          float *o = p.out_f32 + ((size_t)x.col0 * p.M + c * 32) * p.ldo + ch;
          if (ch < p.N) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < nv) o[(size_t)j * p.ldo] = __uint_as_float(v[j]);
          }
        } else if (p.kind == K_DENSE_F32 || p.kind == K_DENSE_RESID) {
          const int row = x.row0 + r;
          if (row < p.M) {
            const int col = x.col0 + c * 32;
            if (p.kind == K_DENSE_F32) {
              float *o = p.out_f32 + (size_t)row * p.ldo + col;
              if (nv == 32) {
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                  *reinterpret_cast<float4 *>(o + j) =
                      make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                                  __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nv) o[j] = __uint_as_float(v[j]);
              }
            } else {
              const float *rs = p.res + (size_t)row * p.ldo + col;
              float *o = p.out_f32 + (size_t)row * p.ldo + col;
              if (nv == 32) {
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                  const float4 rr = *reinterpret_cast<const float4 *>(rs + j);
                  *reinterpret_cast<float4 *>(o + j) =
                      make_float4(__uint_as_float(v[j]) + rr.x, __uint_as_float(v[j + 1]) + rr.y,
                                  __uint_as_float(v[j + 2]) + rr.z, __uint_as_float(v[j + 3]) + rr.w);
                }
              } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  if (j < nv) o[j] = __uint_as_float(v[j]) + rs[j];
              }
            }
          }
        } else if (p.kind == K_MOE_DOWN) {
          const int ch = x.row0 + r;
          float *Y = reinterpret_cast<float *>(p.out);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < nv) Y[(size_t)(x.col0 + c * 32 + j) * p.ld_out + ch] = __uint_as_float(v[j]);
        } else {  // K_MOE_GATE: rows 0-63 gate, 64-127 up of the same channels
          if (q >= 2) {
#pragma unroll
            for (int j = 0; j < 32; ++j) xch[((q - 2) * 32 + lane) * 33 + j] = __uint_as_float(v[j]);
          }
          epi_bar();
          if (q < 2) {
            const int ch = x.row0 + r;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j >= nv) continue;
              const float g = __uint_as_float(v[j]);
              const float up = xch[(q * 32 + lane) * 33 + j];
              const float gl =
                  0.5f * g * (1.0f + tanhf(0.7978845608028654f * (g + 0.044715f * g * g * g)));
              reinterpret_cast<bf16 *>(p.out)[(size_t)(x.col0 + c * 32 + j) * p.ld_out + ch] =
                  __float2bfloat16_rn(gl * up);
            }
          }
          epi_bar();
        }
      }
      if (p.kind == K_SPLIT && p.smem_epi) {  // one TMA store of the [tokens][128] fp32 tile
        fence_proxy_async_smem();
        epi_bar();
        if (warp == 2 && lane == 0) {
          tma_store_3d(&tmC, sA, x.row0, 0, x.col0);
          bulk_commit();
          bulk_wait_all();
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int BN_MAX, int STAGES, int B_BOX>
int launch(const CUtensorMap &tmA, const CUtensorMap &tmB, const Params &p, int units_max,
           const char *name, cudaStream_t s, int ctas_per_sm = 1,
           const CUtensorMap *tmC = nullptr) {
  using C = Cfg<BN_MAX, STAGES>;
  auto k = gemm_tc_kernel<BN_MAX, STAGES, B_BOX>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  const int slots = num_sms() * ctas_per_sm;
  const int grid = units_max < slots ? units_max : slots;
  if (grid <= 0) return DG_OK;
  note_launch(s, name);
  launch_pdl(k, grid, NUM_THREADS, C::SMEM, s, tmA, tmB, tmC ? *tmC : tmA, p);
  return check_launch(name);
}

}  // namespace

// bf16 activations with bf16 weights, or with e4m3 weights that the caller dequantises to bf16
// first (the scales are applied in the epilogue).
bool gemm_tc_supported(int act, int w, int K) {
  return act == DG_BF16 && (w == DG_BF16 || w == DG_E4M3) && K % BK == 0 && K >= BK;
}

// Dense: out[M][N] = A[M][K] * W[N][K]^T (+ res[M][N]), fp32 output.  At batch 1 these are
// latency-bound weight streams (M = 256 tokens), so the channel tiles are narrow (64, or 16 for
// N <= 256) to spread each weight matrix over enough CTAs.  With many token rows (M >= 1024, e.g.
// 32 canvases) the product is compute-bound instead: 128 x 256 tiles, so each activation tile is
// read N / 256 times rather than N / 64 and every MMA is the full 256 columns wide.
int launch_gemm_tc_dense(const void *A, int M, const void *W, int N, int K, float *out,
                         const float *res, int ldo, const char *name, int32_t *st, cudaStream_t s,
                         const float *scale) {
  const int BN = M >= 1024 ? (N <= 128 ? 128 : 256) : (N <= 256 ? 16 : 64);
  const int M_alloc = (M + BM - 1) / BM * BM;  // A has room for whole tiles (caller's layout)
  CUtensorMap ta, tb;
  int rc = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, K, M_alloc, (uint64_t)K * 2, BK,
                        BM);
  if (rc != DG_OK) return rc;
  rc = make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, K, N, (uint64_t)K * 2, BK, BN);
  if (rc != DG_OK) return rc;
  Params p{};
  p.kind = res ? K_DENSE_RESID : K_DENSE_F32;
  p.K = K;
  p.M = M;
  p.N = N;
  p.m_tiles = M_alloc / BM;
  p.bn = BN;
  p.out_f32 = out;
  p.res = res;
  p.scale = scale;
  p.ldo = ldo;
  p.status = st;
  const int units = p.m_tiles * ((N + BN - 1) / BN);
  if (BN == 16) return launch<16, 10, 16>(ta, tb, p, units, name, s);
  if (BN == 256) return launch<256, 4, 256>(ta, tb, p, units, name, s);
  if (BN == 128) return launch<128, 6, 128>(ta, tb, p, units, name, s);
  return launch<64, 8, 64>(ta, tb, p, units, name, s);
}

// Split: part[s][t][n] = sum over k in slice s of W[n][k] X[t][k] (times scale[n] when given), for
// t < T <= 256, n < N (N a multiple of 128), slices s < k_split (K a multiple of 64 k_split).  X is
// the activation buffer [T_alloc][K] with T_alloc >= T rows allocated.
int split_k_slices(int N, int K, int max_slices) {
  const int m_tiles = N / BM, kblocks = K / BK;
  int s = num_sms() / (m_tiles > 0 ? m_tiles : 1);
  if (s > max_slices) s = max_slices;
  if (s < 1) s = 1;
  if (s > kblocks) s = kblocks;
  while (kblocks % s) --s;
  return s;
}

bool split_supported(int act, int w, int T, int N, int K) {
  return gemm_tc_supported(act, w, K) && T > 0 && T <= 256 && N % BM == 0;
}

int launch_gemm_tc_split(const void *W, int N, const void *X, int T, int T_alloc, int K,
                         int k_split, float *part, const char *name, int32_t *st, cudaStream_t s,
                         const float *scale, bool w_static) {
  if (T <= 0 || T > 256 || N % BM || K % (BK * k_split)) return DG_ERR_UNSUPPORTED;
  const int bn = T <= 128 ? 128 : 256;
  CUtensorMap ta, tb;
  int rc = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, K, N, (uint64_t)K * 2, BK, BM);
  if (rc != DG_OK) return rc;
  rc = make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, K, T_alloc, (uint64_t)K * 2, BK,
                    bn);
  if (rc != DG_OK) return rc;
  Params p{};
  p.kind = K_SPLIT;
  p.K = K;
  p.M = T;
  p.N = N;
  p.m_tiles = N / BM;
  p.k_split = k_split;
  p.out_f32 = part;
  p.ldo = N;
  p.scale = scale;
  p.status = st;
  p.a_static = w_static ? 1 : 0;
  const int units = p.m_tiles * k_split;
  // one unit per CTA: the epilogue stages the tile in shared memory and stores it with TMA
  CUtensorMap tc_out;
  p.smem_epi = 0;
  if (units <= num_sms()) {
    rc = make_tmap_3d_f32(&tc_out, part, N, T, k_split, BM, bn, 1);
    if (rc != DG_OK) return rc;
    p.smem_epi = 1;
  }
  if (bn == 128) return launch<128, 6, 128>(ta, tb, p, units, name, s, 1, &tc_out);
  return launch<256, 4, 256>(ta, tb, p, units, name, s, 1, &tc_out);
}

// Experts (swap-AB).  gate_up: W [E][2F][K], X = the routed rows [assignments][K] (permuted order)
// -> a [assignments][F] (bf16).  down: W [E][d][F], X = a -> Y [assignments][d] (fp32).
// Token tile of the expert GEMMs and the depth of their shared-memory ring (weights stream through
// STAGES x 16 KB; the routed tokens take BN_MAX x 128 bytes per stage).
#ifndef DG_MOE_BN
#define DG_MOE_BN 128
#endif
#ifndef DG_MOE_STAGES
#define DG_MOE_STAGES 3
#endif
#ifndef DG_MOE_CTAS_PER_SM
#define DG_MOE_CTAS_PER_SM 2
#endif

int launch_gemm_tc_experts(int gate_up, const void *W, int E, int w_rows, int F, const void *X,
                           int n_assign_max, int K, const GroupTile *tiles,
                           const int32_t *n_tiles_dev, int max_tiles, const int32_t *expert_off,
                           void *out, int ld_out, const char *name, int32_t *st, cudaStream_t s,
                           const float *scale) {
  constexpr int BN_MAX = DG_MOE_BN, B_BOX = 32;
  CUtensorMap ta, tb;
  int rc = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, K, (uint64_t)E * w_rows,
                        (uint64_t)K * 2, BK, gate_up ? 64 : BM);
  if (rc != DG_OK) return rc;
  rc = make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, X, K, n_assign_max, (uint64_t)K * 2,
                    BK, B_BOX);
  if (rc != DG_OK) return rc;
  Params p{};
  p.kind = gate_up ? K_MOE_GATE : K_MOE_DOWN;
  p.K = K;
  p.tiles = tiles;
  p.n_tiles_dev = n_tiles_dev;
  p.expert_off = expert_off;
  p.w_rows = w_rows;
  p.F = F;
  p.m_tiles = gate_up ? F / 64 : w_rows / BM;
  p.ld_out = ld_out;
  p.out = out;
  p.scale = scale;
  p.status = st;
  return launch<BN_MAX, DG_MOE_STAGES, B_BOX>(ta, tb, p, max_tiles * p.m_tiles, name, s,
                                              DG_MOE_CTAS_PER_SM);
}

int experts_tc_tile_tokens() { return DG_MOE_BN; }

}  // namespace dg
