// GEMM on CUDA cores: C = A B^T with fp32 accumulation in k order, for every projection of the
// layer (QKV, output, router, the grouped expert GEMMs) and the LM head.  It is the fp32 path
// of the tiny workload and the always-available path for every dtype; the bf16 hot GEMMs also
// have tensor-core kernels.
//
// Tile 64 x 64 x 16, 256 threads, 4 x 4 outputs per thread.  Grouped mode (the MoE experts,
// model card "diffusiongemma", Mixture-of-Experts bullet) reads a device tile list so that only
// the tiles of experts that received tokens run.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename AT, typename WT>
struct Args {
  const AT *A; int lda;
  const WT *B; int ldb; long long strideB;
  const float *bscale;
  int M, N, K;
  const int32_t *M_dev;
  const int32_t *a_rowmap; int a_rowdiv;
  const GroupTile *tiles; const int32_t *n_tiles; const int32_t *group_off;
};

template <typename AT, typename WT, typename OT, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(Args<AT, WT> g, OT *out, int ldo,
                                                        const OT *res) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int n0 = blockIdx.y * BN;
  int group = 0, m0, arow0 = 0, mlim;
  if (g.tiles) {
    if ((int)blockIdx.x >= *g.n_tiles) return;
    const GroupTile t = g.tiles[blockIdx.x];
    group = t.g;
    m0 = t.m0;
    arow0 = g.group_off[group];
    mlim = g.group_off[group + 1] - arow0;
  } else {
    m0 = blockIdx.x * BM;
    mlim = g.M_dev ? min(*g.M_dev, g.M) : g.M;
  }
  if (m0 >= mlim) return;
  const WT *B = g.B + (long long)group * g.strideB;
  const float *bs = g.bscale ? g.bscale + (long long)group * g.N : nullptr;

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int lr = threadIdx.x >> 2, lk = (threadIdx.x & 3) * 4;
  // source rows for the loads of this thread
  const int am = m0 + lr;
  const AT *arow = nullptr;
  if (am < mlim) {
    int r = arow0 + am;
    if (g.a_rowmap) r = g.a_rowmap[r] / g.a_rowdiv;
    arow = g.A + (long long)r * g.lda;
  }
  const int bn = n0 + lr;
  const WT *brow = (bn < g.N) ? B + (long long)bn * g.ldb : nullptr;

  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < g.K; k0 += BK) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k = k0 + lk + u;
      As[lk + u][lr] = (arow && k < g.K) ? to_f(arow[k]) : 0.f;
      Bs[lk + u][lr] = (brow && k < g.K) ? to_f(brow[k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= mlim) continue;
    const long long orow = (long long)(arow0 + m) * ldo;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      float v = acc[i][j];
      if (bs) v *= bs[n];
      if (EPI == EPI_RESID) v += to_f(res[orow + n]);
      out[orow + n] = from_f<OT>(v);
    }
  }
}

template <typename AT, typename WT>
int run(const GemmDesc &d, int epi, void *out, int ldo, const void *res, cudaStream_t s) {
  Args<AT, WT> a{(const AT *)d.A, d.lda, (const WT *)d.B, d.ldb, d.strideB, d.bscale,
                 d.M, d.N, d.K, d.M_dev, d.a_rowmap, d.a_rowdiv > 0 ? d.a_rowdiv : 1,
                 d.tiles, d.n_tiles, d.group_off};
  const int gx = d.tiles ? d.max_tiles : (d.M + BM - 1) / BM;
  dim3 grid(gx, (d.N + BN - 1) / BN);
  if (gx <= 0) return DG_OK;
  note_launch(s, d.name ? d.name : "gemm_simt");
  if (epi == EPI_F32)
    launch_pdl(gemm_simt_kernel<AT, WT, float, EPI_F32>, grid, 256, 0, s, a, (float *)out, ldo, nullptr);
  else if (epi == EPI_ACT)
    launch_pdl(gemm_simt_kernel<AT, WT, AT, EPI_ACT>, grid, 256, 0, s, a, (AT *)out, ldo, nullptr);
  else
    launch_pdl(gemm_simt_kernel<AT, WT, float, EPI_RESID>, grid, 256, 0, s, a, (float *)out, ldo,
                                                                    (const float *)res);
  return check_launch("gemm_simt");
}

}  // namespace

int launch_gemm_simt(const GemmDesc &d, int epi, void *out, int ldo, const void *res,
                     cudaStream_t s) {
  if (d.act == DG_F32 && d.w == DG_F32) return run<float, float>(d, epi, out, ldo, res, s);
  if (d.act == DG_BF16 && d.w == DG_BF16) return run<bf16, bf16>(d, epi, out, ldo, res, s);
  if (d.act == DG_BF16 && d.w == DG_E4M3) return run<bf16, fp8>(d, epi, out, ldo, res, s);
  return DG_ERR_UNSUPPORTED;
}

}  // namespace dg
