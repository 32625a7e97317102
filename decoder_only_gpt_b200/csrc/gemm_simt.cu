// fp32 SIMT GEMM for the GPT_F32 storage type: C[m,n] = sum_k A(m,k) B(n,k)
// with either operand K-major or MN-major, 64x64x16 tiles, 4x4 outputs per
// thread, and the epilogues of epilogue.cuh (plus the cross-entropy row
// statistics).  bf16 GEMMs run on the tcgen05 kernel of gemm_tc.cu.
#include "epilogue.cuh"

namespace gpt {

namespace {
constexpr int BM = 64, BN = 64, BK = 16;
}

template <typename T, bool AMN, bool BMN>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Cs[BM][BN + 1];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int tr = tid / 16, tc = tid % 16;
  const T* A = static_cast<const T*>(g.A);
  const T* B = static_cast<const T*>(g.B);
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < g.K; k0 += BK) {
    for (int e = tid; e < BM * BK; e += 256) {
      int mm = AMN ? e % BM : e / BK;
      int kk = AMN ? e / BM : e % BK;
      int m = m0 + mm, k = k0 + kk;
      float v = 0.f;
      if (m < g.M && k < g.K) v = to_f(AMN ? A[int64_t(k) * g.lda + m] : A[int64_t(m) * g.lda + k]);
      As[kk][mm] = v;
    }
    for (int e = tid; e < BN * BK; e += 256) {
      int nn = BMN ? e % BN : e / BK;
      int kk = BMN ? e / BN : e % BK;
      int n = n0 + nn, k = k0 + kk;
      float v = 0.f;
      if (n < g.N && k < g.K) v = to_f(BMN ? B[int64_t(k) * g.ldb + n] : B[int64_t(n) * g.ldb + k]);
      Bs[kk][nn] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][tr + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tc + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  if (g.epi == EPI_CE_FWD) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) Cs[tr + 16 * i][tc + 16 * j] = acc[i][j];
    __syncthreads();
    if (tid < BM) {
      const int m = m0 + tid;
      if (m < g.M) {
        const int nend = min(BN, g.n_valid - n0);
        float mx = -INFINITY;
        for (int j = 0; j < nend; ++j) mx = fmaxf(mx, Cs[tid][j]);
        float s = 0.f;
        for (int j = 0; j < nend; ++j) s += expf(Cs[tid][j] - mx);
        g.part_max[int64_t(m) * g.n_part + blockIdx.x] = mx;
        g.part_sum[int64_t(m) * g.n_part + blockIdx.x] = s;
        int y = g.targets[m];
        if (y >= n0 && y < n0 + nend) g.tgt_logit[m] = Cs[tid][y - n0];
      }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + tr + 16 * i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tc + 16 * j;
      if (n < g.N) epi_elem<T>(g, m, n, acc[i][j]);
    }
  }
}

template <typename T>
static int launch_simt(GemmArgs g, cudaStream_t st) {
  dim3 grid(ceil_div(g.N, BN), ceil_div(g.M, BM));
  if (g.epi == EPI_CE_FWD) g.n_part = int(grid.x);
  if (!g.a_mn_major && !g.b_mn_major) gemm_simt_kernel<T, false, false><<<grid, 256, 0, st>>>(g);
  else if (!g.a_mn_major && g.b_mn_major) gemm_simt_kernel<T, false, true><<<grid, 256, 0, st>>>(g);
  else if (g.a_mn_major && !g.b_mn_major) gemm_simt_kernel<T, true, false><<<grid, 256, 0, st>>>(g);
  else gemm_simt_kernel<T, true, true><<<grid, 256, 0, st>>>(g);
  return last_launch_rc();
}

int launch_gemm_simt_f32(const GemmArgs& g, void* stream) {
  // the folded RMSNorm backward is a tensor-core epilogue only
  if (g.epi == EPI_NORM_BWD || g.norm_part_out) return 1;
  return launch_simt<float>(g, (cudaStream_t)stream);
}

int gemm_simt_tile_n() { return BN; }

}  // namespace gpt
