// GEMM on the CUDA cores in fp32 (lazy block updates of the sweep) and fp64 (rank-k
// updates of the factorisation): C = beta*C + alpha * A * op(B).
//
// 128x128 tile per 256-thread CTA, 8x8 outputs per thread, K staged 8 at a time through
// double-buffered shared memory.  All operands are row-major with arbitrary leading
// dimensions; every global access is bounds-checked, so ragged edges need no padding.
//
// In-place use: when C aliases A (or B) the call is still correct as long as each CTA
// is the only reader of the A rows (B columns) it writes, i.e. N <= 128 (M <= 128),
// because a CTA reads all of K before its epilogue writes.  The callers rely on this.
#include "common.cuh"

namespace gptq {
namespace {

constexpr int TM = 128, TN = 128, TK = 8, PAD = 4;

template <typename T, bool TRANSB, typename CT>
__global__ void __launch_bounds__(256) gemm_kernel(int64_t M, int64_t N, int64_t K, T alpha, const T* A,
                                                   int64_t lda, const T* B, int64_t ldb, T beta, CT* C,
                                                   int64_t ldc, int upper) {
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * TM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * TN;
  if (upper && n0 + TN - 1 < m0) return;

  __shared__ __align__(16) T As[2][TK][TM + PAD];
  __shared__ __align__(16) T Bs[2][TK][TN + PAD];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  T ra[4], rb[4];
  auto load_regs = [&](int64_t k0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + 256 * i;
      const int am = e >> 3, ak = e & 7;
      const int64_t gm = m0 + am, gk = k0 + ak;
      ra[i] = (gm < M && gk < K) ? A[gm * lda + gk] : T(0);
      if (TRANSB) {
        const int bn = e >> 3, bk = e & 7;
        const int64_t gn = n0 + bn, gk2 = k0 + bk;
        rb[i] = (gn < N && gk2 < K) ? B[gn * ldb + gk2] : T(0);
      } else {
        const int bk = e >> 7, bn = e & 127;
        const int64_t gn = n0 + bn, gk2 = k0 + bk;
        rb[i] = (gn < N && gk2 < K) ? B[gk2 * ldb + gn] : T(0);
      }
    }
  };
  auto store_smem = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + 256 * i;
      As[buf][e & 7][e >> 3] = ra[i];
      if (TRANSB)
        Bs[buf][e & 7][e >> 3] = rb[i];
      else
        Bs[buf][e >> 7][e & 127] = rb[i];
    }
  };

  T acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = T(0);

  const int64_t nkt = (K + TK - 1) / TK;
  int buf = 0;
  if (nkt > 0) {
    load_regs(0);
    store_smem(0);
  }
  __syncthreads();
  for (int64_t kt = 0; kt < nkt; ++kt) {
    if (kt + 1 < nkt) load_regs((kt + 1) * TK);
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      T a[8], b[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = As[buf][k][ty * 4 + q];
        a[4 + q] = As[buf][k][64 + ty * 4 + q];
        b[q] = Bs[buf][k][tx * 4 + q];
        b[4 + q] = Bs[buf][k][64 + tx * 4 + q];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    if (kt + 1 < nkt) store_smem(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gn >= N) continue;
      CT* cp = C + gm * ldc + gn;
      const T v = alpha * acc[i][j];
      if constexpr (sizeof(CT) > sizeof(T))
        *cp = *cp + static_cast<CT>(v);  // fp32 product, fp64 running value
      else
        *cp = (beta == T(0)) ? v : fma(beta, *cp, v);
    }
  }
}

}  // namespace

int sgemm(cudaStream_t s, int64_t M, int64_t N, int64_t K, float alpha, const float* A, int64_t lda,
          const float* B, int64_t ldb, bool transB, float beta, float* C, int64_t ldc, bool upper) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  dim3 grid(static_cast<unsigned>((N + TN - 1) / TN), static_cast<unsigned>((M + TM - 1) / TM));
  if (grid.y > 65535u) return GPTQ_ERR_UNSUPPORTED;
  if (transB)
    gemm_kernel<float, true, float><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, upper ? 1 : 0);
  else
    gemm_kernel<float, false, float><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, upper ? 1 : 0);
  return after_launch();
}

int dgemm(cudaStream_t s, int64_t M, int64_t N, int64_t K, double alpha, const double* A, int64_t lda,
          const double* B, int64_t ldb, bool transB, double beta, double* C, int64_t ldc, bool upper) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  dim3 grid(static_cast<unsigned>((N + TN - 1) / TN), static_cast<unsigned>((M + TM - 1) / TM));
  if (grid.y > 65535u) return GPTQ_ERR_UNSUPPORTED;
  if (transB)
    gemm_kernel<double, true, double><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, upper ? 1 : 0);
  else
    gemm_kernel<double, false, double><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, upper ? 1 : 0);
  return after_launch();
}

int sgemm_acc64(cudaStream_t s, int64_t M, int64_t N, int64_t K, float alpha, const float* A, int64_t lda,
                const float* B, int64_t ldb, double* C, int64_t ldc) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  dim3 grid(static_cast<unsigned>((N + TN - 1) / TN), static_cast<unsigned>((M + TM - 1) / TM));
  if (grid.y > 65535u) return GPTQ_ERR_UNSUPPORTED;
  gemm_kernel<float, false, double><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, 1.f, C, ldc, 0);
  return after_launch();
}

}  // namespace gptq
