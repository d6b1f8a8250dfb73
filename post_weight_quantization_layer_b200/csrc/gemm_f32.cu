// FP32 GEMM on the CUDA cores, used for the rank-k updates of the factorisation and the
// lazy block updates of the sweep: C = beta*C + alpha * A * op(B).
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

template <bool TRANSB>
__global__ void __launch_bounds__(256) sgemm_kernel(int64_t M, int64_t N, int64_t K, float alpha,
                                                    const float* A, int64_t lda,
                                                    const float* B, int64_t ldb, float beta,
                                                    float* C, int64_t ldc, int upper) {
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * TM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * TN;
  if (upper && n0 + TN - 1 < m0) return;

  __shared__ __align__(16) float As[2][TK][TM + PAD];
  __shared__ __align__(16) float Bs[2][TK][TN + PAD];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  float ra[4], rb[4];
  auto load_regs = [&](int64_t k0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = tid + 256 * i;
      const int am = e >> 3, ak = e & 7;
      const int64_t gm = m0 + am, gk = k0 + ak;
      ra[i] = (gm < M && gk < K) ? A[gm * lda + gk] : 0.f;
      if (TRANSB) {
        const int bn = e >> 3, bk = e & 7;
        const int64_t gn = n0 + bn, gk2 = k0 + bk;
        rb[i] = (gn < N && gk2 < K) ? B[gn * ldb + gk2] : 0.f;
      } else {
        const int bk = e >> 7, bn = e & 127;
        const int64_t gn = n0 + bn, gk2 = k0 + bk;
        rb[i] = (gn < N && gk2 < K) ? B[gk2 * ldb + gn] : 0.f;
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

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

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
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][k][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
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
      float* cp = C + gm * ldc + gn;
      const float v = alpha * acc[i][j];
      *cp = (beta == 0.f) ? v : fmaf(beta, *cp, v);
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
    sgemm_kernel<true><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, upper ? 1 : 0);
  else
    sgemm_kernel<false><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, upper ? 1 : 0);
  return after_launch();
}

}  // namespace gptq
