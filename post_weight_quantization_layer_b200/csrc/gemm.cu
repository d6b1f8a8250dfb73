// fp64 GEMMs of the factorisation (its rank-k updates) and of the sweep (its lazy block
// updates): C = beta*C + alpha * A * op(B).
//
// Two kernels.  dgemm_mma_kernel (below) runs on the fp64 matrix units and takes every
// call whose operands are 16-byte aligned with even leading dimensions, K and N.
// gemm_kernel is the CUDA-core fallback for the rest: 128x128 tile per 256-thread CTA,
// 8x8 outputs per thread, K staged 8 at a time through double-buffered shared memory,
// every global access bounds-checked, so ragged edges need no padding.
#include "common.cuh"

namespace gptq {
namespace {

constexpr int TM = 128, TN = 128, TK = 8, PAD = 4;

template <typename T, bool TRANSB, typename CT>
__global__ void __launch_bounds__(256) gemm_kernel(int64_t M, int64_t N, int64_t K, T alpha, const T* A,
                                                   int64_t lda, const T* B, int64_t ldb, T beta, CT* C,
                                                   int64_t ldc, int upper, int tri) {
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * TM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * TN;
  if (upper && n0 + TN - 1 < m0) return;
  // Triangular operands hold exact zeros outside their triangle; skipping those K ranges
  // leaves every sum unchanged.
  int64_t kbeg = 0, kend = K;
  if (tri & kTriAUpper) kbeg = max(kbeg, m0);            // A(m,k) = 0 for k < m
  if (tri & kTriBUpper) kend = min(kend, n0 + TN);       // B(k,n) = 0 for k > n
  if (tri & kTriBTUpper) kbeg = max(kbeg, n0);           // B(k,n) = 0 for k < n
  kbeg = (kbeg / TK) * TK;

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

  const int64_t nkt = kend > kbeg ? (kend - kbeg + TK - 1) / TK : 0;
  int buf = 0;
  if (nkt > 0) {
    load_regs(kbeg);
    store_smem(0);
  }
  __syncthreads();
  for (int64_t kt = 0; kt < nkt; ++kt) {
    if (kt + 1 < nkt) load_regs(kbeg + (kt + 1) * TK);
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


// ---------------------------------------------------------------------------------------
// fp64 GEMM on the fp64 matrix units (mma.sync m8n8k4; tcgen05 has no fp64 form).
// CTA tile 128x128, K staged 16 at a time through a 3-stage cp.async ring; 8 warps as
// 2 (M) x 4 (N), warp tile 64x32 = 8x4 m8n8 accumulators.  Shared-memory rows are padded
// (20 / 132 doubles) so that every fragment load of a half-warp hits 16 distinct 8-byte
// bank pairs.  Requirements (else the CUDA-core kernel above is used): 16-byte aligned
// operands, even leading dimensions, even K and N.
constexpr int DK = 16, DST = 3;
constexpr int DAP = DK + 4;    // pitch of [row][k] tiles (A, and B when transposed)
template <int BM, int BN>
struct DTile {
  static constexpr int BP = BN + 4;  // pitch of the [k][n] tile (B not transposed)
  static constexpr int A_STAGE = BM * DAP;
  static constexpr int B_STAGE = BN * DAP > DK * BP ? BN * DAP : DK * BP;
  static constexpr int SMEM = DST * (A_STAGE + B_STAGE) * static_cast<int>(sizeof(double));
  static constexpr int WM = BM / 2, WN = BN / 4;  // warp tile (8 warps as 2 x 4)
  static constexpr int MI = WM / 8, NJ = WN / 8;  // m8n8 blocks per warp
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int bytes = pred ? 16 : 0;  // 0: zero-fill, nothing read
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void dmma(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// At most 192 registers a thread (256 threads a CTA): one 128x128 CTA then leaves room on
// its SM for one CTA of the sweep's panel kernel, which runs beside the trailing update.
template <bool TRANSB, int BM, int BN>
__global__ void __maxnreg__(192) dgemm_mma_kernel(int64_t M, int64_t N, int64_t K, double alpha,
                                                           const double* A, int64_t lda, const double* B,
                                                           int64_t ldb, double beta, double* C, int64_t ldc,
                                                           int upper, int tri) {
  using TL = DTile<BM, BN>;
  constexpr int DA_STAGE = TL::A_STAGE, DB_STAGE = TL::B_STAGE, DBP = TL::BP;
  extern __shared__ __align__(16) double dsm[];
  double* As = dsm;
  double* Bs = dsm + DST * DA_STAGE;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  if (upper && n0 + BN - 1 < m0) return;
  int64_t kbeg = 0, kend = K;
  if (tri & kTriAUpper) kbeg = max(kbeg, m0);
  if (tri & kTriBUpper) kend = min(kend, n0 + BN);
  if (tri & kTriBTUpper) kbeg = max(kbeg, n0);
  kbeg = (kbeg / DK) * DK;
  const int64_t nkt = kend > kbeg ? (kend - kbeg + DK - 1) / DK : 0;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp >> 2, wn = warp & 3;
  const int g = lane >> 2, t = lane & 3;

  auto load_stage = [&](int st, int64_t kt) {
    const int64_t k0 = kbeg + kt * DK;
    double* as = As + st * DA_STAGE;
    double* bs = Bs + st * DB_STAGE;
#pragma unroll
    for (int i = 0; i < BM * DK / 2 / 256; ++i) {  // 16-byte chunks of the A tile
      const int c = tid + 256 * i;
      const int row = c >> 3, col = (c & 7) * 2;
      const int64_t gm = m0 + row, gk = k0 + col;
      const bool ok = gm < M && gk < kend;
      cp_async16(as + row * DAP + col, ok ? A + gm * lda + gk : A, ok);
    }
#pragma unroll
    for (int i = 0; i < BN * DK / 2 / 256; ++i) {  // 16-byte chunks of the B tile
      const int c = tid + 256 * i;
      if (TRANSB) {
        const int row = c >> 3, col = (c & 7) * 2;
        const int64_t gn = n0 + row, gk = k0 + col;
        const bool ok = gn < N && gk < kend;
        cp_async16(bs + row * DAP + col, ok ? B + gn * ldb + gk : B, ok);
      } else {
        const int row = c / (BN / 2), col = (c % (BN / 2)) * 2;
        const int64_t gk = k0 + row, gn = n0 + col;
        const bool ok = gk < kend && gn < N;
        cp_async16(bs + row * DBP + col, ok ? B + gk * ldb + gn : B, ok);
      }
    }
  };

  constexpr int MI = TL::MI, NJ = TL::NJ, WM = TL::WM, WN = TL::WN;
  double acc[MI][NJ][2];
#pragma unroll
  for (int i = 0; i < MI; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

#pragma unroll
  for (int st = 0; st < DST - 1; ++st) {
    if (st < nkt) load_stage(st, st);
    cp_async_commit();
  }
  for (int64_t kt = 0; kt < nkt; ++kt) {
    cp_async_wait<DST - 2>();
    __syncthreads();
    if (kt + DST - 1 < nkt) load_stage(static_cast<int>((kt + DST - 1) % DST), kt + DST - 1);
    cp_async_commit();
    const int st = static_cast<int>(kt % DST);
    const double* as = As + st * DA_STAGE;
    const double* bs = Bs + st * DB_STAGE;
#pragma unroll
    for (int kk = 0; kk < DK / 4; ++kk) {
      double a[MI], b[NJ];
#pragma unroll
      for (int i = 0; i < MI; ++i) a[i] = as[(wm * WM + i * 8 + g) * DAP + kk * 4 + t];
#pragma unroll
      for (int j = 0; j < NJ; ++j)
        b[j] = TRANSB ? bs[(wn * WN + j * 8 + g) * DAP + kk * 4 + t] : bs[(kk * 4 + t) * DBP + wn * WN + j * 8 + g];
#pragma unroll
      for (int i = 0; i < MI; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) dmma(acc[i][j], a[i], b[j]);
    }
  }
  cp_async_wait<0>();

  // Epilogue.  Each thread holds element pairs (gn, gn + 1) with gn even; N is even, so a
  // pair is either wholly inside C or wholly outside, and 16-byte aligned.
  // beta == 1 (the accumulating updates): fire-and-forget fp64 reductions, so the CTA does
  // not wait on the latency of reading C; only this CTA writes these elements during the
  // launch, so each one receives exactly one correctly rounded addition C + v.
#pragma unroll
  for (int i = 0; i < MI; ++i) {
    const int64_t gm = m0 + wm * WM + i * 8 + g;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int64_t gn = n0 + wn * WN + j * 8 + 2 * t;
      if (gn >= N) continue;
      double* cp = C + gm * ldc + gn;
      const double v0 = alpha * acc[i][j][0], v1 = alpha * acc[i][j][1];
      if (beta == 1.0) {
        atomicAdd(cp, v0);
        atomicAdd(cp + 1, v1);
      } else if (beta == 0.0) {
        *reinterpret_cast<double2*>(cp) = make_double2(v0, v1);
      } else {
        const double2 c = *reinterpret_cast<const double2*>(cp);
        *reinterpret_cast<double2*>(cp) = make_double2(fma(beta, c.x, v0), fma(beta, c.y, v1));
      }
    }
  }
}

}  // namespace

int dgemm(cudaStream_t s, int64_t M, int64_t N, int64_t K, double alpha, const double* A, int64_t lda,
          const double* B, int64_t ldb, bool transB, double beta, double* C, int64_t ldc, bool upper, int tri) {
  if (M <= 0 || N <= 0) return GPTQ_OK;
  dim3 grid(static_cast<unsigned>((N + TN - 1) / TN), static_cast<unsigned>((M + TM - 1) / TM));
  if (grid.y > 65535u) return GPTQ_ERR_UNSUPPORTED;
  const bool mma_ok = aligned16(A) && aligned16(B) && aligned16(C) && lda % 2 == 0 && ldb % 2 == 0 && ldc % 2 == 0 &&
                      K % 2 == 0 && N % 2 == 0;
  if (mma_ok) {
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(dgemm_mma_kernel<true, 128, 128>), DTile<128, 128>::SMEM));
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(dgemm_mma_kernel<false, 128, 128>), DTile<128, 128>::SMEM));
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(dgemm_mma_kernel<true, 64, 64>), DTile<64, 64>::SMEM));
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(dgemm_mma_kernel<false, 64, 64>), DTile<64, 64>::SMEM));
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(dgemm_mma_kernel<true, 32, 32>), DTile<32, 32>::SMEM));
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(dgemm_mma_kernel<false, 32, 32>), DTile<32, 32>::SMEM));
    // Small products: 64x64 (or 32x32) tiles spread the work over 4x (16x) more SMs.
    const int64_t big_tiles = ((M + 127) / 128) * ((N + 127) / 128);
    const int64_t mid_tiles = ((M + 63) / 64) * ((N + 63) / 64);
    const bool small = big_tiles < 2 * num_sms();
    const bool tiny = mid_tiles < num_sms();
    const int u = upper ? 1 : 0;
    if (tiny) {
      dim3 g32(static_cast<unsigned>((N + 31) / 32), static_cast<unsigned>((M + 31) / 32));
      if (g32.y > 65535u) return GPTQ_ERR_UNSUPPORTED;
      if (transB)
        dgemm_mma_kernel<true, 32, 32><<<g32, 256, DTile<32, 32>::SMEM, s>>>(M, N, K, alpha, A, lda, B, ldb, beta,
                                                                            C, ldc, u, tri);
      else
        dgemm_mma_kernel<false, 32, 32><<<g32, 256, DTile<32, 32>::SMEM, s>>>(M, N, K, alpha, A, lda, B, ldb, beta,
                                                                             C, ldc, u, tri);
    } else if (small) {
      dim3 g64(static_cast<unsigned>((N + 63) / 64), static_cast<unsigned>((M + 63) / 64));
      if (g64.y > 65535u) return GPTQ_ERR_UNSUPPORTED;
      if (transB)
        dgemm_mma_kernel<true, 64, 64><<<g64, 256, DTile<64, 64>::SMEM, s>>>(M, N, K, alpha, A, lda, B, ldb, beta,
                                                                            C, ldc, u, tri);
      else
        dgemm_mma_kernel<false, 64, 64><<<g64, 256, DTile<64, 64>::SMEM, s>>>(M, N, K, alpha, A, lda, B, ldb, beta,
                                                                             C, ldc, u, tri);
    } else if (transB) {
      dgemm_mma_kernel<true, 128, 128><<<grid, 256, DTile<128, 128>::SMEM, s>>>(M, N, K, alpha, A, lda, B, ldb,
                                                                                beta, C, ldc, u, tri);
    } else {
      dgemm_mma_kernel<false, 128, 128><<<grid, 256, DTile<128, 128>::SMEM, s>>>(M, N, K, alpha, A, lda, B, ldb,
                                                                                 beta, C, ldc, u, tri);
    }
    return after_launch();
  }
  if (transB)
    gemm_kernel<double, true, double><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, upper ? 1 : 0,
                                                           tri);
  else
    gemm_kernel<double, false, double><<<grid, 256, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc,
                                                            upper ? 1 : 0, tri);
  return after_launch();
}


}  // namespace gptq
