// Damped inverse-Cholesky factor of the calibration Hessian.
//
// Source: "第5章 GPTQ 实战" §5.1.8, key points 1-2: damp the Hessian with
// damp_percent * mean(diag H) on the diagonal, then take the Cholesky factor of its
// inverse once; row j of that upper factor U holds the compensation coefficients the
// sweep applies when column j is quantized.  With desc_act the Hessian is first
// permuted so that columns run in order of descending diag(H) (AutoGPTQ examples
// guide §1.4, desc_act).
//
// Route: instead of inverting and then factoring (about 5n^3/3 flops), factor the
// damped Hessian from the bottom-right corner, H_d = V V^T with V upper triangular,
// and invert V: inverse(H_d) = V^-T V^-1, so U = V^-1 is exactly the upper factor
// with inverse(H_d) = U^T U and a positive diagonal (2n^3/3 flops).  Both steps are
// blocked with 64-wide blocks: a single-CTA kernel factors and inverts each diagonal
// block in shared memory (and checks every pivot), and the off-diagonal work runs as
// GEMMs.
//
// Precision: the factorisation runs in fp64 and U stays fp64.  The forward error of a
// Cholesky factor grows like cond(H_d) times the working precision; with cond(H_d) ~ 1e4
// (heavy-tailed activation channels) an fp32 factorisation leaves ~1e-5 relative error
// in U, and a sweep over thousands of columns amplifies even fp32 rounding of U into
// different codes.
#include <algorithm>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int NB = 64;  // block width of the factorisation
constexpr int DIAG_THREADS = 512;
constexpr int SP = NB + 1;  // padded pitch of the diagonal block in shared memory
using real = double;     // working precision of the factorisation

// Sum of diag(H) in double.
__global__ void diag_sum_kernel(const float* __restrict__ H, int64_t n, double* out) {
  double s = 0.0;
  for (int64_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) s += H[i * n + i];
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __shared__ double ws[32];
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? ws[threadIdx.x] : 0.0;
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) atomicAdd(out, s);
  }
}

// desc_act order: rank of column i among all columns by (diag descending, index ascending).
// perm[rank] = i, invperm[i] = rank.
__global__ void act_order_rank_kernel(const float* __restrict__ H, int64_t n, int32_t* perm, int32_t* invperm) {
  __shared__ float dj[256];
  const int64_t i = blockIdx.x * 256 + threadIdx.x;
  const float di = (i < n) ? H[i * n + i] : 0.f;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < n; j0 += 256) {
    const int64_t j = j0 + threadIdx.x;
    dj[threadIdx.x] = (j < n) ? H[j * n + j] : 0.f;
    __syncthreads();
    const int lim = static_cast<int>((n - j0) < 256 ? (n - j0) : 256);
    for (int t = 0; t < lim; ++t) {
      const float d = dj[t];
      const int64_t jj = j0 + t;
      rank += (d > di) || (d == di && jj < i);
    }
    __syncthreads();
  }
  if (i < n) {
    const int64_t r = rank < n - 1 ? rank : n - 1;
    perm[r] = static_cast<int32_t>(i);
    invperm[i] = static_cast<int32_t>(r);
  }
}

// A = P H P^T + lambda I with lambda = damp * mean(diag H) (P = permutation, or none).
__global__ void permute_damp_kernel(const float* __restrict__ H, int64_t n, const int32_t* __restrict__ perm,
                                    const double* __restrict__ diag_sum, float damp, real* __restrict__ A) {
  const int64_t i = blockIdx.y;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t pi = perm ? perm[i] : i;
  const int64_t pj = perm ? perm[j] : j;
  real v = H[pi * n + pj];
  if (i == j) v += static_cast<double>(damp) * (*diag_sum / static_cast<double>(n));
  A[i * n + j] = v;
}

// Factor the diagonal block A[k0:k0+nb, k0:k0+nb] (upper part valid) as V V^T with V upper,
// write V back into A, and its inverse into Winv[k0:k0+nb, 0:nb] (ld NB).  A pivot that is
// not positive and finite sets *status = NOT_PD; the factorisation continues with a unit
// pivot so that every later kernel still sees finite numbers.
//
// The block is padded to NB x NB with an identity in its bottom-right corner (no coupling),
// which leaves the real part of V and V^-1 unchanged and lets every size use the same
// power-of-two inverse below.
__global__ void __launch_bounds__(DIAG_THREADS) chol_diag_kernel(real* A, int64_t lda, int64_t k0, int nb,
                                                                 real* Winv, int* status) {
  extern __shared__ real sm[];
  real* S = sm;              // V, [NB][SP]
  real* X = sm + NB * SP;    // V^-1, [NB][SP]
  real* T = X + NB * SP;     // product scratch, [NB/2][SP]
  real* col = T + (NB / 2) * SP;  // scaled column, [NB]
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int e = tid; e < NB * NB; e += DIAG_THREADS) {
    const int i = e / NB, j = e % NB;
    real v = 0;
    if (i < nb && j < nb) {
      if (i <= j) v = A[(k0 + i) * lda + k0 + j];
    } else if (i == j) {
      v = 1;
    }
    S[i * SP + j] = v;
    X[i * SP + j] = 0;
  }
  // Each thread owns fixed elements (i <= j) of the upper triangle for the rank-1 updates.
  constexpr int NUP = NB * (NB + 1) / 2;
  constexpr int SLOTS = (NUP + DIAG_THREADS - 1) / DIAG_THREADS;
  int own[SLOTS];
#pragma unroll
  for (int r = 0; r < SLOTS; ++r) {
    int e = tid + r * DIAG_THREADS, i = 0;
    if (e < NUP) {
      while (e >= NB - i) {
        e -= NB - i;
        ++i;
      }
      own[r] = (i << 8) | (i + e);
    } else {
      own[r] = -1;
    }
  }
  __syncthreads();
  for (int c = NB - 1; c >= 0; --c) {
    real d = S[c * SP + c];
    if (!(d > 0) || !isfinite(d)) {
      if (tid == 0) bad = 1;
      d = 1;
    }
    const real v = sqrt(d);
    if (tid < c) col[tid] = S[tid * SP + c] / v;
    __syncthreads();
    if (tid == 0) S[c * SP + c] = v;
    if (tid < c) S[tid * SP + c] = col[tid];
#pragma unroll
    for (int r = 0; r < SLOTS; ++r) {
      const int o = own[r];
      const int i = o >> 8, j = o & 255;
      if (o >= 0 && j < c) S[i * SP + j] = fma(-col[i], col[j], S[i * SP + j]);
    }
    __syncthreads();
  }

  // X = V^-1 by doubling: invert 16x16 diagonal blocks, then join neighbours with
  // [[A, B], [0, C]]^-1 = [[A^-1, -A^-1 B C^-1], [0, C^-1]].
  {
    const int warp = tid >> 5, lane = tid & 31;
    if (warp < NB / 16 && lane < 16) {
      const int p = warp * 16, j = p + lane;
      X[j * SP + j] = 1 / S[j * SP + j];
      for (int i = j - 1; i >= p; --i) {
        real acc = 0;
        for (int l = i + 1; l <= j; ++l) acc = fma(S[i * SP + l], X[l * SP + j], acc);
        X[i * SP + j] = -acc / S[i * SP + i];
      }
    }
    __syncthreads();
  }
  for (int sz = 16; sz < NB; sz *= 2) {
    const int pairs = NB / (2 * sz);
    // T = B * C^-1 for every pair (B: rows p..p+sz, cols p+sz..p+2sz of V)
    for (int e = tid; e < pairs * sz * sz; e += DIAG_THREADS) {
      const int pr = e / (sz * sz), r = (e / sz) % sz, cc = e % sz;
      const int p = pr * 2 * sz;
      real acc = 0;
      for (int l = 0; l <= cc; ++l) acc = fma(S[(p + r) * SP + p + sz + l], X[(p + sz + l) * SP + p + sz + cc], acc);
      T[(pr * sz + r) * SP + cc] = acc;
    }
    __syncthreads();
    // X12 = -A^-1 * T
    for (int e = tid; e < pairs * sz * sz; e += DIAG_THREADS) {
      const int pr = e / (sz * sz), r = (e / sz) % sz, cc = e % sz;
      const int p = pr * 2 * sz;
      real acc = 0;
      for (int l = r; l < sz; ++l) acc = fma(X[(p + r) * SP + p + l], T[(pr * sz + l) * SP + cc], acc);
      X[(p + r) * SP + p + sz + cc] = -acc;
    }
    __syncthreads();
  }

  for (int e = tid; e < nb * nb; e += DIAG_THREADS) {
    const int i = e / nb, j = e % nb;
    if (i <= j) A[(k0 + i) * lda + k0 + j] = S[i * SP + j];
    Winv[(k0 + i) * NB + j] = X[i * SP + j];
  }
  if (tid == 0 && bad) atomicExch(status, kStatusNotPD);
}

__global__ void set_diag_kernel(real* R, int64_t n, real v) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) R[i * n + i] = v;
}

constexpr int DIAG_SMEM = (2 * NB * SP + (NB / 2) * SP + NB) * static_cast<int>(sizeof(real));

}  // namespace

size_t factor_small_bytes(int64_t n) {
  return static_cast<size_t>(n) * NB * sizeof(real) + 256;
}

size_t factor_work_bytes(int64_t n) { return static_cast<size_t>(n) * n * sizeof(real); }

int factor_hessian(const float* H, int64_t n, float damp, bool desc_act, double* U, int32_t* perm,
                   int32_t* invperm, void* work, void* small, int* status, cudaStream_t s) {
  static cudaError_t attr = cudaFuncSetAttribute(chol_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 DIAG_SMEM);
  if (attr != cudaSuccess) return GPTQ_ERR_CUDA;
  double* dsum = reinterpret_cast<double*>(small);
  real* Winv = reinterpret_cast<real*>(static_cast<char*>(small) + 256);
  real* A = static_cast<real*>(work);   // damped Hessian, then V
  real* R = U;                          // V^-1, written in place into the output

  GPTQ_CUDA(cudaMemsetAsync(dsum, 0, sizeof(double), s));
  diag_sum_kernel<<<std::min<int64_t>((n + 255) / 256, 148), 256, 0, s>>>(H, n, dsum);
  GPTQ_TRY(after_launch());
  if (desc_act) {
    act_order_rank_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(H, n, perm, invperm);
    GPTQ_TRY(after_launch());
  }
  const dim3 rgrid(static_cast<unsigned>((n + 255) / 256), static_cast<unsigned>(n));
  permute_damp_kernel<<<rgrid, 256, 0, s>>>(H, n, desc_act ? perm : nullptr, dsum, damp, A);
  GPTQ_TRY(after_launch());

  // Reverse (bottom-right first) blocked Cholesky: A -> V (upper), H_d = V V^T.
  const int64_t nblk = (n + NB - 1) / NB;
  for (int64_t k = nblk - 1; k >= 0; --k) {
    const int64_t k0 = k * NB;
    const int nb = static_cast<int>(std::min<int64_t>(NB, n - k0));
    chol_diag_kernel<<<1, DIAG_THREADS, DIAG_SMEM, s>>>(A, n, k0, nb, Winv, status);
    GPTQ_TRY(after_launch());
    if (k0 > 0) {
      // Panel: V[0:k0, k] = A[0:k0, k] * V_kk^-T   (in place; N = nb <= 128)
      GPTQ_TRY(dgemm(s, k0, nb, nb, 1.0, A + k0, n, Winv + k0 * NB, NB, true, 0.0, A + k0, n, false));
      // Trailing: A[0:k0, 0:k0] -= V[0:k0, k] V[0:k0, k]^T   (upper tiles only)
      GPTQ_TRY(dgemm(s, k0, k0, nb, -1.0, A + k0, n, A + k0, n, true, 1.0, A, n, true));
    }
  }

  // R = V^-1 by block back substitution on the identity, bottom block row first.
  GPTQ_CUDA(cudaMemsetAsync(R, 0, static_cast<size_t>(n) * n * sizeof(real), s));
  set_diag_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(R, n, 1.0);
  GPTQ_TRY(after_launch());
  for (int64_t k = nblk - 1; k >= 0; --k) {
    const int64_t k0 = k * NB;
    const int nb = static_cast<int>(std::min<int64_t>(NB, n - k0));
    // R[k, k0:] = V_kk^-1 * R[k, k0:]   (in place; M = nb <= 128)
    GPTQ_TRY(dgemm(s, nb, n - k0, nb, 1.0, Winv + k0 * NB, NB, R + k0 * n + k0, n, false, 0.0, R + k0 * n + k0, n,
                   false));
    if (k0 > 0) {
      // R[0:k0, k0:] -= V[0:k0, k] * R[k, k0:]
      GPTQ_TRY(dgemm(s, k0, n - k0, nb, -1.0, A + k0, n, R + k0 * n + k0, n, false, 1.0, R + k0, n, false));
    }
  }
  return GPTQ_OK;
}

}  // namespace gptq
