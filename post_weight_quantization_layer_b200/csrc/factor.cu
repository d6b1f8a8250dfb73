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
// blocked with 128-wide blocks: a single-CTA kernel factors and inverts each diagonal
// block in shared memory (and checks every pivot), and the off-diagonal work runs as
// GEMMs.
#include <algorithm>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int NB = 128;  // block width of the factorisation
constexpr int DIAG_THREADS = 512;
constexpr int SP = NB + 1;  // padded pitch of the diagonal block in shared memory

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
                                    const double* __restrict__ diag_sum, float damp, float* __restrict__ A) {
  const int64_t i = blockIdx.y;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t pi = perm ? perm[i] : i;
  const int64_t pj = perm ? perm[j] : j;
  float v = H[pi * n + pj];
  if (i == j) v += static_cast<float>(static_cast<double>(damp) * (*diag_sum / static_cast<double>(n)));
  A[i * n + j] = v;
}

// Factor the diagonal block A[k0:k0+nb, k0:k0+nb] (upper part valid) as V V^T with V upper,
// write V back into A, and its inverse into Winv[k0:k0+nb, 0:nb] (ld NB).  A pivot that is
// not positive and finite sets *status = NOT_PD; the factorisation continues with a unit
// pivot so that every later kernel still sees finite numbers.
__global__ void __launch_bounds__(DIAG_THREADS) chol_diag_kernel(float* A, int64_t lda, int64_t k0, int nb,
                                                                 float* Winv, int* status) {
  extern __shared__ float sm[];
  float* S = sm;              // V, [NB][SP]
  float* X = sm + NB * SP;    // V^-1, [NB][SP]
  float* col = X + NB * SP;   // scaled column, [NB]
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  for (int e = tid; e < nb * nb; e += DIAG_THREADS) {
    const int i = e / nb, j = e % nb;
    S[i * SP + j] = (i <= j) ? A[(k0 + i) * lda + k0 + j] : 0.f;
  }
  __syncthreads();
  for (int c = nb - 1; c >= 0; --c) {
    float d = S[c * SP + c];
    if (!(d > 0.f) || !isfinite(d)) {
      if (tid == 0) bad = 1;
      d = 1.f;
    }
    const float v = sqrtf(d);
    if (tid < c) col[tid] = S[tid * SP + c] / v;
    __syncthreads();
    if (tid == 0) S[c * SP + c] = v;
    if (tid < c) S[tid * SP + c] = col[tid];
    const int cc = c * c;
    for (int e = tid; e < cc; e += DIAG_THREADS) {
      const int i = e / c, j = e - i * c;
      if (i <= j) S[i * SP + j] = fmaf(-col[i], col[j], S[i * SP + j]);
    }
    __syncthreads();
  }
  // X = V^-1 (upper): thread j solves column j by back substitution.
  if (tid < nb) {
    const int j = tid;
    X[j * SP + j] = 1.f / S[j * SP + j];
    for (int i = j - 1; i >= 0; --i) {
      float s0 = 0.f, s1 = 0.f;
      int l = i + 1;
      for (; l + 1 <= j; l += 2) {
        s0 = fmaf(S[i * SP + l], X[l * SP + j], s0);
        s1 = fmaf(S[i * SP + l + 1], X[(l + 1) * SP + j], s1);
      }
      if (l <= j) s0 = fmaf(S[i * SP + l], X[l * SP + j], s0);
      X[i * SP + j] = -(s0 + s1) / S[i * SP + i];
    }
    for (int i = j + 1; i < nb; ++i) X[i * SP + j] = 0.f;
  }
  __syncthreads();
  for (int e = tid; e < nb * nb; e += DIAG_THREADS) {
    const int i = e / nb, j = e % nb;
    if (i <= j) A[(k0 + i) * lda + k0 + j] = S[i * SP + j];
    Winv[(k0 + i) * NB + j] = X[i * SP + j];
  }
  if (tid == 0 && bad) atomicExch(status, kStatusNotPD);
}

__global__ void set_diag_kernel(float* R, int64_t n, float v) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) R[i * n + i] = v;
}

constexpr int DIAG_SMEM = (2 * NB * SP + NB) * static_cast<int>(sizeof(float));

}  // namespace

size_t factor_small_bytes(int64_t n) {
  return static_cast<size_t>(n) * NB * sizeof(float) + 256;
}

int factor_hessian(const float* H, int64_t n, float damp, bool desc_act, float* U, int32_t* perm,
                   int32_t* invperm, float* work, void* small, int* status, cudaStream_t s) {
  static cudaError_t attr = cudaFuncSetAttribute(chol_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 DIAG_SMEM);
  if (attr != cudaSuccess) return GPTQ_ERR_CUDA;
  double* dsum = reinterpret_cast<double*>(small);
  float* Winv = reinterpret_cast<float*>(static_cast<char*>(small) + 256);
  float* A = work;

  GPTQ_CUDA(cudaMemsetAsync(dsum, 0, sizeof(double), s));
  diag_sum_kernel<<<std::min<int64_t>((n + 255) / 256, 148), 256, 0, s>>>(H, n, dsum);
  GPTQ_TRY(after_launch());
  if (desc_act) {
    act_order_rank_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(H, n, perm, invperm);
    GPTQ_TRY(after_launch());
  }
  {
    dim3 grid(static_cast<unsigned>((n + 255) / 256), static_cast<unsigned>(n));
    permute_damp_kernel<<<grid, 256, 0, s>>>(H, n, desc_act ? perm : nullptr, dsum, damp, A);
    GPTQ_TRY(after_launch());
  }

  // Reverse (bottom-right first) blocked Cholesky: A -> V (upper), H_d = V V^T.
  const int64_t nblk = (n + NB - 1) / NB;
  for (int64_t k = nblk - 1; k >= 0; --k) {
    const int64_t k0 = k * NB;
    const int nb = static_cast<int>(std::min<int64_t>(NB, n - k0));
    chol_diag_kernel<<<1, DIAG_THREADS, DIAG_SMEM, s>>>(A, n, k0, nb, Winv, status);
    GPTQ_TRY(after_launch());
    if (k0 > 0) {
      // Panel: V[0:k0, k] = A[0:k0, k] * V_kk^-T   (in place; N = nb <= 128)
      GPTQ_TRY(sgemm(s, k0, nb, nb, 1.f, A + k0, n, Winv + k0 * NB, NB, true, 0.f, A + k0, n, false));
      // Trailing: A[0:k0, 0:k0] -= V[0:k0, k] V[0:k0, k]^T   (upper tiles only)
      GPTQ_TRY(sgemm(s, k0, k0, nb, -1.f, A + k0, n, A + k0, n, true, 1.f, A, n, true));
    }
  }

  // U = V^-1 by block back substitution on the identity, bottom block row first.
  GPTQ_CUDA(cudaMemsetAsync(U, 0, static_cast<size_t>(n) * n * sizeof(float), s));
  set_diag_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(U, n, 1.f);
  GPTQ_TRY(after_launch());
  for (int64_t k = nblk - 1; k >= 0; --k) {
    const int64_t k0 = k * NB;
    const int nb = static_cast<int>(std::min<int64_t>(NB, n - k0));
    // U[k, k0:] = V_kk^-1 * R[k, k0:]   (in place; M = nb <= 128)
    GPTQ_TRY(sgemm(s, nb, n - k0, nb, 1.f, Winv + k0 * NB, NB, U + k0 * n + k0, n, false, 0.f, U + k0 * n + k0, n,
                   false));
    if (k0 > 0) {
      // R[0:k0, k0:] -= V[0:k0, k] * U[k, k0:]
      GPTQ_TRY(sgemm(s, k0, n - k0, nb, -1.f, A + k0, n, U + k0 * n + k0, n, false, 1.f, U + k0, n, false));
    }
  }
  return GPTQ_OK;
}

}  // namespace gptq
