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
// with inverse(H_d) = U^T U and a positive diagonal (2n^3/3 flops).
//
// Both are done together, recursively.  Split H_d = [[A, B], [B^T, C]] with the larger,
// NB-aligned part C at the bottom right.  Then, with C = V22 V22^T and U22 = V22^-1:
//   P   = B U22^T              (the off-diagonal block V12 of V)
//   A' := A - P P^T            (Schur complement; upper triangle only)
//   T   = P U22
//   U11 = factor-and-invert(A'),  U12 = -U11 T,
// since V^-1 = [[V11^-1, -V11^-1 V12 V22^-1], [0, V22^-1]].  Blocks of at most NB = 128 are
// factored and inverted by one CTA in shared memory (which also checks every pivot);
// everything else is four large products per level: on the fp64 matrix units for nodes whose
// right part is narrower than 1024, on the int8 tensor cores (seven-slice operands, exact
// integer slice products, ozaki.cu) above.  V itself is never stored.
//
// Precision: the factorisation runs in fp64 (the int8 route carries 49 bits of every operand
// and adds exact integer products) and U stays fp64.  The forward error of a Cholesky factor
// grows like cond(H_d) times the working precision; with cond(H_d) ~ 1e4 (heavy-tailed
// activation channels) an fp32 factorisation leaves ~1e-5 relative error in U, and a sweep
// over thousands of columns amplifies even fp32 rounding of U into different codes.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "factor_plan.h"

namespace gptq {
namespace {

using fplan::NB;  // leaf block width of the factorisation
using fplan::node_i8;
using fplan::pad64;
using fplan::Plan;
using fplan::right_part;
constexpr int DIAG_THREADS = 512;
constexpr int SP = NB + 4;      // pitch of the diagonal block in shared memory (fragment loads
constexpr int TP = NB / 2 + 4;  // of m8n8k4 hit 16 distinct bank pairs when pitch = 4 mod 16)
using real = double;     // working precision of the factorisation

// Sum of diag(H) in double, by one CTA of DSUM_THREADS threads in a fixed order (no
// atomics), so that the damping term, and with it the whole factor, is the same bit for
// bit on every call.  At most 65,535 / 1,024 = 64 strided loads a thread.
constexpr int DSUM_THREADS = 1024;
__global__ void __launch_bounds__(DSUM_THREADS) diag_sum_kernel(const float* __restrict__ H, int64_t n, double* out) {
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += DSUM_THREADS) s += H[i * n + i];
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __shared__ double ws[DSUM_THREADS / 32];
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = ws[threadIdx.x];
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) *out = s;
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

// D = sign * A * B for shared-memory blocks (M, N multiples of 8, K of 4), all warps of the
// CTA sharing the m8n8 output tiles, on the fp64 matrix units.  tri & 1: A is upper
// triangular (A[m][k] == 0 for k < m); tri & 2: B is upper triangular (B[k][n] == 0 for
// k > n); those K ranges hold exact zeros and are skipped.
__device__ __forceinline__ void cta_dmma(real* D, int ldd, const real* A, int lda, const real* B, int ldb, int M, int N,
                                         int K, int tri, real sign) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int tn = N / 8;
  for (int tt = warp; tt < (M / 8) * tn; tt += DIAG_THREADS / 32) {
    const int m0 = (tt / tn) * 8, n0 = (tt % tn) * 8;
    int kb = 0, ke = K;
    if (tri & 1) kb = m0;
    if (tri & 2) ke = min(K, n0 + 8);
    kb &= ~3;
    real c0 = 0, c1 = 0;
    for (int k = kb; k < ke; k += 4) {
      const real a0 = A[(m0 + g) * lda + k + t];
      const real b0 = B[(k + t) * ldb + n0 + g];
      asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                   : "+d"(c0), "+d"(c1)
                   : "d"(a0), "d"(b0));
    }
    D[(m0 + g) * ldd + n0 + 2 * t] = sign * c0;
    D[(m0 + g) * ldd + n0 + 2 * t + 1] = sign * c1;
  }
}

// Factor the diagonal block A[k0:k0+nb, k0:k0+nb] (upper part valid) as V V^T with V upper
// and write its inverse into R[k0:k0+nb, k0:k0+nb] (same leading dimension, zeros below the
// diagonal).  A pivot that is not positive and finite sets *status = NOT_PD; the
// factorisation continues with a unit pivot so that every later kernel still sees finite
// numbers.
//
// The block is padded to NB x NB with an identity in its bottom-right corner (no coupling),
// which leaves the real part of V and V^-1 unchanged and lets every size use the same
// power-of-two inverse below.  Everything happens in place in shared memory: S holds the
// block, then V, then V^-1.
__global__ void __launch_bounds__(DIAG_THREADS) chol_diag_kernel(const real* A, int64_t lda, int64_t k0, int nb,
                                                                 real* R, int* status) {
  extern __shared__ real sm[];
  real* S = sm;                         // [NB][SP]
  real* T = S + NB * SP;                // [NB/2][TP] product scratch
  real* col = T + (NB / 2) * TP;        // [NB] scaled column
  real* rdiag = col + NB;               // [NB] 1 / V[j][j]
  real* blk = rdiag + NB;               // [NB/16][16][17] copies of the 16x16 diagonal blocks
  __shared__ int bad;
  // Published 8-column panels of V, double-buffered; row i of a panel column lives at
  // q(i) = i + i/4 so that the 32 lanes of a warp (4 rows each) read it without bank
  // conflicts.
  constexpr int QN = NB + NB / 4;
  __shared__ real pbuf[2][8][QN];
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  // Register blocking: warp w holds columns 8w..8w+7 and lane l rows 4l..4l+3 of the block.
  const int lane = tid & 31, wcol = tid >> 5;
  const int i0 = lane * 4, j0 = wcol * 8;
  const unsigned FULLM = 0xffffffffu;
  real r[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int i = i0 + a, j = j0 + b;
      real v = 0;
      if (i <= j) {
        if (j < nb)
          v = A[(k0 + i) * lda + k0 + j];
        else if (i == j)
          v = 1;
      }
      r[a][b] = v;
    }
  __syncthreads();  // `bad` is initialised before any owner may set it
  // Blocked reverse Cholesky over 8-column panels, right to left.  The warp owning panel p
  // factors it alone with warp shuffles (column c: V[c][c] = sqrt(S[c][c]),
  // V[i][c] = S[i][c] / V[c][c], then the panel's earlier columns get the rank-1 update),
  // publishes it, and every warp holding earlier columns applies the rank-8 update
  // S[i][j] -= sum_k V[i][8p+k] V[j][8p+k].  One barrier per panel; while the next owner
  // factors, the other warps are still applying the previous update.  Elements below the
  // diagonal are updated too (never read, zeroed at the end).
  for (int p = NB / 8 - 1; p >= 0; --p) {
    real(*pb)[QN] = pbuf[p & 1];
    if (wcol == p) {
#pragma unroll
      for (int bc = 7; bc >= 0; --bc) {
        const int c = 8 * p + bc;
        const int src = 2 * p + (bc >> 2);  // lane holding row c (and row 8p+b for b>>2 == bc>>2)
        real d = __shfl_sync(FULLM, r[bc & 3][bc], src);
        if (!(d > 0) || !isfinite(d)) {
          if (lane == src) bad = 1;
          d = 1;
        }
        const real v = sqrt(d);
        const real rv = 1 / v;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const int i = i0 + a;
          if (i < c) r[a][bc] *= rv;
          if (i == c) r[a][bc] = v;
        }
        if (lane == src) rdiag[c] = rv;
#pragma unroll
        for (int b = 0; b < bc; ++b) {
          const real vb = __shfl_sync(FULLM, r[b & 3][bc], 2 * p + (b >> 2));  // V[8p+b][c]
#pragma unroll
          for (int a = 0; a < 4; ++a) r[a][b] = fma(-r[a][bc], vb, r[a][b]);
        }
      }
#pragma unroll
      for (int b = 0; b < 8; ++b)
#pragma unroll
        for (int a = 0; a < 4; ++a) pb[b][(i0 + a) + lane] = r[a][b];  // q(i0+a) = i0 + a + lane
    }
    __syncthreads();
    if (wcol < p) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        real vi[4], vj[8];
#pragma unroll
        for (int a = 0; a < 4; ++a) vi[a] = pb[k][(i0 + a) + lane];
#pragma unroll
        for (int b = 0; b < 8; ++b) vj[b] = pb[k][(j0 + b) + ((j0 + b) >> 2)];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 8; ++b) r[a][b] = fma(-vi[a], vj[b], r[a][b]);
      }
    }
  }
  // V to shared memory for the inverse (zero below the diagonal)
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) S[(i0 + a) * SP + j0 + b] = (i0 + a <= j0 + b) ? r[a][b] : real(0);
  __syncthreads();

  // V^-1 in place by doubling: invert the 16x16 diagonal blocks, then join neighbours with
  // [[A, B], [0, C]]^-1 = [[A^-1, -A^-1 B C^-1], [0, C^-1]].
  {
    const int warp = tid >> 5, lane = tid & 31;
    if (warp < NB / 16) {
      const int p = warp * 16;
      real* b = blk + warp * 16 * 17;
      for (int e = lane; e < 256; e += 32) b[(e >> 4) * 17 + (e & 15)] = S[(p + (e >> 4)) * SP + p + (e & 15)];
      __syncwarp();
      if (lane < 16) {
        const int j = lane;
        real x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = (i == j) ? rdiag[p + i] : real(0);
#pragma unroll
        for (int i = 15; i >= 0; --i) {
          if (i < j) {
            real acc = 0;
#pragma unroll
            for (int l = i + 1; l < 16; ++l)
              if (l <= j) acc = fma(b[i * 17 + l], x[l], acc);
            x[i] = -acc * rdiag[p + i];
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) S[(p + i) * SP + p + j] = x[i];
      }
    }
    __syncthreads();
  }
  for (int sz = 16; sz < NB; sz *= 2) {
    const int pairs = NB / (2 * sz);
    // T = B * C^-1 for every pair (B: rows p..p+sz, cols p+sz..p+2sz, still V there)
    for (int pr = 0; pr < pairs; ++pr) {
      const int p = pr * 2 * sz;
      cta_dmma(T + pr * sz * TP, TP, S + p * SP + p + sz, SP, S + (p + sz) * SP + p + sz, SP, sz, sz, sz, 2, 1);
    }
    __syncthreads();
    // X12 = -A^-1 * T, written over B
    for (int pr = 0; pr < pairs; ++pr) {
      const int p = pr * 2 * sz;
      cta_dmma(S + p * SP + p + sz, SP, S + p * SP + p, SP, T + pr * sz * TP, TP, sz, sz, sz, 1, -1);
    }
    __syncthreads();
  }

  for (int e = tid; e < nb * nb; e += DIAG_THREADS) {
    const int i = e / nb, j = e % nb;
    R[(k0 + i) * lda + k0 + j] = (i <= j) ? S[i * SP + j] : real(0);
  }
  if (tid == 0 && bad) atomicExch(status, kStatusNotPD);
}

constexpr int DIAG_SMEM = (NB * SP + (NB / 2) * TP + 2 * NB + (NB / 16) * 16 * 17) * static_cast<int>(sizeof(real));


struct Scratch {
  real* P;
  real* P0;  // the top level's own P when its T product overlaps the left recursion
  std::vector<real*> T;
  std::vector<int8_t*> SX, SY;
  std::vector<int*> EX, EY;
};

size_t scratch_elems(int64_t n, Scratch* out, real* base, bool overlap) {
  Plan pl;
  fplan::plan(n, 0, pl, static_cast<size_t>(i8f_slices()));
  size_t off = 0;
  auto take = [&](size_t e) {
    real* p = base ? base + off : nullptr;
    off += (e + 31) & ~size_t(31);
    return p;
  };
  auto take_bytes = [&](size_t b) { return reinterpret_cast<char*>(take((b + sizeof(real) - 1) / sizeof(real))); };
  real* P = take(pl.pmax);
  if (out) out->P = P;
  real* P0 = (overlap && !pl.tmax.empty()) ? take(pl.tmax[0]) : nullptr;
  if (out) out->P0 = P0;
  for (size_t d = 0; d < pl.tmax.size(); ++d) {
    real* t = take(pl.tmax[d]);
    int8_t* sx = pl.sx[d] ? reinterpret_cast<int8_t*>(take_bytes(pl.sx[d])) : nullptr;
    int8_t* sy = pl.sy[d] ? reinterpret_cast<int8_t*>(take_bytes(pl.sy[d])) : nullptr;
    int* ex = pl.ex[d] ? reinterpret_cast<int*>(take_bytes(pl.ex[d] * sizeof(int))) : nullptr;
    int* ey = pl.ey[d] ? reinterpret_cast<int*>(take_bytes(pl.ey[d] * sizeof(int))) : nullptr;
    if (out) {
      out->T.push_back(t);
      out->SX.push_back(sx);
      out->SY.push_back(sy);
      out->EX.push_back(ex);
      out->EY.push_back(ey);
    }
  }
  return off;
}

// Overlap of the top level's T = P U22 with the left recursion: T runs on `side` while the
// left half (latency-bound leaves and small GEMMs deeper down) runs on the main stream.
struct Overlap {
  cudaStream_t side = nullptr;
  cudaEvent_t p_ready = nullptr, t_ready = nullptr;
};

// Factor and invert the block [lo, hi) of A (upper triangle valid: the Schur complement
// with respect to every column right of hi); writes U[lo:hi, lo:hi].
int factor_rec(real* A, real* R, int64_t n, int64_t lo, int64_t hi, int depth, Scratch& sc, int* status,
               cudaStream_t s, const Overlap& ov) {
  const int64_t m = hi - lo;
  if (m <= NB) {
    chol_diag_kernel<<<1, DIAG_THREADS, DIAG_SMEM, s>>>(A, n, lo, static_cast<int>(m), R, status);
    return after_launch();
  }
  const int64_t n2 = right_part(m), n1 = m - n2, mid = hi - n2;
  GPTQ_TRY(factor_rec(A, R, n, mid, hi, depth + 1, sc, status, s, ov));
  real* U22 = R + mid * n + mid;
  const bool overlap = depth == 0 && ov.side != nullptr && sc.P0 != nullptr;
  real* P = overlap ? sc.P0 : sc.P;
  real* T = sc.T[depth];
  const size_t d = static_cast<size_t>(depth);
  const bool i8 = node_i8(n2);
  cudaStream_t st = s;
  if (i8) {
    // Int8 route, in negated form so that every product is a subtraction C -= A B:
    //   P' = 0 - B U22^T = -P;  A' = A - P' P'^T;  T = 0 - P' U22 = P U22;  U12 = 0 - U11 T.
    int8_t *SX = sc.SX[d], *SY = sc.SY[d];
    int *EX = sc.EX[d], *EY = sc.EY[d];
    const int64_t K2 = pad64(n2), K1 = pad64(n1);
    GPTQ_TRY(i8f_split_rows(s, A + lo * n + mid, n, n1, n2, K2, SX, EX));
    GPTQ_TRY(i8f_split_rows(s, U22, n, n2, n2, K2, SY, EY));
    GPTQ_CUDA(cudaMemsetAsync(P, 0, static_cast<size_t>(n1) * n2 * sizeof(real), s));
    GPTQ_TRY(i8f_gemm_sub(s, n1, n2, K2, SX, n1, EX, SY, n2, EY, P, n2, /*B[k, c] = U22[c, k]*/ 1, 0));
    GPTQ_TRY(i8f_split_rows(s, P, n2, n1, n2, K2, SX, EX));
    GPTQ_TRY(i8f_gemm_sub(s, n1, n1, K2, SX, n1, EX, SX, n1, EX, A + lo * n + lo, n, 0, /*upper*/ 1));
    if (overlap) {
      GPTQ_CUDA(cudaEventRecord(ov.p_ready, s));
      GPTQ_CUDA(cudaStreamWaitEvent(ov.side, ov.p_ready, 0));
      st = ov.side;
    }
    GPTQ_TRY(i8f_split_cols(st, U22, n, n2, n2, K2, SY, EY));
    GPTQ_CUDA(cudaMemsetAsync(T, 0, static_cast<size_t>(n1) * n2 * sizeof(real), st));
    GPTQ_TRY(i8f_gemm_sub(st, n1, n2, K2, SX, n1, EX, SY, n2, EY, T, n2, /*B[k, c] = U22[k, c]*/ 2, 0));
    if (overlap) GPTQ_CUDA(cudaEventRecord(ov.t_ready, ov.side));
    GPTQ_TRY(factor_rec(A, R, n, lo, mid, depth + 1, sc, status, s, ov));
    if (overlap) GPTQ_CUDA(cudaStreamWaitEvent(s, ov.t_ready, 0));
    GPTQ_TRY(i8f_split_rows(s, R + lo * n + lo, n, n1, n1, K1, SX, EX));
    GPTQ_TRY(i8f_split_cols(s, T, n2, n1, n2, K1, SY, EY));
    // U12 starts at zero (U is cleared before the recursion)
    return i8f_gemm_sub(s, n1, n2, K1, SX, n1, EX, SY, n2, EY, R + lo * n + mid, n, /*A[r, k] = U11[r, k]*/ 3, 0);
  }
  // P = B U22^T
  GPTQ_TRY(dgemm(s, n1, n2, n2, 1.0, A + lo * n + mid, n, U22, n, true, 0.0, P, n2, false, kTriBTUpper));
  // A' = A - P P^T (upper tiles)
  GPTQ_TRY(dgemm(s, n1, n1, n2, -1.0, P, n2, P, n2, true, 1.0, A + lo * n + lo, n, true));
  // T = P U22
  if (overlap) {
    GPTQ_CUDA(cudaEventRecord(ov.p_ready, s));
    GPTQ_CUDA(cudaStreamWaitEvent(ov.side, ov.p_ready, 0));
    st = ov.side;
  }
  GPTQ_TRY(dgemm(st, n1, n2, n2, 1.0, P, n2, U22, n, false, 0.0, T, n2, false, kTriBUpper));
  if (overlap) GPTQ_CUDA(cudaEventRecord(ov.t_ready, ov.side));
  GPTQ_TRY(factor_rec(A, R, n, lo, mid, depth + 1, sc, status, s, ov));
  if (overlap) GPTQ_CUDA(cudaStreamWaitEvent(s, ov.t_ready, 0));
  // U12 = -U11 T
  return dgemm(s, n1, n2, n1, -1.0, R + lo * n + lo, n, T, n2, false, 0.0, R + lo * n + mid, n, false, kTriAUpper);
}

}  // namespace

size_t factor_small_bytes(int64_t n) { return 256; }

size_t factor_work_bytes(int64_t n, bool overlap) {
  return (static_cast<size_t>(n) * n + scratch_elems(n, nullptr, nullptr, overlap)) * sizeof(real);
}

int factor_hessian(const float* H, int64_t n, float damp, bool desc_act, double* U, int32_t* perm,
                   int32_t* invperm, void* work, void* small, int* status, cudaStream_t s, cudaStream_t side,
                   cudaEvent_t ev_p, cudaEvent_t ev_t) {
  GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(chol_diag_kernel), DIAG_SMEM));
  double* dsum = reinterpret_cast<double*>(small);
  real* A = static_cast<real*>(work);  // damped (permuted) Hessian, then Schur complements
  Scratch sc;
  scratch_elems(n, &sc, A + static_cast<size_t>(n) * n, side != nullptr);
  Overlap ov;
  if (side) ov = Overlap{side, ev_p, ev_t};

  diag_sum_kernel<<<1, DSUM_THREADS, 0, s>>>(H, n, dsum);
  GPTQ_TRY(after_launch());
  if (desc_act) {
    act_order_rank_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(H, n, perm, invperm);
    GPTQ_TRY(after_launch());
  }
  const dim3 rgrid(static_cast<unsigned>((n + 255) / 256), static_cast<unsigned>(n));
  permute_damp_kernel<<<rgrid, 256, 0, s>>>(H, n, desc_act ? perm : nullptr, dsum, damp, A);
  GPTQ_TRY(after_launch());
  // U starts as zeros: the GEMMs skip its (exactly zero) lower triangle.
  GPTQ_CUDA(cudaMemsetAsync(U, 0, static_cast<size_t>(n) * n * sizeof(real), s));
  return factor_rec(A, U, n, 0, n, 0, sc, status, s, ov);
}

}  // namespace gptq
