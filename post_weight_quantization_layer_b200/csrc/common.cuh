// Shared host/device helpers of the GPTQ library (internal).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>
#include <utility>
#include <vector>

#include "../../include/gptq.h"

namespace gptq {

// Count of kernels launched by this library (reported by gptq_launch_count).
extern std::atomic<uint64_t> g_launches;

// Launch bookkeeping: count the launch and turn a launch error into a status.
inline int after_launch() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

#define GPTQ_TRY(expr)              \
  do {                              \
    int _st = (expr);               \
    if (_st != GPTQ_OK) return _st; \
  } while (0)

#define GPTQ_CUDA(expr)                                 \
  do {                                                  \
    if ((expr) != cudaSuccess) { return GPTQ_ERR_CUDA; } \
  } while (0)

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Make a kernel's dynamic shared-memory limit on the current device at least `bytes`.  The
// attribute is per device: it is raised for every (device, kernel) pair this process
// launches on (a process may drive several GPUs) whenever a launch needs more than the
// limit set so far (kernels whose shared memory depends on the call's sizes).
// Thread-safe.
int ensure_smem_limit(const void* kernel, int bytes);

inline int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Device status word values shared by the kernels (same numbers as gptq_status).
constexpr int kStatusNotPD = GPTQ_ERR_NOT_PD;
constexpr int kStatusTimeout = GPTQ_ERR_TIMEOUT;

// ---------------------------------------------------------------------------------------------
// Internal entry points implemented in the other translation units.
// All are stream-ordered; they return a gptq_status for host-side launch errors.

// hessian.cu
int launch_hessian(const void* X, int x_dtype, int64_t tokens, int64_t n, float* H, cudaStream_t s);
int hessian_device_status(cudaStream_t s, int clear);
void hessian_wait_test(int skip_loads, uint32_t wait_limit);

// w4a16.cu: Y[M, N] = X[M, K] * Wd[N, K]^T, 16-bit operands (x_dtype), fp32 accumulate, on the
// tcgen05 tensor cores; and its bounded-wait status word.
int gemm_bf16_tn(const void* X, const void* Wd, void* Y, int64_t M, int64_t N, int64_t K, int x_dtype,
                 cudaStream_t s);
int gemm_device_status(int clear);

// gemm.cu: fp64 C[m,n] = beta*C[m,n] + alpha * sum_k A[m*lda+k] * B(k,n),
// B(k,n) = transB ? B[n*ldb+k] : B[k*ldb+n].  upper != 0 skips tiles of C lying entirely
// below its diagonal (m > n for every element).  `tri` declares operands that are
// triangular with exact zeros elsewhere, so that those K ranges are skipped:
constexpr int kTriAUpper = 1;   // A(m,k) == 0 for k < m
constexpr int kTriBUpper = 2;   // B(k,n) == 0 for k > n   (op(B) upper triangular)
constexpr int kTriBTUpper = 4;  // B(k,n) == 0 for k < n   (op(B) = U^T with U upper)
int dgemm(cudaStream_t s, int64_t M, int64_t N, int64_t K, double alpha, const double* A, int64_t lda,
          const double* B, int64_t ldb, bool transB, double beta, double* C, int64_t ldc, bool upper,
          int tri = 0);

// ozaki.cu: the sweep's trailing update C -= A B on the int8 tensor cores, A and B split
// into signed 7-bit slices (rows of A, columns of B) with power-of-two scales.
int i8_slices();
int64_t i8_padded_k(int64_t K);
int i8_split_rows(cudaStream_t s, const double* X, int64_t ldx, int64_t R, int64_t K, int64_t KP, int8_t* S, int* e);
int i8_split_cols(cudaStream_t s, const double* Y, int64_t ldy, int64_t K, int64_t N, int64_t KP, int8_t* S, int* e);
int i8_gemm_sub(cudaStream_t s, int64_t M, int64_t N, int64_t KP, const int8_t* SA, int64_t a_rows, const int* ea,
                const int8_t* SB, int64_t b_cols, const int* eb, int64_t col0, double* C, int64_t ldc,
                int max_ctas);
int i8f_slices();
int i8f_split_rows(cudaStream_t s, const double* X, int64_t ldx, int64_t R, int64_t K, int64_t KP, int8_t* S, int* e);
int i8f_split_cols(cudaStream_t s, const double* Y, int64_t ldy, int64_t K, int64_t N, int64_t KP, int8_t* S,
                   int* e);
int i8f_gemm_sub(cudaStream_t s, int64_t M, int64_t N, int64_t KP, const int8_t* SA, int64_t a_rows, const int* ea,
                 const int8_t* SB, int64_t b_cols, const int* eb, double* C, int64_t ldc, int krange, int upper);
int i8_device_status(int clear);

// factor.cu: U (sweep order, fp64) and perm from H, stream-ordered on s.  `work` holds
// factor_work_bytes(n, side != nullptr), `small` factor_small_bytes(n); `status` is a device
// int.  With a side stream (and two events for its ordering) the top level's T product runs
// on `side`, concurrently with the left half of the recursion; the call leaves no work on
// `side` that s does not wait for.
size_t factor_small_bytes(int64_t n);
size_t factor_work_bytes(int64_t n, bool overlap);
int factor_hessian(const float* H, int64_t n, float damp, bool desc_act, double* U, int32_t* perm,
                   int32_t* invperm, void* work, void* small, int* status, cudaStream_t s,
                   cudaStream_t side = nullptr, cudaEvent_t ev_p = nullptr, cudaEvent_t ev_t = nullptr);

// sweep.cu: everything after the factor.
struct SweepArgs {
  const void* W;
  int w_dtype;
  int64_t n_out, n_in;
  const double* U;
  const int32_t* perm;     // nullptr = identity
  const int32_t* invperm;  // nullptr = identity
  int bits, group_size;
  bool sym, static_groups;
  int blocksize;
  int32_t* qweight;
  float* scales;
  int32_t* zeros;
  int32_t* g_idx;
  // workspace
  double* Wk;       // [n_out, n_in] fp64 working copy of the weights, sweep order
  double* Err;      // [n_out, n_in] fp64 normalised errors, sweep order
  uint8_t* codesT;  // [n_in, n_out] codes in sweep order
  double* loss;     // one double
  int* status;
  gptq_stats* stats;      // may be null
  cudaEvent_t ev[4];      // valid when stats != null
  int low_priority = 0;   // panels and look-ahead on a low-priority lane too
};
int run_sweep(SweepArgs& a, cudaStream_t s, int* panel_width, int* outer_width);

// api.cu: stream-ordered allocation from the library's workspace pool (one pool per device,
// memory kept cached between calls).  pool_alloc returns GPTQ_ERR_OOM on failure.
int pool_alloc(void** p, size_t bytes, cudaStream_t s);
void pool_free(void* p, cudaStream_t s);

// lanes.cu: library-owned streams leased by one call (see the file's header).
enum LanePrio { kLaneHigh = 0, kLaneLow = 1 };
struct Lane {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaEvent_t aux = nullptr, aux2 = nullptr;  // free for the leasing call's own ordering
};
class LaneLease {
 public:
  explicit LaneLease(cudaStream_t s) : s_(s) {}
  ~LaneLease();  // joins every lane into the caller's stream, returns the lanes
  LaneLease(const LaneLease&) = delete;
  LaneLease& operator=(const LaneLease&) = delete;
  // Leases `count` lanes (priority class prio[i] for lane i), each forked from the
  // caller's stream.
  int acquire(int count, const LanePrio* prio);
  Lane& operator[](int i) { return *lanes_[i].first; }

 private:
  cudaStream_t s_;
  int dev_ = 0;
  std::vector<std::pair<Lane*, int>> lanes_;
};

}  // namespace gptq
