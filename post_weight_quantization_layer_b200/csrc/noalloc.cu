// gptq_factor_hessian_noalloc: the damped inverse-Cholesky factor for callers that must
// not allocate device memory.
//
// Some callers cannot call cudaMalloc or any allocating routine: code running inside a
// host that owns all device memory up front (an inference or serving runtime with a
// fixed arena, a real-time loop that forbids allocator calls after start-up, or a plugin
// whose host has capped the allocator), where an allocation would fail or break the
// host's accounting.  This entry point runs the same kernels as gptq_factor_hessian but
// takes its scratch from one fixed array in device memory instead of the library's
// workspace pool.
//
// The scratch lives in the file-scope array below; every GPU that loads this library
// holds it until the process exits.  Host code cannot use the array's name as a device
// address (it names a host-side stand-in), so the device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, on the first call
// made on that device.
#include <map>
#include <mutex>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int64_t kNoAllocMaxN = 1024;  // largest n_in this entry point accepts
constexpr size_t kAlign = 256;
constexpr size_t align_up(size_t b) { return (b + kAlign - 1) & ~(kAlign - 1); }

// Scratch layout for n = kNoAllocMaxN: the factor's fp64 work area (the damped Hessian
// plus the recursion's product buffers: 1,658,880 doubles at n = 1024), the small factor
// buffer (diag sum), the inverse permutation and the status word.  The entry point
// re-checks at run time that the factor's needs fit.
constexpr size_t kWorkBytes = size_t(1658880) * sizeof(double);
constexpr size_t kSmallBytes = 256;
constexpr size_t kPermBytes = static_cast<size_t>(kNoAllocMaxN) * sizeof(int32_t);
constexpr size_t kScratchBytes = align_up(kWorkBytes) + align_up(kSmallBytes) + align_up(kPermBytes) + kAlign;

static __device__ __align__(256) unsigned char g_factor_scratch[kScratchBytes];

__global__ void identity_order_kernel(int32_t* __restrict__ p, int64_t n) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j < n) p[j] = static_cast<int32_t>(j);
}

std::mutex g_mu;
std::map<int, unsigned char*> g_addr;  // device ordinal -> device address of the scratch

// Device address of the scratch on the current device (looked up once per device).
int scratch_address(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_addr.find(dev);
  if (it == g_addr.end()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_factor_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return GPTQ_ERR_CUDA;
    }
    it = g_addr.emplace(dev, static_cast<unsigned char*>(p)).first;
  }
  *out = it->second;
  return GPTQ_OK;
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" int gptq_factor_hessian_noalloc(const float* H, int64_t n_in, float damp_percent, int desc_act,
                                           double* U, int32_t* perm, void* stream) {
  if (!H || !U || !perm) return GPTQ_ERR_INVALID_ARG;
  if (n_in <= 0 || !(damp_percent > 0.f && damp_percent < 1.f)) return GPTQ_ERR_INVALID_ARG;
  if (n_in > kNoAllocMaxN) return GPTQ_ERR_UNSUPPORTED;  // beyond the fixed scratch
  if (n_in % 8 != 0) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned16(H) || !aligned16(U) || !aligned16(perm)) return GPTQ_ERR_UNSUPPORTED;
  if (factor_work_bytes(n_in, false) > kWorkBytes || factor_small_bytes(n_in) > kSmallBytes) return GPTQ_ERR_UNSUPPORTED;

  unsigned char* base = nullptr;
  GPTQ_TRY(scratch_address(&base));
  void* work = base;
  void* small = base + align_up(kWorkBytes);
  int32_t* invperm = reinterpret_cast<int32_t*>(base + align_up(kWorkBytes) + align_up(kSmallBytes));
  int* status = reinterpret_cast<int*>(base + align_up(kWorkBytes) + align_up(kSmallBytes) + align_up(kPermBytes));

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The scratch keeps the previous call's contents: the status word must start at zero
  // (every other piece is fully written before it is read).
  GPTQ_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  GPTQ_TRY(factor_hessian(H, n_in, damp_percent, desc_act != 0, U, perm, invperm, work, small, status, s));
  if (!desc_act) {  // identity order for the caller
    identity_order_kernel<<<static_cast<unsigned>((n_in + 255) / 256), 256, 0, s>>>(perm, n_in);
    GPTQ_TRY(after_launch());
  }
  int h = 0;
  if (cudaMemcpyAsync(&h, status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ_ERR_CUDA;
  return h;
}
