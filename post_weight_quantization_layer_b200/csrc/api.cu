// extern "C" entry points: argument validation, workspace, orchestration, status.
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <memory>
#include <vector>

#include "common.cuh"

namespace gptq {

std::atomic<uint64_t> g_launches{0};

namespace {

constexpr int kVersion = 100;  // 0.1.0

// Library-owned stream-ordered memory pool, one per device.  Its release threshold is
// unbounded, so workspace memory is kept between calls instead of being returned to the
// driver at every synchronisation (re-mapping hundreds of MB per call costs milliseconds).
// gptq_trim_workspace() hands the cached memory back.
std::mutex g_pool_mu;
std::map<int, cudaMemPool_t> g_pools;

cudaMemPool_t workspace_pool() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lk(g_pool_mu);
  auto it = g_pools.find(dev);
  if (it != g_pools.end()) return it->second;
  cudaMemPoolProps props = {};
  props.allocType = cudaMemAllocationTypePinned;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t pool = nullptr;
  if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  uint64_t thr = UINT64_MAX;
  cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
  // No reuse of a block freed on another stream through an inserted wait: concurrent calls
  // (the sweeps of one pipelined layer on their own streams) would queue behind each other.
  int no = 0;
  cudaMemPoolSetAttribute(pool, cudaMemPoolReuseAllowInternalDependencies, &no);
  g_pools[dev] = pool;
  return pool;
}

// Stream-ordered workspace: one allocation carved into aligned pieces.
struct Workspace {
  char* base = nullptr;
  size_t used = 0;
  size_t cap = 0;
  cudaStream_t s = nullptr;
  ~Workspace() {
    if (base) cudaFreeAsync(base, s);
  }
  template <typename T>
  T* take(size_t count) {
    const size_t off = (used + 255) & ~size_t(255);
    used = off + count * sizeof(T);
    return reinterpret_cast<T*>(base + off);
  }
};

size_t padded(size_t bytes) { return (bytes + 255) & ~size_t(255); }

int alloc(Workspace& ws, size_t bytes, cudaStream_t s) {
  ws.s = s;
  ws.cap = bytes;
  cudaMemPool_t pool = workspace_pool();
  if (!pool) return GPTQ_ERR_CUDA;
  cudaError_t e = cudaMallocFromPoolAsync(reinterpret_cast<void**>(&ws.base), bytes, pool, s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    ws.base = nullptr;
    return GPTQ_ERR_OOM;
  }
  return GPTQ_OK;
}

// Read the device status word after the stream drains.
int finish(int* dstatus, cudaStream_t s) {
  int h = 0;
  if (cudaMemcpyAsync(&h, dstatus, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ_ERR_CUDA;
  return h;
}

bool valid_damp(float d) { return d > 0.f && d < 1.f; }  // false for NaN

int check_quant_args(const void* W, int w_dtype, int64_t n_out, int64_t n_in, int bits, int group_size,
                     int blocksize, const void* qweight, const void* scales, const void* zeros, const void* g_idx) {
  if (!W || !qweight || !scales || !zeros || !g_idx) return GPTQ_ERR_INVALID_ARG;
  if (w_dtype != GPTQ_F32 && w_dtype != GPTQ_F16 && w_dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (n_out <= 0 || n_in <= 0) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if (!(group_size == -1 || group_size > 0)) return GPTQ_ERR_INVALID_ARG;
  if (group_size > 0 && n_in % group_size != 0) return GPTQ_ERR_INVALID_ARG;
  if (blocksize <= 0) return GPTQ_ERR_INVALID_ARG;
  if (n_in % 8 != 0 || (n_in * bits) % 32 != 0) return GPTQ_ERR_UNSUPPORTED;
  if (n_in > 65535 || n_out > 65535) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned16(W) || !aligned16(qweight) || !aligned16(scales) || !aligned16(zeros) || !aligned16(g_idx))
    return GPTQ_ERR_UNSUPPORTED;
  return GPTQ_OK;
}

__global__ void invert_perm_kernel(const int32_t* __restrict__ perm, int64_t n, int32_t* __restrict__ invperm,
                                   int* status) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int32_t p = perm[j];
  if (p < 0 || p >= n) {
    atomicExch(status, GPTQ_ERR_INVALID_ARG);
    return;
  }
  invperm[p] = static_cast<int32_t>(j);
}

__global__ void iota_kernel(int32_t* __restrict__ p, int64_t n) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j < n) p[j] = static_cast<int32_t>(j);
}

// A permutation is valid iff invperm[perm[j]] == j for every j (after the scatter).
__global__ void check_perm_kernel(const int32_t* __restrict__ perm, const int32_t* __restrict__ invperm, int64_t n,
                                  int* status) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int32_t p = perm[j];
  if (p < 0 || p >= n || invperm[p] != j) atomicExch(status, GPTQ_ERR_INVALID_ARG);
}

struct Events {
  cudaEvent_t ev[6] = {};
  bool on = false;
  int create(bool want) {
    on = want;
    if (!on) return GPTQ_OK;
    for (auto& e : ev)
      if (cudaEventCreate(&e) != cudaSuccess) return GPTQ_ERR_CUDA;
    return GPTQ_OK;
  }
  ~Events() {
    if (on)
      for (auto& e : ev)
        if (e) cudaEventDestroy(e);
  }
  float ms(int a, int b) {
    float t = 0.f;
    if (on) cudaEventElapsedTime(&t, ev[a], ev[b]);
    return t;
  }
};

int sweep_common(const void* W, int w_dtype, int64_t n_out, int64_t n_in, const double* U, const int32_t* perm,
                 const int32_t* invperm, int bits, int group_size, int sym, int static_groups, int blocksize,
                 int32_t* qweight, float* scales, int32_t* zeros, int32_t* g_idx, double* Wk, double* Err,
                 uint8_t* codesT, double* loss, int* status, cudaStream_t s, gptq_stats* stats, Events& evs,
                 int ev0, bool low_priority = false) {
  SweepArgs a;
  a.W = W;
  a.w_dtype = w_dtype;
  a.n_out = n_out;
  a.n_in = n_in;
  a.U = U;
  a.perm = perm;
  a.invperm = invperm;
  a.bits = bits;
  a.group_size = group_size;
  a.sym = sym != 0;
  a.static_groups = static_groups != 0 && group_size > 0;
  a.blocksize = blocksize;
  a.qweight = qweight;
  a.scales = scales;
  a.zeros = zeros;
  a.g_idx = g_idx;
  a.Wk = Wk;
  a.Err = Err;
  a.codesT = codesT;
  a.loss = loss;
  a.status = status;
  a.stats = stats;
  for (int i = 0; i < 4; ++i) a.ev[i] = evs.on ? evs.ev[ev0 + i] : nullptr;
  a.low_priority = low_priority ? 1 : 0;
  int pw = 0, qw = 0;
  GPTQ_TRY(run_sweep(a, s, &pw, &qw));
  if (stats) {
    stats->panel_width = pw;
    stats->outer_width = qw;
  }
  return GPTQ_OK;
}

// The factor of one Hessian on leased lanes: the recursion on a lane of priority `prio`, the
// top level's T product on a low-priority lane beside it (so it fills the SMs that the left
// half's serial leaf steps leave idle).  Both lanes join back into s when this returns.
// `work` must hold factor_work_bytes(n, true).
int factor_on_lanes(const float* H, int64_t n, float damp, bool desc_act, double* U, int32_t* perm,
                    int32_t* invperm, void* work, void* small, int* status, bool fill_identity, LanePrio prio,
                    cudaStream_t s) {
  LaneLease lanes(s);
  const LanePrio pr[2] = {prio, kLaneLow};
  GPTQ_TRY(lanes.acquire(2, pr));
  cudaStream_t main = lanes[0].st;
  GPTQ_TRY(factor_hessian(H, n, damp, desc_act, U, perm, invperm, work, small, status, main, lanes[1].st,
                          lanes[1].aux, lanes[1].aux2));
  if (fill_identity && !desc_act) {
    iota_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, main>>>(perm, n);
    GPTQ_TRY(after_launch());
  }
  return GPTQ_OK;
}

}  // namespace

int pool_alloc(void** p, size_t bytes, cudaStream_t s) {
  *p = nullptr;
  cudaMemPool_t pool = workspace_pool();
  if (!pool) return GPTQ_ERR_CUDA;
  if (cudaMallocFromPoolAsync(p, bytes, pool, s) != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return GPTQ_ERR_OOM;
  }
  return GPTQ_OK;
}

void pool_free(void* p, cudaStream_t s) {
  if (p) cudaFreeAsync(p, s);
}

}  // namespace gptq

using namespace gptq;

extern "C" {

int gptq_version(void) { return kVersion; }

uint64_t gptq_launch_count(void) { return g_launches.load(); }

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_INVALID_ARG: return "invalid argument";
    case GPTQ_ERR_UNSUPPORTED: return "unsupported size, dtype or alignment";
    case GPTQ_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case GPTQ_ERR_CUDA: return "CUDA error";
    case GPTQ_ERR_OOM: return "workspace allocation failed";
    case GPTQ_ERR_TIMEOUT: return "bounded device wait timed out";
    default: return "unknown status";
  }
}

int gptq_accumulate_hessian(const void* X, int x_dtype, int64_t tokens, int64_t n_in, float* H, void* stream) {
  if (tokens < 0 || n_in <= 0) return GPTQ_ERR_INVALID_ARG;
  if (!H || (!X && tokens > 0)) return GPTQ_ERR_INVALID_ARG;
  if (x_dtype == GPTQ_F32) return GPTQ_ERR_UNSUPPORTED;
  if (x_dtype != GPTQ_F16 && x_dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (n_in % 8 != 0 || n_in > 65535) return GPTQ_ERR_UNSUPPORTED;
  if (tokens == 0) return GPTQ_OK;  // nothing to add; X may be NULL
  if (!aligned16(X) || !aligned16(H)) return GPTQ_ERR_UNSUPPORTED;
  return launch_hessian(X, x_dtype, tokens, n_in, H, static_cast<cudaStream_t>(stream));
}

int gptq_trim_workspace(void) {
  cudaMemPool_t pool = workspace_pool();
  if (!pool) return GPTQ_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return GPTQ_ERR_CUDA;
  return cudaMemPoolTrimTo(pool, 0) == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

int gptq_test_wait_expiry(int skip_loads, uint32_t wait_limit) {
  if (skip_loads && wait_limit == 0) return GPTQ_ERR_INVALID_ARG;  // only with a short limit
  hessian_wait_test(skip_loads, wait_limit);
  return GPTQ_OK;
}

int gptq_device_status(void* stream, int clear) {
  const int h = hessian_device_status(static_cast<cudaStream_t>(stream), clear);
  const int g = gemm_device_status(clear);
  const int i = i8_device_status(clear);
  return h != GPTQ_OK ? h : (g != GPTQ_OK ? g : i);
}

int gptq_factor_hessian(const float* H, int64_t n_in, float damp_percent, int desc_act, double* U, int32_t* perm,
                        void* stream) {
  if (!H || !U || !perm) return GPTQ_ERR_INVALID_ARG;
  if (n_in <= 0 || !valid_damp(damp_percent)) return GPTQ_ERR_INVALID_ARG;
  if (n_in % 8 != 0 || n_in > 65535) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned16(H) || !aligned16(U) || !aligned16(perm)) return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t n = static_cast<size_t>(n_in);
  Workspace ws;
  GPTQ_TRY(alloc(ws, padded(factor_work_bytes(n_in, true)) + padded(factor_small_bytes(n_in)) + padded(n * 4) + 512, s));
  void* work = ws.take<char>(factor_work_bytes(n_in, true));
  void* small = ws.take<char>(factor_small_bytes(n_in));
  int32_t* invperm = ws.take<int32_t>(n);
  int* status = ws.take<int>(1);
  GPTQ_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  GPTQ_TRY(factor_on_lanes(H, n_in, damp_percent, desc_act != 0, U, perm, invperm, work, small, status, true,
                           kLaneHigh, s));
  return finish(status, s);
}

int gptq_factor_hessians(int count, const float* const* H, const int64_t* n_in, float damp_percent,
                         int desc_act, double* const* U, int32_t* const* perm, void* stream, int* statuses) {
  if (count <= 0 || !H || !n_in || !U || !perm) return GPTQ_ERR_INVALID_ARG;
  if (!valid_damp(damp_percent)) return GPTQ_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (!H[i] || !U[i] || !perm[i] || n_in[i] <= 0) return GPTQ_ERR_INVALID_ARG;
    if (n_in[i] % 8 != 0 || n_in[i] > 65535) return GPTQ_ERR_UNSUPPORTED;
    if (!aligned16(H[i]) || !aligned16(U[i]) || !aligned16(perm[i])) return GPTQ_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  size_t bytes = padded(static_cast<size_t>(count) * sizeof(int));
  for (int i = 0; i < count; ++i) {
    const size_t n = static_cast<size_t>(n_in[i]);
    bytes += padded(factor_work_bytes(n_in[i], true)) + padded(factor_small_bytes(n_in[i])) + padded(n * 4);
  }
  Workspace ws;
  GPTQ_TRY(alloc(ws, bytes + 256, s));
  int* status = ws.take<int>(static_cast<size_t>(count));
  GPTQ_CUDA(cudaMemsetAsync(status, 0, static_cast<size_t>(count) * sizeof(int), s));
  // The largest factorisation is the critical path: its lanes have the highest priority.
  int largest = 0;
  for (int i = 1; i < count; ++i)
    if (n_in[i] > n_in[largest]) largest = i;
  // Two lanes per item: its recursion, and its top-level T product beside it.
  std::vector<LanePrio> prio(2 * static_cast<size_t>(count), kLaneLow);
  prio[2 * static_cast<size_t>(largest)] = kLaneHigh;
  {
    LaneLease lanes(s);
    GPTQ_TRY(lanes.acquire(2 * count, prio.data()));
    for (int i = 0; i < count; ++i) {
      const int64_t n = n_in[i];
      void* work = ws.take<char>(factor_work_bytes(n, true));
      void* small = ws.take<char>(factor_small_bytes(n));
      int32_t* invperm = ws.take<int32_t>(static_cast<size_t>(n));
      Lane& li = lanes[2 * i];
      Lane& lt = lanes[2 * i + 1];
      GPTQ_TRY(factor_hessian(H[i], n, damp_percent, desc_act != 0, U[i], perm[i], invperm, work, small, status + i,
                              li.st, lt.st, lt.aux, lt.aux2));
      if (!desc_act) {
        iota_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, li.st>>>(perm[i], n);
        GPTQ_TRY(after_launch());
      }
    }
  }  // every lane joins back into s
  std::vector<int> h(static_cast<size_t>(count), 0);
  if (cudaMemcpyAsync(h.data(), status, static_cast<size_t>(count) * sizeof(int), cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ_ERR_CUDA;
  int first = GPTQ_OK;
  for (int i = 0; i < count; ++i) {
    if (statuses) statuses[i] = h[static_cast<size_t>(i)];
    if (first == GPTQ_OK && h[static_cast<size_t>(i)] != GPTQ_OK) first = h[static_cast<size_t>(i)];
  }
  return first;
}

int gptq_quantize_linears(int n_hessians, const float* const* H, const int64_t* n_in, float damp_percent,
                          int desc_act, double* const* U, int32_t* const* perm, int n_linears,
                          const void* const* W, int w_dtype, const int64_t* n_out, const int* hessian_of, int bits,
                          int group_size, int sym, int static_groups, int blocksize, int32_t* const* qweight,
                          float* const* scales, int32_t* const* zeros, int32_t* const* g_idx,
                          void* const* hessian_ready, void* stream, int* statuses) {
  if (n_hessians <= 0 || n_linears <= 0 || !H || !n_in || !U || !perm || !W || !n_out || !hessian_of || !qweight ||
      !scales || !zeros || !g_idx)
    return GPTQ_ERR_INVALID_ARG;
  if (!valid_damp(damp_percent)) return GPTQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_hessians; ++i) {
    if (!H[i] || !U[i] || !perm[i] || n_in[i] <= 0) return GPTQ_ERR_INVALID_ARG;
    if (n_in[i] % 8 != 0 || n_in[i] > 65535) return GPTQ_ERR_UNSUPPORTED;
    if (!aligned16(H[i]) || !aligned16(U[i]) || !aligned16(perm[i])) return GPTQ_ERR_UNSUPPORTED;
  }
  for (int j = 0; j < n_linears; ++j) {
    if (hessian_of[j] < 0 || hessian_of[j] >= n_hessians) return GPTQ_ERR_INVALID_ARG;
    GPTQ_TRY(check_quant_args(W[j], w_dtype, n_out[j], n_in[hessian_of[j]], bits, group_size, blocksize, qweight[j],
                              scales[j], zeros[j], g_idx[j]));
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  size_t bytes = padded(static_cast<size_t>(n_hessians + n_linears) * sizeof(int));
  for (int i = 0; i < n_hessians; ++i)
    bytes += padded(factor_work_bytes(n_in[i], true)) + padded(factor_small_bytes(n_in[i])) +
             padded(static_cast<size_t>(n_in[i]) * 4);
  for (int j = 0; j < n_linears; ++j) {
    const size_t e = static_cast<size_t>(n_out[j]) * static_cast<size_t>(n_in[hessian_of[j]]);
    bytes += 2 * padded(e * 8) + padded(e) + padded(sizeof(double));
  }
  Workspace ws;  // declared before the leases: freed on s after every lane has joined
  GPTQ_TRY(alloc(ws, bytes + 256, s));
  int* dstat = ws.take<int>(static_cast<size_t>(n_hessians + n_linears));
  GPTQ_CUDA(cudaMemsetAsync(dstat, 0, static_cast<size_t>(n_hessians + n_linears) * sizeof(int), s));
  int largest = 0;
  for (int i = 1; i < n_hessians; ++i)
    if (n_in[i] > n_in[largest]) largest = i;
  std::vector<LanePrio> prio(static_cast<size_t>(n_hessians), kLaneLow);
  prio[static_cast<size_t>(largest)] = kLaneHigh;
  std::vector<int32_t*> invperm(static_cast<size_t>(n_hessians), nullptr);
  Events off;
  GPTQ_TRY(off.create(false));
  {
    // One chain lane per Hessian: its factor, then (forked from it) one lane per linear
    // that reads it.  The sub-leases end before the chain lease (reverse declaration order).
    LaneLease chains(s);
    GPTQ_TRY(chains.acquire(n_hessians, prio.data()));
    // A Hessian finished on another stream: its chain also waits for the caller's event.
    if (hessian_ready)
      for (int i = 0; i < n_hessians; ++i)
        if (hessian_ready[i])
          GPTQ_CUDA(cudaStreamWaitEvent(chains[i].st, static_cast<cudaEvent_t>(hessian_ready[i]), 0));
    std::vector<std::unique_ptr<LaneLease>> subs;
    for (int i = 0; i < n_hessians; ++i) {
      const int64_t n = n_in[i];
      void* work = ws.take<char>(factor_work_bytes(n, true));
      void* small = ws.take<char>(factor_small_bytes(n));
      invperm[static_cast<size_t>(i)] = ws.take<int32_t>(static_cast<size_t>(n));
      GPTQ_TRY(factor_on_lanes(H[i], n, damp_percent, desc_act != 0, U[i], perm[i], invperm[static_cast<size_t>(i)],
                               work, small, dstat + i, true, prio[static_cast<size_t>(i)], chains[i].st));
    }
    for (int i = 0; i < n_hessians; ++i) {
      std::vector<int> mine;
      for (int j = 0; j < n_linears; ++j)
        if (hessian_of[j] == i) mine.push_back(j);
      if (mine.empty()) continue;
      subs.emplace_back(new LaneLease(chains[i].st));
      LaneLease& lease = *subs.back();
      const std::vector<LanePrio> lp(mine.size(), prio[static_cast<size_t>(i)]);
      GPTQ_TRY(lease.acquire(static_cast<int>(mine.size()), lp.data()));
      const int64_t ni = n_in[i];
      for (size_t t = 0; t < mine.size(); ++t) {
        const int j = mine[t];
        const size_t e = static_cast<size_t>(n_out[j]) * static_cast<size_t>(ni);
        double* Wk = ws.take<double>(e);
        double* Err = ws.take<double>(e);
        uint8_t* codesT = ws.take<uint8_t>(e);
        double* loss = ws.take<double>(1);
        GPTQ_TRY(sweep_common(W[j], w_dtype, n_out[j], ni, U[i], desc_act ? perm[i] : nullptr,
                              desc_act ? invperm[static_cast<size_t>(i)] : nullptr, bits, group_size, sym,
                              static_groups, blocksize, qweight[j], scales[j], zeros[j], g_idx[j], Wk, Err, codesT,
                              loss, dstat + n_hessians + j, lease[static_cast<int>(t)].st, nullptr, off, 0,
                              /*low_priority: the largest Hessian's sweeps follow the critical path*/ i != largest));
      }
    }
  }  // every lane joins back into s
  std::vector<int> h(static_cast<size_t>(n_hessians + n_linears), 0);
  if (cudaMemcpyAsync(h.data(), dstat, h.size() * sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ_ERR_CUDA;
  int first = GPTQ_OK;
  for (int j = 0; j < n_linears; ++j) {
    const int hf = h[static_cast<size_t>(hessian_of[j])];
    const int st = hf != GPTQ_OK ? hf : h[static_cast<size_t>(n_hessians + j)];
    if (statuses) statuses[j] = st;
    if (first == GPTQ_OK && st != GPTQ_OK) first = st;
  }
  return first;
}

int gptq_quantize_layer_factored(const void* W, int w_dtype, int64_t n_out, int64_t n_in, const double* U,
                                 const int32_t* perm, int bits, int group_size, int sym, int static_groups,
                                 int blocksize, int32_t* qweight, float* scales, int32_t* zeros, int32_t* g_idx,
                                 void* stream, gptq_stats* stats) {
  GPTQ_TRY(check_quant_args(W, w_dtype, n_out, n_in, bits, group_size, blocksize, qweight, scales, zeros, g_idx));
  if (!U || !perm) return GPTQ_ERR_INVALID_ARG;
  if (!aligned16(U) || !aligned16(perm)) return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t no = static_cast<size_t>(n_out), ni = static_cast<size_t>(n_in);
  Events evs;
  GPTQ_TRY(evs.create(stats != nullptr));
  Workspace ws;
  GPTQ_TRY(alloc(ws, 2 * padded(no * ni * 8) + padded(no * ni) + padded(ni * 4) + 1024, s));
  double* Wk = ws.take<double>(no * ni);
  double* Err = ws.take<double>(no * ni);
  uint8_t* codesT = ws.take<uint8_t>(no * ni);
  int32_t* invperm = ws.take<int32_t>(ni);
  double* loss = ws.take<double>(1);
  int* status = ws.take<int>(1);
  GPTQ_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  const unsigned g1 = static_cast<unsigned>((ni + 255) / 256);
  invert_perm_kernel<<<g1, 256, 0, s>>>(perm, n_in, invperm, status);
  GPTQ_TRY(after_launch());
  check_perm_kernel<<<g1, 256, 0, s>>>(perm, invperm, n_in, status);
  GPTQ_TRY(after_launch());
  GPTQ_TRY(sweep_common(W, w_dtype, n_out, n_in, U, perm, invperm, bits, group_size, sym, static_groups, blocksize,
                        qweight, scales, zeros, g_idx, Wk, Err, codesT, loss, status, s, stats, evs, 0));
  if (stats) GPTQ_CUDA(cudaMemcpyAsync(&stats->damped_loss, loss, sizeof(double), cudaMemcpyDeviceToHost, s));
  const int st = finish(status, s);
  if (stats) {
    stats->ms_prepare = evs.ms(0, 1);
    stats->ms_factor = 0.f;
    stats->ms_sweep = evs.ms(1, 2);
    stats->ms_pack = evs.ms(2, 3);
  }
  return st;
}

int gptq_quantize_layer(const void* W, int w_dtype, int64_t n_out, int64_t n_in, const float* H, int bits,
                        int group_size, float damp_percent, int sym, int desc_act, int static_groups, int blocksize,
                        int32_t* qweight, float* scales, int32_t* zeros, int32_t* g_idx, void* stream,
                        gptq_stats* stats) {
  GPTQ_TRY(check_quant_args(W, w_dtype, n_out, n_in, bits, group_size, blocksize, qweight, scales, zeros, g_idx));
  if (!H) return GPTQ_ERR_INVALID_ARG;
  if (!valid_damp(damp_percent)) return GPTQ_ERR_INVALID_ARG;
  if (!aligned16(H)) return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t no = static_cast<size_t>(n_out), ni = static_cast<size_t>(n_in);
  Events evs;
  GPTQ_TRY(evs.create(stats != nullptr));
  Workspace ws;
  GPTQ_TRY(alloc(ws,
                 padded(factor_work_bytes(n_in, true)) + padded(ni * ni * 8) + padded(factor_small_bytes(n_in)) +
                     2 * padded(ni * 4) + 2 * padded(no * ni * 8) + padded(no * ni) + 1024,
                 s));
  void* work = ws.take<char>(factor_work_bytes(n_in, true));
  double* U = ws.take<double>(ni * ni);
  void* small = ws.take<char>(factor_small_bytes(n_in));
  int32_t* perm = ws.take<int32_t>(ni);
  int32_t* invperm = ws.take<int32_t>(ni);
  double* Wk = ws.take<double>(no * ni);
  double* Err = ws.take<double>(no * ni);
  uint8_t* codesT = ws.take<uint8_t>(no * ni);
  double* loss = ws.take<double>(1);
  int* status = ws.take<int>(1);
  GPTQ_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  if (evs.on) GPTQ_CUDA(cudaEventRecord(evs.ev[4], s));
  GPTQ_TRY(factor_on_lanes(H, n_in, damp_percent, desc_act != 0, U, perm, invperm, work, small, status, false,
                           kLaneHigh, s));
  if (evs.on) GPTQ_CUDA(cudaEventRecord(evs.ev[5], s));
  GPTQ_TRY(sweep_common(W, w_dtype, n_out, n_in, U, desc_act ? perm : nullptr, desc_act ? invperm : nullptr, bits,
                        group_size, sym, static_groups, blocksize, qweight, scales, zeros, g_idx, Wk, Err, codesT,
                        loss, status, s, stats, evs, 0));
  if (stats) GPTQ_CUDA(cudaMemcpyAsync(&stats->damped_loss, loss, sizeof(double), cudaMemcpyDeviceToHost, s));
  const int st = finish(status, s);
  if (stats) {
    stats->ms_factor = evs.ms(4, 5);
    stats->ms_prepare = evs.ms(0, 1);
    stats->ms_sweep = evs.ms(1, 2);
    stats->ms_pack = evs.ms(2, 3);
  }
  return st;
}

}  // extern "C"
