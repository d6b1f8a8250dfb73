// Library-owned streams ("lanes") leased by one call for work that runs concurrently with
// itself: the sweep's look-ahead (panels beside the trailing update) and the batched
// factor (several Hessians at once).
//
// Lanes are created once per device and priority class and kept on a free list, so a call
// pays no stream creation; concurrent calls from several host threads lease disjoint
// lanes, and a lease takes only lanes whose earlier work has drained (the pool grows to the
// largest number of lanes in flight at once).  A lease forks every lane from the caller's stream (the lane starts after all
// work already queued there) and, when it ends, makes the caller's stream wait for all
// work issued on its lanes, on error paths too, so stream-ordered frees of the call's
// workspace on the caller's stream never overtake a lane.
#include <cstddef>
#include <map>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace gptq {
namespace {

std::mutex g_lane_mu;
std::map<std::pair<int, int>, std::vector<Lane*>> g_lane_free;  // (device, priority class)

int create_lane(LanePrio prio, Lane** out) {
  int least = 0, greatest = 0;
  if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return GPTQ_ERR_CUDA;
  Lane* l = new Lane;
  bool ok = cudaStreamCreateWithPriority(&l->st, cudaStreamNonBlocking, prio == kLaneHigh ? greatest : least) ==
            cudaSuccess;
  for (cudaEvent_t* e : {&l->fork, &l->join, &l->aux, &l->aux2})
    ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    for (cudaEvent_t e : {l->fork, l->join, l->aux, l->aux2})
      if (e) cudaEventDestroy(e);
    if (l->st) cudaStreamDestroy(l->st);
    delete l;
    return GPTQ_ERR_CUDA;
  }
  *out = l;
  return GPTQ_OK;
}

}  // namespace

LaneLease::~LaneLease() {
  for (auto& [l, prio] : lanes_) {
    cudaEventRecord(l->join, l->st);
    cudaStreamWaitEvent(s_, l->join, 0);
  }
  std::lock_guard<std::mutex> lk(g_lane_mu);
  for (auto& [l, prio] : lanes_) g_lane_free[{dev_, prio}].push_back(l);
}

int LaneLease::acquire(int count, const LanePrio* prio) {
  if (cudaGetDevice(&dev_) != cudaSuccess) return GPTQ_ERR_CUDA;
  for (int i = 0; i < count; ++i) {
    Lane* l = nullptr;
    {
      // Only a lane whose previous lease has drained: a lane handed back by a call that the
      // host has finished issuing may still hold queued work, and this lease's work would
      // wait behind it (correct, but two concurrent users of the library would run one
      // after the other).  Without an idle lane, a new one is created.
      std::lock_guard<std::mutex> lk(g_lane_mu);
      auto& v = g_lane_free[{dev_, static_cast<int>(prio[i])}];
      for (size_t k = v.size(); k-- > 0;) {
        const cudaError_t q = cudaEventQuery(v[k]->join);
        if (q == cudaSuccess) {
          l = v[k];
          v.erase(v.begin() + static_cast<std::ptrdiff_t>(k));
          break;
        }
        if (q == cudaErrorNotReady) cudaGetLastError();  // "not yet" is not an error: clear it
      }
    }
    if (!l) GPTQ_TRY(create_lane(prio[i], &l));
    lanes_.emplace_back(l, static_cast<int>(prio[i]));
    GPTQ_CUDA(cudaEventRecord(l->fork, s_));
    GPTQ_CUDA(cudaStreamWaitEvent(l->st, l->fork, 0));
  }
  return GPTQ_OK;
}

namespace {
std::mutex g_attr_mu;
std::map<std::pair<int, const void*>, int> g_attr_set;  // (device, kernel) -> limit set so far
}  // namespace

int ensure_smem_limit(const void* kernel, int bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  auto it = g_attr_set.find({dev, kernel});
  if (it != g_attr_set.end() && it->second >= bytes) return GPTQ_OK;  // already high enough
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
    cudaGetLastError();
    return GPTQ_ERR_CUDA;
  }
  g_attr_set[{dev, kernel}] = bytes;
  return GPTQ_OK;
}

}  // namespace gptq
