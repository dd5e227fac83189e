// Tiered expert pool: the routed experts of one layer live as expert blocks in pinned host memory (the
// pages' SSD tier), and an HBM cache of a fixed number of slots (their RAM tier) holds the blocks in use.
// Host-side runtime: residency map, least-recently-used replacement, the host-to-device copies, and the
// ordering of the copies against the kernels that read the slots (CUDA events).  On the device, only the
// remap of a call's expert ids to slot ids runs; the expert forward then runs unchanged over the slot pool.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <vector>

#include "../../include/moe.h"
#include "common.cuh"

namespace moe {
namespace tier {

constexpr int kMaxExperts = 256;

struct Table {
  int32_t slot[kMaxExperts];  // expert -> slot (-1: not resident)
};

// idx_slot[i] = slot of expert idx[i] (expert ids clamped into [0, E) as the forward clamps them); an expert
// that is not resident reports MOE_ERR_INVALID_ARG in err and maps to slot 0.
__global__ void remap_kernel(const int32_t* __restrict__ idx, int n, const __grid_constant__ Table tab, int E,
                             int32_t* __restrict__ idx_slot, int* err) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    int e = idx[i];
    e = e < 0 ? 0 : (e >= E ? E - 1 : e);
    const int s = tab.slot[e];
    if (s < 0) report(err, MOE_ERR_INVALID_ARG);
    idx_slot[i] = s < 0 ? 0 : s;
  }
}

struct Tier {
  const uint8_t* host = nullptr;
  int64_t host_stride = 0;
  int E = 0;
  int64_t bytes = 0;
  uint8_t* slots = nullptr;
  int64_t slot_stride = 0;
  int S = 0;
  std::vector<int32_t> slot_of;     // [E]
  std::vector<int32_t> expert_in;   // [S] (-1: free)
  std::vector<uint64_t> last_use;   // [S] tick of the last acquire or prefetch that wanted the slot's expert
  std::vector<uint8_t> prefetched;  // [S] filled by a prefetch and not acquired since
  uint64_t tick = 0;
  cudaEvent_t use_ev = nullptr;  // recorded by release: the slots' readers so far
  cudaEvent_t pf_ev = nullptr;   // recorded by prefetch: its copies
  bool use_recorded = false, pf_pending = false;
  moe_tier_stats st{};
  std::mutex mu;

  // The distinct experts of a list, clamped into [0, E), in first-seen order.
  std::vector<int32_t> distinct(const int32_t* experts, int n) const {
    std::vector<int32_t> d;
    std::vector<uint8_t> seen(E, 0);
    for (int i = 0; i < n; ++i) {
      int e = experts[i];
      e = e < 0 ? 0 : (e >= E ? E - 1 : e);
      if (!seen[e]) {
        seen[e] = 1;
        d.push_back(e);
      }
    }
    return d;
  }

  uint64_t acq_tick = 0;  // tick of the last acquire

  // A slot to reuse: a free one if any, else the least recently used one last wanted before `limit`.
  int victim(uint64_t limit) const {
    int best = -1;
    for (int s = 0; s < S; ++s) {
      if (expert_in[s] < 0) return s;
      if (last_use[s] < limit && (best < 0 || last_use[s] < last_use[best])) best = s;
    }
    return best;
  }

  bool place(int e, int s, cudaStream_t stream) {
    if (expert_in[s] >= 0) slot_of[expert_in[s]] = -1;
    if (cudaMemcpyAsync(slots + s * slot_stride, host + e * host_stride, static_cast<size_t>(bytes),
                        cudaMemcpyHostToDevice, stream) != cudaSuccess)
      return false;
    expert_in[s] = e;
    slot_of[e] = s;
    last_use[s] = tick;
    return true;
  }
};

}  // namespace tier
}  // namespace moe
