// Host-side launch helpers shared by the translation units of the library.
#pragma once

#include <atomic>
#include <cstdlib>
#include <map>
#include <mutex>

#include <cuda_runtime.h>

namespace dv {

inline std::atomic<uint64_t> g_launches{0};

inline bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DV_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

// Every kernel asks for the largest shared-memory carveout, so that CTAs of
// different kernels (consecutive ones overlapping under programmatic launch,
// and the two streams of the look-ahead) can share an SM without the SM
// having to drain and reconfigure its L1 / shared split. Cached per kernel.
inline std::mutex g_carve_mu;
inline std::map<std::pair<const void*, int>, bool> g_carve_set;

template <typename K>
void prefer_max_shared(K kern) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kern), dev);
  std::lock_guard<std::mutex> lock(g_carve_mu);
  if (g_carve_set.count(key)) return;
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  g_carve_set[key] = true;
}

// Launch with programmatic stream serialisation, so a kernel's launch and
// prologue overlap the tail of the previous kernel on the stream.
template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  prefer_max_shared(kern);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// The highest scheduling priority of the device, given to the kernels of the
// layer's critical path (Q/K/V, attention + W^O, MLP) so that, when the
// look-ahead predictor's kernels on the side streams compete for SMs, the
// critical-path CTAs are placed first. DV_PRIO=0 turns it off. Cached per
// device.
inline int main_priority() {
  static const bool on = [] {
    const char* e = std::getenv("DV_PRIO");
    return !(e && e[0] == '0');
  }();
  if (!on) return 0;
  static int prio[64];
  static bool have[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!have[dev]) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) greatest = 0;
    prio[dev] = greatest;
    have[dev] = true;
  }
  return prio[dev];
}

// launch() with the critical-path priority.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_main(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                               Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributePriority;
  attr[n].val.priority = main_priority();
  ++n;
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  prefer_max_shared(kern);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Launch as thread-block clusters of `cluster_x` CTAs (plus programmatic
// stream serialisation), with the critical-path priority.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                           Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributePriority;
  attr[1].val.priority = main_priority();
  attr[2].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[2].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 3 : 2;
  prefer_max_shared(kern);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Raises a kernel's dynamic shared memory limit to `bytes` when needed (the
// default 48 KB covers static plus dynamic). Cached per kernel and device.
inline std::mutex g_smem_mu;
struct SmemKey {
  const void* fn;
  int dev;
  bool operator<(const SmemKey& o) const { return fn < o.fn || (fn == o.fn && dev < o.dev); }
};
inline std::map<SmemKey, size_t> g_smem_set;

template <typename K>
inline cudaError_t allow_smem(K kern, size_t bytes) {
  if (bytes == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const SmemKey key{reinterpret_cast<const void*>(kern), dev};
  std::lock_guard<std::mutex> lock(g_smem_mu);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) g_smem_set[key] = bytes;
  return e;
}

inline int sm_count() {
  static int n = [] {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
  }();
  return n;
}

// CTAs of the batch-1 neuron-score kernel (predict_b_kernel, one row per
// warp): four per SM unless DV_PB_CTAS gives the count.
inline int pb_ctas() {
  static const int n = [] {
    const char* e = std::getenv("DV_PB_CTAS");
    return e ? std::atoi(e) : 0;
  }();
  return n > 0 ? n : 4 * sm_count();
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
inline bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

inline int nb_bucket(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16; }

// RPW rows per warp and U column steps so that RPW * U = 8 loads per lane.
inline int rpw_for(int K, int E) {
  const int vpl = (K / E + 31) / 32;
  return vpl >= 8 ? 1 : vpl >= 4 ? 2 : vpl >= 2 ? 4 : 8;
}

}  // namespace dv
