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

// Launch as thread-block clusters of `cluster_x` CTAs (plus programmatic
// stream serialisation).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                           Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
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
