// fa_runtime.cu -- per-device launch facts, looked up once and reused by every call.
//
// A decode step of a small batch runs in a few microseconds on the device, so host work per
// call (device attribute queries, raising a kernel's shared-memory limit, occupancy
// queries) would decide its rate. These helpers do each query once per (device, kernel,
// size) under a mutex and answer later calls from a table.
#include <mutex>

#include "fa_host.h"

namespace fa {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxEntries = 256;

struct SmemEntry {
  const void* func;
  int dev, limit;
};
struct OccEntry {
  const void* func;
  int dev, threads;
  size_t smem;
  int blocks;
};

std::mutex g_mu;
int g_sms[kMaxDevices] = {};
SmemEntry g_smem[kMaxEntries];
int g_n_smem = 0;
OccEntry g_occ[kMaxEntries];
int g_n_occ = 0, g_occ_next = 0;

cudaError_t device_index(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return e;
  return (*dev >= 0 && *dev < kMaxDevices) ? cudaSuccess : cudaErrorInvalidDevice;
}

}  // namespace

cudaError_t device_sm_count(int* sms) {
  int dev = 0;
  cudaError_t e = device_index(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sms[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_sms[dev] = n;
  }
  *sms = g_sms[dev];
  return cudaSuccess;
}

cudaError_t raise_smem_limit(const void* func, int bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;  // the default limit
  int dev = 0;
  cudaError_t e = device_index(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_n_smem; ++i) {
    SmemEntry& s = g_smem[i];
    if (s.func == func && s.dev == dev) {
      if (s.limit >= bytes) return cudaSuccess;
      e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e == cudaSuccess) s.limit = bytes;
      return e;
    }
  }
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (g_n_smem < kMaxEntries) g_smem[g_n_smem++] = SmemEntry{func, dev, bytes};
  return cudaSuccess;
}

cudaError_t cached_occupancy(const void* func, int threads, size_t smem, int* blocks) {
  int dev = 0;
  cudaError_t e = device_index(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_n_occ; ++i) {
      const OccEntry& o = g_occ[i];
      if (o.func == func && o.dev == dev && o.threads == threads && o.smem == smem) {
        *blocks = o.blocks;
        return cudaSuccess;
      }
    }
  }
  if ((e = raise_smem_limit(func, (int)smem)) != cudaSuccess) return e;
  int n = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  const int slot = g_n_occ < kMaxEntries ? g_n_occ++ : (g_occ_next++ % kMaxEntries);
  g_occ[slot] = OccEntry{func, dev, threads, smem, n};
  *blocks = n;
  return cudaSuccess;
}

cudaError_t cached_max_clusters(const void* func, int threads, size_t smem, int cluster, int* n) {
  int dev = 0;
  cudaError_t e = device_index(&dev);
  if (e != cudaSuccess) return e;
  // keyed like the occupancy table, with the cluster size in the thread count's high bits
  const int key_threads = threads | (cluster << 16);
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_n_occ; ++i) {
      const OccEntry& o = g_occ[i];
      if (o.func == func && o.dev == dev && o.threads == key_threads && o.smem == smem) {
        *n = o.blocks;
        return cudaSuccess;
      }
    }
  }
  if ((e = raise_smem_limit(func, (int)smem)) != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cluster, 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int c = 0;
  e = cudaOccupancyMaxActiveClusters(&c, func, &cfg);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  const int slot = g_n_occ < kMaxEntries ? g_n_occ++ : (g_occ_next++ % kMaxEntries);
  g_occ[slot] = OccEntry{func, dev, key_threads, smem, c};
  *n = c;
  return cudaSuccess;
}

}  // namespace fa
