// Host-side launch helpers shared by the library's translation units: the SM
// count, the dynamic shared-memory opt-in and occupancy figures, each looked
// up once per device and kept in a process-wide cache.
//
// Every cache is keyed by the device ordinal that is current on the calling
// thread and filled under a mutex, so host threads may call the library at
// the same time, and a kernel used on a second device gets its attribute set
// there too.  These are inline functions, so their static caches are shared
// by every translation unit of the library.
#pragma once

#include <cuda_runtime.h>

#include <mutex>
#include <vector>

namespace nvfp4 {
namespace host {

constexpr int kMaxDevices = 64;

inline std::mutex &cache_mutex() {
  static std::mutex mu;
  return mu;
}

// Ordinal of the current device, or -1.
inline int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

// SM count of the current device (148 on B200; 148 if the query fails).
inline int sm_count() {
  static int cache[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return 148;
  std::lock_guard<std::mutex> lock(cache_mutex());
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

// Opt `fn` in to `bytes` of dynamic shared memory on the current device, once
// per (device, kernel, size).  False if the runtime refuses.
inline bool set_max_dynamic_smem(const void *fn, int bytes) {
  struct Entry { int dev; const void *fn; int bytes; };
  static std::vector<Entry> done;
  const int dev = current_device();
  if (dev < 0) return false;
  std::lock_guard<std::mutex> lock(cache_mutex());
  for (const Entry &e : done)
    if (e.dev == dev && e.fn == fn && e.bytes >= bytes) return true;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done.push_back(Entry{dev, fn, bytes});
  return true;
}

// Resident blocks per SM of `fn` at this block size and dynamic shared memory
// on the current device (at least 1).
inline int blocks_per_sm(const void *fn, int threads, size_t smem) {
  struct Entry { int dev; const void *fn; int threads; size_t smem; int per_sm; };
  static std::vector<Entry> seen;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(cache_mutex());
  for (const Entry &e : seen)
    if (e.dev == dev && e.fn == fn && e.threads == threads && e.smem == smem) return e.per_sm;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, threads, smem) != cudaSuccess || per_sm < 1) {
    (void)cudaGetLastError();
    per_sm = 1;
  }
  seen.push_back(Entry{dev, fn, threads, smem, per_sm});
  return per_sm;
}

}  // namespace host
}  // namespace nvfp4
