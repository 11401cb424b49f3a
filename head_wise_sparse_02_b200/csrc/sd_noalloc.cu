// Fixed device scratch for sparse_decode_attend_noalloc.
//
// The attend launch needs a workspace (per-chunk partial results, the union
// lists of the plan step, the item layout and a few counters).  The regular
// entry point takes it from the caller; the allocation-free one takes it from
// the file-scope array below, which the CUDA runtime places on each device when
// this module is loaded there.  Nothing here allocates: the array's address is
// looked up once per device (with that device current) and cached.
#include <map>
#include <mutex>

#include "sd_internal.cuh"

namespace sd {

namespace {
static __device__ __align__(256) unsigned char g_attend_scratch[kNoAllocScratchBytes];
}  // namespace

cudaError_t noalloc_scratch(void **ptr) {
  static std::mutex mu;
  static std::map<int, void *> addr;                 // device -> scratch address
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  auto it = addr.find(dev);
  if (it == addr.end()) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attend_scratch);
    if (e != cudaSuccess) return e;
    it = addr.emplace(dev, p).first;
  }
  *ptr = it->second;
  return cudaSuccess;
}

}  // namespace sd
