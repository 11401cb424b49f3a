// Fixed device scratch for sparse_decode_attend_noalloc.
//
// The attend launch needs a workspace (per-chunk partial results, the union
// lists of the plan step, the item layout and the merge tickets).  The regular
// entry point takes it from the caller; the allocation-free one takes it from
// the file-scope array below, which the CUDA runtime places on each device when
// this module is loaded there.  Nothing here allocates.  In host code the
// array's name is only a host-side stand-in, so the device address is looked
// up with cudaGetSymbolAddress, with the caller's device current, on every call:
// the lookup is cheap, and an address cached across calls would go stale if the
// device were reset in between.
#include "sd_internal.cuh"

namespace sd {

namespace {
static __device__ __align__(256) unsigned char g_attend_scratch[kNoAllocScratchBytes];
}  // namespace

cudaError_t noalloc_scratch(void **ptr) {
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_attend_scratch);
  if (e != cudaSuccess) return e;
  *ptr = p;
  return cudaSuccess;
}

}  // namespace sd
