// Internal declarations of the sparse decode library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sparse_decode.h"

namespace sd {

constexpr int kMaxGroup = 16;     // q heads per KV head (GQA group) supported
constexpr int kIndexDim = 16;     // r
constexpr int kPage = 16;         // tokens per page

// One KV head's heads of one role (retrieval or local).
struct Group {
  int kv_head;
  int n;                          // heads of this role in the group
  int q_head[kMaxGroup];          // their q-head ids, ascending
  int row[kMaxGroup];             // retrieval: row in sel_idx (rank among retrieval heads)
};

// Device-side view of a context's tables.
struct Tables {
  const Group *ret;               // [n_ret] groups with >= 1 retrieval head
  const Group *loc;               // [n_loc] groups with >= 1 local head
  int n_ret, n_loc;
  int max_ret;                    // largest n over ret groups
  int max_loc;                    // largest n over loc groups
};

struct Shape {
  int Hq, Hkv, d, num_pages, max_pages, H_ret;
  long long max_len;              // max_pages * kPage
};

// ----------------------------------------------------------------- helpers

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// Order-preserving map of a float to an unsigned key (-0 folded onto +0).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(__fadd_rn(f, 0.0f));
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// float64 -> bf16 bits, round to nearest even, from the float64 value itself
// (never through float32).  bf16 keeps 8 significant bits and float32's
// exponent range; the quantum of a value in [2^(e-1), 2^e) is 2^(e-8), with
// the subnormal floor 2^-133.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  if (isnan(x)) return 0x7FC0u;
  const uint16_t sign = (__double_as_longlong(x) < 0) ? 0x8000u : 0u;
  const double a = fabs(x);
  if (a == 0.0) return sign;
  int e;
  frexp(a, &e);                                  // a = m * 2^e, 0.5 <= m < 1
  const int q = max(e - 8, -133);
  const double r = rint(ldexp(a, -q));           // exact scaling, ties to even
  const float y = (float)ldexp(r, q);            // exactly representable, or +inf on overflow
  return sign | (uint16_t)(__float_as_uint(y) >> 16);
}

__device__ __forceinline__ void raise_error(unsigned *err, unsigned bit) {
  if (err) atomicOr(err, bit);
}

// ------------------------------------------------ programmatic dependent launch
// Every kernel of the library is launched with programmatic stream
// serialization (launch_pdl below): its CTAs may be scheduled while the
// previous kernel on the stream is still finishing.  Before its first access to
// memory that earlier work on the stream writes or reads (inputs, outputs,
// workspace), a kernel calls pdl_wait(), which returns once the previous grid
// has completed and its writes are visible; it may only read the library's own
// constant tables before that.  Every kernel calls pdl_wait() on every path,
// early returns included, so that completion stays ordered along the stream.
// pdl_trigger() lets the next kernel be scheduled before this one ends.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// L2 eviction priority of streamed data: cache rows and index pages are read
// once per call, so they are marked evict-first and leave the small tables,
// lists and code of the surrounding kernels in L2
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(p));
  return p;
}
// cudaLaunchKernelEx with programmatic stream serialization, plus an optional
// cluster shape (x CTAs per cluster; 0 = no cluster).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       int cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_x > 0) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error.

cudaError_t launch_index_keys(const uint16_t *k_pre, const int32_t *slots, int T, uint16_t *index_cache,
                              const uint16_t *proj, const Shape &sh, unsigned *err, cudaStream_t st);

struct SelectArgs {
  const uint16_t *q_pre;
  const uint16_t *index_cache;
  const int32_t *page_table;
  const int32_t *seq_lens;
  int32_t *sel_idx;
  int32_t *sel_count;
  long long sel_stride;
  const uint16_t *proj;
  float index_scale;
  int mode;
  float top_p;
  int top_k;
  float top_k_frac;
  float *score_ws;                // global score rows when they do not fit on chip
  uint32_t *flags;                // [batch * n_ret] streaming selection misses
  void *stream_ws;                // streaming selection scratch (histograms, buffers, bitmaps)
  unsigned *err;
  int batch;
  bool pre_scored;                // score_ws already holds every head's scores (exact-score mode)
};

size_t select_workspace_bytes(const Shape &sh, const Tables &tb, int batch, size_t *flags_off);
cudaError_t launch_select(const SelectArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st);
// Exact-score selection: score_ws rows := attn_scale * q . k for every
// retrieval head and cached token (then launch_select with pre_scored).
cudaError_t launch_exact_scores(const SelectArgs &a, const Shape &sh, const Tables &tb, const uint16_t *q,
                                const uint16_t *k_cache, float attn_scale, cudaStream_t st);
// Streaming selection (top-k and top-p): workspace bytes for a batch (0 when
// the shapes are outside what it handles), and its launches; *used = false
// when it did not run and the exact selector must take every item.
size_t stream_workspace_bytes(const Shape &sh, const Tables &tb, int batch, int mode);
cudaError_t launch_select_stream(const SelectArgs &a, const Shape &sh, const Tables &tb, uint32_t *fail,
                                 void *ws_base, cudaStream_t st, bool *used);

struct AttendArgs {
  const uint16_t *q;
  const uint16_t *k_cache;
  const uint16_t *v_cache;
  const int32_t *page_table;
  const int32_t *seq_lens;
  const int32_t *sel_idx;
  const int32_t *sel_count;
  long long sel_stride;
  float *out;
  float attn_scale;
  int window, num_sinks;
  void *ws;                       // attend's part of the workspace (partials, union lists, tickets)
  unsigned *err;
  int batch;
};

size_t attend_workspace_bytes(const Shape &sh, const Tables &tb, int batch);
cudaError_t launch_attend(const AttendArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st);

// Size of the built-in attend scratch of sparse_decode_attend_noalloc.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
// The current device's scratch address (looked up on every call).
cudaError_t noalloc_scratch(void **ptr);

}  // namespace sd
