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

// Bit position of the n-th set bit (0-based) of v, n < popc(v): binary
// search over halves by population count.
__device__ __forceinline__ int nth_set_bit(uint32_t v, int n) {
  int pos = 0;
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) {
    const uint32_t low = v & ((1u << s) - 1u);
    const int c = __popc(low);
    if (n >= c) {
      n -= c;
      v >>= s;
      pos += s;
    } else {
      v = low;
    }
  }
  return pos;
}

// One warp, 32 consecutive bitmap words (word x0 + lane in `bits`): the set
// bits in ascending order are handed out 32 at a time, lane l taking the
// (r + l)-th one, so that whatever a caller stores per bit goes out in
// coalesced rows.  Every lane calls emit(valid, k, w, bit) in every round (so
// that emit may shuffle); when valid, k in [0, total) is the rank of the set
// bit it hands out, found in the word of lane w at bit position `bit`.
// Returns the number of set bits of the 32 words.
template <typename Emit>
__device__ __forceinline__ int warp_emit_bits(uint32_t bits, int lane, Emit &&emit) {
  const unsigned full = 0xFFFFFFFFu;
  const int n = __popc(bits);
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(full, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(full, incl, 31);
  for (int r = 0; r < total; r += 32) {
    const int k = r + lane;
    // the word holding set bit k: the first lane whose inclusive count exceeds k
    int w = 0;
#pragma unroll
    for (int st = 16; st > 0; st >>= 1) {
      const int c = __shfl_sync(full, incl, w + st - 1);
      if (c <= k) w += st;
    }
    const uint32_t wb = __shfl_sync(full, bits, w);
    const int before = __shfl_sync(full, incl - n, w);
    emit(k < total, k, w, nth_set_bit(wb, k - before));
  }
  return total;
}

// warp_emit_bits over W consecutive words per lane (lane l holds words
// W l .. W l + W - 1 of a run of 32 W): fewer, longer steps for sparse bitmaps.
// emit(valid, k, w, j, bit): set bit k of the run lies in word j of lane w.
template <int W, typename Emit>
__device__ __forceinline__ int warp_emit_bits_w(const uint32_t (&bits)[W], int lane, Emit &&emit) {
  const unsigned full = 0xFFFFFFFFu;
  int n = 0;
#pragma unroll
  for (int j = 0; j < W; ++j) n += __popc(bits[j]);
  int incl = n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(full, incl, o);
    if (lane >= o) incl += y;
  }
  const int total = __shfl_sync(full, incl, 31);
  for (int r = 0; r < total; r += 32) {
    const int k = r + lane;
    int w = 0;
#pragma unroll
    for (int st = 16; st > 0; st >>= 1) {
      const int c = __shfl_sync(full, incl, w + st - 1);
      if (c <= k) w += st;
    }
    int rank = k - __shfl_sync(full, incl - n, w);    // rank of the bit among lane w's words
    uint32_t word = 0;
    int jw = 0;
#pragma unroll
    for (int j = 0; j < W; ++j) {
      const uint32_t b = __shfl_sync(full, bits[j], w);
      const int c = __popc(b);
      if (jw == j && rank >= c && j + 1 < W) {
        rank -= c;
        jw = j + 1;
      } else if (jw == j) {
        word = b;
      }
    }
    emit(k < total, k, w, jw, nth_set_bit(word, rank));
  }
  return total;
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

// Where a fused select writes the union lists that attend reads: the plan
// arrays of attend's workspace (union rows of (sequence, retrieval group,
// span of positions): cache row and head mask of each, their count).
struct UnionOut {
  uint32_t *row;                  // [B][n_ret][ns][span]
  uint16_t *mask;                 // [B][n_ret][ns][span]
  int *cnt;                       // [B][n_ret][ns]
  int span, ns;
  bool ret_only;                  // rows address caches of the retrieval groups only
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
// With `uo` (not null) the last pass also builds attend's union lists (one CTA
// per (sequence, retrieval group)) when the shapes allow it; *unioned tells.
cudaError_t launch_select_stream(const SelectArgs &a, const Shape &sh, const Tables &tb, uint32_t *fail,
                                 void *ws_base, cudaStream_t st, bool *used, const UnionOut *uo = nullptr,
                                 bool *unioned = nullptr);
// launch_select with the union lists built by the streaming pass where it can
// (*unioned); the items it flags (exact selector) are left for attend's plan.
cudaError_t launch_select_union(const SelectArgs &a, const Shape &sh, const Tables &tb, const UnionOut &uo,
                                cudaStream_t st, bool *unioned);

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
  // split layout: the paged caches hold only the retrieval KV groups (in
  // ascending KV-head order) and the local groups read the compacted caches
  // local_k / local_v [B][n_loc][num_sinks + window][d]
  bool split;
  const uint16_t *local_k;
  const uint16_t *local_v;
};

// Slot of position `pos` in a compacted local-head cache: sinks first, then a
// ring of `window` slots; -1 when the position is kept nowhere (no window).
__host__ __device__ __forceinline__ long long local_slot(long long pos, int num_sinks, int window) {
  if (pos < num_sinks) return pos;
  return window > 0 ? num_sinks + pos % window : -1;
}

cudaError_t launch_prefill(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *page_table, const int32_t *seq_lens, const int32_t *q_starts, int batch,
                           int total_q, float *out, float attn_scale, int window, int num_sinks, const Shape &sh,
                           const Tables &tb, unsigned *err, cudaStream_t st);

cudaError_t launch_prefill_tc(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                              const int32_t *page_table, const int32_t *seq_lens, const int32_t *q_starts, int batch,
                              int total_q, float *out, float attn_scale, int window, int num_sinks, const Shape &sh,
                              const Tables &tb, unsigned *err, cudaStream_t st);

cudaError_t launch_local_append(const uint16_t *k_new, const uint16_t *v_new, const int32_t *seq_ids,
                                const int32_t *positions, int T, uint16_t *local_k, uint16_t *local_v,
                                const Shape &sh, const Tables &tb, int max_batch, int num_sinks, int window,
                                unsigned *err, cudaStream_t st);

size_t attend_workspace_bytes(const Shape &sh, const Tables &tb, int batch);
// plan_only: null = plan every retrieval item; else the select's miss array
// ([items] flags, count, list): only the listed items are planned, the
// others' union lists are already in the workspace.
cudaError_t launch_attend(const AttendArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st,
                          const uint32_t *plan_only = nullptr);
UnionOut attend_union_view(const Shape &sh, const Tables &tb, int batch, void *attend_ws, bool ret_only);

// Size of the built-in attend scratch of sparse_decode_attend_noalloc.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
// The current device's scratch address (looked up on every call).
cudaError_t noalloc_scratch(void **ptr);

}  // namespace sd
