// C ABI of the sparse decode library: argument validation, the context, the
// workspace layout and the launches.  See include/sparse_decode.h.
#include <atomic>
#include <math.h>
#include <stdio.h>

#include <memory>
#include <string>
#include <vector>

#include "sd_internal.cuh"

namespace sd {
extern std::atomic<int> g_prefill_stall;      // sd_prefill_tc.cu: testing switch of the d = 128 prefill
}

struct sd_ctx {
  sd_config cfg;                      // head_is_retrieval points into `retr`
  std::vector<int32_t> retr;
  int device = 0;
  sd::Shape sh{};
  sd::Tables tb{};                    // device pointers
  std::vector<sd::Group> ret_h, loc_h;
  sd::Group *groups_d = nullptr;      // ret groups then loc groups
  uint16_t *proj_d = nullptr;
  unsigned *err_d = nullptr;
  float attn_scale = 0.f, index_scale = 0.f;
  std::string last_error;
};

namespace {

struct DeviceGuard {
  int prev = -1;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && prev != dev) cudaSetDevice(dev);
    else prev = -1;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

sd_status fail(sd_ctx *ctx, sd_status s, const std::string &msg) {
  if (ctx) ctx->last_error = msg;
  return s;
}

sd_status cuda_fail(sd_ctx *ctx, cudaError_t e, const char *what) {
  return fail(ctx, SD_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Caches, keys and queries are read with 16-byte vector and asynchronous
// copies: their base addresses must be 16-byte aligned.
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0u; }

struct WsLayout {
  size_t scores_off, flags_off, scores_bytes, stream_off, stream_bytes, att_off, total;
};

WsLayout layout(const sd_ctx *ctx, int batch) {
  WsLayout w{};
  w.scores_off = 0;
  size_t foff = 0;
  w.scores_bytes = align256(sd::select_workspace_bytes(ctx->sh, ctx->tb, batch, &foff));
  w.flags_off = w.scores_off + foff;
  w.stream_off = w.scores_off + w.scores_bytes;
  w.stream_bytes = align256(sd::stream_workspace_bytes(ctx->sh, ctx->tb, batch, ctx->cfg.mode));
  w.att_off = w.stream_off + w.stream_bytes;
  w.total = align256(w.att_off + sd::attend_workspace_bytes(ctx->sh, ctx->tb, batch));
  return w;
}

long long max_topk(const sd_ctx *ctx) {
  const long long L = ctx->sh.max_len;
  long long k = ctx->cfg.top_k > 0 ? (long long)ctx->cfg.top_k
                                   : std::max(1LL, (long long)floor((double)ctx->cfg.top_k_frac * (double)L));
  return std::min(k, L);
}

// Rows per (sequence, local KV group) of a compacted local cache.
long long local_rows(const sd_ctx *ctx) { return (long long)ctx->cfg.num_sinks + ctx->cfg.window; }

// attend, alone (joined = false) or after the selection of the same sets
// (joined = true), on the full paged caches (split = false) or on caches of the
// retrieval groups plus compacted local caches (split = true)
sd_status attend_impl(sd_ctx *ctx, const void *q_pre, const void *q, const void *index_cache, const void *k_cache,
                      const void *v_cache, const void *local_k, const void *local_v, const int32_t *page_table,
                      const int32_t *seq_lens, int batch, int32_t *sel_idx, int32_t *sel_count, int sel_stride,
                      float *out, void *workspace, size_t ws_bytes, sd_stream stream, bool joined, bool split) {
  if (!ctx) return SD_ERR_INVALID_ARG;
  if (batch < 0 || batch > ctx->cfg.max_batch) return fail(ctx, SD_ERR_INVALID_ARG, "batch out of range");
  if (batch == 0) return SD_OK;
  const bool ret = ctx->sh.H_ret > 0;
  if (!q || !page_table || !seq_lens || !out) return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
  // with the split layout, caches of a kind of head that is absent may be NULL
  const bool need_paged = !split || ret;
  const bool need_local = split && ctx->tb.n_loc > 0 && local_rows(ctx) > 0;
  if (need_paged && (!k_cache || !v_cache)) return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
  if (need_local && (!local_k || !local_v)) return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || (need_paged && (!aligned16(k_cache) || !aligned16(v_cache))) ||
      (need_local && (!aligned16(local_k) || !aligned16(local_v))))
    return fail(ctx, SD_ERR_INVALID_ARG, "q and the K/V caches must be 16-byte aligned");
  // local cache rows are addressed with 32-bit row numbers inside the kernels
  if (need_local && (long long)batch * ctx->tb.n_loc * local_rows(ctx) >= 0xFFFFFFFFLL)
    return fail(ctx, SD_ERR_UNSUPPORTED, "local caches too large for 32-bit row numbers");
  if (ret) {
    if (!sel_idx || !sel_count) return fail(ctx, SD_ERR_INVALID_ARG, "selection lists required for retrieval heads");
    if (joined) {
      if (!q_pre || !index_cache) return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
      if (!aligned16(q_pre) || !aligned16(index_cache))
        return fail(ctx, SD_ERR_INVALID_ARG, "q_pre and index_cache must be 16-byte aligned");
      const long long need_stride = ctx->cfg.mode == SD_TOP_P ? ctx->sh.max_len : max_topk(ctx);
      if (sel_stride < need_stride)
        return fail(ctx, SD_ERR_INVALID_ARG, "sel_stride smaller than the largest possible set");
    } else if (sel_stride <= 0) {
      return fail(ctx, SD_ERR_INVALID_ARG, "selection lists required for retrieval heads");
    }
  }
  const WsLayout w = layout(ctx, batch);
  if (!workspace || ws_bytes < w.total) return fail(ctx, SD_ERR_WORKSPACE, "workspace too small");
  DeviceGuard dg(ctx->device);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *wsb = static_cast<char *>(workspace);
  bool unioned = false;
  if (joined && ret) {
    sd::SelectArgs a{};
    a.q_pre = static_cast<const uint16_t *>(q_pre);
    a.index_cache = static_cast<const uint16_t *>(index_cache);
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.sel_stride = sel_stride;
    a.proj = ctx->proj_d;
    a.index_scale = ctx->index_scale;
    a.mode = ctx->cfg.mode;
    a.top_p = ctx->cfg.top_p;
    a.top_k = ctx->cfg.top_k;
    a.top_k_frac = ctx->cfg.top_k_frac;
    a.score_ws = reinterpret_cast<float *>(wsb + w.scores_off);
    a.flags = reinterpret_cast<uint32_t *>(wsb + w.flags_off);
    a.stream_ws = w.stream_bytes ? wsb + w.stream_off : nullptr;
    a.err = ctx->err_d;
    a.batch = batch;
    const sd::UnionOut uo = sd::attend_union_view(ctx->sh, ctx->tb, batch, wsb + w.att_off, split);
    const cudaError_t e = sd::launch_select_union(a, ctx->sh, ctx->tb, uo, st, &unioned);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "select launch");
  }
  sd::AttendArgs at{};
  at.q = static_cast<const uint16_t *>(q);
  at.k_cache = static_cast<const uint16_t *>(k_cache);
  at.v_cache = static_cast<const uint16_t *>(v_cache);
  at.page_table = page_table;
  at.seq_lens = seq_lens;
  at.sel_idx = sel_idx;
  at.sel_count = sel_count;
  at.sel_stride = sel_stride;
  at.out = out;
  at.attn_scale = ctx->attn_scale;
  at.window = ctx->cfg.window;
  at.num_sinks = ctx->cfg.num_sinks;
  at.ws = wsb + w.att_off;
  at.err = ctx->err_d;
  at.batch = batch;
  at.split = split;
  at.local_k = static_cast<const uint16_t *>(local_k);
  at.local_v = static_cast<const uint16_t *>(local_v);
  // with the union lists built by select, attend plans only the items the
  // exact selector redid (listed in the miss array)
  const uint32_t *only = unioned ? reinterpret_cast<const uint32_t *>(wsb + w.flags_off) : nullptr;
  const cudaError_t e = sd::launch_attend(at, ctx->sh, ctx->tb, st, only);
  return e == cudaSuccess ? SD_OK : cuda_fail(ctx, e, "attend launch");
}

}  // namespace

extern "C" {

const char *sparse_decode_status_string(sd_status s) {
  switch (s) {
    case SD_OK: return "ok";
    case SD_ERR_INVALID_ARG: return "invalid argument";
    case SD_ERR_UNSUPPORTED: return "unsupported configuration";
    case SD_ERR_WORKSPACE: return "workspace missing or too small";
    case SD_ERR_CUDA: return "CUDA error";
    case SD_ERR_TIMEOUT: return "device-side wait timed out";
    case SD_ERR_DEVICE_DATA: return "device-side check rejected input data";
    case SD_ERR_HOST_MEMORY: return "host allocation failed";
  }
  return "unknown status";
}

const char *sparse_decode_last_error(const sd_ctx *ctx) { return ctx ? ctx->last_error.c_str() : ""; }

int sparse_decode_num_retrieval_heads(const sd_ctx *ctx) { return ctx ? ctx->sh.H_ret : 0; }

sd_status sparse_decode_init(const sd_config *cfg, const void *proj, sd_ctx **out) {
  try {
    if (!out) return SD_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg || !proj || !cfg->head_is_retrieval) return SD_ERR_INVALID_ARG;
    const sd_config &c = *cfg;
    if (c.num_q_heads <= 0 || c.num_kv_heads <= 0 || c.num_q_heads % c.num_kv_heads != 0)
      return SD_ERR_INVALID_ARG;
    if (c.num_q_heads / c.num_kv_heads > sd::kMaxGroup) return SD_ERR_UNSUPPORTED;
    if (c.head_dim != 64 && c.head_dim != 128) return SD_ERR_UNSUPPORTED;
    if (c.index_dim != sd::kIndexDim || c.page_size != sd::kPage) return SD_ERR_UNSUPPORTED;
    if (c.num_pages <= 0 || c.max_batch <= 0 || c.max_pages_per_seq <= 0) return SD_ERR_INVALID_ARG;
    if ((long long)c.max_pages_per_seq * sd::kPage > (1LL << 25)) return SD_ERR_UNSUPPORTED;
    // cache rows are addressed with 32-bit row numbers inside the kernels
    if ((long long)c.num_pages * c.num_kv_heads * sd::kPage >= 0xFFFFFFFFLL) return SD_ERR_UNSUPPORTED;
    if (c.window < 0 || c.num_sinks < 0) return SD_ERR_INVALID_ARG;
    if (c.mode != SD_TOP_P && c.mode != SD_TOP_K) return SD_ERR_INVALID_ARG;
    if (c.mode == SD_TOP_P && !(c.top_p > 0.0f && c.top_p <= 1.0f)) return SD_ERR_INVALID_ARG;
    if (c.mode == SD_TOP_K) {
      if (c.top_k < 0) return SD_ERR_INVALID_ARG;
      if (c.top_k == 0 && !(c.top_k_frac > 0.0f && c.top_k_frac <= 1.0f)) return SD_ERR_INVALID_ARG;
    }
    for (int h = 0; h < c.num_q_heads; ++h)
      if (c.head_is_retrieval[h] != 0 && c.head_is_retrieval[h] != 1) return SD_ERR_INVALID_ARG;

    std::unique_ptr<sd_ctx> holder(new sd_ctx());
    sd_ctx *ctx = holder.get();
    ctx->cfg = c;
    ctx->retr.assign(c.head_is_retrieval, c.head_is_retrieval + c.num_q_heads);
    ctx->cfg.head_is_retrieval = ctx->retr.data();
    cudaGetDevice(&ctx->device);
    const int Hq = c.num_q_heads, Hkv = c.num_kv_heads, G = Hq / Hkv;
    int hr = 0;
    for (int g = 0; g < Hkv; ++g) {
      sd::Group r{}, l{};
      r.kv_head = l.kv_head = g;
      for (int j = 0; j < G; ++j) {
        const int h = g * G + j;
        if (ctx->retr[h]) {
          r.q_head[r.n] = h;
          r.row[r.n] = hr++;
          r.n++;
        } else {
          l.q_head[l.n] = h;
          l.row[l.n] = -1;
          l.n++;
        }
      }
      if (r.n) ctx->ret_h.push_back(r);
      if (l.n) ctx->loc_h.push_back(l);
    }
    ctx->sh.Hq = Hq;
    ctx->sh.Hkv = Hkv;
    ctx->sh.d = c.head_dim;
    ctx->sh.num_pages = c.num_pages;
    ctx->sh.max_pages = c.max_pages_per_seq;
    ctx->sh.H_ret = hr;
    ctx->sh.max_len = (long long)c.max_pages_per_seq * sd::kPage;
    ctx->attn_scale = c.attn_scale > 0.f ? c.attn_scale : (float)(1.0 / sqrt((double)c.head_dim));
    ctx->index_scale = c.index_scale > 0.f ? c.index_scale : (float)(sqrt((double)c.head_dim) / sd::kIndexDim);

    // every host allocation happens before the first device one, so a failed
    // host allocation (caught below) leaves no device memory behind
    const size_t ng = ctx->ret_h.size() + ctx->loc_h.size();
    const size_t proj_bytes = (size_t)Hkv * c.head_dim * sd::kIndexDim * sizeof(uint16_t);
    std::vector<sd::Group> all(ctx->ret_h);
    all.insert(all.end(), ctx->loc_h.begin(), ctx->loc_h.end());
    cudaError_t e = cudaMalloc(&ctx->groups_d, ng * sizeof(sd::Group));
    if (e == cudaSuccess) e = cudaMalloc(&ctx->proj_d, proj_bytes);
    if (e == cudaSuccess) e = cudaMalloc(&ctx->err_d, sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemcpy(ctx->groups_d, all.data(), ng * sizeof(sd::Group), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(ctx->proj_d, proj, proj_bytes, cudaMemcpyDefault);
    if (e == cudaSuccess) e = cudaMemset(ctx->err_d, 0, sizeof(unsigned));
    if (e != cudaSuccess) {
      sparse_decode_destroy(holder.release());
      return SD_ERR_CUDA;
    }
    ctx->tb.ret = ctx->groups_d;
    ctx->tb.loc = ctx->groups_d + ctx->ret_h.size();
    ctx->tb.n_ret = (int)ctx->ret_h.size();
    ctx->tb.n_loc = (int)ctx->loc_h.size();
    for (auto &g : ctx->ret_h) ctx->tb.max_ret = std::max(ctx->tb.max_ret, g.n);
    for (auto &g : ctx->loc_h) ctx->tb.max_loc = std::max(ctx->tb.max_loc, g.n);
    *out = holder.release();
    return SD_OK;
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_workspace_size(const sd_ctx *ctx, int batch, size_t *bytes) {
  try {
    if (!ctx || !bytes) return SD_ERR_INVALID_ARG;
    if (batch < 0 || batch > ctx->cfg.max_batch) return SD_ERR_INVALID_ARG;
    *bytes = layout(ctx, batch).total;
    return SD_OK;
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_index_keys(sd_ctx *ctx, const void *k_pre, const int32_t *slots, int num_tokens,
                                   void *index_cache, sd_stream stream) {
  try {
    if (!ctx) return SD_ERR_INVALID_ARG;
    if (num_tokens < 0) return fail(ctx, SD_ERR_INVALID_ARG, "num_tokens < 0");
    if (num_tokens == 0) return SD_OK;
    if (!k_pre || !slots || !index_cache) return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(k_pre) || !aligned16(index_cache))
      return fail(ctx, SD_ERR_INVALID_ARG, "k_pre and index_cache must be 16-byte aligned");
    DeviceGuard dg(ctx->device);
    cudaError_t e = sd::launch_index_keys(static_cast<const uint16_t *>(k_pre), slots, num_tokens,
                                          static_cast<uint16_t *>(index_cache), ctx->proj_d, ctx->sh,
                                          ctx->err_d, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SD_OK : cuda_fail(ctx, e, "index_keys launch");
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_select(sd_ctx *ctx, const void *q_pre, const void *index_cache,
                               const int32_t *page_table, const int32_t *seq_lens, int batch,
                               int32_t *sel_idx, int32_t *sel_count, int sel_stride, void *workspace,
                               size_t ws_bytes, sd_stream stream) {
  try {
    if (!ctx) return SD_ERR_INVALID_ARG;
    if (batch < 0 || batch > ctx->cfg.max_batch) return fail(ctx, SD_ERR_INVALID_ARG, "batch out of range");
    if (batch == 0 || ctx->sh.H_ret == 0) return SD_OK;
    if (!q_pre || !index_cache || !page_table || !seq_lens || !sel_idx || !sel_count)
      return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q_pre) || !aligned16(index_cache))
      return fail(ctx, SD_ERR_INVALID_ARG, "q_pre and index_cache must be 16-byte aligned");
    const long long need_stride = ctx->cfg.mode == SD_TOP_P ? ctx->sh.max_len : max_topk(ctx);
    if (sel_stride < need_stride)
      return fail(ctx, SD_ERR_INVALID_ARG, "sel_stride smaller than the largest possible set");
    const WsLayout w = layout(ctx, batch);
    if (!workspace || ws_bytes < w.total) return fail(ctx, SD_ERR_WORKSPACE, "workspace too small");
    DeviceGuard dg(ctx->device);
    sd::SelectArgs a{};
    a.q_pre = static_cast<const uint16_t *>(q_pre);
    a.index_cache = static_cast<const uint16_t *>(index_cache);
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.sel_stride = sel_stride;
    a.proj = ctx->proj_d;
    a.index_scale = ctx->index_scale;
    a.mode = ctx->cfg.mode;
    a.top_p = ctx->cfg.top_p;
    a.top_k = ctx->cfg.top_k;
    a.top_k_frac = ctx->cfg.top_k_frac;
    a.score_ws = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.scores_off);
    a.flags = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + w.flags_off);
    a.stream_ws = w.stream_bytes ? static_cast<char *>(workspace) + w.stream_off : nullptr;
    a.err = ctx->err_d;
    a.batch = batch;
    cudaError_t e = sd::launch_select(a, ctx->sh, ctx->tb, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SD_OK : cuda_fail(ctx, e, "select launch");
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_select_exact(sd_ctx *ctx, const void *q, const void *k_cache, const int32_t *page_table,
                                     const int32_t *seq_lens, int batch, int32_t *sel_idx, int32_t *sel_count,
                                     int sel_stride, void *workspace, size_t ws_bytes, sd_stream stream) {
  try {
    if (!ctx) return SD_ERR_INVALID_ARG;
    if (batch < 0 || batch > ctx->cfg.max_batch) return fail(ctx, SD_ERR_INVALID_ARG, "batch out of range");
    if (batch == 0 || ctx->sh.H_ret == 0) return SD_OK;
    if (!q || !k_cache || !page_table || !seq_lens || !sel_idx || !sel_count)
      return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k_cache))
      return fail(ctx, SD_ERR_INVALID_ARG, "q and k_cache must be 16-byte aligned");
    const long long need_stride = ctx->cfg.mode == SD_TOP_P ? ctx->sh.max_len : max_topk(ctx);
    if (sel_stride < need_stride)
      return fail(ctx, SD_ERR_INVALID_ARG, "sel_stride smaller than the largest possible set");
    const WsLayout w = layout(ctx, batch);
    if (!workspace || ws_bytes < w.total) return fail(ctx, SD_ERR_WORKSPACE, "workspace too small");
    DeviceGuard dg(ctx->device);
    sd::SelectArgs a{};
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.sel_stride = sel_stride;
    a.proj = ctx->proj_d;
    a.index_scale = ctx->index_scale;
    a.mode = ctx->cfg.mode;
    a.top_p = ctx->cfg.top_p;
    a.top_k = ctx->cfg.top_k;
    a.top_k_frac = ctx->cfg.top_k_frac;
    a.score_ws = reinterpret_cast<float *>(static_cast<char *>(workspace) + w.scores_off);
    a.flags = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + w.flags_off);
    a.stream_ws = nullptr;
    a.err = ctx->err_d;
    a.batch = batch;
    a.pre_scored = true;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = sd::launch_exact_scores(a, ctx->sh, ctx->tb, static_cast<const uint16_t *>(q),
                                            static_cast<const uint16_t *>(k_cache), ctx->attn_scale, st);
    if (e == cudaSuccess) e = sd::launch_select(a, ctx->sh, ctx->tb, st);
    return e == cudaSuccess ? SD_OK : cuda_fail(ctx, e, "exact-score select launch");
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_attend(sd_ctx *ctx, const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *page_table, const int32_t *seq_lens, int batch,
                               const int32_t *sel_idx, const int32_t *sel_count, int sel_stride, float *out,
                               void *workspace, size_t ws_bytes, sd_stream stream) {
  try {
    return attend_impl(ctx, nullptr, q, nullptr, k_cache, v_cache, nullptr, nullptr, page_table, seq_lens, batch,
                       const_cast<int32_t *>(sel_idx), const_cast<int32_t *>(sel_count), sel_stride, out, workspace,
                       ws_bytes, stream, false, false);
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_select_attend(sd_ctx *ctx, const void *q_pre, const void *q, const void *index_cache,
                                     const void *k_cache, const void *v_cache, const int32_t *page_table,
                                     const int32_t *seq_lens, int batch, int32_t *sel_idx, int32_t *sel_count,
                                     int sel_stride, float *out, void *workspace, size_t ws_bytes, sd_stream stream) {
  try {
    return attend_impl(ctx, q_pre, q, index_cache, k_cache, v_cache, nullptr, nullptr, page_table, seq_lens, batch,
                       sel_idx, sel_count, sel_stride, out, workspace, ws_bytes, stream, true, false);
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_attend_split(sd_ctx *ctx, const void *q, const void *k_ret, const void *v_ret,
                                     const void *local_k, const void *local_v, const int32_t *page_table,
                                     const int32_t *seq_lens, int batch, const int32_t *sel_idx,
                                     const int32_t *sel_count, int sel_stride, float *out, void *workspace,
                                     size_t ws_bytes, sd_stream stream) {
  try {
    return attend_impl(ctx, nullptr, q, nullptr, k_ret, v_ret, local_k, local_v, page_table, seq_lens, batch,
                       const_cast<int32_t *>(sel_idx), const_cast<int32_t *>(sel_count), sel_stride, out, workspace,
                       ws_bytes, stream, false, true);
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_select_attend_split(sd_ctx *ctx, const void *q_pre, const void *q, const void *index_cache,
                                           const void *k_ret, const void *v_ret, const void *local_k,
                                           const void *local_v, const int32_t *page_table, const int32_t *seq_lens,
                                           int batch, int32_t *sel_idx, int32_t *sel_count, int sel_stride,
                                           float *out, void *workspace, size_t ws_bytes, sd_stream stream) {
  try {
    return attend_impl(ctx, q_pre, q, index_cache, k_ret, v_ret, local_k, local_v, page_table, seq_lens, batch,
                       sel_idx, sel_count, sel_stride, out, workspace, ws_bytes, stream, true, true);
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_prefill(sd_ctx *ctx, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *page_table, const int32_t *seq_lens, const int32_t *q_starts,
                                int batch, int total_q, float *out, sd_stream stream) {
  try {
    if (!ctx) return SD_ERR_INVALID_ARG;
    if (batch < 0 || batch > ctx->cfg.max_batch) return fail(ctx, SD_ERR_INVALID_ARG, "batch out of range");
    if (total_q < 0) return fail(ctx, SD_ERR_INVALID_ARG, "total_q < 0");
    if (batch == 0 || total_q == 0) return SD_OK;
    if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !q_starts || !out)
      return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
      return fail(ctx, SD_ERR_INVALID_ARG, "q, the caches and out must be 16-byte aligned");
    DeviceGuard dg(ctx->device);
    const cudaError_t e = sd::launch_prefill(
        static_cast<const uint16_t *>(q), static_cast<const uint16_t *>(k_cache),
        static_cast<const uint16_t *>(v_cache), page_table, seq_lens, q_starts, batch, total_q, out,
        ctx->attn_scale, ctx->cfg.window, ctx->cfg.num_sinks, ctx->sh, ctx->tb, ctx->err_d,
        static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SD_OK : cuda_fail(ctx, e, "prefill launch");
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

int sparse_decode_num_retrieval_groups(const sd_ctx *ctx) { return ctx ? ctx->tb.n_ret : 0; }

int sparse_decode_num_local_groups(const sd_ctx *ctx) { return ctx ? ctx->tb.n_loc : 0; }

sd_status sparse_decode_local_append(sd_ctx *ctx, const void *k_new, const void *v_new, const int32_t *seq_ids,
                                     const int32_t *positions, int num_tokens, void *local_k, void *local_v,
                                     sd_stream stream) {
  try {
    if (!ctx) return SD_ERR_INVALID_ARG;
    if (num_tokens < 0) return fail(ctx, SD_ERR_INVALID_ARG, "num_tokens < 0");
    const long long rows = local_rows(ctx);
    if (num_tokens == 0 || ctx->tb.n_loc == 0 || rows == 0) return SD_OK;
    if (!k_new || !v_new || !seq_ids || !positions || !local_k || !local_v)
      return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(local_k) || !aligned16(local_v))
      return fail(ctx, SD_ERR_INVALID_ARG, "k_new, v_new and the local caches must be 16-byte aligned");
    DeviceGuard dg(ctx->device);
    const cudaError_t e = sd::launch_local_append(
        static_cast<const uint16_t *>(k_new), static_cast<const uint16_t *>(v_new), seq_ids, positions, num_tokens,
        static_cast<uint16_t *>(local_k), static_cast<uint16_t *>(local_v), ctx->sh, ctx->tb, ctx->cfg.max_batch,
        ctx->cfg.num_sinks, ctx->cfg.window, ctx->err_d, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SD_OK : cuda_fail(ctx, e, "local_append launch");
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

sd_status sparse_decode_attend_noalloc(sd_ctx *ctx, const void *q, const void *k_cache, const void *v_cache,
                                       const int32_t *page_table, const int32_t *seq_lens, int batch,
                                       const int32_t *sel_idx, const int32_t *sel_count, int sel_stride,
                                       float *out, sd_stream stream) {
  try {
    if (!ctx) return SD_ERR_INVALID_ARG;
    if (batch < 0 || batch > ctx->cfg.max_batch) return fail(ctx, SD_ERR_INVALID_ARG, "batch out of range");
    if (batch == 0) return SD_OK;
    if (!q || !k_cache || !v_cache || !page_table || !seq_lens || !out)
      return fail(ctx, SD_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
      return fail(ctx, SD_ERR_INVALID_ARG, "q, k_cache and v_cache must be 16-byte aligned");
    if (ctx->sh.H_ret > 0 && (!sel_idx || !sel_count || sel_stride <= 0))
      return fail(ctx, SD_ERR_INVALID_ARG, "selection lists required for retrieval heads");
    const size_t need = sd::attend_workspace_bytes(ctx->sh, ctx->tb, batch);
    if (need > sd::kNoAllocScratchBytes)
      return fail(ctx, SD_ERR_WORKSPACE,
                  "attend needs " + std::to_string(need) + " bytes of scratch for this batch; the built-in scratch holds " +
                      std::to_string(sd::kNoAllocScratchBytes) + " (use sparse_decode_attend with a caller workspace)");
    DeviceGuard dg(ctx->device);
    void *scratch = nullptr;
    cudaError_t e = sd::noalloc_scratch(&scratch);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "scratch lookup");
    sd::AttendArgs a{};
    a.q = static_cast<const uint16_t *>(q);
    a.k_cache = static_cast<const uint16_t *>(k_cache);
    a.v_cache = static_cast<const uint16_t *>(v_cache);
    a.page_table = page_table;
    a.seq_lens = seq_lens;
    a.sel_idx = sel_idx;
    a.sel_count = sel_count;
    a.sel_stride = sel_stride;
    a.out = out;
    a.attn_scale = ctx->attn_scale;
    a.window = ctx->cfg.window;
    a.num_sinks = ctx->cfg.num_sinks;
    a.ws = scratch;
    a.err = ctx->err_d;
    a.batch = batch;
    e = sd::launch_attend(a, ctx->sh, ctx->tb, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SD_OK : cuda_fail(ctx, e, "attend launch");
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

void sparse_decode_testing_stall_prefill(int on) { sd::g_prefill_stall.store(on != 0 ? 1 : 0); }

sd_status sparse_decode_error_word(sd_ctx *ctx, sd_stream stream, uint32_t *word) {
  try {
    if (!ctx) return SD_ERR_INVALID_ARG;
    DeviceGuard dg(ctx->device);
    unsigned v = 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&v, ctx->err_d, sizeof(unsigned), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ctx->err_d, 0, sizeof(unsigned), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "error word read");
    if (word) *word = v;
    if (v == 0) return SD_OK;
    if (v & SD_EBIT_TIMEOUT) return fail(ctx, SD_ERR_TIMEOUT, "device-side wait timed out");
    char buf[96];
    snprintf(buf, sizeof(buf), "device-side check rejected input data (error word 0x%x)", v);
    return fail(ctx, SD_ERR_DEVICE_DATA, buf);
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

void sparse_decode_destroy(sd_ctx *ctx) {
  if (!ctx) return;
  {
    DeviceGuard dg(ctx->device);
    if (ctx->groups_d) cudaFree(ctx->groups_d);
    if (ctx->proj_d) cudaFree(ctx->proj_d);
    if (ctx->err_d) cudaFree(ctx->err_d);
  }
  delete ctx;
}

}  // extern "C"
