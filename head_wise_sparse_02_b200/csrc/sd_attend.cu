// Exact softmax attention over the selected rows (retrieval heads) and over
// sinks + recent window (local heads), split over the rows and merged.
//
// ICS page (gist.science/ar/paper/2605.24168), 3c: sparse decode reads only the
// selected K/V rows, so decode traffic drops from O(N d) to O(k d).
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 1: local heads
// use a sliding window with attention sinks.  AoH page
// (gist.science/ar/paper/2608.06849), Methodology 4: sinks + recent window;
// roles are shared by the heads of a GQA group.
//
// Work item = (sequence b, KV group g, role): a retrieval item's rows are the
// union of its heads' selected positions, a local item's rows are
// [0, sinks) U [N - window, N).  Rows are processed in 16-row tiles.
//
// Three launches:
//   plan  one CTA per (b, retrieval group, span of positions).  Finds each
//         head's sub-list of its ascending selected positions inside the span
//         (warp-cooperative search), marks them in per-head bitmaps and
//         compacts the union into an ordered list of (cache row, head mask):
//         every union row is read once for all the group's heads that
//         selected it.  The page of each row is resolved here, from a
//         shared-memory copy of the span's page-table slice; the union sizes
//         per span are written out.
//   layout one CTA sums the plan's span counts of each retrieval item, lays
//         all items end to end and writes the first tile of each (a prefix
//         sum over the items' tile counts); it also clears the merge tickets,
//         so that no call needs memory that starts at zero.
//   main  a persistent grid, one CTA per resident slot.  CTA c takes the
//         equal share [W c / P, W (c + 1) / P) of all W tiles and walks the
//         items it overlaps (usually one or two), so that its rings run
//         without the start and drain of a grid of small CTAs.  Four warps
//         stream tiles through per-warp cp.async rings (whole rows per
//         instruction, padded row pitch; each warp fetches its tiles' rows
//         from the union lists itself, one tile ahead, so nothing stops the
//         rings inside an item) and run them on the tensor cores in
//         the FlashAttention-2 arrangement: S = Q K^T with mma.m16n8k16 (A =
//         the group's bf16 queries, heads on M; B = K rows by ldmatrix), a
//         masked online softmax per head in base 2, then O += P V with P taken
//         straight from the S fragments, split exactly into bf16 hi + lo terms
//         so that P keeps float32 accuracy (B = V rows by ldmatrix.trans).
//         For every item it touched a CTA merges its warps; an item that lies
//         inside one CTA goes to out directly, otherwise each CTA writes a
//         partial (m, l, acc[d]) and the last to finish (atomic ticket, no
//         waiting) merges the partials with a log-sum-exp combine.
#include <algorithm>
#include <map>
#include <mutex>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;

// plan
constexpr int kPlanThreads = 256;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kSpanMax = 32768;         // positions per plan CTA (max)
constexpr int kPlanCtas = 296;          // plan CTAs aimed for when the items are few (two per SM)

// main
constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kTileRows = 16;
constexpr int kTileRing = 3;            // tiles in flight per warp
constexpr int kMaxGrid = 4096;          // persistent CTAs (partial slots are sized for this)
constexpr int kMergeChunk = 64;         // partial slots weighed per step of the final merge
constexpr int kDensePlanBits = 256;     // union bits per warp step above which lanes write their own rows

// 16-byte copy global -> shared, bypassing L1, with an L2 eviction-priority
// hint (see evict_first_policy)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes), "l"(policy)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d += a * b, bf16 inputs, float32 accumulate
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// the same with rows 8-15 of A zero: only d0, d1 (rows 0-7) are kept, so the
// accumulators of the empty rows need no registers; zu / zf hold 0 (kept in
// one register each by the caller)
__device__ __forceinline__ void mma_bf16_top(float (&d)[2], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1,
                                             uint32_t zu, float zf) {
  [[maybe_unused]] float j0, j1;                    // outputs of the empty rows, discarded
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%5}, {%7,%8}, "
      "{%0,%1,%9,%9};\n"
      : "+f"(d[0]), "+f"(d[1]), "=f"(j0), "=f"(j1)
      : "r"(a0), "r"(zu), "r"(a2), "r"(b0), "r"(b1), "f"(zf));
}
// 2^x by the MUFU unit (PTX ex2.approx.ftz.f32: relative error below 2^-22,
// subnormal results flushed to 0, exp2(-inf) = 0), far inside the float32
// accumulation's own error here
__device__ __forceinline__ float fast_exp2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(r) : "f"(x));
  return r;
}
// two floats -> bf16x2 (x in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(y), "f"(x));
  return r;
}
// p = hi + lo with hi = bf16(p), lo = bf16(p - hi): |p - hi - lo| <= 2^-17 |p|
__device__ __forceinline__ void split_bf16(float x, float y, uint32_t &hi, uint32_t &lo) {
  hi = pack_bf16(x, y);
  lo = pack_bf16(x - bf16_lo(hi), y - bf16_hi(hi));
}

// First index i in [0, n) with arr[i] >= x (n if none), arr ascending; the
// whole warp cooperates.  While the bracket is wider than 31, each lane
// probes 4 of 128 evenly spaced points, the last of which lies at or past hi
// (one dependent round narrows the bracket ~127-fold); then lane j probes
// lo + j, and lane 31 lands at or past hi.  Either way some lane is true.
template <typename T>
__device__ int warp_lower_bound(const T *arr, int n, T x, int lane) {
  int lo = 0, hi = n;                      // answer in [lo, hi]
  while (hi - lo > 31) {
    const int step = (hi - lo + 126) / 127;  // 127 * step >= hi - lo: probe 127 is past hi
    bool ge[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int p = lo + (lane * 4 + j) * step;
      ge[j] = (p < hi) ? (__ldcg(arr + p) >= x) : true;
    }
    const int jf = ge[0] ? 0 : (ge[1] ? 1 : (ge[2] ? 2 : (ge[3] ? 3 : 4)));
    const unsigned bal = __ballot_sync(kFull, jf < 4);
    // probe k = 4 l + j is at lo + k step; probe 127 (lane 31) is always true
    const int l = __ffs(bal) - 1;
    const int first = l * 4 + __shfl_sync(kFull, jf, l);
    const int nhi = std::min(hi, lo + first * step);
    const int nlo = first == 0 ? lo : lo + (first - 1) * step + 1;
    lo = nlo;
    hi = nhi;
  }
  const int p = lo + lane;                 // hi - lo <= 31: lane 31 is past hi
  const bool ge = (p < hi) ? (__ldcg(arr + p) >= x) : true;
  return lo + (__ffs(__ballot_sync(kFull, ge)) - 1);
}

struct AttParams {
  int span;                 // plan: positions per span (power of two, multiple of 32)
  int ns;                   // plan: spans per sequence
  int n_ret_items;          // B * n_ret retrieval items, numbered first
  int ni;                   // all items: then B * n_loc local items
};

// Carving of the attend workspace.
struct AttWs {
  float *partials;          // [(kMaxGrid + ni) slots][GR][D + 2]
  uint32_t *plan_row;       // [B][n_ret][ns][span]: cache row of each union entry
  uint16_t *plan_mask;      // [B][n_ret][ns][span]: heads (bit i = i-th head of the group)
  int *plan_cnt;            // [B][n_ret][ns]
  long long *tstart;        // [ni + 1]: first tile of each item; tstart[ni] = all tiles
  int *item_rows;           // [ni]: rows of each item (layout)
  unsigned *tickets;        // [ni]: partials merged per item (cleared by the layout)
};

__device__ __forceinline__ const Group &item_group(const Tables &tb, const AttParams &ap, int i, int &b,
                                                   bool &is_ret) {
  is_ret = i < ap.n_ret_items;
  if (is_ret) {
    b = i / tb.n_ret;
    return tb.ret[i % tb.n_ret];
  }
  const int j = i - ap.n_ret_items;
  b = j / tb.n_loc;
  return tb.loc[j % tb.n_loc];
}

__device__ __forceinline__ long long clamp_len(const AttendArgs &a, const Shape &sh, int b) {
  const long long N = a.seq_lens[b];
  return N < 0 ? 0 : std::min<long long>(N, sh.max_len);
}

// Tile counts and first tiles of all items, by one CTA (block size a multiple
// of 32, at most 1024).  A retrieval item's rows are the sum of its spans'
// union counts (plan_cnt); a local item's rows follow from N.  Items without
// rows get a zero output here, since no main CTA visits them.  The merge
// tickets of the main kernel are cleared here.
template <int D>
__device__ void item_prefix(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &ap,
                            const AttWs &ws) {
  __shared__ long long wsum[32];
  __shared__ long long carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < ap.ni; base += blockDim.x) {
    const int i = base + tid;
    long long nt = 0;
    if (i < ap.ni) {
      int b;
      bool is_ret;
      const Group &grp = item_group(tb, ap, i, b, is_ret);
      long long rows;
      const long long N0 = a.seq_lens[b];
      if (N0 < 0 || N0 > sh.max_len) raise_error(a.err, SD_EBIT_SEQLEN);
      const long long N = clamp_len(a, sh, b);
      if (is_ret) {
        const int ns_item = (int)((N + ap.span - 1) / ap.span);
        const int *cnt = ws.plan_cnt + ((long long)b * tb.n_ret + i % tb.n_ret) * ap.ns;
        rows = 0;
        for (int s = 0; s < ns_item; ++s) rows += __ldcg(cnt + s);
      } else {
        const long long la = std::min<long long>(a.num_sinks, N);
        const long long lw = std::max<long long>(la, N - a.window);
        rows = la + (N - lw);
      }
      ws.item_rows[i] = (int)rows;
      ws.tickets[i] = 0u;
      nt = (rows + kTileRows - 1) / kTileRows;
      if (rows == 0)
        for (int x = 0; x < grp.n * D; ++x) a.out[((long long)b * sh.Hq + grp.q_head[x / D]) * D + x % D] = 0.0f;
    }
    long long incl = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    long long before = carry, total = 0;
    for (int w = 0; w < nw; ++w) {
      if (w < warp) before += wsum[w];
      total += wsum[w];
    }
    if (i < ap.ni) ws.tstart[i] = before + incl - nt;
    __syncthreads();
    if (tid == 0) carry += total;
    __syncthreads();
  }
  if (tid == 0) ws.tstart[ap.ni] = carry;
}

// The item layout, one CTA, after the plan (when there is one) has summed the
// retrieval items' rows.
template <int D>
__global__ void __launch_bounds__(1024)
attend_prefix_kernel(const AttendArgs a, const Shape sh, const Tables tb, const AttParams ap, const AttWs ws) {
  pdl_wait();
  pdl_trigger();
  item_prefix<D>(a, sh, tb, ap, ws);
}

// ============================================================== plan kernel
// Union list of the span [p0, p1) of retrieval item (b, gi): its length in
// plan_cnt[slot], the list in plan_row / plan_mask.
// hbm: [GR][span / 32] bitmap words; pslice: the span's pages.
template <int GR>
__device__ void plan_span(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &ap,
                          const AttWs &ws, const Group &grp, int b, int gi, int split, uint32_t *hbm, int *pslice) {
  __shared__ int seg_lo[kMaxGroup], seg_hi[kMaxGroup], seg_at[kMaxGroup + 1];
  __shared__ uint32_t wtot[kPlanWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nh = grp.n, g = grp.kv_head;
  const int bwords = ap.span / 32;
  const long long N = clamp_len(a, sh, b);
  const long long slot = ((long long)b * tb.n_ret + gi) * ap.ns + split;
  const long long p0 = (long long)split * ap.span;
  const long long p1 = std::min(N, p0 + ap.span);
  if (p0 >= p1) {
    if (tid == 0) ws.plan_cnt[slot] = 0;
    return;
  }
  // one search per warp: (head, bound) pairs, lower bounds of p0 and p1
  for (int t = warp; t < 2 * nh; t += kPlanWarps) {
    const int i = t >> 1;
    const long long row = (long long)b * sh.H_ret + grp.row[i];
    const int32_t *sel = a.sel_idx + row * a.sel_stride;
    long long c = a.sel_count[row];
    if (c < 0 || c > a.sel_stride) {
      if (lane == 0 && (t & 1) == 0) raise_error(a.err, SD_EBIT_SEL);
      c = c < 0 ? 0 : a.sel_stride;
    }
    const int at = warp_lower_bound<int32_t>(sel, (int)c, (int32_t)((t & 1) ? p1 : p0), lane);
    if (lane == 0) ((t & 1) ? seg_hi : seg_lo)[i] = at;
  }
  for (int o = tid; o < nh * bwords; o += kPlanThreads) hbm[o] = 0u;
  {
    const int32_t *pt = a.page_table + (long long)b * sh.max_pages + p0 / kPage;
    const int npg = (int)((p1 - p0 + kPage - 1) / kPage);
    for (int o = tid; o < npg; o += kPlanThreads) {
      const int page = pt[o];
      pslice[o] = (page >= 0 && page < sh.num_pages) ? page : -1;
    }
  }
  __syncthreads();
  if (tid == 0) {                                    // where each head's entries start in one flat range
    int run = 0;
    for (int i = 0; i < nh; ++i) {
      seg_at[i] = run;
      run += seg_hi[i] - seg_lo[i];
    }
    seg_at[nh] = run;
  }
  __syncthreads();
  // all heads' entries of the span in one flat loop, so that their loads overlap
#pragma unroll 4
  for (int x = tid; x < seg_at[nh]; x += kPlanThreads) {
    int i = 0;
    while (seg_at[i + 1] <= x) ++i;
    const long long pos = a.sel_idx[((long long)b * sh.H_ret + grp.row[i]) * a.sel_stride + seg_lo[i] + (x - seg_at[i])];
    if (pos < p0 || pos >= p1) {                    // not ascending
      raise_error(a.err, SD_EBIT_SEL);
      continue;
    }
    const int off = (int)(pos - p0);
    atomicOr(&hbm[i * bwords + (off >> 5)], 1u << (off & 31));
  }
  __syncthreads();
  // ordered compaction of the union: warp w owns a contiguous run of bitmap
  // words, read lane-strided (32 consecutive words per step, no bank
  // conflicts); a warp scan of the words' union bit counts places each lane's
  // rows, a block-wide sum over the warp totals places the warp
  const int steps = (bwords + kPlanThreads - 1) / kPlanThreads;   // 32-word steps per warp
  const int x0 = warp * steps * 32;
  uint32_t c = 0;
  for (int r = 0; r < steps; ++r) {
    const int x = x0 + r * 32 + lane;
    uint32_t u = 0;
    if (x < bwords)
#pragma unroll
      for (int i = 0; i < GR; ++i) u |= i < nh ? hbm[i * bwords + x] : 0u;
    c += __popc(u);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
  if (lane == 0) wtot[warp] = c;
  __syncthreads();
  uint32_t o = 0, total = 0;
#pragma unroll
  for (int x = 0; x < kPlanWarps; ++x) {
    o += x < warp ? wtot[x] : 0u;
    total += wtot[x];
  }
  uint32_t *rows = ws.plan_row + slot * ap.span;
  uint16_t *masks = ws.plan_mask + slot * ap.span;
  // row of (page, head, slot) = (page * heads + head) * 16 + slot; with a
  // compacted local cache the paged caches hold the retrieval groups only
  const bool ret_only = a.split;
  const uint32_t row_g = (uint32_t)(ret_only ? gi : g) * kPage;
  const uint32_t row_page = (uint32_t)(ret_only ? tb.n_ret : sh.Hkv) * kPage;
  bool bad_page = false;
  for (int r = 0; r < steps; ++r) {
    const int xb = x0 + r * 32;
    const int x = xb + lane;
    uint32_t hw[GR];
    uint32_t u = 0;
#pragma unroll
    for (int i = 0; i < GR; ++i) {
      hw[i] = (x < bwords && i < nh) ? hbm[i * bwords + x] : 0u;
      u |= hw[i];
    }
    const int nl = __popc(u);
    const int step_bits = __reduce_add_sync(kFull, (unsigned)nl);
    if (step_bits >= kDensePlanBits) {
      // dense run: each lane writes the rows of its own word's bits
      int incl = nl;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += y;
      }
      uint32_t at = o + (uint32_t)(incl - nl);
      uint32_t bits = u;
      while (bits) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1u;
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < GR; ++i) m |= ((hw[i] >> bit) & 1u) << i;
        const int off = x * 32 + bit;
        const int page = pslice[off >> 4];
        bad_page |= page < 0;
        rows[at] = page >= 0 ? (uint32_t)page * row_page + row_g + (uint32_t)(off & (kPage - 1)) : 0u;
        masks[at] = (uint16_t)(page >= 0 ? m : 0u);
        ++at;
      }
      o += (uint32_t)step_bits;
      continue;
    }
    // union rows handed out 32 at a time: each store writes consecutive entries
    o += (uint32_t)warp_emit_bits(u, lane, [&](bool valid, int k, int w, int bit) {
      uint32_t m = 0;
#pragma unroll
      for (int i = 0; i < GR; ++i) m |= ((__shfl_sync(kFull, hw[i], w) >> bit) & 1u) << i;   // every lane
      if (!valid) return;
      const int off = (xb + w) * 32 + bit;
      const int page = pslice[off >> 4];
      bad_page |= page < 0;
      rows[o + k] = page >= 0 ? (uint32_t)page * row_page + row_g + (uint32_t)(off & (kPage - 1)) : 0u;
      masks[o + k] = (uint16_t)(page >= 0 ? m : 0u);
    });
  }
  if (bad_page) raise_error(a.err, SD_EBIT_PAGE);
  if (tid == 0) ws.plan_cnt[slot] = (int)total;
}

// dynamic shared memory: [per-head bitmaps: GR x span / 32 words][page slice: span / 16 ints]
// Without `only`: CTA (split, gi, b) plans span `split` of retrieval item
// (b, gi).  With `only` (the select's miss array: [items] flags, count, list),
// the CTAs (split, y) stride over the listed items only.
template <int D, int GR>
__global__ void __launch_bounds__(kPlanThreads)
attend_plan_kernel(const AttendArgs a, const Shape sh, const Tables tb, const AttParams ap, const AttWs ws,
                   const uint32_t *only) {
  const int tid = threadIdx.x;
  const int split = blockIdx.x;
  __shared__ Group grp;
  extern __shared__ uint32_t plan_dyn[];
  int *pslice = reinterpret_cast<int *>(plan_dyn + GR * (ap.span / 32));
  if (only == nullptr && tid == 0) grp = tb.ret[blockIdx.y];
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  if (only == nullptr) {
    plan_span<GR>(a, sh, tb, ap, ws, grp, blockIdx.z, blockIdx.y, split, plan_dyn, pslice);
    return;
  }
  const int n_items = ap.n_ret_items;
  const int listed = (int)__ldcg(only + n_items);
  for (int k = blockIdx.y; k < listed; k += gridDim.y) {
    const int item = (int)__ldcg(only + n_items + 1 + k);
    const int b = item / tb.n_ret, gi = item % tb.n_ret;
    if (tid == 0) grp = tb.ret[gi];
    __syncthreads();
    plan_span<GR>(a, sh, tb, ap, ws, grp, b, gi, split, plan_dyn, pslice);
    __syncthreads();                                 // grp and the bitmaps are reused by the next item
  }
}

// ============================================================== main kernel
struct MainShared {
  Group grp;
  int item;                 // current item
  int last;
};

// dynamic shared memory: [ring: kWarps x kTileRing x (16 K rows + 16 V rows),
//                         rows padded to 2d + 16 bytes: ldmatrix phases hit
//                         distinct banks and every offset is a constant]
//                        [head masks of the tiles in the rings: kWarps x kTileRing x 16 x uint16]
//                        [span prefix of the current item: ns + 1 ints]
// between items the ring holds the warps' (m, l, acc) for the CTA merge
template <int D, int GR>
__global__ void __launch_bounds__(kThreads)
attend_main_kernel(const AttendArgs a, const Shape sh, const Tables tb, const AttParams ap, const AttWs ws) {
  constexpr int KS = D / 16;                         // k-steps of Q K^T
  constexpr int NT = D / 8;                          // n-tiles (8 dims) of P V
  constexpr int kRowB = 2 * D;                       // bytes of one K (or V) row in the cache
  constexpr int kPitch = kRowB + 16;                 // bytes of one row in shared memory
  constexpr int kTileB = 2 * kTileRows * kPitch;     // K tile + V tile
  constexpr int CPR = kRowB / 16;                    // 16-byte chunks per row
  constexpr bool HI = GR > 8;                        // heads 8..15 present
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  __shared__ MainShared S;
  extern __shared__ __align__(128) unsigned char dyn[];
  const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(dyn);
  uint16_t *wmask = reinterpret_cast<uint16_t *>(dyn + (size_t)kWarps * kTileRing * kTileB) +
                    warp * (kTileRing * kTileRows);                       // this warp's tile masks
  int *pre = reinterpret_cast<int *>(dyn + (size_t)kWarps * kTileRing * kTileB + kWarps * kTileRing * kTileRows * 2);
  pdl_wait();
  pdl_trigger();

  // ---- this CTA's share of the tiles -----------------------------------------
  const long long W = __ldcg(ws.tstart + ap.ni);
  // with fewer tiles than CTAs only the first W take part (one tile each), so
  // every CTA between an item's first and last one holds some of its tiles
  const long long P = std::min<long long>(gridDim.x, W), c = blockIdx.x;
  if (c >= P) return;
  const long long t0 = W * c / P, t1 = W * (c + 1) / P;
  // CTA holding tile x: the largest c' with floor(W c' / P) <= x
  auto cta_of = [&](long long x) { return ((x + 1) * P - 1) / W; };
  if (warp == 0) {
    const int i = warp_lower_bound<long long>(ws.tstart, ap.ni + 1, t0 + 1, lane) - 1;   // tstart[i] <= t0 < tstart[i+1]
    if (lane == 0) S.item = i;
  }

  // cp.async mapping: a tile's K rows and its V rows are copied separately
  // (one commit group each), whole rows per instruction (coalesced): lanes
  // [CPR c, CPR (c + 1)) copy row j RPH + c, one 16-byte chunk each
  constexpr int RPH = 32 / CPR;                      // tile rows per copy instruction
  const int c_sub = lane / CPR;                      // which of them
  const int c_ch = lane % CPR;                       // 16-byte chunk of the row
  const uint32_t ring_w = ring0 + warp * (kTileRing * kTileB);
  const unsigned char *kbase = reinterpret_cast<const unsigned char *>(a.k_cache);   // per item, below
  const unsigned char *vbase = reinterpret_cast<const unsigned char *>(a.v_cache);
  // ldmatrix lane addresses inside a tile (plus a constant per k-step / n-tile)
  const int lm = lane >> 3, lr = lane & 7;
  const uint32_t k_lane = (lr + (lm >> 1) * 8) * kPitch + (lm & 1) * 16;   // K: rows (0-7 | 8-15) x chunk (2k | 2k+1)
  const uint32_t v_lane = kTileRows * kPitch + (lr + (lm & 1) * 8) * kPitch + (lm >> 1) * 16;   // V: rows x chunk (n | n+1)
  const float sc = a.attn_scale * kLog2e;
  const uint64_t l2_stream = evict_first_policy();
  uint32_t zu = 0u;
  float zf = 0.0f;
  asm volatile("" : "+r"(zu), "+f"(zf));             // opaque zeros: one register each
  const uint32_t head_bit0 = 1u << gq, head_bit1 = 1u << (gq + 8);

  long long t = t0;
  while (t < t1) {
    __syncthreads();                                   // S.item set; the previous item's smem no longer read
    int item = S.item;
    long long ts = __ldcg(ws.tstart + item), te = __ldcg(ws.tstart + item + 1);
    while (te <= t) {                                  // skip items without tiles
      ++item;
      ts = te;
      te = __ldcg(ws.tstart + item + 1);
    }
    const long long seg_end = std::min(t1, te);
    int b;
    bool is_ret;
    const Group &grp_g = item_group(tb, ap, item, b, is_ret);
    if (tid == 0) S.grp = grp_g;
    const long long N = clamp_len(a, sh, b);
    const long long T = __ldcg(ws.item_rows + item);
    const long long r0 = (t - ts) * kTileRows;
    const long long r1 = std::min(T, (seg_end - ts) * kTileRows);
    const long long first = cta_of(ts), last = cta_of(te - 1);
    const int gi = is_ret ? item % tb.n_ret : 0;
    const long long slot0 = ((long long)b * tb.n_ret + gi) * ap.ns;
    const int ns_item = is_ret ? (int)((N + ap.span - 1) / ap.span) : 0;
    if (is_ret && warp == 0) {
      // exclusive prefix of the item's span counts (32 spans at a time)
      int run = 0;
      for (int s0 = 0; s0 < ns_item; s0 += 32) {
        const int s = s0 + lane;
        const int cnt = s < ns_item ? __ldcg(ws.plan_cnt + slot0 + s) : 0;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFull, incl, o);
          if (lane >= o) incl += y;
        }
        if (s < ns_item) pre[s] = run + incl - cnt;
        run += __shfl_sync(kFull, incl, 31);
      }
      if (lane == 0) pre[ns_item] = run;
    }
    __syncthreads();
    const int nh = S.grp.n;
    const int g = S.grp.kv_head;
    const long long loc_a = std::min<long long>(a.num_sinks, N);
    const long long loc_w = std::max<long long>(loc_a, N - a.window);
    // compacted local cache: rows of (b, local group) start here; the caches
    // the tiles are copied from
    const long long local_base = is_ret ? 0 : (long long)(item - ap.n_ret_items) * (a.num_sinks + a.window);
    kbase = reinterpret_cast<const unsigned char *>(!is_ret && a.split ? a.local_k : a.k_cache);
    vbase = reinterpret_cast<const unsigned char *>(!is_ret && a.split ? a.local_v : a.v_cache);

    // ---- queries: A fragments of Q (heads on M), bf16 ----------------------
    uint32_t qa[KS][4];
    {
      const uint16_t *q0 = gq < nh ? a.q + ((long long)b * sh.Hq + S.grp.q_head[gq]) * D : nullptr;
      const uint16_t *q1 = (HI && gq + 8 < nh) ? a.q + ((long long)b * sh.Hq + S.grp.q_head[gq + 8]) * D : nullptr;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int cc = k * 16 + 2 * tq;
        qa[k][0] = q0 ? *reinterpret_cast<const uint32_t *>(q0 + cc) : 0u;
        qa[k][2] = q0 ? *reinterpret_cast<const uint32_t *>(q0 + cc + 8) : 0u;
        qa[k][1] = q1 ? *reinterpret_cast<const uint32_t *>(q1 + cc) : 0u;
        qa[k][3] = q1 ? *reinterpret_cast<const uint32_t *>(q1 + cc + 8) : 0u;
      }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    // ---- stream the segment's tiles: warp w takes tiles w, w + kWarps, ... -----
    // Lane r < 16 fetches the cache row and head mask of row r of a tile one
    // tile ahead of its copy (registers), so the rings run across the whole
    // segment without staging the list in shared memory.
    const long long rows = r1 - r0;
    const int tiles = (int)((rows + kTileRows - 1) / kTileRows);
    const int mt = tiles > warp ? (tiles - warp + kWarps - 1) / kWarps : 0;
    const uint16_t all = (uint16_t)((1u << nh) - 1u);
    const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
    auto fetch = [&](int q, uint32_t &row, uint32_t &mask) {
      row = 0u;
      mask = 0u;
      if (q >= mt) return;
      const long long gx = r0 + (long long)(warp + q * kWarps) * kTileRows + (lane & 15);
      if (gx < r1) {
        if (is_ret) {
          int lo = 0, hi = ns_item;                    // last span s with pre[s] <= gx
          while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (pre[mid] <= gx) lo = mid;
            else hi = mid;
          }
          const long long e = (slot0 + lo) * ap.span + (gx - pre[lo]);
          row = __ldcg(ws.plan_row + e);
          mask = __ldcg(ws.plan_mask + e);
        } else {
          const long long pos = gx < loc_a ? gx : loc_w + (gx - loc_a);
          if (a.split) {                               // compacted: sinks, then a ring of the window
            row = (uint32_t)(local_base + local_slot(pos, a.num_sinks, a.window));
            mask = all;
          } else {
            const int page = pt[pos / kPage];
            const bool ok = page >= 0 && page < sh.num_pages;
            if (!ok) raise_error(a.err, SD_EBIT_PAGE);
            row = ok ? (uint32_t)(((long long)page * sh.Hkv + g) * kPage + (pos % kPage)) : 0u;
            mask = ok ? all : 0u;
          }
        }
      }
    };
    // tile q's rows: rows past the segment repeat the tile's first row (finite
    // data) and are masked out; the masks go to the warp's slot of tile q
    auto prep = [&](int q, uint32_t row, uint32_t mask) -> uint32_t {
      if (q < mt) {
        const long long gx0 = r0 + (long long)(warp + q * kWarps) * kTileRows;
        const uint32_t first = __shfl_sync(kFull, row, 0);
        if (gx0 + (lane & 15) >= r1) row = first;
        if (lane < kTileRows) wmask[(q % kTileRing) * kTileRows + lane] = (uint16_t)mask;
      }
      return row;
    };
    // copy the K rows (half 0) or the V rows (half 1) of tile q: one commit group
    auto issue_half = [&](int q, uint32_t row, int half) {
      if (q < mt) {
        const uint32_t dst = ring_w + (q % kTileRing) * kTileB + half * (kTileRows * kPitch) + c_ch * 16 +
                             c_sub * kPitch;
        const unsigned char *src = (half ? vbase : kbase) + c_ch * 16;
#pragma unroll
        for (int j = 0; j < kTileRows / RPH; ++j) {
          const uint32_t rj = __shfl_sync(kFull, row, j * RPH + c_sub);
          cp_async16(dst + j * RPH * kPitch, src + (size_t)rj * kRowB, 16, l2_stream);
        }
      }
      cp_async_commit();
    };
    uint32_t nrow, nmask;
    fetch(0, nrow, nmask);
#pragma unroll
    for (int q = 0; q < kTileRing; ++q) {
      const uint32_t row = prep(q, nrow, nmask);
      fetch(q + 1, nrow, nmask);
      issue_half(q, row, 0);
      issue_half(q, row, 1);
    }

    // Groups in flight: K and V of the next kTileRing tiles.  K of tile
    // q + kTileRing is issued as soon as S(q) has read K(q) (during the
    // softmax and P V of tile q), V of tile q + kTileRing after P V(q); at
    // both waits 2 kTileRing - 1 younger groups may stay pending.
    for (int q = 0; q < mt; ++q) {
      cp_async_wait<2 * kTileRing - 1>();              // K(q)
      __syncwarp();
      const uint32_t kt = ring_w + (q % kTileRing) * kTileB;
        // S = Q K^T: n-tile j holds rows 8j .. 8j + 7 of the tile
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int k = 0; k < KS; ++k) {
          uint32_t kb[4];
          ldsm_x4(kb, kt + k_lane + k * 32);
          if constexpr (HI) {
            mma_bf16(s[0], qa[k][0], qa[k][1], qa[k][2], qa[k][3], kb[0], kb[1]);
            mma_bf16(s[1], qa[k][0], qa[k][1], qa[k][2], qa[k][3], kb[2], kb[3]);
          } else {
            float u0[2] = {s[0][0], s[0][1]}, u1[2] = {s[1][0], s[1][1]};
            mma_bf16_top(u0, qa[k][0], qa[k][2], kb[0], kb[1], zu, zf);
            mma_bf16_top(u1, qa[k][0], qa[k][2], kb[2], kb[3], zu, zf);
            s[0][0] = u0[0]; s[0][1] = u0[1]; s[1][0] = u1[0]; s[1][1] = u1[1];
          }
        }
        // head masks of rows 2tq, 2tq + 1 (j = 0) and 8 + 2tq, 9 + 2tq (j = 1)
        const uint16_t *ms = wmask + (q % kTileRing) * kTileRows;
        const uint32_t mk0 = *reinterpret_cast<const uint32_t *>(ms + 2 * tq);
        const uint32_t mk1 = *reinterpret_cast<const uint32_t *>(ms + 8 + 2 * tq);
        const uint32_t mr[4] = {mk0 & 0xFFFFu, mk0 >> 16, mk1 & 0xFFFFu, mk1 >> 16};
        __syncwarp();                                  // K(q) and the masks of q read by all lanes
        const uint32_t rowR = prep(q + kTileRing, nrow, nmask);
        fetch(q + kTileRing + 1, nrow, nmask);
        issue_half(q + kTileRing, rowR, 0);
        float p[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const uint32_t mm = mr[2 * j + e];
            p[j][e] = (mm & head_bit0) ? s[j][e] * sc : -INFINITY;
            p[j][2 + e] = (HI && (mm & head_bit1)) ? s[j][2 + e] * sc : -INFINITY;
          }
        // online softmax per head (head gq: p[.][0..1]; head gq + 8: p[.][2..3])
        float x0m = fmaxf(fmaxf(p[0][0], p[0][1]), fmaxf(p[1][0], p[1][1]));
        x0m = fmaxf(x0m, __shfl_xor_sync(kFull, x0m, 1));
        x0m = fmaxf(x0m, __shfl_xor_sync(kFull, x0m, 2));
        const float mn0 = fmaxf(m0, x0m);
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
        const float al0 = mn0 == m0 ? 1.f : fast_exp2(m0 - mu0);
        m0 = mn0;
        float al1 = 1.f;
        if (HI) {
          float x1m = fmaxf(fmaxf(p[0][2], p[0][3]), fmaxf(p[1][2], p[1][3]));
          x1m = fmaxf(x1m, __shfl_xor_sync(kFull, x1m, 1));
          x1m = fmaxf(x1m, __shfl_xor_sync(kFull, x1m, 2));
          const float mn1 = fmaxf(m1, x1m);
          const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
          al1 = mn1 == m1 ? 1.f : fast_exp2(m1 - mu1);
          m1 = mn1;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            p[j][2] = fast_exp2(p[j][2] - mu1);
            p[j][3] = fast_exp2(p[j][3] - mu1);
          }
          l1 = fmaf(l1, al1, (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]));
        } else {
#pragma unroll
          for (int j = 0; j < 2; ++j) p[j][2] = p[j][3] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          p[j][0] = fast_exp2(p[j][0] - mu0);
          p[j][1] = fast_exp2(p[j][1] - mu0);
        }
        l0 = fmaf(l0, al0, (p[0][0] + p[0][1]) + (p[1][0] + p[1][1]));
        if (__any_sync(kFull, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
          for (int nn = 0; nn < NT; ++nn) {
            o[nn][0] *= al0;
            o[nn][1] *= al0;
            o[nn][2] *= al1;
            o[nn][3] *= al1;
          }
        }
        // P as the A operand (heads x 16 rows), hi + lo
        cp_async_wait<2 * kTileRing - 1>();            // V(q)
        __syncwarp();
        uint32_t ph[4], pl[4];
        split_bf16(p[0][0], p[0][1], ph[0], pl[0]);  // head gq,     rows 2tq, 2tq+1
        split_bf16(p[0][2], p[0][3], ph[1], pl[1]);  // head gq + 8, rows 2tq, 2tq+1
        split_bf16(p[1][0], p[1][1], ph[2], pl[2]);  // head gq,     rows 8+2tq, 9+2tq
        split_bf16(p[1][2], p[1][3], ph[3], pl[3]);  // head gq + 8, rows 8+2tq, 9+2tq
#pragma unroll
        for (int nn = 0; nn < NT; nn += 2) {
          uint32_t vb[4];
          ldsm_x4_t(vb, kt + v_lane + nn * 16);
          if constexpr (HI) {
            mma_bf16(o[nn], ph[0], ph[1], ph[2], ph[3], vb[0], vb[1]);
            mma_bf16(o[nn], pl[0], pl[1], pl[2], pl[3], vb[0], vb[1]);
            mma_bf16(o[nn + 1], ph[0], ph[1], ph[2], ph[3], vb[2], vb[3]);
            mma_bf16(o[nn + 1], pl[0], pl[1], pl[2], pl[3], vb[2], vb[3]);
          } else {
            float u0[2] = {o[nn][0], o[nn][1]}, u1[2] = {o[nn + 1][0], o[nn + 1][1]};
            mma_bf16_top(u0, ph[0], ph[2], vb[0], vb[1], zu, zf);
            mma_bf16_top(u0, pl[0], pl[2], vb[0], vb[1], zu, zf);
            mma_bf16_top(u1, ph[0], ph[2], vb[2], vb[3], zu, zf);
            mma_bf16_top(u1, pl[0], pl[2], vb[2], vb[3], zu, zf);
            o[nn][0] = u0[0]; o[nn][1] = u0[1]; o[nn + 1][0] = u1[0]; o[nn + 1][1] = u1[1];
          }
        }
        __syncwarp();
        issue_half(q + kTileRing, rowR, 1);
      }
      cp_async_wait<0>();
    // per-lane partial sums of l -> per head
    l0 += __shfl_xor_sync(kFull, l0, 1);
    l0 += __shfl_xor_sync(kFull, l0, 2);
    l1 += __shfl_xor_sync(kFull, l1, 1);
    l1 += __shfl_xor_sync(kFull, l1, 2);

    // ---- merge the warps of the CTA ------------------------------------------
    __syncthreads();                                   // ring and lists no longer read
    float *cm = reinterpret_cast<float *>(dyn);                  // [kWarps][16]
    float *cl = cm + kWarps * 16;                                // [kWarps][16]
    float *cacc = cl + kWarps * 16;                              // [kWarps][GR][D]
    if (tq == 0) {
      cm[warp * 16 + gq] = m0;
      cl[warp * 16 + gq] = l0;
      cm[warp * 16 + gq + 8] = m1;
      cl[warp * 16 + gq + 8] = l1;
    }
#pragma unroll
    for (int nn = 0; nn < NT; ++nn) {
      const int cc = nn * 8 + 2 * tq;
      if (gq < GR) {
        cacc[(warp * GR + gq) * D + cc] = o[nn][0];
        cacc[(warp * GR + gq) * D + cc + 1] = o[nn][1];
      }
      if (HI && gq + 8 < GR) {
        cacc[(warp * GR + gq + 8) * D + cc] = o[nn][2];
        cacc[(warp * GR + gq + 8) * D + cc + 1] = o[nn][3];
      }
    }
    __syncthreads();
    const bool alone = first == last;                  // the whole item is in this CTA
    float *part = ws.partials + ((c + item) * GR) * (long long)(D + 2);
    for (int x = tid; x < nh * (D + 2); x += kThreads) {
      const int i = x / (D + 2), cc = x % (D + 2);
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) M = fmaxf(M, cm[w * 16 + i]);
      if (alone) {
        if (cc < 2) continue;
        float num = 0.0f, den = 0.0f;
        if (M > -INFINITY) {
#pragma unroll
          for (int w = 0; w < kWarps; ++w) {
            const float f = exp2f(cm[w * 16 + i] - M);
            den = fmaf(f, cl[w * 16 + i], den);
            num = fmaf(f, cacc[(w * GR + i) * D + (cc - 2)], num);
          }
        }
        a.out[((long long)b * sh.Hq + S.grp.q_head[i]) * D + (cc - 2)] = den > 0.0f ? num / den : 0.0f;
        continue;
      }
      float v;
      if (cc == 0) {
        v = M;
      } else {
        v = 0.0f;
        if (M > -INFINITY) {
#pragma unroll
          for (int w = 0; w < kWarps; ++w) {
            const float f = exp2f(cm[w * 16 + i] - M);
            v += f * (cc == 1 ? cl[w * 16 + i] : cacc[(w * GR + i) * D + (cc - 2)]);
          }
        }
      }
      part[i * (D + 2) + cc] = v;
    }
    if (!alone) {
      __threadfence();
      __syncthreads();
      if (tid == 0) S.last = (atomicAdd(ws.tickets + item, 1u) == (unsigned)(last - first));
      __syncthreads();
      if (S.last) {
        __threadfence();
        // the last segment of the item: merge partial slots first + item .. last
        // + item.  Per head i the reference M_i = max_s m_s; then, kMergeChunk
        // slots at a time, the weights f_is = 2^(m_s - M_i) (0 for an empty
        // slot) go to shared memory and every output sums f_is o_s[cc] with
        // independent loads (an item can span a few hundred CTAs)
        const int np = (int)(last - first + 1);
        constexpr long long PS = (long long)GR * (D + 2);            // stride of the partial slots
        constexpr int OPT = (GR * D + kThreads - 1) / kThreads;     // outputs per thread, at most
        const float *pbase = ws.partials + (first + item) * PS;
        float *fw = reinterpret_cast<float *>(dyn);                  // [GR][kMergeChunk]
        float *sM = fw + GR * kMergeChunk;                           // [GR]
        float *sden = sM + GR;                                       // [GR]
        for (int i = warp; i < nh; i += kWarps) {
          float M = -INFINITY;
          for (int s = lane; s < np; s += 32) M = fmaxf(M, __ldcg(pbase + s * PS + i * (D + 2)));
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
          if (lane == 0) {
            sM[i] = M;
            sden[i] = 0.0f;
          }
        }
        float num[OPT];
#pragma unroll
        for (int u = 0; u < OPT; ++u) num[u] = 0.0f;
        for (int s0 = 0; s0 < np; s0 += kMergeChunk) {
          const int nc = np - s0 < kMergeChunk ? np - s0 : kMergeChunk;
          __syncthreads();                             // M ready; the previous chunk's weights consumed
          for (int x = tid; x < nh * kMergeChunk; x += kThreads) {
            const int i = x / kMergeChunk, sl = x % kMergeChunk;
            float f = 0.0f;
            if (sl < nc) {
              const float ms = __ldcg(pbase + (s0 + sl) * PS + i * (D + 2));
              f = (ms == -INFINITY || sM[i] == -INFINITY) ? 0.0f : exp2f(ms - sM[i]);
            }
            fw[i * kMergeChunk + sl] = f;
          }
          __syncthreads();
          for (int i = warp; i < nh; i += kWarps) {
            float dsum = 0.0f;
            for (int sl = lane; sl < nc; sl += 32)
              dsum = fmaf(fw[i * kMergeChunk + sl], __ldcg(pbase + (s0 + sl) * PS + i * (D + 2) + 1), dsum);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dsum += __shfl_xor_sync(kFull, dsum, off);
            if (lane == 0) sden[i] += dsum;
          }
#pragma unroll
          for (int u = 0; u < OPT; ++u) {
            const int x = tid + u * kThreads;
            if (x < nh * D) {
              const int i = x / D, cc = x % D;
              const float *pp = pbase + s0 * PS + i * (D + 2) + 2 + cc;
              const float *fi = fw + i * kMergeChunk;
              float acc = num[u];
#pragma unroll 8
              for (int sl = 0; sl < nc; ++sl) acc = fmaf(fi[sl], __ldcg(pp + sl * PS), acc);
              num[u] = acc;
            }
          }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < OPT; ++u) {
          const int x = tid + u * kThreads;
          if (x < nh * D) {
            const int i = x / D, cc = x % D;
            a.out[((long long)b * sh.Hq + S.grp.q_head[i]) * D + cc] = sden[i] > 0.0f ? num[u] / sden[i] : 0.0f;
          }
        }
      }
    }
    t = seg_end;
    if (tid == 0) S.item = item + 1;
  }
}

// ==================================================================== host
int pow2_ceil(long long x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

int group_rows_att(const Tables &tb) { return pow2_ceil(std::max(1, std::max(tb.max_ret, tb.max_loc))); }

AttParams att_params(const Shape &sh, const Tables &tb, int batch) {
  AttParams p{};
  const long long L = sh.max_len;
  // spans per sequence: about four, more when the retrieval items are few, so
  // that the plan still has about kPlanCtas CTAs (its work is split by span)
  const long long items = std::max(1LL, (long long)batch * tb.n_ret);
  const long long want = std::max(4LL, (kPlanCtas + items - 1) / items);
  p.span = (int)std::max(256LL, std::min<long long>(kSpanMax, pow2_ceil((L + want - 1) / want)));
  p.ns = (int)((L + p.span - 1) / p.span);
  p.n_ret_items = batch * tb.n_ret;
  p.ni = batch * (tb.n_ret + tb.n_loc);
  return p;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct AttLayout {
  size_t partials, plan_row, plan_mask, plan_cnt, tstart, counters, total;
};

AttLayout att_layout(const Shape &sh, const Tables &tb, int batch) {
  const AttParams p = att_params(sh, tb, batch);
  AttLayout L{};
  const size_t entries = (size_t)batch * tb.n_ret * p.ns * p.span;
  size_t o = 0;
  L.partials = o;  o = align256(o + (size_t)(kMaxGrid + p.ni) * group_rows_att(tb) * (sh.d + 2) * sizeof(float));
  L.plan_row = o;  o = align256(o + entries * 4);
  L.plan_mask = o; o = align256(o + entries * 2);
  L.plan_cnt = o;  o = align256(o + (size_t)batch * tb.n_ret * p.ns * 4);
  L.tstart = o;    o = align256(o + (size_t)(p.ni + 1) * 8);
  L.counters = o;  o = align256(o + (size_t)p.ni * 2 * 4);           // item_rows, tickets
  L.total = o;
  return L;
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, size_t> done;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair((const void *)kern, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

// resident CTAs of a kernel on this device (cached)
template <typename K>
int resident_ctas(K kern, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair((const void *)kern, dev);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int occ = 0, sms = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;                                        // not cached: retried next call
  }
  const int n = std::max(1, std::min(kMaxGrid, occ * sms));
  cache.emplace(key, n);
  return n;
}

template <int D, int GR>
cudaError_t launch_t(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &p, const AttWs &ws,
                     cudaStream_t st, const uint32_t *only) {
  cudaError_t e;
  if (tb.n_ret > 0) {
    const size_t pbytes = (size_t)GR * (p.span / 32) * 4 + (size_t)(p.span / kPage) * 4;
    e = set_smem(attend_plan_kernel<D, GR>, pbytes);
    if (e != cudaSuccess) return e;
    // the listed items only (usually none): a few CTAs per span stride over them
    const dim3 grid = only ? dim3(p.ns, (unsigned)std::min(p.n_ret_items, 4), 1) : dim3(p.ns, tb.n_ret, a.batch);
    e = launch_pdl(attend_plan_kernel<D, GR>, grid, dim3(kPlanThreads), pbytes, st, 0, a, sh, tb, p, ws, only);
    if (e != cudaSuccess) return e;
  }
  e = launch_pdl(attend_prefix_kernel<D>, dim3(1), dim3(1024), 0, st, 0, a, sh, tb, p, ws);
  if (e != cudaSuccess) return e;
  const size_t ring = (size_t)kWarps * kTileRing * (2 * kTileRows * (2 * D + 16));
  const size_t lists = (size_t)kWarps * kTileRing * kTileRows * 2 + (size_t)(p.ns + 1) * 4;
  const size_t merge = std::max((size_t)kWarps * 32 * 4 + (size_t)kWarps * GR * D * 4,
                                (size_t)GR * (kMergeChunk + 2) * 4);
  const size_t bytes = std::max(ring + lists, merge);
  e = set_smem(attend_main_kernel<D, GR>, bytes);
  if (e != cudaSuccess) return e;
  const int grid = resident_ctas(attend_main_kernel<D, GR>, kThreads, bytes);
  if (grid <= 0) return cudaErrorInvalidConfiguration;
  return launch_pdl(attend_main_kernel<D, GR>, dim3(grid), dim3(kThreads), bytes, st, 0, a, sh, tb, p, ws);
}

template <int D>
cudaError_t dispatch_gr(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &p,
                        const AttWs &ws, cudaStream_t st, const uint32_t *only) {
  switch (group_rows_att(tb)) {
    case 1: return launch_t<D, 1>(a, sh, tb, p, ws, st, only);
    case 2: return launch_t<D, 2>(a, sh, tb, p, ws, st, only);
    case 4: return launch_t<D, 4>(a, sh, tb, p, ws, st, only);
    case 8: return launch_t<D, 8>(a, sh, tb, p, ws, st, only);
    default: return launch_t<D, 16>(a, sh, tb, p, ws, st, only);
  }
}

}  // namespace

size_t attend_workspace_bytes(const Shape &sh, const Tables &tb, int batch) {
  return att_layout(sh, tb, batch).total;
}

UnionOut attend_union_view(const Shape &sh, const Tables &tb, int batch, void *attend_ws, bool ret_only) {
  const AttLayout L = att_layout(sh, tb, batch);
  const AttParams p = att_params(sh, tb, batch);
  char *base = static_cast<char *>(attend_ws);
  return UnionOut{reinterpret_cast<uint32_t *>(base + L.plan_row), reinterpret_cast<uint16_t *>(base + L.plan_mask),
                  reinterpret_cast<int *>(base + L.plan_cnt), p.span, p.ns, ret_only};
}

cudaError_t launch_attend(const AttendArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st,
                          const uint32_t *plan_only) {
  if (a.batch == 0) return cudaSuccess;
  const AttLayout L = att_layout(sh, tb, a.batch);
  const AttParams p = att_params(sh, tb, a.batch);
  char *base = static_cast<char *>(a.ws);
  AttWs ws{};
  ws.partials = reinterpret_cast<float *>(base + L.partials);
  ws.plan_row = reinterpret_cast<uint32_t *>(base + L.plan_row);
  ws.plan_mask = reinterpret_cast<uint16_t *>(base + L.plan_mask);
  ws.plan_cnt = reinterpret_cast<int *>(base + L.plan_cnt);
  ws.tstart = reinterpret_cast<long long *>(base + L.tstart);
  ws.item_rows = reinterpret_cast<int *>(base + L.counters);
  ws.tickets = reinterpret_cast<unsigned *>(ws.item_rows + p.ni);
  return sh.d == 128 ? dispatch_gr<128>(a, sh, tb, p, ws, st, plan_only)
                     : dispatch_gr<64>(a, sh, tb, p, ws, st, plan_only);
}

}  // namespace sd
