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
// Two launches:
//   plan  one CTA per (sequence b, KV group g with retrieval heads, span of
//         positions).  Finds each head's sub-list of its ascending selected
//         positions inside the span (warp-cooperative search), marks them in
//         per-head bitmaps and compacts the union into an ordered list of
//         (cache row, head mask): every union row is read once for all the
//         group's heads that selected it.  The page of each row is resolved
//         here, from a shared-memory copy of the span's page-table slice.
//   main  one CTA per (b, g, role, chunk).  A retrieval chunk is an equal share
//         of the (b, g) union list (the span lists concatenated); a local chunk
//         is a run of 1024 rows of [0, sinks) U [N - window, N).  Four warps
//         stream 16-row K/V tiles through per-warp cp.async rings (XOR-swizzled
//         16-byte chunks) and run them on the tensor cores in the
//         FlashAttention-2 arrangement: S = Q K^T with mma.m16n8k16 (A = the
//         group's bf16 queries, heads on M; B = K rows by ldmatrix), a masked
//         online softmax per head in base 2, then O += P V with P taken
//         straight from the S fragments, split exactly into bf16 hi + lo terms
//         so that P keeps float32 accuracy (B = V rows by ldmatrix.trans).
//         Each CTA merges its warps and writes one partial (m, l, acc[d]) per
//         (b, head, chunk); the last CTA of a (b, g, role) to finish (atomic
//         ticket, no waiting) merges the partials with a log-sum-exp combine
//         into out[b, h, :] and resets the ticket.
#include <algorithm>
#include <cmath>
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
constexpr int kSpanMax = 8192;          // positions per plan CTA (max)

// main
constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kTileRows = 16;
constexpr int kTileRing = 2;            // tiles in flight per warp
constexpr int kPassRows = 1024;         // list entries staged in shared memory per pass
constexpr int kSpanLoc = 1024;          // local rows per chunk
constexpr int kChunksRet = 16;          // retrieval chunks per (b, g), at most
constexpr int kRowsPerChunk = 512;      // retrieval: aim for at least this many rows per chunk

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
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
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// the same with rows 8-15 of A zero: only d0, d1 (rows 0-7) are kept, so the
// accumulators of the empty rows need no registers
__device__ __forceinline__ void mma_bf16_top(float (&d)[2], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  float j0, j1;
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%5}, {%7,%8}, "
      "{%0,%1,%9,%9};\n"
      : "+f"(d[0]), "+f"(d[1]), "=f"(j0), "=f"(j1)
      : "r"(a0), "r"(0u), "r"(a2), "r"(b0), "r"(b1), "f"(0.0f));
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

// First index i in [0, n) with arr[i] >= x (n if none); whole warp cooperates.
// Lanes 0..30 probe inside [lo, hi); lane 31 always lands at or past hi and
// acts as the sentinel, so some lane is always true.
__device__ int warp_lower_bound(const int32_t *arr, int n, int x, int lane) {
  int lo = 0, hi = n;                      // answer in [lo, hi]
  while (hi - lo > 31) {
    const int step = (hi - lo + 30) / 31;  // 31 * step >= hi - lo
    const int p = lo + lane * step;
    const bool ge = (p < hi) ? (__ldg(arr + p) >= x) : true;
    const int first = __ffs(__ballot_sync(kFull, ge)) - 1;
    const int nhi = std::min(hi, lo + first * step);
    const int nlo = first == 0 ? lo : lo + (first - 1) * step + 1;
    lo = nlo;
    hi = nhi;
  }
  const int p = lo + lane;                 // hi - lo <= 31: lane 31 is past hi
  const bool ge = (p < hi) ? (__ldg(arr + p) >= x) : true;
  return lo + (__ffs(__ballot_sync(kFull, ge)) - 1);
}

struct AttParams {
  int span;                 // plan: positions per span (power of two, multiple of 32)
  int ns;                   // plan: spans per sequence
  int c_r, c_l;             // main: chunks per retrieval / local item
  int c_max;                // partial slots per (b, head)
};

// Carving of the attend workspace.
struct AttWs {
  float *partials;          // [B][Hq][c_max][D + 2]
  uint32_t *plan_row;       // [B][n_ret][ns][span]: cache row of each union entry
  uint16_t *plan_mask;      // [B][n_ret][ns][span]: heads (bit i = i-th head of the group)
  int *plan_cnt;            // [B][n_ret][ns]
  unsigned *tickets;        // [B][Hkv][2]
};

// ============================================================== plan kernel
// dynamic shared memory: [per-head bitmaps: GR x span / 32 words][page slice: span / 16 ints]
template <int GR>
__global__ void __launch_bounds__(kPlanThreads)
attend_plan_kernel(const AttendArgs a, const Shape sh, const Tables tb, const AttParams ap, const AttWs ws) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, gi = blockIdx.y, b = blockIdx.z;
  __shared__ Group grp;
  __shared__ int seg_lo[kMaxGroup], seg_hi[kMaxGroup];
  __shared__ uint32_t wtot[kPlanWarps];
  extern __shared__ uint32_t plan_dyn[];
  const int bwords = ap.span / 32;
  uint32_t *hbm = plan_dyn;
  int *pslice = reinterpret_cast<int *>(plan_dyn + GR * bwords);
  if (tid == 0) grp = tb.ret[gi];
  __syncthreads();
  const int nh = grp.n, g = grp.kv_head;
  long long N = a.seq_lens[b];
  if (N < 0 || N > sh.max_len) {
    if (tid == 0 && split == 0 && gi == 0) raise_error(a.err, SD_EBIT_SEQLEN);
    N = N < 0 ? 0 : sh.max_len;
  }
  const long long slot = ((long long)b * tb.n_ret + gi) * ap.ns + split;
  const long long p0 = (long long)split * ap.span;
  const long long p1 = std::min(N, p0 + ap.span);
  if (p0 >= N) {
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
    const int at = warp_lower_bound(sel, (int)c, (int)((t & 1) ? p1 : p0), lane);
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
  for (int i = 0; i < nh; ++i) {
    const int32_t *sel = a.sel_idx + ((long long)b * sh.H_ret + grp.row[i]) * a.sel_stride;
    for (int e = seg_lo[i] + tid; e < seg_hi[i]; e += kPlanThreads) {
      const long long pos = sel[e];
      if (pos < p0 || pos >= p1) {                  // not ascending
        raise_error(a.err, SD_EBIT_SEL);
        continue;
      }
      const int off = (int)(pos - p0);
      atomicOr(&hbm[i * bwords + (off >> 5)], 1u << (off & 31));
    }
  }
  __syncthreads();
  // ordered compaction of the union: contiguous word ranges per thread
  const int wpt = (bwords + kPlanThreads - 1) / kPlanThreads;
  const int w0 = tid * wpt, w1 = std::min(bwords, w0 + wpt);
  uint32_t c = 0;
  for (int x = w0; x < w1; ++x) {
    uint32_t u = 0;
    for (int i = 0; i < nh; ++i) u |= hbm[i * bwords + x];
    c += __popc(u);
  }
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  uint32_t base = 0, total = 0;
  for (int x = 0; x < kPlanWarps; ++x) {
    if (x < warp) base += wtot[x];
    total += wtot[x];
  }
  uint32_t o = base + incl - c;
  uint32_t *rows = ws.plan_row + slot * ap.span;
  uint16_t *masks = ws.plan_mask + slot * ap.span;
  for (int x = w0; x < w1; ++x) {
    uint32_t u = 0;
    for (int i = 0; i < nh; ++i) u |= hbm[i * bwords + x];
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      uint32_t m = 0;
      for (int i = 0; i < nh; ++i) m |= ((hbm[i * bwords + x] >> bit) & 1u) << i;
      const int off = x * 32 + bit;
      const int page = pslice[off / kPage];
      if (page < 0) raise_error(a.err, SD_EBIT_PAGE);
      rows[o] = page >= 0 ? (uint32_t)(((long long)page * sh.Hkv + g) * kPage + (off % kPage)) : 0u;
      masks[o] = (uint16_t)(page >= 0 ? m : 0u);
      ++o;
    }
  }
  if (tid == 0) ws.plan_cnt[slot] = (int)total;
}

// ============================================================== main kernel
struct MainShared {
  Group grp;
  int last;
};

// dynamic shared memory: [ring: kWarps x kTileRing x (16 K rows + 16 V rows)]
//                        [pass list: kPassRows x uint32 cache row]
//                        [kPassRows + 16 x uint16 head mask]
//                        [span prefix: ns + 1 ints]
// after the row loop the ring holds the warps' (m, l, acc) for the CTA merge
template <int D, int GR>
__global__ void __launch_bounds__(kThreads)
attend_main_kernel(const AttendArgs a, const Shape sh, const Tables tb, const AttParams ap, const AttWs ws) {
  constexpr int KS = D / 16;                         // k-steps of Q K^T
  constexpr int NT = D / 8;                          // n-tiles (8 dims) of P V
  constexpr int kRowB = 2 * D;                       // bytes of one K (or V) row
  constexpr int kTileB = 2 * kTileRows * kRowB;      // K tile + V tile
  constexpr int CPR = kRowB / 16;                    // 16-byte chunks per row
  constexpr bool HI = GR > 8;                        // heads 8..15 present
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  __shared__ MainShared S;
  extern __shared__ __align__(128) unsigned char dyn[];
  const uint32_t ring0 = (uint32_t)__cvta_generic_to_shared(dyn);
  uint32_t *lrow = reinterpret_cast<uint32_t *>(dyn + (size_t)kWarps * kTileRing * kTileB);
  uint16_t *lmask = reinterpret_cast<uint16_t *>(lrow + kPassRows);
  int *pre = reinterpret_cast<int *>(lmask + kPassRows + kTileRows);

  // ---- decode the work item ------------------------------------------------
  long long bid = blockIdx.x;
  const long long n_ret_items = (long long)a.batch * tb.n_ret * ap.c_r;
  const bool is_ret = bid < n_ret_items;
  int b, gi, chunk, nc;
  if (is_ret) {
    b = (int)(bid / ((long long)tb.n_ret * ap.c_r));
    const long long rem = bid % ((long long)tb.n_ret * ap.c_r);
    gi = (int)(rem / ap.c_r);
    chunk = (int)(rem % ap.c_r);
    nc = ap.c_r;
  } else {
    bid -= n_ret_items;
    b = (int)(bid / ((long long)tb.n_loc * ap.c_l));
    const long long rem = bid % ((long long)tb.n_loc * ap.c_l);
    gi = (int)(rem / ap.c_l);
    chunk = (int)(rem % ap.c_l);
    nc = ap.c_l;
  }
  if (tid == 0) S.grp = is_ret ? tb.ret[gi] : tb.loc[gi];
  __syncthreads();
  const int nh = S.grp.n;
  const int g = S.grp.kv_head;
  long long N = a.seq_lens[b];
  if (N < 0 || N > sh.max_len) {
    if (tid == 0 && chunk == 0 && !is_ret && gi == 0) raise_error(a.err, SD_EBIT_SEQLEN);
    N = N < 0 ? 0 : sh.max_len;
  }

  // ---- rows of this chunk: [r0, r1) of the item's row sequence ---------------
  long long r0 = 0, r1 = 0;
  long long loc_a = 0, loc_w = 0;
  const long long slot0 = ((long long)b * tb.n_ret + gi) * ap.ns;
  const int ns_item = is_ret ? (int)std::min<long long>(ap.ns, (N + ap.span - 1) / ap.span) : 0;
  if (is_ret) {
    // exclusive prefix of the span counts (warp 0, 32 spans at a time)
    if (warp == 0) {
      int run = 0;
      for (int s0 = 0; s0 < ns_item; s0 += 32) {
        const int s = s0 + lane;
        const int c = s < ns_item ? ws.plan_cnt[slot0 + s] : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(kFull, incl, o);
          if (lane >= o) incl += y;
        }
        if (s < ns_item) pre[s] = run + incl - c;
        run += __shfl_sync(kFull, incl, 31);
      }
      if (lane == 0) pre[ns_item] = run;
    }
    __syncthreads();
    const long long T = pre[ns_item];
    const long long per = ((T + nc - 1) / nc + kTileRows - 1) / kTileRows * kTileRows;
    r0 = std::min(T, (long long)chunk * per);
    r1 = std::min(T, r0 + per);
  } else {
    loc_a = std::min<long long>(a.num_sinks, N);
    loc_w = std::max<long long>(loc_a, N - a.window);
    const long long L = loc_a + (N - loc_w);
    r0 = std::min(L, (long long)chunk * kSpanLoc);
    r1 = std::min(L, r0 + kSpanLoc);
  }

  // ---- queries: A fragments of Q (heads on M), bf16 ------------------------
  uint32_t qa[KS][4];
  {
    const uint16_t *q0 = gq < nh ? a.q + ((long long)b * sh.Hq + S.grp.q_head[gq]) * D : nullptr;
    const uint16_t *q1 = (HI && gq + 8 < nh) ? a.q + ((long long)b * sh.Hq + S.grp.q_head[gq + 8]) * D : nullptr;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const int c = k * 16 + 2 * tq;
      qa[k][0] = q0 ? *reinterpret_cast<const uint32_t *>(q0 + c) : 0u;
      qa[k][2] = q0 ? *reinterpret_cast<const uint32_t *>(q0 + c + 8) : 0u;
      qa[k][1] = q1 ? *reinterpret_cast<const uint32_t *>(q1 + c) : 0u;
      qa[k][3] = q1 ? *reinterpret_cast<const uint32_t *>(q1 + c + 8) : 0u;
    }
  }
  const float sc = a.attn_scale * kLog2e;
  const uint32_t head_bit0 = 1u << gq, head_bit1 = 1u << (gq + 8);

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  // cp.async mapping: lane -> tile row lane / 2, one half of its 16-byte chunks
  const int crow = lane >> 1, chalf = lane & 1;
  const uint32_t ring_w = ring0 + warp * (kTileRing * kTileB);
  const unsigned char *kbase = reinterpret_cast<const unsigned char *>(a.k_cache);
  const unsigned char *vbase = reinterpret_cast<const unsigned char *>(a.v_cache);
  // byte offset of 16-byte chunk `ch` of tile row `row`: chunks XOR-swizzled by row % 8
  auto swz = [](int row, int ch) -> uint32_t { return (uint32_t)(row * kRowB + ((ch ^ (row & 7)) << 4)); };
  const int lm = lane >> 3, lr = lane & 7;
  const int k_row = lr + (lm >> 1) * 8, k_chk = lm & 1;       // K: rows (0-7 | 8-15) x chunk (2k | 2k+1)
  const int v_row = lr + (lm & 1) * 8, v_chk = lm >> 1;       // V: rows (0-7 | 8-15) x chunk (n | n+1)

  for (long long ps = r0; ps < r1; ps += kPassRows) {
    const int n = (int)std::min<long long>(kPassRows, r1 - ps);
    __syncthreads();                                   // the previous pass no longer reads the list
    // ---- stage the pass's list entries -------------------------------------
    if (is_ret) {
      for (int x = tid; x < n; x += kThreads) {
        const long long gx = ps + x;
        int lo = 0, hi = ns_item;                      // last span s with pre[s] <= gx
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (pre[mid] <= gx) lo = mid;
          else hi = mid;
        }
        const long long e = (slot0 + lo) * ap.span + (gx - pre[lo]);
        lrow[x] = ws.plan_row[e];
        lmask[x] = ws.plan_mask[e];
      }
    } else {
      const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
      const uint16_t all = (uint16_t)((1u << nh) - 1u);
      for (int x = tid; x < n; x += kThreads) {
        const long long rr = ps + x;
        const long long pos = rr < loc_a ? rr : loc_w + (rr - loc_a);
        const int page = pt[pos / kPage];
        const bool ok = page >= 0 && page < sh.num_pages;
        if (!ok) raise_error(a.err, SD_EBIT_PAGE);
        lrow[x] = ok ? (uint32_t)(((long long)page * sh.Hkv + g) * kPage + (pos % kPage)) : 0u;
        lmask[x] = ok ? all : (uint16_t)0;
      }
    }
    const int tiles = (n + kTileRows - 1) / kTileRows;
    for (int x = n + tid; x < tiles * kTileRows; x += kThreads) lmask[x] = 0;
    __syncthreads();

    // ---- stream the pass's tiles: warp w takes tiles w, w + 4, ... ----------
    const int mt = tiles > warp ? (tiles - warp + kWarps - 1) / kWarps : 0;
    auto issue = [&](int t) {
      if (t < mt) {
        const int x = (warp + t * kWarps) * kTileRows + crow;
        const bool ok = x < n;
        const size_t row = ok ? lrow[x] : 0u;
        const unsigned char *ks = kbase + row * kRowB;
        const unsigned char *vs = vbase + row * kRowB;
        const uint32_t dst = ring_w + (t % kTileRing) * kTileB;
#pragma unroll 2                                 // full unrolling keeps 16 addresses live
        for (int j = 0; j < CPR / 2; ++j) {
          const int ch = chalf * (CPR / 2) + j;
          const uint32_t off = swz(crow, ch);
          cp_async16(dst + off, ks + ch * 16, ok ? 16 : 0);
          cp_async16(dst + kTileRows * kRowB + off, vs + ch * 16, ok ? 16 : 0);
        }
      }
      cp_async_commit();
    };
#pragma unroll
    for (int t = 0; t < kTileRing; ++t) issue(t);

    for (int t = 0; t < mt; ++t) {
      cp_async_wait<kTileRing - 1>();
      __syncwarp();
      const uint32_t kt = ring_w + (t % kTileRing) * kTileB;
      const uint32_t vt = kt + kTileRows * kRowB;
      const int x0 = (warp + t * kWarps) * kTileRows;
      // S = Q K^T: n-tile j holds rows 8j .. 8j + 7 of the tile
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        uint32_t kb[4];
        ldsm_x4(kb, kt + swz(k_row, 2 * k + k_chk));
        if constexpr (HI) {
          mma_bf16(s[0], qa[k][0], qa[k][1], qa[k][2], qa[k][3], kb[0], kb[1]);
          mma_bf16(s[1], qa[k][0], qa[k][1], qa[k][2], qa[k][3], kb[2], kb[3]);
        } else {
          float t0[2] = {s[0][0], s[0][1]}, t1[2] = {s[1][0], s[1][1]};
          mma_bf16_top(t0, qa[k][0], qa[k][2], kb[0], kb[1]);
          mma_bf16_top(t1, qa[k][0], qa[k][2], kb[2], kb[3]);
          s[0][0] = t0[0]; s[0][1] = t0[1]; s[1][0] = t1[0]; s[1][1] = t1[1];
        }
      }
      // head masks of rows 2tq, 2tq + 1 (j = 0) and 8 + 2tq, 9 + 2tq (j = 1)
      const uint32_t mk0 = *reinterpret_cast<const uint32_t *>(lmask + x0 + 2 * tq);
      const uint32_t mk1 = *reinterpret_cast<const uint32_t *>(lmask + x0 + 8 + 2 * tq);
      const uint32_t mr[4] = {mk0 & 0xFFFFu, mk0 >> 16, mk1 & 0xFFFFu, mk1 >> 16};
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
      const float al0 = exp2f(m0 - mu0);
      m0 = mn0;
      float al1 = 1.f;
      if (HI) {
        float x1m = fmaxf(fmaxf(p[0][2], p[0][3]), fmaxf(p[1][2], p[1][3]));
        x1m = fmaxf(x1m, __shfl_xor_sync(kFull, x1m, 1));
        x1m = fmaxf(x1m, __shfl_xor_sync(kFull, x1m, 2));
        const float mn1 = fmaxf(m1, x1m);
        const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
        al1 = exp2f(m1 - mu1);
        m1 = mn1;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          p[j][2] = exp2f(p[j][2] - mu1);
          p[j][3] = exp2f(p[j][3] - mu1);
        }
        l1 = fmaf(l1, al1, (p[0][2] + p[0][3]) + (p[1][2] + p[1][3]));
      } else {
#pragma unroll
        for (int j = 0; j < 2; ++j) p[j][2] = p[j][3] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        p[j][0] = exp2f(p[j][0] - mu0);
        p[j][1] = exp2f(p[j][1] - mu0);
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
      uint32_t ph[4], pl[4];
      split_bf16(p[0][0], p[0][1], ph[0], pl[0]);    // head gq,     rows 2tq, 2tq+1
      split_bf16(p[0][2], p[0][3], ph[1], pl[1]);    // head gq + 8, rows 2tq, 2tq+1
      split_bf16(p[1][0], p[1][1], ph[2], pl[2]);    // head gq,     rows 8+2tq, 9+2tq
      split_bf16(p[1][2], p[1][3], ph[3], pl[3]);    // head gq + 8, rows 8+2tq, 9+2tq
#pragma unroll
      for (int nn = 0; nn < NT; nn += 2) {
        uint32_t vb[4];
        ldsm_x4_t(vb, vt + swz(v_row, nn + v_chk));
        if constexpr (HI) {
          mma_bf16(o[nn], ph[0], ph[1], ph[2], ph[3], vb[0], vb[1]);
          mma_bf16(o[nn], pl[0], pl[1], pl[2], pl[3], vb[0], vb[1]);
          mma_bf16(o[nn + 1], ph[0], ph[1], ph[2], ph[3], vb[2], vb[3]);
          mma_bf16(o[nn + 1], pl[0], pl[1], pl[2], pl[3], vb[2], vb[3]);
        } else {
          float u0[2] = {o[nn][0], o[nn][1]}, u1[2] = {o[nn + 1][0], o[nn + 1][1]};
          mma_bf16_top(u0, ph[0], ph[2], vb[0], vb[1]);
          mma_bf16_top(u0, pl[0], pl[2], vb[0], vb[1]);
          mma_bf16_top(u1, ph[0], ph[2], vb[2], vb[3]);
          mma_bf16_top(u1, pl[0], pl[2], vb[2], vb[3]);
          o[nn][0] = u0[0]; o[nn][1] = u0[1]; o[nn + 1][0] = u1[0]; o[nn + 1][1] = u1[1];
        }
      }
      __syncwarp();
      issue(t + kTileRing);
    }
    cp_async_wait<0>();
  }
  // per-lane partial sums of l -> per head
  l0 += __shfl_xor_sync(kFull, l0, 1);
  l0 += __shfl_xor_sync(kFull, l0, 2);
  l1 += __shfl_xor_sync(kFull, l1, 1);
  l1 += __shfl_xor_sync(kFull, l1, 2);

  // ---- merge the warps of the CTA, write the partial -----------------------
  __syncthreads();                                   // ring and lists no longer read
  float *cm = reinterpret_cast<float *>(dyn);                    // [kWarps][16]
  float *cl = cm + kWarps * 16;                                  // [kWarps][16]
  float *cacc = cl + kWarps * 16;                                // [kWarps][GR][D]
  if (tq == 0) {
    cm[warp * 16 + gq] = m0;
    cl[warp * 16 + gq] = l0;
    cm[warp * 16 + gq + 8] = m1;
    cl[warp * 16 + gq + 8] = l1;
  }
#pragma unroll
  for (int nn = 0; nn < NT; ++nn) {
    const int c = nn * 8 + 2 * tq;
    if (gq < GR) {
      cacc[(warp * GR + gq) * D + c] = o[nn][0];
      cacc[(warp * GR + gq) * D + c + 1] = o[nn][1];
    }
    if (HI && gq + 8 < GR) {
      cacc[(warp * GR + gq + 8) * D + c] = o[nn][2];
      cacc[(warp * GR + gq + 8) * D + c + 1] = o[nn][3];
    }
  }
  __syncthreads();
  const int role = is_ret ? 0 : 1;
  for (int x = tid; x < nh * (D + 2); x += kThreads) {
    const int i = x / (D + 2), c = x % (D + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, cm[w * 16 + i]);
    float v;
    if (c == 0) {
      v = M;
    } else {
      v = 0.0f;
      if (M > -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float f = exp2f(cm[w * 16 + i] - M);
          v += f * (c == 1 ? cl[w * 16 + i] : cacc[(w * GR + i) * D + (c - 2)]);
        }
      }
    }
    const long long h = S.grp.q_head[i];
    ws.partials[(((long long)b * sh.Hq + h) * ap.c_max + chunk) * (D + 2) + c] = v;
  }
  __threadfence();
  __syncthreads();
  unsigned *ticket = ws.tickets + ((long long)b * sh.Hkv + g) * 2 + role;
  if (tid == 0) S.last = (atomicAdd(ticket, 1u) == (unsigned)(nc - 1));
  __syncthreads();
  if (!S.last) return;
  __threadfence();

  // ---- last CTA of the item: merge all chunks into out ----------------------
  for (int x = tid; x < nh * D; x += kThreads) {
    const int i = x / D, c = x % D;
    const long long h = S.grp.q_head[i];
    const float *pp = ws.partials + ((long long)b * sh.Hq + h) * ap.c_max * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < nc; ++s) M = fmaxf(M, __ldcg(pp + (long long)s * (D + 2)));
    float num = 0.0f, den = 0.0f;
    if (M > -INFINITY) {
      for (int s = 0; s < nc; ++s) {
        const float ms = __ldcg(pp + (long long)s * (D + 2));
        if (ms == -INFINITY) continue;
        const float f = exp2f(ms - M);
        den = fmaf(f, __ldcg(pp + (long long)s * (D + 2) + 1), den);
        num = fmaf(f, __ldcg(pp + (long long)s * (D + 2) + 2 + c), num);
      }
    }
    a.out[((long long)b * sh.Hq + h) * D + c] = den > 0.0f ? num / den : 0.0f;
  }
  if (tid == 0) atomicExch(ticket, 0u);
}

// ==================================================================== host
int pow2_ceil(long long x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

int group_rows_att(const Tables &tb) { return pow2_ceil(std::max(1, std::max(tb.max_ret, tb.max_loc))); }

// bound: most union rows one retrieval item can hold in this call
AttParams att_params(const Shape &sh, const Tables &tb, long long window, long long sinks, long long bound) {
  AttParams p{};
  const long long L = sh.max_len;
  p.span = (int)std::max(256LL, std::min<long long>(kSpanMax, pow2_ceil((L + 15) / 16)));
  p.ns = (int)((L + p.span - 1) / p.span);
  p.c_r = (int)std::max(1LL, std::min<long long>(kChunksRet, (std::min(bound, L) + kRowsPerChunk - 1) / kRowsPerChunk));
  p.c_l = 0;
  if (tb.n_loc > 0) {
    const long long rows = std::min<long long>(L, window + sinks);
    p.c_l = (int)std::max(1LL, (rows + kSpanLoc - 1) / kSpanLoc);
  }
  // partial slots: the largest chunk count any call can use
  p.c_max = (int)std::max<long long>(kChunksRet, (L + kSpanLoc - 1) / kSpanLoc);
  return p;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct AttLayout {
  size_t partials, plan_row, plan_mask, plan_cnt, tickets, total;
};

AttLayout att_layout(const Shape &sh, const Tables &tb, int batch) {
  const AttParams p = att_params(sh, tb, 0, 0, sh.max_len);
  AttLayout L{};
  const size_t entries = (size_t)batch * tb.n_ret * p.ns * p.span;
  size_t o = 0;
  L.partials = o;  o = align256(o + (size_t)batch * sh.Hq * p.c_max * (sh.d + 2) * sizeof(float));
  L.plan_row = o;  o = align256(o + entries * 4);
  L.plan_mask = o; o = align256(o + entries * 2);
  L.plan_cnt = o;  o = align256(o + (size_t)batch * tb.n_ret * p.ns * 4);
  L.tickets = o;   o = align256(o + (size_t)batch * sh.Hkv * 2 * sizeof(unsigned));
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

// Chunks per retrieval item, at most c_hi.  Chunks are equal shares of an
// item's rows, so CTAs finish in waves: pick the count whose last wave is
// fullest, preferring more chunks when the difference is small.
template <typename K>
int pick_chunks(K kern, size_t smem, long long items, int c_hi, long long other_blocks) {
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, int> slots_of;
  if (items <= 0 || c_hi <= 1) return std::max(1, c_hi);
  int dev = 0;
  cudaGetDevice(&dev);
  int slots = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    const auto key = std::make_pair((const void *)kern, dev);
    auto it = slots_of.find(key);
    if (it == slots_of.end()) {
      int occ = 0, sms = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        occ = sms = 0;
      }
      it = slots_of.emplace(key, occ * sms).first;
    }
    slots = it->second;
  }
  if (slots <= 0) return c_hi;
  auto eff = [&](int c) {
    const double w = (double)(items * c + other_blocks) / slots;
    return w / std::ceil(w);
  };
  double best = 0.0;
  for (int c = 1; c <= c_hi; ++c) best = std::max(best, eff(c));
  int pick = 1;
  for (int c = 1; c <= c_hi; ++c)
    if (eff(c) >= best - 0.03) pick = c;
  return pick;
}

template <int D, int GR>
cudaError_t launch_t(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &p, const AttWs &ws,
                     cudaStream_t st) {
  if (tb.n_ret > 0) {
    const size_t pbytes = (size_t)GR * (p.span / 32) * 4 + (size_t)(p.span / kPage) * 4;
    cudaError_t e = set_smem(attend_plan_kernel<GR>, pbytes);
    if (e != cudaSuccess) return e;
    attend_plan_kernel<GR><<<dim3(p.ns, tb.n_ret, a.batch), kPlanThreads, pbytes, st>>>(a, sh, tb, p, ws);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t ring = (size_t)kWarps * kTileRing * (2 * kTileRows * 2 * D);
  const size_t lists = (size_t)kPassRows * 4 + (size_t)(kPassRows + kTileRows) * 2 + (size_t)(p.ns + 1) * 4;
  const size_t merge = (size_t)kWarps * 32 * 4 + (size_t)kWarps * GR * D * 4;
  const size_t bytes = std::max(ring + lists, merge);
  cudaError_t e = set_smem(attend_main_kernel<D, GR>, bytes);
  if (e != cudaSuccess) return e;
  AttParams q = p;
  q.c_r = pick_chunks(attend_main_kernel<D, GR>, bytes, (long long)a.batch * tb.n_ret, p.c_r,
                      (long long)a.batch * tb.n_loc * p.c_l);
  const long long blocks = (long long)a.batch * ((long long)tb.n_ret * q.c_r + (long long)tb.n_loc * q.c_l);
  if (blocks == 0) return cudaSuccess;
  attend_main_kernel<D, GR><<<(unsigned)blocks, kThreads, bytes, st>>>(a, sh, tb, q, ws);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_gr(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &p,
                        const AttWs &ws, cudaStream_t st) {
  switch (group_rows_att(tb)) {
    case 1: return launch_t<D, 1>(a, sh, tb, p, ws, st);
    case 2: return launch_t<D, 2>(a, sh, tb, p, ws, st);
    case 4: return launch_t<D, 4>(a, sh, tb, p, ws, st);
    case 8: return launch_t<D, 8>(a, sh, tb, p, ws, st);
    default: return launch_t<D, 16>(a, sh, tb, p, ws, st);
  }
}

}  // namespace

size_t attend_workspace_bytes(const Shape &sh, const Tables &tb, int batch) {
  return att_layout(sh, tb, batch).total;
}

cudaError_t launch_attend(const AttendArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st) {
  if (a.batch == 0) return cudaSuccess;
  const AttLayout L = att_layout(sh, tb, a.batch);
  char *base = static_cast<char *>(a.ws);
  AttWs ws{};
  ws.partials = reinterpret_cast<float *>(base + L.partials);
  ws.plan_row = reinterpret_cast<uint32_t *>(base + L.plan_row);
  ws.plan_mask = reinterpret_cast<uint16_t *>(base + L.plan_mask);
  ws.plan_cnt = reinterpret_cast<int *>(base + L.plan_cnt);
  ws.tickets = reinterpret_cast<unsigned *>(base + L.tickets);
  const long long bound = tb.n_ret > 0 ? (long long)std::max(1, tb.max_ret) * a.sel_stride : 0;
  const AttParams p = att_params(sh, tb, a.window, a.num_sinks, bound);
  cudaError_t e = cudaMemsetAsync(ws.tickets, 0, (size_t)a.batch * sh.Hkv * 2 * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  return sh.d == 128 ? dispatch_gr<128>(a, sh, tb, p, ws, st) : dispatch_gr<64>(a, sh, tb, p, ws, st);
}

}  // namespace sd
