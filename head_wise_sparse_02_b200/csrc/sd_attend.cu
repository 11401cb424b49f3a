// Exact softmax attention over the selected rows (retrieval heads) and over
// sinks + recent window (local heads), split over the context and merged.
//
// ICS page (gist.science/ar/paper/2605.24168), 3c: sparse decode reads only the
// selected K/V rows, so decode traffic drops from O(N d) to O(k d).
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 1: local heads
// use a sliding window with attention sinks.  AoH page
// (gist.science/ar/paper/2608.06849), Methodology 4: sinks + recent window;
// roles are shared by the heads of a GQA group.
//
// Work item = (sequence b, KV group g, role, split):
//   retrieval  split s covers positions [s*span, (s+1)*span); the CTA finds
//              each head's sub-list of its (ascending) selected positions with
//              a warp-cooperative search, marks them in per-head bitmaps of the
//              span, and compacts the union into an ordered list of
//              (position, head mask): every union row is read once for all the
//              group's heads that selected it;
//   local      split s covers rows [s*span_l, (s+1)*span_l) of the enumerated
//              set [0, sinks) U [N - window, N); every local head of the group
//              uses every row.
// Rows stream through a per-warp cp.async ring (one 16-byte copy per lane per
// row: lanes 0-15 the K row, lanes 16-31 the V row), so the bytes in flight
// live in shared memory, not in registers.  Each warp keeps a float32 online
// softmax per head in base 2 (lane l holds d/32 consecutive elements); the CTA
// merges its warps and writes one partial (m, l, acc[d]) per (b, head, split);
// the last CTA of a (b, g, role) to finish (atomic ticket, no waiting) merges
// the partials with a log-sum-exp combine into out[b, h, :] and resets the
// ticket.
#include <algorithm>
#include <map>
#include <mutex>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kRing = 8;                // rows in flight per warp
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSpanRetMax = 8192;       // positions per retrieval split (max)
constexpr int kSpanLoc = 1024;          // rows per local split

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
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

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

struct AttShared {
  Group grp;
  int seg_lo[kMaxGroup];
  int seg_hi[kMaxGroup];
  int n_union;
  uint32_t wtot[kWarps];
  int last;
};

struct AttParams {
  int ns_r, span_r, ns_l, ns_max;
};

// dynamic shared memory: [ring: kWarps x kRing rows x 4D bytes]
//                        [union list: span_r x uint32 (offset << 16 | mask)]
//                        [per-head bitmaps: GR x span_r / 32 words]
// after the row loop it holds the warps' (m, l, acc) for the CTA merge
template <int D, int GR>
__global__ void __launch_bounds__(kThreads)
attend_kernel(const AttendArgs a, const Shape sh, const Tables tb, const AttParams ap) {
  constexpr int E = D / 32;                         // elements per lane
  constexpr int kRowBytes = 4 * D;                  // K row + V row, bf16
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ AttShared S;
  extern __shared__ __align__(128) unsigned char dyn[];
  unsigned char *ring = dyn;
  uint32_t *ulist = reinterpret_cast<uint32_t *>(dyn + (size_t)kWarps * kRing * kRowBytes);
  uint32_t *hbm = ulist + ap.span_r;
  const int bwords = ap.span_r / 32;

  // ---- decode the work item ------------------------------------------------
  long long bid = blockIdx.x;
  const long long n_ret_items = (long long)a.batch * tb.n_ret * ap.ns_r;
  const bool is_ret = bid < n_ret_items;
  int b, gi, split, ns;
  if (is_ret) {
    b = (int)(bid / ((long long)tb.n_ret * ap.ns_r));
    const long long rem = bid % ((long long)tb.n_ret * ap.ns_r);
    gi = (int)(rem / ap.ns_r);
    split = (int)(rem % ap.ns_r);
    ns = ap.ns_r;
  } else {
    bid -= n_ret_items;
    const int nsl = std::max(ap.ns_l, 1);
    b = (int)(bid / ((long long)tb.n_loc * nsl));
    const long long rem = bid % ((long long)tb.n_loc * nsl);
    gi = (int)(rem / nsl);
    split = (int)(rem % nsl);
    ns = nsl;
  }
  if (tid == 0) S.grp = is_ret ? tb.ret[gi] : tb.loc[gi];
  __syncthreads();
  const int nh = S.grp.n;
  const int g = S.grp.kv_head;
  long long N = a.seq_lens[b];
  if (N < 0 || N > sh.max_len) {
    if (tid == 0 && split == 0) raise_error(a.err, SD_EBIT_SEQLEN);
    N = N < 0 ? 0 : sh.max_len;
  }
  const int32_t *pt = a.page_table + (long long)b * sh.max_pages;

  // ---- rows of this item ---------------------------------------------------
  int n_rows = 0;
  long long p0 = 0;                                  // retrieval: first position of the span
  long long loc_a = 0, loc_w = 0, row0 = 0;          // local: sinks, window start, first row
  if (is_ret) {
    p0 = (long long)split * ap.span_r;
    const long long p1 = std::min(N, p0 + ap.span_r);
    if (p0 < N) {
      for (int i = warp; i < nh; i += kWarps) {
        const int32_t *row = a.sel_idx + ((long long)b * sh.H_ret + S.grp.row[i]) * a.sel_stride;
        long long c = a.sel_count[(long long)b * sh.H_ret + S.grp.row[i]];
        if (c < 0 || c > a.sel_stride) {
          if (lane == 0) raise_error(a.err, SD_EBIT_SEL);
          c = c < 0 ? 0 : a.sel_stride;
        }
        const int lo = warp_lower_bound(row, (int)c, (int)p0, lane);
        const int hi = warp_lower_bound(row, (int)c, (int)p1, lane);
        if (lane == 0) {
          S.seg_lo[i] = lo;
          S.seg_hi[i] = hi;
        }
      }
      for (int o = tid; o < nh * bwords; o += kThreads) hbm[o] = 0u;
      __syncthreads();
      for (int i = 0; i < nh; ++i) {
        const int32_t *row = a.sel_idx + ((long long)b * sh.H_ret + S.grp.row[i]) * a.sel_stride;
        for (int e = S.seg_lo[i] + tid; e < S.seg_hi[i]; e += kThreads) {
          const long long pos = row[e];
          if (pos < p0 || pos >= p1) {
            raise_error(a.err, SD_EBIT_SEL);
            continue;
          }
          const int off = (int)(pos - p0);
          atomicOr(&hbm[i * bwords + (off >> 5)], 1u << (off & 31));
        }
      }
      __syncthreads();
      // ordered compaction of the union: contiguous word ranges per thread
      const int wpt = (bwords + kThreads - 1) / kThreads;
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
      if (lane == 31) S.wtot[warp] = incl;
      __syncthreads();
      uint32_t base = 0, total = 0;
      for (int x = 0; x < kWarps; ++x) {
        if (x < warp) base += S.wtot[x];
        total += S.wtot[x];
      }
      uint32_t o = base + incl - c;
      for (int x = w0; x < w1; ++x) {
        uint32_t u = 0;
        for (int i = 0; i < nh; ++i) u |= hbm[i * bwords + x];
        while (u) {
          const int bit = __ffs(u) - 1;
          u &= u - 1;
          uint32_t m = 0;
          for (int i = 0; i < nh; ++i) m |= ((hbm[i * bwords + x] >> bit) & 1u) << i;
          ulist[o++] = ((uint32_t)(x * 32 + bit) << 16) | m;
        }
      }
      if (tid == 0) S.n_union = (int)total;
      __syncthreads();
      n_rows = S.n_union;
    }
  } else {
    loc_a = std::min<long long>(a.num_sinks, N);
    loc_w = std::max<long long>(loc_a, N - a.window);
    const long long L = loc_a + (N - loc_w);
    row0 = (long long)split * kSpanLoc;
    n_rows = (int)std::max<long long>(0, std::min<long long>(kSpanLoc, L - row0));
  }
  const uint32_t all_mask = (nh >= 32) ? 0xFFFFFFFFu : ((1u << nh) - 1u);

  // ---- per-warp row ring: rows warp, warp + 8, ... ----------------------------
  const uint32_t ring_base = (uint32_t)__cvta_generic_to_shared(ring) + warp * (kRing * kRowBytes);
  const int nq = n_rows > warp ? (n_rows - warp + kWarps - 1) / kWarps : 0;
  auto row_info = [&](int u, long long &pos, uint32_t &m) {
    if (is_ret) {
      const uint32_t e = ulist[u];
      pos = p0 + (e >> 16);
      m = e & 0xFFFFu;
    } else {
      const long long rr = row0 + u;
      pos = rr < loc_a ? rr : loc_w + (rr - loc_a);
      m = all_mask;
    }
  };
  // lanes [0, D/8) copy the K row, lanes [16, 16 + D/8) the V row
  const int half = lane >> 4, hl = lane & 15;
  const bool copier = hl < D / 8;
  auto issue = [&](int q) {
    if (q < nq) {
      long long pos;
      uint32_t m;
      row_info(warp + q * kWarps, pos, m);
      const int page = pt[pos / kPage];
      const bool ok = page >= 0 && page < sh.num_pages;
      if (!ok && lane == 0) raise_error(a.err, SD_EBIT_PAGE);
      const long long off = (((long long)page * sh.Hkv + g) * kPage + (pos % kPage)) * D + hl * 8;
      const uint16_t *src = (half ? a.v_cache : a.k_cache) + (ok ? off : 0);
      if (copier)
        cp_async16(ring_base + (q % kRing) * kRowBytes + half * (2 * D) + hl * 16, src, ok ? 16 : 0);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int q = 0; q < kRing; ++q) issue(q);

  float qv[GR][E];
  {
    const float sc = a.attn_scale * kLog2e;
#pragma unroll
    for (int i = 0; i < GR; ++i) {
#pragma unroll
      for (int e = 0; e < E; ++e) qv[i][e] = 0.0f;
      if (i < nh) {
        const uint16_t *qp = a.q + ((long long)b * sh.Hq + S.grp.q_head[i]) * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) qv[i][e] = bf16_to_f32(qp[e]) * sc;
      }
    }
  }
  float m_[GR], l_[GR], acc[GR][E];
#pragma unroll
  for (int i = 0; i < GR; ++i) {
    m_[i] = -INFINITY;
    l_[i] = 0.0f;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[i][e] = 0.0f;
  }
  for (int q = 0; q < nq; ++q) {
    cp_async_wait<kRing - 1>();
    __syncwarp();
    long long pos;
    uint32_t m;
    row_info(warp + q * kWarps, pos, m);
    const int page = pt[pos / kPage];
    if (page < 0 || page >= sh.num_pages) m = 0u;
    const unsigned char *slot = ring + (size_t)(warp * kRing + q % kRing) * kRowBytes;
    float kf[E], vf[E];
    if constexpr (E == 4) {
      const uint2 kw = *reinterpret_cast<const uint2 *>(slot + lane * 8);
      const uint2 vw = *reinterpret_cast<const uint2 *>(slot + 2 * D + lane * 8);
      kf[0] = bf16_lo(kw.x); kf[1] = bf16_hi(kw.x); kf[2] = bf16_lo(kw.y); kf[3] = bf16_hi(kw.y);
      vf[0] = bf16_lo(vw.x); vf[1] = bf16_hi(vw.x); vf[2] = bf16_lo(vw.y); vf[3] = bf16_hi(vw.y);
    } else {
      const uint32_t kw = *reinterpret_cast<const uint32_t *>(slot + lane * 4);
      const uint32_t vw = *reinterpret_cast<const uint32_t *>(slot + 2 * D + lane * 4);
      kf[0] = bf16_lo(kw); kf[1] = bf16_hi(kw);
      vf[0] = bf16_lo(vw); vf[1] = bf16_hi(vw);
    }
    __syncwarp();
    issue(q + kRing);
#pragma unroll
    for (int i = 0; i < GR; ++i) {
      if (!((m >> i) & 1u)) continue;
      float dot = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) dot = fmaf(qv[i][e], kf[e], dot);
      dot = warp_sum(dot);
      const float mn = fmaxf(m_[i], dot);
      const float alpha = exp2f(m_[i] - mn);
      const float p = exp2f(dot - mn);
      l_[i] = fmaf(l_[i], alpha, p);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[i][e] = fmaf(acc[i][e], alpha, p * vf[e]);
      m_[i] = mn;
    }
  }
  cp_async_wait<0>();

  // ---- merge the warps of the CTA, write the partial -----------------------
  __syncthreads();                                   // ring and union list no longer read
  float *cm = reinterpret_cast<float *>(dyn);                    // [kWarps][GR]
  float *cl = cm + kWarps * GR;                                  // [kWarps][GR]
  float *cacc = cl + kWarps * GR;                                // [kWarps][GR][D]
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < GR; ++i) {
      cm[warp * GR + i] = m_[i];
      cl[warp * GR + i] = l_[i];
    }
  }
#pragma unroll
  for (int i = 0; i < GR; ++i)
#pragma unroll
    for (int e = 0; e < E; ++e) cacc[(warp * GR + i) * D + lane * E + e] = acc[i][e];
  __syncthreads();
  const int role = is_ret ? 0 : 1;
  for (int o = tid; o < nh * (D + 2); o += kThreads) {
    const int i = o / (D + 2), c = o % (D + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, cm[w * GR + i]);
    float v;
    if (c == 0) {
      v = M;
    } else {
      v = 0.0f;
      if (M > -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float f = exp2f(cm[w * GR + i] - M);
          v += f * (c == 1 ? cl[w * GR + i] : cacc[(w * GR + i) * D + (c - 2)]);
        }
      }
    }
    const long long h = S.grp.q_head[i];
    a.partials[(((long long)b * sh.Hq + h) * ap.ns_max + split) * (D + 2) + c] = v;
  }
  __threadfence();
  __syncthreads();
  unsigned *ticket = a.tickets + ((long long)b * sh.Hkv + g) * 2 + role;
  if (tid == 0) S.last = (atomicAdd(ticket, 1u) == (unsigned)(ns - 1));
  __syncthreads();
  if (!S.last) return;
  __threadfence();

  // ---- last CTA of the item: merge all splits into out ----------------------
  for (int o = tid; o < nh * D; o += kThreads) {
    const int i = o / D, c = o % D;
    const long long h = S.grp.q_head[i];
    const float *pp = a.partials + ((long long)b * sh.Hq + h) * ap.ns_max * (D + 2);
    float M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, __ldcg(pp + (long long)s * (D + 2)));
    float num = 0.0f, den = 0.0f;
    if (M > -INFINITY) {
      for (int s = 0; s < ns; ++s) {
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

int pow2_ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

int group_rows_att(const Tables &tb) { return pow2_ceil(std::max(1, std::max(tb.max_ret, tb.max_loc))); }

AttParams att_params(const Shape &sh, const Tables &tb, int window, int sinks) {
  AttParams p{};
  const long long L = sh.max_len;
  const int span = pow2_ceil((int)std::max<long long>(1, (L + 15) / 16));
  p.span_r = std::max(256, std::min(kSpanRetMax, span));
  p.ns_r = (int)((L + p.span_r - 1) / p.span_r);
  p.ns_l = 0;
  if (tb.n_loc > 0) {
    const long long rows = std::min<long long>(L, (long long)window + sinks);
    p.ns_l = (int)std::max<long long>(1, (rows + kSpanLoc - 1) / kSpanLoc);
  }
  // partial rows are laid out with the largest split count any call can use
  p.ns_max = (int)std::max<long long>(p.ns_r, (L + kSpanLoc - 1) / kSpanLoc);
  return p;
}

size_t att_smem(int D, int GR, int span_r) {
  const size_t ring = (size_t)kWarps * kRing * 4 * D;
  const size_t lists = (size_t)span_r * 4 + (size_t)GR * (span_r / 32) * 4;
  const size_t merge = (size_t)kWarps * GR * (D + 2) * 4;
  return std::max(ring + lists, merge);
}

template <int D, int GR>
cudaError_t launch_t(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &p, cudaStream_t st) {
  auto kern = attend_kernel<D, GR>;
  const size_t bytes = att_smem(D, GR, p.span_r);
  static std::mutex mu;
  static std::map<int, size_t> configured;     // device -> dynamic smem bytes set
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = configured.find(dev);
    if (it == configured.end() || it->second < bytes) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
      if (e != cudaSuccess) return e;
      configured[dev] = bytes;
    }
  }
  const long long blocks = (long long)a.batch * ((long long)tb.n_ret * p.ns_r + (long long)tb.n_loc * p.ns_l);
  if (blocks == 0) return cudaSuccess;
  kern<<<(unsigned)blocks, kThreads, bytes, st>>>(a, sh, tb, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_gr(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttParams &p, cudaStream_t st) {
  switch (group_rows_att(tb)) {
    case 1: return launch_t<D, 1>(a, sh, tb, p, st);
    case 2: return launch_t<D, 2>(a, sh, tb, p, st);
    case 4: return launch_t<D, 4>(a, sh, tb, p, st);
    case 8: return launch_t<D, 8>(a, sh, tb, p, st);
    default: return launch_t<D, 16>(a, sh, tb, p, st);
  }
}

}  // namespace

size_t attend_workspace_bytes(const Shape &sh, const Tables &tb, int batch, size_t *tickets_off) {
  const AttParams p = att_params(sh, tb, 0, 0);
  size_t part = (size_t)batch * sh.Hq * (size_t)p.ns_max * (sh.d + 2) * sizeof(float);
  part = (part + 255) / 256 * 256;
  if (tickets_off) *tickets_off = part;
  return part + (size_t)batch * sh.Hkv * 2 * sizeof(unsigned);
}

cudaError_t launch_attend(const AttendArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st) {
  if (a.batch == 0) return cudaSuccess;
  const AttParams p = att_params(sh, tb, a.window, a.num_sinks);
  cudaError_t e = cudaMemsetAsync(a.tickets, 0, (size_t)a.batch * sh.Hkv * 2 * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  return sh.d == 128 ? dispatch_gr<128>(a, sh, tb, p, st) : dispatch_gr<64>(a, sh, tb, p, st);
}

}  // namespace sd
