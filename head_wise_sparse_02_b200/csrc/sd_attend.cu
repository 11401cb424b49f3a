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
//              a warp-cooperative search, merges them into a union with a head
//              mask per position, and reads every union row once for all the
//              group's heads that selected it;
//   local      split s covers rows [s*span, (s+1)*span) of the enumerated set
//              [0, sinks) U [N - window, N); every local head of the group uses
//              every row.
// Each warp walks its rows with several rows' K/V slices in flight (each lane
// holds d/32 consecutive elements), keeps a float32 online softmax per head in
// base 2, and the CTA merges its warps.  The partial (m, l, acc[d]) of each
// (b, head, split) goes to the workspace; the last CTA of a (b, g, role) to
// finish (atomic ticket, no waiting) merges the partials with a log-sum-exp
// combine into out[b, h, :] and resets the ticket.
#include <algorithm>
#include <map>
#include <mutex>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kRowsInFlight = 8;        // per warp
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSpanRet = 2048;          // positions per retrieval split (max)
constexpr int kSpanLoc = 512;           // rows per local split

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

template <int E>
struct Slice;
template <>
struct Slice<4> {                        // d = 128: 4 bf16 per lane
  uint2 v;
  __device__ void load(const uint16_t *p) { v = __ldg(reinterpret_cast<const uint2 *>(p)); }
  __device__ void zero() { v = make_uint2(0u, 0u); }
  __device__ void unpack(float *f) const {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x); f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
  }
};
template <>
struct Slice<2> {                        // d = 64: 2 bf16 per lane
  uint32_t v;
  __device__ void load(const uint16_t *p) { v = __ldg(reinterpret_cast<const uint32_t *>(p)); }
  __device__ void zero() { v = 0u; }
  __device__ void unpack(float *f) const { f[0] = bf16_lo(v); f[1] = bf16_hi(v); }
};

struct AttShared {
  Group grp;
  int seg_lo[kMaxGroup];
  int seg_hi[kMaxGroup];
  int n_union;
  int warp_base[kWarps + 1];
  int last;
};

template <int D, int GR>
__global__ void __launch_bounds__(kThreads)
attend_kernel(const AttendArgs a, const Shape sh, const Tables tb, int ns_r, int span_r, int ns_l,
              int ns_max) {
  constexpr int E = D / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ AttShared S;
  __shared__ float cm[kWarps][GR], cl[kWarps][GR];
  extern __shared__ __align__(16) unsigned char dyn[];
  uint32_t *bm = reinterpret_cast<uint32_t *>(dyn);         // [span_r] head masks per position
  int32_t *upos = reinterpret_cast<int32_t *>(bm + span_r);  // [span_r] union positions
  uint32_t *umask = reinterpret_cast<uint32_t *>(upos + span_r);
  float *cacc = reinterpret_cast<float *>(dyn);             // reused after the loop: [kWarps][GR][D]

  // ---- decode the work item ------------------------------------------------
  long long bid = blockIdx.x;
  const long long n_ret_items = (long long)a.batch * tb.n_ret * ns_r;
  const bool is_ret = bid < n_ret_items;
  int b, gi, split, ns;
  if (is_ret) {
    b = (int)(bid / ((long long)tb.n_ret * ns_r));
    const long long rem = bid % ((long long)tb.n_ret * ns_r);
    gi = (int)(rem / ns_r);
    split = (int)(rem % ns_r);
    ns = ns_r;
  } else {
    bid -= n_ret_items;
    const int ns_l_ = std::max(ns_l, 1);
    b = (int)(bid / ((long long)tb.n_loc * ns_l_));
    const long long rem = bid % ((long long)tb.n_loc * ns_l_);
    gi = (int)(rem / ns_l_);
    split = (int)(rem % ns_l_);
    ns = ns_l_;
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
  long long loc_a = 0, loc_w = 0, row0 = 0;       // local: sinks count, window start, first row
  if (is_ret) {
    const long long p0 = (long long)split * span_r;
    const long long p1 = std::min(N, p0 + span_r);
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
      for (int o = tid; o < span_r; o += kThreads) bm[o] = 0u;
      __syncthreads();
      for (int i = 0; i < nh; ++i) {
        const int32_t *row = a.sel_idx + ((long long)b * sh.H_ret + S.grp.row[i]) * a.sel_stride;
        for (int e = S.seg_lo[i] + tid; e < S.seg_hi[i]; e += kThreads) {
          const long long pos = row[e];
          if (pos < p0 || pos >= p1) {
            raise_error(a.err, SD_EBIT_SEL);
            continue;
          }
          atomicOr(&bm[pos - p0], 1u << i);
        }
      }
      __syncthreads();
      // ordered compaction: warp w owns a contiguous quarter of the span
      const int q = (span_r + kWarps - 1) / kWarps;
      const int q0 = warp * q, q1 = std::min(span_r, q0 + q);
      int c = 0;
      for (int base = q0; base < q1; base += 32) {
        const int o = base + lane;
        c += __popc(__ballot_sync(kFull, o < q1 && bm[o] != 0u));
      }
      if (lane == 0) S.warp_base[warp + 1] = c;
      __syncthreads();
      if (tid == 0) {
        S.warp_base[0] = 0;
        for (int w = 0; w < kWarps; ++w) S.warp_base[w + 1] += S.warp_base[w];
        S.n_union = S.warp_base[kWarps];
      }
      __syncthreads();
      int off = S.warp_base[warp];
      for (int base = q0; base < q1; base += 32) {
        const int o = base + lane;
        const uint32_t m = (o < q1) ? bm[o] : 0u;
        const unsigned bal = __ballot_sync(kFull, m != 0u);
        if (m) {
          const int dst = off + __popc(bal & ((1u << lane) - 1u));
          upos[dst] = (int32_t)(p0 + o);
          umask[dst] = m;
        }
        off += __popc(bal);
      }
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

  // ---- gather + online softmax --------------------------------------------
  float qv[GR][E];
  {
    const float sc = a.attn_scale * kLog2e;
#pragma unroll
    for (int i = 0; i < GR; ++i) {
      float f[E];
      if (i < nh) {
        Slice<E> s;
        s.load(a.q + ((long long)b * sh.Hq + S.grp.q_head[i]) * D + lane * E);
        s.unpack(f);
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) f[e] = 0.0f;
      }
#pragma unroll
      for (int e = 0; e < E; ++e) qv[i][e] = f[e] * sc;
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
  const uint32_t all_mask = (nh >= 32) ? 0xFFFFFFFFu : ((1u << nh) - 1u);
  for (int u0 = warp * kRowsInFlight; u0 < n_rows; u0 += kWarps * kRowsInFlight) {
    Slice<E> ks[kRowsInFlight], vs[kRowsInFlight];
    uint32_t mk[kRowsInFlight];
#pragma unroll
    for (int r = 0; r < kRowsInFlight; ++r) {
      const int u = u0 + r;
      mk[r] = 0u;
      ks[r].zero();
      vs[r].zero();
      if (u < n_rows) {
        long long pos;
        uint32_t m;
        if (is_ret) {
          pos = upos[u];
          m = umask[u];
        } else {
          const long long rr = row0 + u;
          pos = rr < loc_a ? rr : loc_w + (rr - loc_a);
          m = all_mask;
        }
        const int page = pt[pos / kPage];
        if (page >= 0 && page < sh.num_pages) {
          const long long off = (((long long)page * sh.Hkv + g) * kPage + (pos % kPage)) * D + lane * E;
          ks[r].load(a.k_cache + off);
          vs[r].load(a.v_cache + off);
          mk[r] = m;
        } else if (lane == 0) {
          raise_error(a.err, SD_EBIT_PAGE);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsInFlight; ++r) {
      if (mk[r] == 0u) continue;
      float kf[E], vf[E];
      ks[r].unpack(kf);
      vs[r].unpack(vf);
#pragma unroll
      for (int i = 0; i < GR; ++i) {
        if (!((mk[r] >> i) & 1u)) continue;
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
  }

  // ---- merge the warps of the CTA, write the partial -----------------------
  __syncthreads();                                   // union arrays are no longer read
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < GR; ++i) {
      cm[warp][i] = m_[i];
      cl[warp][i] = l_[i];
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
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, cm[w][i]);
    float v;
    if (c == 0) {
      v = M;
    } else {
      v = 0.0f;
      if (M > -INFINITY) {
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
          const float f = exp2f(cm[w][i] - M);
          v += f * (c == 1 ? cl[w][i] : cacc[(w * GR + i) * D + (c - 2)]);
        }
      }
    }
    const long long h = S.grp.q_head[i];
    a.partials[(((long long)b * sh.Hq + h) * ns_max + split) * (D + 2) + c] = v;
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
    const float *pp = a.partials + ((long long)b * sh.Hq + h) * ns_max * (D + 2);
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

struct AttPlan {
  int ns_r, span_r, ns_l, ns_max;
  size_t dyn_bytes;
};

AttPlan make_plan(const Shape &sh, const Tables &tb, int D) {
  AttPlan p{};
  const long long L = sh.max_len;
  int span = pow2_ceil((int)std::max<long long>(1, (L + 31) / 32));
  span = std::max(256, std::min(kSpanRet, span));
  p.span_r = span;
  p.ns_r = (int)((L + span - 1) / span);
  p.ns_l = 0;
  if (tb.n_loc > 0) {
    // rows of a local set: at most sinks + window, never more than the context
    p.ns_l = 1;   // refined at launch from the window size
  }
  p.ns_max = p.ns_r;
  const int GR = pow2_ceil(std::max(1, std::max(tb.max_ret, tb.max_loc)));
  const size_t uni = (size_t)span * 3 * sizeof(uint32_t);
  const size_t comb = (size_t)kWarps * GR * D * sizeof(float);
  p.dyn_bytes = std::max(uni, comb);
  return p;
}

template <int D, int GR>
cudaError_t launch_t(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttPlan &p, cudaStream_t st) {
  auto kern = attend_kernel<D, GR>;
  static std::mutex mu;
  static std::map<int, size_t> configured;     // device -> dynamic smem bytes set
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = configured.find(dev);
    if (it == configured.end() || it->second < p.dyn_bytes) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.dyn_bytes);
      if (e != cudaSuccess) return e;
      configured[dev] = p.dyn_bytes;
    }
  }
  const long long blocks = (long long)a.batch * ((long long)tb.n_ret * p.ns_r + (long long)tb.n_loc * p.ns_l);
  if (blocks == 0) return cudaSuccess;
  kern<<<(unsigned)blocks, kThreads, p.dyn_bytes, st>>>(a, sh, tb, p.ns_r, p.span_r, p.ns_l, p.ns_max);
  return cudaGetLastError();
}

template <int D>
cudaError_t dispatch_gr(const AttendArgs &a, const Shape &sh, const Tables &tb, const AttPlan &p, cudaStream_t st) {
  switch (pow2_ceil(std::max(1, std::max(tb.max_ret, tb.max_loc)))) {
    case 1: return launch_t<D, 1>(a, sh, tb, p, st);
    case 2: return launch_t<D, 2>(a, sh, tb, p, st);
    case 4: return launch_t<D, 4>(a, sh, tb, p, st);
    case 8: return launch_t<D, 8>(a, sh, tb, p, st);
    default: return launch_t<D, 16>(a, sh, tb, p, st);
  }
}

AttPlan full_plan(const Shape &sh, const Tables &tb, int window, int sinks) {
  AttPlan p = make_plan(sh, tb, sh.d);
  if (tb.n_loc > 0) {
    const long long rows = std::min<long long>(sh.max_len, (long long)window + sinks);
    p.ns_l = (int)std::max<long long>(1, (rows + kSpanLoc - 1) / kSpanLoc);
  }
  p.ns_max = std::max(p.ns_r, p.ns_l);
  return p;
}

}  // namespace

size_t attend_workspace_bytes(const Shape &sh, const Tables &tb, int batch, size_t *tickets_off) {
  // The local split count depends on the window; size for the worst case
  // (every split of the longest context).
  const AttPlan p = make_plan(sh, tb, sh.d);
  const long long ns_max = std::max<long long>(p.ns_r, (sh.max_len + kSpanLoc - 1) / kSpanLoc);
  size_t part = (size_t)batch * sh.Hq * (size_t)ns_max * (sh.d + 2) * sizeof(float);
  part = (part + 255) / 256 * 256;
  if (tickets_off) *tickets_off = part;
  return part + (size_t)batch * sh.Hkv * 2 * sizeof(unsigned);
}

cudaError_t launch_attend(const AttendArgs &a0, const Shape &sh, const Tables &tb, cudaStream_t st) {
  if (a0.batch == 0) return cudaSuccess;
  AttendArgs a = a0;
  const AttPlan p0 = full_plan(sh, tb, a.window, a.num_sinks);
  // partial rows are laid out with the worst-case split count used for sizing
  AttPlan p = p0;
  p.ns_max = (int)std::max<long long>(p.ns_r, (sh.max_len + kSpanLoc - 1) / kSpanLoc);
  cudaError_t e = cudaMemsetAsync(a.tickets, 0, (size_t)a.batch * sh.Hkv * 2 * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  return sh.d == 128 ? dispatch_gr<128>(a, sh, tb, p, st) : dispatch_gr<64>(a, sh, tb, p, st);
}

}  // namespace sd
