// Fixed-budget (top-k) selection in one pass over the index.
//
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 2-3 and 5: the
// tokens of a retrieval head are scored in the r = 16 index space and a fixed
// top-k budget is taken; the threshold comes from a histogram, without
// sorting.  ICS page (gist.science/ar/paper/2605.24168), 2 and 3a: exact
// ("Oracle") top-k at ~2% of the context.
//
// One thread-block cluster of C CTAs per (sequence, KV group); each CTA owns a
// page-aligned chunk of the context and reads its index entries once.
//
//   1. Scores on the tensor cores: a 16-token page of the index of one KV
//      head (16 x 16 bf16) is the A operand of mma.m16n8k16; the B operand
//      holds q~ of the group's heads split into three bf16 terms
//      (q~ = hi + mid + lo, each the bf16 rounding of the remainder), so the
//      float32 accumulation reproduces the float32 score to ~2^-24 relative.
//   2. Each CTA first scores a strided sample of its pages (<= 64 pages) and
//      derives from it a conservative score window [t_lo, t_hi): t_lo is a
//      sample quantile safely below the k-th score, t_hi the sample maximum.
//      The cluster agrees on the widest window (min of t_lo, max of t_hi).
//   3. Streaming the rest of the chunk, every score at or above t_lo goes to
//      a small per-head list (score, position) and, when below t_hi, to a
//      512-bin linear histogram of the window.  Nothing else is kept.
//   4. The histograms are reduced across the cluster (distributed shared
//      memory); the bin holding the k-th score is found scanning down from
//      the top, and the few tokens of that bin are sent to the head's owner
//      CTA, which ranks them exactly by (score desc, position asc).  This
//      yields the threshold as a (score, position) pair.
//   5. Each CTA marks its selected list entries in a bitmap of its chunk and
//      writes their positions in ascending order at its cluster offset.
// If the window misses (list overflow, k-th score outside the window, too
// many candidates in the cut bin), the cluster flags its work item and the
// exact general kernel recomputes it.
#include <cooperative_groups.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "sd_internal.cuh"

namespace cg = cooperative_groups;

namespace sd {
namespace {

constexpr int kT = 256;
constexpr int kW = kT / 32;
constexpr int kBins = 512;            // window histogram
constexpr int kTopClass = kBins;      // class of scores at or above t_hi
constexpr int kSampleTiles = 64;      // sampled pages per CTA
constexpr int kSampleBins = 64;
constexpr int kCap = 1024;            // cut-bin candidates ranked exactly per head
constexpr int kMaxCluster = 16;
constexpr int kUnroll = 4;            // pages in flight per warp
constexpr unsigned kFull = 0xFFFFFFFFu;

struct TopkParams {
  int tc_cap;                         // tokens per CTA (capacity, multiple of 16)
  int list_cap;                       // list entries per head per CTA
  int own_slots;                      // heads owned per CTA
  uint32_t *fail;                     // [items]: 1 = needs the exact general kernel
};

struct TkShared {
  Group grp;
  uint32_t qs[3][kMaxGroup][kIndexDim / 2];   // q~ terms hi / mid / lo, bf16 pairs
  uint32_t smax[kMaxGroup], smin[kMaxGroup];
  uint32_t tlo_key[kMaxGroup], thi_key[kMaxGroup];
  float tlo[kMaxGroup], thi[kMaxGroup], inv[kMaxGroup];
  uint32_t list_n[kMaxGroup];
  uint32_t top_n[kMaxGroup];
  uint32_t overflow;
  uint32_t slice_cnt[kMaxGroup];
  int cut[kMaxGroup];
  long long need_c[kMaxGroup];
  int fail;
  uint32_t above_local[kMaxGroup];
  uint32_t cand_n[kMaxGroup];
  unsigned long long tau_sk[kMaxGroup];
  uint32_t wtot[kW];
};

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}

__device__ __forceinline__ double bf16_bits_to_f64(uint16_t h) { return (double)__uint_as_float(uint32_t(h) << 16); }

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;\n" ::: "memory"); }

// sort key: ascending order = score descending, then position ascending
__device__ __forceinline__ unsigned long long sort_key(float s, uint32_t pos) {
  return ((unsigned long long)(~order_key(s)) << 32) | pos;
}

struct TkLayout {
  size_t sample, whist, wred, list, cand, occ, bitmap, total;
};

__host__ __device__ inline TkLayout tk_layout(int GR, int tc_cap, int list_cap, int own_slots) {
  TkLayout L{};
  size_t o = 0;
  L.list = o;   o += (size_t)GR * list_cap * 8;
  L.cand = o;   o += (size_t)own_slots * kCap * 8;
  L.sample = o; o += (size_t)GR * kSampleTiles * 16 * 4;
  L.whist = o;  o += (size_t)GR * kBins * 4;
  L.wred = o;   o += (size_t)GR * kBins * 4;
  L.occ = o;    o += (size_t)own_slots * kMaxCluster * 4;
  L.bitmap = o; o += (size_t)GR * (tc_cap / 32) * 4;
  L.total = o;
  return L;
}

template <int GR>
__global__ void __launch_bounds__(kT, 2)
topk_kernel(const SelectArgs a, const Shape sh, const Group *__restrict__ groups, int n_groups,
            const TopkParams tp) {
  constexpr int HB = (GR + 3) / 4;                   // 4-head blocks of the MMA
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int item = blockIdx.y;
  const int b = item / n_groups, gi = item % n_groups;

  __shared__ TkShared S;
  extern __shared__ __align__(16) unsigned char dyn[];
  const TkLayout L = tk_layout(GR, tp.tc_cap, tp.list_cap, tp.own_slots);
  unsigned long long *list = reinterpret_cast<unsigned long long *>(dyn + L.list);
  unsigned long long *cand = reinterpret_cast<unsigned long long *>(dyn + L.cand);
  float *sample = reinterpret_cast<float *>(dyn + L.sample);
  uint32_t *whist = reinterpret_cast<uint32_t *>(dyn + L.whist);
  uint32_t *wred = reinterpret_cast<uint32_t *>(dyn + L.wred);
  uint32_t *occ = reinterpret_cast<uint32_t *>(dyn + L.occ);
  uint32_t *bitmap = reinterpret_cast<uint32_t *>(dyn + L.bitmap);
  const int words = tp.tc_cap / 32;

  if (tid == 0) S.grp = groups[gi];
  __syncthreads();
  const int nr = S.grp.n;
  const int g = S.grp.kv_head;

  long long N = a.seq_lens[b];
  if (N < 0 || N > sh.max_len) {
    if (tid == 0 && rank == 0) raise_error(a.err, SD_EBIT_SEQLEN);
    N = N < 0 ? 0 : sh.max_len;
  }
  const long long per_cta = ((N + C - 1) / C + kPage - 1) / kPage * kPage;
  const long long t0 = std::min(N, (long long)rank * per_cta);
  const long long t1 = std::min(N, t0 + per_cta);
  const int cnt = (int)(t1 - t0);
  const int ntiles = (cnt + kPage - 1) / kPage;

  auto sel_row = [&](int i) { return a.sel_idx + ((long long)b * sh.H_ret + S.grp.row[i]) * a.sel_stride; };
  auto count_slot = [&](int i) { return a.sel_count + (long long)b * sh.H_ret + S.grp.row[i]; };

  long long kb = a.top_k > 0 ? (long long)a.top_k
                             : std::max(1LL, (long long)floor((double)a.top_k_frac * (double)N));
  kb = std::min(kb, N);
  if (N == 0 || kb >= N) {                           // the whole context (or nothing)
    for (int i = 0; i < nr; ++i) {
      int32_t *row = sel_row(i);
      for (long long t = t0 + tid; t < t1; t += kT) {
        if (t < a.sel_stride) row[t] = (int32_t)t;
        else raise_error(a.err, SD_EBIT_SEL);
      }
      if (rank == 0 && tid == 0) *count_slot(i) = (int32_t)std::min(N, a.sel_stride);
    }
    if (rank == 0 && tid == 0) tp.fail[item] = 0u;
    return;
  }

  // ---- q~ = c P_g^T q_pre in float64, split into three bf16 terms ----------
  for (int o = tid; o < kMaxGroup * kIndexDim; o += kT) {
    const int i = o / kIndexDim, j = o % kIndexDim;
    uint16_t hi = 0, mid = 0, lo = 0;
    if (i < nr) {
      const uint16_t *qrow = a.q_pre + ((long long)b * sh.Hq + S.grp.q_head[i]) * sh.d;
      const uint16_t *P = a.proj + (long long)g * sh.d * kIndexDim;
      double acc = 0.0;
      for (int e = 0; e < sh.d; ++e)
        acc = fma((double)bf16_to_f32(qrow[e]), (double)bf16_to_f32(P[e * kIndexDim + j]), acc);
      acc *= (double)a.index_scale;
      hi = f64_to_bf16_rne(acc);
      const double r1 = acc - bf16_bits_to_f64(hi);
      mid = f64_to_bf16_rne(r1);
      lo = f64_to_bf16_rne(r1 - bf16_bits_to_f64(mid));
    }
    uint16_t *q0 = reinterpret_cast<uint16_t *>(&S.qs[0][i][0]);
    uint16_t *q1 = reinterpret_cast<uint16_t *>(&S.qs[1][i][0]);
    uint16_t *q2 = reinterpret_cast<uint16_t *>(&S.qs[2][i][0]);
    q0[j] = hi;
    q1[j] = mid;
    q2[j] = lo;
  }
  if (tid < kMaxGroup) {
    S.smax[tid] = 0u;
    S.smin[tid] = 0xFFFFFFFFu;
    S.list_n[tid] = 0u;
    S.top_n[tid] = 0u;
    S.cand_n[tid] = 0u;
    S.above_local[tid] = 0u;
  }
  if (tid == 0) {
    S.overflow = 0u;
    S.fail = 0;
  }
  for (int o = tid; o < GR * kBins; o += kT) whist[o] = 0u;
  for (int o = tid; o < tp.own_slots * kMaxCluster; o += kT) occ[o] = 0u;
  for (int o = tid; o < GR * words; o += kT) bitmap[o] = 0u;
  __syncthreads();

  // B fragments: column n = gq of the first MMA carries head 4hb + gq/2, term
  // gq%2 (hi, mid); of the second MMA, the lo term for even gq, zero for odd.
  uint32_t bf[HB][2][2];
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) {
    const int head = hb * 4 + (gq >> 1);
    const int part = gq & 1;
    bf[hb][0][0] = S.qs[part][head][tq];
    bf[hb][0][1] = S.qs[part][head][tq + 4];
    bf[hb][1][0] = part == 0 ? S.qs[2][head][tq] : 0u;
    bf[hb][1][1] = part == 0 ? S.qs[2][head][tq + 4] : 0u;
  }
  const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
  const uint16_t *icache = a.index_cache;

  auto load_tile = [&](int tile, uint32_t (&af)[4]) -> bool {
    const long long pos0 = t0 + (long long)tile * kPage;
    const int page = pt[pos0 / kPage];
    if (page < 0 || page >= sh.num_pages) {
      if (lane == 0) raise_error(a.err, SD_EBIT_PAGE);
      af[0] = af[1] = af[2] = af[3] = 0u;
      return false;
    }
    const uint32_t *pg =
        reinterpret_cast<const uint32_t *>(icache + ((long long)page * sh.Hkv + g) * (kPage * kIndexDim));
    af[0] = __ldg(pg + gq * 8 + tq);
    af[1] = __ldg(pg + (gq + 8) * 8 + tq);
    af[2] = __ldg(pg + gq * 8 + tq + 4);
    af[3] = __ldg(pg + (gq + 8) * 8 + tq + 4);
    return true;
  };
  // scores of rows gq and gq + 8 for head 4hb + tq
  auto score_tile = [&](const uint32_t (&af)[4], float (&out)[HB][2]) {
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
      float d[4], e[4];
      mma_16816(d, af, bf[hb][0][0], bf[hb][0][1]);
      mma_16816(e, af, bf[hb][1][0], bf[hb][1][1]);
      out[hb][0] = (d[0] + d[1]) + e[0];
      out[hb][1] = (d[2] + d[3]) + e[2];
    }
  };

  // ---- 1. sample --------------------------------------------------------------
  const int st = std::max(1, (ntiles + kSampleTiles - 1) / kSampleTiles);
  const int ns = (ntiles + st - 1) / st;
  {
    float smx[HB], smn[HB];
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
      smx[hb] = -INFINITY;
      smn[hb] = INFINITY;
    }
    for (int j = warp; j < ns; j += kW) {
      const int tile = j * st;
      uint32_t af[4];
      const bool ok = load_tile(tile, af);
      float sc[HB][2];
      score_tile(af, sc);
#pragma unroll
      for (int hb = 0; hb < HB; ++hb) {
        const int h = hb * 4 + tq;
        if (h >= GR) continue;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = gq + 8 * r;
          const bool valid = ok && tile * kPage + row < cnt;
          const float v = valid ? sc[hb][r] : -INFINITY;
          sample[h * (kSampleTiles * 16) + j * 16 + row] = v;
          if (valid) {
            smx[hb] = fmaxf(smx[hb], v);
            smn[hb] = fminf(smn[hb], v);
          }
        }
      }
    }
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        smx[hb] = fmaxf(smx[hb], __shfl_xor_sync(kFull, smx[hb], o));
        smn[hb] = fminf(smn[hb], __shfl_xor_sync(kFull, smn[hb], o));
      }
      const int h = hb * 4 + tq;
      if (gq == 0 && h < nr && smx[hb] > -INFINITY) {
        atomicMax(&S.smax[h], order_key(smx[hb]));
        atomicMin(&S.smin[h], order_key(smn[hb]));
      }
    }
  }
  __syncthreads();
  // local window estimate from a 64-bin histogram of the sample
  uint32_t *shist = wred;                            // scratch until the reduction
  for (int o = tid; o < GR * kSampleBins; o += kT) shist[o] = 0u;
  __syncthreads();
  int n_sample = 0;                                  // valid sample tokens (same for every head)
  for (int j = 0; j < ns; ++j) n_sample += std::max(0, std::min(16, cnt - j * st * kPage));
  for (int o = tid; o < nr * ns * 16; o += kT) {
    const int h = o / (ns * 16), r = o % (ns * 16);
    const float v = sample[h * (kSampleTiles * 16) + r];
    if (v == -INFINITY) continue;
    const float lo = key_to_float(S.smin[h]), hi = key_to_float(S.smax[h]);
    const float inv = hi > lo ? (float)kSampleBins / (hi - lo) : 0.0f;
    const int bin = std::min(kSampleBins - 1, std::max(0, __float2int_rz((v - lo) * inv)));
    atomicAdd(&shist[h * kSampleBins + bin], 1u);
  }
  __syncthreads();
  if (tid < nr) {
    const int h = tid;
    uint32_t lo_key = 0xFFFFFFFFu, hi_key = 0u;      // neutral for the cluster min / max
    if (n_sample > 0 && S.smax[h] != 0u) {
      const double mu = (double)n_sample * (double)kb / (double)N;
      const double r = ceil(mu + 6.0 * sqrt(mu) + 8.0);
      hi_key = S.smax[h];
      if (r < (double)n_sample) {
        const float lo = key_to_float(S.smin[h]), hi = key_to_float(S.smax[h]);
        uint32_t cum = 0;
        int blo = 0;
        for (int bin = kSampleBins - 1; bin >= 0; --bin) {
          cum += shist[h * kSampleBins + bin];
          if ((double)cum >= r) {
            blo = bin;
            break;
          }
        }
        const float edge = lo + (float)blo * ((hi - lo) / (float)kSampleBins);
        lo_key = order_key(edge);
      } else {
        lo_key = 0u;                                 // no estimate: the window starts at -inf
      }
    }
    S.tlo_key[h] = lo_key;
    S.thi_key[h] = hi_key;
  }
  cluster.sync();                                    // B1: local windows published
  for (int h = warp; h < nr; h += kW) {
    uint32_t lo = lane < C ? *cluster.map_shared_rank(&S.tlo_key[h], lane) : 0xFFFFFFFFu;
    uint32_t hi = lane < C ? *cluster.map_shared_rank(&S.thi_key[h], lane) : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = std::min(lo, __shfl_xor_sync(kFull, lo, o));
      hi = std::max(hi, __shfl_xor_sync(kFull, hi, o));
    }
    if (lane == 0) {
      const float flo = (lo == 0u || lo == 0xFFFFFFFFu) ? -INFINITY : key_to_float(lo);
      const float fhi = key_to_float(hi);
      S.tlo[h] = flo;
      S.thi[h] = fhi;
      S.inv[h] = (flo > -INFINITY && fhi > flo) ? (float)kBins / (fhi - flo) : 0.0f;
    }
  }
  __syncthreads();

  // ---- 2. stream the chunk, keep the window ----------------------------------
  auto classify = [&](int h, int i, float s) {
    int cls;
    if (s >= S.thi[h]) {
      cls = kTopClass;
      atomicAdd(&S.top_n[h], 1u);
    } else if (s >= S.tlo[h]) {
      cls = std::min(kBins - 1, std::max(0, __float2int_rz((s - S.tlo[h]) * S.inv[h])));
      atomicAdd(&whist[h * kBins + cls], 1u);
    } else {
      return;
    }
    const uint32_t slot = atomicAdd(&S.list_n[h], 1u);
    if (slot < (uint32_t)tp.list_cap)
      list[(size_t)h * tp.list_cap + slot] = ((unsigned long long)__float_as_uint(s) << 32) | (uint32_t)i;
    else
      S.overflow = 1u;
  };
  for (int base = warp; base < ntiles; base += kW * kUnroll) {
    uint32_t af[kUnroll][4];
    bool ok[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int tile = base + u * kW;
      ok[u] = false;
      if (tile < ntiles && tile % st != 0) ok[u] = load_tile(tile, af[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!ok[u]) continue;
      const int tile = base + u * kW;
      float sc[HB][2];
      score_tile(af[u], sc);
#pragma unroll
      for (int hb = 0; hb < HB; ++hb) {
        const int h = hb * 4 + tq;
        if (h >= nr) continue;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int i = tile * kPage + gq + 8 * r;
          if (i < cnt) classify(h, i, sc[hb][r]);
        }
      }
    }
  }
  for (int o = tid; o < nr * ns * 16; o += kT) {     // sampled pages
    const int h = o / (ns * 16), r = o % (ns * 16);
    const int i = (r / 16) * st * kPage + (r % 16);
    const float v = sample[h * (kSampleTiles * 16) + r];
    if (i < cnt && v > -INFINITY) classify(h, i, v);
  }
  __syncthreads();
  cluster.sync();                                    // B2: histograms and lists complete

  // ---- 3. cluster reduction of the window histogram, cut bin ----------------
  const int per = kBins / C;
  const int d0 = rank * per;
  for (int base = 0; base < nr * kBins; base += kT) {
    const int it = base + tid;
    const bool okk = it < nr * kBins;
    const int c = it % C, rest = it / C;
    const int h = rest / per, bin = d0 + rest % per;
    uint32_t v = okk ? *cluster.map_shared_rank(&whist[h * kBins + bin], c) : 0u;
    for (int o = 1; o < C; o <<= 1) v += __shfl_xor_sync(kFull, v, o);
    if (okk && c == 0) wred[h * kBins + bin] = v;
  }
  __syncthreads();
  for (int h = warp; h < nr; h += kW) {
    uint32_t sc = 0u;
    for (int j = lane; j < per; j += 32) sc += wred[h * kBins + d0 + j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sc += __shfl_xor_sync(kFull, sc, o);
    if (lane == 0) S.slice_cnt[h] = sc;
  }
  __syncthreads();
  cluster.sync();                                    // B3: owner slices reduced
  if (warp == 0) {
    uint32_t f = lane < C ? *cluster.map_shared_rank(&S.overflow, lane) : 0u;
    f = __reduce_or_sync(kFull, f);
    if (lane == 0 && f) S.fail = 1;
  }
  for (int h = warp; h < nr; h += kW) {
    const uint32_t topc = lane < C ? *cluster.map_shared_rank(&S.top_n[h], lane) : 0u;
    const long long top_total = __reduce_add_sync(kFull, topc);
    const long long need = kb - top_total;
    const uint32_t lc = lane < C ? *cluster.map_shared_rank(&S.slice_cnt[h], lane) : 0u;
    long long suf = lc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_down_sync(kFull, suf, o);
      if (lane + o < 32) suf += y;
    }
    const bool reach = lane < C && lc > 0u && need > 0 && suf >= need;
    const unsigned bal = __ballot_sync(kFull, reach);
    bool bad = need <= 0 || bal == 0u;
    int cut = -1;
    long long above = 0, ncut = 0;
    if (!bad) {
      const int cs = 31 - __clz(bal);
      above = __shfl_sync(kFull, suf, cs) - (long long)__shfl_sync(kFull, lc, cs);
      for (int top = per; top > 0 && cut < 0; top -= 32) {
        const int j = top - 32 + lane;
        const bool in = j >= 0 && j < per;
        const uint32_t dc = in ? *cluster.map_shared_rank(&wred[h * kBins + cs * per + j], cs) : 0u;
        long long sk = dc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const long long y = __shfl_down_sync(kFull, sk, o);
          if (lane + o < 32) sk += y;
        }
        const unsigned b2 = __ballot_sync(kFull, in && dc > 0u && above + sk >= need);
        if (b2) {
          const int l = 31 - __clz(b2);
          cut = cs * per + top - 32 + l;
          ncut = __shfl_sync(kFull, (long long)dc, l);
          above += __shfl_sync(kFull, sk, l) - ncut;
        } else {
          above += __shfl_sync(kFull, sk, 0);
        }
      }
      bad = cut < 0 || ncut > kCap;
    }
    if (lane == 0) {
      S.cut[h] = cut;
      S.need_c[h] = need - above;
      if (bad) S.fail = 1;
    }
  }
  __syncthreads();
  if (S.fail) {                                      // uniform across the cluster
    if (rank == 0 && tid == 0) tp.fail[item] = 1u;
    cluster.sync();                                  // peers may still read this CTA's memory
    return;
  }
  if (rank == 0 && tid == 0) tp.fail[item] = 0u;

  // ---- 4. candidates of the cut bin to the owner; local counts above it -----
  auto class_of = [&](int h, float s) -> int {
    if (s >= S.thi[h]) return kTopClass;
    return std::min(kBins - 1, std::max(0, __float2int_rz((s - S.tlo[h]) * S.inv[h])));
  };
  for (int h = 0; h < nr; ++h) {
    const int n = (int)std::min<uint32_t>(S.list_n[h], (uint32_t)tp.list_cap);
    const int cut = S.cut[h];
    const int owner = h % C, slot = h / C;
    uint32_t above = 0u;
    for (int e = tid; e < n; e += kT) {
      const unsigned long long ent = list[(size_t)h * tp.list_cap + e];
      const float s = __uint_as_float((uint32_t)(ent >> 32));
      const uint32_t i = (uint32_t)ent;
      const int cls = class_of(h, s);
      if (cls > cut) {
        ++above;
      } else if (cls == cut) {
        uint32_t *cn = cluster.map_shared_rank(&S.cand_n[slot], owner);
        const uint32_t idx = atomicAdd(cn, 1u);
        if (idx < (uint32_t)kCap) {
          unsigned long long *dst = cluster.map_shared_rank(cand + (size_t)slot * kCap + idx, owner);
          *dst = sort_key(s, (uint32_t)(t0 + i));
        }
      }
    }
    above = __reduce_add_sync(kFull, above);
    if (lane == 0 && above) atomicAdd(&S.above_local[h], above);
  }
  __syncthreads();
  cluster.sync();                                    // B4: candidates delivered

  // ---- 5. owners rank their candidates exactly --------------------------------
  for (int slot = 0; slot < tp.own_slots; ++slot) {
    const int h = rank + slot * C;
    if (h >= nr) break;
    const int n = (int)std::min<uint32_t>(S.cand_n[slot], (uint32_t)kCap);
    const long long need_c = S.need_c[h];
    const unsigned long long *cs = cand + (size_t)slot * kCap;
    for (int e = tid; e < n; e += kT) {
      const unsigned long long me = cs[e];
      int rk = 0;
      for (int j = 0; j < n; ++j) rk += cs[j] < me;
      if (rk == need_c - 1) S.tau_sk[slot] = me;
      if (rk < need_c) {
        const long long pos = (long long)(me & 0xFFFFFFFFull);
        const int c = (int)std::min<long long>(C - 1, pos / per_cta);
        atomicAdd(&occ[slot * kMaxCluster + c], 1u);
      }
    }
  }
  __syncthreads();
  cluster.sync();                                    // B5: thresholds published

  // ---- 6. offsets, ordered write ---------------------------------------------
  unsigned long long tau[kMaxGroup];
  long long off[kMaxGroup];
  for (int h = 0; h < nr; ++h) {
    const int owner = h % C, slot = h / C;
    tau[h] = *cluster.map_shared_rank(&S.tau_sk[slot], owner);
    const long long ab = lane < C ? (long long)*cluster.map_shared_rank(&S.above_local[h], lane) : 0LL;
    const long long oc = lane < C ? (long long)*cluster.map_shared_rank(&occ[slot * kMaxCluster + lane], owner) : 0LL;
    const long long mine = ab + oc;
    const long long before = __reduce_add_sync(kFull, (unsigned)(lane < rank ? mine : 0LL));
    const long long total = __reduce_add_sync(kFull, (unsigned)mine);
    off[h] = before;
    if (rank == 0 && tid == 0) {
      if (total > a.sel_stride) raise_error(a.err, SD_EBIT_SEL);
      *count_slot(h) = (int32_t)std::min(total, a.sel_stride);
    }
  }
  cluster_arrive();                                  // no more reads of peer memory
  for (int h = 0; h < nr; ++h) {
    const int n = (int)std::min<uint32_t>(S.list_n[h], (uint32_t)tp.list_cap);
    const int cut = S.cut[h];
    for (int e = tid; e < n; e += kT) {
      const unsigned long long ent = list[(size_t)h * tp.list_cap + e];
      const float s = __uint_as_float((uint32_t)(ent >> 32));
      const uint32_t i = (uint32_t)ent;
      const int cls = class_of(h, s);
      const bool sel = cls > cut || (cls == cut && sort_key(s, (uint32_t)(t0 + i)) <= tau[h]);
      if (sel) atomicOr(&bitmap[h * words + (i >> 5)], 1u << (i & 31));
    }
  }
  __syncthreads();
  const int nwords = (cnt + 31) / 32;
  const int wpt = (nwords + kT - 1) / kT;            // bitmap words per thread
  for (int h = 0; h < nr; ++h) {
    int32_t *row = sel_row(h);
    const int w0 = tid * wpt;
    uint32_t c = 0;
    for (int w = w0; w < std::min(nwords, w0 + wpt); ++w) c += __popc(bitmap[h * words + w]);
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) S.wtot[warp] = incl;
    __syncthreads();
    uint32_t wbase = 0;
    for (int w = 0; w < warp; ++w) wbase += S.wtot[w];
    long long o = off[h] + wbase + incl - c;
    for (int w = w0; w < std::min(nwords, w0 + wpt); ++w) {
      uint32_t bits = bitmap[h * words + w];
      while (bits) {
        const int bit = __ffs(bits) - 1;
        bits &= bits - 1;
        if (o < a.sel_stride) row[o] = (int32_t)(t0 + w * 32 + bit);
        else raise_error(a.err, SD_EBIT_SEL);
        ++o;
      }
    }
    __syncthreads();
  }
  cluster_wait();
}

int pow2_floor(int x) {
  int p = 1;
  while (p * 2 <= x) p <<= 1;
  return p;
}

template <int GR>
struct TkCache {
  std::mutex mu;
  std::map<int, size_t> attr;
  std::map<std::tuple<int, size_t, int>, int> clusters;
};

template <int GR>
TkCache<GR> &tk_cache() {
  static TkCache<GR> c;
  return c;
}

template <int GR>
cudaError_t tk_attrs(int dev, size_t bytes) {
  auto &c = tk_cache<GR>();
  std::lock_guard<std::mutex> lk(c.mu);
  auto it = c.attr.find(dev);
  if (it != c.attr.end() && it->second >= bytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(topk_kernel<GR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(topk_kernel<GR>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) c.attr[dev] = bytes;
  return e;
}

template <int GR>
cudaLaunchConfig_t tk_config(int C, int items, size_t bytes, cudaStream_t st, cudaLaunchAttribute *attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, items, 1);
  cfg.blockDim = dim3(kT, 1, 1);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int GR>
int tk_fits(int dev, int C, size_t bytes) {
  if (tk_attrs<GR>(dev, bytes) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  auto &c = tk_cache<GR>();
  const auto key = std::make_tuple(dev, bytes, C);
  {
    std::lock_guard<std::mutex> lk(c.mu);
    auto it = c.clusters.find(key);
    if (it != c.clusters.end()) return it->second;
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = tk_config<GR>(C, 1, bytes, 0, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, topk_kernel<GR>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(c.mu);
  c.clusters[key] = n;
  return n;
}

struct TkPlan {
  int C, tc_cap, list_cap, own_slots;
  size_t bytes;
};

TkPlan tk_plan(const Shape &sh, int GR) {
  TkPlan p{};
  p.C = std::min(kMaxCluster, pow2_floor(std::max(1, sh.max_pages)));
  p.tc_cap = (int)(((sh.max_len + p.C - 1) / p.C + kPage - 1) / kPage * kPage);
  p.tc_cap = (p.tc_cap + 31) / 32 * 32;
  p.list_cap = std::max(256, (p.tc_cap / 8 + 31) / 32 * 32);
  p.own_slots = (GR + p.C - 1) / p.C;
  p.bytes = tk_layout(GR, p.tc_cap, p.list_cap, p.own_slots).total;
  return p;
}

template <int GR>
cudaError_t tk_launch(const SelectArgs &a, const Shape &sh, const Tables &tb, uint32_t *fail, int dev,
                      cudaStream_t st, bool *used) {
  *used = false;
  const TkPlan p = tk_plan(sh, GR);
  if (p.bytes + sizeof(TkShared) > 227 * 1024) return cudaSuccess;
  if (tk_fits<GR>(dev, p.C, p.bytes) == 0) return cudaSuccess;
  cudaError_t e = tk_attrs<GR>(dev, p.bytes);
  if (e != cudaSuccess) return e;
  TopkParams tp{p.tc_cap, p.list_cap, p.own_slots, fail};
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = tk_config<GR>(p.C, a.batch * tb.n_ret, p.bytes, st, attr);
  e = cudaLaunchKernelEx(&cfg, topk_kernel<GR>, a, sh, tb.ret, tb.n_ret, tp);
  if (e == cudaSuccess) *used = true;
  return e;
}

}  // namespace

cudaError_t launch_select_topk_stream(const SelectArgs &a, const Shape &sh, const Tables &tb, uint32_t *fail,
                                      cudaStream_t st, bool *used) {
  int dev = 0;
  cudaGetDevice(&dev);
  int gr = 1;
  while (gr < tb.max_ret) gr <<= 1;
  switch (gr) {
    case 1: return tk_launch<1>(a, sh, tb, fail, dev, st, used);
    case 2: return tk_launch<2>(a, sh, tb, fail, dev, st, used);
    case 4: return tk_launch<4>(a, sh, tb, fail, dev, st, used);
    case 8: return tk_launch<8>(a, sh, tb, fail, dev, st, used);
    default: return tk_launch<16>(a, sh, tb, fail, dev, st, used);
  }
}

}  // namespace sd
