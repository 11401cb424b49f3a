// Index scoring + top-p / top-k selection for retrieval heads.
//
// RTPurbo page (gist.science/ar/paper/2605.16928):
//   Methodology 2  relevance is scored in an r = 16 space: s_j = c <P^T q, k~_j>;
//   Methodology 3  dynamic top-p: attention mass (softmax of the index scores)
//                  is accumulated in descending order until the cumulative
//                  threshold p is reached; fixed top-k is the alternative;
//   Methodology 5  the threshold is found with a histogram, without sorting.
// ICS page (gist.science/ar/paper/2605.24168), 2: "Oracle Top-K" = exact top-k.
//
// This is the exact selector.  It takes the items the streaming selectors
// (sd_select_stream.cu) flag as misses, or every item when those cannot run
// (shapes outside them).
//
// Design (one thread-block cluster per (sequence b, KV group g)):
//   * the C CTAs of the cluster split the sequence's N_b tokens into C
//     contiguous, page-aligned chunks;
//   * every CTA streams its chunk of the index once from HBM (two 16-byte
//     loads per token), computes the float32 scores of all retrieval heads of
//     the group and keeps them on chip (shared memory) -- or, when they do not
//     fit, in a workspace row that stays L2-resident for the cluster's
//     lifetime;
//   * the threshold is an exact radix search on an order-preserving 32-bit key
//     of the score, 8 bits per pass (4 passes); each pass builds per-CTA
//     digit histograms (counts; for top-p also float64 softmax mass), reduces
//     them across the cluster through distributed shared memory, and narrows
//     the key prefix to the digit where the cumulative count (k) or mass
//     (p * Z) is reached, scanning from the top digit down;
//   * the selected positions (key > tau, plus ties at tau: all of them for
//     top-p, the lowest positions for top-k) are written in ascending order:
//     per-warp counts, a cluster-wide exclusive scan, then ordered ballots.
// No CTA ever waits on another CTA outside hardware cluster barriers.
#include <cooperative_groups.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "sd_internal.cuh"

namespace cg = cooperative_groups;

namespace sd {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kRadix = 256;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxCluster = 16;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Max over the lanes that share (lane % stride); stride is a power of two.
__device__ __forceinline__ float warp_max_strided(float v, int stride) {
  for (int o = 16; o >= stride; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Warp-aggregated histogram update: lanes with the same digit are combined so
// that each distinct digit costs one shared-memory atomic per warp.
template <bool TOPP>
__device__ __forceinline__ void hist_add(uint32_t *cnt, double *mass, bool act, uint32_t dg, float w,
                                         int lane) {
  const uint32_t tag = act ? dg : (0x100u | (uint32_t)lane);
  const unsigned peers = __match_any_sync(kFull, tag);
  const int leader = __ffs(peers) - 1;
  if constexpr (TOPP) {
    float gsum = w;
    unsigned multi = __ballot_sync(kFull, act && lane == leader && __popc(peers) > 1);
    while (multi) {
      const int src = __ffs(multi) - 1;
      multi &= multi - 1;
      const unsigned gm = __shfl_sync(kFull, peers, src);
      const float v = warp_sum(((gm >> lane) & 1u) ? w : 0.0f);
      if (lane == src) gsum = v;
    }
    if (act && lane == leader) {
      atomicAdd(&cnt[dg], (uint32_t)__popc(peers));
      atomicAdd(&mass[dg], (double)gsum);
    }
  } else {
    if (act && lane == leader) atomicAdd(&cnt[dg], (uint32_t)__popc(peers));
  }
}

struct SelShared {
  Group grp;
  float qt[kMaxGroup][kIndexDim];
  uint32_t cmax_key[kMaxGroup];
  float M[kMaxGroup];
  uint32_t prefix[kMaxGroup];
  long long need[kMaxGroup];     // top-k: tokens still to take among the candidates
  double target[kMaxGroup];      // top-p: mass still to take among the candidates
  uint32_t slice_cnt[kMaxGroup];
  double slice_mass[kMaxGroup];
  uint32_t wgt[kWarps][kMaxGroup];
  uint32_t weq[kWarps][kMaxGroup];
  uint32_t cgt[kMaxGroup];
  uint32_t ceq[kMaxGroup];
  long long out_off[kMaxGroup];
  long long my_ties[kMaxGroup];
};

// GR: score rows held per CTA (power of two >= the group's retrieval heads).
template <int GR, bool TOPP, bool SMEM>
__device__ __forceinline__ void select_item(const SelectArgs &a, const Shape &sh, const Group *__restrict__ groups,
                                            int n_groups, int tc_cap, int item, SelShared &S, unsigned char *dyn) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = item / n_groups;
  const int gi = item % n_groups;
  double *hmass = reinterpret_cast<double *>(dyn);                    // [GR][256] (top-p)
  double *rmass = hmass + (TOPP ? GR * kRadix : 0);                  // [GR][256] (top-p)
  uint32_t *hcnt = reinterpret_cast<uint32_t *>(rmass + (TOPP ? GR * kRadix : 0));
  uint32_t *rcnt = hcnt + GR * kRadix;
  float *scores = reinterpret_cast<float *>(rcnt + GR * kRadix);     // [GR][tc_cap] (SMEM)

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

  auto sel_row = [&](int i) {
    return a.sel_idx + ((long long)b * sh.H_ret + S.grp.row[i]) * a.sel_stride;
  };
  auto count_slot = [&](int i) { return a.sel_count + (long long)b * sh.H_ret + S.grp.row[i]; };

  // ---- degenerate sets: empty context, p >= 1, k_b >= N_b --------------
  long long kb = 0;
  bool keep_all;
  if (TOPP) {
    keep_all = a.top_p >= 1.0f;
  } else {
    kb = a.top_k > 0 ? (long long)a.top_k
                     : std::max(1LL, (long long)floor((double)a.top_k_frac * (double)N));
    kb = std::min(kb, N);
    keep_all = kb >= N;
  }
  if (N == 0 || keep_all) {
    for (int i = 0; i < nr; ++i) {
      int32_t *row = sel_row(i);
      for (long long t = t0 + tid; t < t1; t += kThreads) {
        if (t < a.sel_stride) row[t] = (int32_t)t;
        else raise_error(a.err, SD_EBIT_SEL);
      }
      if (rank == 0 && tid == 0) *count_slot(i) = (int32_t)std::min(N, a.sel_stride);
    }
    return;
  }

  auto score_ptr = [&](int h) -> float * {
    if constexpr (SMEM) return scores + (size_t)h * tc_cap;
    else return a.score_ws + ((long long)b * sh.H_ret + S.grp.row[h]) * sh.max_len + t0;
  };

  // ---- q~ = c * P_g^T q_pre (float64 accumulation) ----------------------
  // (scores written beforehand by the exact-score kernel: only their maxima)
  for (int o = tid; o < kMaxGroup * kIndexDim && !a.pre_scored; o += kThreads) {
    const int i = o / kIndexDim, j = o % kIndexDim;
    float v = 0.0f;
    if (i < nr) {
      const uint16_t *qrow = a.q_pre + ((long long)b * sh.Hq + S.grp.q_head[i]) * sh.d;
      const uint16_t *P = a.proj + (long long)g * sh.d * kIndexDim;
      double acc = 0.0;
      for (int e = 0; e < sh.d; ++e)
        acc = fma((double)bf16_to_f32(qrow[e]), (double)bf16_to_f32(P[e * kIndexDim + j]), acc);
      v = (float)((double)a.index_scale * acc);
    }
    S.qt[i][j] = v;
  }
  if (tid < kMaxGroup) S.cmax_key[tid] = 0u;
  __syncthreads();

  if (a.pre_scored) {
    // ---- the score rows are given (exact-score mode): the CTA's maxima, and
    // with room on chip a copy of its chunk of every row, read once here
    // instead of at every radix pass
    for (int h = 0; h < nr; ++h) {
      const float *src = a.score_ws + ((long long)b * sh.H_ret + S.grp.row[h]) * sh.max_len + t0;
      float m = -INFINITY;
      if constexpr (SMEM) {
        float *dst = score_ptr(h);
        for (int i = tid; i < cnt; i += kThreads) {
          const float v = __ldcg(src + i);
          dst[i] = v;
          m = fmaxf(m, v);
        }
      } else {
        for (int i = tid; i < cnt; i += kThreads) m = fmaxf(m, src[i]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
      if (lane == 0 && m > -INFINITY) atomicMax(&S.cmax_key[h], order_key(m));
    }
  }
  // ---- stream the index, score, keep scores on chip ----------------------
  if (!a.pre_scored) {
    constexpr int HPB = GR < 4 ? GR : 4;          // heads per thread
    constexpr int HB = GR / HPB;                  // head blocks (threads per token)
    const int hb = tid % HB;
    const int TS = kThreads / HB;
    float q[HPB][kIndexDim];
#pragma unroll
    for (int h = 0; h < HPB; ++h)
#pragma unroll
      for (int j = 0; j < kIndexDim; ++j) q[h][j] = S.qt[hb * HPB + h][j];
    float tmax[HPB];
#pragma unroll
    for (int h = 0; h < HPB; ++h) tmax[h] = -INFINITY;
    float *sp[HPB];
#pragma unroll
    for (int h = 0; h < HPB; ++h) sp[h] = (hb * HPB + h < nr) ? score_ptr(hb * HPB + h) : nullptr;
    const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
    constexpr int U = 4;
    for (int i0 = tid / HB; i0 < cnt; i0 += TS * U) {
      uint4 raw[U][2];
      bool ok[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * TS;
        ok[u] = false;
        if (i < cnt) {
          const long long t = t0 + i;
          const int page = pt[t / kPage];
          if (page >= 0 && page < sh.num_pages) {
            const uint4 *row = reinterpret_cast<const uint4 *>(
                a.index_cache + (((long long)page * sh.Hkv + g) * kPage + (t % kPage)) * kIndexDim);
            raw[u][0] = __ldg(row);
            raw[u][1] = __ldg(row + 1);
            ok[u] = true;
          } else {
            raise_error(a.err, SD_EBIT_PAGE);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * TS;
        if (i >= cnt) break;
        float k[kIndexDim];
        const uint32_t w[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                               raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          k[2 * j] = bf16_lo(w[j]);
          k[2 * j + 1] = bf16_hi(w[j]);
        }
#pragma unroll
        for (int h = 0; h < HPB; ++h) {
          float s = 0.0f;
#pragma unroll
          for (int j = 0; j < kIndexDim; ++j) s = fmaf(q[h][j], k[j], s);
          if (!ok[u]) s = -INFINITY;
          if (sp[h]) {
            sp[h][i] = s;
            tmax[h] = fmaxf(tmax[h], s);
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < HPB; ++h) {
      const float m = warp_max_strided(tmax[h], HB);
      if (lane < HB && hb * HPB + h < nr && m > -INFINITY) atomicMax(&S.cmax_key[hb * HPB + h], order_key(m));
    }
  }
  if (!SMEM) __threadfence_block();
  __syncthreads();

  // ---- cluster max (top-p needs the softmax reference) --------------------
  if (TOPP) {
    cluster.sync();
    if (warp < nr) {                   // warp h reads the C CTA maxima, one per lane
      uint32_t m = lane < C ? *cluster.map_shared_rank(&S.cmax_key[warp], lane) : 0u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = std::max(m, __shfl_xor_sync(kFull, m, o));
      if (lane == 0) S.M[warp] = key_to_float(m);
    }
  }
  if (tid < nr) {
    S.prefix[tid] = 0u;
    S.need[tid] = kb;
  }
  __syncthreads();

  const int per = kRadix / C;        // digits owned by each CTA in the reduction
  const int d0 = rank * per;

  // ---- radix passes -------------------------------------------------------
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int o = tid; o < GR * kRadix; o += kThreads) {
      hcnt[o] = 0u;
      if (TOPP) hmass[o] = 0.0;
    }
    __syncthreads();
    for (int h = 0; h < nr; ++h) {
      const uint32_t pre = S.prefix[h];
      const float M = TOPP ? S.M[h] : 0.0f;
      const float *sc = score_ptr(h);
      for (int base = warp * 32; base < cnt; base += kThreads) {
        const int i = base + lane;
        bool act = i < cnt;
        const float s = act ? sc[i] : 0.0f;
        const uint32_t key = order_key(s);
        if (pass > 0) act = act && ((key >> (shift + 8)) == pre);
        if (__ballot_sync(kFull, act) == 0u) continue;
        const float w = (TOPP && act) ? exp2f((s - M) * kLog2e) : 0.0f;
        hist_add<TOPP>(hcnt + h * kRadix, hmass + h * kRadix, act, (key >> shift) & 0xFFu, w, lane);
      }
    }
    __syncthreads();
    cluster.sync();
    // owner reduction of this CTA's digit slice: one remote load per lane,
    // items ordered (head, digit, cta) with the CTA index fastest so that the
    // C values of one digit sit in C adjacent lanes (C divides 32)
    for (int base = 0; base < nr * kRadix; base += kThreads) {
      const int it = base + tid;
      const bool ok = it < nr * kRadix;
      const int c = it % C, rest = it / C;
      const int h = rest / per, dg = d0 + rest % per;
      uint32_t vc = 0u;
      double vm = 0.0;
      if (ok) {
        vc = *cluster.map_shared_rank(&hcnt[h * kRadix + dg], c);
        if (TOPP) vm = *cluster.map_shared_rank(&hmass[h * kRadix + dg], c);
      }
      for (int o = 1; o < C; o <<= 1) {
        vc += __shfl_xor_sync(kFull, vc, o);
        if (TOPP) vm += __shfl_xor_sync(kFull, vm, o);
      }
      if (ok && c == 0) {
        rcnt[h * kRadix + dg] = vc;
        if (TOPP) rmass[h * kRadix + dg] = vm;
      }
    }
    __syncthreads();
    if (warp < nr) {                   // slice totals, warp h
      uint32_t sc = 0u;
      double sm = 0.0;
      for (int j = lane; j < per; j += 32) {
        sc += rcnt[warp * kRadix + d0 + j];
        if (TOPP) sm += rmass[warp * kRadix + d0 + j];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sc += __shfl_xor_sync(kFull, sc, o);
        if (TOPP) sm += __shfl_xor_sync(kFull, sm, o);
      }
      if (lane == 0) {
        S.slice_cnt[warp] = sc;
        S.slice_mass[warp] = sm;
      }
    }
    __syncthreads();
    cluster.sync();
    // every CTA, warp h: locate the cut digit scanning from the highest digit
    // down; lanes hold slices (then digits) and suffix sums give the running
    // amount above each of them
    if (warp < nr) {
      const int h = warp;
      const uint32_t lc = lane < C ? *cluster.map_shared_rank(&S.slice_cnt[h], lane) : 0u;
      const double lm = (TOPP && lane < C) ? *cluster.map_shared_rank(&S.slice_mass[h], lane) : 0.0;
      if (TOPP && pass == 0) {
        double Z = lm;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Z += __shfl_xor_sync(kFull, Z, o);
        if (lane == 0) S.target[h] = (double)a.top_p * Z;
      }
      __syncwarp();
      const double need_m = TOPP ? S.target[h] : 0.0;
      const long long need_k = S.need[h];
      // suffix sums over lanes: value at lane c = sum over lanes >= c
      long long suf_k = lc;
      double suf_m = lm;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long yk = __shfl_down_sync(kFull, suf_k, o);
        const double ym = __shfl_down_sync(kFull, suf_m, o);
        if (lane + o < 32) {
          suf_k += yk;
          suf_m += ym;
        }
      }
      bool reach = lane < C && lc > 0u && (TOPP ? suf_m >= need_m : suf_k >= need_k);
      unsigned bal = __ballot_sync(kFull, reach);
      int cs;
      if (bal) {
        cs = 31 - __clz(bal);          // highest slice where the amount is reached
      } else {                         // rounding left it unreached: lowest non-empty slice
        const unsigned nz = __ballot_sync(kFull, lane < C && lc > 0u);
        cs = nz ? __ffs(nz) - 1 : 0;
      }
      // amount strictly above slice cs
      long long acc_k = __shfl_sync(kFull, suf_k, cs) - (long long)__shfl_sync(kFull, lc, cs);
      double acc_m = __shfl_sync(kFull, suf_m, cs) - __shfl_sync(kFull, lm, cs);
      int cut = -1;
      int lowest_nz = -1;
      for (int top = per; top > 0 && cut < 0; top -= 32) {
        const int j = top - 32 + lane;          // digits of this chunk, highest chunk first
        const int dg = cs * per + j;
        const bool in = j >= 0 && j < per;
        const uint32_t dc = in ? *cluster.map_shared_rank(&rcnt[h * kRadix + dg], cs) : 0u;
        const double dm = (TOPP && in) ? *cluster.map_shared_rank(&rmass[h * kRadix + dg], cs) : 0.0;
        long long sk = dc;
        double smv = dm;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const long long yk = __shfl_down_sync(kFull, sk, o);
          const double ym = __shfl_down_sync(kFull, smv, o);
          if (lane + o < 32) {
            sk += yk;
            smv += ym;
          }
        }
        const bool r2 = in && dc > 0u && (TOPP ? acc_m + smv >= need_m : acc_k + sk >= need_k);
        const unsigned b2 = __ballot_sync(kFull, r2);
        const unsigned nz2 = __ballot_sync(kFull, in && dc > 0u);
        if (b2) {
          const int l = 31 - __clz(b2);
          cut = cs * per + top - 32 + l;
          acc_k += __shfl_sync(kFull, sk, l) - (long long)__shfl_sync(kFull, dc, l);
          acc_m += __shfl_sync(kFull, smv, l) - __shfl_sync(kFull, dm, l);
        } else {
          if (nz2) {
            const int l = __ffs(nz2) - 1;
            lowest_nz = cs * per + top - 32 + l;
          }
          acc_k += __shfl_sync(kFull, sk, 0);
          acc_m += __shfl_sync(kFull, smv, 0);
        }
      }
      if (cut < 0) {                   // rounding: take the lowest non-empty digit of the slice
        cut = lowest_nz < 0 ? cs * per : lowest_nz;
        const uint32_t dc = *cluster.map_shared_rank(&rcnt[h * kRadix + cut], cs);
        const double dm = TOPP ? *cluster.map_shared_rank(&rmass[h * kRadix + cut], cs) : 0.0;
        acc_k -= dc;
        acc_m -= dm;
      }
      if (lane == 0) {
        S.prefix[h] = (S.prefix[h] << 8) | (uint32_t)cut;
        if (TOPP) S.target[h] = need_m - acc_m;
        S.need[h] = need_k - acc_k;
      }
    }
    __syncthreads();
  }

  // ---- ordered compaction -------------------------------------------------
  const int wr = ((cnt + kWarps - 1) / kWarps + 31) / 32 * 32;     // tokens per warp
  const int w0 = std::min(cnt, warp * wr), w1 = std::min(cnt, w0 + wr);
  for (int h = 0; h < nr; ++h) {
    const uint32_t tk = S.prefix[h];
    const float *sc = score_ptr(h);
    uint32_t gt = 0, eq = 0;
    for (int base = w0; base < w1; base += 32) {
      const int i = base + lane;
      const bool act = i < w1;
      const uint32_t key = act ? order_key(sc[i]) : 0u;
      gt += __popc(__ballot_sync(kFull, act && key > tk));
      eq += __popc(__ballot_sync(kFull, act && key == tk));
    }
    if (lane == 0) {
      S.wgt[warp][h] = gt;
      S.weq[warp][h] = eq;
    }
  }
  __syncthreads();
  if (tid < nr) {
    uint32_t gt = 0, eq = 0;
    for (int w = 0; w < kWarps; ++w) {
      gt += S.wgt[w][tid];
      eq += S.weq[w][tid];
    }
    S.cgt[tid] = gt;
    S.ceq[tid] = eq;
  }
  __syncthreads();
  cluster.sync();
  if (warp < nr) {
    const int h = warp;
    const long long gc = lane < C ? (long long)*cluster.map_shared_rank(&S.cgt[h], lane) : 0LL;
    const long long ec = lane < C ? (long long)*cluster.map_shared_rank(&S.ceq[h], lane) : 0LL;
    long long gt_before = lane < rank ? gc : 0, eq_before = lane < rank ? ec : 0;
    long long tot_gt = gc, tot_eq = ec;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt_before += __shfl_xor_sync(kFull, gt_before, o);
      eq_before += __shfl_xor_sync(kFull, eq_before, o);
      tot_gt += __shfl_xor_sync(kFull, tot_gt, o);
      tot_eq += __shfl_xor_sync(kFull, tot_eq, o);
    }
    if (lane == 0) {
      const long long ties_total = TOPP ? tot_eq : std::min(S.need[h], tot_eq);
      const long long ties_before = std::min(eq_before, ties_total);
      S.my_ties[h] = std::max(0LL, std::min((long long)S.ceq[h], ties_total - eq_before));
      S.out_off[h] = gt_before + ties_before;
      const long long total = tot_gt + ties_total;
      if (rank == 0) {
        if (total > a.sel_stride) raise_error(a.err, SD_EBIT_SEL);
        *count_slot(h) = (int32_t)std::min(total, a.sel_stride);
      }
    }
  }
  cluster.sync();   // no CTA leaves while others still read its shared memory
  for (int h = 0; h < nr; ++h) {
    const uint32_t tk = S.prefix[h];
    const float *sc = score_ptr(h);
    int32_t *row = sel_row(h);
    long long off = S.out_off[h];
    long long ties_left = S.my_ties[h];
    for (int w = 0; w < warp; ++w) {
      const long long wt = std::min<long long>(S.weq[w][h], std::max(0LL, ties_left));
      off += S.wgt[w][h] + wt;
      ties_left -= S.weq[w][h];
    }
    const long long wtb = std::min<long long>(S.weq[warp][h], std::max(0LL, ties_left));
    long long eq_seen = 0;
    for (int base = w0; base < w1; base += 32) {
      const int i = base + lane;
      const bool act = i < w1;
      const uint32_t key = act ? order_key(sc[i]) : 0u;
      const bool is_eq = act && key == tk;
      const unsigned eqb = __ballot_sync(kFull, is_eq);
      const unsigned lt = (1u << lane) - 1u;
      const bool sel = (act && key > tk) || (is_eq && eq_seen + __popc(eqb & lt) < wtb);
      const unsigned sb = __ballot_sync(kFull, sel);
      if (sel) {
        const long long o = off + __popc(sb & lt);
        if (o < a.sel_stride) row[o] = (int32_t)(t0 + i);
        else raise_error(a.err, SD_EBIT_SEL);
      }
      off += __popc(sb);
      eq_seen += __popc(eqb);
    }
  }
}

// One cluster per work item (sequence, retrieval KV group).  With `flags`
// (layout: a flag per item, then the count of flagged items, then their
// list), the grid's clusters stride over the listed items only (items whose
// streaming top-k or top-p window missed); otherwise item = blockIdx.y.
template <int GR, bool TOPP, bool SMEM>
__global__ void __launch_bounds__(kThreads, 1)
select_kernel(const SelectArgs a, const Shape sh, const Group *__restrict__ groups, int n_groups,
              int tc_cap, const uint32_t *__restrict__ flags) {
  __shared__ SelShared S;
  extern __shared__ __align__(16) unsigned char dyn[];
  pdl_wait();
  pdl_trigger();
  const int n_items = a.batch * n_groups;
  const int n = flags ? (int)flags[n_items] : n_items;
  for (int k = blockIdx.y; k < n; k += gridDim.y) {
    const int item = flags ? (int)flags[n_items + 1 + k] : k;
    __syncthreads();
    select_item<GR, TOPP, SMEM>(a, sh, groups, n_groups, tc_cap, item, S, dyn);
  }
}

struct Plan {
  int cluster;
  bool smem;
  int tc_cap;
  size_t dyn_bytes;
};

int pow2_ceil(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

size_t hist_bytes(int GR, bool topp) {
  return (size_t)GR * kRadix * (2 * sizeof(uint32_t) + (topp ? 2 * sizeof(double) : 0));
}

int group_rows(const Tables &tb) { return pow2_ceil(std::max(1, tb.max_ret)); }

Plan make_plan(const Shape &sh, const Tables &tb, int batch, bool topp, int smem_limit, int sms) {
  const int GR = group_rows(tb);
  const int items = std::max(1, batch * tb.n_ret);
  int C = pow2_ceil((2 * sms + items - 1) / items);      // about two CTAs per SM over all items
  C = std::min(C, kMaxCluster);
  const int max_c = std::max(1, std::min(kMaxCluster, 1 << (31 - __builtin_clz(std::max(1, sh.max_pages)))));
  C = std::min(C, max_c);
  Plan p{};
  for (int c = C; c <= max_c; c <<= 1) {
    const int tc = (int)(((sh.max_len + c - 1) / c + kPage - 1) / kPage * kPage);
    const size_t bytes = hist_bytes(GR, topp) + (size_t)GR * tc * sizeof(float);
    if (bytes + sizeof(SelShared) <= (size_t)smem_limit) {
      p.cluster = c;
      p.smem = true;
      p.tc_cap = tc;
      p.dyn_bytes = bytes;
      return p;
    }
  }
  p.cluster = max_c;
  p.smem = false;
  p.tc_cap = (int)(((sh.max_len + max_c - 1) / max_c + kPage - 1) / kPage * kPage);
  p.dyn_bytes = hist_bytes(GR, topp);
  return p;
}

// Per kernel instantiation and device: the dynamic shared memory attribute
// and the cluster occupancy check are set / queried once, not per call.
template <int GR, bool TOPP, bool SMEM>
struct KernelCache {
  std::mutex mu;
  std::map<int, size_t> attr_bytes;                      // device -> bytes configured
  std::map<std::tuple<int, size_t, int>, int> clusters;  // (device, bytes, cluster) -> active clusters
};

template <int GR, bool TOPP, bool SMEM>
KernelCache<GR, TOPP, SMEM> &kcache() {
  static KernelCache<GR, TOPP, SMEM> c;
  return c;
}

template <int GR, bool TOPP, bool SMEM>
cudaError_t ensure_attrs(int dev, size_t bytes) {
  auto &c = kcache<GR, TOPP, SMEM>();
  std::lock_guard<std::mutex> lk(c.mu);
  auto it = c.attr_bytes.find(dev);
  if (it != c.attr_bytes.end() && it->second >= bytes) return cudaSuccess;
  auto kern = select_kernel<GR, TOPP, SMEM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) c.attr_bytes[dev] = bytes;
  return e;
}

template <int GR, bool TOPP, bool SMEM>
int active_clusters(int dev, const Plan &p) {
  if (ensure_attrs<GR, TOPP, SMEM>(dev, p.dyn_bytes) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  auto &c = kcache<GR, TOPP, SMEM>();
  const auto key = std::make_tuple(dev, p.dyn_bytes, p.cluster);
  {
    std::lock_guard<std::mutex> lk(c.mu);
    auto it = c.clusters.find(key);
    if (it != c.clusters.end()) return it->second;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.cluster, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = p.dyn_bytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, select_kernel<GR, TOPP, SMEM>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(c.mu);
  c.clusters[key] = n;
  return n;
}

template <int GR, bool TOPP, bool SMEM>
cudaError_t launch_t(const SelectArgs &a, const Shape &sh, const Tables &tb, const Plan &p, int dev,
                     cudaStream_t st, const uint32_t *flags, int grid_y) {
  cudaError_t e = ensure_attrs<GR, TOPP, SMEM>(dev, p.dyn_bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(select_kernel<GR, TOPP, SMEM>, dim3(p.cluster, grid_y, 1), dim3(kThreads), p.dyn_bytes, st,
                    p.cluster, a, sh, tb.ret, tb.n_ret, p.tc_cap, flags);
}

template <bool TOPP, bool SMEM>
int active_clusters_gr(const Tables &tb, const Plan &p, int dev) {
  switch (group_rows(tb)) {
    case 1: return active_clusters<1, TOPP, SMEM>(dev, p);
    case 2: return active_clusters<2, TOPP, SMEM>(dev, p);
    case 4: return active_clusters<4, TOPP, SMEM>(dev, p);
    case 8: return active_clusters<8, TOPP, SMEM>(dev, p);
    default: return active_clusters<16, TOPP, SMEM>(dev, p);
  }
}

template <bool TOPP, bool SMEM>
cudaError_t dispatch_gr(const SelectArgs &a, const Shape &sh, const Tables &tb, const Plan &p, int dev,
                        cudaStream_t st, const uint32_t *flags, int grid_y) {
  switch (group_rows(tb)) {
    case 1: return launch_t<1, TOPP, SMEM>(a, sh, tb, p, dev, st, flags, grid_y);
    case 2: return launch_t<2, TOPP, SMEM>(a, sh, tb, p, dev, st, flags, grid_y);
    case 4: return launch_t<4, TOPP, SMEM>(a, sh, tb, p, dev, st, flags, grid_y);
    case 8: return launch_t<8, TOPP, SMEM>(a, sh, tb, p, dev, st, flags, grid_y);
    default: return launch_t<16, TOPP, SMEM>(a, sh, tb, p, dev, st, flags, grid_y);
  }
}

// Per device, looked up once: the opt-in shared memory per block and the
// number of multiprocessors.
struct DeviceLimits {
  int smem;
  int sms;
};

DeviceLimits device_limits() {
  int dev = 0, v = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return DeviceLimits{v > 0 ? v : 48 * 1024, n > 0 ? n : 1};
}

}  // namespace

size_t select_workspace_bytes(const Shape &sh, const Tables &tb, int batch, size_t *flags_off) {
  // global score rows (used when the scores of a chunk do not fit on chip),
  // then one flag per work item, the count of flagged items and their list
  size_t rows = (size_t)batch * sh.H_ret * (size_t)sh.max_len * sizeof(float);
  rows = (rows + 255) / 256 * 256;
  if (flags_off) *flags_off = rows;
  return rows + (2 * (size_t)batch * std::max(1, tb.n_ret) + 1) * sizeof(uint32_t);
}

namespace {
cudaError_t launch_select_impl(const SelectArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st,
                               const UnionOut *uo, bool *unioned);
}  // namespace

cudaError_t launch_select(const SelectArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st) {
  return launch_select_impl(a, sh, tb, st, nullptr, nullptr);
}

cudaError_t launch_select_union(const SelectArgs &a, const Shape &sh, const Tables &tb, const UnionOut &uo,
                                cudaStream_t st, bool *unioned) {
  return launch_select_impl(a, sh, tb, st, &uo, unioned);
}

namespace {
cudaError_t launch_select_impl(const SelectArgs &a, const Shape &sh, const Tables &tb, cudaStream_t st,
                               const UnionOut *uo, bool *unioned) {
  if (unioned) *unioned = false;
  if (tb.n_ret == 0 || a.batch == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  const bool topp = a.mode == SD_TOP_P;
  static std::mutex mu;
  static std::map<int, DeviceLimits> limits;
  DeviceLimits lim;
  {
    std::lock_guard<std::mutex> lk(mu);
    auto it = limits.find(dev);
    if (it == limits.end()) it = limits.emplace(dev, device_limits()).first;
    lim = it->second;
  }
  Plan p = make_plan(sh, tb, a.batch, topp, lim.smem, lim.sms);
  // A cluster whose CTAs cannot be co-resident would fail to launch: fall back
  // to the portable size with scores in the workspace.
  const int fits = topp ? (p.smem ? active_clusters_gr<true, true>(tb, p, dev) : active_clusters_gr<true, false>(tb, p, dev))
                        : (p.smem ? active_clusters_gr<false, true>(tb, p, dev) : active_clusters_gr<false, false>(tb, p, dev));
  if (fits == 0) {
    const int c = std::min(p.cluster, 8);
    p.cluster = c;
    p.smem = false;
    p.tc_cap = (int)(((sh.max_len + c - 1) / c + kPage - 1) / kPage * kPage);
    p.dyn_bytes = hist_bytes(group_rows(tb), topp);
  }
  // exact-score mode: the score rows are in the workspace already and every
  // item goes through the exact selector; a CTA copies its chunk of them on
  // chip when the plan has room for it (else it reads them there at each pass)
  const int items = a.batch * tb.n_ret;
  bool used = false;
  if (!a.pre_scored) {
    cudaError_t e = launch_select_stream(a, sh, tb, a.flags, a.stream_ws, st, &used, uo, unioned);
    if (e != cudaSuccess) return e;
  }
  // after the streaming passes: exact recomputation of the items whose window
  // missed (usually none); without them: every item
  const uint32_t *flags = used ? a.flags : nullptr;
  // with the streaming passes the exact selector usually has nothing to do:
  // a few clusters stride over the flagged items (one wave of CTAs to launch)
  const int gy = used ? std::min(items, 4) : items;
  if (topp)
    return p.smem ? dispatch_gr<true, true>(a, sh, tb, p, dev, st, flags, gy)
                  : dispatch_gr<true, false>(a, sh, tb, p, dev, st, flags, gy);
  return p.smem ? dispatch_gr<false, true>(a, sh, tb, p, dev, st, flags, gy)
                : dispatch_gr<false, false>(a, sh, tb, p, dev, st, flags, gy);
}

}  // namespace

}  // namespace sd
