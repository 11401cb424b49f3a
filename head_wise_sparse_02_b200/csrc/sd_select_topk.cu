// Fixed-budget (top-k) selection: one streaming pass over the index.
//
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 2-3 and 5: the
// tokens of a retrieval head are scored in the r = 16 index space and a fixed
// top-k budget is kept; the threshold comes from a histogram, without
// sorting.  ICS page (gist.science/ar/paper/2605.24168), 2 and 3a: exact
// ("Oracle") top-k at ~2% of the context.
//
// Three launches, none of which waits on another CTA:
//   K0 window  one CTA per (sequence, KV group).  Computes q~ = c P_g^T q_pre
//              (float64, rounded to float32, split exactly into three bf16
//              terms) and scores a strided sample of <= 256 pages; from the
//              sample it sets, per head, a conservative score window
//              [t_lo, t_hi): t_lo a sample quantile safely below the k-th
//              score, t_hi the sample maximum.  Zeroes the head's buffer
//              counter.
//   K1 stream  many CTAs, each 512 pages of one (sequence, KV group): pages
//              arrive through a per-warp cp.async ring (16 bytes per lane,
//              XOR-swizzled rows), ldmatrix + mma.m16n8k16 score all heads of
//              the group at once (A = the 16 x 16 bf16 index page, B = the q~
//              terms), and every score at or above t_lo goes, with its
//              position, to a lane-private staging area in shared memory and
//              from there, in batches, to a per-head buffer.  Most scores
//              fail the single compare and cost nothing more.
//   K2 resolve one CTA per (sequence, retrieval head): histograms the
//              buffered scores over 512 bins of [t_lo, t_hi) (plus one bin for
//              scores >= t_hi), scans from the top for the bin holding the
//              k-th score and, while that bin holds many tokens, splits it
//              into 512 sub-bins and scans again (three levels at most); ranks
//              the tokens of the final bin exactly by (score desc, position
//              asc), marks the selected positions in a bitmap of the context
//              and writes them in ascending order.
// If the window misses (buffer overflow, k-th score outside the window, too
// many tokens in the cut bin), K2 flags the work item and the exact general
// kernel recomputes it.
#include <cuda_bf16.h>

#include <algorithm>
#include <map>
#include <mutex>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kBins = 512;            // window histogram bins (+1 slot: scores >= t_hi)
// K0: sampled pages per (sequence, group); the sample store is capped at 96 KB
__host__ __device__ constexpr int sample_pages(int GR) { return GR <= 4 ? 256 : (GR == 8 ? 192 : 96); }
constexpr int kSampleBins = 256;
constexpr int kChunkPages = 512;      // K1: pages per CTA
constexpr int kRing = 8;              // K1: pages in flight per warp (even); 4 CTAs per SM
// K1: staged buffer entries per (lane, head block); an iteration adds <= 4
__host__ __device__ constexpr int stage_lane(int GR) { return GR <= 4 ? 10 : (GR == 8 ? 8 : 5); }
constexpr int kCap = 2048;            // K2: cut-bin tokens ranked exactly
constexpr int kLevels = 3;            // K2: histogram levels (the cut bin is split again)
constexpr int kRefine = 64;           // K2: a cut bin above this many tokens is split again
constexpr int kPer2 = 16;             // K2: buffer entries held in registers per thread
constexpr int kPageBytes = kPage * kIndexDim * 2;   // 512 B: one page of one KV head
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
// byte offset of the 16-byte half `half` of row `row` inside a staged page;
// halves of rows 4-7 and 12-15 are swapped so that the eight rows an ldmatrix
// phase reads fall in distinct banks
__device__ __forceinline__ uint32_t page_off(int row, int half) {
  return (uint32_t)(row * 32 + ((half ^ ((row >> 2) & 1)) << 4));
}
__device__ __forceinline__ uint16_t bf16_rn(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float(uint32_t(h) << 16); }

// class of a score in the window of its head: kBins for scores >= t_hi, else
// the linear bin of [t_lo, t_hi); the same arithmetic in K1 and K2
__device__ __forceinline__ int window_bin(float s, float tlo, float thi, float inv) {
  if (s >= thi) return kBins;
  return min(kBins - 1, max(0, __float2int_rz((s - tlo) * inv)));
}

// One warp: the highest bin c of hist[0, nb) (nb a multiple of 32, at most
// 1024) whose suffix count sum_{b >= c} hist[b] reaches need (need >= 1);
// -1 when the whole histogram holds fewer.  *above = sum_{b > c} hist[b],
// *count = hist[c].  Each lane first sums its own nb / 32 consecutive bins,
// one suffix scan over the 32 group totals picks the group, a second one
// inside the group picks the bin.
__device__ int warp_cut_bin(const uint32_t *hist, int nb, uint32_t need, int lane, uint32_t *above,
                            uint32_t *count) {
  const int G = nb >> 5;
  uint32_t tot = 0;
  for (int j = 0; j < G; ++j) tot += hist[lane * G + j];
  uint32_t suf = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(kFull, suf, o);
    if (lane + o < 32) suf += y;
  }
  const unsigned bal = __ballot_sync(kFull, suf >= need);
  if (!bal) return -1;
  const int grp = 31 - __clz(bal);
  const uint32_t acc = __shfl_sync(kFull, suf - tot, grp);     // bins of the groups above grp
  const uint32_t c = lane < G ? hist[grp * G + lane] : 0u;
  uint32_t s2 = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(kFull, s2, o);
    if (lane + o < 32) s2 += y;
  }
  const unsigned bal2 = __ballot_sync(kFull, lane < G && acc + s2 >= need);
  const int j = 31 - __clz(bal2);                              // bal2 != 0: the group reaches need
  *count = __shfl_sync(kFull, c, j);
  *above = acc + __shfl_sync(kFull, s2, j) - *count;
  return grp * G + j;
}

struct TopkWs {
  uint32_t *qsplit;                   // [rows][24]: bf16 pairs of the q~ terms hi, mid, lo
  float4 *win;                        // [rows]: t_lo, t_hi, 1 / bin width, unused
  uint32_t *bcount;                   // [rows] buffer entries written
  int *rowitem;                       // [rows] work item of the row
  unsigned long long *buf;            // [rows][cap]: order key << 32 | position
  uint32_t *fail;                     // [items] flags, [1] count, [items] list of flagged items
  int items;
  int cap;
};

// B fragments of mma.m16n8k16 for head block hb: column n = gq of the first
// MMA carries head 4hb + gq/2, term gq%2 (hi, mid); of the second, the lo term
// for even gq and zero for odd gq.
struct BFrag {
  uint32_t v[2][2];
};
__device__ __forceinline__ BFrag load_bfrag(const uint32_t *qs /* [16 heads][24] */, int hb, int gq, int tq) {
  const int head = hb * 4 + (gq >> 1);
  const int part = gq & 1;
  const uint32_t *q = qs + head * 24;
  BFrag f;
  f.v[0][0] = q[part * 8 + tq];
  f.v[0][1] = q[part * 8 + tq + 4];
  f.v[1][0] = part == 0 ? q[16 + tq] : 0u;
  f.v[1][1] = part == 0 ? q[16 + tq + 4] : 0u;
  return f;
}
template <int HB>
__device__ __forceinline__ void score_frag(const uint32_t (&af)[4], const BFrag (&bf)[HB], float (&out)[HB][2]) {
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) {
    float d[4], e[4];
    mma_16816(d, af, bf[hb].v[0][0], bf[hb].v[0][1]);
    mma_16816(e, af, bf[hb].v[1][0], bf[hb].v[1][1]);
    out[hb][0] = (d[0] + d[1]) + e[0];               // row gq
    out[hb][1] = (d[2] + d[3]) + e[2];               // row gq + 8
  }
}

__device__ __forceinline__ long long topk_budget(const SelectArgs &a, long long N) {
  long long kb = a.top_k > 0 ? (long long)a.top_k
                             : std::max(1LL, (long long)floor((double)a.top_k_frac * (double)N));
  return std::min(kb, N);
}

// ------------------------------------------------------------------- K0
constexpr int kT0 = 512;

template <int GR>
__global__ void __launch_bounds__(kT0)
topk_window_kernel(const SelectArgs a, const Shape sh, const Group *__restrict__ groups, int n_groups,
                   const TopkWs ws) {
  constexpr int HB = (GR + 3) / 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int item = blockIdx.x;
  const int b = item / n_groups, gi = item % n_groups;
  constexpr int SP = sample_pages(GR);
  __shared__ Group grp;
  __shared__ uint32_t qs[16 * 24];
  __shared__ uint32_t smax[GR], smin[GR];
  __shared__ float hlo[GR], hinv[GR];
  __shared__ int spage[SP];
  extern __shared__ __align__(16) unsigned char dyn0[];
  float (*sample)[SP * 16] = reinterpret_cast<float (*)[SP * 16]>(dyn0);
  uint32_t (*shist)[kSampleBins] = reinterpret_cast<uint32_t (*)[kSampleBins]>(dyn0 + (size_t)GR * SP * 16 * 4);
  if (tid == 0) grp = groups[gi];
  __syncthreads();
  const int nr = grp.n, g = grp.kv_head;
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  const long long kb = topk_budget(a, N);
  if (tid == 0) {
    ws.fail[item] = 0u;
    if (item == 0) ws.fail[ws.items] = 0u;           // count of flagged items
  }
  if (tid < nr) {
    ws.bcount[(long long)b * sh.H_ret + grp.row[tid]] = 0u;
    ws.rowitem[(long long)b * sh.H_ret + grp.row[tid]] = item;
  }
  if (N == 0 || kb >= N) return;                     // K1 skips, K2 keeps everything

  // q~ in float64 (one warp per head, lanes split d) -> float32 -> hi/mid/lo
  for (int i = warp; i < 16; i += kT0 / 32) {
    double acc[kIndexDim];
#pragma unroll
    for (int j = 0; j < kIndexDim; ++j) acc[j] = 0.0;
    if (i < nr) {
      const uint16_t *qrow = a.q_pre + ((long long)b * sh.Hq + grp.q_head[i]) * sh.d;
      const uint16_t *P = a.proj + (long long)g * sh.d * kIndexDim;
      for (int e = lane; e < sh.d; e += 32) {
        const double qe = (double)bf16_to_f32(qrow[e]);
        const uint4 p0 = __ldg(reinterpret_cast<const uint4 *>(P + e * kIndexDim));
        const uint4 p1 = __ldg(reinterpret_cast<const uint4 *>(P + e * kIndexDim + 8));
        const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc[2 * j] = fma(qe, (double)bf16_lo(pw[j]), acc[2 * j]);
          acc[2 * j + 1] = fma(qe, (double)bf16_hi(pw[j]), acc[2 * j + 1]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kIndexDim; ++j)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(kFull, acc[j], o);
    if (lane < kIndexDim) {
      double v = 0.0;
#pragma unroll
      for (int j = 0; j < kIndexDim; ++j) v = (lane == j) ? acc[j] : v;
      const float x = (float)(v * (double)a.index_scale);
      const uint16_t hi = bf16_rn(x);
      const float r1 = x - bf16_val(hi);             // exact in float32
      const uint16_t mid = bf16_rn(r1);
      const uint16_t lo = bf16_rn(r1 - bf16_val(mid));
      uint16_t *q16 = reinterpret_cast<uint16_t *>(qs + i * 24);
      q16[lane] = hi;
      q16[16 + lane] = mid;
      q16[32 + lane] = lo;
    }
  }
  if (tid < GR) {
    smax[tid] = 0u;
    smin[tid] = 0xFFFFFFFFu;
  }
  for (int o = tid; o < GR * kSampleBins; o += kT0) (&shist[0][0])[o] = 0u;
  __syncthreads();
  for (int o = tid; o < nr * 24; o += kT0)           // publish the q~ terms for K1
    ws.qsplit[((long long)b * sh.H_ret + grp.row[o / 24]) * 24 + o % 24] = qs[o];

  // sample: pages j * st, j < ns; their page ids first, all at once
  const int pages = (int)((N + kPage - 1) / kPage);
  int st = 1;
  while ((long long)st * SP < pages) st <<= 1;
  const int ns = (pages + st - 1) / st;
  const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
  for (int j = tid; j < ns; j += kT0) {
    const int page = pt[j * st];
    const bool ok = page >= 0 && page < sh.num_pages;
    spage[j] = ok ? page : -1;
    if (!ok) raise_error(a.err, SD_EBIT_PAGE);
  }
  __syncthreads();
  BFrag bf[HB];
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) bf[hb] = load_bfrag(qs, hb, gq, tq);
  const uint16_t *icache = a.index_cache + (long long)g * (kPage * kIndexDim);
  const long long page_stride = (long long)sh.Hkv * (kPage * kIndexDim);
  float smx[HB], smn[HB];
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) {
    smx[hb] = -INFINITY;
    smn[hb] = INFINITY;
  }
  constexpr int U = 16;
  for (int j0 = warp; j0 < ns; j0 += (kT0 / 32) * U) {
    uint32_t af[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * (kT0 / 32);
      af[u][0] = af[u][1] = af[u][2] = af[u][3] = 0u;
      const int page = j < ns ? spage[j] : -1;
      if (page >= 0) {
        const uint32_t *pg = reinterpret_cast<const uint32_t *>(icache + page * page_stride);
        af[u][0] = __ldg(pg + gq * 8 + tq);
        af[u][1] = __ldg(pg + (gq + 8) * 8 + tq);
        af[u][2] = __ldg(pg + gq * 8 + tq + 4);
        af[u][3] = __ldg(pg + (gq + 8) * 8 + tq + 4);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * (kT0 / 32);
      if (j >= ns) break;
      const bool ok = spage[j] >= 0;
      float sc[HB][2];
      score_frag<HB>(af[u], bf, sc);
#pragma unroll
      for (int hb = 0; hb < HB; ++hb) {
        const int h = hb * 4 + tq;
        if (h >= GR) continue;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = gq + 8 * r;
          const bool valid = ok && (long long)j * st * kPage + row < N;
          const float v = valid ? sc[hb][r] : -INFINITY;
          sample[h][j * 16 + row] = v;
          if (valid) {
            smx[hb] = fmaxf(smx[hb], v);
            smn[hb] = fminf(smn[hb], v);
          }
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
      atomicMax(&smax[h], order_key(smx[hb]));
      atomicMin(&smin[h], order_key(smn[hb]));
    }
  }
  __syncthreads();
  if (tid < nr) {
    const float lo = key_to_float(smin[tid]), hi = key_to_float(smax[tid]);
    hlo[tid] = lo;
    hinv[tid] = (smax[tid] != 0u && hi > lo) ? (float)kSampleBins / (hi - lo) : 0.0f;
  }
  __syncthreads();
  for (int o = tid; o < nr * ns * 16; o += kT0) {
    const int h = o / (ns * 16), r = o % (ns * 16);
    const float v = sample[h][r];
    if (v == -INFINITY) continue;
    atomicAdd(&shist[h][std::min(kSampleBins - 1, std::max(0, __float2int_rz((v - hlo[h]) * hinv[h])))], 1u);
  }
  __syncthreads();
  // one warp per head: the highest bin whose suffix count reaches r
  for (int h = warp; h < nr; h += kT0 / 32) {
    // valid sample tokens: every sampled page is full except possibly the last
    const long long m = (long long)(ns - 1) * kPage + std::min<long long>(kPage, N - (long long)(ns - 1) * st * kPage);
    float tlo = -INFINITY, thi = INFINITY;
    if (smax[h] != 0u) {
      const float lo = hlo[h], hi = key_to_float(smax[h]);
      thi = hi;
      const double mu = (double)m * (double)kb / (double)N;
      const double r = ceil(mu + 6.0 * sqrt(mu) + 8.0);
      if (r < (double)m) {
        uint32_t above, cnt;
        const int c = warp_cut_bin(shist[h], kSampleBins, (uint32_t)r, lane, &above, &cnt);
        const int blo = c < 0 ? 0 : c;
        tlo = lo + (float)blo * ((hi - lo) / (float)kSampleBins);
      }
    }
    const float inv = (tlo > -INFINITY && thi > tlo) ? (float)kBins / (thi - tlo) : 0.0f;
    if (lane == 0) ws.win[(long long)b * sh.H_ret + grp.row[h]] = make_float4(tlo, thi, inv, 0.0f);
  }
}

// ------------------------------------------------------------------- K1
constexpr int kT1 = 256;
constexpr int kW1 = kT1 / 32;

template <int GR>
__global__ void __launch_bounds__(kT1)
topk_stream_kernel(const SelectArgs a, const Shape sh, const Group *__restrict__ groups, int n_groups,
                   const TopkWs ws) {
  constexpr int HB = (GR + 3) / 4;
  constexpr int SL = stage_lane(GR);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  // item fastest in the launch order: CTAs of all KV groups for the same
  // chunk of pages run together, so reads of the groups' 512-byte slices of a
  // page (adjacent in the index cache) meet in the same DRAM rows
  const int item = blockIdx.x;
  const int b = item / n_groups, gi = item % n_groups;
  extern __shared__ __align__(128) unsigned char dyn1[];
  unsigned char (*ring)[kRing][kPageBytes] = reinterpret_cast<unsigned char (*)[kRing][kPageBytes]>(dyn1);
  // lane-private staging: entry e of (warp, head block hb) for lane l at stage[warp][hb][e][l]
  unsigned long long (*stage)[HB][SL][32] =
      reinterpret_cast<unsigned long long (*)[HB][SL][32]>(dyn1 + (size_t)kW1 * kRing * kPageBytes);
  __shared__ int32_t pt_s[kChunkPages];
  __shared__ uint32_t qs[16 * 24];
  __shared__ Group grp;
  if (tid == 0) grp = groups[gi];
  __syncthreads();
  const int nr = grp.n, g = grp.kv_head;
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  const long long kb = topk_budget(a, N);
  if (N == 0 || kb >= N) return;
  const int pages = (int)((N + kPage - 1) / kPage);
  const int p0 = blockIdx.y * kChunkPages;
  if (p0 >= pages) return;
  const int np = pages - p0 < kChunkPages ? pages - p0 : kChunkPages;
  {
    // page id -> page * Hkv + g (the 512-byte index block of this KV head), or -1
    const int32_t *pt = a.page_table + (long long)b * sh.max_pages + p0;
    for (int o = tid; o < np; o += kT1) {
      const int page = pt[o];
      const bool ok = page >= 0 && page < sh.num_pages;
      pt_s[o] = ok ? page * sh.Hkv + g : -1;
      if (!ok) raise_error(a.err, SD_EBIT_PAGE);
    }
    for (int o = tid; o < 16 * 24; o += kT1) {
      const int i = o / 24;
      qs[o] = i < nr ? ws.qsplit[((long long)b * sh.H_ret + grp.row[i]) * 24 + o % 24] : 0u;
    }
  }
  __syncthreads();

  // per-warp ring: this warp reads pages warp, warp + 8, ... of the chunk
  const uint32_t ring_base = (uint32_t)__cvta_generic_to_shared(&ring[warp][0][0]);
  const unsigned char *iblk = reinterpret_cast<const unsigned char *>(a.index_cache) + lane * 16;
  const uint32_t st_off = page_off(lane >> 1, lane & 1);
  const int nq = np > warp ? (np - warp + kW1 - 1) / kW1 : 0;
  auto issue = [&](int q) {
    if (q < nq) {
      const int blk = pt_s[warp + q * kW1];
      cp_async16(ring_base + (q % kRing) * kPageBytes + st_off, iblk + (size_t)(blk >= 0 ? blk : 0) * kPageBytes,
                 blk >= 0 ? 16 : 0);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int q = 0; q < kRing; ++q) issue(q);

  BFrag bf[HB];
  float tlo[HB];
  long long row_of[HB];
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) {
    bf[hb] = load_bfrag(qs, hb, gq, tq);
    const int h = hb * 4 + tq;
    row_of[hb] = h < nr ? (long long)b * sh.H_ret + grp.row[h] : 0;
    tlo[hb] = h < nr ? ws.win[row_of[hb]].x : INFINITY;   // absent heads keep nothing
  }
  uint32_t cnt[HB];
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) cnt[hb] = 0u;
  // move the warp's staged entries to the heads' buffers: the 8 lanes of a
  // head (same tq) take consecutive ranges of one reservation
  auto flush = [&]() {
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
      const int h = hb * 4 + tq;
      uint32_t incl = cnt[hb];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t tot = __shfl_sync(kFull, incl, 28 + tq);
      uint32_t base = 0u;
      if (gq == 0 && h < nr && tot > 0u) base = atomicAdd(&ws.bcount[row_of[hb]], tot);
      base = __shfl_sync(kFull, base, tq) + (incl - cnt[hb]);
      if (h < nr) {
        unsigned long long *dst = ws.buf + row_of[hb] * ws.cap;
        for (uint32_t e = 0; e < cnt[hb]; ++e)
          if (base + e < (uint32_t)ws.cap) dst[base + e] = stage[warp][hb][e][lane];
      }
      cnt[hb] = 0u;
    }
    __syncwarp();
  };
  const uint32_t ld = ring_base + page_off((lane & 7) + ((lane >> 3) & 1) * 8, lane >> 4);
  const uint32_t n32 = (uint32_t)N;
  // two pages per iteration (q, q + 1); one cp.async group per page
  for (int q = 0; q < nq; q += 2) {
    cp_async_wait<kRing - 2>();
    __syncwarp();
    uint32_t af[2][4];
    ldmatrix_x4(af[0], ld + (q % kRing) * kPageBytes);
    ldmatrix_x4(af[1], ld + ((q + 1) % kRing) * kPageBytes);
    __syncwarp();
    const int pl = warp + q * kW1;                   // page within the chunk
    const bool ok0 = pt_s[pl] >= 0;
    const bool ok1 = q + 1 < nq && pt_s[pl + kW1] >= 0;
    issue(q + kRing);
    issue(q + kRing + 1);
    float sc[2][HB][2];
    score_frag<HB>(af[0], bf, sc[0]);
    score_frag<HB>(af[1], bf, sc[1]);
    const uint32_t pos0 = (uint32_t)(p0 + pl) * kPage + gq;
    bool full = false;
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
#pragma unroll
      for (int u = 0; u < 2; ++u) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint32_t pos = pos0 + u * (kW1 * kPage) + 8 * r;
          const float s = sc[u][hb][r];
          if ((u ? ok1 : ok0) && s >= tlo[hb] && pos < n32) {
            stage[warp][hb][cnt[hb]][lane] = ((unsigned long long)order_key(s) << 32) | pos;
            ++cnt[hb];
          }
        }
      }
      full |= cnt[hb] > (uint32_t)(SL - 4);
    }
    if (__any_sync(kFull, full)) flush();
  }
  flush();
  cp_async_wait<0>();
}

// ------------------------------------------------------------------- K2
constexpr int kT2 = 256;

__global__ void __launch_bounds__(kT2, 4)
topk_resolve_kernel(const SelectArgs a, const Shape sh, const TopkWs ws) {
  extern __shared__ uint32_t bitmap[];               // [max_len / 32]
  __shared__ unsigned long long cand[kCap];
  __shared__ uint32_t hist[kBins + 1];
  __shared__ uint32_t n_cand;
  __shared__ int fail_s, done_s;
  __shared__ long long need_s;
  __shared__ int cutv[kLevels];
  __shared__ float llo[kLevels], linv[kLevels];
  __shared__ uint32_t wtot[kT2 / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.y, hr = blockIdx.x;
  const long long row = (long long)b * sh.H_ret + hr;
  int32_t *out = a.sel_idx + row * a.sel_stride;
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  const long long kb = topk_budget(a, N);
  if (N == 0 || kb >= N) {
    for (long long t = tid; t < N; t += kT2) {
      if (t < a.sel_stride) out[t] = (int32_t)t;
      else raise_error(a.err, SD_EBIT_SEL);
    }
    if (tid == 0) a.sel_count[row] = (int32_t)std::min(N, a.sel_stride);
    return;
  }
  const float4 w = ws.win[row];
  const uint32_t nbuf = ws.bcount[row];
  const unsigned long long *buf = ws.buf + row * ws.cap;
  const int n = (int)std::min<uint32_t>(nbuf, (uint32_t)ws.cap);
  const int words = (int)((N + 31) / 32);
  for (int o = tid; o < words; o += kT2) bitmap[o] = 0u;
  if (tid == 0) {
    llo[0] = w.x;
    linv[0] = w.z;
    need_s = kb;
    fail_s = 0;
    done_s = 0;
    n_cand = 0u;
  }
  // bin of a score at level L: level 0 is the window histogram (bin kBins:
  // scores >= t_hi); level L > 0 splits the cut bin of level L - 1 into kBins
  // linear sub-bins.  Bins are non-decreasing in the score at every level.
  auto bin_at = [&](float v, int L) -> int {
    if (L == 0) return window_bin(v, w.x, w.y, w.z);
    return min(kBins - 1, max(0, __float2int_rz((v - llo[L]) * linv[L])));
  };
  // this thread's first kPer2 entries, loaded once (the passes below reread
  // only entries past kPer2 * kT2 from memory)
  unsigned long long ent[kPer2];
#pragma unroll
  for (int j = 0; j < kPer2; ++j) {
    const int e = tid + j * kT2;
    ent[j] = e < n ? buf[e] : 0ull;
  }
  // the cut bin: refine while it holds more than kRefine tokens
  int L = 0;
  for (; L < kLevels; ++L) {
    for (int o = tid; o <= kBins; o += kT2) hist[o] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kPer2; ++j) {
      const int e = tid + j * kT2;
      if (e < n) {
        const float v = key_to_float((uint32_t)(ent[j] >> 32));
        bool play = true;
        for (int l = 0; l < L; ++l) play = play && bin_at(v, l) == cutv[l];
        if (play) atomicAdd(&hist[bin_at(v, L)], 1u);
      }
    }
    for (int e = tid + kPer2 * kT2; e < n; e += kT2) {
      const float v = key_to_float((uint32_t)(buf[e] >> 32));
      bool play = true;
      for (int l = 0; l < L; ++l) play = play && bin_at(v, l) == cutv[l];
      if (play) atomicAdd(&hist[bin_at(v, L)], 1u);
    }
    __syncthreads();
    // warp 0 finds the bin holding the cut among the level's bins
    if (warp == 0) {
      const long long need = need_s - (L == 0 ? (long long)hist[kBins] : 0LL);
      uint32_t above = 0, ncut = 0;
      const int cut = need > 0 ? warp_cut_bin(hist, kBins, (uint32_t)need, lane, &above, &ncut) : -1;
      const long long acc = above;
      if (lane == 0) {
        if (need <= 0 || cut < 0 || nbuf > (uint32_t)ws.cap) {
          fail_s = 1;
        } else {
          cutv[L] = cut;
          need_s = need - acc;                       // tokens still to take from the cut bin
          const bool last = ncut <= kRefine || L + 1 == kLevels;
          if (last && ncut > kCap) fail_s = 1;
          if (!last) {
            llo[L + 1] = llo[L] + (float)cut / linv[L];
            linv[L + 1] = linv[L] * (float)kBins;
          }
          done_s = last;
        }
      }
    }
    __syncthreads();
    if (fail_s || done_s) break;
  }
  if (fail_s) {
    if (tid == 0) {
      const int it = ws.rowitem[row];
      if (atomicExch(&ws.fail[it], 1u) == 0u) ws.fail[ws.items + 1 + atomicAdd(&ws.fail[ws.items], 1u)] = (uint32_t)it;
    }
    return;
  }
  const int nlev = L + 1;
  // classify: above the cut path -> selected; on it -> candidate
  auto classify = [&](unsigned long long en) {
    const uint32_t key = (uint32_t)(en >> 32), pos = (uint32_t)en;
    const float v = key_to_float(key);
    int rel = 0;
    for (int l = 0; l < nlev && rel == 0; ++l) {
      const int bl = bin_at(v, l);
      rel = bl > cutv[l] ? 1 : (bl < cutv[l] ? -1 : 0);
    }
    if (rel > 0) {
      atomicOr(&bitmap[pos >> 5], 1u << (pos & 31));
    } else if (rel == 0) {
      const uint32_t at = atomicAdd(&n_cand, 1u);
      if (at < (uint32_t)kCap) cand[at] = ((unsigned long long)(~key) << 32) | pos;   // ascending = better first
    }
  };
#pragma unroll
  for (int j = 0; j < kPer2; ++j)
    if (tid + j * kT2 < n) classify(ent[j]);
  for (int e = tid + kPer2 * kT2; e < n; e += kT2) classify(buf[e]);
  __syncthreads();
  // rank the cut bin exactly: the need_c best by (score desc, position asc)
  const int nc = (int)std::min<uint32_t>(n_cand, (uint32_t)kCap);
  const long long need_c = need_s;
  for (int e = tid; e < nc; e += kT2) {
    const unsigned long long me = cand[e];
    int rk = 0;
    for (int j = 0; j < nc; ++j) rk += cand[j] < me;
    if (rk < need_c) {
      const uint32_t pos = (uint32_t)me;
      atomicOr(&bitmap[pos >> 5], 1u << (pos & 31));
    }
  }
  __syncthreads();
  // ordered write: contiguous word ranges per thread, block-wide prefix
  const int wpt = (words + kT2 - 1) / kT2;
  const int w0 = tid * wpt, w1 = std::min(words, w0 + wpt);
  uint32_t c = 0;
  for (int x = w0; x < w1; ++x) c += __popc(bitmap[x]);
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  uint32_t base = 0, total = 0;
  for (int x = 0; x < kT2 / 32; ++x) {
    if (x < warp) base += wtot[x];
    total += wtot[x];
  }
  long long o = base + incl - c;
  for (int x = w0; x < w1; ++x) {
    uint32_t bits = bitmap[x];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      if (o < a.sel_stride) out[o] = x * 32 + bit;
      else raise_error(a.err, SD_EBIT_SEL);
      ++o;
    }
  }
  if (tid == 0) {
    if ((long long)total > a.sel_stride) raise_error(a.err, SD_EBIT_SEL);
    a.sel_count[row] = (int32_t)std::min<long long>(total, a.sel_stride);
  }
}

// ------------------------------------------------------------------- host
struct TopkPlan {
  int cap;
  size_t bitmap_bytes;
  bool ok;
};

TopkPlan topk_plan(const Shape &sh, const Tables &tb) {
  TopkPlan p{};
  p.cap = (int)std::min<long long>(sh.max_len, std::max<long long>(4096, sh.max_len / 8));
  p.bitmap_bytes = (size_t)((sh.max_len + 31) / 32) * 4;
  p.ok = tb.max_ret <= 16 && p.bitmap_bytes <= 160 * 1024 && sh.max_len < (1LL << 31);
  return p;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct TopkLayout {
  size_t qsplit, win, bcount, rowitem, buf, total;
};

TopkLayout topk_layout(const Shape &sh, int batch, int cap) {
  TopkLayout L{};
  const size_t rows = (size_t)batch * std::max(1, sh.H_ret);
  size_t o = 0;
  L.qsplit = o;  o = align256(o + rows * 24 * 4);
  L.win = o;     o = align256(o + rows * 16);
  L.bcount = o;  o = align256(o + rows * 4);
  L.rowitem = o; o = align256(o + rows * 4);
  L.buf = o;     o = align256(o + rows * (size_t)cap * 8);
  L.total = o;
  return L;
}

// dynamic shared memory attributes, set once per kernel and device
template <typename K>
cudaError_t set_smem_once(K kern, size_t bytes) {
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

template <int GR>
cudaError_t topk_launch(const SelectArgs &a, const Shape &sh, const Tables &tb, const TopkWs &ws,
                        size_t bitmap_bytes, cudaStream_t st) {
  const int items = a.batch * tb.n_ret;
  const size_t smem0 = (size_t)GR * sample_pages(GR) * 16 * 4 + (size_t)GR * kSampleBins * 4;
  const size_t smem1 = (size_t)kW1 * kRing * kPageBytes + (size_t)kW1 * ((GR + 3) / 4) * stage_lane(GR) * 32 * 8;
  cudaError_t e = set_smem_once(topk_window_kernel<GR>, smem0);
  if (e == cudaSuccess) e = set_smem_once(topk_stream_kernel<GR>, smem1);
  if (e == cudaSuccess) e = set_smem_once(topk_resolve_kernel, bitmap_bytes);
  if (e != cudaSuccess) return e;
  topk_window_kernel<GR><<<items, kT0, smem0, st>>>(a, sh, tb.ret, tb.n_ret, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int chunks = (int)((sh.max_pages + kChunkPages - 1) / kChunkPages);
  topk_stream_kernel<GR><<<dim3(items, chunks), kT1, smem1, st>>>(a, sh, tb.ret, tb.n_ret, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topk_resolve_kernel<<<dim3(sh.H_ret, a.batch), kT2, bitmap_bytes, st>>>(a, sh, ws);
  return cudaGetLastError();
}

}  // namespace

size_t topk_workspace_bytes(const Shape &sh, const Tables &tb, int batch) {
  const TopkPlan p = topk_plan(sh, tb);
  if (!p.ok) return 0;
  return topk_layout(sh, batch, p.cap).total;
}

cudaError_t launch_select_topk_stream(const SelectArgs &a, const Shape &sh, const Tables &tb, uint32_t *fail,
                                      void *ws_base, cudaStream_t st, bool *used) {
  *used = false;
  const TopkPlan p = topk_plan(sh, tb);
  if (!p.ok || ws_base == nullptr) return cudaSuccess;
  const TopkLayout L = topk_layout(sh, a.batch, p.cap);
  char *base = static_cast<char *>(ws_base);
  TopkWs ws{};
  ws.qsplit = reinterpret_cast<uint32_t *>(base + L.qsplit);
  ws.win = reinterpret_cast<float4 *>(base + L.win);
  ws.bcount = reinterpret_cast<uint32_t *>(base + L.bcount);
  ws.rowitem = reinterpret_cast<int *>(base + L.rowitem);
  ws.buf = reinterpret_cast<unsigned long long *>(base + L.buf);
  ws.fail = fail;
  ws.items = a.batch * tb.n_ret;
  ws.cap = p.cap;
  int gr = 1;
  while (gr < tb.max_ret) gr <<= 1;
  cudaError_t e;
  switch (gr) {
    case 1: e = topk_launch<1>(a, sh, tb, ws, p.bitmap_bytes, st); break;
    case 2: e = topk_launch<2>(a, sh, tb, ws, p.bitmap_bytes, st); break;
    case 4: e = topk_launch<4>(a, sh, tb, ws, p.bitmap_bytes, st); break;
    case 8: e = topk_launch<8>(a, sh, tb, ws, p.bitmap_bytes, st); break;
    default: e = topk_launch<16>(a, sh, tb, ws, p.bitmap_bytes, st); break;
  }
  if (e == cudaSuccess) *used = true;
  return e;
}

}  // namespace sd
