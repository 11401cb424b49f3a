// Streaming selection: top-k and top-p without a sort, in passes over the
// index that no CTA waits on.
//
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 2-3 and 5: the
// tokens of a retrieval head are scored in the r = 16 index space; a fixed
// top-k budget, or a dynamic top-p set (softmax mass of the index scores
// accumulated from the top until it reaches p), is kept, and the threshold
// comes from a histogram, without sorting.  ICS page
// (gist.science/ar/paper/2605.24168), 2 and 3a: exact ("Oracle") top-k at ~2%
// of the context.
//
// Every pass streams the index through per-warp cp.async rings (16 bytes per
// lane, XOR-swizzled rows, L2 evict-first) and scores all heads of a KV group
// at once with ldmatrix + mma.m16n8k16 (A = the 16 x 16 bf16 index page, B =
// the q~ terms).  One bulk copy (cp.async.bulk) per 512-byte page, issued by
// one lane and counted on an mbarrier, was measured 1.6x slower here: more
// instructions per page and one CTA less per SM.
//
// K0 window  one CTA per (sequence, KV group).  Computes q~ = c P_g^T q_pre
//            (float64, rounded to float32, split exactly into three bf16
//            terms) and scores a strided sample of <= 256 pages; from the
//            sample it sets, per head, a score window [t_lo, t_hi): t_lo a
//            sample quantile safely below the threshold, t_hi the sample
//            maximum.  Zeroes the head's counters.
//
// top-k (three launches)
//   K1 stream  many CTAs, each 512 pages of one (sequence, KV group): every
//              score at or above t_lo goes, with its position, to a
//              lane-private staging area in shared memory and from there, in
//              batches, to a per-head buffer.  Most scores fail the single
//              compare and cost nothing more.
//   K2 resolve one CTA per (sequence, retrieval head): histograms the
//              buffered scores over 2048 bins of [t_lo, t_hi) (plus one bin
//              for scores >= t_hi), scans from the top for the bin holding
//              the k-th score and, while that bin holds many tokens, splits
//              it into 2048 sub-bins and scans again (three levels at most);
//              ranks the tokens of the final bin exactly by (score desc,
//              position asc), marks the selected positions in a bitmap of the
//              context and writes them in ascending order.
//
// In the joined select + attend call with many items, K2 of either mode runs
// fused: one CTA per (sequence, retrieval KV group) resolves all its heads and
// writes the group's union list straight into attend's workspace.
//
// top-p (four launches; the softmax mass of a head is known only after a
// whole pass, so the index is streamed twice)
//   K1 mass    per chunk: the softmax weight w = 2^((s - t_hi) log2 e) of
//              every score goes to a float64 sum (scores below t_lo) or to a
//              1024-bin mass histogram of [t_lo, t_hi) plus one bin for scores
//              >= t_hi, kept per CTA in shared memory and added to the head's
//              histogram at the end.
//   K1 cut     per chunk: every CTA derives the same cut bin from the head's
//              histogram (the highest bin whose mass, with the mass above
//              it, reaches p Z); tokens of higher bins go to a bitmap of the
//              context, tokens of the cut bin to the head's candidate buffer.
//   K2 resolve one CTA per (sequence, retrieval head): an exact radix search
//              over the candidates' order keys (9 bits per level, float64
//              mass per digit) finds the threshold score tau inside the cut
//              bin; candidates >= tau join the bitmap, which is written out
//              in ascending order.  Ties at tau are all kept.
//
// If the window misses (top-k: buffer overflow, k-th score outside the
// window, too many tokens in the cut bin; top-p: the cut below t_lo, too many
// candidates, a weight out of float range), K2 flags the work item and the
// exact general kernel recomputes it.
#include <cuda_bf16.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <type_traits>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kBins = 512;            // window histogram bins (+1 slot: scores >= t_hi)
// K0: sampled pages per (sequence, group); the sample store is capped at 96 KB
__host__ __device__ constexpr int sample_pages(int GR) { return GR <= 4 ? 256 : (GR == 8 ? 192 : 96); }
constexpr int kSampleBins = 256;
// set bits per warp step above which write_ascending's lanes write their own
// bits (the union lists keep the coalesced emission: measured faster there)
constexpr int kDenseBits = 256;
constexpr int kChunkPages = 512;      // K1: pages per CTA (at most; fewer when the items are few)
constexpr int kRing = 8;              // K1: pages in flight per warp (even); 4 CTAs per SM
// K1: staged buffer entries per (lane, head block); an iteration adds <= 4
__host__ __device__ constexpr int stage_lane(int GR) { return GR <= 4 ? 10 : (GR == 8 ? 8 : 5); }
constexpr int kBinsK = 2048;          // top-k K2: bins of the window and of each refinement level
constexpr int kCap = 2048;            // K2: cut-bin tokens ranked exactly
constexpr int kLevels = 3;            // K2: histogram levels (the cut bin is split again)
constexpr int kRefine = 256;          // K2: a cut bin above this many tokens is split again
// K2: buffer entries held in registers per thread (the rest of the buffer is
// read from L2 at each pass), by the launch's register budget: with 64
// registers a thread, 16 entries (32 registers) spilled; the fused union
// resolve, whose union walk needs more of them, holds 8
__host__ __device__ constexpr int per_thread_entries(int cta_threads, int ctas_per_sm) {
  return 65536 / (cta_threads * ctas_per_sm) > 64 ? 16 : (cta_threads >= 1024 ? 8 : 12);
}
constexpr int kRestBatch = 4;         // K2: buffer entries past the registers loaded at once per thread
constexpr int kPageBytes = kPage * kIndexDim * 2;   // 512 B: one page of one KV head
constexpr unsigned kFull = 0xFFFFFFFFu;
// top-p window (K0): the sample's kExcl highest tokens are left out of its
// mass estimate (one planted needle in the sample must not make the mass look
// concentrated); the mass below t_lo is estimated kMassSafety times over; the
// count above t_lo gets kCountSigmas standard deviations (plus 8) of margin
constexpr int kExcl = 8;
constexpr double kMassSafety = 2.0;
constexpr double kCountSigmas = 6.0;
constexpr int kBinsP = 1024;          // top-p window bins (+1 slot: scores >= t_hi); 32 per lane of a warp
constexpr int kCapP = 4096;           // top-p: cut-bin candidates per head
constexpr float kLog2e = 1.4426950408889634f;
// top-p: a score this far above t_hi (nats) is flagged, so that no float
// weight, nor a chunk's float sum of up to 512 x 16 x 16 of them, overflows
constexpr float kMaxLogit = 60.0f;

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
template <int NB = kBins>
__device__ __forceinline__ int window_bin(float s, float tlo, float thi, float inv) {
  if (s >= thi) return NB;
  return min(NB - 1, max(0, __float2int_rz((s - tlo) * inv)));
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

// One warp, float64 masses: the cut bin of a top-p head.  hist[0, kBinsP)
// holds the mass of the window's bins, hist[kBinsP] that of scores >= t_hi,
// zlo that of scores below t_lo.  Returns the highest bin c whose mass plus
// the mass above it reaches need = p Z (kBinsP when the top bin alone does),
// with *above = the mass strictly above c; -1 when the window's bins together
// fall short (the threshold lies below t_lo).  Every step is a fixed sequence
// of shuffles, so every caller reading the same histogram gets the same bin.
__device__ int warp_cut_mass(const double *hist, double zlo, double p, int lane, double *above, double *need) {
  constexpr int G = kBinsP / 32;
  double tot = 0.0;
  for (int j = 0; j < G; ++j) tot += hist[lane * G + j];
  double zw = tot;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) zw += __shfl_xor_sync(kFull, zw, o);   // the same on every lane
  const double top = hist[kBinsP];
  const double nd = p * ((zlo + zw) + top);
  *need = nd;
  *above = 0.0;
  if (top >= nd) return kBinsP;
  const double n2 = nd - top;
  double suf = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_down_sync(kFull, suf, o);
    if (lane + o < 32) suf += y;
  }
  const unsigned bal = __ballot_sync(kFull, suf >= n2);
  if (!bal) return -1;
  const int grp = 31 - __clz(bal);
  const double acc = __shfl_sync(kFull, suf - tot, grp);
  const double c = lane < G ? hist[grp * G + lane] : 0.0;
  double s2 = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_down_sync(kFull, s2, o);
    if (lane + o < 32) s2 += y;
  }
  unsigned bal2 = __ballot_sync(kFull, lane < G && acc + s2 >= n2);
  // summed in another order the group may fall short by a rounding: its
  // lowest bin with mass then
  if (!bal2) {
    const unsigned nz = __ballot_sync(kFull, lane < G && c > 0.0);
    bal2 = nz & (0u - nz);
  }
  const int j = bal2 ? 31 - __clz(bal2) : 0;
  *above = top + acc + __shfl_sync(kFull, s2, j) - __shfl_sync(kFull, c, j);
  return grp * G + j;
}

struct StreamWs {
  uint32_t *qsplit;                   // [rows][24]: bf16 pairs of the q~ terms hi, mid, lo
  float4 *win;                        // [rows]: t_lo, t_hi, 1 / bin width, unused
  uint32_t *bcount;                   // [rows] buffer entries written
  int *rowitem;                       // [rows] work item of the row
  unsigned long long *buf;            // [rows][cap]: order key << 32 | position
  uint32_t *fail;                     // [items] flags, [1] count, [items] list of flagged items
  double *hist;                       // top-p: [rows][kBinsP + 1] softmax mass per window bin
  double *zlo;                        // top-p: [rows] softmax mass below t_lo
  uint32_t *rflag;                    // top-p: [rows] nonzero: the window cannot resolve the row
  uint32_t *bits;                     // top-p: [rows][bwords] tokens above the cut bin
  long long bwords;
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

// t_lo of a top-p head from its sample (one warp): m valid sample tokens out
// of N, cnt / mass the sample's histograms over kSampleBins bins of [lo, hi]
// (mass relative to the sample maximum hi).  The mass below a bin edge t is
// estimated as (N / m) x the sample's mass below t; the total as that scaled
// mass up to the bin of the kExcl-th highest sample token plus the mass above
// it unscaled (heavy sampled tokens are real but need not be typical).  t_lo
// is the highest edge whose estimated mass below, taken kMassSafety times,
// stays within (1 - p) of the total, lowered further to hold kCountSigmas
// standard deviations (plus 8) more sample tokens; the sample minimum when
// that asks for more tokens than the sample has.
__device__ float topp_window_lo(const uint32_t *cnt, const float *mass, float lo, float hi, long long m,
                                long long N, double p, int lane) {
  constexpr int PB = kSampleBins / 32;               // bins per lane
  uint32_t above, ncut;
  int cx = warp_cut_bin(cnt, kSampleBins, (uint32_t)kExcl, lane, &above, &ncut);
  if (cx < 0) cx = 0;
  double lm[PB];
  double tot = 0.0;
#pragma unroll
  for (int j = 0; j < PB; ++j) {
    lm[j] = (double)mass[lane * PB + j];
    tot += lm[j];
  }
  double incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  const double before = incl - tot;                  // mass of the bins below this lane's
  const double total = __shfl_sync(kFull, incl, 31);
  double upto = 0.0, run = before;
#pragma unroll
  for (int j = 0; j < PB; ++j) {
    run += lm[j];
    if (lane * PB + j == cx) upto = run;             // mass of bins <= cx
  }
  upto = __shfl_sync(kFull, upto, cx / PB);
  const double sc = (double)N / (double)m;
  const double thr = (1.0 - p) * (sc * upto + (total - upto));
  int best = 0;
  run = before;
#pragma unroll
  for (int j = 0; j < PB; ++j) {
    const int c = lane * PB + j;
    if (c <= cx && sc * run * kMassSafety <= thr) best = c;
    run += lm[j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(kFull, best, o));
  uint32_t cc = 0;
#pragma unroll
  for (int j = 0; j < PB; ++j)
    if (lane * PB + j >= best) cc += cnt[lane * PB + j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cc += __shfl_xor_sync(kFull, cc, o);
  const double r = ceil((double)cc + kCountSigmas * sqrt((double)cc) + 8.0);
  if (r >= (double)m) return lo;
  const int c = warp_cut_bin(cnt, kSampleBins, (uint32_t)r, lane, &above, &ncut);
  return lo + (float)(c < 0 ? 0 : c) * ((hi - lo) / (float)kSampleBins);
}

// keep every token: an empty context, k_b >= N_b (top-k) or p >= 1 (top-p)
template <bool TOPP>
__device__ __forceinline__ bool keeps_all(const SelectArgs &a, long long N) {
  if (N == 0) return true;
  if constexpr (TOPP) return a.top_p >= 1.0f;
  else return topk_budget(a, N) >= N;
}

template <int GR, bool TOPP>
__global__ void __launch_bounds__(kT0)
window_kernel(const SelectArgs a, const Shape sh, const Group *__restrict__ groups, int n_groups,
              const StreamWs ws) {
  constexpr int HB = (GR + 3) / 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int item = blockIdx.x;
  const int b = item / n_groups, gi = item % n_groups;
  constexpr int SP = sample_pages(GR);
  __shared__ Group grp;
  __shared__ uint32_t qs[16 * 24];
  __shared__ uint32_t smax[GR], smin[GR];
  __shared__ float hlo[GR], hinv[GR], hhi[GR];
  __shared__ int spage[SP];
  extern __shared__ __align__(16) unsigned char dyn0[];
  float (*sample)[SP * 16] = reinterpret_cast<float (*)[SP * 16]>(dyn0);
  uint32_t (*shist)[kSampleBins] = reinterpret_cast<uint32_t (*)[kSampleBins]>(dyn0 + (size_t)GR * SP * 16 * 4);
  // top-p: softmax mass of the sample per bin, relative to the sample maximum
  float (*smass)[kSampleBins] =
      reinterpret_cast<float (*)[kSampleBins]>(dyn0 + (size_t)GR * SP * 16 * 4 + (size_t)GR * kSampleBins * 4);
  if (tid == 0) grp = groups[gi];
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int nr = grp.n, g = grp.kv_head;
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  const long long kb = TOPP ? 0 : topk_budget(a, N);
  if (tid == 0) {
    ws.fail[item] = 0u;
    if (item == 0) ws.fail[ws.items] = 0u;           // count of flagged items
  }
  if (tid < nr) {
    const long long row = (long long)b * sh.H_ret + grp.row[tid];
    ws.bcount[row] = 0u;
    ws.rowitem[row] = item;
    if constexpr (TOPP) {
      ws.zlo[row] = 0.0;
      ws.rflag[row] = 0u;
    }
  }
  if constexpr (TOPP) {
    for (int o = tid; o < nr * (kBinsP + 1); o += kT0)
      ws.hist[((long long)b * sh.H_ret + grp.row[o / (kBinsP + 1)]) * (kBinsP + 1) + o % (kBinsP + 1)] = 0.0;
  }
  if (keeps_all<TOPP>(a, N)) return;                 // K1 skips, K2 keeps everything

  // q~ in float64 (one warp per head, lanes split d) -> float32 -> hi/mid/lo;
  // the terms of absent heads stay zero
  for (int o = tid; o < 16 * 24; o += kT0) qs[o] = 0u;
  __syncthreads();
  for (int i = warp; i < nr; i += kT0 / 32) {
    double acc[kIndexDim];
#pragma unroll
    for (int j = 0; j < kIndexDim; ++j) acc[j] = 0.0;
    {
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
  for (int o = tid; o < GR * kSampleBins; o += kT0) {
    (&shist[0][0])[o] = 0u;
    if constexpr (TOPP) (&smass[0][0])[o] = 0.0f;
  }
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
    hhi[tid] = hi;
    hinv[tid] = (smax[tid] != 0u && hi > lo) ? (float)kSampleBins / (hi - lo) : 0.0f;
  }
  __syncthreads();
  for (int h = 0; h < nr; ++h) {
    const float lo = hlo[h], iv = hinv[h], hi = hhi[h];
    for (int r = tid; r < ns * 16; r += kT0) {
      const float v = sample[h][r];
      if (v == -INFINITY) continue;
      const int bin = std::min(kSampleBins - 1, std::max(0, __float2int_rz((v - lo) * iv)));
      atomicAdd(&shist[h][bin], 1u);
      if constexpr (TOPP) atomicAdd(&smass[h][bin], exp2f((v - hi) * kLog2e));
    }
  }
  __syncthreads();
  // one warp per head: the highest bin whose suffix count reaches r
  for (int h = warp; h < nr; h += kT0 / 32) {
    // valid sample tokens: every sampled page is full except possibly the last
    const long long m = (long long)(ns - 1) * kPage + std::min<long long>(kPage, N - (long long)(ns - 1) * st * kPage);
    const long long row = (long long)b * sh.H_ret + grp.row[h];
    if constexpr (TOPP) {
      // no valid sample token (bad page ids): nothing is binned, K2 flags the row
      float tlo = INFINITY, thi = 0.0f;
      if (smax[h] != 0u) {
        thi = hhi[h];
        tlo = topp_window_lo(shist[h], smass[h], hlo[h], thi, m, N, (double)a.top_p, lane);
      } else if (lane == 0) {
        ws.rflag[row] = 1u;
      }
      const float inv = thi > tlo ? (float)kBinsP / (thi - tlo) : 0.0f;
      if (lane == 0) ws.win[row] = make_float4(tlo, thi, inv, 0.0f);
      continue;
    }
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
    const float inv = (tlo > -INFINITY && thi > tlo) ? (float)kBinsK / (thi - tlo) : 0.0f;
    if (lane == 0) ws.win[row] = make_float4(tlo, thi, inv, 0.0f);
  }
}

// ------------------------------------------------------------------- K1
constexpr int kT1 = 256;
constexpr int kW1 = kT1 / 32;

// What a K1 launch does with each score.
enum StreamMode { kStageTopk = 0, kMassTopp = 1, kCutTopp = 2 };

// dynamic shared memory of a K1 launch: the rings, then the staging area
// (kStageTopk, kCutTopp), the chunk's bitmap (kCutTopp) or the mass
// histograms (kMassTopp)
__host__ __device__ constexpr size_t stream_stage_bytes(int GR, int MODE) {
  return MODE == kMassTopp ? 0 : (size_t)kW1 * ((GR + 3) / 4) * stage_lane(GR) * 32 * 8;
}
__host__ __device__ constexpr size_t stream_smem_bytes(int GR, int MODE) {
  return (size_t)kW1 * kRing * kPageBytes + stream_stage_bytes(GR, MODE) +
         (MODE == kMassTopp ? (size_t)GR * (kBinsP + 1) * 4 : 0) +
         (MODE == kCutTopp ? (size_t)GR * (kChunkPages / 2) * 4 : 0);
}

template <int GR, int MODE>
__global__ void __launch_bounds__(kT1)
stream_kernel(const SelectArgs a, const Shape sh, const Group *__restrict__ groups, int n_groups,
              const StreamWs ws, int chunk) {
  constexpr int HB = (GR + 3) / 4;
  constexpr int SL = stage_lane(GR);
  constexpr bool TOPP = MODE != kStageTopk;
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
  unsigned char *tail = dyn1 + (size_t)kW1 * kRing * kPageBytes + stream_stage_bytes(GR, MODE);
  // kMassTopp: per-head mass histograms; kCutTopp: per-head bitmap of the chunk
  float (*shm)[kBinsP + 1] = reinterpret_cast<float (*)[kBinsP + 1]>(tail);
  uint32_t (*sbits)[kChunkPages / 2] = reinterpret_cast<uint32_t (*)[kChunkPages / 2]>(tail);
  __shared__ int32_t pt_s[kChunkPages];
  __shared__ uint32_t qs[16 * 24];
  __shared__ int cut_s[GR];
  __shared__ Group grp;
  if (tid == 0) grp = groups[gi];
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int nr = grp.n, g = grp.kv_head;
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  if (keeps_all<TOPP>(a, N)) return;
  const int pages = (int)((N + kPage - 1) / kPage);
  const int p0 = blockIdx.y * chunk;                 // chunk: a multiple of 64 pages, at most kChunkPages
  if (p0 >= pages) return;
  const int np = pages - p0 < chunk ? pages - p0 : chunk;
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
    if constexpr (MODE == kMassTopp)
      for (int o = tid; o < GR * (kBinsP + 1); o += kT1) (&shm[0][0])[o] = 0.0f;
    if constexpr (MODE == kCutTopp) {
      for (int o = tid; o < GR * (kChunkPages / 2); o += kT1) (&sbits[0][0])[o] = 0u;
      // the cut bin of each head, from the mass pass (warp h, head h)
      for (int h = warp; h < GR; h += kW1) {
        int c = kBinsP + 1;                          // absent heads: nothing is above the cut
        if (h < nr) {
          const long long row = (long long)b * sh.H_ret + grp.row[h];
          double above, need;
          c = warp_cut_mass(ws.hist + row * (kBinsP + 1), ws.zlo[row], (double)a.top_p, lane, &above, &need);
          if (c < 0) c = kBinsP + 1;                 // the threshold lies below t_lo: K2 flags the row
        }
        if (lane == 0) cut_s[h] = c;
      }
    }
  }
  __syncthreads();

  // per-warp ring: this warp reads pages warp, warp + 8, ... of the chunk
  const uint32_t ring_base = (uint32_t)__cvta_generic_to_shared(&ring[warp][0][0]);
  const unsigned char *iblk = reinterpret_cast<const unsigned char *>(a.index_cache) + lane * 16;
  const uint32_t st_off = page_off(lane >> 1, lane & 1);
  const int nq = np > warp ? (np - warp + kW1 - 1) / kW1 : 0;
  const uint64_t l2_stream = evict_first_policy();
  auto issue = [&](int q) {
    if (q < nq) {
      const int blk = pt_s[warp + q * kW1];
      cp_async16(ring_base + (q % kRing) * kPageBytes + st_off, iblk + (size_t)(blk >= 0 ? blk : 0) * kPageBytes,
                 blk >= 0 ? 16 : 0, l2_stream);
    }
    cp_async_commit();
  };
#pragma unroll
  for (int q = 0; q < kRing; ++q) issue(q);

  BFrag bf[HB];
  float tlo[HB], thi[HB], inv[HB];
  int cut[HB];
  double zl[HB];                                     // kMassTopp: this lane's mass below t_lo
  long long row_of[HB];
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) {
    bf[hb] = load_bfrag(qs, hb, gq, tq);
    const int h = hb * 4 + tq;
    row_of[hb] = h < nr ? (long long)b * sh.H_ret + grp.row[h] : 0;
    const float4 wv = h < nr ? ws.win[row_of[hb]] : make_float4(INFINITY, 0.0f, 0.0f, 0.0f);
    tlo[hb] = wv.x;                                  // absent heads keep nothing
    thi[hb] = wv.y;
    inv[hb] = wv.z;
    cut[hb] = MODE == kCutTopp && h < GR ? cut_s[h] : 0;
    zl[hb] = 0.0;
  }
  bool wide = false;                                 // kMassTopp: a weight beyond float range
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
          const bool valid = (u ? ok1 : ok0) && pos < n32;
          if constexpr (MODE == kStageTopk) {
            if (valid && s >= tlo[hb]) {
              stage[warp][hb][cnt[hb]][lane] = ((unsigned long long)order_key(s) << 32) | pos;
              ++cnt[hb];
            }
          } else if constexpr (MODE == kMassTopp) {
            const int h = hb * 4 + tq;
            if (valid && h < nr) {
              const float w = exp2f((s - thi[hb]) * kLog2e);
              wide |= s - thi[hb] > kMaxLogit;
              if (s < tlo[hb]) zl[hb] += (double)w;
              else atomicAdd(&shm[h][window_bin<kBinsP>(s, tlo[hb], thi[hb], inv[hb])], w);
            }
          } else {
            if (valid && hb * 4 + tq < nr && s >= tlo[hb]) {
              const int bin = window_bin<kBinsP>(s, tlo[hb], thi[hb], inv[hb]);
              if (bin > cut[hb]) {
                const uint32_t loc = pos - (uint32_t)p0 * kPage;
                atomicOr(&sbits[hb * 4 + tq][loc >> 5], 1u << (pos & 31));
              } else if (bin == cut[hb]) {
                stage[warp][hb][cnt[hb]][lane] = ((unsigned long long)order_key(s) << 32) | pos;
                ++cnt[hb];
              }
            }
          }
        }
      }
      full |= cnt[hb] > (uint32_t)(SL - 4);
    }
    if constexpr (MODE != kMassTopp)
      if (__any_sync(kFull, full)) flush();
  }
  if constexpr (MODE != kMassTopp) flush();
  cp_async_wait<0>();
  if constexpr (MODE == kMassTopp) {
    // the chunk's masses join the heads' histograms; the lanes of a head
    // (same tq) sum their float64 masses below t_lo first
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) {
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) zl[hb] += __shfl_xor_sync(kFull, zl[hb], o);
      if (gq == 0 && hb * 4 + tq < nr && zl[hb] != 0.0) atomicAdd(&ws.zlo[row_of[hb]], zl[hb]);
    }
    // a weight out of float range: the item goes to the exact selector
    if (__any_sync(kFull, wide) && lane == 0) atomicOr(&ws.rflag[(long long)b * sh.H_ret + grp.row[0]], 2u);
    __syncthreads();
    for (int o = tid; o < nr * (kBinsP + 1); o += kT1) {
      const int h = o / (kBinsP + 1), bin = o % (kBinsP + 1);
      const float v = shm[h][bin];
      if (v != 0.0f) atomicAdd(&ws.hist[((long long)b * sh.H_ret + grp.row[h]) * (kBinsP + 1) + bin], (double)v);
    }
  }
  if constexpr (MODE == kCutTopp) {
    // the chunk's words of the heads' bitmaps (512 pages = 256 words; the
    // chunk starts on a word boundary)
    __syncthreads();
    const int nw = (np + 1) / 2;
    for (int o = tid; o < nr * nw; o += kT1) {
      const int h = o / nw, w = o % nw;
      ws.bits[((long long)b * sh.H_ret + grp.row[h]) * ws.bwords + p0 / 2 + w] = sbits[h][w];
    }
  }
}

// ------------------------------------------------------------------- K2
constexpr int kT2 = 256;

// K2 runs per head on a group of kT2 threads: alone in its CTA (the per-head
// resolve kernels) or as one of several groups of a CTA that resolves every
// retrieval head of a KV group and then builds the group's union list for
// attend.  A group's barrier is __syncthreads when it is alone, otherwise the
// named barrier 1 + id over its kT2 threads.
struct HeadGroup {
  int t;                    // thread index in the group
  int id;                   // group index in the CTA
  bool alone;
  __device__ __forceinline__ void sync() const {
    if (alone) __syncthreads();
    else asm volatile("bar.sync %0, %1;\n" ::"r"(1 + id), "n"(kT2) : "memory");
  }
};

// Group-wide: the positions set in bitmap[0, words) go to out in ascending
// order, their number to sel_count[row].  Warp w owns a contiguous run of
// words, 128 per step (four consecutive words per lane, one 16-byte load, no
// bank conflicts); the set bits of a step are handed out 32 at a time, so
// every store instruction writes consecutive positions; a group-wide sum over
// the warps' totals places each warp.  The bitmap is read in whole 16-byte
// words (its allocation is rounded up to them).  wtot: kT2 / 32 words of
// shared memory.
__device__ void write_ascending(const SelectArgs &a, const HeadGroup &hg, const uint32_t *bitmap, int words,
                                int32_t *out, long long row, uint32_t *wtot) {
  constexpr int NW = kT2 / 32;
  constexpr int WPL = 4;                             // words per lane and step
  const int lane = hg.t & 31, warp = hg.t >> 5;
  const int steps = (words + NW * 32 * WPL - 1) / (NW * 32 * WPL);
  const int w0 = warp * steps * 32 * WPL;
  auto load = [&](int x, uint32_t (&v)[WPL]) {       // words x .. x + 3 (x a multiple of 4)
    const uint4 q = x < words ? *reinterpret_cast<const uint4 *>(bitmap + x) : make_uint4(0u, 0u, 0u, 0u);
    v[0] = q.x;
    v[1] = x + 1 < words ? q.y : 0u;
    v[2] = x + 2 < words ? q.z : 0u;
    v[3] = x + 3 < words ? q.w : 0u;
  };
  uint32_t c = 0;
  for (int r = 0; r < steps; ++r) {
    uint32_t v[WPL];
    load(w0 + (r * 32 + lane) * WPL, v);
#pragma unroll
    for (int j = 0; j < WPL; ++j) c += __popc(v[j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
  if (lane == 0) wtot[warp] = c;
  hg.sync();
  long long off = 0, total = 0;
#pragma unroll
  for (int x = 0; x < NW; ++x) {
    const uint32_t t = wtot[x];
    off += x < warp ? t : 0u;
    total += t;
  }
  bool over = false;
  for (int r = 0; r < steps; ++r) {
    const int x0 = w0 + r * 32 * WPL;
    uint32_t v[WPL];
    load(x0 + lane * WPL, v);
    int nl = 0;
#pragma unroll
    for (int j = 0; j < WPL; ++j) nl += __popc(v[j]);
    const int step_bits = __reduce_add_sync(kFull, (unsigned)nl);
    if (step_bits >= kDenseBits) {
      // dense run: each lane writes its own bits (consecutive slots per lane),
      // far fewer instructions than handing bits out 32 at a time
      int incl = nl;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      long long o = off + incl - nl;
#pragma unroll
      for (int j = 0; j < WPL; ++j) {
        uint32_t bits = v[j];
        const int base = (x0 + lane * WPL + j) * 32;
        while (bits) {
          const int bit = __ffs(bits) - 1;
          bits &= bits - 1u;
          if (o < a.sel_stride) out[o] = base + bit;
          else over = true;
          ++o;
        }
      }
      off += step_bits;
    } else {
      off += warp_emit_bits_w<WPL>(v, lane, [&](bool valid, int k, int w, int j, int bit) {
        const long long o = off + k;
        if (valid) {
          if (o < a.sel_stride) out[o] = (x0 + w * WPL + j) * 32 + bit;
          else over = true;
        }
      });
    }
  }
  if (over) raise_error(a.err, SD_EBIT_SEL);
  if (hg.t == 0) {
    if (total > a.sel_stride) raise_error(a.err, SD_EBIT_SEL);
    a.sel_count[row] = (int32_t)std::min<long long>(total, a.sel_stride);
  }
}

// Group-wide: every position 0 .. N - 1 (a head that keeps all its tokens);
// with `bitmap`, also every bit of [0, N) (for the union).
__device__ void write_all(const SelectArgs &a, const HeadGroup &hg, long long N, int32_t *out, long long row,
                          uint32_t *bitmap) {
  for (long long t = hg.t; t < N; t += kT2) {
    if (t < a.sel_stride) out[t] = (int32_t)t;
    else raise_error(a.err, SD_EBIT_SEL);
  }
  if (bitmap)
    for (long long x = hg.t; x < (N + 31) / 32; x += kT2)
      bitmap[x] = (x + 1) * 32 <= N ? 0xFFFFFFFFu : ((1u << (N & 31)) - 1u);
  if (hg.t == 0) a.sel_count[row] = (int32_t)std::min(N, a.sel_stride);
}

// K2 flags the work item of a row whose window missed (once per item).
__device__ void flag_item(const StreamWs &ws, long long row) {
  const int it = ws.rowitem[row];
  if (atomicExch(&ws.fail[it], 1u) == 0u) ws.fail[ws.items + 1 + atomicAdd(&ws.fail[ws.items], 1u)] = (uint32_t)it;
}

// Group-wide: the highest bin c of hist[0, kBinsK) whose suffix count reaches
// need (need >= 1).  Thread t holds bins [8 t, 8 t + 8); a group-wide suffix
// sum over the threads' totals finds the thread holding the cut, which scans
// its own bins.  Writes c, the count strictly above it and hist[c] to res
// (res[0] = -1 when the bins together hold fewer than need).  wsum: kT2 / 32
// words of shared memory.
__device__ void block_cut_bin(const HeadGroup &hg, const uint32_t *hist, long long need, uint32_t *wsum, int *res) {
  constexpr int PT = kBinsK / kT2;
  static_assert(PT == 8, "two 16-byte loads per thread");
  const int tid = hg.t, lane = tid & 31, warp = tid >> 5;
  const uint4 h0 = reinterpret_cast<const uint4 *>(hist)[2 * tid];
  const uint4 h1 = reinterpret_cast<const uint4 *>(hist)[2 * tid + 1];
  const uint32_t v[PT] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  uint32_t tot = 0;
#pragma unroll
  for (int j = 0; j < PT; ++j) tot += v[j];
  uint32_t suf = tot;                                  // sum over this and the higher lanes of the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(kFull, suf, o);
    if (lane + o < 32) suf += y;
  }
  if (lane == 0) wsum[warp] = suf;
  hg.sync();
  long long above = 0;
#pragma unroll
  for (int w = 0; w < kT2 / 32; ++w) above += w > warp ? wsum[w] : 0u;
  long long run = above + (suf - tot);                 // count above this thread's bins
  if (run < need && run + tot >= need) {
#pragma unroll
    for (int j = PT - 1; j >= 0; --j) {
      if (run + v[j] >= need) {
        res[0] = tid * PT + j;
        res[1] = (int)run;
        res[2] = (int)v[j];
        break;
      }
      run += v[j];
    }
  }
}

// Shared memory of one top-k head group (besides its bitmap).
struct TopkSmem {
  unsigned long long cand[kCap];
  __align__(16) uint32_t hist[kBinsK + 4];
  uint32_t n_cand;
  int res[3];
  int fail, done;
  long long need;
  int cutv[kLevels];
  float llo[kLevels], linv[kLevels];
  uint32_t wtot[kT2 / 32];
};

// top-k K2 of one (sequence b, retrieval head row hr).  The head's buffered
// entries (every score >= t_lo) are histogrammed over kBinsK bins of
// [t_lo, t_hi) plus one bin for scores >= t_hi; the bin holding the k-th
// score is split again while it holds more than kRefine tokens (kLevels
// levels at most); entries above the cut path are selected, the cut bin's are
// ranked exactly by (score desc, position asc).  Leaves the set in `bitmap`
// (bits of [0, N)) and writes it out; false when the window missed (the item
// is flagged for the exact selector and nothing is written).  PER: buffer
// entries held in registers per thread.
template <int PER>
__device__ bool resolve_topk(const SelectArgs &a, const Shape &sh, const StreamWs &ws, int b, int hr,
                             const HeadGroup &hg, TopkSmem &S, uint32_t *bitmap, bool union_bits) {
  const int tid = hg.t, lane = tid & 31;
  const long long row = (long long)b * sh.H_ret + hr;
  int32_t *out = a.sel_idx + row * a.sel_stride;
  // one round of independent loads: the length, the window, the buffer count
  // and the first PER * kT2 buffer slots (inside the row: reads stop at cap)
  long long N = a.seq_lens[b];
  const float4 w = ws.win[row];
  const uint32_t nbuf = ws.bcount[row];
  const unsigned long long *buf = ws.buf + row * ws.cap;
  unsigned long long ent[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = tid + j * kT2;
    ent[j] = e < ws.cap ? __ldcg(buf + e) : 0ull;
  }
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  const long long kb = topk_budget(a, N);
  if (N == 0 || kb >= N) {
    write_all(a, hg, N, out, row, union_bits ? bitmap : nullptr);
    return true;
  }
  const int n = (int)std::min<uint32_t>(nbuf, (uint32_t)ws.cap);
  const int words = (int)((N + 31) / 32);
  for (int o = tid; o < (words + 3) / 4; o += kT2) reinterpret_cast<uint4 *>(bitmap)[o] = make_uint4(0u, 0u, 0u, 0u);
  if (tid == 0) {
    S.llo[0] = w.x;
    S.linv[0] = w.z;
    S.need = kb;
    S.fail = nbuf > (uint32_t)ws.cap;
    S.done = 0;
    S.n_cand = 0u;
  }
  // bin of a score at level L: level 0 is the window histogram (bin kBinsK:
  // scores >= t_hi); level L > 0 splits the cut bin of level L - 1 into kBinsK
  // linear sub-bins.  Bins are non-decreasing in the score at every level.
  auto bin_at = [&](float v, int L) -> int {
    if (L == 0) return window_bin<kBinsK>(v, w.x, w.y, w.z);
    return min(kBinsK - 1, max(0, __float2int_rz((v - S.llo[L]) * S.linv[L])));
  };
  // the entries past the registers are read from the buffer (L2) at each pass
  const int rest0 = PER * kT2;
  // the cut bin: refine while it holds more than kRefine tokens
  int L = 0;
  for (; L < kLevels; ++L) {
    for (int o = tid; o <= kBinsK; o += kT2) S.hist[o] = 0u;
    hg.sync();
    if (S.fail) break;
    auto add = [&](unsigned long long en) {
      const float v = key_to_float((uint32_t)(en >> 32));
      bool play = true;
      for (int l = 0; l < L; ++l) play = play && bin_at(v, l) == S.cutv[l];
      if (play) atomicAdd(&S.hist[bin_at(v, L)], 1u);
    };
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (tid + j * kT2 < n) add(ent[j]);
    for (int e0 = rest0 + tid; e0 < n; e0 += kRestBatch * kT2) {
      unsigned long long v[kRestBatch];              // independent loads first
#pragma unroll
      for (int u = 0; u < kRestBatch; ++u) v[u] = e0 + u * kT2 < n ? __ldcg(buf + e0 + u * kT2) : 0ull;
#pragma unroll
      for (int u = 0; u < kRestBatch; ++u)
        if (e0 + u * kT2 < n) add(v[u]);
    }
    if (tid == 0) S.res[0] = -1;
    hg.sync();
    const long long need = S.need - (L == 0 ? (long long)S.hist[kBinsK] : 0LL);
    if (need > 0) block_cut_bin(hg, S.hist, need, S.wtot, S.res);
    hg.sync();
    if (tid == 0) {
      const int cut = S.res[0];
      if (need <= 0 || cut < 0) {
        S.fail = 1;
      } else {
        const uint32_t ncut = (uint32_t)S.res[2];
        S.cutv[L] = cut;
        S.need = need - S.res[1];                      // tokens still to take from the cut bin
        const bool last = ncut <= (uint32_t)kRefine || L + 1 == kLevels;
        if (last && ncut > (uint32_t)kCap) S.fail = 1;
        if (!last) {
          S.llo[L + 1] = S.llo[L] + (float)cut / S.linv[L];
          S.linv[L + 1] = S.linv[L] * (float)kBinsK;
        }
        S.done = last;
      }
    }
    hg.sync();
    if (S.fail || S.done) break;
  }
  if (S.fail) {
    if (tid == 0) flag_item(ws, row);
    return false;
  }
  const int nlev = L + 1;
  // classify: above the cut path -> selected; on it -> candidate.  Every lane
  // of a warp takes part (invalid entries included) so that candidates are
  // appended with one atomic per warp.
  auto classify = [&](unsigned long long en, bool valid) {
    const uint32_t key = (uint32_t)(en >> 32), pos = (uint32_t)en;
    const float v = key_to_float(key);
    int rel = 0;
    for (int l = 0; l < nlev && rel == 0; ++l) {
      const int bl = bin_at(v, l);
      rel = bl > S.cutv[l] ? 1 : (bl < S.cutv[l] ? -1 : 0);
    }
    if (valid && rel > 0) atomicOr(&bitmap[pos >> 5], 1u << (pos & 31));
    const bool isc = valid && rel == 0;
    const unsigned m = __ballot_sync(kFull, isc);
    if (m) {
      const int leader = __ffs(m) - 1;
      uint32_t base = 0;
      if (lane == leader) base = atomicAdd(&S.n_cand, (uint32_t)__popc(m));
      base = __shfl_sync(kFull, base, leader);
      const uint32_t at = base + __popc(m & ((1u << lane) - 1u));
      if (isc && at < (uint32_t)kCap) S.cand[at] = ((unsigned long long)(~key) << 32) | pos;   // ascending = better first
    }
  };
#pragma unroll
  for (int j = 0; j < PER; ++j) classify(ent[j], tid + j * kT2 < n);
  for (int e0 = rest0; e0 < n; e0 += kRestBatch * kT2) {
    unsigned long long v[kRestBatch];
#pragma unroll
    for (int u = 0; u < kRestBatch; ++u) {
      const int e = e0 + u * kT2 + tid;
      v[u] = e < n ? __ldcg(buf + e) : 0ull;
    }
#pragma unroll
    for (int u = 0; u < kRestBatch; ++u) classify(v[u], e0 + u * kT2 + tid < n);
  }
  hg.sync();
  // rank the cut bin exactly: the need_c best by (score desc, position asc)
  const int nc = (int)std::min<uint32_t>(S.n_cand, (uint32_t)kCap);
  const long long need_c = S.need;
  for (int e = tid; e < nc; e += kT2) {
    const unsigned long long me = S.cand[e];
    int rk = 0;
    for (int j = 0; j < nc; ++j) rk += S.cand[j] < me;
    if (rk < need_c) {
      const uint32_t pos = (uint32_t)me;
      atomicOr(&bitmap[pos >> 5], 1u << (pos & 31));
    }
  }
  hg.sync();
  write_ascending(a, hg, bitmap, words, out, row, S.wtot);
  return true;
}

// One warp, over kBins radix digits with counts and float64 masses: the
// highest non-empty digit whose mass plus the mass above it reaches need
// (need <= 0: the highest non-empty digit).  When rounding leaves every digit
// short, the lowest non-empty digit (all of the level is kept).  *above = the
// mass of the digits above the one returned.
__device__ int warp_cut_digit(const uint32_t *cnt, const double *mass, double need, int lane, double *above) {
  constexpr int G = kBins / 32;
  double tot = 0.0;
  uint32_t nz = 0u;
  for (int j = 0; j < G; ++j) {
    tot += mass[lane * G + j];
    nz += cnt[lane * G + j];
  }
  double suf = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_down_sync(kFull, suf, o);
    if (lane + o < 32) suf += y;
  }
  const unsigned bal = __ballot_sync(kFull, nz > 0u && suf >= need);
  const unsigned any = __ballot_sync(kFull, nz > 0u);
  const int grp = bal ? 31 - __clz(bal) : (any ? __ffs(any) - 1 : 0);
  const double acc = __shfl_sync(kFull, suf - tot, grp);
  const uint32_t c = lane < G ? cnt[grp * G + lane] : 0u;
  const double m = lane < G ? mass[grp * G + lane] : 0.0;
  double s2 = m;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_down_sync(kFull, s2, o);
    if (lane + o < 32) s2 += y;
  }
  const unsigned bal2 = __ballot_sync(kFull, lane < G && c > 0u && acc + s2 >= need);
  const unsigned any2 = __ballot_sync(kFull, lane < G && c > 0u);
  const int j = bal2 ? 31 - __clz(bal2) : (any2 ? __ffs(any2) - 1 : 0);
  *above = acc + __shfl_sync(kFull, s2, j) - __shfl_sync(kFull, m, j);
  return grp * G + j;
}

// Shared memory of one top-p head group (besides its bitmap).
struct ToppSmem {
  unsigned long long cand[kCapP];
  uint32_t dcnt[kBins];
  double dmass[kBins];
  int fail;
  double need;
  uint32_t kmin, kmax, prefix;
  uint32_t wtot[kT2 / 32];
};

// top-p K2 of one (sequence b, retrieval head row hr): the tokens above the
// cut bin (the cut pass's bitmap) plus the cut bin's candidates at or above
// the exact threshold, found by a radix search over their order keys with
// float64 mass per digit.  As resolve_topk for the bitmap, the output and a
// miss.
__device__ bool resolve_topp(const SelectArgs &a, const Shape &sh, const StreamWs &ws, int b, int hr,
                             const HeadGroup &hg, ToppSmem &S, uint32_t *bitmap, bool union_bits) {
  const int tid = hg.t, lane = tid & 31, warp = tid >> 5;
  const long long row = (long long)b * sh.H_ret + hr;
  int32_t *out = a.sel_idx + row * a.sel_stride;
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  if (keeps_all<true>(a, N)) {
    write_all(a, hg, N, out, row, union_bits ? bitmap : nullptr);
    return true;
  }
  const float thi = ws.win[row].y;
  if (warp == 0) {
    double above, need;
    const int c = warp_cut_mass(ws.hist + row * (kBinsP + 1), ws.zlo[row], (double)a.top_p, lane, &above, &need);
    if (lane == 0) {
      S.fail = c < 0 || ws.rflag[row] != 0u || ws.bcount[row] > (uint32_t)ws.cap;
      S.need = need - above;                           // mass still to take from the cut bin
      S.kmin = 0xFFFFFFFFu;
      S.kmax = 0u;
      S.prefix = 0u;
    }
  }
  hg.sync();
  if (S.fail) {
    if (tid == 0) flag_item(ws, row);
    return false;
  }
  // the bitmap of the tokens above the cut bin, and the cut bin's candidates
  const int words = (int)((N + 31) / 32);
  const uint32_t *bits = ws.bits + row * ws.bwords;
  for (int o = tid; o < words; o += kT2) bitmap[o] = bits[o];
  const int n = (int)ws.bcount[row];
  const unsigned long long *buf = ws.buf + row * ws.cap;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int e = tid; e < n; e += kT2) {
    const unsigned long long v = buf[e];
    S.cand[e] = v;
    lo = min(lo, (uint32_t)(v >> 32));
    hi = max(hi, (uint32_t)(v >> 32));
  }
  if (lo != 0xFFFFFFFFu) {
    atomicMin(&S.kmin, lo);
    atomicMax(&S.kmax, hi);
  }
  hg.sync();
  if (n > 0) {
    // exact radix search over the order keys' offsets from the smallest:
    // the largest key whose suffix mass reaches need (9 bits per level)
    const uint32_t kmin = S.kmin, span = S.kmax - kmin;
    int rem = span ? 32 - __clz(span) : 0;           // offset bits not yet decided
    const int top = rem;
    uint32_t prefix = 0u;
    double need = S.need;
    while (rem > 0) {
      const int sh2 = rem > 9 ? rem - 9 : 0;
      for (int o = tid; o < kBins; o += kT2) {
        S.dcnt[o] = 0u;
        S.dmass[o] = 0.0;
      }
      hg.sync();
      // lanes of a warp holding the same digit add their count and mass
      // first, and one of them updates the shared bins (the candidates of a
      // cut bin crowd into a few digits at the first levels)
      for (int e0 = 0; e0 < n; e0 += kT2) {
        const int e = e0 + tid;
        bool part = false;
        uint32_t d = 0u;
        double wt = 0.0;
        if (e < n) {
          const uint32_t key = (uint32_t)(S.cand[e] >> 32), off = key - kmin;
          part = rem == top || (off >> rem) == prefix;
          if (part) {
            d = (off >> sh2) & ((1u << (rem - sh2)) - 1u);
            wt = (double)exp2f((key_to_float(key) - thi) * kLog2e);
          }
        }
        const unsigned pm = __ballot_sync(kFull, part);
        if (part) {
          const unsigned peers = __match_any_sync(pm, d);
          double sum = 0.0;
          for (unsigned m = peers; m; m &= m - 1u) sum += __shfl_sync(peers, wt, __ffs(m) - 1);
          if (lane == __ffs(peers) - 1) {
            atomicAdd(&S.dcnt[d], (uint32_t)__popc(peers));
            atomicAdd(&S.dmass[d], sum);
          }
        }
      }
      hg.sync();
      if (warp == 0) {
        double above;
        const int d = warp_cut_digit(S.dcnt, S.dmass, need, lane, &above);
        if (lane == 0) {
          S.need = need - above;
          S.prefix = (prefix << (rem - sh2)) | (uint32_t)d;
        }
      }
      hg.sync();
      need = S.need;
      prefix = S.prefix;
      rem = sh2;
    }
    const uint32_t tau = kmin + prefix;              // the threshold's key: every candidate >= it is kept
    for (int e = tid; e < n; e += kT2) {
      const unsigned long long v = S.cand[e];
      if ((uint32_t)(v >> 32) >= tau) {
        const uint32_t pos = (uint32_t)v;
        atomicOr(&bitmap[pos >> 5], 1u << (pos & 31));
      }
    }
  }
  hg.sync();
  write_ascending(a, hg, bitmap, words, out, row, S.wtot);
  return true;
}

// Per-head K2: one CTA per (sequence, retrieval head).  dynamic shared
// memory: the head's bitmap of the context [max_len / 32 words, rounded up to
// 16 bytes].
__global__ void __launch_bounds__(kT2, 4)
topk_resolve_kernel(const SelectArgs a, const Shape sh, const StreamWs ws) {
  extern __shared__ __align__(16) uint32_t bitmap[];
  __shared__ TopkSmem S;
  pdl_wait();
  pdl_trigger();
  const HeadGroup hg{(int)threadIdx.x, 0, true};
  resolve_topk<per_thread_entries(kT2, 4)>(a, sh, ws, blockIdx.y, blockIdx.x, hg, S, bitmap, false);
}

__global__ void __launch_bounds__(kT2, 4)
topp_resolve_kernel(const SelectArgs a, const Shape sh, const StreamWs ws) {
  extern __shared__ __align__(16) uint32_t bitmap[];
  __shared__ ToppSmem S;
  pdl_wait();
  pdl_trigger();
  const HeadGroup hg{(int)threadIdx.x, 0, true};
  resolve_topp(a, sh, ws, blockIdx.y, blockIdx.x, hg, S, bitmap, false);
}

// K2 of the decode step with the union: one CTA per (sequence, retrieval KV
// group), one group of kT2 threads per retrieval head of the group (NG >= the
// group's heads).  Each group resolves its head into a bitmap of the context
// and writes the head's list; then the whole CTA walks the heads' bitmaps over
// the spans of attend's plan (the item's spans side by side, a share of the
// warps each) and writes each span's union list there: (cache row, head mask)
// in ascending position order, and its length.
// An item with a missed window is left to the exact selector and to attend's
// plan.  dynamic shared memory: [NG bitmaps of bm_bytes][NG head smem].
template <bool TOPP, int NG>
__global__ void __launch_bounds__(NG * kT2, 1)
resolve_union_kernel(const SelectArgs a, const Shape sh, const StreamWs ws, const Group *__restrict__ groups,
                     int n_groups, const UnionOut uo, int bm_bytes) {
  using Smem = typename std::conditional<TOPP, ToppSmem, TopkSmem>::type;
  constexpr int NWC = NG * kT2 / 32;                 // warps of the CTA
  extern __shared__ __align__(16) unsigned char dynu[];
  __shared__ Group grp;
  __shared__ int any_fail;
  __shared__ uint32_t ctot[NWC];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int item = blockIdx.x;
  const int b = item / n_groups, gi = item % n_groups;
  if (tid == 0) {
    grp = groups[gi];
    any_fail = 0;
  }
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int nr = grp.n, g = grp.kv_head;
  const int k = tid / kT2;
  const HeadGroup hg{tid % kT2, k, false};
  auto bitmap_of = [&](int i) { return reinterpret_cast<uint32_t *>(dynu + (size_t)i * bm_bytes); };
  Smem &S = *reinterpret_cast<Smem *>(dynu + (size_t)NG * bm_bytes + (size_t)k * sizeof(Smem));
  if (k < nr) {
    const bool ok = TOPP ? resolve_topp(a, sh, ws, b, grp.row[k], hg, reinterpret_cast<ToppSmem &>(S), bitmap_of(k), true)
                         : resolve_topk<per_thread_entries(NG * kT2, 1)>(a, sh, ws, b, grp.row[k], hg,
                                                                      reinterpret_cast<TopkSmem &>(S), bitmap_of(k), true);
    if (!ok && hg.t == 0) any_fail = 1;
  }
  __syncthreads();
  if (any_fail) return;                              // planned by attend after the exact selector

  // ---- the group's union list: the item's spans side by side ---------------------
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  const int words = (int)((N + 31) / 32);
  const int span_words = uo.span / 32;
  const int ns_item = (int)((N + uo.span - 1) / uo.span);
  // row of (page, head, slot) = (page * heads + head) * 16 + slot, over all KV
  // heads or over the retrieval groups only
  const uint32_t row_g = (uint32_t)(uo.ret_only ? gi : g) * kPage;
  const uint32_t row_page = (uint32_t)(uo.ret_only ? n_groups : sh.Hkv) * kPage;
  const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
  bool bad_page = false;
  // P spans at a time, WPS warps on each: warp `sub` of a span takes its words
  // [sub * steps * 32, (sub + 1) * steps * 32) in steps of 32 (one per lane)
  constexpr int kPre = 4;                            // steps whose page ids are loaded up front
  const int P = ns_item < NWC ? ns_item : NWC;
  const int WPS = P > 0 ? NWC / P : NWC;
  const int sub = warp % WPS, first = warp - sub;
  for (int sp0 = 0; sp0 < ns_item; sp0 += P) {
    const int sp = sp0 + warp / WPS;
    const bool act = warp / WPS < P && sp < ns_item;
    const int x_lo = act ? sp * span_words : 0;
    const int x_hi = act ? std::min(words, x_lo + span_words) : 0;
    const int steps = (x_hi - x_lo + WPS * 32 - 1) / (WPS * 32);
    const int w0 = x_lo + sub * steps * 32;
    // the two pages of each word of the first steps, in flight during the
    // count (pages at or past the sequence's end are never read)
    auto pages_of = [&](int x, int &p0, int &p1) {
      const long long q0 = (long long)x * 32;
      p0 = (x < x_hi && q0 < N) ? pt[q0 >> 4] : -1;
      p1 = (x < x_hi && q0 + 16 < N) ? pt[(q0 >> 4) + 1] : -1;
    };
    int pre0[kPre], pre1[kPre];
#pragma unroll
    for (int r = 0; r < kPre; ++r) {
      pre0[r] = pre1[r] = -1;
      if (r < steps) pages_of(w0 + r * 32 + lane, pre0[r], pre1[r]);
    }
    uint32_t c = 0;
    for (int r = 0; r < steps; ++r) {
      const int x = w0 + r * 32 + lane;
      uint32_t u = 0;
#pragma unroll
      for (int i = 0; i < NG; ++i) u |= (x < x_hi && i < nr) ? bitmap_of(i)[x] : 0u;
      c += __popc(u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(kFull, c, o);
    if (lane == 0) ctot[warp] = c;
    __syncthreads();
    uint32_t off = 0, total = 0;
    for (int x = first; x < first + WPS; ++x) {
      off += x < warp ? ctot[x] : 0u;
      total += ctot[x];
    }
    const long long slot = ((long long)b * n_groups + gi) * uo.ns + (act ? sp : 0);   // attend's plan slot
    uint32_t *rows = uo.row + slot * uo.span;
    uint16_t *masks = uo.mask + slot * uo.span;
    auto step = [&](int r, int pg0, int pg1) {       // warp-wide: words w0 + 32 r + lane
      const int xb = w0 + r * 32;
      const int x = xb + lane;
      uint32_t hw[NG];
      uint32_t u = 0;
#pragma unroll
      for (int i = 0; i < NG; ++i) {
        hw[i] = (x < x_hi && i < nr) ? bitmap_of(i)[x] : 0u;
        u |= hw[i];
      }
      off += (uint32_t)warp_emit_bits(u, lane, [&](bool valid, int kk, int w, int bit) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < NG; ++i) m |= ((__shfl_sync(kFull, hw[i], w) >> bit) & 1u) << i;   // every lane
        const int pa = __shfl_sync(kFull, pg0, w), pb = __shfl_sync(kFull, pg1, w);
        if (!valid) return;
        const int pos = (xb + w) * 32 + bit;
        const int page = bit < 16 ? pa : pb;
        const bool ok = page >= 0 && page < sh.num_pages;
        bad_page |= !ok;
        rows[off + kk] = ok ? (uint32_t)page * row_page + row_g + (uint32_t)(pos & (kPage - 1)) : 0u;
        masks[off + kk] = (uint16_t)(ok ? m : 0u);
      });
    };
#pragma unroll
    for (int r = 0; r < kPre; ++r)
      if (r < steps) step(r, pre0[r], pre1[r]);
    for (int r = kPre; r < steps; ++r) {
      int p0, p1;
      pages_of(w0 + r * 32 + lane, p0, p1);
      step(r, p0, p1);
    }
    if (act && sub == 0 && lane == 0) uo.cnt[slot] = (int)total;
    __syncthreads();                                 // ctot is reused by the next spans
  }
  if (bad_page) raise_error(a.err, SD_EBIT_PAGE);
}

// ------------------------------------------------------------------- host
struct StreamPlan {
  int cap;
  size_t bitmap_bytes;
  long long bwords;                   // top-p bitmap words per row
  bool ok;
};

StreamPlan stream_plan(const Shape &sh, const Tables &tb, int mode) {
  StreamPlan p{};
  p.cap = mode == SD_TOP_P ? kCapP
                           : (int)std::min<long long>(sh.max_len, std::max<long long>(4096, sh.max_len / 8));
  p.bitmap_bytes = (size_t)((sh.max_len + 127) / 128) * 16;      // whole 16-byte words
  p.bwords = mode == SD_TOP_P ? ((long long)sh.max_pages + 1) / 2 : 0;
  p.ok = tb.max_ret <= 16 && p.bitmap_bytes <= 160 * 1024 && sh.max_len < (1LL << 31);
  return p;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct StreamLayout {
  size_t qsplit, win, bcount, rowitem, buf, hist, zlo, rflag, bits, total;
};

StreamLayout stream_layout(const Shape &sh, int batch, const StreamPlan &p) {
  StreamLayout L{};
  const size_t rows = (size_t)batch * std::max(1, sh.H_ret);
  size_t o = 0;
  L.qsplit = o;  o = align256(o + rows * 24 * 4);
  L.win = o;     o = align256(o + rows * 16);
  L.bcount = o;  o = align256(o + rows * 4);
  L.rowitem = o; o = align256(o + rows * 4);
  L.buf = o;     o = align256(o + rows * (size_t)p.cap * 8);
  if (p.bwords) {
    L.hist = o;  o = align256(o + rows * (kBinsP + 1) * 8);
    L.zlo = o;   o = align256(o + rows * 8);
    L.rflag = o; o = align256(o + rows * 4);
    L.bits = o;  o = align256(o + rows * (size_t)p.bwords * 4);
  }
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

// The last pass: the per-head resolve, or, with `uo`, at most four retrieval
// heads per group whose bitmaps and scratch fit in one CTA, and enough items
// to fill half the multiprocessors, the resolve with the group's union list
// (*unioned).
// SMs of the current device (looked up once; 1 if the query fails)
int sm_count() {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
      sms = n;
  }
  return std::max(sms, 1);
}

template <bool TOPP, int GR>
cudaError_t launch_resolve(const SelectArgs &a, const Shape &sh, const Tables &tb, const StreamWs &ws,
                           size_t bitmap_bytes, const UnionOut *uo, bool *unioned, cudaStream_t st) {
  using Smem = typename std::conditional<TOPP, ToppSmem, TopkSmem>::type;
  auto *per_head = TOPP ? topp_resolve_kernel : topk_resolve_kernel;
  constexpr int NG = GR <= 4 ? GR : 4;
  const size_t ubytes = (size_t)NG * (bitmap_bytes + sizeof(Smem));
  if (unioned) *unioned = false;
  // one CTA per item: worth it when the items fill at least half the GPU
  // (fewer, and the per-head CTAs' parallelism wins)
  if (uo && GR <= 4 && ubytes <= 227 * 1024 && 2 * a.batch * tb.n_ret >= sm_count()) {
    auto *kern = resolve_union_kernel<TOPP, NG>;
    cudaError_t e = set_smem_once(kern, ubytes);
    if (e != cudaSuccess) return e;
    e = launch_pdl(kern, dim3(a.batch * tb.n_ret), dim3(NG * kT2), ubytes, st, 0, a, sh, ws, tb.ret, tb.n_ret, *uo,
                   (int)bitmap_bytes);
    if (e == cudaSuccess && unioned) *unioned = true;
    return e;
  }
  cudaError_t e = set_smem_once(per_head, bitmap_bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(per_head, dim3(sh.H_ret, a.batch), dim3(kT2), bitmap_bytes, st, 0, a, sh, ws);
}

template <int GR>
cudaError_t stream_launch(const SelectArgs &a, const Shape &sh, const Tables &tb, const StreamWs &ws,
                          size_t bitmap_bytes, const UnionOut *uo, bool *unioned, cudaStream_t st) {
  const bool topp = a.mode == SD_TOP_P;
  const int items = a.batch * tb.n_ret;
  // pages per K1 CTA: 512, or fewer (a multiple of 64) when items x chunks
  // would leave SMs idle, so that small batches still spread over the GPU
  int chunk = kChunkPages;
  while (chunk > 64 && (long long)items * ((sh.max_pages + chunk - 1) / chunk) < 2LL * sm_count()) chunk /= 2;
  const int chunks = (int)((sh.max_pages + chunk - 1) / chunk);
  const dim3 g1(items, chunks);
  const size_t smem0 = (size_t)GR * sample_pages(GR) * 16 * 4 + (size_t)GR * kSampleBins * 4 * (topp ? 2 : 1);
  cudaError_t e;
  if (!topp) {
    const size_t smem1 = stream_smem_bytes(GR, kStageTopk);
    e = set_smem_once(window_kernel<GR, false>, smem0);
    if (e == cudaSuccess) e = set_smem_once(stream_kernel<GR, kStageTopk>, smem1);
    if (e != cudaSuccess) return e;
    e = launch_pdl(window_kernel<GR, false>, dim3(items), dim3(kT0), smem0, st, 0, a, sh, tb.ret, tb.n_ret, ws);
    if (e == cudaSuccess)
      e = launch_pdl(stream_kernel<GR, kStageTopk>, g1, dim3(kT1), smem1, st, 0, a, sh, tb.ret, tb.n_ret, ws, chunk);
    if (e == cudaSuccess) e = launch_resolve<false, GR>(a, sh, tb, ws, bitmap_bytes, uo, unioned, st);
    return e;
  }
  const size_t smem_m = stream_smem_bytes(GR, kMassTopp), smem_c = stream_smem_bytes(GR, kCutTopp);
  e = set_smem_once(window_kernel<GR, true>, smem0);
  if (e == cudaSuccess) e = set_smem_once(stream_kernel<GR, kMassTopp>, smem_m);
  if (e == cudaSuccess) e = set_smem_once(stream_kernel<GR, kCutTopp>, smem_c);
  if (e != cudaSuccess) return e;
  e = launch_pdl(window_kernel<GR, true>, dim3(items), dim3(kT0), smem0, st, 0, a, sh, tb.ret, tb.n_ret, ws);
  if (e == cudaSuccess)
    e = launch_pdl(stream_kernel<GR, kMassTopp>, g1, dim3(kT1), smem_m, st, 0, a, sh, tb.ret, tb.n_ret, ws, chunk);
  if (e == cudaSuccess)
    e = launch_pdl(stream_kernel<GR, kCutTopp>, g1, dim3(kT1), smem_c, st, 0, a, sh, tb.ret, tb.n_ret, ws, chunk);
  if (e == cudaSuccess) e = launch_resolve<true, GR>(a, sh, tb, ws, bitmap_bytes, uo, unioned, st);
  return e;
}

}  // namespace

size_t stream_workspace_bytes(const Shape &sh, const Tables &tb, int batch, int mode) {
  const StreamPlan p = stream_plan(sh, tb, mode);
  if (!p.ok) return 0;
  return stream_layout(sh, batch, p).total;
}

cudaError_t launch_select_stream(const SelectArgs &a, const Shape &sh, const Tables &tb, uint32_t *fail,
                                 void *ws_base, cudaStream_t st, bool *used, const UnionOut *uo, bool *unioned) {
  *used = false;
  if (unioned) *unioned = false;
  const StreamPlan p = stream_plan(sh, tb, a.mode);
  if (!p.ok || ws_base == nullptr) return cudaSuccess;
  const StreamLayout L = stream_layout(sh, a.batch, p);
  char *base = static_cast<char *>(ws_base);
  StreamWs ws{};
  ws.qsplit = reinterpret_cast<uint32_t *>(base + L.qsplit);
  ws.win = reinterpret_cast<float4 *>(base + L.win);
  ws.bcount = reinterpret_cast<uint32_t *>(base + L.bcount);
  ws.rowitem = reinterpret_cast<int *>(base + L.rowitem);
  ws.buf = reinterpret_cast<unsigned long long *>(base + L.buf);
  if (p.bwords) {
    ws.hist = reinterpret_cast<double *>(base + L.hist);
    ws.zlo = reinterpret_cast<double *>(base + L.zlo);
    ws.rflag = reinterpret_cast<uint32_t *>(base + L.rflag);
    ws.bits = reinterpret_cast<uint32_t *>(base + L.bits);
  }
  ws.bwords = p.bwords;
  ws.fail = fail;
  ws.items = a.batch * tb.n_ret;
  ws.cap = p.cap;
  int gr = 1;
  while (gr < tb.max_ret) gr <<= 1;
  cudaError_t e;
  switch (gr) {
    case 1: e = stream_launch<1>(a, sh, tb, ws, p.bitmap_bytes, uo, unioned, st); break;
    case 2: e = stream_launch<2>(a, sh, tb, ws, p.bitmap_bytes, uo, unioned, st); break;
    case 4: e = stream_launch<4>(a, sh, tb, ws, p.bitmap_bytes, uo, unioned, st); break;
    case 8: e = stream_launch<8>(a, sh, tb, ws, p.bitmap_bytes, uo, unioned, st); break;
    default: e = stream_launch<16>(a, sh, tb, ws, p.bitmap_bytes, uo, unioned, st); break;
  }
  if (e == cudaSuccess) *used = true;
  return e;
}

}  // namespace sd
