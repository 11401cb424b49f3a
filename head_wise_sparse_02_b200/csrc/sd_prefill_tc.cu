// Head-wise prefill on the 5th-generation tensor cores (tcgen05, accumulators
// in tensor memory), d = 128.  Same operation as sd_prefill.cu: the query at
// position i of a retrieval head attends to keys 0 .. i, of a local head to
// the sinks and the window ending at i (RTPurbo page, Methodology 1; AoH page,
// Methodology 4).
//
// One CTA (8 warps) per (128 consecutive query positions of one sequence, one
// query head).  Two threads own query row r (warps w and w + 4 read the same
// TMEM lane quarter), each one half of the row's columns of S and O; they
// trade their partial row maximum and sum through shared memory at the
// barriers the tile already has.  Per key tile of
// 64 positions:
//   S[128 x 64]  = Q[128 x 128] K^T     one tcgen05.mma per 16 dims (A = Q, B = K,
//                                       both K-major in shared memory), into TMEM
//   P            = 2^(S log2e scale - m) (masked), split P = P_hi + P_lo in bf16,
//                  stored by each thread into its TMEM lane
//   O[128 x 128] += P_hi V + P_lo V      (A = P from TMEM, B = V MN-major in
//                                       shared memory), into TMEM
// One elected thread issues the MMAs; tcgen05.commit arrives on an mbarrier
// that the CTA waits on (bounded: a wait that runs out sets SD_EBIT_TIMEOUT).
// The running maximum of a row is only moved when a tile raises it by more than
// 8 (log2 units); O is then rescaled in tensor memory (ld, scale, st), so most
// tiles skip that round trip and P stays below 2^8.  K and V tiles are double
// buffered: K(i + 2) is fetched as soon as S(i) has read K(i), V(i + 1) as soon
// as P V(i - 1) has read V(i - 1).  Two CTAs share an SM (96 KB of shared
// memory, 256 TMEM columns each), so one's softmax overlaps the other's MMAs.
//
// Shared-memory operand layouts are the canonical no-swizzle ones: 8 rows x
// 16 bytes per core matrix (128 contiguous bytes); for a K-major operand the
// two core matrices of one 16-element K step are LBO = 128 bytes apart and
// consecutive 8-row groups SBO apart; for the MN-major V the 8-key groups are
// LBO = 128 bytes apart and consecutive 8-dim chunks SBO apart.  In TMEM, A
// (= P) has one row per lane and two 16-bit K elements per 32-bit column.
#include <algorithm>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 256;                // 8 warps: two per TMEM lane quarter
constexpr int kD = 128;                 // head dimension
constexpr int kM = 128;                 // query rows per CTA
constexpr int kN = 64;                  // keys per tile
constexpr float kRescale = 8.0f;        // log2 growth of a row maximum that triggers a rescale of O
constexpr long long kWaitSpins = 1LL << 26;

// shared memory (bytes)
constexpr int kQBytes = kM * kD * 2;    // 32 KB, K-major, SBO 2048
constexpr int kKBytes = kN * kD * 2;    // 16 KB, K-major, SBO 2048
constexpr int kVBytes = kN * kD * 2;    // 16 KB, MN-major, SBO 1024
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;          // two buffers
constexpr int kOffV = kOffK + 2 * kKBytes;      // two buffers
constexpr int kSmem = kOffV + 2 * kVBytes;      // 96 KB: two CTAs per SM
constexpr int kTmemCols = 256;                  // O: columns 0..127, S: 128..191, P hi: 192..223, P lo: 224..255

// tcgen05 instruction descriptor, kind::f16: bf16 A and B, float32 D, M = 128
__host__ __device__ constexpr uint32_t idesc(int n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(kM >> 4) << 24);
}
// shared-memory matrix descriptor, no swizzle, sm_100 version field
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
__device__ __forceinline__ void umma(uint32_t tmem, uint64_t da, uint64_t db, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem),
      "l"(da), "l"(db), "r"(id), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
// the same with A read from tensor memory (lane = row, two 16-bit K elements per column)
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(id), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void cp_async_wait2() { asm volatile("cp.async.wait_group 2;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_st32u(uint32_t addr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16u(uint32_t addr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}
// wait for completion `phase` (0, 1, 0, ...) of an mbarrier; false after kWaitSpins polls
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t phase) {
  for (long long it = 0; it < kWaitSpins; ++it) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
                 "selp.b32 %0, 1, 0, P1;\n\t}\n"
                 : "=r"(done)
                 : "r"(mbar), "r"(phase)
                 : "memory");
    if (done) return true;
  }
  return false;
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ float fast_exp2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16(float x, float y) {     // x in the low half, round to nearest even
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(y), "f"(x));
  return r;
}

// 32 consecutive float32 columns of this warp's 32 TMEM lanes (lane = row)
__device__ __forceinline__ void tmem_ld32(uint32_t addr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
}
__device__ __forceinline__ void tmem_st32(uint32_t addr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

struct TcArgs {
  const uint16_t *q;              // [total_q, Hq, 128]
  const uint16_t *k_cache, *v_cache;
  const int32_t *page_table, *seq_lens, *q_starts;
  float *out;                     // [total_q, Hq, 128]
  float attn_scale;
  int window, num_sinks, batch, total_q;
  unsigned *err;
};

// Key tiles (64 positions) of a CTA, ascending, without repeats: retrieval rows
// read [0, p_last]; local rows the sinks [0, min(S, p_last + 1)) and the window
// [max(0, p0 - W + 1), p_last].
struct Tiles {
  int a0, a1, b0, b1;
  __device__ int count() const { return (a1 - a0) + (b1 - b0); }
  __device__ int at(int i) const { return i < a1 - a0 ? a0 + i : b0 + (i - (a1 - a0)); }
};

__device__ Tiles tiles_for(bool ret, long long p0, long long p_last, int S, int W) {
  Tiles t{0, 0, 0, 0};
  if (ret) {
    t.a1 = (int)(p_last / kN) + 1;
    return t;
  }
  const long long s_end = std::min<long long>(S, p_last + 1);
  if (s_end > 0) t.a1 = (int)((s_end - 1) / kN) + 1;
  if (W > 0) {
    int lo = (int)(std::max<long long>(0, p0 - W + 1) / kN);
    const int hi = (int)(p_last / kN) + 1;
    lo = std::max(lo, t.a1);
    if (lo < hi) {
      if (lo == t.a1) t.a1 = hi;
      else {
        t.b0 = lo;
        t.b1 = hi;
      }
    }
  }
  return t;
}

__global__ void __launch_bounds__(kThreads, 2)
prefill_tc_kernel(const TcArgs a, const Shape sh, const Tables tb) {
  extern __shared__ __align__(1024) unsigned char sm[];
  __shared__ __align__(8) uint64_t mbar[2];          // 0: S ready, 1: P V done
  __shared__ uint32_t tslot;
  __shared__ int s_b, s_t, s_bad;
  __shared__ int s_pg[128 * (kN / kPage)];
  __shared__ float s_max[2][kM], s_sum[2][kM];         // per row: the two column halves' partial max / sum
  __shared__ Group s_grp;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gr = blockIdx.y, hidx = blockIdx.z;
  const bool ret = gr < tb.n_ret;
  pdl_wait();
  pdl_trigger();

  // ---- which (sequence, 128-row query tile): handed out last first
  if (warp == 0) {
    const int want = (int)gridDim.x - 1 - (int)blockIdx.x;
    int base = 0, found_b = -1, found_t = 0;
    for (int c = 0; c < a.batch && found_b < 0; c += 32) {
      const int b = c + lane;
      int nt = 0;
      if (b < a.batch) {
        const int t = a.q_starts[b + 1] - a.q_starts[b];
        nt = t > 0 ? (t + kM - 1) / kM : 0;
      }
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned hit = __ballot_sync(kFull, b < a.batch && want < base + incl && want >= base + incl - nt);
      if (hit) {
        const int src = __ffs(hit) - 1;
        const int ex = __shfl_sync(kFull, incl - nt, src);
        found_b = c + src;
        found_t = want - base - ex;
      }
      base += __shfl_sync(kFull, incl, 31);
    }
    if (lane == 0) {
      s_b = found_b;
      s_t = found_t;
      s_bad = 0;
      s_grp = ret ? tb.ret[gr] : tb.loc[gr - tb.n_ret];
    }
  }
  __syncthreads();
  const int b = s_b;
  if (b < 0 || hidx >= s_grp.n) return;              // past the last tile, or past the group's heads
  const int qs = a.q_starts[b];
  const int T = a.q_starts[b + 1] - qs;
  const long long N = a.seq_lens[b];
  if (N < 0 || N > sh.max_len || T > N || qs < 0 || qs + T > a.total_q) {
    if (tid == 0) raise_error(a.err, SD_EBIT_SEQLEN);
    return;
  }
  const int qh = s_grp.q_head[hidx], g = s_grp.kv_head;
  const int row0 = s_t * kM;
  const int nrows = T - row0 < kM ? T - row0 : kM;
  const long long p0 = N - T + row0, p_last = p0 + nrows - 1;
  const Tiles tr = tiles_for(ret, p0, p_last, a.num_sinks, a.window);
  const int ntiles = tr.count();
  const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
  const uint32_t mb_s = (uint32_t)__cvta_generic_to_shared(&mbar[0]);
  const uint32_t mb_o = (uint32_t)__cvta_generic_to_shared(&mbar[1]);

  // ---- copies: Q once; K / V tiles of 64 keys (rows past p_last or on a bad
  // page are zero-filled)
  {
    const uint16_t *qrow0 = a.q + ((long long)(qs + row0) * sh.Hq + qh) * kD;
    for (int c = tid; c < kM * 16; c += kThreads) {
      const int r = c >> 4, c8 = c & 15;
      const bool ok = r < nrows;
      const uint16_t *src = ok ? qrow0 + (long long)r * sh.Hq * kD + c8 * 8 : a.q;
      cp_async16(sbase + kOffQ + (r >> 3) * 2048 + c8 * 128 + (r & 7) * 16, src, ok ? 16 : 0);
    }
  }
  // Page ids of the CTA's key tiles, 4 per tile, in a shared ring of 128
  // tiles filled 64 tiles at a time, 64 tiles ahead of their copies, so that
  // no page-table load sits on the path of a tile (-1: past p_last or a bad id)
  auto fill_pages = [&](int t0) {
    for (int e = tid; e < 64 * (kN / kPage); e += kThreads) {
      const int t = t0 + e / (kN / kPage), u = e % (kN / kPage);
      int val = -1;
      if (t < ntiles) {
        const long long key = (long long)tr.at(t) * kN + u * kPage;
        if (key <= p_last) {
          val = pt[key / kPage];
          if (val < 0 || val >= sh.num_pages) {
            raise_error(a.err, SD_EBIT_PAGE);
            val = -1;
          }
        }
      }
      s_pg[(t & 127) * (kN / kPage) + u] = val;
    }
  };
  fill_pages(0);
  fill_pages(64);
  __syncthreads();
  // Copies of a tile: thread tid takes the 16-byte chunk c8 = tid % 16 of row
  // r0 = tid / 16 of each of the tile's four pages (x = page), so its
  // shared-memory offsets are fixed up to x (rows r0 + 16 x: 8-row group
  // r0 / 8 + 2 x, row r0 % 8 within it).
  const int r0 = tid >> 4, c8 = tid & 15;
  auto issue_kv = [&](int t, const uint16_t *cache, uint32_t dst0, uint32_t xstride) {
    const int kt = tr.at(t);
    const int *pg = s_pg + (t & 127) * (kN / kPage);
    const unsigned char *base = reinterpret_cast<const unsigned char *>(cache) + c8 * 16;
#pragma unroll
    for (int x = 0; x < kN / kPage; ++x) {
      const int page = pg[x];
      const bool ok = page >= 0 && (long long)kt * kN + x * kPage + r0 <= p_last;
      const unsigned char *src =
          ok ? base + ((((size_t)page * sh.Hkv + g) * kPage + r0) * (size_t)(2 * kD)) : base;
      cp_async16(dst0 + x * xstride, src, ok ? 16 : 0);
    }
  };
  // K: K-major (8-row group -> 2048 bytes); V: MN-major (8-key group -> 128 bytes)
  auto issue_k = [&](int t, int buf) {                // t: position in the CTA's tile list
    issue_kv(t, a.k_cache, sbase + kOffK + buf * kKBytes + (r0 >> 3) * 2048 + c8 * 128 + (r0 & 7) * 16, 2u * 2048u);
  };
  auto issue_v = [&](int t, int buf) {
    issue_kv(t, a.v_cache, sbase + kOffV + buf * kVBytes + c8 * 1024 + (r0 >> 3) * 128 + (r0 & 7) * 16, 2u * 128u);
  };
  if (ntiles > 0) issue_k(0, 0);
  cp_async_commit();
  if (ntiles > 1) issue_k(1, 1);
  cp_async_commit();
  if (ntiles > 0) issue_v(0, 0);
  cp_async_commit();

  // ---- barriers and tensor memory
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mb_s));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mb_o));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(&tslot)),
                 "r"((uint32_t)kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = tslot;
  const uint32_t t_o = tmem, t_s = tmem + 128, t_ph = tmem + 192, t_pl = tmem + 224;
  // warp w reads TMEM lanes 32 (w % 4) .. + 31 (rows) and column half w / 4
  const int quarter = warp & 3, half = warp >> 2;
  const int row = quarter * 32 + lane;                // this thread's query row
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  const long long pos = p0 + row;
  const float sc = a.attn_scale * kLog2e;
  float m_ref = -INFINITY, l = 0.0f;
  bool waited_ok = true;
  // S(0) before the loop; then in iteration i the tensor cores compute S(i + 1)
  // while the CTA turns S(i) into P(i), and P V(i) while it reads S(i + 1)
  auto issue_s = [&](int t) {
    const uint32_t kb = sbase + kOffK + (t & 1) * kKBytes;
#pragma unroll
    for (int s = 0; s < kD / 16; ++s)
      umma(t_s, sdesc(sbase + kOffQ + s * 256, 128, 2048), sdesc(kb + s * 256, 128, 2048), idesc(kN, false),
           s > 0 ? 1u : 0u);
    umma_commit(mb_s);
  };
  cp_async_wait2();                                   // Q and K(0)
  fence_async_smem();
  __syncthreads();
  if (tid == 0 && ntiles > 0) {
    tc_after_sync();
    issue_s(0);
  }
  for (int i = 0; i < ntiles; ++i) {
    const long long j0 = (long long)tr.at(i) * kN;
    if (!mbar_wait(mb_s, (uint32_t)(i & 1))) {        // S(i) is in tensor memory, K(i)'s buffer is free
      waited_ok = false;
      s_bad = 1;
    }
    tc_after_sync();
    if (i + 2 < ntiles) issue_k(i + 2, i & 1);
    cp_async_commit();
    // ---- this row's scores
    constexpr int kH = kN / 2;                        // this thread's columns of S
    float p[kH];
    tmem_ld32(t_s + lane_off + half * kH, p);
    const long long jb = j0 + half * kH;              // position of column 0 of this half
    // ---- masked scores of this half; the row's partial maximum goes to the
    // other half's thread through shared memory at the barrier below.  Every row
    // of the CTA sees the whole tile when its keys lie at or before p0 and, for
    // local rows, are all sinks or all inside the last row's window.
    const bool full = j0 + kN - 1 <= p0 &&
                      (ret || j0 + kN - 1 < a.num_sinks || j0 > p_last - a.window);
    if (!full) {
      const int jr = (int)(pos - jb);                 // column j is seen when j <= jr and, for a local
      const int js = a.num_sinks - (int)jb;           // head, j < js (a sink) or j > jw (in the window)
      const int jw = jr - a.window;
#pragma unroll
      for (int j = 0; j < kH; ++j) {
        const bool ok = j <= jr && (ret || j < js || j > jw);
        p[j] = ok ? p[j] : -INFINITY;
      }
    }
    {
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = p[u];
#pragma unroll
      for (int j = 8; j < kH; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], p[j]);
      s_max[half][row] = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
    }
    cp_async_wait2();                                 // K(i + 1) landed
    fence_async_smem();
    tc_before_sync();
    __syncthreads();                                  // S(i) read by every thread: its columns may be rewritten
    if (s_bad) break;
    if (tid == 0 && i + 1 < ntiles) {
      tc_after_sync();
      issue_s(i + 1);
    }
    if ((i & 63) == 0 && i > 0) fill_pages(i + 64);  // the ring slots of tiles i - 64 .. i - 1 are done with
    // ---- softmax weights (the scale folded into the exponent: p = 2^(s sc - m))
    const float mt = fmaxf(s_max[0][row], s_max[1][row]) * sc;   // the same on both halves' threads
    float factor = 1.0f;
    if (mt > -INFINITY) {
      if (m_ref == -INFINITY) {
        m_ref = mt;                                   // first keys of the row: O and l are still zero
      } else if (mt > m_ref + kRescale) {
        factor = fast_exp2(m_ref - mt);
        m_ref = mt;
      }
    }
    const float nm = m_ref == -INFINITY ? 0.0f : -m_ref;
    float ps8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kH; ++j) {
      p[j] = fast_exp2(fmaf(p[j], sc, nm));           // 2^(-inf) = 0 for masked keys
      ps8[j & 7] += p[j];
    }
    s_sum[half][row] = ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
    // ---- P V(i - 1) must be done before O or P change and before V(i - 1)'s buffer is refilled
    if (i > 0 && !mbar_wait(mb_o, (uint32_t)((i - 1) & 1))) {
      waited_ok = false;
      s_bad = 1;
    }
    tc_after_sync();
    if (i + 1 < ntiles) issue_v(i + 1, (i + 1) & 1);
    cp_async_commit();
    if (__any_sync(kFull, factor != 1.0f)) {          // rescale this warp's rows of O (its column half)
#pragma unroll 1
      for (int c = half * (kD / 2); c < (half + 1) * (kD / 2); c += 32) {
        float o[32];
        tmem_ld32(t_o + lane_off + c, o);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] *= factor;
        tmem_st32(t_o + lane_off + c, o);
      }
    }
    // P = hi + lo in bf16 into tensor memory: column c holds keys 2c (low half) and 2c + 1
    {
      uint32_t h[kH / 2], w[kH / 2];
#pragma unroll
      for (int c = 0; c < kH / 2; ++c) {
        const float x = p[2 * c], y = p[2 * c + 1];
        h[c] = pack_bf16(x, y);
        w[c] = pack_bf16(x - __uint_as_float(h[c] << 16), y - __uint_as_float(h[c] & 0xFFFF0000u));
      }
      tmem_st16u(t_ph + lane_off + half * (kH / 2), h);
      tmem_st16u(t_pl + lane_off + half * (kH / 2), w);
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    cp_async_wait2();                                 // V(i) landed
    fence_async_smem();
    tc_before_sync();
    __syncthreads();                                  // P and O in place, V(i) visible: the tensor cores may go
    l = l * factor + (s_sum[half][row] + s_sum[half ^ 1][row]);
    if (s_bad) break;
    if (tid == 0) {
      tc_after_sync();
      const uint32_t vb = sbase + kOffV + (i & 1) * kVBytes;
#pragma unroll
      for (int s = 0; s < kN / 16; ++s)
        umma_ts(t_o, t_ph + s * 8, sdesc(vb + s * 256, 128, 1024), idesc(kD, true), (i > 0 || s > 0) ? 1u : 0u);
#pragma unroll
      for (int s = 0; s < kN / 16; ++s)
        umma_ts(t_o, t_pl + s * 8, sdesc(vb + s * 256, 128, 1024), idesc(kD, true), 1u);
      umma_commit(mb_o);
    }
  }
  cp_async_wait_all();
  if (ntiles > 0 && !s_bad && !mbar_wait(mb_o, (uint32_t)((ntiles - 1) & 1))) waited_ok = false;
  tc_after_sync();

  // ---- O / l to the output rows (this thread: its row's column half)
  float *orow = a.out + ((long long)(qs + row0 + row) * sh.Hq + qh) * kD;
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
  const bool use_o = ntiles > 0 && !__syncthreads_or(!waited_ok || s_bad);
#pragma unroll 1
  for (int c = half * (kD / 2); c < (half + 1) * (kD / 2); c += 32) {
    float o[32];
    if (use_o) tmem_ld32(t_o + lane_off + c, o);
#pragma unroll
    for (int j = 0; j < 32; ++j) o[j] = use_o ? o[j] * inv : 0.0f;
    if (row < nrows)
#pragma unroll
      for (int j = 0; j < 32; j += 4) *reinterpret_cast<float4 *>(orow + c + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
  }
  if (!use_o && ntiles > 0 && tid == 0) raise_error(a.err, SD_EBIT_TIMEOUT);
  tc_before_sync();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTmemCols));
}

}  // namespace

cudaError_t launch_prefill_tc(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                              const int32_t *page_table, const int32_t *seq_lens, const int32_t *q_starts, int batch,
                              int total_q, float *out, float attn_scale, int window, int num_sinks, const Shape &sh,
                              const Tables &tb, unsigned *err, cudaStream_t st) {
  if (batch == 0 || total_q == 0 || tb.n_ret + tb.n_loc == 0) return cudaSuccess;
  static_assert(kSmem <= 113 * 1024, "two CTAs per SM");
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  TcArgs a{q, k_cache, v_cache, page_table, seq_lens, q_starts, out, attn_scale, window, num_sinks, batch, total_q, err};
  const long long tiles = (long long)(total_q + kM - 1) / kM + batch;   // >= sum_b ceil(T_b / 128)
  const int heads = std::max(tb.max_ret, tb.max_loc);
  const dim3 grid((unsigned)tiles, (unsigned)(tb.n_ret + tb.n_loc), (unsigned)heads);
  return launch_pdl(prefill_tc_kernel, grid, dim3(kThreads), (size_t)kSmem, st, 0, a, sh, tb);
}

}  // namespace sd
