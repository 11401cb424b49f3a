// Head-wise prefill on the 5th-generation tensor cores (tcgen05, accumulators
// in tensor memory), d = 128.  Same operation as sd_prefill.cu: the query at
// position i of a retrieval head attends to keys 0 .. i, of a local head to
// the sinks and the window ending at i (RTPurbo page, Methodology 1; AoH page,
// Methodology 4).
//
// One CTA per (128 consecutive query positions of one sequence, two query
// heads of one KV group): both heads read the same key tiles, so each K / V
// tile is fetched once for two heads.  Warp roles:
//   warps 0-3, 4-7   softmax of head slot 0, 1: thread = query row (warp w
//                    reads TMEM lanes 32 (w % 4) ..), the whole 64-key row of S
//   warps 8-9        copies of the K / V tiles (cp.async, four buffers each)
//   warp 10          the MMA warp: one elected lane issues every MMA
// Tensor memory of head slot s (columns from 256 s): O 0..127 (float32), S / P
// 128..191, Q 192..255 (bf16 pairs).  Per key tile of 64 positions:
//   S_s[128 x 64]  = Q_s[128 x 128] K^T   (A = Q from TMEM, B = K K-major in
//                                          shared memory)
//   P_s            = 2^(S log2e scale - m) (masked), split P = P_hi + P_lo in
//                    bf16 and stored over S_s's own columns by each thread
//   O_s[128 x 128] += P_hi V + P_lo V      (A = P from TMEM, B = V MN-major in
//                                          shared memory)
// Q in tensor memory keeps the S MMAs off the shared-memory bandwidth (only K
// is read there), and P over S keeps two heads within the 512 columns.  The MMA
// warp issues, per head, P V(i) and then S(i + 1) into the same columns (the
// tensor cores run one thread's MMAs in order, so S(i + 1) overwrites P(i) only
// after P V(i) has read it), and commits both to one mbarrier: its arrival
// tells the softmax warps that S(i + 1) is there and that O holds P V(i).  While
// one head's softmax runs, the tensor cores work on the other head.
// The hand-offs are mbarriers, no CTA-wide barrier inside the loop: a K / V
// buffer is full when every copy thread's cp.async.mbarrier.arrive has fired
// (its copies landed; the MMA warp then fences them to the async proxy), and a
// buffer slot (K and V of one tile) is free when tcgen05.commit says that the
// tile's S and P V MMAs of both heads are done; S_s is full
// when tcgen05.commit arrives; P_s is stored when each softmax warp arrives.
// Every wait is bounded (a poll count and 2 s of the global timer) and also
// ends when another role has given up (a shared flag): the CTA then sets
// SD_EBIT_TIMEOUT, waits for its own MMAs and copies, writes zeros and frees
// its tensor memory.  A test-only switch (sparse_decode_testing_stall_prefill)
// makes the MMA warp first wait on an mbarrier that nothing arrives at, so
// that the tests can check this path.
//
// The softmax reference of a row (log2 units) is set by the first keys it sees
// and moved only when a tile's weights against it sum past 2^64 or overflow;
// then S is read again, the reference becomes the tile's maximum and O is
// rescaled in tensor memory (ld, scale, st).  Most tiles so skip both the row
// maximum and the rescale; P (hi + lo) and O keep their relative precision at
// any magnitude up to 2^64.
//
// Shared-memory operand layouts are the canonical no-swizzle ones: 8 rows x
// 16 bytes per core matrix (128 contiguous bytes); for the K-major K the two
// core matrices of one 16-element K step are LBO = 128 bytes apart and
// consecutive 8-row groups SBO apart; for the MN-major V the 8-key groups are
// LBO = 128 bytes apart and consecutive 8-dim chunks SBO apart.  In TMEM, an A
// operand (Q, P) has one row per lane and two 16-bit K elements per 32-bit
// column.
#include <algorithm>
#include <atomic>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSoftmaxThreads = 256;    // two warpgroups, one per head slot
constexpr int kLoadThreads = 64;        // warps 8-9
constexpr int kThreads = kSoftmaxThreads + kLoadThreads + 32;   // + the MMA warp
constexpr int kMmaWarp = (kSoftmaxThreads + kLoadThreads) / 32;
constexpr int kD = 128;                 // head dimension
constexpr int kM = 128;                 // query rows per CTA
constexpr int kN = 64;                  // keys per tile
constexpr int kStages = 4;              // K and V buffers
constexpr float kBig = 1.8446744e19f;   // 2^64: a tile whose weights sum past this moves the reference
constexpr long long kWaitSpins = 1LL << 26;
constexpr unsigned long long kWaitNs = 2000000000ull;

// shared memory (bytes)
constexpr int kKBytes = kN * kD * 2;    // 16 KB, K-major, SBO 2048
constexpr int kVBytes = kN * kD * 2;    // 16 KB, MN-major, SBO 1024
constexpr int kOffK = 0;                        // kStages buffers
constexpr int kOffV = kOffK + kStages * kKBytes;
constexpr int kSmem = kOffV + kStages * kVBytes;   // 128 KB: one CTA per SM
// tensor memory: per head slot s, from column 256 s: O 0..127, S / P 128..191
// (P hi 128..159, P lo 160..191), Q 192..255
constexpr int kTmemCols = 512;

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
// tcgen05.mma, kind::f16, A read from tensor memory (lane = row, two 16-bit K
// elements per column), B from shared memory; ACC = false overwrites D.  The
// whole (converged) warp executes it and one elected lane issues, so the
// operands stay warp-uniform and the enable-input-d flag is an immediate.
template <bool ACC>
__device__ __forceinline__ void umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db, uint32_t id) {
  if (ACC)
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 1;\n\t}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(id));
  else
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 0;\n\t}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(db), "r"(id));
}
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
// arrive on an mbarrier once the MMAs issued so far have completed; the same
// elected lane as the MMAs (the lowest active lane of the full warp)
__device__ __forceinline__ void umma_commit(uint32_t mbar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(mbar)
      : "memory");
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for completion `phase` (0, 1, 0, ...) of an mbarrier.  False when the
// shared abort flag (if given) is up, because another role gave up, or after
// kWaitSpins polls or kWaitNs of the global timer, whichever comes first; a
// wait that runs out raises the flag itself, so that every other role stops at
// its next wait.
__device__ __forceinline__ bool mbar_wait(uint32_t mbar, uint32_t phase, volatile int *abort) {
  unsigned long long t0 = 0;
  for (long long it = 0; it < kWaitSpins; ++it) {
    uint32_t done;
    asm volatile("{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2;\n\t"
                 "selp.b32 %0, 1, 0, P1;\n\t}\n"
                 : "=r"(done)
                 : "r"(mbar), "r"(phase)
                 : "memory");
    if (done) return true;
    if (abort != nullptr && *abort) return false;
    if ((it & 255) == 0) {
      const unsigned long long t = global_ns();
      if (it == 0) t0 = t;
      else if (t - t0 > kWaitNs) break;
    }
  }
  if (abort != nullptr) *abort = 1;
  return false;
}
__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// arrive on an mbarrier once every cp.async this thread has issued so far has
// landed; the arrival counts toward the barrier's expected count
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t mbar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(mbar) : "memory");
}
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
// 64 consecutive float32 columns (two loads, one wait)
__device__ __forceinline__ void tmem_ld32x2(uint32_t addr, float (&v)[64]) {
  uint32_t r[64];
#define SD_TMEM_LD32(A, R)                                                                                            \
  asm volatile(                                                                                                      \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"              \
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                                     \
      : "=r"(R[0]), "=r"(R[1]), "=r"(R[2]), "=r"(R[3]), "=r"(R[4]), "=r"(R[5]), "=r"(R[6]), "=r"(R[7]), "=r"(R[8]),   \
        "=r"(R[9]), "=r"(R[10]), "=r"(R[11]), "=r"(R[12]), "=r"(R[13]), "=r"(R[14]), "=r"(R[15]), "=r"(R[16]),      \
        "=r"(R[17]), "=r"(R[18]), "=r"(R[19]), "=r"(R[20]), "=r"(R[21]), "=r"(R[22]), "=r"(R[23]), "=r"(R[24]),     \
        "=r"(R[25]), "=r"(R[26]), "=r"(R[27]), "=r"(R[28]), "=r"(R[29]), "=r"(R[30]), "=r"(R[31])                   \
      : "r"(A))
  SD_TMEM_LD32(addr, r);
  SD_TMEM_LD32(addr + 32, (r + 32));
#undef SD_TMEM_LD32
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 64; ++j) v[j] = __uint_as_float(r[j]);
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
  int stall;                      // testing: the MMA warp first waits on a barrier nothing arrives at
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

__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const TcArgs a, const Shape sh, const Tables tb) {
  extern __shared__ __align__(1024) unsigned char sm[];
  // mbarriers: K / V buffer full (copy warps) and free (MMA commit); per head
  // slot Q stored and P stored (softmax warps), S full (MMA commit: S(i) and
  // the P V before it), the last P V done (MMA commit); the MMA thread's drain
  __shared__ __align__(8) uint64_t bar_kfull[kStages], bar_vfull[kStages], bar_free[kStages];
  __shared__ __align__(8) uint64_t bar_qfull[2], bar_sfull[2], bar_pfull[2], bar_odone[2], bar_drain, bar_never;
  __shared__ uint32_t tslot;
  __shared__ int s_b, s_t;
  __shared__ volatile int s_bad;
  __shared__ Group s_grp;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gr = blockIdx.y, pair = blockIdx.z;
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
  const int nh = b < 0 ? 0 : (s_grp.n - 2 * pair < 2 ? s_grp.n - 2 * pair : 2);   // head slots of this CTA
  if (nh <= 0) return;                                 // past the last tile, or past the group's heads
  const int qs = a.q_starts[b];
  const int T = a.q_starts[b + 1] - qs;
  const long long N = a.seq_lens[b];
  if (N < 0 || N > sh.max_len || T > N || qs < 0 || qs + T > a.total_q) {
    if (tid == 0) raise_error(a.err, SD_EBIT_SEQLEN);
    return;
  }
  const int g = s_grp.kv_head;
  const int row0 = s_t * kM;
  const int nrows = T - row0 < kM ? T - row0 : kM;
  const long long p0 = N - T + row0, p_last = p0 + nrows - 1;
  const Tiles tr = tiles_for(ret, p0, p_last, a.num_sinks, a.window);
  const int ntiles = tr.count();
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(sm);
  auto bar = [](uint64_t *p) { return (uint32_t)__cvta_generic_to_shared(p); };

  // ---- barriers, tensor memory
  if (tid == 0) {
    for (int k = 0; k < kStages; ++k) {
      mbar_init(bar(&bar_kfull[k]), kLoadThreads);
      mbar_init(bar(&bar_vfull[k]), kLoadThreads);
      mbar_init(bar(&bar_free[k]), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar(&bar_sfull[k]), 1);
      mbar_init(bar(&bar_qfull[k]), 4);
      mbar_init(bar(&bar_pfull[k]), 4);
      mbar_init(bar(&bar_odone[k]), 1);
    }
    mbar_init(bar(&bar_drain), 1);
    mbar_init(bar(&bar_never), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(&tslot)),
                 "r"((uint32_t)kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tmem = tslot;

  if (tid < kSoftmaxThreads) {
    // ================= softmax: head slot s, query row `row`
    const int s = warp >> 2, quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t t_o = tmem + 256u * s + lane_off, t_s = t_o + 128, t_q = t_o + 192;
    const long long pos = p0 + row;
    const float sc = a.attn_scale * kLog2e;
    float m_ref = -INFINITY, l = 0.0f;
    bool ok = true;
    if (s < nh) {
      const int qh = s_grp.q_head[2 * pair + s];
      // ---- this row's query into tensor memory (zeros past the last row)
      {
        uint32_t qv[32];
        const uint4 *qrow = reinterpret_cast<const uint4 *>(a.q + ((long long)(qs + row0 + row) * sh.Hq + qh) * kD);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 v = row < nrows ? qrow[half * 8 + c] : make_uint4(0u, 0u, 0u, 0u);
            qv[4 * c] = v.x;
            qv[4 * c + 1] = v.y;
            qv[4 * c + 2] = v.z;
            qv[4 * c + 3] = v.w;
          }
          tmem_st32u(t_q + half * 32, qv);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(&bar_qfull[s]));
      }
      const uint32_t b_sfull = bar(&bar_sfull[s]), b_pfull = bar(&bar_pfull[s]);
      for (int i = 0; i < ntiles; ++i) {
        const long long j0 = (long long)tr.at(i) * kN;
        // S(i) in tensor memory, and O holds P V(i - 1)
        ok = __all_sync(kFull, mbar_wait(b_sfull, (uint32_t)(i & 1), &s_bad));
        if (!ok) break;
        tc_after_sync();
        float p[kN];
        // ---- masked scores.  Every row of the CTA sees the whole tile when its
        // keys lie at or before p0 and, for local rows, are all sinks or all
        // inside the last row's window.
        const bool full = j0 + kN - 1 <= p0 && (ret || j0 + kN - 1 < a.num_sinks || j0 > p_last - a.window);
        auto load_scores = [&]() {                    // warp-collective
          tmem_ld32x2(t_s, p);
          if (!full) {
            const int jr = (int)(pos - j0);           // column j is seen when j <= jr and, for a local
            const int js = a.num_sinks - (int)j0;     // head, j < js (a sink) or j > jw (in the window)
            const int jw = jr - a.window;
#pragma unroll
            for (int j = 0; j < kN; ++j) {
              const bool seen = j <= jr && (ret || j < js || j > jw);
              p[j] = seen ? p[j] : -INFINITY;
            }
          }
        };
        auto scaled_max = [&]() {                     // the tile's maximum of this row, times sc
          float mx8[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mx8[u] = p[u];
#pragma unroll
          for (int j = 8; j < kN; ++j) mx8[j & 7] = fmaxf(mx8[j & 7], p[j]);
          return fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                       fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * sc;
        };
        float ps8[8];
        auto weights = [&]() {                        // p = 2^(s sc - m_ref); 2^(-inf) = 0 for masked keys
          const float nm = m_ref == -INFINITY ? 0.0f : -m_ref;
#pragma unroll
          for (int u = 0; u < 8; ++u) ps8[u] = 0.0f;
#pragma unroll
          for (int j = 0; j < kN; ++j) {
            p[j] = fast_exp2(fmaf(p[j], sc, nm));
            ps8[j & 7] += p[j];
          }
          return ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
        };
        load_scores();
        // ---- softmax weights against the row's reference m_ref (log2 units),
        // which is set by the first keys the row sees and only moved when a
        // tile's weights against it sum past kBig (or overflow): then S is read
        // again, m_ref becomes the tile's maximum and O is rescaled.  Most tiles
        // thus skip the row maximum altogether; P and O keep their relative
        // precision at any magnitude up to kBig.
        float factor = 1.0f;
        if (__any_sync(kFull, m_ref == -INFINITY)) {
          const float mt = scaled_max();
          if (m_ref == -INFINITY) m_ref = mt;         // O and l are still zero; -inf again if no key is seen
        }
        float psum = weights();
        if (__any_sync(kFull, !(psum <= kBig))) {
          const bool moved = !(psum <= kBig);
          load_scores();
          const float mt = scaled_max();
          if (moved && mt > m_ref) {
            factor = fast_exp2(m_ref - mt);
            m_ref = mt;
          }
          psum = weights();
        }
        if (__any_sync(kFull, factor != 1.0f)) {      // rescale this warp's rows of O
#pragma unroll 1
          for (int c = 0; c < kD; c += 32) {
            float o[32];
            tmem_ld32(t_o + c, o);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] *= factor;
            tmem_st32(t_o + c, o);
          }
        }
        // P = hi + lo in bf16 over S: column c of each half holds keys 2c (low
        // half) and 2c + 1
        {
          uint32_t h[kN / 2];
#pragma unroll
          for (int c = 0; c < kN / 2; ++c) h[c] = pack_bf16(p[2 * c], p[2 * c + 1]);
          tmem_st32u(t_s, h);
#pragma unroll
          for (int c = 0; c < kN / 2; ++c)
            h[c] = pack_bf16(p[2 * c] - __uint_as_float(h[c] << 16), p[2 * c + 1] - __uint_as_float(h[c] & 0xFFFF0000u));
          tmem_st32u(t_s + kN / 2, h);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(b_pfull);          // P(i) and O in place: P V(i) may go
        l = l * factor + psum;
      }
      if (ok && ntiles > 0) {                         // the last P V
        ok = __all_sync(kFull, mbar_wait(bar(&bar_odone[s]), 0u, &s_bad));
        tc_after_sync();
      }
      // ---- O / l to the output row
      const bool use_o = ok && ntiles > 0;
      float *orow = a.out + ((long long)(qs + row0 + row) * sh.Hq + qh) * kD;
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;
#pragma unroll 1
      for (int c = 0; c < kD; c += 32) {
        float o[32];
        if (use_o) tmem_ld32(t_o + c, o);
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = use_o ? o[j] * inv : 0.0f;
        if (row < nrows)
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4 *>(orow + c + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
      }
    }
  } else if (warp < kMmaWarp) {
    // ================= copies of the K / V tiles: thread lt takes the 16-byte
    // chunk c8 of rows r0 + 4 x (x = 0..15) of each tile, so its shared-memory
    // offsets are fixed up to x (K: 8-row group x / 2, row r0 + 4 (x % 2) in it;
    // V: 8-key group x / 2, the same row)
    const int lt = tid - kSoftmaxThreads, r0 = lt >> 4, c8 = lt & 15;
    const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
    const uint32_t k_dst = sbase + kOffK + (uint32_t)(c8 * 128 + r0 * 16);
    const uint32_t v_dst = sbase + kOffV + (uint32_t)(c8 * 1024 + r0 * 16);
    const unsigned char *kbase = reinterpret_cast<const unsigned char *>(a.k_cache) + c8 * 16;
    const unsigned char *vbase = reinterpret_cast<const unsigned char *>(a.v_cache) + c8 * 16;
    // The copies of a tile complete asynchronously: each thread's
    // cp.async.mbarrier.arrive.noinc counts on the buffer's "full" barrier once
    // all its copies so far have landed (the MMA thread fences them to the
    // async proxy after its wait), so up to kStages tiles are in flight.
    // page ids of the tile after the current one are loaded while the current
    // tile's copies are issued (kPastEnd past p_last); checked one iteration later
    constexpr int kPastEnd = -0x7FFFFFFF - 1;
    auto raw_pages = [&](int t) {
      const long long k0 = (long long)tr.at(t) * kN;
      int4 v;
      v.x = k0 <= p_last ? pt[k0 / kPage] : kPastEnd;
      v.y = k0 + kPage <= p_last ? pt[k0 / kPage + 1] : kPastEnd;
      v.z = k0 + 2 * kPage <= p_last ? pt[k0 / kPage + 2] : kPastEnd;
      v.w = k0 + 3 * kPage <= p_last ? pt[k0 / kPage + 3] : kPastEnd;
      return v;
    };
    auto checked = [&](int id) {                      // -1: zero-fill; a bad id also sets the error bit
      if (id == kPastEnd) return -1;
      if (id < 0 || id >= sh.num_pages) {
        raise_error(a.err, SD_EBIT_PAGE);
        return -1;
      }
      return id;
    };
    bool ok = true;
    int4 nxt = ntiles > 0 ? raw_pages(0) : make_int4(kPastEnd, kPastEnd, kPastEnd, kPastEnd);
    for (int i = 0; i < ntiles; ++i) {
      const int bi = i % kStages;
      const uint32_t par = (uint32_t)(((i / kStages) + 1) & 1);   // completion i / kStages - 1: tile i - kStages
      const long long k0 = (long long)tr.at(i) * kN;
      const int pgs[kN / kPage] = {checked(nxt.x), checked(nxt.y), checked(nxt.z), checked(nxt.w)};
      if (i + 1 < ntiles) nxt = raw_pages(i + 1);
      long long so[kN / 4];                           // byte offsets of this thread's rows (-1: zero-fill)
#pragma unroll
      for (int x = 0; x < kN / 4; ++x) {
        const int r = r0 + 4 * x;                     // key row of the tile
        const int page = pgs[r / kPage];
        so[x] = page >= 0 && k0 + r <= p_last
                    ? (long long)((((size_t)page * sh.Hkv + g) * kPage + (r % kPage)) * (size_t)(2 * kD))
                    : -1;
      }
      if (i >= kStages) ok = __all_sync(kFull, mbar_wait(bar(&bar_free[bi]), par, &s_bad));
      if (!ok) break;
#pragma unroll
      for (int x = 0; x < kN / 4; ++x)
        cp_async16(k_dst + bi * kKBytes + (x >> 1) * 2048 + (x & 1) * 64, so[x] >= 0 ? kbase + so[x] : kbase,
                   so[x] >= 0 ? 16 : 0);
      cp_async_arrive_noinc(bar(&bar_kfull[bi]));
#pragma unroll
      for (int x = 0; x < kN / 4; ++x)
        cp_async16(v_dst + bi * kVBytes + (x >> 1) * 128 + (x & 1) * 64, so[x] >= 0 ? vbase + so[x] : vbase,
                   so[x] >= 0 ? 16 : 0);
      cp_async_arrive_noinc(bar(&bar_vfull[bi]));
    }
    cp_async_wait_all();
  } else if (ntiles > 0) {
    // ================= the MMA warp: every lane runs this code and waits; one
    // elected lane issues the MMAs and commits
    // descriptors of the operands' first K step, built once: the K step k and
    // the buffer b only move the start address, i.e. add (offset >> 4) to the
    // descriptor's low field
    const uint64_t dk0 = sdesc(sbase + kOffK, 128, 2048);
    const uint64_t dv0 = sdesc(sbase + kOffV, 128, 1024);
    constexpr uint32_t id_s = idesc(kN, false), id_o = idesc(kD, true);
    auto issue_s = [&](int t, int s) {                // S_s(t) = Q_s K(t)^T, Q from TMEM
      const uint64_t dk = dk0 + (uint64_t)((t % kStages) * (kKBytes >> 4));
      const uint32_t to = tmem + 256u * s;
      umma_ts<false>(to + 128, to + 192, dk, id_s);
#pragma unroll
      for (int k = 1; k < kD / 16; ++k) umma_ts<true>(to + 128, to + 192 + k * 8, dk + k * 16, id_s);
      umma_commit(bar(&bar_sfull[s]));                // also covers the P V issued before it
    };
    auto issue_pv = [&](int t, int s) {               // O_s += (P_hi + P_lo) V(t), P from TMEM (over S)
      const uint64_t dv = dv0 + (uint64_t)((t % kStages) * (kVBytes >> 4));
      const uint32_t to = tmem + 256u * s;
      if (t == 0) umma_ts<false>(to, to + 128, dv, id_o);
      else umma_ts<true>(to, to + 128, dv, id_o);
#pragma unroll
      for (int k = 1; k < kN / 16; ++k) umma_ts<true>(to, to + 128 + k * 8, dv + k * 16, id_o);
#pragma unroll
      for (int k = 0; k < kN / 16; ++k) umma_ts<true>(to, to + 160 + k * 8, dv + k * 16, id_o);
    };
    bool ok = true;
    if (a.stall) ok = __all_sync(kFull, mbar_wait(bar(&bar_never), 0u, &s_bad));   // runs out: the test of the bounds
    ok = ok && __all_sync(kFull, mbar_wait(bar(&bar_kfull[0]), 0u, &s_bad));
    fence_async_smem();                               // the copy warps' writes, to the async proxy
    for (int s = 0; s < nh && ok; ++s) {
      ok = __all_sync(kFull, mbar_wait(bar(&bar_qfull[s]), 0u, &s_bad));
      tc_after_sync();
      if (ok) issue_s(0, s);
    }
    for (int i = 0; i < ntiles && ok; ++i) {
      const bool more = i + 1 < ntiles;
      // V(i) and K(i + 1) landed; one fence to the async proxy for both
      ok = __all_sync(kFull, mbar_wait(bar(&bar_vfull[i % kStages]), (uint32_t)((i / kStages) & 1), &s_bad));
      if (ok && more)
        ok = __all_sync(kFull, mbar_wait(bar(&bar_kfull[(i + 1) % kStages]), (uint32_t)(((i + 1) / kStages) & 1),
                                         &s_bad));
      fence_async_smem();
      // per head: P V(i), then S(i + 1) into the same columns
      for (int s = 0; s < nh && ok; ++s) {
        ok = __all_sync(kFull, mbar_wait(bar(&bar_pfull[s]), (uint32_t)(i & 1), &s_bad));
        tc_after_sync();
        if (!ok) break;
        issue_pv(i, s);
        if (more) issue_s(i + 1, s);
        else umma_commit(bar(&bar_odone[s]));
      }
      if (!ok) break;
      umma_commit(bar(&bar_free[i % kStages]));       // K(i) and V(i): S(i) and P V(i) of both heads are done
    }
    // every MMA issued above completes before tensor memory is freed (this
    // wait ignores the abort flag; the MMAs depend on nothing and finish)
    umma_commit(bar(&bar_drain));
    if (!__all_sync(kFull, mbar_wait(bar(&bar_drain), 0u, nullptr))) s_bad = 1;
  }

  // ---- every role ends here
  tc_before_sync();
  __syncthreads();
  if (tid == 0 && s_bad) raise_error(a.err, SD_EBIT_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kTmemCols));
  }
}

}  // namespace

std::atomic<int> g_prefill_stall{0};

cudaError_t launch_prefill_tc(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                              const int32_t *page_table, const int32_t *seq_lens, const int32_t *q_starts, int batch,
                              int total_q, float *out, float attn_scale, int window, int num_sinks, const Shape &sh,
                              const Tables &tb, unsigned *err, cudaStream_t st) {
  if (batch == 0 || total_q == 0 || tb.n_ret + tb.n_loc == 0) return cudaSuccess;
  static_assert(kSmem > 114 * 1024 && kSmem <= 227 * 1024, "one CTA per SM: it holds all 512 TMEM columns");
  cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) return e;
  TcArgs a{q, k_cache, v_cache, page_table, seq_lens, q_starts, out, attn_scale, window, num_sinks, batch, total_q, err,
           g_prefill_stall.load()};
  const long long tiles = (long long)(total_q + kM - 1) / kM + batch;   // >= sum_b ceil(T_b / 128)
  const int heads = std::max(tb.max_ret, tb.max_loc);
  const dim3 grid((unsigned)tiles, (unsigned)(tb.n_ret + tb.n_loc), (unsigned)((heads + 1) / 2));
  return launch_pdl(prefill_tc_kernel, grid, dim3(kThreads), (size_t)kSmem, st, 0, a, sh, tb);
}

}  // namespace sd
