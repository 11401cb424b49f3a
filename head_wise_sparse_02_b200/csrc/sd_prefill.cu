// Head-wise prefill attention: the queries of a chunk attend causally, each
// retrieval head to every earlier key, each local head to the sinks plus the
// window ending at its own position.
//
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 1: local heads
// run a sliding window with attention sinks through inference, while the
// retrieval heads keep their full KV during prefill (sparse selection starts
// at decode); its results report the prefill speed-up over dense attention
// growing with the context.  AoH page (gist.science/ar/paper/2608.06849),
// Methodology 4: streaming heads keep sinks plus a recent window, with
// standard chunked prefill.
//
// One CTA per (16 consecutive query positions of one sequence, KV group,
// role): four warps, warp w takes head w of the group's heads of that role
// (heads 4.., 8.. in further passes), its 16 query rows on the M side of the
// MMAs.  The group's keys and values stream through a two-stage shared-memory
// ring in tiles of 64 positions (4 pages, whole 2d-byte rows per cp.async
// chunk set) shared by the four warps: S = Q K^T and O += P V on the tensor
// cores (mma.sync m16n8k16, bf16 in, float32 accumulation, P split into
// bf16 hi + lo so that the weights keep 16 bits), online softmax in base 2.
// Tiles outside every row's key range are never loaded: a retrieval CTA
// reads tiles 0 .. p_last / 64, a local CTA the sink tiles and the window
// tiles only.  K/V tiles are re-read by the CTAs of later query tiles of the
// same sequence, so they keep the default L2 policy.
#include <algorithm>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kQT = 16;                 // query positions per CTA
constexpr int kKT = 64;                 // key positions per tile (4 pages)

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
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
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

template <int D>
__host__ __device__ constexpr int row_pitch() {
  return 2 * D + 16;                                 // bytes of one staged K or V row (padded)
}
template <int D>
__host__ __device__ constexpr size_t stage_bytes() {
  return (size_t)2 * kKT * row_pitch<D>();           // K tile + V tile
}

struct PrefillArgs {
  const uint16_t *q;              // [total_q, Hq, d]
  const uint16_t *k_cache, *v_cache;
  const int32_t *page_table, *seq_lens, *q_starts;
  float *out;                     // [total_q, Hq, d]
  float attn_scale;
  int window, num_sinks, batch, total_q;
  unsigned *err;
};

// Key tiles of a CTA, ascending and without repeats: retrieval rows read
// [0, p_last]; local rows the sinks [0, min(S, p_last + 1)) and the window
// [max(0, p0 - W + 1), p_last].
struct TileRange {
  int a0, a1;                     // first range of tiles [a0, a1)
  int b0, b1;                     // second range [b0, b1), after the first
  __device__ int count() const { return (a1 - a0) + (b1 - b0); }
  __device__ int at(int i) const { return i < a1 - a0 ? a0 + i : b0 + (i - (a1 - a0)); }
};

__device__ TileRange tiles_of(bool ret, long long p0, long long p_last, int S, int W) {
  TileRange t{0, 0, 0, 0};
  if (ret) {
    t.a1 = (int)(p_last / kKT) + 1;
    return t;
  }
  const long long s_end = std::min<long long>(S, p_last + 1);          // sink keys [0, s_end)
  const long long w_lo = std::max<long long>(0, p0 - W + 1);           // window keys [w_lo, p_last]
  const bool has_w = W > 0;
  if (s_end > 0) t.a1 = (int)((s_end - 1) / kKT) + 1;
  if (has_w) {
    int lo = (int)(w_lo / kKT);
    const int hi = (int)(p_last / kKT) + 1;
    lo = std::max(lo, t.a1);                                           // tiles already in the sink range
    if (lo < hi) {
      if (lo == t.a1) t.a1 = hi;                                       // contiguous: one range
      else {
        t.b0 = lo;
        t.b1 = hi;
      }
    }
  }
  return t;
}

template <int D>
__global__ void __launch_bounds__(kThreads)
prefill_kernel(const PrefillArgs a, const Shape sh, const Tables tb) {
  constexpr int KS = D / 16;                         // k-steps over the head dimension
  constexpr int NT = D / 8;                          // n-tiles of the output
  constexpr int PITCH = row_pitch<D>();
  constexpr int CPR = 2 * D / 16;                    // 16-byte chunks per row
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_b, s_t;
  __shared__ Group s_grp;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int gr = blockIdx.y;
  const bool ret = gr < tb.n_ret;
  pdl_wait();
  pdl_trigger();

  // ---- which (sequence, query tile): tiles numbered sequence by sequence,
  // handed out last first (the longest key ranges start first)
  if (warp == 0) {
    const int want = (int)gridDim.x - 1 - (int)blockIdx.x;
    int base = 0, found_b = -1, found_t = 0;
    for (int c = 0; c < a.batch && found_b < 0; c += 32) {
      const int b = c + lane;
      int nt = 0;
      if (b < a.batch) {
        const int t = a.q_starts[b + 1] - a.q_starts[b];
        nt = t > 0 ? (t + kQT - 1) / kQT : 0;
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
      s_grp = ret ? tb.ret[gr] : tb.loc[gr - tb.n_ret];
    }
  }
  __syncthreads();
  const int b = s_b;
  if (b < 0) return;                                 // past the last tile
  const int qs = a.q_starts[b];
  const int T = a.q_starts[b + 1] - qs;
  long long N = a.seq_lens[b];
  if (N < 0 || N > sh.max_len || T > N || qs < 0 || qs + T > a.total_q) {
    if (tid == 0) raise_error(a.err, SD_EBIT_SEQLEN);
    return;
  }
  const int row0 = s_t * kQT;                        // first query row of the tile within the chunk
  const int nrows = T - row0 < kQT ? T - row0 : kQT;
  const long long p0 = N - T + row0, p_last = p0 + nrows - 1;
  const int g = s_grp.kv_head, nh = s_grp.n;
  const TileRange tr = tiles_of(ret, p0, p_last, a.num_sinks, a.window);
  const int ntiles = tr.count();
  const int32_t *pt = a.page_table + (long long)b * sh.max_pages;
  const float sc = a.attn_scale * kLog2e;
  const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(smem);

  // cp.async of key tile `kt` into stage `st`: 64 rows x CPR chunks of K and of V
  auto issue = [&](int kt, int st) {
    const uint32_t kdst = sbase + st * (uint32_t)stage_bytes<D>();
    const uint32_t vdst = kdst + kKT * PITCH;
    // the tile's four page ids first (independent loads), then the copies
    int pg[kKT / kPage];
#pragma unroll
    for (int u = 0; u < kKT / kPage; ++u) {
      const long long key = (long long)kt * kKT + u * kPage;
      int page = key <= p_last ? pt[key / kPage] : -1;
      if (key <= p_last && (page < 0 || page >= sh.num_pages)) {
        raise_error(a.err, SD_EBIT_PAGE);
        page = -1;
      }
      pg[u] = page;
    }
#pragma unroll
    for (int x = 0; x < kKT * CPR / kThreads; ++x) {
      const int c = tid + kThreads * x;
      const int r = c / CPR, ch = c % CPR;
      const long long key = (long long)kt * kKT + r;
      const int page = key <= p_last ? pg[r / kPage] : -1;
      const size_t off = page >= 0 ? (((size_t)page * sh.Hkv + g) * kPage + (size_t)(key % kPage)) * (2 * D) + ch * 16 : 0;
      const int bytes = page >= 0 ? 16 : 0;          // rows past p_last or on a bad page are zero-filled
      cp_async16(kdst + r * PITCH + ch * 16, reinterpret_cast<const unsigned char *>(a.k_cache) + off, bytes);
      cp_async16(vdst + r * PITCH + ch * 16, reinterpret_cast<const unsigned char *>(a.v_cache) + off, bytes);
    }
    cp_async_commit();
  };

  // ldmatrix lane offsets: K (keys x dims, non-transposed) and V (transposed)
  const int lm = lane >> 3, lr = lane & 7;
  const uint32_t k_lane = (lr + (lm >> 1) * 8) * PITCH + (lm & 1) * 16;
  const uint32_t v_lane = (lr + (lm & 1) * 8) * PITCH + (lm >> 1) * 16;

  for (int hc = 0; hc < nh; hc += kWarps) {
    const int hi = hc + warp;                        // this warp's head (index in the group's list)
    const bool active = hi < nh;
    const int qh = active ? s_grp.q_head[hi] : 0;
    // Q fragments: rows gq / gq + 8 are query rows row0 + gq / + 8 of head qh
    uint32_t qa[KS][4];
    {
      const bool v0 = active && gq < nrows, v1 = active && gq + 8 < nrows;
      const uint16_t *q0 = a.q + ((long long)(qs + row0 + gq) * sh.Hq + qh) * D;
      const uint16_t *q1 = a.q + ((long long)(qs + row0 + gq + 8) * sh.Hq + qh) * D;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        const int cc = k * 16 + 2 * tq;
        qa[k][0] = v0 ? *reinterpret_cast<const uint32_t *>(q0 + cc) : 0u;
        qa[k][1] = v1 ? *reinterpret_cast<const uint32_t *>(q1 + cc) : 0u;
        qa[k][2] = v0 ? *reinterpret_cast<const uint32_t *>(q0 + cc + 8) : 0u;
        qa[k][3] = v1 ? *reinterpret_cast<const uint32_t *>(q1 + cc + 8) : 0u;
      }
    }
    const long long pos0 = p0 + gq, pos1 = p0 + gq + 8;   // positions of this thread's two rows
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    if (ntiles > 0) issue(tr.at(0), 0);
    for (int i = 0; i < ntiles; ++i) {
      if (i + 1 < ntiles) {
        issue(tr.at(i + 1), (i + 1) & 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();                               // tile i is in shared memory for every warp
      const int kt = tr.at(i);
      const long long j0 = (long long)kt * kKT;
      const uint32_t kb = sbase + (i & 1) * (uint32_t)stage_bytes<D>();
      const uint32_t vb = kb + kKT * PITCH;
      if (active) {
        // ---- S = Q K^T over the tile's 64 keys
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
        for (int k = 0; k < KS; ++k)
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            uint32_t r[4];
            ldsm_x4(r, kb + np * 16 * PITCH + k * 32 + k_lane);
            mma_bf16(s[2 * np], qa[k], r[0], r[1]);
            mma_bf16(s[2 * np + 1], qa[k], r[2], r[3]);
          }
        // ---- masks: key j is seen by the row at position p when j <= p and,
        // for a local head, j < S or j > p - W; the whole tile is inside every
        // row's range in the common case
        const bool full = (j0 + kKT - 1 <= p0) &&
                          (ret || j0 + kKT - 1 < a.num_sinks || j0 >= p_last - a.window + 1);
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const long long j = j0 + n * 8 + 2 * tq + (e & 1);
            const long long p = e < 2 ? pos0 : pos1;
            float v = s[n][e] * sc;
            if (!full) {
              const bool ok = j <= p && (ret || j < a.num_sinks || j > p - a.window);
              v = ok ? v : -INFINITY;
            }
            s[n][e] = v;
            if (e < 2) mx0 = fmaxf(mx0, v);
            else mx1 = fmaxf(mx1, v);
          }
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float ref0 = mn0 == -INFINITY ? 0.f : mn0, ref1 = mn1 == -INFINITY ? 0.f : mn1;
        const float c0 = fast_exp2(m0 - ref0), c1 = fast_exp2(m1 - ref1);   // exp2(-inf) = 0 on the first tile
        m0 = mn0;
        m1 = mn1;
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int n = 0; n < 8; ++n) {
          s[n][0] = fast_exp2(s[n][0] - ref0);
          s[n][1] = fast_exp2(s[n][1] - ref0);
          s[n][2] = fast_exp2(s[n][2] - ref1);
          s[n][3] = fast_exp2(s[n][3] - ref1);
          ps0 += s[n][0] + s[n][1];
          ps1 += s[n][2] + s[n][3];
        }
        l0 = l0 * c0 + ps0;
        l1 = l1 * c1 + ps1;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          o[n][0] *= c0;
          o[n][1] *= c0;
          o[n][2] *= c1;
          o[n][3] *= c1;
        }
        // ---- O += P V, P = hi + lo in bf16
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          uint32_t ph[4], pl[4];
          ph[0] = pack_bf16(s[2 * kp][0], s[2 * kp][1]);
          ph[1] = pack_bf16(s[2 * kp][2], s[2 * kp][3]);
          ph[2] = pack_bf16(s[2 * kp + 1][0], s[2 * kp + 1][1]);
          ph[3] = pack_bf16(s[2 * kp + 1][2], s[2 * kp + 1][3]);
          pl[0] = pack_bf16(s[2 * kp][0] - bf16_lo(ph[0]), s[2 * kp][1] - bf16_hi(ph[0]));
          pl[1] = pack_bf16(s[2 * kp][2] - bf16_lo(ph[1]), s[2 * kp][3] - bf16_hi(ph[1]));
          pl[2] = pack_bf16(s[2 * kp + 1][0] - bf16_lo(ph[2]), s[2 * kp + 1][1] - bf16_hi(ph[2]));
          pl[3] = pack_bf16(s[2 * kp + 1][2] - bf16_lo(ph[3]), s[2 * kp + 1][3] - bf16_hi(ph[3]));
#pragma unroll
          for (int dp = 0; dp < NT / 2; ++dp) {
            uint32_t r[4];
            ldsm_x4_t(r, vb + kp * 16 * PITCH + dp * 32 + v_lane);
            mma_bf16(o[2 * dp], ph, r[0], r[1]);
            mma_bf16(o[2 * dp + 1], ph, r[2], r[3]);
            mma_bf16(o[2 * dp], pl, r[0], r[1]);
            mma_bf16(o[2 * dp + 1], pl, r[2], r[3]);
          }
        }
      }
      __syncthreads();                               // stage i & 1 is free for tile i + 2
    }

    // ---- normalise and store the valid rows
    if (active) {
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, off);
        l1 += __shfl_xor_sync(kFull, l1, off);
      }
      const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
      float *out0 = a.out + ((long long)(qs + row0 + gq) * sh.Hq + qh) * D;
      float *out1 = a.out + ((long long)(qs + row0 + gq + 8) * sh.Hq + qh) * D;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int c = n * 8 + 2 * tq;
        if (gq < nrows) *reinterpret_cast<float2 *>(out0 + c) = make_float2(o[n][0] * inv0, o[n][1] * inv0);
        if (gq + 8 < nrows) *reinterpret_cast<float2 *>(out1 + c) = make_float2(o[n][2] * inv1, o[n][3] * inv1);
      }
    }
  }
}

template <int D>
cudaError_t launch_d(const PrefillArgs &a, const Shape &sh, const Tables &tb, int total_q, cudaStream_t st) {
  const size_t smem = 2 * stage_bytes<D>();
  static_assert(2 * stage_bytes<D>() <= 227 * 1024, "two stages fit in shared memory");
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // an upper bound on the query tiles: sum_b ceil(T_b / 16) <= total_q / 16 + batch
  const long long tiles = (long long)(total_q + kQT - 1) / kQT + a.batch;
  const dim3 grid((unsigned)tiles, (unsigned)(tb.n_ret + tb.n_loc));
  return launch_pdl(prefill_kernel<D>, grid, dim3(kThreads), smem, st, 0, a, sh, tb);
}

}  // namespace

cudaError_t launch_prefill(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                           const int32_t *page_table, const int32_t *seq_lens, const int32_t *q_starts, int batch,
                           int total_q, float *out, float attn_scale, int window, int num_sinks, const Shape &sh,
                           const Tables &tb, unsigned *err, cudaStream_t st) {
  if (batch == 0 || total_q == 0 || tb.n_ret + tb.n_loc == 0) return cudaSuccess;
  // d = 128 runs on the tcgen05 kernel (sd_prefill_tc.cu); this mma.sync one serves d = 64
  if (sh.d == 128)
    return launch_prefill_tc(q, k_cache, v_cache, page_table, seq_lens, q_starts, batch, total_q, out, attn_scale,
                             window, num_sinks, sh, tb, err, st);
  PrefillArgs a{q, k_cache, v_cache, page_table, seq_lens, q_starts, out, attn_scale, window, num_sinks, batch,
                total_q, err};
  return launch_d<64>(a, sh, tb, total_q, st);
}

}  // namespace sd
