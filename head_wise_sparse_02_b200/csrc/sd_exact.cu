// Exact-score selection: retrieval heads scored by their true attention
// logits instead of the r = 16 index.
//
// ICS page (gist.science/ar/paper/2605.24168), 2: the study's reference
// selector ("Oracle Top-K") keeps the tokens with the highest exact attention
// scores; 3c: decode traffic then still reads every key once per step (the
// scores need the full keys), which is what the index avoids.
//
//   score_ws[(b * H_ret + row(h)) * L + t] = attn_scale * <q[b, h], k_t>,  t < N_b
//
// One CTA per (sequence, retrieval KV group, chunk of kChunk pages); four
// warps, each streaming its pages (16 keys of one KV head, d bf16 each, padded
// row pitch) through a cp.async ring and scoring them on the tensor cores:
// A = 16 keys x 16 dims by ldmatrix, B = the group's bf16 queries (exact, heads
// on N, eight per MMA), float32 accumulation.  The exact selector then finds
// each head's top-k / top-p threshold over the score rows.
#include <algorithm>

#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 64;              // pages per CTA
constexpr int kRing = 4;                // pages in flight per warp

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes), "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d = a * b (fresh accumulator), bf16 inputs, float32 accumulate
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__host__ __device__ constexpr size_t ring_bytes() {
  return (size_t)kWarps * kRing * kPage * (2 * D + 16);
}

// HB: head blocks of eight heads (ceil(GR / 8)).
template <int D, int HB>
__global__ void __launch_bounds__(kThreads)
exact_score_kernel(const SelectArgs a, const Shape sh, const Group *__restrict__ groups, int n_groups,
                   const uint16_t *__restrict__ q, const uint16_t *__restrict__ k_cache, float attn_scale) {
  constexpr int KS = D / 16;                         // k-steps over the head dimension
  constexpr int kRowB = 2 * D;                       // bytes of one key
  constexpr int kPitch = kRowB + 16;                 // bytes of one key in shared memory
  constexpr int kPageB = kPage * kPitch;
  constexpr int CPL = kPage * kRowB / 16 / 32;       // 16-byte chunks per lane and page
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int item = blockIdx.x;
  const int b = item / n_groups, gi = item % n_groups;
  extern __shared__ __align__(128) unsigned char dyn[];
  __shared__ Group grp;
  __shared__ int32_t pt_s[kChunk];
  if (tid == 0) grp = groups[gi];
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int nr = grp.n, g = grp.kv_head;
  long long N = a.seq_lens[b];
  N = N < 0 ? 0 : std::min<long long>(N, sh.max_len);
  const int pages = (int)((N + kPage - 1) / kPage);
  const int p0 = blockIdx.y * kChunk;
  if (p0 >= pages) return;
  const int np = pages - p0 < kChunk ? pages - p0 : kChunk;
  {
    const int32_t *pt = a.page_table + (long long)b * sh.max_pages + p0;
    for (int o = tid; o < np; o += kThreads) {
      const int page = pt[o];
      const bool ok = page >= 0 && page < sh.num_pages;
      pt_s[o] = ok ? page : -1;
      if (!ok) raise_error(a.err, SD_EBIT_PAGE);
    }
  }
  __syncthreads();

  // B fragments: column n = gq carries head 8 hb + gq, rows k = the dims
  uint32_t bq[HB][KS][2];
#pragma unroll
  for (int hb = 0; hb < HB; ++hb) {
    const int h = hb * 8 + gq;
    const uint16_t *qr = h < nr ? q + ((long long)b * sh.Hq + grp.q_head[h]) * D : nullptr;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      bq[hb][kk][0] = qr ? *reinterpret_cast<const uint32_t *>(qr + kk * 16 + 2 * tq) : 0u;
      bq[hb][kk][1] = qr ? *reinterpret_cast<const uint32_t *>(qr + kk * 16 + 2 * tq + 8) : 0u;
    }
  }
  float *srow[HB][2];                                // score rows of heads 8 hb + 2 tq (+1)
#pragma unroll
  for (int hb = 0; hb < HB; ++hb)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int h = hb * 8 + 2 * tq + c;
      srow[hb][c] = h < nr ? a.score_ws + ((long long)b * sh.H_ret + grp.row[h]) * sh.max_len : nullptr;
    }

  // per-warp ring: this warp scores pages warp, warp + 4, ... of the chunk
  const uint32_t ring = (uint32_t)__cvta_generic_to_shared(dyn) + warp * (kRing * kPageB);
  const unsigned char *kb = reinterpret_cast<const unsigned char *>(k_cache);
  const uint64_t l2_stream = evict_first_policy();
  const int nq = np > warp ? (np - warp + kWarps - 1) / kWarps : 0;
  auto issue = [&](int i) {
    if (i < nq) {
      const int page = pt_s[warp + i * kWarps];
      const unsigned char *src = kb + ((size_t)(page >= 0 ? page : 0) * sh.Hkv + g) * (kPage * kRowB);
#pragma unroll
      for (int j = 0; j < CPL; ++j) {
        const int c = lane + 32 * j;                 // 16-byte chunk of the page
        const int r = c / (kRowB / 16), x = c % (kRowB / 16);
        cp_async16(ring + (i % kRing) * kPageB + r * kPitch + x * 16, src + r * kRowB + x * 16, page >= 0 ? 16 : 0,
                   l2_stream);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < kRing - 1; ++i) issue(i);
  // ldmatrix rows: lanes 0-7 / 8-15 keys 0-7 / 8-15 (dims 0-7), lanes 16-31 the same keys (dims 8-15)
  const uint32_t ld = (uint32_t)(((lane & 7) + ((lane >> 3) & 1) * 8) * kPitch + (lane >> 4) * 16);
  for (int i = 0; i < nq; ++i) {
    issue(i + kRing - 1);
    cp_async_wait<kRing - 1>();
    __syncwarp();
    const uint32_t tile = ring + (i % kRing) * kPageB + ld;
    float acc[HB][4];
#pragma unroll
    for (int hb = 0; hb < HB; ++hb) acc[hb][0] = acc[hb][1] = acc[hb][2] = acc[hb][3] = 0.0f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t af[4];
      ldsm_x4(af, tile + kk * 32);
#pragma unroll
      for (int hb = 0; hb < HB; ++hb) mma_bf16(acc[hb], af, bq[hb][kk][0], bq[hb][kk][1]);
    }
    __syncwarp();                                    // the slot is free for the copy issued next
    const int pl = warp + i * kWarps;
    const bool ok = pt_s[pl] >= 0;
    const long long t0 = (long long)(p0 + pl) * kPage;
#pragma unroll
    for (int hb = 0; hb < HB; ++hb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float *dst = srow[hb][e & 1];
        const long long t = t0 + gq + 8 * (e >> 1);
        if (dst && t < N) dst[t] = ok ? acc[hb][e] * attn_scale : -INFINITY;
      }
  }
  cp_async_wait<0>();
}

template <int D>
cudaError_t launch_d(const SelectArgs &a, const Shape &sh, const Tables &tb, const uint16_t *q, const uint16_t *k_cache,
                     float attn_scale, cudaStream_t st) {
  static_assert(ring_bytes<D>() <= 227 * 1024, "ring fits in shared memory");
  const dim3 grid(a.batch * tb.n_ret, (unsigned)((sh.max_pages + kChunk - 1) / kChunk));
  const size_t smem = ring_bytes<D>();
  cudaError_t e;
  if (tb.max_ret <= 8) {
    e = cudaFuncSetAttribute(exact_score_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(exact_score_kernel<D, 1>, grid, dim3(kThreads), smem, st, 0, a, sh, tb.ret, tb.n_ret, q, k_cache,
                      attn_scale);
  }
  e = cudaFuncSetAttribute(exact_score_kernel<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(exact_score_kernel<D, 2>, grid, dim3(kThreads), smem, st, 0, a, sh, tb.ret, tb.n_ret, q, k_cache,
                    attn_scale);
}

}  // namespace

cudaError_t launch_exact_scores(const SelectArgs &a, const Shape &sh, const Tables &tb, const uint16_t *q,
                                const uint16_t *k_cache, float attn_scale, cudaStream_t st) {
  if (tb.n_ret == 0 || a.batch == 0) return cudaSuccess;
  return sh.d == 128 ? launch_d<128>(a, sh, tb, q, k_cache, attn_scale, st)
                     : launch_d<64>(a, sh, tb, q, k_cache, attn_scale, st);
}

}  // namespace sd
