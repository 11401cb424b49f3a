// Index keys: k~ = bf16_rne(P_g^T k_pre) for newly cached tokens.
//
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 2: retrieval
// heads estimate relevance in an r = 16 dimensional space obtained by
// projecting pre-RoPE keys (and queries).  The index entry of a token is the
// projection of its key, stored as bf16 (32 bytes per token and KV head).
//
// Accumulation is float64: every product of two bf16 values is exact in
// float64 and the running sum is rounded at 2^-53, so the single final
// rounding to bf16 (round to nearest even, from the float64 value) agrees with
// rounding the exact dot product except when that exact value lies within
// ~2^-45 relative of a bf16 rounding midpoint.
#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kRows = 16;          // (token) rows per block, one KV head per block
constexpr int kThreads = kRows * kIndexDim;

template <int D>
__global__ void __launch_bounds__(kThreads)
index_keys_kernel(const uint16_t *__restrict__ k_pre, const int32_t *__restrict__ slots, int T,
                  uint16_t *__restrict__ index_cache, const uint16_t *__restrict__ proj, int Hkv,
                  int num_pages, unsigned *err) {
  static_assert(D % 8 == 0, "whole 16-byte loads");
  __shared__ double Ps[D][kIndexDim];
  __shared__ double Ks[kRows][D + 1];
  const int g = blockIdx.y;
  const int t0 = blockIdx.x * kRows;
  const int tid = threadIdx.x;
  // the projection is the context's own copy: loaded before waiting for the
  // previous kernel on the stream
  const uint4 *P = reinterpret_cast<const uint4 *>(proj + (size_t)g * D * kIndexDim);
#pragma unroll
  for (int i = tid; i < D * kIndexDim / 8; i += kThreads) {
    const uint4 v = __ldg(P + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = i * 8 + 2 * j;
      Ps[e / kIndexDim][e % kIndexDim] = (double)bf16_lo(w[j]);
      Ps[(e + 1) / kIndexDim][(e + 1) % kIndexDim] = (double)bf16_hi(w[j]);
    }
  }
  pdl_wait();
  pdl_trigger();
  const int row = tid / kIndexDim, j = tid % kIndexDim;
  const int t = t0 + row;
  const long long slot = t < T ? (long long)slots[t] : -1;     // issued with the key loads
#pragma unroll
  for (int i = tid; i < kRows * D / 8; i += kThreads) {
    const int r = i / (D / 8), c = (i % (D / 8)) * 8, tr = t0 + r;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (tr < T) v = *reinterpret_cast<const uint4 *>(k_pre + ((size_t)tr * Hkv + g) * D + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      Ks[r][c + 2 * q] = (double)bf16_lo(w[q]);
      Ks[r][c + 2 * q + 1] = (double)bf16_hi(w[q]);
    }
  }
  __syncthreads();
  if (t >= T) return;
  // four interleaved partial sums (shorter dependent chains), added at the end
  double acc4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 8
  for (int i = 0; i < D; i += 4)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc4[u] = fma(Ks[row][i + u], Ps[i + u][j], acc4[u]);
  const double acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
  if (slot < 0 || slot >= (long long)num_pages * kPage) {
    if (j == 0) raise_error(err, SD_EBIT_SLOT);
    return;
  }
  const long long page = slot / kPage, off = slot % kPage;
  index_cache[((page * Hkv + g) * kPage + off) * kIndexDim + j] = f64_to_bf16_rne(acc);
}

}  // namespace

cudaError_t launch_index_keys(const uint16_t *k_pre, const int32_t *slots, int T, uint16_t *index_cache,
                              const uint16_t *proj, const Shape &sh, unsigned *err, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  dim3 grid((T + kRows - 1) / kRows, sh.Hkv);
  if (sh.d == 128)
    return launch_pdl(index_keys_kernel<128>, grid, dim3(kThreads), 0, st, 0, k_pre, slots, T, index_cache, proj,
                      sh.Hkv, sh.num_pages, err);
  return launch_pdl(index_keys_kernel<64>, grid, dim3(kThreads), 0, st, 0, k_pre, slots, T, index_cache, proj,
                    sh.Hkv, sh.num_pages, err);
}

}  // namespace sd
