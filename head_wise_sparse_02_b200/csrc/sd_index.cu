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
  __shared__ double Ps[D][kIndexDim];
  __shared__ double Ks[kRows][D + 1];
  const int g = blockIdx.y;
  const int t0 = blockIdx.x * kRows;
  const uint16_t *P = proj + (size_t)g * D * kIndexDim;
  for (int i = threadIdx.x; i < D * kIndexDim; i += kThreads)
    Ps[i / kIndexDim][i % kIndexDim] = (double)bf16_to_f32(P[i]);    // the context's own copy
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < kRows * D; i += kThreads) {
    const int row = i / D, c = i % D, t = t0 + row;
    Ks[row][c] = (t < T) ? (double)bf16_to_f32(k_pre[((size_t)t * Hkv + g) * D + c]) : 0.0;
  }
  __syncthreads();
  const int row = threadIdx.x / kIndexDim, j = threadIdx.x % kIndexDim;
  const int t = t0 + row;
  if (t >= T) return;
  // four interleaved partial sums (shorter dependent chains), added at the end
  double acc4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 8
  for (int i = 0; i < D; i += 4)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc4[u] = fma(Ks[row][i + u], Ps[i + u][j], acc4[u]);
  const double acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
  const long long slot = slots[t];
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
