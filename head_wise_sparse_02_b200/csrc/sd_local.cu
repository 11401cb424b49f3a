// Compacted caches of the local heads: each (sequence, local KV group) keeps
// only the rows it can ever attend to, the sinks and a ring of the window.
//
// RTPurbo page (gist.science/ar/paper/2605.16928), Methodology 1: local heads
// attend through a sliding window with attention sinks, so their K/V need not
// be kept for the whole context; AoH page (gist.science/ar/paper/2608.06849),
// Methodology 4: streaming heads keep sinks plus a recent window, and the
// saving is the KV memory of those heads.
//
//   slot(pos) = pos                          pos < num_sinks
//             = num_sinks + pos % window     otherwise (window > 0)
//
// Positions [N - window, N) of a sequence of length N occupy distinct ring
// slots, and no sink slot is shared with the ring, so once every position of
// the sequence has been appended in order the compacted rows are exactly the
// local set of a decode step at length N.
#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kThreads = 128;
constexpr int kWarpsPerCta = kThreads / 32;

// One warp per (token, local KV group): lanes [0, D/8) copy the key row, lanes
// [16, 16 + D/8) the value row, 16 bytes each.
template <int D>
__global__ void __launch_bounds__(kThreads)
local_append_kernel(const uint16_t *__restrict__ k_new, const uint16_t *__restrict__ v_new,
                    const int32_t *__restrict__ seq_ids, const int32_t *__restrict__ positions, int T,
                    uint16_t *__restrict__ local_k, uint16_t *__restrict__ local_v, int Hkv,
                    const Group *__restrict__ loc, int n_loc, int max_batch, long long max_len, int num_sinks,
                    int window, unsigned *err) {
  constexpr int CH = D / 8;                          // 16-byte chunks per row
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * kWarpsPerCta + (threadIdx.x >> 5);
  pdl_wait();
  pdl_trigger();
  if (w >= (long long)T * n_loc) return;
  const int t = (int)(w / n_loc), li = (int)(w % n_loc);
  const int seq = seq_ids[t];
  const int pos = positions[t];
  if (seq < 0 || seq >= max_batch || pos < 0 || pos >= max_len) {
    if (lane == 0 && li == 0) raise_error(err, SD_EBIT_SLOT);
    return;
  }
  const long long slot = local_slot(pos, num_sinks, window);
  if (slot < 0) return;                              // kept nowhere: no window
  const int g = loc[li].kv_head;
  const bool is_v = lane >= 16;
  const int c = lane & 15;
  if (c >= CH) return;
  const uint4 *src = reinterpret_cast<const uint4 *>((is_v ? v_new : k_new) + ((long long)t * Hkv + g) * D) + c;
  uint4 *dst = reinterpret_cast<uint4 *>((is_v ? local_v : local_k) +
                                         (((long long)seq * n_loc + li) * (num_sinks + window) + slot) * D) + c;
  *dst = __ldg(src);
}

}  // namespace

cudaError_t launch_local_append(const uint16_t *k_new, const uint16_t *v_new, const int32_t *seq_ids,
                                const int32_t *positions, int T, uint16_t *local_k, uint16_t *local_v,
                                const Shape &sh, const Tables &tb, int max_batch, int num_sinks, int window,
                                unsigned *err, cudaStream_t st) {
  const long long warps = (long long)T * tb.n_loc;
  if (warps == 0) return cudaSuccess;
  const dim3 grid((unsigned)((warps + kWarpsPerCta - 1) / kWarpsPerCta));
  if (sh.d == 128)
    return launch_pdl(local_append_kernel<128>, grid, dim3(kThreads), 0, st, 0, k_new, v_new, seq_ids, positions, T,
                      local_k, local_v, sh.Hkv, tb.loc, tb.n_loc, max_batch, sh.max_len, num_sinks, window, err);
  return launch_pdl(local_append_kernel<64>, grid, dim3(kThreads), 0, st, 0, k_new, v_new, seq_ids, positions, T,
                    local_k, local_v, sh.Hkv, tb.loc, tb.n_loc, max_batch, sh.max_len, num_sinks, window, err);
}

}  // namespace sd
