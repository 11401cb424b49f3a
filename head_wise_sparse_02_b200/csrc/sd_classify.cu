// Data-free head classifier: the effective rank of every query head's kernel
// attention operator, from the frozen query and key projections alone.
//
// AoH page (gist.science/ar/paper/2608.06849), Methodology 1-3: head h's
// operator is M_h = W_K^T W_Q (d_model x d_model); its effective rank is the
// exponential of the Shannon entropy of its normalised nonzero singular
// values; those singular values follow from the d_head x d_head Gram matrices
// W_Q W_Q^T and W_K W_K^T (the page's C_h is their product).
//
// The singular values are taken here without forming C_h (a non-symmetric
// product whose small eigenvalues carry only sqrt(eps) relative accuracy
// after the square root): with the Gram matrices factored as
// W_Q W_Q^T = L_q L_q^T and W_K W_K^T = L_k L_k^T (lower triangular; W^T = U L^T
// is a thin QR of W^T), M_h = U_k (L_k^T L_q) U_q^T, so the nonzero singular
// values of M_h are those of the d_head x d_head matrix X = L_k^T L_q, and
// X X^T is similar to C_h.  One-sided (Hestenes) Jacobi rotations
// orthogonalise the columns of X; the singular values are the column norms.
//
//   gram_kernel      G = W W^T of each d_head-row block (a query head or a KV
//                    head of one layer), float64 sums of exact bf16 products
//   cholesky_kernel  G = L L^T in place, a pivot at or below
//                    d_head * eps * max diag G zeroes its column (rank-deficient
//                    blocks factor as semi-definite)
//   jacobi_kernel    X = L_k^T L_q in shared memory, parallel cyclic Jacobi
//                    sweeps (round-robin pairings; each warp takes several
//                    column pairs of a round, their reductions interleaved),
//                    then ER from the column norms
//
// Everything is float64: this runs once per model, and its output is a
// ranking.
#include <float.h>

#include <algorithm>
#include <vector>

#include "head_classifier.h"
#include "sd_internal.cuh"

namespace sd {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 64;          // Gram output tile (rows x columns)
constexpr int kChunk = 32;         // d_model columns staged per step
constexpr int kMaxSweeps = 60;     // Jacobi sweeps before a head is reported as not converged
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ double bf16_bits_to_f64(uint32_t bits) { return (double)__uint_as_float(bits << 16); }

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

// Pointer to the d_head x d_model block of matrix `mat` = layer * (Hq + Hkv) + idx:
// query head idx (< Hq) or KV head idx - Hq of that layer.
__device__ __forceinline__ const uint16_t *block_of(const uint16_t *w_q, const uint16_t *w_k, int mat, int Hq, int Hkv,
                                                    int D, int d_model) {
  const int layer = mat / (Hq + Hkv), idx = mat % (Hq + Hkv);
  return idx < Hq ? w_q + ((long long)layer * Hq + idx) * D * d_model
                  : w_k + ((long long)layer * Hkv + (idx - Hq)) * D * d_model;
}

// One 64 x 64 tile (bi, bj), bi <= bj, of G = W W^T for one block W.  Thread
// (ty, tx) owns rows ty + 8 a and columns tx + 8 c (a, c < 8): 16 shared-memory
// loads per 64 FMAs.
constexpr int kGramThreads = 64;

template <int D>
__global__ void __launch_bounds__(kGramThreads)
gram_kernel(const uint16_t *__restrict__ w_q, const uint16_t *__restrict__ w_k, int d_model, int Hq, int Hkv,
            double *__restrict__ gram) {
  constexpr int NB = D / kTile;
  __shared__ double As[kChunk][kTile + 1];
  __shared__ double Bs[kChunk][kTile + 1];
  const int tid = threadIdx.x, ty = tid / 8, tx = tid % 8;
  int bi = 0, bj = blockIdx.x;                     // tile index -> (bi, bj) with bi <= bj
  while (bj >= NB - bi) {
    bj -= NB - bi;
    ++bi;
  }
  bj += bi;
  const int mat = blockIdx.y;
  pdl_wait();
  pdl_trigger();
  const uint16_t *W = block_of(w_q, w_k, mat, Hq, Hkv, D, d_model);
  const uint16_t *wa = W + (long long)(bi * kTile) * d_model;
  const uint16_t *wb = W + (long long)(bj * kTile) * d_model;
  double acc[8][8] = {};
  for (int k0 = 0; k0 < d_model; k0 += kChunk) {
    // staging: 64 rows x 32 columns of each block = 256 16-byte pieces, 4 per thread
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int piece = tid + kGramThreads * x;
      const int lr = piece / 4, lk = (piece % 4) * 8;
      const uint4 va = *reinterpret_cast<const uint4 *>(wa + (long long)lr * d_model + k0 + lk);
      const uint4 vb = *reinterpret_cast<const uint4 *>(wb + (long long)lr * d_model + k0 + lk);
      const uint32_t ua[4] = {va.x, va.y, va.z, va.w}, ub[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        As[lk + 2 * e][lr] = bf16_bits_to_f64(ua[e] & 0xFFFFu);
        As[lk + 2 * e + 1][lr] = bf16_bits_to_f64(ua[e] >> 16);
        Bs[lk + 2 * e][lr] = bf16_bits_to_f64(ub[e] & 0xFFFFu);
        Bs[lk + 2 * e + 1][lr] = bf16_bits_to_f64(ub[e] >> 16);
      }
    }
    __syncthreads();
#pragma unroll 2
    for (int k = 0; k < kChunk; ++k) {
      double a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        a[i] = As[k][ty + 8 * i];
        b[i] = Bs[k][tx + 8 * i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  double *G = gram + (size_t)mat * D * D;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = bi * kTile + ty + 8 * i, c = bj * kTile + tx + 8 * j;
      G[(size_t)r * D + c] = acc[i][j];
      if (bi != bj) G[(size_t)c * D + r] = acc[i][j];
    }
}

// G = L L^T in place (right-looking, column by column), one CTA per matrix,
// the lower triangle packed in shared memory (row i at i (i + 1) / 2: 66 KB at
// d_head 128, three CTAs per SM); writes L with zeros above the diagonal.
template <int D>
__host__ __device__ constexpr size_t chol_smem() {
  return (size_t)D * (D + 1) / 2 * sizeof(double);
}

template <int D>
__global__ void __launch_bounds__(kThreads) cholesky_kernel(double *__restrict__ gram) {
  extern __shared__ __align__(16) double a[];        // packed lower triangle
  __shared__ double s_tol;
  const int tid = threadIdx.x, lane = tid & 31, ty = tid / 16, tx = tid % 16;
  auto at = [&](int i, int j) -> double & { return a[i * (i + 1) / 2 + j]; };
  pdl_wait();
  pdl_trigger();
  double *G = gram + (size_t)blockIdx.x * D * D;
  for (int i = tid / 32; i < D; i += kThreads / 32)
    for (int j = lane; j <= i; j += 32) at(i, j) = G[i * D + j];
  __syncthreads();
  if (tid < 32) {
    double m = 0.0;
    for (int i = lane; i < D; i += 32) m = fmax(m, at(i, i));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(kFull, m, o));
    if (lane == 0) s_tol = m * D * DBL_EPSILON;
  }
  __syncthreads();
  const double tol = s_tol;
  for (int k = 0; k < D; ++k) {
    const double piv = at(k, k);
    const double lkk = piv > tol ? sqrt(piv) : 0.0;
    const double inv = lkk > 0.0 ? 1.0 / lkk : 0.0;
    __syncthreads();                                 // every thread has the pivot before column k changes
    for (int i = k + 1 + tid; i < D; i += kThreads) at(i, k) *= inv;
    if (tid == 0) at(k, k) = lkk;
    __syncthreads();
    for (int i = k + 1 + ty; i < D; i += 16) {       // trailing lower triangle: a_ij -= l_ik l_jk, k < j <= i
      const double lik = at(i, k);
      double *row = a + i * (i + 1) / 2;
      for (int j = k + 1 + tx; j <= i; j += 16) row[j] -= lik * at(j, k);
    }
    __syncthreads();
  }
  for (int i = tid / 32; i < D; i += kThreads / 32)
    for (int j = lane; j < D; j += 32) G[i * D + j] = j <= i ? at(i, j) : 0.0;
}

// Rotation of a column pair (alpha = |x_p|^2, beta = |x_q|^2, gamma = x_p.x_q)
// that makes the pair orthogonal: tan = t, the root of t^2 + 2 zeta t - 1 = 0
// of smaller magnitude, zeta = (beta - alpha) / (2 gamma) (Rutishauser's
// form).  t is taken in float32 (fast reciprocal and root): an angle off by
// ~1e-7 relative only leaves a residual gamma ~1e-7 times the old one for a
// later sweep.  cos = (1 + t^2)^(-1/2) must keep cos^2 + sin^2 = 1 to float64
// rounding (the rotations must preserve the column norms), so it starts from
// the float32 reciprocal square root and takes two Newton steps in float64,
// y <- y (3 - x y^2) / 2, each squaring the relative error (1e-7 -> 1e-14 ->
// below double rounding).  Returns cos; *t gets the tangent.
__device__ __forceinline__ double rot_cos(double alpha, double beta, double gamma, double &t) {
  const float den = 2.0f * (float)gamma;
  float tf = 0.0f;                                   // gamma below float range: no rotation
  if (den != 0.0f) {
    const float zeta = (float)(beta - alpha) / den;
    const float az = fabsf(zeta);
    tf = (zeta >= 0.0f ? 1.0f : -1.0f) / (az + sqrtf(fmaf(az, az, 1.0f)));   // 0 when zeta^2 overflows
  }
  t = (double)tf;
  const double x = fma(t, t, 1.0);
  double y = (double)rsqrtf((float)x);
  y = y * fma(-0.5 * x * y, y, 1.5);
  y = y * fma(-0.5 * x * y, y, 1.5);
  return y;
}

template <int D>
__host__ __device__ constexpr size_t jacobi_smem() {
  return (size_t)D * D * sizeof(double) + 2 * (size_t)16 * D * sizeof(double);
}

// One CTA per (layer, query head): X = L_k^T L_q, one-sided Jacobi, ER.
// threads of the Jacobi kernel: 4 column pairs per warp and round
template <int D>
__host__ __device__ constexpr int jacobi_threads() {
  return D / 2 / 4 * 32;
}

template <int D>
__global__ void __launch_bounds__(jacobi_threads<D>(), 1)
jacobi_kernel(const double *__restrict__ gram, int Hq, int Hkv, double *__restrict__ eff_rank) {
  constexpr int kJThreads = jacobi_threads<D>();
  constexpr int kWarps = kJThreads / 32;
  constexpr int TR = D / (kJThreads / 16), TC = D / 16;   // rows, columns of X per thread (register tile)
  static_assert(TR >= 1 && D % (kJThreads / 16) == 0, "X tile");
  extern __shared__ __align__(16) double smem[];
  double *Xc = smem;                                 // X column-major: Xc[j * D + i] = X_ij
  double *sk = smem + D * D;                         // 16 staged rows of L_k
  double *sq = sk + 16 * D;                          // 16 staged rows of L_q
  __shared__ double sig[D];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, ty = tid / 16, tx = tid % 16;
  const int layer = blockIdx.x / Hq, h = blockIdx.x % Hq, g = h / (Hq / Hkv);
  pdl_wait();
  pdl_trigger();
  const double *Lq = gram + ((size_t)layer * (Hq + Hkv) + h) * D * D;
  const double *Lk = gram + ((size_t)layer * (Hq + Hkv) + Hq + g) * D * D;

  // ---- X_ij = sum_k Lk[k][i] Lq[k][j]: rows i = ty + (threads / 16) a,
  // columns j = tx + 16 c
  {
    constexpr int RS = kJThreads / 16;               // row stride of a thread's tile
    double acc[TR][TC] = {};
    for (int k0 = 0; k0 < D; k0 += 16) {
      for (int x = tid; x < 16 * D; x += kJThreads) {
        sk[x] = Lk[(size_t)k0 * D + x];
        sq[x] = Lq[(size_t)k0 * D + x];
      }
      __syncthreads();
#pragma unroll 2
      for (int k = 0; k < 16; ++k) {
        double u[TR], v[TC];
#pragma unroll
        for (int t = 0; t < TR; ++t) u[t] = sk[k * D + ty + RS * t];
#pragma unroll
        for (int t = 0; t < TC; ++t) v[t] = sq[k * D + tx + 16 * t];
#pragma unroll
        for (int a = 0; a < TR; ++a)
#pragma unroll
          for (int c = 0; c < TC; ++c) acc[a][c] = fma(u[a], v[c], acc[a][c]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < TR; ++a)
#pragma unroll
      for (int c = 0; c < TC; ++c) Xc[(tx + 16 * c) * D + ty + RS * a] = acc[a][c];
  }
  __syncthreads();

  // ---- one-sided Jacobi: rotate column pairs until every pair is orthogonal
  // to D * eps relative; round r pairs (r, D-1) and ((r+m) mod (D-1),
  // (r-m) mod (D-1)) for m = 1 .. D/2-1, every pair once per sweep
  // Warp w takes pairs m = w * PPW .. w * PPW + PPW - 1 of each round, all at
  // once: their partial sums, reductions and rotations interleave, so the
  // shuffle latency of one pair hides behind the others'.
  constexpr int PPW = D / 2 / kWarps;                // pairs per warp and round
  static_assert(PPW % 4 == 0, "the pair sums are split over the four quarters of a warp");
  constexpr int RPL = D / 32;                        // rows per lane
  const double tol2 = (D * DBL_EPSILON) * (D * DBL_EPSILON);
  bool converged = false;
  for (int sweep = 0; sweep < kMaxSweeps && !converged; ++sweep) {
    int rotated = 0;
    for (int r = 0; r < D - 1; ++r) {
      double al[PPW], be[PPW], ga[PPW];
      double xu[PPW][RPL], xv[PPW][RPL];             // this lane's rows of the pairs' columns, read once
      int cp[PPW], cq[PPW];
#pragma unroll
      for (int j = 0; j < PPW; ++j) {
        const int m = warp * PPW + j;
        cp[j] = m == 0 ? D - 1 : (r + m) % (D - 1);
        cq[j] = m == 0 ? r : (r - m + (D - 1)) % (D - 1);
        al[j] = be[j] = ga[j] = 0.0;
#pragma unroll
        for (int e = 0; e < RPL; ++e) {
          const double u = Xc[cp[j] * D + lane + 32 * e], v = Xc[cq[j] * D + lane + 32 * e];
          xu[j][e] = u;
          xv[j][e] = v;
          al[j] = fma(u, u, al[j]);
          be[j] = fma(v, v, be[j]);
          ga[j] = fma(u, v, ga[j]);
        }
      }
      // The pairs' sums (al, be, ga) over the warp, reduce-scatter style: two
      // halving exchanges leave each quarter of the warp (lane bits 4 and 3)
      // with the partial sums of NP of the pairs, a butterfly over those lanes
      // completes them, the quarter computes their rotations, and three
      // exchanges give every lane the rotations of all PPW pairs.
      constexpr int NV = 3 * PPW, NP = PPW / 4;
      const int b4 = (lane >> 4) & 1, b3 = (lane >> 3) & 1;
      double w1[NV / 2], w2[NV / 4];
#pragma unroll
      for (int k = 0; k < NV / 2; ++k) {             // lanes 0-15 keep pairs 0 .. PPW/2-1, lanes 16-31 the rest
        const int lo = k, hi = NV / 2 + k;
        const double vlo = lo % 3 == 0 ? al[lo / 3] : (lo % 3 == 1 ? be[lo / 3] : ga[lo / 3]);
        const double vhi = hi % 3 == 0 ? al[hi / 3] : (hi % 3 == 1 ? be[hi / 3] : ga[hi / 3]);
        w1[k] = (b4 ? vhi : vlo) + __shfl_xor_sync(kFull, b4 ? vlo : vhi, 16);
      }
#pragma unroll
      for (int k = 0; k < NV / 4; ++k) {             // then lane bit 3 halves the kept pairs again
        const double vlo = w1[k], vhi = w1[NV / 4 + k];
        w2[k] = (b3 ? vhi : vlo) + __shfl_xor_sync(kFull, b3 ? vlo : vhi, 8);
      }
#pragma unroll
      for (int o = 4; o > 0; o >>= 1)
#pragma unroll
        for (int k = 0; k < NV / 4; ++k) w2[k] += __shfl_xor_sync(kFull, w2[k], o);
      // this quarter's pairs G4 * PPW/2 + G3 * NP + p (G4 = b4, G3 = b3): c, s
      // (s = 0: no rotation; a rotating pair has |t| > 0, so s != 0)
      double cg[NP], sg[NP];
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        const double A = w2[3 * q], Bv = w2[3 * q + 1], Gv = w2[3 * q + 2];
        cg[q] = 1.0;
        sg[q] = 0.0;
        if (Gv * Gv > tol2 * (A * Bv)) {             // |gamma| > tol sqrt(alpha beta), without the root
          double t;
          cg[q] = rot_cos(A, Bv, Gv, t);
          sg[q] = cg[q] * t;
          rotated = 1;
        }
      }
      double c8[NP], s8[NP], c16[NP], s16[NP], c24[NP], s24[NP];
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        c8[q] = __shfl_xor_sync(kFull, cg[q], 8);
        s8[q] = __shfl_xor_sync(kFull, sg[q], 8);
        c16[q] = __shfl_xor_sync(kFull, cg[q], 16);
        s16[q] = __shfl_xor_sync(kFull, sg[q], 16);
        c24[q] = __shfl_xor_sync(kFull, cg[q], 24);
        s24[q] = __shfl_xor_sync(kFull, sg[q], 24);
      }
#pragma unroll
      for (int j = 0; j < PPW; ++j) {
        const int G4 = j / (PPW / 2), G3 = (j / NP) & 1, q = j % NP;
        const bool f4 = G4 != b4, f3 = G3 != b3;
        const double c = f4 ? (f3 ? c24[q] : c16[q]) : (f3 ? c8[q] : cg[q]);
        const double sn = f4 ? (f3 ? s24[q] : s16[q]) : (f3 ? s8[q] : sg[q]);
        if (sn != 0.0) {
#pragma unroll
          for (int e = 0; e < RPL; ++e) {
            const double u = xu[j][e], v = xv[j][e];
            Xc[cp[j] * D + lane + 32 * e] = c * u - sn * v;
            Xc[cq[j] * D + lane + 32 * e] = sn * u + c * v;
          }
        }
      }
      __syncthreads();
    }
    converged = __syncthreads_or(rotated) == 0;
  }

  // ---- singular values (column norms) and the effective rank
  for (int j = warp; j < D; j += kWarps) {
    double s2 = 0.0;
#pragma unroll
    for (int i = lane; i < D; i += 32) s2 = fma(Xc[j * D + i], Xc[j * D + i], s2);
    s2 = warp_sum(s2);
    if (lane == 0) sig[j] = sqrt(s2);
  }
  __syncthreads();
  if (warp == 0) {
    double mx = 0.0;
    for (int j = lane; j < D; j += 32) mx = fmax(mx, sig[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(kFull, mx, o));
    const double cut = mx * D * DBL_EPSILON;       // nonzero singular values: above the numerical-rank threshold
    double total = 0.0;
    for (int j = lane; j < D; j += 32) total += sig[j] > cut ? sig[j] : 0.0;
    total = warp_sum(total);
    double ent = 0.0;
    if (total > 0.0)
      for (int j = lane; j < D; j += 32)
        if (sig[j] > cut) {
          const double p = sig[j] / total;
          ent -= p * log(p);
        }
    ent = warp_sum(ent);
    if (lane == 0) eff_rank[blockIdx.x] = converged ? exp(ent) : __longlong_as_double(0x7ff8000000000000LL);
  }
}

template <int D>
cudaError_t launch_er_d(const uint16_t *w_q, const uint16_t *w_k, int L, int d_model, int Hq, int Hkv, double *er,
                        double *gram, cudaStream_t st) {
  constexpr int NB = D / kTile;
  const int mats = L * (Hq + Hkv);
  cudaError_t e = launch_pdl(gram_kernel<D>, dim3(NB * (NB + 1) / 2, mats), dim3(kGramThreads), 0, st, 0, w_q, w_k,
                             d_model, Hq, Hkv, gram);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(cholesky_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)chol_smem<D>());
  if (e != cudaSuccess) return e;
  e = launch_pdl(cholesky_kernel<D>, dim3(mats), dim3(kThreads), chol_smem<D>(), st, 0, gram);
  if (e != cudaSuccess) return e;
  static_assert(jacobi_smem<D>() + D * sizeof(double) <= 227 * 1024, "Jacobi tile fits in shared memory");
  e = cudaFuncSetAttribute(jacobi_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)jacobi_smem<D>());
  if (e != cudaSuccess) return e;
  return launch_pdl(jacobi_kernel<D>, dim3(L * Hq), dim3(jacobi_threads<D>()), jacobi_smem<D>(), st, 0,
                    (const double *)gram, Hq, Hkv, er);
}

}  // namespace

size_t head_er_workspace_bytes(int L, int Hq, int Hkv, int D) {
  return (size_t)L * (Hq + Hkv) * D * D * sizeof(double);
}

cudaError_t launch_head_effective_rank(const uint16_t *w_q, const uint16_t *w_k, int L, int d_model, int Hq, int Hkv,
                                       int D, double *er, void *ws, cudaStream_t st) {
  double *gram = static_cast<double *>(ws);
  return D == 128 ? launch_er_d<128>(w_q, w_k, L, d_model, Hq, Hkv, er, gram, st)
                  : launch_er_d<64>(w_q, w_k, L, d_model, Hq, Hkv, er, gram, st);
}

}  // namespace sd

extern "C" {

sd_status sparse_decode_head_er_workspace_size(int num_layers, int num_q_heads, int num_kv_heads, int head_dim,
                                               size_t *bytes) {
  if (!bytes || num_layers < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return SD_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SD_ERR_UNSUPPORTED;
  *bytes = sd::head_er_workspace_bytes(num_layers, num_q_heads, num_kv_heads, head_dim);
  return SD_OK;
}

sd_status sparse_decode_head_effective_rank(const void *w_q, const void *w_k, int num_layers, int d_model,
                                            int num_q_heads, int num_kv_heads, int head_dim, double *eff_rank,
                                            void *workspace, size_t ws_bytes, sd_stream stream) {
  if (num_layers < 0 || d_model <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return SD_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SD_ERR_UNSUPPORTED;
  if (d_model % 32 != 0) return SD_ERR_UNSUPPORTED;
  if (num_layers == 0) return SD_OK;
  if ((long long)num_layers * (num_q_heads + num_kv_heads) > 65535LL * 1024) return SD_ERR_UNSUPPORTED;
  if (!w_q || !w_k || !eff_rank) return SD_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(w_q) & 15u) || (reinterpret_cast<uintptr_t>(w_k) & 15u)) return SD_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < sd::head_er_workspace_bytes(num_layers, num_q_heads, num_kv_heads, head_dim))
    return SD_ERR_WORKSPACE;
  const cudaError_t e = sd::launch_head_effective_rank(
      static_cast<const uint16_t *>(w_q), static_cast<const uint16_t *>(w_k), num_layers, d_model, num_q_heads,
      num_kv_heads, head_dim, eff_rank, workspace, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SD_OK : SD_ERR_CUDA;
}

sd_status sparse_decode_classify_heads(const double *eff_rank, int num_q_heads, int num_kv_heads,
                                       int num_retrieval_groups, int32_t *head_is_retrieval) {
  try {
    if (!eff_rank || !head_is_retrieval || num_q_heads <= 0 || num_kv_heads <= 0 ||
        num_q_heads % num_kv_heads != 0 || num_retrieval_groups < 0 || num_retrieval_groups > num_kv_heads)
      return SD_ERR_INVALID_ARG;
    const int G = num_q_heads / num_kv_heads;
    std::vector<double> pooled(num_kv_heads);
    for (int g = 0; g < num_kv_heads; ++g) {
      double total = 0.0;
      for (int h = g * G; h < (g + 1) * G; ++h) total += eff_rank[h];
      pooled[g] = total / G;
    }
    std::vector<int> order(num_kv_heads);
    for (int g = 0; g < num_kv_heads; ++g) order[g] = g;
    std::stable_sort(order.begin(), order.end(), [&](int x, int y) {
      const bool nx = pooled[x] != pooled[x], ny = pooled[y] != pooled[y];
      if (nx != ny) return ny;                       // numbers before NaN
      return !nx && pooled[x] < pooled[y];
    });
    std::vector<char> chosen(num_kv_heads, 0);
    for (int i = 0; i < num_retrieval_groups; ++i) chosen[order[i]] = 1;
    for (int h = 0; h < num_q_heads; ++h) head_is_retrieval[h] = chosen[h / G] ? 1 : 0;
    return SD_OK;
  } catch (...) {
    return SD_ERR_HOST_MEMORY;
  }
}

}  // extern "C"
