// Newton-Schulz for thin matrices: the short side m is at most THIN_M (32).
//
// The iteration is the one of "Muon and MuonClip: orthogonalised updates for
// LLM training", §2 (A = X X^T, B = bA + cA^2, X <- aX + BX) and "MuonClip:
// speed, then stability", §02, in the oriented frame (X is m x n, m <= n).
// With m this small the products are not tensor-core contractions: A and B
// are at most 32 x 32, and both A = X X^T and X <- (aI + B) X stream the long
// side of X once, a few dozen flops per element.  So the work runs on CUDA
// cores in fp32, with the iterate kept in fp32:
//
//   thin_gram_kernel   per chunk of THIN_COLS columns of X: the upper
//                      triangle of that chunk's X X^T (iteration 0 first
//                      builds X0 = s (hi + lo) from the momentum kernel's two
//                      bf16 halves of U and stores it in fp32)
//   thin_poly_kernel   per matrix: A = the chunks' partial sums in a fixed
//                      order, then P = aI + bA + cA^2 (fp32, 32 x 32 slot)
//   thin_apply_kernel  per chunk: X <- P X, column by column, in place; the
//                      last iteration writes W = (1 - lr wd) W - lr rms X
//                      instead (NorMuon: keeps X, the fp32 NS output)
//
// X is kept in the weight's stored layout [rows][ld]: oriented element (p, j)
// is at p*ld + j for a wide matrix and at j*ld + p for a tall one.  All
// reductions use a fixed order, so results are bitwise reproducible.
#pragma once

#include "ptx.cuh"

namespace mc {

constexpr int THIN_M = 32;                               // largest short side
constexpr int THIN_COLS = 256;                           // columns of X per CTA
constexpr int THIN_THREADS = 256;
constexpr int THIN_PAIRS = THIN_M * (THIN_M + 1) / 2;    // partial-sum slots per CTA
constexpr int THIN_PMAT = THIN_M * THIN_M;               // fp32 slot of P per matrix

struct ThinEntry {
  const __nv_bfloat16* xh;  // hi half of U, bf16(U), stored layout [rows][ld]
  const __nv_bfloat16* xl;  // lo half of U, bf16(U - hi)
  float* xf;                // fp32 iterate, stored layout [rows][ld]
  void* w;                  // weight rows x cols (row stride cols); NULL: keep O in xf
  float* u;                 // optional update output rows x cols
  float* pmat;              // P = aI + bA + cA^2, m x m in a THIN_M x THIN_M slot
  long long ld;             // row stride of xh, xl, xf
  long long cols;           // row stride of w and u
  long long n;              // long side (columns of the oriented X)
  long long cta_begin;      // first CTA of this matrix in the chunk launches
  int m;                    // short side, 1 .. THIN_M
  int tall;                 // rows > cols: oriented X is the stored matrix transposed
  int w_f32;
  int prob;                 // index into the per-matrix scale table
  float rms;                // rms_scale * sqrt(max(rows, cols))
  int pad_;
};

__device__ __forceinline__ long long thin_at(const ThinEntry& E, int p, long long j) {
  return E.tall ? j * E.ld + p : (long long)p * E.ld + j;
}

// Upper-triangle pair index t -> (p, q), p <= q < m, row by row.
__device__ __forceinline__ void thin_pair(int t, int m, int& p, int& q) {
  p = 0;
  while (t >= m - p) {
    t -= m - p;
    ++p;
  }
  q = p + t;
}

__device__ __forceinline__ int thin_find(const ThinEntry* __restrict__ tab, int n, long long cta) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid].cta_begin <= cta) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(THIN_THREADS) thin_gram_kernel(const ThinEntry* __restrict__ tab, int n,
                                                                 float* __restrict__ partials,
                                                                 const float* __restrict__ scale, int first) {
  const ThinEntry& E = tab[thin_find(tab, n, blockIdx.x)];
  const long long j0 = ((long long)blockIdx.x - E.cta_begin) * THIN_COLS;
  const int cols = static_cast<int>(E.n - j0 < THIN_COLS ? E.n - j0 : THIN_COLS);
  const int m = E.m;
  __shared__ float xs[THIN_M][THIN_COLS + 1];
  const float s = first ? scale[E.prob] : 1.f;
  for (int t = threadIdx.x; t < m * cols; t += THIN_THREADS) {
    // consecutive threads walk memory in order: along j for a wide matrix,
    // along p (the stored row) for a tall one
    const int p = E.tall ? t % m : t / cols;
    const int jj = E.tall ? t / m : t % cols;
    const long long a = thin_at(E, p, j0 + jj);
    float x;
    if (first) {
      // s = 0 marks a non-finite NS input: the iterate starts at zero
      x = s == 0.f ? 0.f : s * (__bfloat162float(E.xh[a]) + __bfloat162float(E.xl[a]));
      E.xf[a] = x;
    } else {
      x = E.xf[a];
    }
    xs[p][jj] = x;
  }
  __syncthreads();
  float* out = partials + (long long)blockIdx.x * THIN_PAIRS;
  const int npairs = m * (m + 1) / 2;
  for (int t = threadIdx.x; t < npairs; t += THIN_THREADS) {
    int p, q;
    thin_pair(t, m, p, q);
    float acc = 0.f;
    for (int jj = 0; jj < cols; ++jj) acc = fmaf(xs[p][jj], xs[q][jj], acc);
    out[t] = acc;
  }
}

// One CTA per matrix: warp w sums pairs w, w + 8, ... over the chunks (lanes
// stride the chunks, fp64, fixed shuffle tree), then P = aI + bA + cA^2.
__global__ void __launch_bounds__(THIN_THREADS) thin_poly_kernel(const ThinEntry* __restrict__ tab,
                                                                 const float* __restrict__ partials, float a,
                                                                 float b, float c) {
  const ThinEntry& E = tab[blockIdx.x];
  const int m = E.m;
  const long long nch = (E.n + THIN_COLS - 1) / THIN_COLS;
  __shared__ float A[THIN_M][THIN_M];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npairs = m * (m + 1) / 2;
  for (int t = warp; t < npairs; t += THIN_THREADS / 32) {
    double acc = 0.0;
    for (long long ch = lane; ch < nch; ch += 32) acc += partials[(E.cta_begin + ch) * THIN_PAIRS + t];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      int p, q;
      thin_pair(t, m, p, q);
      A[p][q] = static_cast<float>(acc);
      A[q][p] = static_cast<float>(acc);
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < m * m; t += THIN_THREADS) {
    const int p = t / m, q = t % m;
    float aa = 0.f;
    for (int r = 0; r < m; ++r) aa = fmaf(A[p][r], A[r][q], aa);
    E.pmat[p * THIN_M + q] = fmaf(c, aa, b * A[p][q]) + (p == q ? a : 0.f);
  }
}

// X <- P X, one thread per column of the oriented X; on the last iteration
// (when the entry has a weight) W = decay W + step * X_new instead.
// lr_wd: optional device (lr, wd) replacing decay = 1 - lr*wd and neg_lr = -lr.
__global__ void __launch_bounds__(THIN_THREADS) thin_apply_kernel(const ThinEntry* __restrict__ tab, int n,
                                                                  int last, float decay, float neg_lr,
                                                                  const float* __restrict__ lr_wd) {
  if (lr_wd) {
    decay = __fsub_rn(1.f, __fmul_rn(lr_wd[0], lr_wd[1]));
    neg_lr = -lr_wd[0];
  }
  const ThinEntry& E = tab[thin_find(tab, n, blockIdx.x)];
  const long long j0 = ((long long)blockIdx.x - E.cta_begin) * THIN_COLS;
  const int cols = static_cast<int>(E.n - j0 < THIN_COLS ? E.n - j0 : THIN_COLS);
  const int m = E.m;
  __shared__ float Ps[THIN_M][THIN_M];
  for (int t = threadIdx.x; t < THIN_M * THIN_M; t += THIN_THREADS) {
    const int p = t / THIN_M, q = t % THIN_M;
    Ps[p][q] = (p < m && q < m) ? E.pmat[p * THIN_M + q] : 0.f;
  }
  __syncthreads();
  const bool write_w = last && E.w != nullptr;
  const float step = neg_lr * E.rms;
  for (int jj = threadIdx.x; jj < cols; jj += THIN_THREADS) {
    const long long j = j0 + jj;
    float x[THIN_M];
#pragma unroll
    for (int p = 0; p < THIN_M; ++p) x[p] = p < m ? E.xf[thin_at(E, p, j)] : 0.f;
#pragma unroll
    for (int p = 0; p < THIN_M; ++p) {
      if (p >= m) break;
      float y = 0.f;
#pragma unroll
      for (int q = 0; q < THIN_M; ++q) y = fmaf(Ps[p][q], x[q], y);
      if (!write_w) {
        E.xf[thin_at(E, p, j)] = y;
      } else {
        // stored (row, col) of oriented element (p, j)
        const long long e = E.tall ? j * E.cols + p : (long long)p * E.cols + j;
        if (E.u) E.u[e] = E.rms * y;
        if (E.w_f32) {
          float* w = static_cast<float*>(E.w) + e;
          *w = fmaf(step, y, decay * *w);
        } else {
          __nv_bfloat16* w = static_cast<__nv_bfloat16*>(E.w) + e;
          *w = __float2bfloat16_rn(fmaf(step, y, decay * __bfloat162float(*w)));
        }
      }
    }
  }
}

}  // namespace mc
