// Bandwidth-bound kernels of the MuonClip step (CUDA cores, 128-bit accesses).
//
//  momentum_kernel   M <- mu*M + G;  U = G + mu*M (Nesterov) or M;  writes U as
//                    two bf16 halves, hi = bf16(U) (the first MMA operand) and
//                    lo = bf16(U - hi) (same row-major layout as the weight), and
//                    one fp64 partial of ||U||_F^2 per CTA.
//                    ("MuonClip: speed, then stability", §02 momentum; "Muon and
//                    MuonClip: orthogonalised updates for LLM training", §2
//                    Frobenius normalisation.)
//  norm_finalize     sums each matrix's partials in a fixed order (bitwise
//                    deterministic) and stores s = 1 / max(||U||_F, eps); a
//                    non-finite ||U||_F (U holds a NaN or Inf) gives s = 0,
//                    which the first Newton-Schulz products turn into a zero
//                    iterate, and raises MC_DEV_ERR_NONFINITE.
//  qk_keys_*         order-preserving int encoding of the per-head S_max.
//  qk_clip_kernel    gamma_h = tau / S_max_h when S_max_h > tau; rows of head h
//                    in W_q scaled by gamma^alpha, in W_k by gamma^(1-alpha)
//                    ("MuonClip: speed, then stability", §05).
//  qk_gamma_kernel   gamma_h and the clipped-head mask alone.
//  qk_clip_slices_kernel
//                    the same rescale over an explicit map of weight slices,
//                    each with its head and exponent: multi-head latent
//                    attention scales the head's content query and content key
//                    by gamma^(1/2) and its rotary query by gamma, and leaves
//                    the rotary key that all heads share alone ("MuonClip:
//                    speed, then stability", §06; "Muon and MuonClip:
//                    orthogonalised updates for LLM training", "MuonClip:
//                    QK-clip, per head, adapted to MLA").
//  normuon_rowsq_kernel, normuon_finalize_kernel, normuon_apply_kernel
//                    NorMuon after Newton-Schulz ("About Muon: Muon At Scale",
//                    "Certain Neurons Still Dominate"): per-row sums of
//                    squares of O, the per-row second moment and row factors
//                    (with the rescale to ||O||_F folded in), then the scaled
//                    update with decoupled decay.
#pragma once

#include <climits>

#include "ptx.cuh"

namespace mc {

constexpr int MOM_THREADS = 256;
constexpr long long MOM_ELEMS_PER_CTA = 32768;

struct MomEntry {
  const void* g;        // gradient, rows x cols row-major (bf16 or fp32)
  float* m;             // momentum, rows x cols row-major, updated in place
  __nv_bfloat16* xl;    // lo half of the iterate, bf16(U - bf16(U)) [rows][ld]
  __nv_bfloat16* xb;    // bf16 iterate (its hi half) [rows][ld]
  long long rows, cols, ld;
  long long cta_begin;  // first CTA of this matrix in the launch
  int g_f32;
  int vec;              // cols % 8 == 0 (then ld == cols and rows are 32-byte aligned)
  int orig;             // index of the matrix in the caller's list
  int pad_;
};

__device__ __forceinline__ void load_g8(const void* g, long long idx, int g_f32, float (&x)[8]) {
  if (g_f32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(g) + idx);
    float4 a = p[0], b = p[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
    uint4 a = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(g) + idx);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void momentum8(const float (&g)[8], float4 ma, float4 mb, float mu, int nesterov,
                                          float* m_out, __nv_bfloat16* xl_out, __nv_bfloat16* xb_out,
                                          double& acc) {
  float m[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
  float u[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    m[i] = fmaf(mu, m[i], g[i]);
    u[i] = nesterov ? fmaf(mu, m[i], g[i]) : m[i];
    acc += static_cast<double>(u[i]) * static_cast<double>(u[i]);
  }
  float4* mp = reinterpret_cast<float4*>(m_out);
  mp[0] = make_float4(m[0], m[1], m[2], m[3]);
  mp[1] = make_float4(m[4], m[5], m[6], m[7]);
  float lo[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) lo[i] = u[i] - __bfloat162float(__float2bfloat16_rn(u[i]));
  uint4 b;
  b.x = pack_bf16x2(u[0], u[1]);
  b.y = pack_bf16x2(u[2], u[3]);
  b.z = pack_bf16x2(u[4], u[5]);
  b.w = pack_bf16x2(u[6], u[7]);
  *reinterpret_cast<uint4*>(xb_out) = b;
  uint4 l;
  l.x = pack_bf16x2(lo[0], lo[1]);
  l.y = pack_bf16x2(lo[2], lo[3]);
  l.z = pack_bf16x2(lo[4], lo[5]);
  l.w = pack_bf16x2(lo[6], lo[7]);
  *reinterpret_cast<uint4*>(xl_out) = l;
}

__global__ void __launch_bounds__(MOM_THREADS) momentum_kernel(const MomEntry* __restrict__ tab, int n,
                                                               double* __restrict__ partials, float mu,
                                                               int nesterov) {
  // Find the matrix this CTA works on: largest i with tab[i].cta_begin <= blockIdx.x.
  int lo = 0, hi = n - 1;
  const long long cta = blockIdx.x;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid].cta_begin <= cta) lo = mid; else hi = mid - 1;
  }
  const MomEntry* e = tab + lo;
  const void* gp = e->g;
  float* mp = e->m;
  __nv_bfloat16* xl = e->xl;
  __nv_bfloat16* xb = e->xb;
  const long long cols = e->cols, ld = e->ld;
  const long long total = e->rows * cols;
  const int g_f32 = e->g_f32;
  const long long e0 = (cta - e->cta_begin) * MOM_ELEMS_PER_CTA;
  const long long e1 = (e0 + MOM_ELEMS_PER_CTA < total) ? e0 + MOM_ELEMS_PER_CTA : total;
  double acc = 0.0;
  if (e->vec) {
    // Two groups of 8 elements per thread in flight: both groups' loads are
    // issued before either is used.
    constexpr long long STEP = MOM_THREADS * 8;
    for (long long idx = e0 + threadIdx.x * 8; idx < e1; idx += 2 * STEP) {
      const long long j = idx + STEP;
      const bool two = j < e1;
      float g0[8], g1[8];
      load_g8(gp, idx, g_f32, g0);
      const float4* m0p = reinterpret_cast<const float4*>(mp + idx);
      const float4 m0a = m0p[0], m0b = m0p[1];
      float4 m1a = make_float4(0.f, 0.f, 0.f, 0.f), m1b = m1a;
      if (two) {
        load_g8(gp, j, g_f32, g1);
        const float4* m1p = reinterpret_cast<const float4*>(mp + j);
        m1a = m1p[0];
        m1b = m1p[1];
      }
      momentum8(g0, m0a, m0b, mu, nesterov, mp + idx, xl + idx, xb + idx, acc);
      if (two) momentum8(g1, m1a, m1b, mu, nesterov, mp + j, xl + j, xb + j, acc);
    }
  } else {
    for (long long idx = e0 + threadIdx.x; idx < e1; idx += MOM_THREADS) {
      const float g = g_f32 ? static_cast<const float*>(gp)[idx]
                            : __bfloat162float(static_cast<const __nv_bfloat16*>(gp)[idx]);
      const float m = fmaf(mu, mp[idx], g);
      mp[idx] = m;
      const float u = nesterov ? fmaf(mu, m, g) : m;
      acc += static_cast<double>(u) * static_cast<double>(u);
      const long long row = idx / cols, col = idx - row * cols;
      const __nv_bfloat16 h = __float2bfloat16_rn(u);
      xb[row * ld + col] = h;
      xl[row * ld + col] = __float2bfloat16_rn(u - __bfloat162float(h));
    }
  }
  // Fixed-order block reduction (deterministic).
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ double wsum[MOM_THREADS / 32];
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < MOM_THREADS / 32; ++w) s += wsum[w];
    partials[cta] = s;
  }
}

// One warp per matrix.  The fp64 sum of squares of finite fp32 values cannot
// overflow (at most 2^36 terms below 2^256 each), so the norm is finite
// exactly when every element of U is.
__global__ void norm_finalize_kernel(const MomEntry* __restrict__ tab, int n, const double* __restrict__ partials,
                                     long long total_ctas, float eps, float* __restrict__ scale,
                                     float* __restrict__ norms_out, int* __restrict__ err) {
  const int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (i >= n) return;
  const long long b = tab[i].cta_begin;
  const long long e = (i + 1 < n) ? tab[i + 1].cta_begin : total_ctas;
  double s = 0.0;
  for (long long k = b + lane; k < e; k += 32) s += partials[k];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    const double nrm = sqrt(s);
    const double den = nrm > static_cast<double>(eps) ? nrm : static_cast<double>(eps);
    const bool finite = isfinite(nrm);
    scale[i] = finite ? static_cast<float>(1.0 / den) : 0.f;
    if (!finite && err) atomicOr(err, MC_DEV_ERR_NONFINITE);
    if (norms_out) norms_out[tab[i].orig] = static_cast<float>(nrm);
  }
}

// A parameter table of up to BYTES carried in the launch's own parameters:
// the launch copies them, so the caller's host buffer is free as soon as the
// launch returns, no host memory is read later, and the upload stays valid
// when the launch is captured into a CUDA graph.  The launch queue holds the
// whole parameter block, so a table takes the smallest size that fits; the
// largest (32720 bytes of parameters) stays under the 32764-byte limit.
constexpr unsigned TABLE_BLOB_MAX = 32704;
template <unsigned BYTES>
struct TableBlob {
  uint4* dst;     // 16-byte aligned
  unsigned n16;   // 16-byte words to copy, <= BYTES / 16
  unsigned pad_;
  uint4 data[BYTES / 16];
};
static_assert(sizeof(TableBlob<TABLE_BLOB_MAX>) <= 32764, "kernel parameters");

template <unsigned BYTES>
__global__ void table_fill_kernel(const __grid_constant__ TableBlob<BYTES> b) {
  for (unsigned i = threadIdx.x; i < b.n16; i += blockDim.x) b.dst[i] = b.data[i];
}

__global__ void qk_keys_init_kernel(int* keys, int H) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) keys[h] = INT_MIN;
}

__global__ void qk_keys_decode_kernel(const int* keys, float* smax, int H) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) smax[h] = keys[h] == INT_MIN ? -INFINITY : ordered_to_float(keys[h]);
}

// grid (H*dh, 2): one CTA per row of W_q (y = 0) or W_k (y = 1).
__global__ void qk_clip_kernel(__nv_bfloat16* __restrict__ wq, __nv_bfloat16* __restrict__ wk, int H, int dh,
                               int D, const float* __restrict__ smax, float tau, float alpha,
                               float* __restrict__ gamma_out, int* __restrict__ mask_out, int vec) {
  const int row = blockIdx.x;
  const int which = blockIdx.y;
  const int h = row / dh;
  const float s = smax[h];
  const bool clip = s > tau;  // S_max == tau (or NaN) does not clip
  const float gamma = clip ? tau / s : 1.f;
  if (which == 0 && row == h * dh && threadIdx.x == 0) {
    if (gamma_out) gamma_out[h] = gamma;
    if (mask_out) mask_out[h] = clip ? 1 : 0;
  }
  if (!clip) return;
  const float ex = which == 0 ? alpha : 1.f - alpha;
  const float f = (ex == 0.5f) ? sqrtf(gamma) : powf(gamma, ex);
  __nv_bfloat16* w = (which == 0 ? wq : wk) + static_cast<long long>(row) * D;
  if (vec) {
    for (int c = threadIdx.x * 8; c < D; c += blockDim.x * 8) {
      uint4 a = *reinterpret_cast<uint4*>(w + c);
      uint32_t x[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float lo = __uint_as_float(x[i] << 16) * f;
        const float hi = __uint_as_float(x[i] & 0xFFFF0000u) * f;
        x[i] = pack_bf16x2(lo, hi);
      }
      *reinterpret_cast<uint4*>(w + c) = make_uint4(x[0], x[1], x[2], x[3]);
    }
  } else {
    for (int c = threadIdx.x; c < D; c += blockDim.x) w[c] = __float2bfloat16_rn(__bfloat162float(w[c]) * f);
  }
}

// ---------------------------------------------------------------- NorMuon
struct NormEntry {
  const float* o;        // NS output, rows x ld fp32 (stored, un-oriented layout)
  float* v;              // per-row second moment [rows], updated in place
  void* w;               // weight rows x cols (bf16 or fp32)
  float* u;              // optional update output rows x cols
  long long rows, cols, ld;
  long long row_base;    // first slot of this matrix in the row arrays
  long long cta_begin;   // first CTA of this matrix in the apply launch
  float rms;             // rms_scale * sqrt(max(rows, cols))
  int w_f32;
  int vec;               // cols % 8 == 0 (then ld == cols)
  int pad_;
};

constexpr int NORM_THREADS = 256;

// First entry whose `key` field exceeds x, minus one (entries sorted by key).
template <typename F>
__device__ __forceinline__ int find_entry(int n, long long x, F key) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (key(mid) <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// One warp per row: sum of squares of the row of O, fixed lane order and a
// fixed shuffle tree (deterministic).
__global__ void normuon_rowsq_kernel(const NormEntry* __restrict__ tab, int n, long long total_rows,
                                     float* __restrict__ rowsq) {
  const long long gr = (long long)blockIdx.x * (NORM_THREADS / 32) + (threadIdx.x >> 5);
  if (gr >= total_rows) return;
  const int lane = threadIdx.x & 31;
  const int k = find_entry(n, gr, [&](int i) { return tab[i].row_base; });
  const NormEntry& E = tab[k];
  const long long i = gr - E.row_base;
  const float* o = E.o + i * E.ld;
  float acc = 0.f;
  const long long c4 = E.cols & ~3LL;
  for (long long j = 4 * lane; j < c4; j += 128) {
    const float4 x = *reinterpret_cast<const float4*>(o + j);
    acc = fmaf(x.x, x.x, acc);
    acc = fmaf(x.y, x.y, acc);
    acc = fmaf(x.z, x.z, acc);
    acc = fmaf(x.w, x.w, acc);
  }
  for (long long j = c4 + lane; j < E.cols; j += 32) acc = fmaf(o[j], o[j], acc);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) rowsq[E.row_base + i] = acc;
}

// One CTA per matrix: v <- beta2 v + (1 - beta2) rowsq / cols, f = 1/(sqrt(v)+eps),
// then every row factor times ||O||_F / ||f o O||_F (fp64 sums, fixed order).
__global__ void normuon_finalize_kernel(const NormEntry* __restrict__ tab, const float* __restrict__ rowsq,
                                        float* __restrict__ rowf, float beta2, float eps) {
  const NormEntry& E = tab[blockIdx.x];
  __shared__ double red_a[NORM_THREADS], red_b[NORM_THREADS];
  __shared__ float g_sh;
  double a = 0.0, b = 0.0;
  const float inv_cols = 1.f / static_cast<float>(E.cols);
  for (long long i = threadIdx.x; i < E.rows; i += NORM_THREADS) {
    const float q = rowsq[E.row_base + i];
    const float vn = fmaf(beta2, E.v[i], (1.f - beta2) * (q * inv_cols));
    E.v[i] = vn;
    const float f = 1.f / (sqrtf(vn) + eps);
    rowf[E.row_base + i] = f;
    a += static_cast<double>(q);
    b += static_cast<double>(f) * static_cast<double>(f) * static_cast<double>(q);
  }
  red_a[threadIdx.x] = a;
  red_b[threadIdx.x] = b;
  __syncthreads();
  for (int w = NORM_THREADS / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) {
      red_a[threadIdx.x] += red_a[threadIdx.x + w];
      red_b[threadIdx.x] += red_b[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) g_sh = red_b[0] > 0.0 ? static_cast<float>(sqrt(red_a[0] / red_b[0])) : 0.f;
  __syncthreads();
  const float g = g_sh;
  for (long long i = threadIdx.x; i < E.rows; i += NORM_THREADS) rowf[E.row_base + i] *= g;
}

// W <- decay W + step * (rowf_i O_ij), update_out = rms * rowf_i O_ij;
// MOM_ELEMS_PER_CTA elements of one matrix per CTA, 8 at a time when rows are
// 16-byte multiples.
// lr_wd: optional device (lr, wd) replacing decay = 1 - lr*wd and neg_lr = -lr.
__global__ void normuon_apply_kernel(const NormEntry* __restrict__ tab, int n, const float* __restrict__ rowf,
                                     float decay, float neg_lr, const float* __restrict__ lr_wd) {
  if (lr_wd) {
    decay = __fsub_rn(1.f, __fmul_rn(lr_wd[0], lr_wd[1]));
    neg_lr = -lr_wd[0];
  }
  const int k = find_entry(n, blockIdx.x, [&](int i) { return tab[i].cta_begin; });
  const NormEntry& E = tab[k];
  const long long total = E.rows * E.cols;
  const long long e0 = (blockIdx.x - E.cta_begin) * MOM_ELEMS_PER_CTA;
  const long long e1 = e0 + MOM_ELEMS_PER_CTA < total ? e0 + MOM_ELEMS_PER_CTA : total;
  const float step = neg_lr * E.rms;
  const float* rf = rowf + E.row_base;
  if (E.vec) {
    for (long long e = e0 + 8LL * threadIdx.x; e < e1; e += 8LL * NORM_THREADS) {
      const long long i = e / E.cols;
      const float f = rf[i];
      const float4 o0 = *reinterpret_cast<const float4*>(E.o + e);
      const float4 o1 = *reinterpret_cast<const float4*>(E.o + e + 4);
      const float x[8] = {f * o0.x, f * o0.y, f * o0.z, f * o0.w, f * o1.x, f * o1.y, f * o1.z, f * o1.w};
      if (E.u) {
        float4* U = reinterpret_cast<float4*>(E.u + e);
        U[0] = make_float4(E.rms * x[0], E.rms * x[1], E.rms * x[2], E.rms * x[3]);
        U[1] = make_float4(E.rms * x[4], E.rms * x[5], E.rms * x[6], E.rms * x[7]);
      }
      if (E.w_f32) {
        float4* W = reinterpret_cast<float4*>(static_cast<float*>(E.w) + e);
        float4 a = W[0], b = W[1];
        a = make_float4(fmaf(step, x[0], decay * a.x), fmaf(step, x[1], decay * a.y),
                        fmaf(step, x[2], decay * a.z), fmaf(step, x[3], decay * a.w));
        b = make_float4(fmaf(step, x[4], decay * b.x), fmaf(step, x[5], decay * b.y),
                        fmaf(step, x[6], decay * b.z), fmaf(step, x[7], decay * b.w));
        W[0] = a;
        W[1] = b;
      } else {
        uint4* W = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(E.w) + e);
        uint4 a = *W;
        uint32_t wv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float lo = fmaf(step, x[2 * t], decay * __uint_as_float(wv[t] << 16));
          const float hi = fmaf(step, x[2 * t + 1], decay * __uint_as_float(wv[t] & 0xFFFF0000u));
          wv[t] = pack_bf16x2(lo, hi);
        }
        *W = make_uint4(wv[0], wv[1], wv[2], wv[3]);
      }
    }
  } else {
    for (long long e = e0 + threadIdx.x; e < e1; e += NORM_THREADS) {
      const long long i = e / E.cols, j = e - i * E.cols;
      const float x = rf[i] * E.o[i * E.ld + j];
      if (E.u) E.u[e] = E.rms * x;
      if (E.w_f32) {
        float* W = static_cast<float*>(E.w) + e;
        *W = fmaf(step, x, decay * *W);
      } else {
        __nv_bfloat16* W = static_cast<__nv_bfloat16*>(E.w) + e;
        *W = __float2bfloat16_rn(fmaf(step, x, decay * __bfloat162float(*W)));
      }
    }
  }
}

__global__ void qk_gamma_kernel(const float* __restrict__ smax, int H, float tau, float* __restrict__ gamma_out,
                                int* __restrict__ mask_out) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= H) return;
  const float s = smax[h];
  const bool clip = s > tau;
  if (gamma_out) gamma_out[h] = clip ? tau / s : 1.f;
  if (mask_out) mask_out[h] = clip ? 1 : 0;
}

// One launch covers up to CLIP_MAX_SLICES slices; CTA b rescales one row,
// the row of the slice whose cumulative row range holds b.
constexpr int CLIP_MAX_SLICES = 48;
struct ClipSlice {
  void* w;               // row-major matrix, `cols` elements per row
  long long row_begin;   // first row of the slice
  long long cols;
  float exponent;        // rows *= gamma_head ^ exponent
  int head;
  int f32;               // 1 fp32, 0 bf16
  int vec;               // rows are 16-byte aligned and a whole number of 16-byte chunks
};
struct ClipTable {
  ClipSlice s[CLIP_MAX_SLICES];
  long long row_end[CLIP_MAX_SLICES];  // cumulative: slice i owns CTAs [row_end[i-1], row_end[i])
  int n;
};
static_assert(sizeof(ClipTable) + 64 <= 4096, "clip table must fit the classic 4 KiB parameter limit");

__global__ void qk_clip_slices_kernel(const __grid_constant__ ClipTable T, const float* __restrict__ smax,
                                      float tau) {
  const long long b = blockIdx.x;
  int lo = 0, hi = T.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (T.row_end[mid] > b) hi = mid;
    else lo = mid + 1;
  }
  const ClipSlice& S = T.s[lo];
  const float sm = smax[S.head];
  if (!(sm > tau)) return;  // S_max == tau (or NaN) does not clip: rows stay bit-for-bit
  const float gamma = tau / sm;
  const float f = S.exponent == 0.5f ? sqrtf(gamma) : (S.exponent == 1.f ? gamma : powf(gamma, S.exponent));
  const long long row = S.row_begin + (b - (lo ? T.row_end[lo - 1] : 0));
  if (S.f32) {
    float* w = static_cast<float*>(S.w) + row * S.cols;
    if (S.vec) {
      for (long long c = threadIdx.x * 4; c < S.cols; c += blockDim.x * 4) {
        float4 a = *reinterpret_cast<float4*>(w + c);
        a.x *= f; a.y *= f; a.z *= f; a.w *= f;
        *reinterpret_cast<float4*>(w + c) = a;
      }
    } else {
      for (long long c = threadIdx.x; c < S.cols; c += blockDim.x) w[c] *= f;
    }
  } else {
    __nv_bfloat16* w = static_cast<__nv_bfloat16*>(S.w) + row * S.cols;
    if (S.vec) {
      for (long long c = threadIdx.x * 8; c < S.cols; c += blockDim.x * 8) {
        uint4 a = *reinterpret_cast<uint4*>(w + c);
        uint32_t x[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          x[i] = pack_bf16x2(__uint_as_float(x[i] << 16) * f, __uint_as_float(x[i] & 0xFFFF0000u) * f);
        *reinterpret_cast<uint4*>(w + c) = make_uint4(x[0], x[1], x[2], x[3]);
      }
    } else {
      for (long long c = threadIdx.x; c < S.cols; c += blockDim.x) w[c] = __float2bfloat16_rn(__bfloat162float(w[c]) * f);
    }
  }
}

}  // namespace mc
