// Bandwidth-bound kernels of the MuonClip step (CUDA cores, 128-bit accesses).
//
//  momentum_kernel   M <- mu*M + G;  U = G + mu*M (Nesterov) or M;  writes U as
//                    the fp32 iterate and its bf16 copy (same row-major layout as
//                    the weight), and one fp64 partial of ||U||_F^2 per CTA.
//                    ("MuonClip: speed, then stability", §02 momentum; "Muon and
//                    MuonClip: orthogonalised updates for LLM training", §2
//                    Frobenius normalisation.)
//  norm_finalize     sums each matrix's partials in a fixed order (bitwise
//                    deterministic) and stores s = 1 / max(||U||_F, eps).
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
#pragma once

#include <climits>

#include "ptx.cuh"

namespace mc {

constexpr int MOM_THREADS = 256;
constexpr long long MOM_ELEMS_PER_CTA = 32768;

struct MomEntry {
  const void* g;        // gradient, rows x cols row-major (bf16 or fp32)
  float* m;             // momentum, rows x cols row-major, updated in place
  float* xf;            // fp32 iterate [rows][ld]
  __nv_bfloat16* xb;    // bf16 iterate [rows][ld]
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
                                          float* m_out, float* xf_out, __nv_bfloat16* xb_out, double& acc) {
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
  float4* xp = reinterpret_cast<float4*>(xf_out);
  xp[0] = make_float4(u[0], u[1], u[2], u[3]);
  xp[1] = make_float4(u[4], u[5], u[6], u[7]);
  uint4 b;
  b.x = pack_bf16x2(u[0], u[1]);
  b.y = pack_bf16x2(u[2], u[3]);
  b.z = pack_bf16x2(u[4], u[5]);
  b.w = pack_bf16x2(u[6], u[7]);
  *reinterpret_cast<uint4*>(xb_out) = b;
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
  float* xf = e->xf;
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
      momentum8(g0, m0a, m0b, mu, nesterov, mp + idx, xf + idx, xb + idx, acc);
      if (two) momentum8(g1, m1a, m1b, mu, nesterov, mp + j, xf + j, xb + j, acc);
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
      xf[row * ld + col] = u;
      xb[row * ld + col] = __float2bfloat16_rn(u);
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

// One warp per matrix.
__global__ void norm_finalize_kernel(const MomEntry* __restrict__ tab, int n, const double* __restrict__ partials,
                                     long long total_ctas, float eps, float* __restrict__ scale,
                                     float* __restrict__ norms_out) {
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
    scale[i] = static_cast<float>(1.0 / den);
    if (norms_out) norms_out[tab[i].orig] = static_cast<float>(nrm);
  }
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
