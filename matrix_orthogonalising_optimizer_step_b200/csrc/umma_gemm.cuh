// Grouped, persistent tcgen05 GEMM for sm_100a with the MuonClip epilogues.
//
// One kernel computes D = A * B^T tile by tile (a CTA pair's 256 x 256 or
// 256 x 512 fp32 accumulator in TMEM) for up to MAX_GROUPS groups of equally
// shaped problems, and hands each finished tile to a fused epilogue:
//
//   EPI_GRAM        A_k   = s^2 * X X^T            (symmetric: upper tiles only,
//                                                  each element stored twice;
//                                                  dead diagonal blocks skipped)
//   EPI_POLY        B_k   = b*A + c*(A A) [+ a*I]  (symmetric, mirrored store)
//   EPI_APPLY_MIXED X_k+1 = s * (a*X + B X)        (a*X from the hi + lo copy of the
//                                                  iterate; stores the bf16 iterate
//                                                  and, when flagged, its lo half)
//   EPI_APPLY       X_k+1 = P X, P = aI+bA+cA^2    (stores the bf16 iterate, and the
//                                                  fp32 NS output for NorMuon)
//   EPI_APPLY_FINAL W     = (1 - lr*wd) W - lr * rms * X_N   (last iteration; X_N
//                                                  never touches memory)
//
// Precision: operands are bf16, accumulation fp32.  While singular values are
// still small (the first two iterations) the a*X term is taken from a
// two-part copy of the iterate, hi = bf16(X) (the MMA operand itself) plus
// lo = bf16(X - hi), about 16 significant bits, so only B X sees a rounded X
// (emulated against an fp32 copy: the same error to within 1 %); afterwards a*I is folded
// into B, because once the singular values sit in the polynomial's band
// |a + b s^2 + c s^4| (the factor on a rounded X in P X) is smaller than
// |b s^2 + c s^4| (the factor in B X).
//   EPI_STORE       plain bf16 store (Q/K projection)
//   EPI_CAUSALMAX   per-head max over j <= i of the score tile (QK-Clip's S_max);
//                   the score tile is never stored
//
// The quintic Newton-Schulz step these epilogues implement is the one printed in
// "Muon and MuonClip: orthogonalised updates for LLM training", §2 (A = X X^T,
// X = aX + (bA + cA A)X) and "MuonClip: speed, then stability", §02; the apply
// is §03's W <- W - eta (O + lambda W) with O scaled by 0.2 sqrt(max(m, n)).
//
// Execution: CTA pairs (clusters of 2, one CTA per SM) run 2-SM tensor-core
// MMAs (tcgen05 cta_group::2): a 256 x 256 or 256 x 512 output tile per pair
// (see TileCfg), of which each CTA holds 128 rows in its own TMEM.  Each CTA
// stages its 128 rows of A and its 128 rows of every 256-column B block (the
// pair's B is split between the two SMs).  No TMA multicast is used.
//
// Warp roles (320 threads per CTA):
//   warp 0      TMA producer: ring of stages, each one or two k-blocks of
//               {A 128x64, one or two B 128x64} bf16 tiles (TileCfg::KPS),
//               128-byte swizzled, K-major or MN-major per group.  Both CTAs'
//               copies complete on the leader CTA's "full" barrier.
//   warp 1      TMEM allocation (512 columns, both CTAs, 2-SM form); in the
//               leader CTA one thread issues tcgen05.mma (M=256, N=256, K=16;
//               two per k-step for WIDE tiles) and commits to both CTAs'
//               "empty" and "accumulator full" barriers.
//   warps 2..   epilogue: warp w reads TMEM lanes 32*(w%4)..+31 and column
//               group (w-2)/4 of the tile; the leader's "accumulator empty"
//               barrier counts both CTAs' epilogue warps.  Whole 32-row
//               blocks move to and from global memory through a per-warp
//               shared-memory buffer (TMA where the operand has a tensor map,
//               else coalesced rows; see epi_tma_block and epi_fast64).
// Every role starts after griddepcontrol.wait: the prologue (barriers, TMEM,
// tensor-map prefetch) may overlap the previous kernel of the stream when the
// launch allows programmatic serialisation.
#pragma once

#include <climits>

#include "ptx.cuh"

namespace mc {

constexpr int BM = 256, BK = 64;
constexpr int HALF = 128;                               // rows of A and of each B block per CTA
constexpr int MMA_N = 256;                              // N of one MMA instruction
constexpr uint32_t A_STAGE_BYTES = HALF * BK * 2;       // 16 KiB
constexpr uint32_t B_STAGE_BYTES = HALF * BK * 2;       // 16 KiB per B block
constexpr uint32_t MN_BOX_BYTES = 64 * BK * 2;          // one {64 MN, 64 K} box: 8 KiB
constexpr int NUM_EPI_WARPS = 8;                         // multiple of 4 (one per TMEM lane quarter)
constexpr int EPI_COL_GROUPS = NUM_EPI_WARPS / 4;        // warps sharing a lane quarter split its columns
constexpr int GEMM_THREADS = 64 + NUM_EPI_WARPS * 32;
static_assert(NUM_EPI_WARPS % 4 == 0, "epilogue warps cover the four TMEM lane quarters evenly");
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_GROUPS = 4;
constexpr int GEMM_BARRIER_BYTES = 256;

// Two tile shapes per CTA pair:
//   WIDE = 0: 256 x 256, two 256-column accumulators (the next tile's MMAs
//             overlap this tile's epilogue), 3 stages of 64 KB per CTA, each
//             two k-blocks under one pair of barriers (eight MMAs per round
//             trip, as WIDE = 1 has);
//   WIDE = 1: 256 x 512, one 512-column accumulator, 4 stages of 48 KB per
//             CTA.  Sharing each A tile between two N=256 MMAs cuts the
//             operand bytes per MMA cycle from 64 to 48 per SM, below the
//             TMA feed limit; the epilogue is then not overlapped, so WIDE
//             suits the phases whose epilogue is light.
// EPI_CAUSALMAX keeps one running maximum per head in shared memory (for up to
// this many heads) and flushes it to global memory once, at the end.
constexpr int SMEM_HEADS = 4096;

template <int WIDE>
struct TileCfg {
  static constexpr int N = MMA_N << WIDE;               // tile columns per pair
  static constexpr int NB = 1 << WIDE;                  // B blocks (MMAs per k-step)
  static constexpr int KPS = WIDE ? 1 : 2;              // k-blocks per stage
  static constexpr int STAGES = WIDE ? 4 : 3;
  static constexpr int NACC = WIDE ? 1 : 2;             // accumulator buffers
  static constexpr uint32_t KB_BYTES = A_STAGE_BYTES + NB * B_STAGE_BYTES;  // one k-block, one CTA
  static constexpr uint32_t PAIR_KB_BYTES = 2 * KB_BYTES;
  static constexpr uint32_t STAGE_BYTES = KPS * KB_BYTES;
  static constexpr size_t SMEM_BYTES = 1024 + size_t(STAGES) * STAGE_BYTES + GEMM_BARRIER_BYTES;
  static constexpr size_t SMEM_BYTES_HEADS = SMEM_BYTES + 4 * size_t(SMEM_HEADS);
  static_assert(NACC * N <= int(TMEM_COLS), "accumulators exceed TMEM");
};
constexpr size_t GEMM_SMEM_BYTES =
    TileCfg<0>::SMEM_BYTES > TileCfg<1>::SMEM_BYTES ? TileCfg<0>::SMEM_BYTES : TileCfg<1>::SMEM_BYTES;
static_assert(TileCfg<0>::SMEM_BYTES_HEADS <= 232448, "shared memory per CTA");

enum Sched : int { SCHED_DENSE = 0, SCHED_SYM = 1, SCHED_CAUSAL = 2 };
enum Layout : int { LAYOUT_BATCHED = 0, LAYOUT_HEADS = 1 };
enum Epi : int {
  EPI_GRAM = 0,
  EPI_POLY = 1,
  EPI_APPLY = 2,
  EPI_APPLY_FINAL = 3,
  EPI_STORE = 4,
  EPI_CAUSALMAX = 5,
  EPI_APPLY_MIXED = 6   // EPI_APPLY whose a*X term comes from the iterate's hi + lo halves
};

// The apply epilogues: X' = s(aX + BX) (EPI_APPLY_MIXED, a*X from hi + lo),
// X' = P X (EPI_APPLY) and the last iteration's weight update (EPI_APPLY_FINAL,
// either form, chosen at run time by xf_read).
template <int EPI>
__host__ __device__ constexpr bool is_apply_epi() {
  return EPI == EPI_APPLY || EPI == EPI_APPLY_MIXED || EPI == EPI_APPLY_FINAL;
}


// Epilogues that move bf16 row blocks to or from global memory stage them
// through one 4 KiB shared-memory buffer per epilogue warp (32 rows x 64
// columns); see warp_rows_from_frags / warp_store_rows64.
constexpr int EPI_BUF_BYTES = 32 * 64 * 2;
template <int EPI>
__host__ __device__ constexpr bool epi_uses_row_buffers() {
  return EPI == EPI_GRAM || EPI == EPI_POLY || is_apply_epi<EPI>() || EPI == EPI_STORE;
}

template <int EPI, int WIDE>
constexpr size_t gemm_smem_bytes() {
  return EPI == EPI_CAUSALMAX ? TileCfg<WIDE>::SMEM_BYTES_HEADS
                              : TileCfg<WIDE>::SMEM_BYTES +
                                    (epi_uses_row_buffers<EPI>() ? size_t(NUM_EPI_WARPS) * EPI_BUF_BYTES : 0);
}
static_assert(TileCfg<1>::SMEM_BYTES + size_t(NUM_EPI_WARPS) * EPI_BUF_BYTES <= 232448, "shared memory per CTA");
static_assert(TileCfg<0>::SMEM_BYTES + size_t(NUM_EPI_WARPS) * EPI_BUF_BYTES <= 232448, "shared memory per CTA");

struct GemmGroup {
  int M, N, K;             // D is M x N, contraction K
  int count;               // independent problems in the group
  int tiles_m, tiles_n;    // ceil(M / BM), ceil(N / BN)
  long long tiles_per_prob;
  long long tile_start;    // first global tile of this group
  int sched, layout, heads;
  int k_split;             // LAYOUT_HEADS: contraction columns [0, k_split) come from
                           // maps slot 0, the rest from slot 1 (0 = no split)
  int a_mn, b_mn;          // operand major-ness: 0 K-major, 1 MN-major
  int prob_base;           // index of problem 0 in the per-matrix scale table
  int band;                // dense raster: n-tiles per band
  int nshift;              // log2(tile columns / 256): 0 or 1 (WIDE tiles)
  // ---- epilogue operands ----
  void* d;                 // bf16 output [count][M][d_ld]
  long long d_ld, d_bs;
  const void* src;         // bf16 epilogue source (EPI_POLY)
  long long src_ld, src_bs;
  const __nv_bfloat16* xh; // EPI_APPLY*: hi half of the iterate (its bf16 copy)
  long long xh_ld, xh_bs;
  __nv_bfloat16* xl;       // EPI_APPLY*: lo half of the iterate, bf16(X - hi)
  long long xl_ld, xl_bs;
  float* xf;               // EPI_APPLY: fp32 copy of the new iterate (when xf_write)
  long long xf_ld, xf_bs;
  int xf_read;             // EPI_APPLY*: take a*X from hi + lo
  int xl_write;            // EPI_APPLY: store the new iterate's lo half to xl
  int xf_write;            // EPI_APPLY: store the new (last) iterate in fp32 to xf instead of d
  void* const* w_ptrs;     // per-problem weight (EPI_APPLY_FINAL), row-major M x N
  float* const* u_ptrs;    // per-problem update output, entries may be null
  const float* scale;      // per-problem s, or null for 1
  int w_f32;               // weight dtype: 1 fp32, 0 bf16
  int w_vec;               // weight rows 16-byte aligned
  int mask_causal;         // EPI_CAUSALMAX
  int* keys;               // EPI_CAUSALMAX: order-preserving ints, one per head
  float coef_acc, coef_src;
  float diag;              // EPI_POLY: added on the diagonal (a for P = aI + B)
  float decay, step, rms;  // EPI_APPLY_FINAL
  const float* lr_wd;      // EPI_APPLY_FINAL: device (lr, wd) replacing decay and step, or null
  float out_scale;         // EPI_CAUSALMAX: 1/sqrt(d_head)
  int tma_epi;             // the group's epilogue tensor maps are set (map_eo, map_ei, map_ei2)
};

// The last apply's W <- decay W + step O coefficients: the group's own, or
// computed when the kernel runs from a device (lr, wd) pair, with the same
// fp32 operations (and roundings) as the host's 1 - lr*wd and -lr*rms.
__device__ __forceinline__ void final_coefs(const GemmGroup& G, float& decay, float& step) {
  if (G.lr_wd) {
    const float lr = G.lr_wd[0], wd = G.lr_wd[1];
    decay = __fsub_rn(1.f, __fmul_rn(lr, wd));
    step = __fmul_rn(-lr, G.rms);
  } else {
    decay = G.decay;
    step = G.step;
  }
}

template <int EPI>
__device__ __forceinline__ bool apply_reads_x(const GemmGroup& G) {
  if constexpr (EPI == EPI_APPLY_MIXED) return true;
  else if constexpr (EPI == EPI_APPLY) return false;
  else return G.xf_read != 0;
}

struct GemmParams {
  CUtensorMap map_a[MAX_GROUPS];
  CUtensorMap map_b[MAX_GROUPS];
  // Epilogue tensor maps per group, boxes of 32 rows x 64 columns (128-byte
  // swizzle) or 32 x 32 (64-byte swizzle, EPI_APPLY_MIXED): the output, and
  // the one or two inputs (EPI_POLY: the b*A source; EPI_APPLY_MIXED: the
  // iterate's hi half, and its lo half, which is also written).
  CUtensorMap map_eo[MAX_GROUPS];
  CUtensorMap map_ei[MAX_GROUPS];
  CUtensorMap map_ei2[MAX_GROUPS];
  GemmGroup g[MAX_GROUPS];
  int num_groups;
  long long total_tiles;
  int* err;
};
static_assert(sizeof(GemmParams) <= 4096, "kernel parameters must fit the classic 4 KiB limit");

// ------------------------------------------------------------------ tiling
// Tiles (i, j) of 256 rows x (256 << nshift) columns.  SYM keeps the tiles
// that reach the upper triangle (j >= i >> nshift); CAUSAL keeps those that
// reach the lower triangle including the diagonal (j <= i >> nshift).
__host__ __device__ inline long long sched_row_count(int sched, int i, int tiles_n, int nshift) {
  if (sched == SCHED_SYM) return tiles_n - (i >> nshift);
  if (sched == SCHED_CAUSAL) return ((i >> nshift) + 1) < tiles_n ? ((i >> nshift) + 1) : tiles_n;
  return tiles_n;
}
__host__ __device__ inline long long sched_tiles_per_prob(int sched, int tiles_m, int tiles_n, int nshift) {
  if (sched == SCHED_DENSE) return (long long)tiles_m * tiles_n;
  long long t = 0;
  for (int i = 0; i < tiles_m; ++i) t += sched_row_count(sched, i, tiles_n, nshift);
  return t;
}

struct TileInfo {
  int g, prob, tm, tn, num_kb;
};

// A symmetric-output tile of 256 rows x 512 columns whose first 256 columns
// lie wholly below the diagonal (odd tile rows, first kept tile): only its
// second N block holds kept entries, so the first block is neither loaded,
// multiplied nor drained.
template <int NB>
__host__ __device__ inline bool sym_skip_first_block(const GemmGroup& G, const TileInfo& ti) {
  return NB == 2 && G.sched == SCHED_SYM && 2 * ti.tn + 1 <= ti.tm;
}

__host__ __device__ inline void decode_tile(const GemmGroup* groups, int num_groups, long long t,
                                            TileInfo& ti) {
  int g = 0;
  while (g + 1 < num_groups && t >= groups[g + 1].tile_start) ++g;
  const GemmGroup& G = groups[g];
  long long local = t - G.tile_start;
  const long long prob = local / G.tiles_per_prob;
  long long tl = local - prob * G.tiles_per_prob;
  int tm = 0, tn = 0;
  if (G.sched == SCHED_DENSE) {
    const int band = G.band;
    const long long per_band = (long long)G.tiles_m * band;
    const int bidx = (int)(tl / per_band);
    const long long x = tl - (long long)bidx * per_band;
    const int rem = G.tiles_n - bidx * band;
    const int w = rem < band ? rem : band;
    tm = (int)(x / w);
    tn = bidx * band + (int)(x % w);
  } else {
    int i = 0;
    while (true) {
      const long long cnt = sched_row_count(G.sched, i, G.tiles_n, G.nshift);
      if (tl < cnt) break;
      tl -= cnt;
      ++i;
    }
    tm = i;
    tn = (G.sched == SCHED_SYM ? (i >> G.nshift) : 0) + (int)tl;
  }
  ti.g = g;
  ti.prob = (int)prob;
  ti.tm = tm;
  ti.tn = tn;
  ti.num_kb = (G.K + BK - 1) / BK;
}

// -------------------------------------------------------------- epilogues
__device__ __forceinline__ void load_bf16x16(const __nv_bfloat16* p, float (&x)[16]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
  uint4 a = q[0], b = q[1];
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void store_bf16x16(__nv_bfloat16* p, const float (&x)[16]) {
  uint4 a, b;
  a.x = pack_bf16x2(x[0], x[1]);
  a.y = pack_bf16x2(x[2], x[3]);
  a.z = pack_bf16x2(x[4], x[5]);
  a.w = pack_bf16x2(x[6], x[7]);
  b.x = pack_bf16x2(x[8], x[9]);
  b.y = pack_bf16x2(x[10], x[11]);
  b.z = pack_bf16x2(x[12], x[13]);
  b.w = pack_bf16x2(x[14], x[15]);
  uint4* q = reinterpret_cast<uint4*>(p);
  q[0] = a;
  q[1] = b;
}
__device__ __forceinline__ void load_f32x16(const float* p, float (&x)[16]) {
  const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 v = q[i];
    x[4 * i] = v.x;
    x[4 * i + 1] = v.y;
    x[4 * i + 2] = v.z;
    x[4 * i + 3] = v.w;
  }
}
__device__ __forceinline__ void store_f32x16(float* p, const float (&x)[16]) {
  float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) q[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}

// Symmetric store of one 16-column chunk of row r: element (r, c) with c >= r
// goes to (r, c) and, when c > r, also to (c, r).  Across a warp r runs over
// 32 consecutive rows, so each mirrored store is one 64-byte segment.
__device__ __forceinline__ void store_sym_chunk(__nv_bfloat16* D, long long ld, int M, int r, int c0,
                                                const float (&v)[16]) {
  if (r >= M) return;
  if (c0 >= r && c0 + 16 <= M) {
    store_bf16x16(D + (long long)r * ld + c0, v);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int c = c0 + j;
      if (c >= r && c < M) D[(long long)r * ld + c] = __float2bfloat16_rn(v[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int c = c0 + j;
    if (c > r && c < M) D[(long long)c * ld + r] = __float2bfloat16_rn(v[j]);
  }
}

// Each epilogue thread owns one row r of the tile and walks its columns in
// chunks of 16: the global operands of a chunk are requested first
// (epi_prefetch), then its accumulator columns are read from TMEM, so the two
// latencies overlap, then the chunk is finished (epi_finish).

// Global operands of one chunk, kept as raw 128-bit words until used:
// x = the b*A source (EPI_POLY, bf16: x[0..1]) or the iterate's hi and lo
// halves (EPI_APPLY* with xf_read: x[0..1] and x[2..3]); w = the weight
// (EPI_APPLY_FINAL, bf16 or fp32).
struct EpiPre {
  uint4 x[4];
  uint4 w[4];
};

// `valid` columns are in range; `vec`: the 16 elements may be read as two
// 16-byte words (aligned row and full chunk), else element by element.
__device__ __forceinline__ void raw_load_bf16x16(const __nv_bfloat16* p, int valid, bool vec, uint4& q0,
                                                 uint4& q1) {
  if (vec && valid >= 16) {
    const uint4* s = reinterpret_cast<const uint4*>(p);
    q0 = s[0];
    q1 = s[1];
  } else {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lo = (2 * i < valid) ? static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p + 2 * i)) : 0u;
      const uint32_t hi =
          (2 * i + 1 < valid) ? static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(p + 2 * i + 1)) : 0u;
      w[i] = lo | (hi << 16);
    }
    q0 = make_uint4(w[0], w[1], w[2], w[3]);
    q1 = make_uint4(w[4], w[5], w[6], w[7]);
  }
}
__device__ __forceinline__ void raw_load_bf16x16(const __nv_bfloat16* p, int valid, bool vec, uint4 (&q)[4]) {
  raw_load_bf16x16(p, valid, vec, q[0], q[1]);
}
__device__ __forceinline__ void raw_load_f32x16(const float* p, int valid, bool vec, uint4 (&q)[4]) {
  if (vec && valid >= 16) {
    const uint4* s = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = s[i];
  } else {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = (i < valid) ? __float_as_uint(p[i]) : 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) q[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
}
__device__ __forceinline__ void raw_to_bf16x16(const uint4 (&q)[4], float (&x)[16]) {
  const uint32_t w[8] = {q[0].x, q[0].y, q[0].z, q[0].w, q[1].x, q[1].y, q[1].z, q[1].w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
// hi + lo halves (x[0..1] and x[2..3], bf16 each) back to fp32; the sum is exact.
__device__ __forceinline__ void raw_hilo_to_f32x16(const uint4 (&q)[4], float (&x)[16]) {
  const uint32_t h[8] = {q[0].x, q[0].y, q[0].z, q[0].w, q[1].x, q[1].y, q[1].z, q[1].w};
  const uint32_t l[8] = {q[2].x, q[2].y, q[2].z, q[2].w, q[3].x, q[3].y, q[3].z, q[3].w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = __uint_as_float(h[i] << 16) + __uint_as_float(l[i] << 16);
    x[2 * i + 1] = __uint_as_float(h[i] & 0xFFFF0000u) + __uint_as_float(l[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void raw_to_f32x16(const uint4 (&q)[4], float (&x)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[4 * i] = __uint_as_float(q[i].x);
    x[4 * i + 1] = __uint_as_float(q[i].y);
    x[4 * i + 2] = __uint_as_float(q[i].z);
    x[4 * i + 3] = __uint_as_float(q[i].w);
  }
}

template <int EPI>
__device__ __forceinline__ void epi_prefetch(const GemmGroup& G, int prob, int r, int c0, EpiPre& pre) {
  if (r >= G.M) return;
  const int valid = G.N - c0;
  if (valid <= 0) return;
  if constexpr (EPI == EPI_POLY) {
    const __nv_bfloat16* S =
        static_cast<const __nv_bfloat16*>(G.src) + (long long)prob * G.src_bs + (long long)r * G.src_ld;
    raw_load_bf16x16(S + c0, valid, true, pre.x);
  } else if constexpr (is_apply_epi<EPI>()) {
    if (apply_reads_x<EPI>(G)) {
      const __nv_bfloat16* Xh = G.xh + (long long)prob * G.xh_bs + (long long)r * G.xh_ld;
      const __nv_bfloat16* Xl = G.xl + (long long)prob * G.xl_bs + (long long)r * G.xl_ld;
      raw_load_bf16x16(Xh + c0, valid, true, pre.x[0], pre.x[1]);
      raw_load_bf16x16(Xl + c0, valid, true, pre.x[2], pre.x[3]);
    }
    if constexpr (EPI == EPI_APPLY_FINAL) {
      const long long row = (long long)r * G.N;
      if (G.w_f32) {
        raw_load_f32x16(static_cast<const float*>(G.w_ptrs[prob]) + row + c0, valid, G.w_vec != 0, pre.w);
      } else {
        raw_load_bf16x16(static_cast<const __nv_bfloat16*>(G.w_ptrs[prob]) + row + c0, valid, G.w_vec != 0,
                         pre.w);
      }
    }
  }
}

template <int EPI>
__device__ __forceinline__ void epi_finish(const GemmGroup& G, int prob, int r, int c0, float* v,
                                           const EpiPre& pre, float& run_max) {
  const bool full = (r < G.M) && (c0 + 16 <= G.N);
  if constexpr (EPI == EPI_GRAM) {
    float s2 = 1.f;
    if (G.scale) {
      const float s = G.scale[G.prob_base + prob];
      s2 = s * s;
    }
    // s = 0 marks a non-finite NS input: its Gram is zero, not NaN
    float o[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j] = s2 == 0.f ? 0.f : v[j] * s2;
    __nv_bfloat16* D = static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs;
    store_sym_chunk(D, G.d_ld, G.M, r, c0, o);
  } else if constexpr (EPI == EPI_POLY) {
    if (r >= G.M) return;
    float x[16];
    raw_to_bf16x16(pre.x, x);
    float o[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j] = fmaf(G.coef_acc, v[j], G.coef_src * x[j]) + (c0 + j == r ? G.diag : 0.f);
    __nv_bfloat16* D = static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs;
    store_sym_chunk(D, G.d_ld, G.M, r, c0, o);
  } else if constexpr (is_apply_epi<EPI>()) {
    if (r >= G.M) return;
    const float s = G.scale ? G.scale[G.prob_base + prob] : 1.f;
    float o[16];
    if (apply_reads_x<EPI>(G)) {
      float x[16];
      raw_hilo_to_f32x16(pre.x, x);
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = s * fmaf(G.coef_src, x[j], v[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = s * v[j];
    }
    if (s == 0.f) {  // a non-finite NS input: the first iterate is zero, not NaN
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = 0.f;
    }
    if constexpr (EPI == EPI_APPLY || EPI == EPI_APPLY_MIXED) {
      float* X = G.xf_write ? G.xf + (long long)prob * G.xf_bs + (long long)r * G.xf_ld : nullptr;
      __nv_bfloat16* XL = G.xl_write ? G.xl + (long long)prob * G.xl_bs + (long long)r * G.xl_ld : nullptr;
      __nv_bfloat16* D =
          static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs + (long long)r * G.d_ld;
      float lo[16];
      if (G.xl_write) {
#pragma unroll
        for (int j = 0; j < 16; ++j) lo[j] = o[j] - __bfloat162float(__float2bfloat16_rn(o[j]));
      }
      if (full) {
        if (G.xf_write) store_f32x16(X + c0, o);
        if (G.xl_write) store_bf16x16(XL + c0, lo);
        if (!G.xf_write) store_bf16x16(D + c0, o);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (c0 + j < G.N) {
            if (G.xf_write) X[c0 + j] = o[j];
            if (G.xl_write) XL[c0 + j] = __float2bfloat16_rn(lo[j]);
            if (!G.xf_write) D[c0 + j] = __float2bfloat16_rn(o[j]);
          }
      }
    } else {
      const long long row = (long long)r * G.N;
      float* U = G.u_ptrs ? G.u_ptrs[prob] : nullptr;
      if (U) {
        float u[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) u[j] = G.rms * o[j];
        if (full && (G.N % 4 == 0)) {
          store_f32x16(U + row + c0, u);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < G.N) U[row + c0 + j] = u[j];
        }
      }
      float w[16];
      if (G.w_f32) {
        raw_to_f32x16(pre.w, w);
      } else {
        raw_to_bf16x16(pre.w, w);
      }
      float nw[16], decay, step;
      final_coefs(G, decay, step);
#pragma unroll
      for (int j = 0; j < 16; ++j) nw[j] = fmaf(step, o[j], decay * w[j]);
      if (G.w_f32) {
        float* W = static_cast<float*>(G.w_ptrs[prob]) + row;
        if (full && G.w_vec) {
          store_f32x16(W + c0, nw);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < G.N) W[c0 + j] = nw[j];
        }
      } else {
        __nv_bfloat16* W = static_cast<__nv_bfloat16*>(G.w_ptrs[prob]) + row;
        if (full && G.w_vec) {
          store_bf16x16(W + c0, nw);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < G.N) W[c0 + j] = __float2bfloat16_rn(nw[j]);
        }
      }
    }
  } else if constexpr (EPI == EPI_STORE) {
    if (r >= G.M) return;
    __nv_bfloat16* D =
        static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs + (long long)r * G.d_ld;
    if (full) {
      store_bf16x16(D + c0, *reinterpret_cast<const float(*)[16]>(v));
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c0 + j < G.N) D[c0 + j] = __float2bfloat16_rn(v[j]);
    }
  } else if constexpr (EPI == EPI_CAUSALMAX) {
    if (r >= G.M) return;
    if (c0 + 16 <= G.N && (!G.mask_causal || c0 + 15 <= r)) {
      // Whole chunk inside the mask and the bounds: a tree of three-input
      // maxima (8 instructions for 16 scores), no compares.
      const float a0 = fmax3(v[0], v[1], v[2]), a1 = fmax3(v[3], v[4], v[5]), a2 = fmax3(v[6], v[7], v[8]);
      const float a3 = fmax3(v[9], v[10], v[11]), a4 = fmax3(v[12], v[13], v[14]);
      run_max = fmax3(run_max, fmax3(a0, a1, a2), fmax3(a3, a4, v[15]));
    } else {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int c = c0 + j;
        const bool ok = (c < G.N) && (!G.mask_causal || c <= r);
        if (ok) run_max = fmaxf(run_max, v[j]);
      }
    }
  }
}

// ---------------------------------------------------- coalesced row blocks
// The accumulator gives each epilogue thread one row of the tile, so a warp's
// 16-byte accesses to global memory would each touch 32 rows (32 L1
// wavefronts).  Whole blocks of 32 rows x 64 bf16 columns go through the
// warp's shared-memory buffer instead: global memory is read and written four
// 128-byte row segments per warp instruction, and each thread reads or writes
// its own row in shared memory.  The buffer's 16-byte chunks are XOR-swizzled
// by row, so neither side has bank conflicts.
__device__ __forceinline__ uint32_t epi_swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// Fragments of rows 0..31, columns 0..63 of the block at `base` (row stride
// ld elements): fragment k of lane l is row 4k + l/8, columns 8(l%8)..+7.
__device__ __forceinline__ void warp_issue_rows64(const __nv_bfloat16* base, long long ld, int lane, uint4 (&g)[8]) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    g[k] = *reinterpret_cast<const uint4*>(base + (long long)(4 * k + (lane >> 3)) * ld + (lane & 7) * 8);
}

// The fragments, regrouped so that lane l holds row l: out[i] = columns 2i, 2i+1.
__device__ __forceinline__ void warp_rows_from_frags(const uint4 (&g)[8], int lane, uint8_t* buf, uint32_t (&out)[32]) {
#pragma unroll
  for (int k = 0; k < 8; ++k) *reinterpret_cast<uint4*>(buf + epi_swz(4 * k + (lane >> 3), lane & 7)) = g[k];
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(buf + epi_swz(lane, c));
    out[4 * c] = v.x;
    out[4 * c + 1] = v.y;
    out[4 * c + 2] = v.z;
    out[4 * c + 3] = v.w;
  }
  __syncwarp();
}

// Lane l's row `in` (bf16 pairs) to row l of the block at `base`.
__device__ __forceinline__ void warp_store_rows64(__nv_bfloat16* base, long long ld, int lane, uint8_t* buf,
                                                  const uint32_t (&in)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4*>(buf + epi_swz(lane, c)) = make_uint4(in[4 * c], in[4 * c + 1], in[4 * c + 2], in[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int k0 = 0; k0 < 8; k0 += 4) {  // four fragments at a time (registers)
    uint4 g[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      g[k] = *reinterpret_cast<const uint4*>(buf + epi_swz(4 * (k0 + k) + (lane >> 3), lane & 7));
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<uint4*>(base + (long long)(4 * (k0 + k) + (lane >> 3)) * ld + (lane & 7) * 8) = g[k];
  }
  __syncwarp();
}

// The same for blocks of 32 rows x 32 columns (64-byte rows; 2 KiB of the
// buffer), for the epilogue that holds two operands: fragment k of lane l is
// row 8k + l/4, columns 8(l%4)..+7; chunks are swizzled by (row / 2) % 4.
__device__ __forceinline__ uint32_t epi_swz32(int row, int chunk) {
  return static_cast<uint32_t>(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}
// One warp's 32 rows x 32 fp32 columns (each thread's `in` is its own row)
// to global memory: own row into the buffer (128 bytes, swizzled chunks),
// then four 128-byte row segments per warp store.
__device__ __forceinline__ void warp_store_rows32f(float* base, long long ld, int lane, uint8_t* buf,
                                                   const float* in) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<float4*>(buf + epi_swz(lane, c)) = make_float4(in[4 * c], in[4 * c + 1], in[4 * c + 2], in[4 * c + 3]);
  __syncwarp();
#pragma unroll
  for (int k0 = 0; k0 < 8; k0 += 4) {
    float4 g[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      g[k] = *reinterpret_cast<const float4*>(buf + epi_swz(4 * (k0 + k) + (lane >> 3), lane & 7));
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<float4*>(base + (long long)(4 * (k0 + k) + (lane >> 3)) * ld + (lane & 7) * 4) = g[k];
  }
  __syncwarp();
}

__device__ __forceinline__ void warp_issue_rows32(const __nv_bfloat16* base, long long ld, int lane, uint4 (&g)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k)
    g[k] = *reinterpret_cast<const uint4*>(base + (long long)(8 * k + (lane >> 2)) * ld + (lane & 3) * 8);
}
__device__ __forceinline__ void warp_rows_from_frags32(const uint4 (&g)[4], int lane, uint8_t* buf, uint32_t (&out)[16]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(buf + epi_swz32(8 * k + (lane >> 2), lane & 3)) = g[k];
  __syncwarp();
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(buf + epi_swz32(lane, c));
    out[4 * c] = v.x;
    out[4 * c + 1] = v.y;
    out[4 * c + 2] = v.z;
    out[4 * c + 3] = v.w;
  }
  __syncwarp();
}
__device__ __forceinline__ void warp_store_rows32(__nv_bfloat16* base, long long ld, int lane, uint8_t* buf,
                                                  const uint32_t (&in)[16]) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(buf + epi_swz32(lane, c)) = make_uint4(in[4 * c], in[4 * c + 1], in[4 * c + 2], in[4 * c + 3]);
  __syncwarp();
  uint4 g[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) g[k] = *reinterpret_cast<const uint4*>(buf + epi_swz32(8 * k + (lane >> 2), lane & 3));
#pragma unroll
  for (int k = 0; k < 4; ++k)
    *reinterpret_cast<uint4*>(base + (long long)(8 * k + (lane >> 2)) * ld + (lane & 3) * 8) = g[k];
  __syncwarp();
}

__device__ __forceinline__ void pack_row64(const float (&o)[64], uint32_t (&out)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) out[i] = pack_bf16x2(o[2 * i], o[2 * i + 1]);
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Whether a warp's 32 x 64 block (rows r0.., columns c0..) takes the
// coalesced path: every row and column in range, rows 16-byte aligned, no
// fp32 operand, and for the symmetric outputs every column strictly above
// every row (the block's elements are all stored directly and mirrored).
// Columns of the blocks that take the coalesced path: 32 for the epilogue that
// holds two operands (EPI_APPLY_MIXED), 64 for the others.
template <int EPI>
__host__ __device__ constexpr int epi_fast_cols() {
  return EPI == EPI_APPLY_MIXED ? 32 : 64;
}

template <int EPI>
__device__ __forceinline__ bool epi_fast_ok(const GemmGroup& G, int prob, int r0, int c0) {
  if (r0 + 32 > G.M || c0 + epi_fast_cols<EPI>() > G.N) return false;
  if constexpr (EPI == EPI_GRAM || EPI == EPI_POLY) {
    if (c0 <= r0 + 31 || (G.d_ld & 7) != 0) return false;
    if constexpr (EPI == EPI_POLY) {
      if ((G.src_ld & 7) != 0) return false;
    }
    return true;
  } else if constexpr (EPI == EPI_APPLY || EPI == EPI_APPLY_MIXED) {
    if ((G.d_ld & 7) != 0 || (G.xl_write && (G.xl_ld & 7) != 0)) return false;
    if (G.xf_write && (EPI == EPI_APPLY_MIXED || G.tma_epi || (G.xf_ld & 3) != 0)) return false;
    if (EPI == EPI_APPLY_MIXED && ((G.xh_ld | G.xl_ld) & 7) != 0) return false;
    return true;
  } else if constexpr (EPI == EPI_APPLY_FINAL) {
    return !G.xf_read && !G.w_f32 && G.w_vec && !(G.u_ptrs && G.u_ptrs[prob]);
  } else if constexpr (EPI == EPI_STORE) {
    return (G.d_ld & 7) == 0;
  } else {
    return false;
  }
}

// The epilogue of one warp's 32 x 64 block through the coalesced path (see
// epi_finish for what each epilogue computes; EPI_APPLY_MIXED has its own,
// epi_fast32_mixed).  The block's global operand is requested first, then its
// accumulator columns are read from TMEM.
template <int EPI>
__device__ __forceinline__ void epi_fast64(const GemmGroup& G, int prob, int r0, int c0, int lane, uint32_t taddr,
                                           uint8_t* buf) {
  static_assert(EPI != EPI_APPLY_MIXED, "the mixed apply uses epi_fast32_mixed");
  if (lane == 0) bulk_wait_read_all();  // no tensor store of the warp still reads the buffer
  __syncwarp();
  uint4 ga[8];
  if constexpr (EPI == EPI_POLY) {
    warp_issue_rows64(static_cast<const __nv_bfloat16*>(G.src) + (long long)prob * G.src_bs + (long long)r0 * G.src_ld + c0,
                      G.src_ld, lane, ga);
  } else if constexpr (EPI == EPI_APPLY_FINAL) {
    warp_issue_rows64(static_cast<const __nv_bfloat16*>(G.w_ptrs[prob]) + (long long)r0 * G.N + c0, G.N, lane, ga);
  }
  float v[64];  // the accumulator columns, turned into the block's outputs in place
  tmem_ld64(taddr, v);
  uint32_t pk[32];
  if constexpr (EPI == EPI_GRAM) {
    float s2 = 1.f;
    if (G.scale) {
      const float sc = G.scale[G.prob_base + prob];
      s2 = sc * sc;
    }
#pragma unroll
    for (int j = 0; j < 64; ++j) v[j] = s2 == 0.f ? 0.f : v[j] * s2;
  } else if constexpr (EPI == EPI_POLY) {
    uint32_t x[32];
    warp_rows_from_frags(ga, lane, buf, x);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      v[2 * i] = fmaf(G.coef_acc, v[2 * i], G.coef_src * bf16_lo(x[i]));
      v[2 * i + 1] = fmaf(G.coef_acc, v[2 * i + 1], G.coef_src * bf16_hi(x[i]));
    }
  } else if constexpr (is_apply_epi<EPI>()) {
    const float sc = G.scale ? G.scale[G.prob_base + prob] : 1.f;
    {
#pragma unroll
      for (int j = 0; j < 64; ++j) v[j] = sc * v[j];
    }
    if (sc == 0.f) {  // a non-finite NS input: the first iterate is zero, not NaN
#pragma unroll
      for (int j = 0; j < 64; ++j) v[j] = 0.f;
    }
  }

  if constexpr (EPI == EPI_GRAM || EPI == EPI_POLY) {
    __nv_bfloat16* D = static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs;
    pack_row64(v, pk);
    warp_store_rows64(D + (long long)r0 * G.d_ld + c0, G.d_ld, lane, buf, pk);
    // the mirror image: column c0+j of rows r0..r0+31 is one 64-byte segment
    // of row c0+j, written by the warp in one store
    unsigned short* pm = reinterpret_cast<unsigned short*>(D + (long long)c0 * G.d_ld + r0 + lane);
    const long long ld = G.d_ld;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      pm[0] = static_cast<unsigned short>(pk[i] & 0xFFFFu);
      pm[ld] = static_cast<unsigned short>(pk[i] >> 16);
      pm += 2 * ld;
    }
  } else if constexpr (EPI == EPI_APPLY) {
    if (G.xf_write) {
      // the NS output in fp32 (NorMuon's row pass reads it), two 32-column
      // halves; nothing reads a bf16 copy of the last iterate
      float* X = G.xf + (long long)prob * G.xf_bs + (long long)r0 * G.xf_ld + c0;
      warp_store_rows32f(X, G.xf_ld, lane, buf, v);
      warp_store_rows32f(X + 32, G.xf_ld, lane, buf, v + 32);
    } else {
      __nv_bfloat16* D = static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs + (long long)r0 * G.d_ld + c0;
      pack_row64(v, pk);
      warp_store_rows64(D, G.d_ld, lane, buf, pk);
    }
  } else if constexpr (EPI == EPI_APPLY_FINAL) {
    warp_rows_from_frags(ga, lane, buf, pk);
    float decay, step;
    final_coefs(G, decay, step);
#pragma unroll
    for (int i = 0; i < 32; ++i)
      pk[i] = pack_bf16x2(fmaf(step, v[2 * i], decay * bf16_lo(pk[i])),
                          fmaf(step, v[2 * i + 1], decay * bf16_hi(pk[i])));
    warp_store_rows64(static_cast<__nv_bfloat16*>(G.w_ptrs[prob]) + (long long)r0 * G.N + c0, G.N, lane, buf, pk);
  } else if constexpr (EPI == EPI_STORE) {
    pack_row64(v, pk);
    warp_store_rows64(static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs + (long long)r0 * G.d_ld + c0,
                      G.d_ld, lane, buf, pk);
  }
}

// EPI_APPLY_MIXED through the coalesced path, a 32 x 32 block: X' = s(aX + BX)
// with aX from the iterate's hi and lo halves, stored as bf16 (and its lo
// half when flagged).
__device__ __forceinline__ void epi_fast32_mixed(const GemmGroup& G, int prob, int r0, int c0, int lane,
                                                 uint32_t taddr, uint8_t* buf) {
  if (lane == 0) bulk_wait_read_all();  // no tensor store of the warp still reads the buffer
  __syncwarp();
  uint4 gh[4], gl[4];
  warp_issue_rows32(G.xh + (long long)prob * G.xh_bs + (long long)r0 * G.xh_ld + c0, G.xh_ld, lane, gh);
  warp_issue_rows32(G.xl + (long long)prob * G.xl_bs + (long long)r0 * G.xl_ld + c0, G.xl_ld, lane, gl);
  float v[32];
  tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(v));
  tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(v + 16));
  uint32_t xh[16], xl[16];
  warp_rows_from_frags32(gh, lane, buf, xh);
  warp_rows_from_frags32(gl, lane, buf, xl);
  const float sc = G.scale ? G.scale[G.prob_base + prob] : 1.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[2 * i] = sc * fmaf(G.coef_src, bf16_lo(xh[i]) + bf16_lo(xl[i]), v[2 * i]);
    v[2 * i + 1] = sc * fmaf(G.coef_src, bf16_hi(xh[i]) + bf16_hi(xl[i]), v[2 * i + 1]);
  }
  if (sc == 0.f) {  // a non-finite NS input: the first iterate is zero, not NaN
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = 0.f;
  }
  // hi = bf16(o) and lo = bf16(o - hi)
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    xh[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    xl[i] = pack_bf16x2(v[2 * i] - bf16_lo(xh[i]), v[2 * i + 1] - bf16_hi(xh[i]));
  }
  warp_store_rows32(static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs + (long long)r0 * G.d_ld + c0, G.d_ld,
                    lane, buf, xh);
  if (G.xl_write)
    warp_store_rows32(G.xl + (long long)prob * G.xl_bs + (long long)r0 * G.xl_ld + c0, G.xl_ld, lane, buf, xl);
}

// The coalesced path with tensor copies, for groups that carry epilogue maps:
// the block's inputs arrive by TMA loads into the warp's buffer (completing on
// the warp's barrier `ebar`) and its outputs leave by a TMA store from it, so
// the global side takes no load or store instructions; each thread only reads
// and writes its own row of the buffer (the buffer's swizzle is the maps'
// 128- or 64-byte swizzle).  Returns false if the loads' wait timed out.
template <int EPI>
__device__ __forceinline__ bool epi_tma_block(const GemmParams& P, int gi, const GemmGroup& G, int prob, int r0, int c0,
                                              int lane, uint32_t taddr, uint8_t* buf, uint32_t ebar, uint32_t& ephase,
                                              bool& load_pending, volatile int* abort_flag) {
  constexpr int COLS = epi_fast_cols<EPI>();
  constexpr int NLOAD = EPI == EPI_APPLY_MIXED ? 2 : (EPI == EPI_POLY ? 1 : 0);
  const uint32_t sbuf = smem_u32(buf);
  if (lane == 0) {
    bulk_wait_read_all();  // the previous block's store has read the buffer
    if constexpr (NLOAD > 0) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(ebar, uint32_t(NLOAD) * 32u * COLS * 2u);
      tma_load_3d(sbuf, &P.map_ei[gi], ebar, c0, r0, prob);
      if constexpr (NLOAD == 2) tma_load_3d(sbuf + 2048, &P.map_ei2[gi], ebar, c0, r0, prob);
    }
  }
  if constexpr (NLOAD > 0) load_pending = true;
  __syncwarp();
  float v[COLS];
  if constexpr (COLS == 64) {
    tmem_ld64(taddr, v);
  } else {
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(v));
    tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(v + 16));
  }
  if constexpr (NLOAD > 0) {
    const bool got = wait_bounded(ebar, ephase, abort_flag, P.err);
    if (!__all_sync(0xffffffffu, got)) return false;
    ephase ^= 1;
    load_pending = false;
  }
  uint32_t pk[COLS / 2];
  if constexpr (EPI == EPI_GRAM) {
    float s2 = 1.f;
    if (G.scale) {
      const float sc = G.scale[G.prob_base + prob];
      s2 = sc * sc;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(s2 == 0.f ? 0.f : v[2 * i] * s2, s2 == 0.f ? 0.f : v[2 * i + 1] * s2);
  } else if constexpr (EPI == EPI_POLY) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint4 x = *reinterpret_cast<const uint4*>(buf + epi_swz(lane, c));
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = 4 * c + t;
        pk[i] = pack_bf16x2(fmaf(G.coef_acc, v[2 * i], G.coef_src * bf16_lo(xs[t])),
                            fmaf(G.coef_acc, v[2 * i + 1], G.coef_src * bf16_hi(xs[t])));
      }
    }
  } else if constexpr (EPI == EPI_APPLY) {
    const float sc = G.scale ? G.scale[G.prob_base + prob] : 1.f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
      pk[i] = sc == 0.f ? 0u : pack_bf16x2(sc * v[2 * i], sc * v[2 * i + 1]);
  } else if constexpr (EPI == EPI_APPLY_MIXED) {
    const float sc = G.scale ? G.scale[G.prob_base + prob] : 1.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 h = *reinterpret_cast<const uint4*>(buf + epi_swz32(lane, c));
      const uint4 l = *reinterpret_cast<const uint4*>(buf + 2048 + epi_swz32(lane, c));
      const uint32_t hs[4] = {h.x, h.y, h.z, h.w}, ls[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = 4 * c + t;
        v[2 * i] = sc * fmaf(G.coef_src, bf16_lo(hs[t]) + bf16_lo(ls[t]), v[2 * i]);
        v[2 * i + 1] = sc * fmaf(G.coef_src, bf16_hi(hs[t]) + bf16_hi(ls[t]), v[2 * i + 1]);
      }
    }
    if (sc == 0.f) {  // a non-finite NS input: the first iterate is zero, not NaN
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  } else {  // EPI_STORE
#pragma unroll
    for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
  }
  // own row of the outputs into the buffer, then one tensor store per output
  if constexpr (COLS == 64) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(buf + epi_swz(lane, c)) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4*>(buf + epi_swz32(lane, c)) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    if constexpr (EPI == EPI_APPLY_MIXED) {
      if (G.xl_write) {
        uint32_t lo[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int i = 4 * c + t;
            lo[t] = pack_bf16x2(v[2 * i] - bf16_lo(pk[i]), v[2 * i + 1] - bf16_hi(pk[i]));
          }
          *reinterpret_cast<uint4*>(buf + 2048 + epi_swz32(lane, c)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(&P.map_eo[gi], sbuf, c0, r0, prob);
    if constexpr (EPI == EPI_APPLY_MIXED) {
      if (G.xl_write) tma_store_3d(&P.map_ei2[gi], sbuf + 2048, c0, r0, prob);
    }
    bulk_commit_group();
  }
  if constexpr (EPI == EPI_GRAM || EPI == EPI_POLY) {
    // the mirror image, as in epi_fast64
    __nv_bfloat16* D = static_cast<__nv_bfloat16*>(G.d) + (long long)prob * G.d_bs;
    unsigned short* pm = reinterpret_cast<unsigned short*>(D + (long long)c0 * G.d_ld + r0 + lane);
    const long long ld = G.d_ld;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      pm[0] = static_cast<unsigned short>(pk[i] & 0xFFFFu);
      pm[ld] = static_cast<unsigned short>(pk[i] >> 16);
      pm += 2 * ld;
    }
  }
  return true;
}

// Chunks per batch.  One for the NS phases: measured against batches of four
// chunks (one 64-column TMEM load, all global loads issued first) on the same
// GPU, the single-chunk drain was as fast or faster.  Eight for the causal
// max (a warp's whole 128 columns: two TMEM loads in flight, one wait), whose
// epilogue has no global operands and is bound by the TMEM load latency.
template <int EPI>
struct EpiBatch {
  static constexpr int CH = (EPI == EPI_CAUSALMAX) ? 8 : 1;
};

// ------------------------------------------------------------------ kernel
template <int EPI, int WIDE>
__global__ void __launch_bounds__(GEMM_THREADS, 1) umma_gemm_kernel(const __grid_constant__ GemmParams P) {
  using T = TileCfg<WIDE>;
  constexpr int STAGES = T::STAGES;
  constexpr int NACC = T::NACC;
  constexpr uint32_t STAGE_BYTES = T::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // [stages][epilogue row buffers (1 KiB-aligned, 4 KiB per warp)][barriers][head maxima]
  constexpr size_t BUF_BYTES = epi_uses_row_buffers<EPI>() ? size_t(NUM_EPI_WARPS) * EPI_BUF_BYTES : 0;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + BUF_BYTES);
  uint64_t* full_bar = bars;                          // [STAGES]  used in the leader only
  uint64_t* empty_bar = bars + STAGES;                // [STAGES]  every CTA
  uint64_t* tfull_bar = bars + 2 * STAGES;            // [NACC]    every CTA
  uint64_t* tempty_bar = bars + 2 * STAGES + NACC;    // [NACC]    used in the leader only
  uint64_t* drain_bar = bars + 2 * STAGES + 2 * NACC; // [1]       leader
  uint64_t* epi_bar = drain_bar + 1;                  // [NUM_EPI_WARPS] epilogue tensor loads
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + NUM_EPI_WARPS);
  static_assert((2 * 6 + 2 * 2 + 1 + NUM_EPI_WARPS) * 8 + 8 <= GEMM_BARRIER_BYTES, "barrier block");
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* head_max = reinterpret_cast<int*>(smem + STAGES * STAGE_BYTES + BUF_BYTES + GEMM_BARRIER_BYTES);  // EPI_CAUSALMAX
  const int nheads_smem = (EPI == EPI_CAUSALMAX && P.g[0].heads <= SMEM_HEADS) ? P.g[0].heads : 0;
  for (int i = threadIdx.x; i < nheads_smem; i += blockDim.x) head_max[i] = INT_MIN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0 = leader (issues the MMAs)
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < NACC; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), 2 * NUM_EPI_WARPS);
    }
    mbar_init(smem_u32(drain_bar), 1);
    for (int w = 0; w < NUM_EPI_WARPS; ++w) mbar_init(smem_u32(&epi_bar[w]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int g = 0; g < P.num_groups; ++g) {
      prefetch_tmap(&P.map_a[g]);
      prefetch_tmap(&P.map_b[g]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touches only the parameters, shared memory and TMEM, so
  // it may overlap the previous kernel's last tiles; no global memory is read
  // or written before that kernel has completed.
  griddep_launch_dependents();
  griddep_wait();
  const long long total = P.total_tiles;
  const long long first_tile = blockIdx.x >> 1;
  const long long tile_step = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0;          // leader: bit s set once stage s was filled
      uint32_t fill_parity = 0;     // leader: parity of stage s's latest fill
      bool ok = true;
      for (long long t = first_tile; ok && t < total; t += tile_step) {
        TileInfo ti;
        decode_tile(P.g, P.num_groups, t, ti);
        const GemmGroup& G = P.g[ti.g];
        const CUtensorMap* ma = &P.map_a[ti.g];
        const CUtensorMap* mb = &P.map_b[ti.g];
        const int m0 = ti.tm * BM + HALF * static_cast<int>(rank);
        const int n0 = ti.tn * T::N + HALF * static_cast<int>(rank);
        for (int kb0 = 0; kb0 < ti.num_kb; kb0 += T::KPS) {
          const int nk = ti.num_kb - kb0 < T::KPS ? ti.num_kb - kb0 : T::KPS;
          if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_u32(&full_bar[stage]);
          const bool skip0 = sym_skip_first_block<T::NB>(G, ti);
          if (leader) {
            // both CTAs of the pair skip the same block (it depends on the tile only)
            mbar_arrive_expect_tx(fb_local, uint32_t(nk) * (skip0 ? T::PAIR_KB_BYTES - 2 * B_STAGE_BYTES
                                                                   : T::PAIR_KB_BYTES));
            filled |= 1u << stage;
            fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t fb = mapa_shared(fb_local, 0);
          for (int j = 0; j < nk; ++j) {
            const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES + j * T::KB_BYTES);
            const int k0 = (kb0 + j) * BK;
            if (G.layout == LAYOUT_HEADS) {
              const int bb = ti.prob / G.heads, hh = ti.prob % G.heads;
              // A split contraction concatenates two per-head operand pairs along K
              // (MLA's content and rotary parts); the second key operand has one
              // head shared by all query heads.
              const bool second = G.k_split > 0 && k0 >= G.k_split;
              const CUtensorMap* qa = second ? &P.map_a[1] : ma;
              const CUtensorMap* kb_map = second ? &P.map_b[1] : mb;
              const int kk = second ? k0 - G.k_split : k0;
              const int hk = second ? 0 : hh;
              tma_load_4d_pair(sa, qa, fb, kk, hh, m0, bb);
#pragma unroll
              for (int h = 0; h < T::NB; ++h)
                tma_load_4d_pair(sa + A_STAGE_BYTES + h * B_STAGE_BYTES, kb_map, fb, kk, hk, n0 + h * MMA_N, bb);
            } else {
              if (!G.a_mn) {
                tma_load_3d_pair(sa, ma, fb, k0, m0, ti.prob);
              } else {
                tma_load_3d_pair(sa, ma, fb, m0, k0, ti.prob);
                tma_load_3d_pair(sa + MN_BOX_BYTES, ma, fb, m0 + 64, k0, ti.prob);
              }
#pragma unroll
              for (int h = 0; h < T::NB; ++h) {
                if (h == 0 && skip0) continue;
                const uint32_t sb = sa + A_STAGE_BYTES + h * B_STAGE_BYTES;
                const int nh = n0 + h * MMA_N;
                if (!G.b_mn) {
                  tma_load_3d_pair(sb, mb, fb, k0, nh, ti.prob);
                } else {
                  tma_load_3d_pair(sb, mb, fb, nh, k0, ti.prob);
                  tma_load_3d_pair(sb + MN_BOX_BYTES, mb, fb, nh + 64, k0, ti.prob);
                }
              }
            }
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // The leader's full barriers count both CTAs' copies: wait for every
      // copy of the pair to land before anyone leaves.
      if (leader)
        for (int s = 0; s < STAGES; ++s)
          if (filled & (1u << s)) {
            volatile int no_abort = 0;
            wait_bounded(smem_u32(&full_bar[s]), (fill_parity >> s) & 1u, &no_abort, nullptr, kDrainLimitCycles);
          }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t s0 = smem_u32(smem);
      for (long long t = first_tile; ok && t < total; t += tile_step) {
        TileInfo ti;
        decode_tile(P.g, P.num_groups, t, ti);
        const GemmGroup& G = P.g[ti.g];
        const uint32_t idesc = idesc_bf16_f32(BM, MMA_N, G.a_mn, G.b_mn);
        const uint32_t a_lbo = G.a_mn ? MN_BOX_BYTES : 16u;
        const uint32_t b_lbo = G.b_mn ? MN_BOX_BYTES : 16u;
        const uint32_t a_kstep = G.a_mn ? 16u * 128u : 32u;
        const uint32_t b_kstep = G.b_mn ? 16u * 128u : 32u;
        if (!wait_bounded(smem_u32(&tempty_bar[acc]), acc_phase ^ 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * T::N;
        // Descriptors of stage 0; the stage, the k-step and the B block only
        // move the start-address field (address >> 4 in the low 14 bits, no
        // carry out of it since shared memory ends below 2^18).
        const uint64_t ad0 = smem_desc_sw128(s0, a_lbo, 1024);
        const uint64_t bd0 = smem_desc_sw128(s0 + A_STAGE_BYTES, b_lbo, 1024);
        const bool skip0 = sym_skip_first_block<T::NB>(G, ti);
        for (int kb0 = 0; kb0 < ti.num_kb; kb0 += T::KPS) {
          const int nk = ti.num_kb - kb0 < T::KPS ? ti.num_kb - kb0 : T::KPS;
          // The TMA writes are made visible by the barrier's complete_tx; the
          // MMAs read them through the same async proxy.
          if (!wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, P.err)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int j = 0; j < T::KPS; ++j) {
            if (j >= nk) break;
            const uint64_t soff = static_cast<uint64_t>((stage * STAGE_BYTES + j * T::KB_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t ad = ad0 + soff + ((kk * a_kstep) >> 4);
#pragma unroll
              for (int h = 0; h < T::NB; ++h) {
                if (h == 0 && skip0) continue;
                const uint64_t bd = bd0 + soff + ((h * B_STAGE_BYTES + kk * b_kstep) >> 4);
                umma_bf16_pair(d_tmem + h * MMA_N, ad, bd, idesc, ((kb0 + j) | kk) != 0);
              }
            }
          }
          umma_commit_pair_mc(smem_u32(&empty_bar[stage]), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair_mc(smem_u32(&tfull_bar[acc]), 0x3);
        if (++acc == NACC) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // Every MMA of the pair completes before TMEM is released.
      umma_commit_pair(smem_u32(drain_bar));
      volatile int no_abort = 0;
      wait_bounded(smem_u32(drain_bar), 0, &no_abort, nullptr, kDrainLimitCycles);
    }
  } else {
    // ------------------------------------------------------- epilogue
    constexpr int WCOLS = T::N / EPI_COL_GROUPS;  // columns per epilogue warp
    const int q = warp & 3;                       // TMEM lane quarter this warp may read
    const int half = (warp - 2) >> 2;             // which column group of the tile
    uint8_t* epi_buf = smem + STAGES * STAGE_BYTES + (warp - 2) * EPI_BUF_BYTES;
    const uint32_t ebar = smem_u32(&epi_bar[warp - 2]);
    uint32_t ephase = 0;
    bool load_pending = false;
    uint32_t tempty_leader[NACC];
#pragma unroll
    for (int b = 0; b < NACC; ++b) tempty_leader[b] = mapa_shared(smem_u32(&tempty_bar[b]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (long long t = first_tile; t < total; t += tile_step) {
      TileInfo ti;
      decode_tile(P.g, P.num_groups, t, ti);
      const GemmGroup& G = P.g[ti.g];
      // Every lane waits; the warp proceeds only if all lanes saw the phase
      // complete, so a timeout can never split the warp before the
      // warp-collective TMEM loads below.
      const bool ok = wait_bounded(smem_u32(&tfull_bar[acc]), acc_phase, abort_flag, P.err);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int r = ti.tm * BM + HALF * static_cast<int>(rank) + q * 32 + lane;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * T::N + half * WCOLS;
      float run_max = -INFINITY;
      constexpr int CH = EpiBatch<EPI>::CH;
      // With two column groups, group 0 is exactly the first N block.
      static_assert(T::NB == 1 || EPI_COL_GROUPS == T::NB, "column groups match the N blocks");
      const bool idle = half == 0 && sym_skip_first_block<T::NB>(G, ti);
      const int cbase = ti.tn * T::N + half * WCOLS;
      // Last row of this warp: a chunk that starts beyond it lies above the
      // diagonal for every lane, as do all later chunks (causal max only).
      const int r_warp_last = ti.tm * BM + HALF * static_cast<int>(rank) + q * 32 + 31;
      const int r0w = r_warp_last - 31;             // first row of this warp
      bool tile_ok = true;                          // false: an epilogue load's wait timed out
#pragma unroll 1
      for (int cb = 0; cb < (idle ? 0 : WCOLS / 16); cb += CH) {
        if constexpr (EPI == EPI_CAUSALMAX) {
          if (G.mask_causal && cbase + cb * 16 > r_warp_last) break;
        }
        if constexpr (epi_uses_row_buffers<EPI>()) {
          // a whole 32-row block through the coalesced path when it can
          constexpr int FB = epi_fast_cols<EPI>() / 16;
          if (cb % FB == 0 && epi_fast_ok<EPI>(G, ti.prob, r0w, cbase + cb * 16)) {
            if constexpr (EPI != EPI_APPLY_FINAL) {
              if (G.tma_epi) {
                if (!epi_tma_block<EPI>(P, ti.g, G, ti.prob, r0w, cbase + cb * 16, lane, t_row + cb * 16, epi_buf, ebar,
                                        ephase, load_pending, abort_flag)) {
                  tile_ok = false;
                  break;
                }
                cb += FB - 1;
                continue;
              }
            }
            if constexpr (EPI == EPI_APPLY_MIXED) {
              epi_fast32_mixed(G, ti.prob, r0w, cbase + cb * 16, lane, t_row + cb * 16, epi_buf);
            } else {
              epi_fast64<EPI>(G, ti.prob, r0w, cbase + cb * 16, lane, t_row + cb * 16, epi_buf);
            }
            cb += FB - 1;
            continue;
          }
        }
        EpiPre pre[CH];
#pragma unroll
        for (int b = 0; b < CH; ++b) epi_prefetch<EPI>(G, ti.prob, r, cbase + (cb + b) * 16, pre[b]);
        float v[CH * 16];
        if constexpr (CH == 8) {
          tmem_ld128(t_row + cb * 16, v);
        } else if constexpr (CH == 4) {
          tmem_ld64(t_row + cb * 16, v);
        } else {
          static_assert(CH == 1, "one 16-, 64- or 128-column TMEM drain per batch");
          tmem_ld16(t_row + cb * 16, *reinterpret_cast<float(*)[16]>(v));
        }
#pragma unroll
        for (int b = 0; b < CH; ++b)
          epi_finish<EPI>(G, ti.prob, r, cbase + (cb + b) * 16, v + b * 16, pre[b], run_max);
      }
      if (!tile_ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
      if constexpr (EPI == EPI_CAUSALMAX) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) run_max = fmaxf(run_max, __shfl_xor_sync(0xffffffffu, run_max, o));
        if (lane == 0 && run_max > -INFINITY) {
          const int h = ti.prob % G.heads;
          const int key = float_to_ordered(run_max * G.out_scale);
          if (nheads_smem) {
            atomicMax(&head_max[h], key);
          } else {
            atomicMax(&G.keys[h], key);
          }
        }
      }
      if (++acc == NACC) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if constexpr (epi_uses_row_buffers<EPI>()) {
      // the warp's tensor stores complete, and a load abandoned on a timeout
      // lands, before the CTA's shared memory is released
      if (lane == 0) {
        bulk_wait_all();
        if (load_pending) {
          volatile int no_abort = 0;
          wait_bounded(ebar, ephase, &no_abort, nullptr, kDrainLimitCycles);
        }
      }
      __syncwarp();
    }
  }

  // Nobody leaves (or frees TMEM) while the peer may still signal this CTA's
  // barriers or read its shared memory.
  tc_fence_before();
  __syncthreads();
  if constexpr (EPI == EPI_CAUSALMAX) {
    for (int i = threadIdx.x; i < nheads_smem; i += blockDim.x)
      if (head_max[i] != INT_MIN) atomicMax(&P.g[0].keys[i], head_max[i]);
  }
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace mc
