// Per-head causal max of the pre-softmax logit with the query block held
// resident: S_max[h] = max over b, i and j <= i of (q_{b,i,h} . k_{b,j,h}) / sqrt(d)
// ("Muon and MuonClip: orthogonalised updates for LLM training", "The
// exploding-logit problem"; "MuonClip: speed, then stability", §05).
//
// A CTA pair owns one task (b, h, query block i of 256 rows: 128 per CTA) at
// a time, loads that block's Q once and keeps it in shared memory, then
// streams the key blocks j = 0 .. i (all blocks without the causal mask)
// through a ring of stages, one key block (all its k-blocks) per stage, so
// that one barrier round trip feeds a whole tile's MMAs.  Per key block the pair runs a
// 256 x 256 x d tile on the tensor cores (tcgen05, cta_group::2) into one of
// two TMEM accumulators, so the epilogue's max over one tile overlaps the
// next tile's MMAs.  Only the key blocks move per tile (half of what a tile
// that reloads both operands moves), and the per-head running max stays in
// registers for the whole task.  The score matrix is never stored.
//
// Tasks go head by head (all query blocks of one (b, h) in a row, the longest
// first under the causal mask), task t to pair t mod npairs, so the pairs that
// work on one head at the same time share its key blocks in L2.  The contraction may be split in two
// (multi-head latent attention: content columns [0, k_split) from operand
// slot 0, rotary columns from slot 1, whose key has one head shared by all).
//
// Warp roles (RM_THREADS per CTA), as in umma_gemm.cuh:
//   warp 0      TMA producer: the task's Q block, then the key k-blocks
//   warp 1      TMEM allocation; in the leader CTA one thread issues the MMAs
//   warps 2..   epilogue (RM_EPI_WARPS): warp w reads TMEM lanes 32*(w%4)..
//               and column group (w-2)/4 of the 256-column tile
// Every wait is bounded (wait_bounded); on a timeout the roles drain their
// in-flight copies and MMAs before TMEM is freed.
#pragma once

#include <climits>

#include "ptx.cuh"
#include "umma_gemm.cuh"

namespace mc {

constexpr int RM_STAGES_MAX = 8;
// Epilogue warps: four per TMEM lane quarter would give each 64 of a tile's
// 256 columns, two give each 128.
constexpr int RM_EPI_WARPS = 8;
constexpr int RM_THREADS = 64 + 32 * RM_EPI_WARPS;
constexpr int RM_COLS = MMA_N / (RM_EPI_WARPS / 4);  // columns per epilogue warp
static_assert(RM_EPI_WARPS % 4 == 0 && (RM_COLS == 64 || RM_COLS == 128), "epilogue split");
constexpr int RM_KB_MAX = 4;                 // contraction up to 256 columns
constexpr uint32_t RM_KB_BYTES = HALF * BK * 2;  // one CTA's 128 rows x 64 columns: 16 KiB

struct RowMaxParams {
  CUtensorMap map_q[2];  // [dims {d, H, S, B}, box {64, 1, 128, 1}]; slot 1: rotary part
  CUtensorMap map_k[2];
  int S, B, H;
  int nkb;               // k-blocks of 64 columns in the contraction
  int k_split;           // 0, or the first column taken from slot 1 (a multiple of 64)
  int stages;            // key ring depth in key blocks of nkb k-blocks, 1 <= stages <= RM_STAGES_MAX
  int causal;
  int nblk;              // ceil(S / 256)
  long long tasks;       // B * H * nblk
  float out_scale;       // 1 / sqrt(d)
  int* keys;             // per-head order-preserving ints (global)
  int* err;
};

// Shared memory: Q double buffer, key ring, barriers, per-head maxima.
__host__ __device__ constexpr size_t rowmax_smem_bytes(int nkb, int stages) {
  return 1024 + size_t(2 + stages) * nkb * RM_KB_BYTES + GEMM_BARRIER_BYTES + 4 * size_t(SMEM_HEADS);
}

struct RmTask {
  int b, h, i, jn;  // jn: key blocks of this task
};

// Task order: head-major takes all query blocks of one (b, h) in a row, so
// that the pairs working on one head at the same time share its key blocks in
// L2; level-major (false) takes every (b, h) at one query-block level before
// the next.  Measured on the B4 S4096 H32 dh128 layer: 0.272 against 0.273 ms.
constexpr bool kRowmaxHeadMajor = true;

__device__ __forceinline__ RmTask rowmax_task(const RowMaxParams& P, long long t) {
  const long long bh_count = (long long)P.B * P.H;
  const int level = kRowmaxHeadMajor ? static_cast<int>(t % P.nblk) : static_cast<int>(t / bh_count);
  const long long bh = kRowmaxHeadMajor ? t / P.nblk : t - (long long)level * bh_count;
  RmTask k;
  k.i = P.causal ? P.nblk - 1 - level : level;
  k.b = static_cast<int>(bh / P.H);
  k.h = static_cast<int>(bh % P.H);
  k.jn = P.causal ? k.i + 1 : P.nblk;
  return k;
}

__global__ void __launch_bounds__(RM_THREADS, 1) qk_rowmax_kernel(const __grid_constant__ RowMaxParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nkb = P.nkb, STG = P.stages;
  uint8_t* q_smem = smem;                                  // [2][nkb] x 16 KiB
  uint8_t* k_smem = smem + size_t(2 * nkb) * RM_KB_BYTES;  // [STG][nkb] x 16 KiB
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + size_t(2 + STG) * nkb * RM_KB_BYTES);
  uint64_t* full_bar = bars;                               // [RM_STAGES_MAX] leader
  uint64_t* empty_bar = bars + RM_STAGES_MAX;              // [RM_STAGES_MAX] every CTA
  uint64_t* tfull_bar = bars + 2 * RM_STAGES_MAX;          // [2] every CTA
  uint64_t* tempty_bar = tfull_bar + 2;                    // [2] leader
  uint64_t* qfull_bar = tempty_bar + 2;                    // [2] leader
  uint64_t* qempty_bar = qfull_bar + 2;                    // [2] every CTA
  uint64_t* drain_bar = qempty_bar + 2;                    // [1] leader
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * RM_STAGES_MAX + 9) * 8 + 8 <= GEMM_BARRIER_BYTES, "barrier block");
  int* head_max = reinterpret_cast<int*>(smem + size_t(2 + STG) * nkb * RM_KB_BYTES + GEMM_BARRIER_BYTES);
  const int nheads_smem = P.H <= SMEM_HEADS ? P.H : 0;
  for (int i = threadIdx.x; i < nheads_smem; i += blockDim.x) head_max[i] = INT_MIN;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < RM_STAGES_MAX; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&tfull_bar[b]), 1);
      mbar_init(smem_u32(&tempty_bar[b]), 2 * RM_EPI_WARPS);
      mbar_init(smem_u32(&qfull_bar[b]), 1);
      mbar_init(smem_u32(&qempty_bar[b]), 1);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.map_q[0]);
    prefetch_tmap(&P.map_k[0]);
    if (P.k_split) {
      prefetch_tmap(&P.map_q[1]);
      prefetch_tmap(&P.map_k[1]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long first_task = blockIdx.x >> 1;
  const long long task_step = gridDim.x >> 1;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0, fill_parity = 0;    // leader: key stages, as in umma_gemm.cuh
      uint32_t qfilled = 0, qfill_parity = 0;  // leader: Q buffers
      bool ok = true;
      long long qi = 0;
      for (long long t = first_task; ok && t < P.tasks; t += task_step, ++qi) {
        const RmTask T = rowmax_task(P, t);
        const int qb = static_cast<int>(qi & 1);
        const uint32_t qph = static_cast<uint32_t>((qi >> 1) & 1);
        if (!wait_bounded(smem_u32(&qempty_bar[qb]), qph ^ 1, abort_flag, P.err)) {
          ok = false;
          break;
        }
        const uint32_t qfb_local = smem_u32(&qfull_bar[qb]);
        if (leader) {
          mbar_arrive_expect_tx(qfb_local, 2u * nkb * RM_KB_BYTES);
          qfilled |= 1u << qb;
          qfill_parity = (qfill_parity & ~(1u << qb)) | (qph << qb);
        }
        const uint32_t qfb = mapa_shared(qfb_local, 0);
        const int m0 = T.i * BM + HALF * static_cast<int>(rank);
        for (int kb = 0; kb < nkb; ++kb) {
          const int k0 = kb * BK;
          const bool second = P.k_split > 0 && k0 >= P.k_split;
          tma_load_4d_pair(smem_u32(q_smem + size_t(qb * nkb + kb) * RM_KB_BYTES), second ? &P.map_q[1] : &P.map_q[0],
                           qfb, second ? k0 - P.k_split : k0, T.h, m0, T.b);
        }
        for (int j = 0; ok && j < T.jn; ++j) {
          const int n0 = j * BM + HALF * static_cast<int>(rank);
          if (!wait_bounded(smem_u32(&empty_bar[stage]), phase ^ 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          const uint32_t fb_local = smem_u32(&full_bar[stage]);
          if (leader) {
            mbar_arrive_expect_tx(fb_local, 2u * nkb * RM_KB_BYTES);
            filled |= 1u << stage;
            fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
          }
          const uint32_t fb = mapa_shared(fb_local, 0);
          for (int kb = 0; kb < nkb; ++kb) {
            const int k0 = kb * BK;
            const bool second = P.k_split > 0 && k0 >= P.k_split;
            tma_load_4d_pair(smem_u32(k_smem + size_t(stage * nkb + kb) * RM_KB_BYTES),
                             second ? &P.map_k[1] : &P.map_k[0], fb, second ? k0 - P.k_split : k0, second ? 0 : T.h,
                             n0, T.b);
          }
          if (++stage == STG) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // The leader's barriers count both CTAs' copies: every copy of the pair
      // lands before anyone leaves.
      if (leader) {
        volatile int no_abort = 0;
        for (int s = 0; s < STG; ++s)
          if (filled & (1u << s))
            wait_bounded(smem_u32(&full_bar[s]), (fill_parity >> s) & 1u, &no_abort, nullptr, kDrainLimitCycles);
        for (int b = 0; b < 2; ++b)
          if (qfilled & (1u << b))
            wait_bounded(smem_u32(&qfull_bar[b]), (qfill_parity >> b) & 1u, &no_abort, nullptr, kDrainLimitCycles);
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
      long long qi = 0;
      const uint32_t idesc = idesc_bf16_f32(BM, MMA_N, 0, 0);
      const uint64_t qd0 = smem_desc_sw128(smem_u32(q_smem), 16u, 1024);
      const uint64_t kd0 = smem_desc_sw128(smem_u32(k_smem), 16u, 1024);
      for (long long t = first_task; ok && t < P.tasks; t += task_step, ++qi) {
        const RmTask T = rowmax_task(P, t);
        const int qb = static_cast<int>(qi & 1);
        const uint32_t qph = static_cast<uint32_t>((qi >> 1) & 1);
        if (!wait_bounded(smem_u32(&qfull_bar[qb]), qph, abort_flag, P.err)) {
          ok = false;
          break;
        }
        for (int j = 0; ok && j < T.jn; ++j) {
          if (!wait_bounded(smem_u32(&tempty_bar[acc]), acc_phase ^ 1, abort_flag, P.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * MMA_N;
          if (!wait_bounded(smem_u32(&full_bar[stage]), phase, abort_flag, P.err)) {
            ok = false;
            break;
          }
          for (int kb = 0; kb < nkb; ++kb) {
            const uint64_t qoff = static_cast<uint64_t>((size_t(qb * nkb + kb) * RM_KB_BYTES) >> 4);
            const uint64_t koff = static_cast<uint64_t>((size_t(stage * nkb + kb) * RM_KB_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_bf16_pair(d_tmem, qd0 + qoff + ((kk * 32u) >> 4), kd0 + koff + ((kk * 32u) >> 4), idesc,
                             (kb | kk) != 0);
          }
          umma_commit_pair_mc(smem_u32(&empty_bar[stage]), 0x3);
          if (++stage == STG) {
            stage = 0;
            phase ^= 1;
          }
          umma_commit_pair_mc(smem_u32(&tfull_bar[acc]), 0x3);
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1;
        }
        if (!ok) break;
        // the task's last MMA has read its Q block: both CTAs may refill it
        umma_commit_pair_mc(smem_u32(&qempty_bar[qb]), 0x3);
      }
      umma_commit_pair(smem_u32(drain_bar));
      volatile int no_abort = 0;
      wait_bounded(smem_u32(drain_bar), 0, &no_abort, nullptr, kDrainLimitCycles);
    }
  } else {
    // ------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter
    const int cg = (warp - 2) >> 2;         // column group of the 256-column tile
    uint32_t tempty_leader[2];
    for (int b = 0; b < 2; ++b) tempty_leader[b] = mapa_shared(smem_u32(&tempty_bar[b]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (long long t = first_task; ok && t < P.tasks; t += task_step) {
      const RmTask T = rowmax_task(P, t);
      const int r = T.i * BM + HALF * static_cast<int>(rank) + q * 32 + lane;
      const int r_warp_last = T.i * BM + HALF * static_cast<int>(rank) + q * 32 + 31;
      float run_max = -INFINITY;
      for (int j = 0; j < T.jn; ++j) {
        const bool got = wait_bounded(smem_u32(&tfull_bar[acc]), acc_phase, abort_flag, P.err);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int c0 = j * BM + cg * RM_COLS;
        // a warp whose columns all lie above its last row has nothing to read
        const bool dead = P.causal && c0 > r_warp_last;
        if (!dead) {
          float v[RM_COLS];
          const uint32_t ta = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * MMA_N + cg * RM_COLS;
          if constexpr (RM_COLS == 128) {
            tmem_ld128(ta, v);
          } else {
            tmem_ld64(ta, v);
          }
          if (r < P.S) {
            if (c0 + RM_COLS <= P.S && (!P.causal || c0 + RM_COLS - 1 <= r)) {
              float m = run_max;
#pragma unroll
              for (int x = 0; x < RM_COLS; x += 8)
                m = fmax3(m, fmax3(v[x], v[x + 1], v[x + 2]),
                          fmax3(fmax3(v[x + 3], v[x + 4], v[x + 5]), v[x + 6], v[x + 7]));
              run_max = m;
            } else {
#pragma unroll
              for (int x = 0; x < RM_COLS; ++x) {
                const int c = c0 + x;
                if (c < P.S && (!P.causal || c <= r)) run_max = fmaxf(run_max, v[x]);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) run_max = fmaxf(run_max, __shfl_xor_sync(0xffffffffu, run_max, o));
      if (lane == 0 && run_max > -INFINITY) {
        const int key = float_to_ordered(run_max * P.out_scale);
        if (nheads_smem) {
          atomicMax(&head_max[T.h], key);
        } else {
          atomicMax(&P.keys[T.h], key);
        }
      }
    }
  }

  // Nobody leaves (or frees TMEM) while the peer may still signal this CTA's
  // barriers or read its shared memory.
  tc_fence_before();
  __syncthreads();
  for (int i = threadIdx.x; i < nheads_smem; i += blockDim.x)
    if (head_max[i] != INT_MIN) atomicMax(&P.keys[i], head_max[i]);
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace mc
