// Host engine and C ABI of the MuonClip step library (see include/muonclip.h).
//
// mc_muon_step splits the list into pieces of at most 2^29 elements and
// enqueues, per piece, on the caller's stream:
//   1. momentum_kernel       one launch over every matrix of the piece
//                            (momentum, Nesterov, the iterate's bf16 hi and lo
//                            halves, ||U||^2 partials)
//   2. norm_finalize_kernel  s = 1 / max(||U||_F, eps) per matrix
//   3. ns_steps x { GRAM, POLY, APPLY } grouped tcgen05 GEMM launches; the last
//      APPLY writes W directly (decay + scaled update), so the final iterate
//      never goes to memory (NorMuon: it goes out in fp32 for the row pass).
// Matrices with equal (rows, cols, weight dtype) form one problem group; their
// iterates sit back to back in the workspace so that one 3-D TMA descriptor
// covers the whole group.  Tall matrices (rows > cols) are never transposed in
// memory: the Gram product reads them MN-major and the apply multiplies from
// the right (X B instead of B X), which is the oriented iteration transposed.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "muonclip.h"
#include "ptx.cuh"
#include "qk_rowmax.cuh"
#include "stream_kernels.cuh"
#include "thin_ns.cuh"
#include "umma_gemm.cuh"

#define MC_API extern "C" __attribute__((visibility("default")))

namespace mc {
__device__ int g_device_error = 0;
}

namespace {

using namespace mc;

thread_local std::string t_last_error;

int fail(int code, const std::string& msg) {
  t_last_error = msg;
  return code;
}

#define MC_CUDA(expr)                                                                      \
  do {                                                                                     \
    cudaError_t e_ = (expr);                                                               \
    if (e_ != cudaSuccess) return fail(MC_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e_)); \
  } while (0)

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Largest dynamic shared memory a CTA may opt into on sm_100.
constexpr int kSmemOptIn = 232448;
// Newton-Schulz iterations that take a*X from the iterate's hi + lo halves.
constexpr int kMixedIters = 2;

struct DeviceState {
  bool init = false;
  int sms = 0;
  int pair_clusters = 0;  // CTA pairs of the GEMM kernel that fit on the device at once
  int cc_major = 0, cc_minor = 0;
  int* err_ptr = nullptr;
  void* own_ws = nullptr;
  size_t own_ws_bytes = 0;
  // mc_muon_step_host_grads: a non-blocking stream for the gradient copies and
  // events that order each chunk's compute after its copies
  cudaStream_t copy_stream = nullptr;
  std::vector<cudaEvent_t> chunk_ev;
};

std::mutex g_mu;
std::map<int, DeviceState> g_devices;
EncodeTiledFn g_encode = nullptr;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int EPI, int WIDE>
cudaError_t set_gemm_attr() {
  return cudaFuncSetAttribute(umma_gemm_kernel<EPI, WIDE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(gemm_smem_bytes<EPI, WIDE>()));
}

// Caller holds g_mu.
int device_state(DeviceState** out) {
  int dev = 0;
  MC_CUDA(cudaGetDevice(&dev));
  DeviceState& st = g_devices[dev];
  if (!st.init) {
    MC_CUDA(cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev));
    MC_CUDA(cudaDeviceGetAttribute(&st.cc_major, cudaDevAttrComputeCapabilityMajor, dev));
    MC_CUDA(cudaDeviceGetAttribute(&st.cc_minor, cudaDevAttrComputeCapabilityMinor, dev));
    if (st.cc_major != 10 || st.cc_minor != 0)
      return fail(MC_ERR_UNSUPPORTED, "device " + std::to_string(dev) + " has compute capability " +
                                          std::to_string(st.cc_major) + "." + std::to_string(st.cc_minor) +
                                          "; this library is built for sm_100a (B200)");
    MC_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&st.err_ptr), g_device_error));
    MC_CUDA((set_gemm_attr<EPI_GRAM, 1>()));
    MC_CUDA((set_gemm_attr<EPI_POLY, 1>()));
    MC_CUDA((set_gemm_attr<EPI_APPLY, 1>()));
    MC_CUDA((set_gemm_attr<EPI_APPLY_FINAL, 1>()));
    MC_CUDA((set_gemm_attr<EPI_GRAM, 0>()));
    MC_CUDA((set_gemm_attr<EPI_POLY, 0>()));
    MC_CUDA((set_gemm_attr<EPI_APPLY, 0>()));
    MC_CUDA((set_gemm_attr<EPI_APPLY_FINAL, 0>()));
    MC_CUDA((set_gemm_attr<EPI_APPLY_MIXED, 1>()));
    MC_CUDA((set_gemm_attr<EPI_APPLY_MIXED, 0>()));
    MC_CUDA((set_gemm_attr<EPI_STORE, 1>()));
    MC_CUDA((set_gemm_attr<EPI_CAUSALMAX, 0>()));
    MC_CUDA(cudaFuncSetAttribute(qk_rowmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemOptIn));
    {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(static_cast<unsigned>(st.sms & ~1));
      cfg.blockDim = dim3(GEMM_THREADS);
      cfg.dynamicSmemBytes = gemm_smem_bytes<EPI_CAUSALMAX, 0>();
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      MC_CUDA(cudaOccupancyMaxActiveClusters(&clusters, umma_gemm_kernel<EPI_CAUSALMAX, 0>, &cfg));
      if (clusters < 1) return fail(MC_ERR_UNSUPPORTED, "no CTA pair of the GEMM kernel fits on this device");
      st.pair_clusters = clusters;
    }
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      MC_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn)
        return fail(MC_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    st.init = true;
  }
  *out = &st;
  return MC_OK;
}

// ----------------------------------------------------------- profiling
enum Kind : int { K_MOMENTUM, K_FINALIZE, K_GRAM, K_POLY, K_APPLY_MIXED, K_APPLY, K_APPLY_FINAL, K_QK_PROJ,
                  K_QK_CMAX, K_QK_KEYS, K_QK_CLIP, K_MLA_PROJ, K_MLA_CMAX, K_QK_CLIP_SLICES, K_NORM_ROWS,
                  K_NORM_APPLY, K_TABLE_UPLOAD, K_NS_THIN, K_COUNT };
const char* const kKindNames[K_COUNT] = {"momentum",  "norm_finalize",  "ns_gram", "ns_poly",
                                         "ns_apply_mixed", "ns_apply", "ns_apply_final", "qk_proj",
                                         "qk_causal_max", "qk_keys", "qk_clip", "mla_proj",
                                         "mla_causal_max", "qk_clip_slices", "normuon_rows",
                                         "normuon_apply", "table_upload", "ns_thin"};
struct ProfRec {
  int kind;
  cudaEvent_t b, e;
  double flops, flops_exec, flops_dense, bytes;
};
thread_local bool t_prof = false;
thread_local std::vector<ProfRec> t_recs;

// Brackets one launch with CUDA events on its stream while profiling is on.
struct ProfScope {
  bool on = false;
  ProfRec r{};
  cudaStream_t s;
  ProfScope(int kind, cudaStream_t st, double flops = 0, double flops_exec = 0, double bytes = 0,
            double flops_dense = -1) : s(st) {
    if (!t_prof || kind < 0) return;
    r.kind = kind;
    r.flops = flops;
    r.flops_exec = flops_exec;
    r.flops_dense = flops_dense < 0 ? flops : flops_dense;
    r.bytes = bytes;
    if (cudaEventCreate(&r.b) != cudaSuccess) return;
    if (cudaEventCreate(&r.e) != cudaSuccess) {
      cudaEventDestroy(r.b);
      return;
    }
    on = cudaEventRecord(r.b, s) == cudaSuccess;
  }
  ~ProfScope() {
    if (!on) return;
    cudaEventRecord(r.e, s);
    t_recs.push_back(r);
  }
};

// One launch of table_fill_kernel<BYTES> with `n` bytes (n <= BYTES).
template <unsigned BYTES>
int fill_launch(const uint8_t* host, size_t n, uint8_t* dst, cudaStream_t s) {
  static thread_local TableBlob<BYTES> blob;  // off the stack
  blob.dst = reinterpret_cast<uint4*>(dst);
  blob.n16 = static_cast<unsigned>(n / 16);
  std::memcpy(blob.data, host, n);
  ProfScope prof(K_TABLE_UPLOAD, s, 0, 0, static_cast<double>(n));
  table_fill_kernel<BYTES><<<1, 256, 0, s>>>(blob);
  MC_CUDA(cudaGetLastError());
  return MC_OK;
}

// Copy a host table (a multiple of 16 bytes) to 16-byte aligned device
// memory, in launches of table_fill_kernel that carry it in their parameters.
// Stream-ordered like any launch, it never waits on the host, the host buffer
// may be reused at once, and a captured graph keeps its own copy of the bytes.
int upload(const void* host, size_t bytes, void* dst, cudaStream_t s) {
  if (bytes % 16 != 0 || !aligned16(dst)) return fail(MC_ERR_INVAL, "internal: table upload not 16-byte aligned");
  const uint8_t* h = static_cast<const uint8_t*>(host);
  uint8_t* d = static_cast<uint8_t*>(dst);
  for (size_t off = 0; off < bytes;) {
    const size_t n = std::min<size_t>(TABLE_BLOB_MAX, bytes - off);
    int rc = n <= 1024   ? fill_launch<1024>(h + off, n, d + off, s)
             : n <= 4096 ? fill_launch<4096>(h + off, n, d + off, s)
                         : fill_launch<TABLE_BLOB_MAX>(h + off, n, d + off, s);
    if (rc != MC_OK) return rc;
    off += n;
  }
  return MC_OK;
}

int own_workspace(DeviceState& st, size_t bytes, void** ws) {
  if (st.own_ws_bytes < bytes) {
    if (st.own_ws) {
      MC_CUDA(cudaDeviceSynchronize());
      MC_CUDA(cudaFree(st.own_ws));
      st.own_ws = nullptr;
      st.own_ws_bytes = 0;
    }
    MC_CUDA(cudaMalloc(&st.own_ws, bytes));
    st.own_ws_bytes = bytes;
  }
  *ws = st.own_ws;
  return MC_OK;
}

// bf16 tensor map (128-byte swizzle unless given), zero fill out of bounds.
int make_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
             const uint32_t* box, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gs[i] = strides[i];
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gd, gs, bx, es,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MC_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string(r));
  return MC_OK;
}

// [count][rows][ld] bf16, box {box_cols, box_rows, 1}
int map_batched(CUtensorMap* map, const void* base, int64_t count, int64_t rows, int64_t cols, int64_t ld,
                uint32_t box_rows, uint32_t box_cols = 64, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  const uint64_t dims[3] = {uint64_t(cols), uint64_t(rows), uint64_t(count)};
  const uint64_t strides[2] = {uint64_t(ld) * 2, uint64_t(rows) * uint64_t(ld) * 2};
  const uint32_t box[3] = {box_cols, box_rows, 1};
  return make_map(map, base, 3, dims, strides, box, swizzle);
}

// Epilogue map of a [count][rows][ld] bf16 matrix for the coalesced tensor
// path: boxes of 32 rows x 64 columns (128-byte swizzle) or, when `narrow`,
// 32 x 32 (64-byte swizzle).  `*ok` is false (and nothing is encoded) when the
// matrix is smaller than one box; the epilogue then keeps its other paths.
int map_epilogue(CUtensorMap* map, bool* ok, const void* base, int64_t count, int64_t rows, int64_t cols, int64_t ld,
                 bool narrow) {
  const uint32_t bc = narrow ? 32 : 64;
  *ok = rows >= 32 && cols >= bc && ld % 8 == 0;
  if (!*ok) return MC_OK;
  return map_batched(map, base, count, rows, cols, ld, 32, bc,
                     narrow ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

double gemm_exec_flops(const GemmParams& p) {
  double f = 0;
  for (int i = 0; i < p.num_groups; ++i) {
    const GemmGroup& G = p.g[i];
    const double kpad = double((G.K + BK - 1) / BK) * BK;
    f += double(G.tiles_per_prob) * G.count * 2.0 * BM * double(MMA_N << G.nshift) * kpad;
  }
  return f;
}

// Persistent launch in clusters of two CTAs (one 2-SM MMA pair each), as
// many pairs as fit on the device at once, at most one per tile.
// Programmatic stream serialisation for the Newton-Schulz GEMMs: a kernel so
// launched may begin (its prologue: barriers, TMEM, tensor-map prefetch) while
// the previous kernel of the stream finishes its last tiles; it touches global
// memory only after griddepcontrol.wait, i.e. once that kernel has completed
// and its writes are visible, so stream order is kept for all memory effects.
// Measured A/B on one box: one fp32 256 x 512 step 0.269 -> 0.239 ms, the MoE
// set 98.1 -> 97.2 ms, 64 x 1024^2 1.943 -> 1.933 ms; the QK layer (projection
// and causal max) gained nothing, so its launches keep plain stream order.
void set_pdl(cudaLaunchAttribute& a, bool on) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = on ? 1 : 0;
}

template <int EPI, int WIDE>
cudaError_t launch_pairs(const GemmParams& p, int pair_clusters, cudaStream_t s) {
  const long long pairs = std::min<long long>(pair_clusters, p.total_tiles);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_pdl(attr[1], EPI != EPI_STORE && EPI != EPI_CAUSALMAX);
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = gemm_smem_bytes<EPI, WIDE>();
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, umma_gemm_kernel<EPI, WIDE>, p);
}

template <int EPI, int WIDE>
int launch_gemm(const GemmParams& p, const DeviceState& st, cudaStream_t s, int kind, double flops,
                double flops_dense = -1) {
  if (p.total_tiles <= 0) return MC_OK;
  ProfScope prof(kind, s, flops, gemm_exec_flops(p), 0, flops_dense);
  MC_CUDA((launch_pairs<EPI, WIDE>(p, st.pair_clusters, s)));
  return MC_OK;
}

// `wide`: 1 for 256 x 512 tiles (TileCfg<1>), 0 for 256 x 256.
void finish_group(GemmParams& p, int gi, GemmGroup& G, int wide) {
  const int tile_n = MMA_N << wide;
  G.nshift = wide;
  G.tiles_m = (G.M + BM - 1) / BM;
  G.tiles_n = (G.N + tile_n - 1) / tile_n;
  G.tiles_per_prob = sched_tiles_per_prob(G.sched, G.tiles_m, G.tiles_n, G.nshift);
  G.tile_start = p.total_tiles;
  if (G.band <= 0) G.band = 8;
  p.total_tiles += G.tiles_per_prob * G.count;
  p.g[gi] = G;
  p.num_groups = gi + 1;
}

// Key-ring depth of qk_rowmax_kernel for a contraction of nkb k-blocks: as
// many stages as fit beside the Q double buffer, at most RM_STAGES_MAX.
int rowmax_stages(int nkb) {
  const long long room = kSmemOptIn - 1024 - GEMM_BARRIER_BYTES - 4LL * SMEM_HEADS - 2LL * nkb * RM_KB_BYTES;
  return static_cast<int>(std::min<long long>(RM_STAGES_MAX, room / (nkb * (long long)RM_KB_BYTES)));
}

// Per-head max of the score tiles, scores never stored.  `cm` holds the Q and
// K maps (slot 1: the rotary part of a split contraction) and the group as
// the tile GEMM takes them.  A contraction of at most RM_KB_MAX k-blocks runs
// the row-owned kernel (Q resident, only key blocks stream); a longer one the
// tile GEMM with the max epilogue.
int launch_causal_max(const GemmParams& cm, const DeviceState& st, cudaStream_t s, int kind, double flops,
                      bool profiled) {
  const GemmGroup& G = cm.g[0];
  const int nkb = (G.K + BK - 1) / BK;
  const int stages = rowmax_stages(nkb);
  if (nkb > RM_KB_MAX || stages < 1) {
    if (!profiled) {
      if (cm.total_tiles > 0) MC_CUDA((launch_pairs<EPI_CAUSALMAX, 0>(cm, st.pair_clusters, s)));
      return MC_OK;
    }
    return launch_gemm<EPI_CAUSALMAX, 0>(cm, st, s, kind, flops);
  }
  RowMaxParams R;
  std::memset(&R, 0, sizeof(R));
  R.map_q[0] = cm.map_a[0];
  R.map_k[0] = cm.map_b[0];
  R.map_q[1] = cm.map_a[1];
  R.map_k[1] = cm.map_b[1];
  R.S = G.M;
  R.H = G.heads;
  R.B = G.count / G.heads;
  R.nkb = nkb;
  R.k_split = G.k_split;
  R.stages = stages;
  R.causal = G.mask_causal;
  R.nblk = (G.M + BM - 1) / BM;
  R.tasks = static_cast<long long>(G.count) * R.nblk;
  R.out_scale = G.out_scale;
  R.keys = G.keys;
  R.err = cm.err;
  if (R.tasks <= 0) return MC_OK;
  const double nb = R.nblk;
  const double tiles = double(G.count) * (R.causal ? nb * (nb + 1) / 2 : nb * nb);
  ProfScope prof(profiled ? kind : -1, s, flops, tiles * 2.0 * BM * MMA_N * nkb * BK);
  const long long pairs = std::min<long long>(st.pair_clusters, R.tasks);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(RM_THREADS);
  cfg.dynamicSmemBytes = rowmax_smem_bytes(nkb, stages);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  MC_CUDA(cudaLaunchKernelEx(&cfg, qk_rowmax_kernel, R));
  return MC_OK;
}

// Newton-Schulz phases whose contraction is at most this long use the
// 256 x 256 tile with two accumulators (WIDE = 0), so one tile's epilogue
// overlaps the next tile's MMAs; longer ones the 256 x 512 tile with one
// accumulator (WIDE = 1), which shares each A tile between two MMAs and so
// stays under the per-SM operand feed limit, but exposes its epilogue.  With a
// short contraction the main loop of a tile is short and the exposed epilogue
// (its global reads and writes) would cost more than the narrower tile loses.
// The plain apply (X' = (aI + B) X, bf16 out, nothing read) has the lightest
// epilogue and takes the wide tile at every length.
constexpr int kNarrowMaxK = 2048;

// Up to MAX_GROUPS problem groups of one launch, with their work figures.
struct GemmBatch {
  GemmParams p;
  double f = 0, fd = 0;
  int n = 0;
};

// eo / ei / ei2: the group's epilogue maps (output, inputs), or NULL: when eo
// is given the group's full blocks move by tensor copies (GemmGroup::tma_epi).
void add_to_batch(std::vector<GemmBatch>& v, const DeviceState& st, const CUtensorMap& ma, const CUtensorMap& mb,
                  const GemmGroup& G, int wide, double flops, double flops_dense, const CUtensorMap* eo = nullptr,
                  const CUtensorMap* ei = nullptr, const CUtensorMap* ei2 = nullptr) {
  if (v.empty() || v.back().n == MAX_GROUPS) {
    v.emplace_back();
    std::memset(&v.back().p, 0, sizeof(GemmParams));
    v.back().p.err = st.err_ptr;
  }
  GemmBatch& b = v.back();
  b.p.map_a[b.n] = ma;
  b.p.map_b[b.n] = mb;
  GemmGroup g = G;
  g.tma_epi = eo != nullptr ? 1 : 0;
  if (eo) b.p.map_eo[b.n] = *eo;
  if (ei) b.p.map_ei[b.n] = *ei;
  if (ei2) b.p.map_ei2[b.n] = *ei2;
  finish_group(b.p, b.n, g, wide);
  b.f += flops;
  b.fd += flops_dense;
  ++b.n;
}

// ------------------------------------------------------------------ muon plan
struct NsGroup {
  int64_t rows = 0, cols = 0;
  int w_f32 = 0;
  bool tall = false;
  int64_t m = 0, n = 0;   // min, max
  int64_t ld = 0;         // row stride of the iterate
  int64_t ldm = 0;        // row stride of A and B
  bool thin = false;       // m <= THIN_M (32): the fp32 CUDA-core iteration of thin_ns.cuh
  std::vector<int> members;
  int prob_base = 0;
  size_t off_xb[2] = {0, 0}, off_xl = 0, off_xf = 0, off_a = 0, off_b = 0, off_wptr = 0, off_uptr = 0;
};

struct MuonLayout {
  std::vector<NsGroup> groups;
  std::vector<int> order;   // workspace order -> caller index
  std::vector<long long> cta_begin;
  long long total_ctas = 0;
  size_t off_tab = 0, tab_bytes = 0, off_partials = 0, off_scale = 0, total = 0;
  // NorMuon only: NormEntry[n] inside the table block, and two fp32 row arrays
  bool normuon = false;
  size_t off_ntab = 0, off_rowsq = 0, off_rowf = 0;
  long long total_rows = 0;
  // thin matrices: ThinEntry[n_thin] inside the table block, the chunk
  // partial sums of A and the P matrices
  int n_thin = 0;
  long long thin_ctas = 0;
  size_t off_ttab = 0, off_tpart = 0, off_pmat = 0;
};

// 1 - lr*wd as two rounded fp32 operations (the kernels that read a device
// (lr, wd) pair do the same, so both routes give the same bits).
float host_decay(const mc_hparams* hp) {
  volatile float t = hp->lr * hp->wd;
  return 1.f - t;
}

int validate_muon(const mc_param* params, int n, const mc_hparams* hp) {
  if (n < 0) return fail(MC_ERR_INVAL, "n must be >= 0");
  if (n > 0 && !params) return fail(MC_ERR_INVAL, "params is NULL");
  if (!hp) return fail(MC_ERR_INVAL, "hp is NULL");
  if (hp->ns_steps < 1 || hp->ns_steps >= 100) return fail(MC_ERR_INVAL, "ns_steps must be in [1, 100)");
  const float vals[] = {hp->mu, hp->lr, hp->wd, hp->a, hp->b, hp->c, hp->eps, hp->rms_scale};
  for (float v : vals)
    if (!std::isfinite(v)) return fail(MC_ERR_INVAL, "non-finite hyper-parameter");
  if (hp->coeffs)
    for (int i = 0; i < 3 * hp->ns_steps; ++i)
      if (!std::isfinite(hp->coeffs[i])) return fail(MC_ERR_INVAL, "non-finite coefficient in hp->coeffs");
  if (!(hp->eps > 0.f)) return fail(MC_ERR_INVAL, "eps must be > 0");
  if (hp->lr_wd && (reinterpret_cast<uintptr_t>(hp->lr_wd) & 3u) != 0)
    return fail(MC_ERR_ALIGN, "hp->lr_wd must be 4-byte aligned");
  for (int i = 0; i < n; ++i) {
    const mc_param& q = params[i];
    const std::string at = "params[" + std::to_string(i) + "]: ";
    if (!q.w || !q.g || !q.m) return fail(MC_ERR_INVAL, at + "NULL w, g or m");
    if (q.rows < 1 || q.cols < 1) return fail(MC_ERR_INVAL, at + "rows and cols must be >= 1");
    if (q.rows > (1 << 24) || q.cols > (1 << 24) || q.rows * q.cols > (int64_t(1) << 36))
      return fail(MC_ERR_INVAL, at + "matrix too large");
    if ((q.w_dtype != MC_F32 && q.w_dtype != MC_BF16) || (q.g_dtype != MC_F32 && q.g_dtype != MC_BF16))
      return fail(MC_ERR_INVAL, at + "dtype must be MC_F32 or MC_BF16");
    if (q.w == static_cast<const void*>(q.g) || q.w == static_cast<void*>(q.m) ||
        q.g == static_cast<const void*>(q.m))
      return fail(MC_ERR_INVAL, at + "w, g and m must not alias");
    if (!aligned16(q.w) || !aligned16(q.g) || !aligned16(q.m) || (q.update_out && !aligned16(q.update_out)))
      return fail(MC_ERR_ALIGN, at + "pointers must be 16-byte aligned");
  }
  return MC_OK;
}

void plan_muon(const mc_param* params, int n, MuonLayout& L, bool normuon = false) {
  L.normuon = normuon;
  std::map<std::tuple<int64_t, int64_t, int>, int> index;
  for (int i = 0; i < n; ++i) {
    const auto key = std::make_tuple(params[i].rows, params[i].cols, params[i].w_dtype == MC_F32 ? 1 : 0);
    auto it = index.find(key);
    if (it == index.end()) {
      NsGroup g;
      g.rows = params[i].rows;
      g.cols = params[i].cols;
      g.w_f32 = params[i].w_dtype == MC_F32;
      g.tall = g.rows > g.cols;
      g.m = std::min(g.rows, g.cols);
      g.n = std::max(g.rows, g.cols);
      g.ld = round8(g.cols);
      g.ldm = round8(g.m);
      g.thin = g.m <= THIN_M;
      index[key] = static_cast<int>(L.groups.size());
      L.groups.push_back(g);
      it = index.find(key);
    }
    L.groups[it->second].members.push_back(i);
  }
  size_t off = 0;
  int pb = 0;
  for (auto& g : L.groups) {
    g.prob_base = pb;
    pb += static_cast<int>(g.members.size());
    for (int i : g.members) L.order.push_back(i);
  }
  // Momentum kernel CTA split, in workspace order.
  L.cta_begin.resize(n);
  long long ctas = 0;
  for (int k = 0; k < n; ++k) {
    const mc_param& q = params[L.order[k]];
    L.cta_begin[k] = ctas;
    ctas += (q.rows * q.cols + MOM_ELEMS_PER_CTA - 1) / MOM_ELEMS_PER_CTA;
  }
  L.total_ctas = ctas;
  // Tables: MomEntry[n], then per group w_ptrs[count] and u_ptrs[count].
  L.off_tab = 0;
  off = align_up(sizeof(MomEntry) * n, 256);
  for (auto& g : L.groups) {
    g.off_wptr = off;
    off += sizeof(void*) * g.members.size();
    g.off_uptr = off;
    off += sizeof(void*) * g.members.size();
  }
  if (normuon) {
    off = align_up(off, 256);
    L.off_ntab = off;
    off += sizeof(NormEntry) * n;
  }
  for (const auto& g : L.groups) {
    if (!g.thin) continue;
    for (size_t j = 0; j < g.members.size(); ++j)
      L.thin_ctas += (g.n + THIN_COLS - 1) / THIN_COLS;
    L.n_thin += static_cast<int>(g.members.size());
  }
  if (L.n_thin) {
    off = align_up(off, 256);
    L.off_ttab = off;
    off += sizeof(ThinEntry) * size_t(L.n_thin);
  }
  L.tab_bytes = off;
  off = align_up(off, 1024);
  L.off_partials = off;
  off = align_up(off + sizeof(double) * ctas, 1024);
  L.off_scale = off;
  off = align_up(off + sizeof(float) * n, 1024);
  for (auto& g : L.groups) {
    const size_t cnt = g.members.size();
    const size_t xe = cnt * size_t(g.rows) * size_t(g.ld);
    const size_t ae = cnt * size_t(g.m) * size_t(g.ldm);
    g.off_xb[0] = off; off = align_up(off + 2 * xe, 1024);   // U's hi half (momentum kernel)
    g.off_xl = off;    off = align_up(off + 2 * xe, 1024);   // U's lo half
    if (g.thin) {        // fp32 iterate; no GEMM operands
      g.off_xf = off;    off = align_up(off + 4 * xe, 1024);
      continue;
    }
    g.off_xb[1] = off; off = align_up(off + 2 * xe, 1024);
    if (normuon) {       // NorMuon's row pass reads the NS output in fp32
      g.off_xf = off;    off = align_up(off + 4 * xe, 1024);
    }
    g.off_a = off;     off = align_up(off + 2 * ae, 1024);
    g.off_b = off;     off = align_up(off + 2 * ae, 1024);
  }
  if (L.n_thin) {
    L.off_tpart = off;
    off = align_up(off + sizeof(float) * THIN_PAIRS * size_t(L.thin_ctas), 1024);
    L.off_pmat = off;
    off = align_up(off + sizeof(float) * THIN_PMAT * size_t(L.n_thin), 1024);
  }
  if (normuon) {
    for (int i = 0; i < n; ++i) L.total_rows += params[i].rows;
    L.off_rowsq = off;
    off = align_up(off + sizeof(float) * size_t(L.total_rows), 1024);
    L.off_rowf = off;
    off = align_up(off + sizeof(float) * size_t(L.total_rows), 1024);
  }
  L.total = std::max<size_t>(off, 1024);
}

// K-major maps use 128-row boxes (each CTA of a pair stages 128 rows of an
// operand); MN-major maps use {64, 64} boxes.
struct GroupMaps {
  CUtensorMap x_k[2], x_mn[2], a_k, b_k;
  // epilogue maps (see map_epilogue): A and B, the iterate by 64 and by 32
  // columns, its lo half by 32 columns
  CUtensorMap a_e, b_e, x_e64[2], x_e32[2], xl_e32;
  bool ok_ab = false, ok_x64 = false, ok_x32 = false;
};

int build_group_maps(const NsGroup& g, uint8_t* ws, GroupMaps& M) {
  const int64_t cnt = static_cast<int64_t>(g.members.size());
  for (int par = 0; par < 2; ++par) {
    const void* xb = ws + g.off_xb[par];
    int rc;
    if ((rc = map_batched(&M.x_k[par], xb, cnt, g.rows, g.cols, g.ld, HALF)) != MC_OK) return rc;
    if ((rc = map_batched(&M.x_mn[par], xb, cnt, g.rows, g.cols, g.ld, 64)) != MC_OK) return rc;
  }
  int rc;
  if ((rc = map_batched(&M.a_k, ws + g.off_a, cnt, g.m, g.m, g.ldm, HALF)) != MC_OK) return rc;
  if ((rc = map_batched(&M.b_k, ws + g.off_b, cnt, g.m, g.m, g.ldm, HALF)) != MC_OK) return rc;
  bool ok = true;
  if ((rc = map_epilogue(&M.a_e, &M.ok_ab, ws + g.off_a, cnt, g.m, g.m, g.ldm, false)) != MC_OK) return rc;
  if ((rc = map_epilogue(&M.b_e, &ok, ws + g.off_b, cnt, g.m, g.m, g.ldm, false)) != MC_OK) return rc;
  for (int par = 0; par < 2; ++par) {
    const void* xb = ws + g.off_xb[par];
    if ((rc = map_epilogue(&M.x_e64[par], &M.ok_x64, xb, cnt, g.rows, g.cols, g.ld, false)) != MC_OK) return rc;
    if ((rc = map_epilogue(&M.x_e32[par], &M.ok_x32, xb, cnt, g.rows, g.cols, g.ld, true)) != MC_OK) return rc;
  }
  if ((rc = map_epilogue(&M.xl_e32, &ok, ws + g.off_xl, cnt, g.rows, g.cols, g.ld, true)) != MC_OK) return rc;
  return MC_OK;
}

GemmGroup base_group(const NsGroup& g) {
  GemmGroup G;
  std::memset(&G, 0, sizeof(G));
  G.count = static_cast<int>(g.members.size());
  G.layout = LAYOUT_BATCHED;
  G.heads = 1;
  G.prob_base = g.prob_base;
  G.band = 8;
  return G;
}

}  // namespace

// =========================================================================
MC_API const char* mc_last_error(void) { return t_last_error.c_str(); }

namespace {
size_t pieces_workspace(const mc_param* params, int n, bool normuon);
}  // namespace

MC_API size_t mc_muon_workspace_size(const mc_param* params, int n, const mc_hparams* hp) {
  if (validate_muon(params, n, hp) != MC_OK) return 0;
  return pieces_workspace(params, n, false);
}

namespace {
int validate_normuon(const mc_param* params, int n, const mc_normuon* nm) {
  if (!nm) return fail(MC_ERR_INVAL, "nm is NULL");
  if (!std::isfinite(nm->beta2) || nm->beta2 < 0.f || nm->beta2 >= 1.f)
    return fail(MC_ERR_INVAL, "nm->beta2 must be in [0, 1)");
  if (!std::isfinite(nm->eps) || nm->eps < 0.f) return fail(MC_ERR_INVAL, "nm->eps must be finite and >= 0");
  if (n > 0 && !nm->v) return fail(MC_ERR_INVAL, "nm->v is NULL");
  for (int i = 0; i < n; ++i) {
    const float* v = nm->v[i];
    const std::string at = "nm->v[" + std::to_string(i) + "]: ";
    if (!v) return fail(MC_ERR_INVAL, at + "NULL");
    if (!aligned16(v)) return fail(MC_ERR_ALIGN, at + "must be 16-byte aligned");
    if (static_cast<const void*>(v) == params[i].w || static_cast<const void*>(v) == params[i].g ||
        v == params[i].m)
      return fail(MC_ERR_INVAL, at + "aliases w, g or m");
  }
  return MC_OK;
}

int run_muon(const mc_param* params, int n, const mc_hparams* hp, const mc_normuon* nm, void* workspace,
             size_t workspace_bytes, float* norms_out, cudaStream_t s, uint8_t* tab_dev);
void build_muon_table(const mc_param* params, int n, const mc_hparams* hp, const mc_normuon* nm, uint8_t* ws,
                      const MuonLayout& L, uint8_t* tab);
}  // namespace

namespace {
// The list is processed in consecutive pieces of at most this many elements
// (at least one matrix each), every piece reusing one workspace.  Measured on
// the 7B-shaped set (7.8e9 elements) on one GPU: 1, 2, 4, 8, 16 and 32 pieces
// took 605, 584, 560, 553, 551 and 550 ms; 16 pieces it is, with a workspace
// about 18 x smaller than one pass would need.
constexpr double kPieceElems = 536870912.0;

std::vector<int> split_pieces(const mc_param* params, int n) {
  std::vector<int> b{0};
  double acc = 0;
  for (int i = 0; i < n; ++i) {
    const double e = double(params[i].rows) * double(params[i].cols);
    if (i > b.back() && acc + e > kPieceElems) {
      b.push_back(i);
      acc = 0;
    }
    acc += e;
  }
  b.push_back(n);
  return b;
}

// Workspace of a call that runs the list in pieces: one compute region that
// every piece reuses in turn, then every piece's device tables, all built on
// the host and uploaded in one copy at the start of the call (so the call
// never waits on the host for an earlier piece).
struct PiecesPlan {
  std::vector<int> bounds;
  std::vector<MuonLayout> layouts;
  std::vector<size_t> tab_off;
  size_t compute = 0, total = 0;
};

void plan_pieces(const mc_param* params, std::vector<int> bounds, bool normuon, PiecesPlan& P) {
  P.bounds = std::move(bounds);
  const int np = static_cast<int>(P.bounds.size()) - 1;
  P.layouts.resize(static_cast<size_t>(np));
  for (int k = 0; k < np; ++k) {
    plan_muon(params + P.bounds[k], P.bounds[k + 1] - P.bounds[k], P.layouts[size_t(k)], normuon);
    P.compute = std::max(P.compute, P.layouts[size_t(k)].total);
  }
  size_t off = align_up(P.compute, 1024);
  for (int k = 0; k < np; ++k) {
    P.tab_off.push_back(off);
    off = align_up(off + P.layouts[size_t(k)].tab_bytes, 256);
  }
  P.total = align_up(off, 1024);
}

size_t pieces_workspace(const mc_param* params, int n, bool normuon) {
  PiecesPlan P;
  plan_pieces(params, split_pieces(params, n), normuon, P);
  return P.total;
}

// Every piece's tables, built on the host, in one upload (caller holds g_mu).
int upload_piece_tables(DeviceState& st, const mc_param* params, const mc_hparams* hp, const mc_normuon* nm,
                        const PiecesPlan& P, uint8_t* ws, cudaStream_t s) {
  const size_t t0 = P.tab_off.front();
  std::vector<uint8_t> tabs(P.total - t0, 0);
  mc_normuon sub{};
  for (size_t k = 0; k + 1 < P.bounds.size(); ++k) {
    const mc_normuon* pn = nullptr;
    if (nm) {
      sub = *nm;
      sub.v = nm->v + P.bounds[k];
      pn = &sub;
    }
    build_muon_table(params + P.bounds[k], P.bounds[k + 1] - P.bounds[k], hp, pn, ws, P.layouts[k],
                     tabs.data() + (P.tab_off[k] - t0));
  }
  (void)st;
  return upload(tabs.data(), tabs.size(), ws + t0, s);
}

// mc_muon_step / mc_normuon_step body: the tables of every piece in one
// upload, then one run_muon per piece.
int run_pieces(const mc_param* params, int n, const mc_hparams* hp, const mc_normuon* nm, void* workspace,
               size_t workspace_bytes, float* norms_out, cudaStream_t s) {
  PiecesPlan P;
  plan_pieces(params, split_pieces(params, n), nm != nullptr, P);
  uint8_t* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != MC_OK) return rc;
    if (workspace) {
      if (workspace_bytes < P.total)
        return fail(MC_ERR_NOSPC, "workspace has " + std::to_string(workspace_bytes) + " bytes, needs " +
                                      std::to_string(P.total));
    } else if ((rc = own_workspace(*st, P.total, &workspace)) != MC_OK) {
      return rc;
    }
    ws = static_cast<uint8_t*>(workspace);
    if ((rc = upload_piece_tables(*st, params, hp, nm, P, ws, s)) != MC_OK) return rc;
  }
  mc_normuon sub{};
  for (size_t k = 0; k + 1 < P.bounds.size(); ++k) {
    const mc_normuon* pn = nullptr;
    if (nm) {
      sub = *nm;
      sub.v = nm->v + P.bounds[k];
      pn = &sub;
    }
    const int rc = run_muon(params + P.bounds[k], P.bounds[k + 1] - P.bounds[k], hp, pn, ws, P.compute,
                            norms_out ? norms_out + P.bounds[k] : nullptr, s, ws + P.tab_off[k]);
    if (rc != MC_OK) return rc;
  }
  return MC_OK;
}
}  // namespace

MC_API size_t mc_normuon_workspace_size(const mc_param* params, int n, const mc_hparams* hp) {
  if (validate_muon(params, n, hp) != MC_OK || n == 0) return 0;
  return pieces_workspace(params, n, true);
}

int check_out_align(const float* norms_out, const void* workspace) {
  if (norms_out && !aligned16(norms_out)) return fail(MC_ERR_ALIGN, "norms_out must be 16-byte aligned");
  if (workspace && !aligned16(workspace)) return fail(MC_ERR_ALIGN, "workspace must be 16-byte aligned");
  return MC_OK;
}

// Pieces of the host-gradient step, in order: the first ones ramp up
// geometrically, from total/256 of the gradient bytes by x1.75 each, to
// total/chunks, the size the rest keep.  The step takes about 1.9x longer
// per byte than the upload, so a piece 1.75x the size of the one before
// still lands before that one's step ends: only the small first upload is
// exposed.  Returns the piece boundaries (first entry 0, last n).
std::vector<int> split_chunks(const mc_param* params, int n, int chunks) {
  auto bytes = [&](int i) {
    return double(params[i].rows) * double(params[i].cols) * (params[i].g_dtype == MC_F32 ? 4 : 2);
  };
  double total = 0;
  for (int i = 0; i < n; ++i) total += bytes(i);
  const double even = total / chunks;
  double target = chunks > 1 ? std::min(even, total / 256.0) : total;
  std::vector<int> b{0};
  double acc = 0;
  for (int i = 0; i < n; ++i) {
    acc += bytes(i);
    if (i + 1 < n && acc >= target) {
      b.push_back(i + 1);
      acc = 0;
      target = std::min(even, target * 1.75);
    }
  }
  b.push_back(n);
  return b;
}

MC_API int mc_normuon_step(const mc_param* params, int n, const mc_hparams* hp, const mc_normuon* nm,
                           void* workspace, size_t workspace_bytes, float* norms_out, void* stream) {
  int rc = validate_muon(params, n, hp);
  if (rc != MC_OK) return rc;
  if ((rc = validate_normuon(params, n, nm)) != MC_OK) return rc;
  if ((rc = check_out_align(norms_out, workspace)) != MC_OK) return rc;
  if (n == 0) return MC_OK;
  return run_pieces(params, n, hp, nm, workspace, workspace_bytes, norms_out, static_cast<cudaStream_t>(stream));
}

MC_API int mc_muon_step(const mc_param* params, int n, const mc_hparams* hp, void* workspace,
                        size_t workspace_bytes, float* norms_out, void* stream) {
  int rc = validate_muon(params, n, hp);
  if (rc != MC_OK) return rc;
  if ((rc = check_out_align(norms_out, workspace)) != MC_OK) return rc;
  if (n == 0) return MC_OK;
  return run_pieces(params, n, hp, nullptr, workspace, workspace_bytes, norms_out,
                    static_cast<cudaStream_t>(stream));
}

// Workspace of mc_muon_step_host_grads: as for mc_muon_step, with the pieces
// of split_chunks.  Every piece's tables go up before the first gradient copy
// (a table upload queued behind the gradient copies would wait for all of
// them in the copy engine, and so would the first piece).
void plan_host_grads(const mc_param* params, int n, int chunks, PiecesPlan& P) {
  plan_pieces(params, split_chunks(params, n, chunks), false, P);
}

MC_API size_t mc_muon_host_grads_workspace_size(const mc_param* params, int n, const mc_hparams* hp, int chunks) {
  if (validate_muon(params, n, hp) != MC_OK || n == 0 || chunks < 1) return 0;
  PiecesPlan P;
  plan_host_grads(params, n, chunks, P);
  return P.total;
}

MC_API int mc_muon_step_host_grads(const mc_param* params, const void* const* g_host, int n, const mc_hparams* hp,
                                   int chunks, void* workspace, size_t workspace_bytes, float* norms_out,
                                   void* stream) {
  int rc = validate_muon(params, n, hp);
  if (rc != MC_OK) return rc;
  if ((rc = check_out_align(norms_out, workspace)) != MC_OK) return rc;
  if (chunks < 1) return fail(MC_ERR_INVAL, "chunks must be >= 1");
  if (n > 0 && !g_host) return fail(MC_ERR_INVAL, "g_host is NULL");
  for (int i = 0; i < n; ++i)
    if (!g_host[i]) return fail(MC_ERR_INVAL, "g_host[" + std::to_string(i) + "] is NULL");
  if (n == 0) return MC_OK;
  PiecesPlan P;
  plan_host_grads(params, n, chunks, P);
  const std::vector<int>& b = P.bounds;
  const int nch = static_cast<int>(b.size()) - 1;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<cudaEvent_t> done(static_cast<size_t>(nch));
  uint8_t* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* st = nullptr;
    if ((rc = device_state(&st)) != MC_OK) return rc;
    if (workspace) {
      if (workspace_bytes < P.total)
        return fail(MC_ERR_NOSPC, "workspace has " + std::to_string(workspace_bytes) + " bytes, needs " +
                                      std::to_string(P.total));
    } else if ((rc = own_workspace(*st, P.total, &workspace)) != MC_OK) {
      return rc;
    }
    ws = static_cast<uint8_t*>(workspace);
    // every piece's tables, in one upload, ahead of the gradient copies
    if ((rc = upload_piece_tables(*st, params, hp, nullptr, P, ws, s)) != MC_OK) return rc;
    if (!st->copy_stream) MC_CUDA(cudaStreamCreateWithFlags(&st->copy_stream, cudaStreamNonBlocking));
    while (static_cast<int>(st->chunk_ev.size()) < nch + 1) {
      cudaEvent_t e;
      MC_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
      st->chunk_ev.push_back(e);
    }
    // Copies start only after the work already queued on `stream` (which may
    // still read the previous gradients, and includes the table upload); each
    // piece's step waits for its own copies.
    MC_CUDA(cudaEventRecord(st->chunk_ev[nch], s));
    MC_CUDA(cudaStreamWaitEvent(st->copy_stream, st->chunk_ev[nch], 0));
    for (int k = 0; k < nch; ++k) {
      for (int i = b[k]; i < b[k + 1]; ++i) {
        const size_t bytes = size_t(params[i].rows) * size_t(params[i].cols) * (params[i].g_dtype == MC_F32 ? 4 : 2);
        MC_CUDA(cudaMemcpyAsync(const_cast<void*>(params[i].g), g_host[i], bytes, cudaMemcpyHostToDevice,
                                st->copy_stream));
      }
      MC_CUDA(cudaEventRecord(st->chunk_ev[k], st->copy_stream));
      done[static_cast<size_t>(k)] = st->chunk_ev[k];
    }
  }
  // Piece k's step waits only for piece k's copies, so the copies of later
  // pieces run under the GEMMs of earlier ones.  Its tables are already on
  // the device, so it queues no copy of its own.
  for (int k = 0; k < nch; ++k) {
    MC_CUDA(cudaStreamWaitEvent(s, done[static_cast<size_t>(k)], 0));
    if ((rc = run_muon(params + b[k], b[k + 1] - b[k], hp, nullptr, ws, P.compute,
                       norms_out ? norms_out + b[k] : nullptr, s, ws + P.tab_off[size_t(k)])) != MC_OK)
      return rc;
  }
  return MC_OK;
}

namespace {
// Host image of the device tables of one call (MomEntry[n], the per-group
// weight and update pointer arrays, NormEntry[n] for NorMuon), for a layout
// whose workspace starts at `ws`.
void build_muon_table(const mc_param* params, int n, const mc_hparams* hp, const mc_normuon* nm, uint8_t* ws,
                      const MuonLayout& L, uint8_t* tab) {
  std::memset(tab, 0, L.tab_bytes);
  MomEntry* ent = reinterpret_cast<MomEntry*>(tab);
  std::vector<float*> o32(static_cast<size_t>(n), nullptr);  // NorMuon: fp32 NS output per matrix
  int k = 0;
  for (const auto& g : L.groups) {
    const size_t xe = size_t(g.rows) * size_t(g.ld);
    for (size_t j = 0; j < g.members.size(); ++j, ++k) {
      const mc_param& q = params[g.members[j]];
      MomEntry& e = ent[k];
      e.g = q.g;
      e.m = q.m;
      e.xl = reinterpret_cast<__nv_bfloat16*>(ws + g.off_xl) + j * xe;
      if (L.normuon) o32[static_cast<size_t>(k)] = reinterpret_cast<float*>(ws + g.off_xf) + j * xe;
      e.xb = reinterpret_cast<__nv_bfloat16*>(ws + g.off_xb[0]) + j * xe;
      e.rows = q.rows;
      e.cols = q.cols;
      e.ld = g.ld;
      e.cta_begin = L.cta_begin[k];
      e.g_f32 = q.g_dtype == MC_F32;
      e.vec = (q.cols % 8) == 0;
      e.orig = g.members[j];
      void** wp = reinterpret_cast<void**>(tab + g.off_wptr);
      float** up = reinterpret_cast<float**>(tab + g.off_uptr);
      wp[j] = q.w;
      up[j] = q.update_out;
    }
  }
  if (L.n_thin) {
    ThinEntry* te = reinterpret_cast<ThinEntry*>(tab + L.off_ttab);
    int t = 0, kk = 0;
    long long ctas = 0;
    for (const auto& g : L.groups) {
      const size_t xe = size_t(g.rows) * size_t(g.ld);
      for (size_t j = 0; j < g.members.size(); ++j, ++kk) {
        if (!g.thin) continue;
        const mc_param& q = params[g.members[j]];
        ThinEntry& e = te[t];
        e.xh = reinterpret_cast<const __nv_bfloat16*>(ws + g.off_xb[0]) + j * xe;
        e.xl = reinterpret_cast<const __nv_bfloat16*>(ws + g.off_xl) + j * xe;
        e.xf = reinterpret_cast<float*>(ws + g.off_xf) + j * xe;
        e.w = nm ? nullptr : q.w;  // NorMuon keeps O in xf for its row pass
        e.u = nm ? nullptr : q.update_out;
        e.pmat = reinterpret_cast<float*>(ws + L.off_pmat) + size_t(t) * THIN_PMAT;
        e.ld = g.ld;
        e.cols = q.cols;
        e.n = g.n;
        e.cta_begin = ctas;
        e.m = static_cast<int>(g.m);
        e.tall = g.tall ? 1 : 0;
        e.w_f32 = q.w_dtype == MC_F32;
        e.prob = g.prob_base + static_cast<int>(j);
        e.rms = hp->rms_scale * std::sqrt(static_cast<float>(std::max(q.rows, q.cols)));
        ctas += (g.n + THIN_COLS - 1) / THIN_COLS;
        ++t;
      }
    }
  }
  if (nm) {
    NormEntry* ne = reinterpret_cast<NormEntry*>(tab + L.off_ntab);
    long long rb = 0;
    for (int kk = 0; kk < n; ++kk) {
      const mc_param& q = params[ent[kk].orig];
      NormEntry& e = ne[kk];
      e.o = o32[static_cast<size_t>(kk)];
      e.v = nm->v[ent[kk].orig];
      e.w = q.w;
      e.u = q.update_out;
      e.rows = q.rows;
      e.cols = q.cols;
      e.ld = ent[kk].ld;
      e.row_base = rb;
      e.cta_begin = L.cta_begin[kk];
      e.rms = hp->rms_scale * std::sqrt(static_cast<float>(std::max(q.rows, q.cols)));
      e.w_f32 = q.w_dtype == MC_F32;
      e.vec = (q.cols % 8) == 0;
      rb += q.rows;
    }
  }
}

// One piece of the list; `tab_dev`: where the caller uploaded its tables.
int run_muon(const mc_param* params, int n, const mc_hparams* hp, const mc_normuon* nm, void* workspace,
             size_t workspace_bytes, float* norms_out, cudaStream_t s, uint8_t* tab_dev) {
  int rc = MC_OK;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st)) != MC_OK) return rc;

  MuonLayout L;
  plan_muon(params, n, L, nm != nullptr);
  if (workspace) {
    if (workspace_bytes < L.total)
      return fail(MC_ERR_NOSPC, "workspace has " + std::to_string(workspace_bytes) + " bytes, needs " +
                                    std::to_string(L.total));
  } else if ((rc = own_workspace(*st, L.total, &workspace)) != MC_OK) {
    return rc;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  // ---- device tables (uploaded by the caller, ahead of every piece)
  uint8_t* tb = tab_dev;

  // ---- momentum, Nesterov, fp32/bf16 iterate, norm partials
  const MomEntry* dtab = reinterpret_cast<const MomEntry*>(tb);
  double* partials = reinterpret_cast<double*>(ws + L.off_partials);
  float* scale = reinterpret_cast<float*>(ws + L.off_scale);
  double mom_bytes = 0;
  for (int i = 0; i < n; ++i)
    mom_bytes += double(params[i].rows) * double(params[i].cols) * ((params[i].g_dtype == MC_F32 ? 4 : 2) + 8 + 4);
  {
    ProfScope prof(K_MOMENTUM, s, 0, 0, mom_bytes);
    momentum_kernel<<<static_cast<unsigned>(L.total_ctas), MOM_THREADS, 0, s>>>(dtab, n, partials, hp->mu,
                                                                                 hp->nesterov ? 1 : 0);
    MC_CUDA(cudaGetLastError());
  }
  {
    ProfScope prof(K_FINALIZE, s);
    norm_finalize_kernel<<<(n * 32 + 255) / 256, 256, 0, s>>>(dtab, n, partials, L.total_ctas, hp->eps, scale,
                                                              norms_out, st->err_ptr);
    MC_CUDA(cudaGetLastError());
  }

  // ---- tensor maps
  std::vector<GroupMaps> maps(L.groups.size());
  std::vector<int> tc;  // groups on the tensor cores (the others take the thin path)
  for (size_t gi = 0; gi < L.groups.size(); ++gi) {
    if (L.groups[gi].thin) continue;
    tc.push_back(static_cast<int>(gi));
    if ((rc = build_group_maps(L.groups[gi], ws, maps[gi])) != MC_OK) return rc;
  }
  const ThinEntry* ttab = reinterpret_cast<const ThinEntry*>(tb + L.off_ttab);
  float* tpart = reinterpret_cast<float*>(ws + L.off_tpart);
  double thin_flops = 0;
  for (const auto& g : L.groups)
    if (g.thin)
      thin_flops += double(g.members.size()) * (4.0 * double(g.m) * double(g.m) * double(g.n) +
                                                2.0 * double(g.m) * double(g.m) * double(g.m));

  // ---- Newton-Schulz iterations, MAX_GROUPS problem groups per launch.
  // Iterations it < kMixedIters take a*X from the hi + lo iterate; later ones
  // fold a*I into B (see the precision note in umma_gemm.cuh).
  const int ng = static_cast<int>(tc.size());
  for (int it = 0; it < hp->ns_steps; ++it) {
    const int par = it & 1;
    const bool first = it == 0, last = it + 1 == hp->ns_steps;
    const bool mixed = it < kMixedIters;
    const float ca = hp->coeffs ? hp->coeffs[3 * it] : hp->a;
    const float cb = hp->coeffs ? hp->coeffs[3 * it + 1] : hp->b;
    const float cc = hp->coeffs ? hp->coeffs[3 * it + 2] : hp->c;
    // Batches of up to MAX_GROUPS problem groups per launch, one list per
    // phase and tile shape (see kNarrowMaxK); every Gram launch of the
    // iteration is enqueued before any polynomial launch, and those before
    // any apply launch, so each group's three phases stay in order.
    std::vector<GemmBatch> grams[2], polys[2], applies[2];
    for (int ti = 0; ti < ng; ++ti) {
      const int gi = tc[static_cast<size_t>(ti)];
      const NsGroup& g = L.groups[gi];
      const GroupMaps& Mp = maps[gi];
      const double cnt = double(g.members.size()), dm = double(g.m), dn = double(g.n);
      const int wide_gram = g.n > kNarrowMaxK ? 1 : 0;   // contraction n
      const int wide_m = g.m > kNarrowMaxK ? 1 : 0;      // contraction m (polynomial, apply)
      const int wide_apply = (wide_m || (!mixed && !last)) ? 1 : 0;
      // A = s^2 X X^T  (oriented; tall matrices read MN-major: X^T X)
      GemmGroup G = base_group(g);
      G.M = G.N = static_cast<int>(g.m);
      G.K = static_cast<int>(g.n);
      G.sched = SCHED_SYM;
      G.a_mn = G.b_mn = g.tall ? 1 : 0;
      G.d = ws + g.off_a;
      G.d_ld = g.ldm;
      G.d_bs = g.m * g.ldm;
      G.scale = first ? scale : nullptr;
      // symmetric: the entries on and above the diagonal, 2n flops each
      add_to_batch(grams[wide_gram], *st, g.tall ? Mp.x_mn[par] : Mp.x_k[par], g.tall ? Mp.x_mn[par] : Mp.x_k[par], G,
                   wide_gram, dm * (dm + 1) * dn * cnt, 2.0 * dm * dm * dn * cnt, Mp.ok_ab ? &Mp.a_e : nullptr);
      // B = b A + c A A
      G = base_group(g);
      G.M = G.N = G.K = static_cast<int>(g.m);
      G.sched = SCHED_SYM;
      G.src = ws + g.off_a;
      G.src_ld = g.ldm;
      G.src_bs = g.m * g.ldm;
      G.d = ws + g.off_b;
      G.d_ld = g.ldm;
      G.d_bs = g.m * g.ldm;
      G.coef_acc = cc;
      G.coef_src = cb;
      G.diag = mixed ? 0.f : ca;
      add_to_batch(polys[wide_m], *st, Mp.a_k, Mp.a_k, G, wide_m, dm * dm * (dm + 1) * cnt, 2.0 * dm * dm * dm * cnt,
                   Mp.ok_ab ? &Mp.b_e : nullptr, &Mp.a_e);
      // X' = s (a X + B X)   (tall: s (a X + X B), in the stored layout)
      G = base_group(g);
      G.M = static_cast<int>(g.rows);
      G.N = static_cast<int>(g.cols);
      G.K = static_cast<int>(g.m);
      G.sched = SCHED_DENSE;
      G.a_mn = 0;
      G.b_mn = g.tall ? 0 : 1;
      G.xh = reinterpret_cast<const __nv_bfloat16*>(ws + g.off_xb[par]);
      G.xh_ld = g.ld;
      G.xh_bs = g.rows * g.ld;
      G.xl = reinterpret_cast<__nv_bfloat16*>(ws + g.off_xl);
      G.xl_ld = g.ld;
      G.xl_bs = g.rows * g.ld;
      G.xf = nm ? reinterpret_cast<float*>(ws + g.off_xf) : nullptr;
      G.xf_ld = g.ld;
      G.xf_bs = g.rows * g.ld;
      G.xf_read = mixed ? 1 : 0;
      G.xl_write = (!last && it + 1 < kMixedIters) ? 1 : 0;
      // NorMuon keeps the last iterate (the NS output O) in fp32 for the row pass.
      G.xf_write = (last && nm) ? 1 : 0;
      G.d = ws + g.off_xb[par ^ 1];
      G.d_ld = g.ld;
      G.d_bs = g.rows * g.ld;
      G.scale = first ? scale : nullptr;
      G.coef_src = ca;
      if (last && !nm) {
        G.w_ptrs = reinterpret_cast<void* const*>(tb + g.off_wptr);
        bool any_u = false;
        for (int i : g.members) any_u |= params[i].update_out != nullptr;
        G.u_ptrs = any_u ? reinterpret_cast<float* const*>(tb + g.off_uptr) : nullptr;
        G.w_f32 = g.w_f32;
        G.w_vec = g.w_f32 ? (g.cols % 4 == 0) : (g.cols % 8 == 0);
        G.rms = hp->rms_scale * std::sqrt(static_cast<float>(std::max(g.rows, g.cols)));
        G.decay = host_decay(hp);
        G.step = -hp->lr * G.rms;
        G.lr_wd = hp->lr_wd;
      }
      const double fa = 2.0 * dm * dm * dn * cnt;
      // epilogue maps: none for the last apply (each weight has its own
      // pointer); the iterate by 32 columns with its lo half for the mixed
      // apply, by 64 columns for the plain one
      const bool final_apply = last && !nm;
      const CUtensorMap* eo = nullptr;
      const CUtensorMap* ei = nullptr;
      const CUtensorMap* ei2 = nullptr;
      if (!final_apply && mixed && Mp.ok_x32) {
        eo = &Mp.x_e32[par ^ 1];
        ei = &Mp.x_e32[par];
        ei2 = &Mp.xl_e32;
      } else if (!final_apply && !mixed && Mp.ok_x64 && !(last && nm)) {
        // (NorMuon's last apply writes the fp32 NS output through the
        // warp-coalesced path instead)
        eo = &Mp.x_e64[par ^ 1];
      }
      add_to_batch(applies[wide_apply], *st, g.tall ? Mp.x_k[par] : Mp.b_k, g.tall ? Mp.b_k : Mp.x_mn[par], G,
                   wide_apply, fa, fa, eo, ei, ei2);
    }
    for (int w = 0; w < 2; ++w)
      for (const auto& b : grams[w])
        if ((rc = w ? launch_gemm<EPI_GRAM, 1>(b.p, *st, s, K_GRAM, b.f, b.fd)
                    : launch_gemm<EPI_GRAM, 0>(b.p, *st, s, K_GRAM, b.f, b.fd)) != MC_OK)
          return rc;
    for (int w = 0; w < 2; ++w)
      for (const auto& b : polys[w])
        if ((rc = w ? launch_gemm<EPI_POLY, 1>(b.p, *st, s, K_POLY, b.f, b.fd)
                    : launch_gemm<EPI_POLY, 0>(b.p, *st, s, K_POLY, b.f, b.fd)) != MC_OK)
          return rc;
    for (int w = 0; w < 2; ++w)
      for (const auto& b : applies[w]) {
        if (last && !nm) {
          rc = w ? launch_gemm<EPI_APPLY_FINAL, 1>(b.p, *st, s, K_APPLY_FINAL, b.f)
                 : launch_gemm<EPI_APPLY_FINAL, 0>(b.p, *st, s, K_APPLY_FINAL, b.f);
        } else if (mixed) {
          rc = w ? launch_gemm<EPI_APPLY_MIXED, 1>(b.p, *st, s, K_APPLY_MIXED, b.f)
                 : launch_gemm<EPI_APPLY_MIXED, 0>(b.p, *st, s, K_APPLY_MIXED, b.f);
        } else {
          rc = w ? launch_gemm<EPI_APPLY, 1>(b.p, *st, s, K_APPLY, b.f) : launch_gemm<EPI_APPLY, 0>(b.p, *st, s, K_APPLY, b.f);
        }
      if (rc != MC_OK) return rc;
    }
    if (L.n_thin) {
      // thin matrices: fp32 Gram chunks, P = aI + bA + cA^2, X <- P X (the
      // last iteration writes W, or keeps O for NorMuon)
      ProfScope prof(K_NS_THIN, s, thin_flops, thin_flops);
      thin_gram_kernel<<<static_cast<unsigned>(L.thin_ctas), THIN_THREADS, 0, s>>>(ttab, L.n_thin, tpart, scale,
                                                                                  first ? 1 : 0);
      MC_CUDA(cudaGetLastError());
      thin_poly_kernel<<<static_cast<unsigned>(L.n_thin), THIN_THREADS, 0, s>>>(ttab, tpart, ca, cb, cc);
      MC_CUDA(cudaGetLastError());
      thin_apply_kernel<<<static_cast<unsigned>(L.thin_ctas), THIN_THREADS, 0, s>>>(
          ttab, L.n_thin, last ? 1 : 0, host_decay(hp), -hp->lr, hp->lr_wd);
      MC_CUDA(cudaGetLastError());
    }
  }
  if (nm) {
    // NorMuon: row sums of squares of O, then the row factors, then the update.
    const NormEntry* ntab = reinterpret_cast<const NormEntry*>(tb + L.off_ntab);
    float* rowsq = reinterpret_cast<float*>(ws + L.off_rowsq);
    float* rowf = reinterpret_cast<float*>(ws + L.off_rowf);
    double o_bytes = 0, w_bytes = 0;
    for (int i = 0; i < n; ++i) {
      const double el = double(params[i].rows) * double(params[i].cols);
      o_bytes += 4.0 * el;
      w_bytes += el * (4.0 + 2.0 * (params[i].w_dtype == MC_F32 ? 4 : 2) + (params[i].update_out ? 4 : 0));
    }
    {
      ProfScope prof(K_NORM_ROWS, s, 0, 0, o_bytes);
      const long long rows_per_cta = NORM_THREADS / 32;
      normuon_rowsq_kernel<<<static_cast<unsigned>((L.total_rows + rows_per_cta - 1) / rows_per_cta),
                             NORM_THREADS, 0, s>>>(ntab, n, L.total_rows, rowsq);
      MC_CUDA(cudaGetLastError());
      normuon_finalize_kernel<<<static_cast<unsigned>(n), NORM_THREADS, 0, s>>>(ntab, rowsq, rowf, nm->beta2,
                                                                                nm->eps);
      MC_CUDA(cudaGetLastError());
    }
    {
      ProfScope prof(K_NORM_APPLY, s, 0, 0, w_bytes);
      normuon_apply_kernel<<<static_cast<unsigned>(L.total_ctas), NORM_THREADS, 0, s>>>(
          ntab, n, rowf, host_decay(hp), -hp->lr, hp->lr_wd);
      MC_CUDA(cudaGetLastError());
    }
  }
  return MC_OK;
}
}  // namespace

// =========================================================================
namespace {
struct QkLayout {
  size_t off_q, off_k, off_keys, total;
};
QkLayout plan_qk(int B, int S, int H, int dh) {
  QkLayout L;
  const size_t qe = size_t(B) * size_t(S) * size_t(H) * size_t(dh);
  L.off_q = 0;
  L.off_k = align_up(2 * qe, 1024);
  L.off_keys = align_up(L.off_k + 2 * qe, 1024);
  L.total = align_up(L.off_keys + sizeof(int) * size_t(H), 1024);
  return L;
}
int validate_qk_dims(int B, int S, int D, int H, int dh) {
  if (B < 1 || S < 1 || D < 1 || H < 1 || dh < 1) return fail(MC_ERR_INVAL, "B, S, D, H, dh must be >= 1");
  if (D % 8 || dh % 8) return fail(MC_ERR_INVAL, "D and dh must be multiples of 8");
  if (int64_t(B) * S > (int64_t(1) << 31) - 1 || int64_t(H) * dh > (1 << 24) || D > (1 << 24))
    return fail(MC_ERR_INVAL, "problem too large");
  return MC_OK;
}
}  // namespace

MC_API size_t mc_qk_workspace_size(int B, int S, int D, int H, int dh) {
  if (validate_qk_dims(B, S, D, H, dh) != MC_OK) return 0;
  return plan_qk(B, S, H, dh).total;
}

MC_API int mc_qk_max_logit(const void* x, const void* wq, const void* wk, int B, int S, int D, int H, int dh,
                           int causal, float* smax_out, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_qk_dims(B, S, D, H, dh);
  if (rc != MC_OK) return rc;
  if (!x || !wq || !wk || !smax_out) return fail(MC_ERR_INVAL, "NULL x, wq, wk or smax_out");
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wk) || !aligned16(smax_out) ||
      (workspace && !aligned16(workspace)))
    return fail(MC_ERR_ALIGN, "pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st)) != MC_OK) return rc;
  const QkLayout L = plan_qk(B, S, H, dh);
  if (workspace) {
    if (workspace_bytes < L.total)
      return fail(MC_ERR_NOSPC, "workspace has " + std::to_string(workspace_bytes) + " bytes, needs " +
                                    std::to_string(L.total));
  } else if ((rc = own_workspace(*st, L.total, &workspace)) != MC_OK) {
    return rc;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* keys = reinterpret_cast<int*>(ws + L.off_keys);
  const int HD = H * dh;
  const int64_t BS = int64_t(B) * S;

  {
    ProfScope prof(K_QK_KEYS, s);
    qk_keys_init_kernel<<<(H + 255) / 256, 256, 0, s>>>(keys, H);
    MC_CUDA(cudaGetLastError());
  }

  // Q = X W_q^T and K = X W_k^T, bf16 out, one launch.
  GemmParams proj;
  std::memset(&proj, 0, sizeof(proj));
  proj.err = st->err_ptr;
  for (int which = 0; which < 2; ++which) {
    if ((rc = map_batched(&proj.map_a[which], x, 1, BS, D, D, HALF)) != MC_OK) return rc;
    if ((rc = map_batched(&proj.map_b[which], which == 0 ? wq : wk, 1, HD, D, D, HALF)) != MC_OK) return rc;
    GemmGroup G;
    std::memset(&G, 0, sizeof(G));
    G.M = static_cast<int>(BS);
    G.N = HD;
    G.K = D;
    G.count = 1;
    G.sched = SCHED_DENSE;
    G.layout = LAYOUT_BATCHED;
    G.heads = 1;
    G.band = 8;
    G.d = ws + (which == 0 ? L.off_q : L.off_k);
    G.d_ld = HD;
    // the projection's full 32 x 64 output blocks leave by tensor stores
    bool e_ok = false;
    if ((rc = map_epilogue(&proj.map_eo[which], &e_ok, G.d, 1, BS, HD, HD, false)) != MC_OK) return rc;
    G.tma_epi = e_ok ? 1 : 0;
    finish_group(proj, which, G, 1);
  }
  if ((rc = launch_gemm<EPI_STORE, 1>(proj, *st, s, K_QK_PROJ, 2.0 * 2.0 * double(BS) * HD * D)) != MC_OK)
    return rc;

  // Per-head causal max of Q K^T / sqrt(dh), scores never stored.
  GemmParams cm;
  std::memset(&cm, 0, sizeof(cm));
  cm.err = st->err_ptr;
  {
    const uint64_t dims[4] = {uint64_t(dh), uint64_t(H), uint64_t(S), uint64_t(B)};
    const uint64_t strides[3] = {uint64_t(dh) * 2, uint64_t(HD) * 2, uint64_t(S) * uint64_t(HD) * 2};
    const uint32_t box_q[4] = {64, 1, HALF, 1};
    const uint32_t box_k[4] = {64, 1, HALF, 1};
    if ((rc = make_map(&cm.map_a[0], ws + L.off_q, 4, dims, strides, box_q)) != MC_OK) return rc;
    if ((rc = make_map(&cm.map_b[0], ws + L.off_k, 4, dims, strides, box_k)) != MC_OK) return rc;
    GemmGroup G;
    std::memset(&G, 0, sizeof(G));
    G.M = G.N = S;
    G.K = dh;
    G.count = B * H;
    G.heads = H;
    G.layout = LAYOUT_HEADS;
    G.sched = causal ? SCHED_CAUSAL : SCHED_DENSE;
    G.band = 8;
    G.mask_causal = causal ? 1 : 0;
    G.keys = keys;
    G.out_scale = 1.f / std::sqrt(static_cast<float>(dh));
    finish_group(cm, 0, G, 0);
  }
  const double pairs = causal ? double(S) * (double(S) + 1) / 2 : double(S) * S;
  if ((rc = launch_causal_max(cm, *st, s, K_QK_CMAX, 2.0 * dh * pairs * B * H, true)) != MC_OK) return rc;
  {
    ProfScope prof(K_QK_KEYS, s);
    qk_keys_decode_kernel<<<(H + 255) / 256, 256, 0, s>>>(keys, smax_out, H);
    MC_CUDA(cudaGetLastError());
  }
  return MC_OK;
}

MC_API int mc_qk_clip(void* wq, void* wk, int H, int dh, int D, const float* smax, float tau, float alpha,
                      float* gamma_out, int32_t* mask_out, void* stream) {
  if (H < 1 || dh < 1 || D < 1) return fail(MC_ERR_INVAL, "H, dh, D must be >= 1");
  if (int64_t(H) * dh > (1 << 24) || D > (1 << 24)) return fail(MC_ERR_INVAL, "problem too large");
  if (!wq || !wk || !smax) return fail(MC_ERR_INVAL, "NULL wq, wk or smax");
  if (wq == wk) return fail(MC_ERR_INVAL, "wq and wk must not alias");
  if (!std::isfinite(tau) || !(tau > 0.f)) return fail(MC_ERR_INVAL, "tau must be finite and > 0");
  if (!std::isfinite(alpha) || alpha < 0.f || alpha > 1.f) return fail(MC_ERR_INVAL, "alpha must be in [0, 1]");
  if (!aligned16(wq) || !aligned16(wk) || !aligned16(smax) || (gamma_out && !aligned16(gamma_out)) ||
      (mask_out && !aligned16(mask_out)))
    return fail(MC_ERR_ALIGN, "pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != MC_OK) return rc;
  const dim3 grid(static_cast<unsigned>(H * dh), 2);
  ProfScope prof(K_QK_CLIP, s);
  qk_clip_kernel<<<grid, 256, 0, s>>>(static_cast<__nv_bfloat16*>(wq), static_cast<__nv_bfloat16*>(wk), H, dh, D,
                                      smax, tau, alpha, gamma_out, mask_out, D % 8 == 0 ? 1 : 0);
  MC_CUDA(cudaGetLastError());
  return MC_OK;
}

// =========================================================================
// QK-Clip over an explicit slice map (MLA and fused projection layouts).
MC_API int mc_qk_clip_slices(const mc_clip_slice* slices, int n, const float* smax, int H, float tau,
                             float* gamma_out, int32_t* mask_out, void* stream) {
  if (n < 0 || (n > 0 && !slices)) return fail(MC_ERR_INVAL, "slices must be non-NULL when n > 0, and n >= 0");
  if (H < 1 || H > (1 << 24)) return fail(MC_ERR_INVAL, "H must be in [1, 2^24]");
  if (!smax) return fail(MC_ERR_INVAL, "NULL smax");
  if (!std::isfinite(tau) || !(tau > 0.f)) return fail(MC_ERR_INVAL, "tau must be finite and > 0");
  if (!aligned16(smax) || (gamma_out && !aligned16(gamma_out)) || (mask_out && !aligned16(mask_out)))
    return fail(MC_ERR_ALIGN, "pointers must be 16-byte aligned");
  struct Span {
    uintptr_t lo, hi;
    int idx;
  };
  std::vector<Span> spans;
  spans.reserve(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    const mc_clip_slice& c = slices[i];
    const std::string at = "slices[" + std::to_string(i) + "]: ";
    if (!c.w) return fail(MC_ERR_INVAL, at + "NULL w");
    if (c.dtype != MC_F32 && c.dtype != MC_BF16) return fail(MC_ERR_INVAL, at + "dtype must be MC_F32 or MC_BF16");
    if (c.reserved != 0) return fail(MC_ERR_INVAL, at + "reserved must be 0");
    if (c.cols < 1 || c.row_begin < 0 || c.row_end <= c.row_begin)
      return fail(MC_ERR_INVAL, at + "need cols >= 1 and 0 <= row_begin < row_end");
    if (c.row_end > (int64_t(1) << 40) / c.cols || c.row_end - c.row_begin > INT_MAX)
      return fail(MC_ERR_INVAL, at + "slice too large");
    if (c.head < 0 || c.head >= H) return fail(MC_ERR_INVAL, at + "head out of [0, H)");
    if (!std::isfinite(c.exponent) || c.exponent < 0.f || c.exponent > 1.f)
      return fail(MC_ERR_INVAL, at + "exponent must be in [0, 1]");
    if (!aligned16(c.w)) return fail(MC_ERR_ALIGN, at + "w must be 16-byte aligned");
    const uintptr_t es = c.dtype == MC_F32 ? 4 : 2;
    const uintptr_t base = reinterpret_cast<uintptr_t>(c.w);
    spans.push_back({base + uintptr_t(c.row_begin) * uintptr_t(c.cols) * es,
                     base + uintptr_t(c.row_end) * uintptr_t(c.cols) * es, i});
  }
  std::sort(spans.begin(), spans.end(), [](const Span& a, const Span& b) { return a.lo < b.lo; });
  for (size_t i = 1; i < spans.size(); ++i)
    if (spans[i].lo < spans[i - 1].hi)
      return fail(MC_ERR_INVAL, "slices[" + std::to_string(spans[i - 1].idx) + "] and slices[" +
                                    std::to_string(spans[i].idx) + "] overlap in memory");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc != MC_OK) return rc;
  if (gamma_out || mask_out) {
    ProfScope prof(K_QK_KEYS, s);
    qk_gamma_kernel<<<(H + 255) / 256, 256, 0, s>>>(smax, H, tau, gamma_out, mask_out);
    MC_CUDA(cudaGetLastError());
  }
  ClipTable T;
  std::memset(&T, 0, sizeof(T));
  double bytes = 0;
  auto flush = [&]() -> int {
    if (T.n == 0) return MC_OK;
    ProfScope prof(K_QK_CLIP_SLICES, s, 0, 0, bytes);
    qk_clip_slices_kernel<<<static_cast<unsigned>(T.row_end[T.n - 1]), 256, 0, s>>>(T, smax, tau);
    MC_CUDA(cudaGetLastError());
    std::memset(&T, 0, sizeof(T));
    bytes = 0;
    return MC_OK;
  };
  for (int i = 0; i < n; ++i) {
    const mc_clip_slice& c = slices[i];
    if (c.exponent == 0.f) continue;  // gamma^0 = 1: nothing to write
    const long long rows = c.row_end - c.row_begin;
    const long long prev = T.n ? T.row_end[T.n - 1] : 0;
    if (T.n == CLIP_MAX_SLICES || prev + rows > INT_MAX) {
      if ((rc = flush()) != MC_OK) return rc;
    }
    const long long base = T.n ? T.row_end[T.n - 1] : 0;
    const int es = c.dtype == MC_F32 ? 4 : 2;
    ClipSlice& d = T.s[T.n];
    d.w = c.w;
    d.row_begin = c.row_begin;
    d.cols = c.cols;
    d.exponent = c.exponent;
    d.head = c.head;
    d.f32 = c.dtype == MC_F32 ? 1 : 0;
    d.vec = (c.cols * es) % 16 == 0 ? 1 : 0;
    T.row_end[T.n] = base + rows;
    ++T.n;
    bytes += 2.0 * double(rows) * double(c.cols) * es;  // read + write if the head clips
  }
  return flush();
}

// =========================================================================
// Per-head causal max logit of multi-head latent attention.
namespace {
struct MlaLayout {
  size_t off_qc, off_kc, off_qr, off_kr, off_keys, total;
};
MlaLayout plan_mla(int B, int S, int H, int dc, int dr) {
  MlaLayout L;
  const size_t bs = size_t(B) * size_t(S);
  L.off_qc = 0;
  L.off_kc = align_up(L.off_qc + 2 * bs * size_t(H) * size_t(dc), 1024);
  L.off_qr = align_up(L.off_kc + 2 * bs * size_t(H) * size_t(dc), 1024);
  L.off_kr = align_up(L.off_qr + 2 * bs * size_t(H) * size_t(dr), 1024);
  L.off_keys = align_up(L.off_kr + 2 * bs * size_t(dr), 1024);
  L.total = align_up(L.off_keys + sizeof(int) * size_t(H), 1024);
  return L;
}
int validate_mla_dims(int B, int S, int D, int H, int dc, int dr) {
  if (B < 1 || S < 1 || D < 1 || H < 1 || dc < 1 || dr < 1)
    return fail(MC_ERR_INVAL, "B, S, D, H, dc, dr must be >= 1");
  if (D % 8 || dr % 8) return fail(MC_ERR_INVAL, "D and dr must be multiples of 8");
  if (dc % BK) return fail(MC_ERR_INVAL, "dc must be a multiple of 64");
  if (int64_t(B) * S > (int64_t(1) << 31) - 1 || int64_t(H) * dc > (1 << 24) || int64_t(H) * dr > (1 << 24) ||
      D > (1 << 24))
    return fail(MC_ERR_INVAL, "problem too large");
  return MC_OK;
}
}  // namespace

MC_API size_t mc_mla_workspace_size(int B, int S, int D, int H, int dc, int dr) {
  if (validate_mla_dims(B, S, D, H, dc, dr) != MC_OK) return 0;
  return plan_mla(B, S, H, dc, dr).total;
}

MC_API int mc_mla_max_logit(const void* x, const void* wqc, const void* wkc, const void* wqr, const void* wkr,
                            int B, int S, int D, int H, int dc, int dr, int causal, float* smax_out,
                            void* workspace, size_t workspace_bytes, void* stream) {
  int rc = validate_mla_dims(B, S, D, H, dc, dr);
  if (rc != MC_OK) return rc;
  if (!x || !wqc || !wkc || !wqr || !wkr || !smax_out)
    return fail(MC_ERR_INVAL, "NULL x, wqc, wkc, wqr, wkr or smax_out");
  if (!aligned16(x) || !aligned16(wqc) || !aligned16(wkc) || !aligned16(wqr) || !aligned16(wkr) ||
      !aligned16(smax_out) || (workspace && !aligned16(workspace)))
    return fail(MC_ERR_ALIGN, "pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st)) != MC_OK) return rc;
  const MlaLayout L = plan_mla(B, S, H, dc, dr);
  if (workspace) {
    if (workspace_bytes < L.total)
      return fail(MC_ERR_NOSPC, "workspace has " + std::to_string(workspace_bytes) + " bytes, needs " +
                                    std::to_string(L.total));
  } else if ((rc = own_workspace(*st, L.total, &workspace)) != MC_OK) {
    return rc;
  }
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* keys = reinterpret_cast<int*>(ws + L.off_keys);
  const int64_t BS = int64_t(B) * S;
  {
    ProfScope prof(K_QK_KEYS, s);
    qk_keys_init_kernel<<<(H + 255) / 256, 256, 0, s>>>(keys, H);
    MC_CUDA(cudaGetLastError());
  }

  // q^C = X W_qC^T, k^C = X W_kC^T, q^R = X W_qR^T, k^R = X W_kR^T: one launch.
  GemmParams proj;
  std::memset(&proj, 0, sizeof(proj));
  proj.err = st->err_ptr;
  const void* wts[4] = {wqc, wkc, wqr, wkr};
  const int outs[4] = {H * dc, H * dc, H * dr, dr};
  const size_t offs[4] = {L.off_qc, L.off_kc, L.off_qr, L.off_kr};
  double proj_flops = 0;
  for (int which = 0; which < 4; ++which) {
    if ((rc = map_batched(&proj.map_a[which], x, 1, BS, D, D, HALF)) != MC_OK) return rc;
    if ((rc = map_batched(&proj.map_b[which], wts[which], 1, outs[which], D, D, HALF)) != MC_OK) return rc;
    GemmGroup G;
    std::memset(&G, 0, sizeof(G));
    G.M = static_cast<int>(BS);
    G.N = outs[which];
    G.K = D;
    G.count = 1;
    G.sched = SCHED_DENSE;
    G.layout = LAYOUT_BATCHED;
    G.heads = 1;
    G.band = 8;
    G.d = ws + offs[which];
    G.d_ld = outs[which];
    bool e_ok = false;
    if ((rc = map_epilogue(&proj.map_eo[which], &e_ok, G.d, 1, BS, outs[which], outs[which], false)) != MC_OK)
      return rc;
    G.tma_epi = e_ok ? 1 : 0;
    finish_group(proj, which, G, 1);
    proj_flops += 2.0 * double(BS) * outs[which] * D;
  }
  if ((rc = launch_gemm<EPI_STORE, 1>(proj, *st, s, K_MLA_PROJ, proj_flops)) != MC_OK) return rc;

  // s_h(i, j) = (q^C_hi . k^C_hj + q^R_hi . k^R_j) / sqrt(dc + dr): one contraction
  // of length dc + dr whose first dc columns come from the content pair and
  // the rest from the rotary pair (the rotary key has a single shared head).
  GemmParams cm;
  std::memset(&cm, 0, sizeof(cm));
  cm.err = st->err_ptr;
  {
    const uint32_t box[4] = {64, 1, HALF, 1};
    const uint64_t dc_dims[4] = {uint64_t(dc), uint64_t(H), uint64_t(S), uint64_t(B)};
    const uint64_t dc_str[3] = {uint64_t(dc) * 2, uint64_t(H) * dc * 2, uint64_t(S) * H * dc * 2};
    const uint64_t qr_dims[4] = {uint64_t(dr), uint64_t(H), uint64_t(S), uint64_t(B)};
    const uint64_t qr_str[3] = {uint64_t(dr) * 2, uint64_t(H) * dr * 2, uint64_t(S) * H * dr * 2};
    const uint64_t kr_dims[4] = {uint64_t(dr), 1, uint64_t(S), uint64_t(B)};
    const uint64_t kr_str[3] = {uint64_t(dr) * 2, uint64_t(dr) * 2, uint64_t(S) * dr * 2};
    if ((rc = make_map(&cm.map_a[0], ws + L.off_qc, 4, dc_dims, dc_str, box)) != MC_OK) return rc;
    if ((rc = make_map(&cm.map_b[0], ws + L.off_kc, 4, dc_dims, dc_str, box)) != MC_OK) return rc;
    if ((rc = make_map(&cm.map_a[1], ws + L.off_qr, 4, qr_dims, qr_str, box)) != MC_OK) return rc;
    if ((rc = make_map(&cm.map_b[1], ws + L.off_kr, 4, kr_dims, kr_str, box)) != MC_OK) return rc;
    GemmGroup G;
    std::memset(&G, 0, sizeof(G));
    G.M = G.N = S;
    G.K = dc + dr;
    G.k_split = dc;
    G.count = B * H;
    G.heads = H;
    G.layout = LAYOUT_HEADS;
    G.sched = causal ? SCHED_CAUSAL : SCHED_DENSE;
    G.band = 8;
    G.mask_causal = causal ? 1 : 0;
    G.keys = keys;
    G.out_scale = 1.f / std::sqrt(static_cast<float>(dc + dr));
    finish_group(cm, 0, G, 0);
  }
  const double pairs = causal ? double(S) * (double(S) + 1) / 2 : double(S) * S;
  if ((rc = launch_causal_max(cm, *st, s, K_MLA_CMAX, 2.0 * (dc + dr) * pairs * B * H, true)) != MC_OK)
    return rc;
  {
    ProfScope prof(K_QK_KEYS, s);
    qk_keys_decode_kernel<<<(H + 255) / 256, 256, 0, s>>>(keys, smax_out, H);
    MC_CUDA(cudaGetLastError());
  }
  return MC_OK;
}

// Self-test of the bounded wait: one thread waits on an mbarrier that
// expects an arrival nobody makes, so the wait runs out after `limit` cycles,
// raises the abort flag and sets the device error word, and the kernel
// returns normally.
namespace mc {
__global__ void bounded_wait_selftest_kernel(int* err, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(smem_u32(&bar), 0, &abort_flag, err, limit);
}
}  // namespace mc

MC_API size_t mc_struct_size(int which) {
  switch (which) {
    case 0: return sizeof(mc_param);
    case 1: return sizeof(mc_hparams);
    case 2: return sizeof(mc_normuon);
    case 3: return sizeof(mc_clip_slice);
    case 4: return sizeof(mc_kernel_stat);
    default: return 0;
  }
}

MC_API int mc_selftest_bounded_wait(long long limit_cycles, void* stream) {
  if (limit_cycles < 1000 || limit_cycles > kWaitLimitCycles)
    return fail(MC_ERR_INVAL, "limit_cycles must be in [1000, 2^32]");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  const int rc = device_state(&st);
  if (rc != MC_OK) return rc;
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(st->err_ptr, limit_cycles);
  MC_CUDA(cudaGetLastError());
  return MC_OK;
}

MC_API int mc_device_status(void) {
  MC_CUDA(cudaDeviceSynchronize());
  int v = 0;
  MC_CUDA(cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)));
  if (v == 0) return MC_OK;
  const int zero = 0;
  MC_CUDA(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)));
  if (v & MC_DEV_ERR_TIMEOUT)
    return fail(MC_ERR_DEVICE, "a kernel abandoned a bounded wait (device error word " + std::to_string(v) + ")");
  return fail(MC_ERR_NONFINITE, "a Muon step met a non-finite Newton-Schulz input (a NaN or Inf gradient or "
                                "momentum); that matrix's norms_out entry is not finite and its W only decayed");
}

// =========================================================================
// Polar Express coefficient schedule (host only).
namespace {
// Gaussian elimination with partial pivoting on an augmented 4 x 5 system.
bool solve4(double (&m)[4][5], double (&x)[4]) {
  for (int col = 0; col < 4; ++col) {
    int piv = col;
    for (int r = col + 1; r < 4; ++r)
      if (std::fabs(m[r][col]) > std::fabs(m[piv][col])) piv = r;
    if (!(std::fabs(m[piv][col]) > 1e-300)) return false;
    if (piv != col)
      for (int k = 0; k < 5; ++k) std::swap(m[col][k], m[piv][k]);
    for (int r = col + 1; r < 4; ++r) {
      const double f = m[r][col] / m[col][col];
      for (int k = col; k < 5; ++k) m[r][k] -= f * m[col][k];
    }
  }
  for (int r = 3; r >= 0; --r) {
    double acc = m[r][4];
    for (int k = r + 1; k < 4; ++k) acc -= m[r][k] * x[k];
    x[r] = acc / m[r][r];
  }
  return true;
}

// Odd quintic closest to 1 in the max norm on [lo, hi]: Remez exchange over
// four alternation points (the two ends and the two interior extrema).
bool minimax_quintic(double lo, double hi, double& a, double& b, double& c) {
  const double kPi = 3.14159265358979323846;
  double pts[4];
  for (int k = 0; k < 4; ++k) pts[k] = lo + (hi - lo) * 0.5 * (1.0 - std::cos(kPi * k / 3.0));
  for (int it = 0; it < 200; ++it) {
    double m[4][5], sol[4];
    for (int i = 0; i < 4; ++i) {
      const double x = pts[i], x2 = x * x;
      m[i][0] = x;
      m[i][1] = x * x2;
      m[i][2] = x * x2 * x2;
      m[i][3] = (i & 1) ? -1.0 : 1.0;
      m[i][4] = 1.0;
    }
    if (!solve4(m, sol)) return false;
    a = sol[0];
    b = sol[1];
    c = sol[2];
    // p'(x) = a + 3b x^2 + 5c x^4 = 0: a quadratic in y = x^2
    const double disc = 9.0 * b * b - 20.0 * a * c;
    // No two interior extrema: the points cannot move, keep this solution.
    if (disc < 0.0 || c == 0.0) return true;
    const double sq = std::sqrt(disc);
    double ys[2] = {(-3.0 * b - sq) / (10.0 * c), (-3.0 * b + sq) / (10.0 * c)};
    double inner[2];
    int cnt = 0;
    for (double y : ys)
      if (y > 0.0) {
        const double x = std::sqrt(y);
        if (x > lo && x < hi && cnt < 2) inner[cnt++] = x;
      }
    if (cnt != 2) return true;
    if (inner[0] > inner[1]) std::swap(inner[0], inner[1]);
    const double next[4] = {lo, inner[0], inner[1], hi};
    double moved = 0.0;
    for (int k = 0; k < 4; ++k) moved = std::max(moved, std::fabs(next[k] - pts[k]));
    for (int k = 0; k < 4; ++k) pts[k] = next[k];
    if (moved <= 1e-15 * hi) return true;
  }
  return true;
}
}  // namespace

MC_API int mc_polar_express_coeffs(int steps, double l0, double safety, float* coeffs_out) {
  if (steps < 1 || steps >= 100) return fail(MC_ERR_INVAL, "steps must be in [1, 100)");
  if (!(l0 > 0.0 && l0 < 1.0)) return fail(MC_ERR_INVAL, "l0 must be in (0, 1)");
  if (!std::isfinite(safety) || safety < 0.0) return fail(MC_ERR_INVAL, "safety must be finite and >= 0");
  if (!coeffs_out) return fail(MC_ERR_INVAL, "NULL coeffs_out");
  std::vector<double> co(3 * static_cast<size_t>(steps));
  double lo = l0, hi = 1.0;
  for (int t = 0; t < steps; ++t) {
    double a = 15.0 / 8.0, b = -10.0 / 8.0, c = 3.0 / 8.0;
    if (hi - lo >= 1e-3 && !minimax_quintic(lo, hi, a, b, c))
      return fail(MC_ERR_UNSUPPORTED, "the Remez exchange did not converge at step " + std::to_string(t));
    co[3 * t] = a;
    co[3 * t + 1] = b;
    co[3 * t + 2] = c;
    const double l2 = lo * lo;
    lo = a * lo + b * lo * l2 + c * lo * l2 * l2;
    hi = 2.0 - lo;
  }
  const double s = 1.0 + safety;
  for (int t = 0; t < steps; ++t) {
    const bool last = t + 1 == steps;
    coeffs_out[3 * t] = static_cast<float>(last ? co[3 * t] : co[3 * t] / s);
    coeffs_out[3 * t + 1] = static_cast<float>(last ? co[3 * t + 1] : co[3 * t + 1] / (s * s * s));
    coeffs_out[3 * t + 2] = static_cast<float>(last ? co[3 * t + 2] : co[3 * t + 2] / (s * s * s * s * s));
  }
  return MC_OK;
}

// =========================================================================
// Ownership plan for the sharded data-parallel step (host only).
MC_API int mc_shard_plan(const int64_t* rows, const int64_t* cols, int n, int ns_steps, int world,
                         int32_t* owner_out, double* load_out) {
  if (n < 0 || world < 1 || ns_steps < 1) return fail(MC_ERR_INVAL, "need n >= 0, world >= 1, ns_steps >= 1");
  if (n > 0 && (!rows || !cols || !owner_out)) return fail(MC_ERR_INVAL, "NULL rows, cols or owner_out");
  std::vector<double> cost(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    if (rows[i] < 1 || cols[i] < 1) return fail(MC_ERR_INVAL, "matrix " + std::to_string(i) + " has a dimension < 1");
    const double m = static_cast<double>(std::min(rows[i], cols[i]));
    const double nn = static_cast<double>(std::max(rows[i], cols[i]));
    cost[static_cast<size_t>(i)] = ns_steps * (4.0 * m * m * nn + 2.0 * m * m * m);
  }
  std::vector<int> order(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) order[static_cast<size_t>(i)] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[size_t(a)] > cost[size_t(b)]; });
  std::vector<double> load(static_cast<size_t>(world), 0.0);
  for (int i : order) {
    int best = 0;
    for (int r = 1; r < world; ++r)
      if (load[size_t(r)] < load[size_t(best)]) best = r;
    owner_out[i] = best;
    load[size_t(best)] += cost[size_t(i)];
  }
  if (load_out)
    for (int r = 0; r < world; ++r) load_out[r] = load[size_t(r)];
  return MC_OK;
}

MC_API int mc_profile_begin(void) {
  for (auto& r : t_recs) {
    cudaEventDestroy(r.b);
    cudaEventDestroy(r.e);
  }
  t_recs.clear();
  t_prof = true;
  return MC_OK;
}

MC_API int mc_profile_end(mc_kernel_stat* out, int max_rows, int* rows) {
  t_prof = false;
  mc_kernel_stat acc[K_COUNT];
  std::memset(acc, 0, sizeof(acc));
  int rc = MC_OK;
  for (auto& r : t_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.e) != cudaSuccess || cudaEventElapsedTime(&ms, r.b, r.e) != cudaSuccess) {
      rc = fail(MC_ERR_CUDA, "profiling event could not be read");
    }
    mc_kernel_stat& a = acc[r.kind];
    a.launches += 1;
    a.total_ms += ms;
    a.flops += r.flops;
    a.flops_executed += r.flops_exec;
    a.flops_dense_equiv += r.flops_dense;
    a.bytes += r.bytes;
    cudaEventDestroy(r.b);
    cudaEventDestroy(r.e);
  }
  t_recs.clear();
  int k = 0;
  for (int i = 0; i < K_COUNT; ++i) {
    if (acc[i].launches == 0) continue;
    if (out && k < max_rows) {
      out[k] = acc[i];
      std::strncpy(out[k].name, kKindNames[i], sizeof(out[k].name) - 1);
    }
    ++k;
  }
  if (rows) *rows = k;
  return rc;
}

// =========================================================================
// Allocation-free S_max (mc_qk_max_logit_static).  Its Q/K scratch is this
// file-scope device array; host code must not pass the array's name to a
// kernel (on the host it is only a stand-in), so each device's address is
// looked up once with cudaGetSymbolAddress while that device is current.
static __device__ __align__(256) uint8_t g_qk_static_scratch[MC_QK_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
void* g_qk_static_addr[kMaxDevices] = {};  // guarded by g_mu

int qk_static_scratch(void** out) {
  int dev = 0;
  MC_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(MC_ERR_UNSUPPORTED, "device ordinal out of range");
  if (!g_qk_static_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_qk_static_scratch);
    if (e != cudaSuccess || !p)
      return fail(MC_ERR_CUDA, std::string("cudaGetSymbolAddress of the static scratch failed: ") +
                                   cudaGetErrorString(e));
    g_qk_static_addr[dev] = p;
  }
  *out = g_qk_static_addr[dev];
  return MC_OK;
}

template <int EPI, int WIDE>
int launch_gemm_unprofiled(const GemmParams& p, const DeviceState& st, cudaStream_t s) {
  if (p.total_tiles <= 0) return MC_OK;
  MC_CUDA((launch_pairs<EPI, WIDE>(p, st.pair_clusters, s)));
  return MC_OK;
}
}  // namespace

MC_API int mc_qk_max_logit_static(const void* x, const void* wq, const void* wk, int B, int S, int D, int H,
                                  int dh, int causal, float* smax_out, void* stream) {
  int rc = validate_qk_dims(B, S, D, H, dh);
  if (rc != MC_OK) return rc;
  if (!x || !wq || !wk || !smax_out) return fail(MC_ERR_INVAL, "NULL x, wq, wk or smax_out");
  if (!aligned16(x) || !aligned16(wq) || !aligned16(wk) || !aligned16(smax_out))
    return fail(MC_ERR_ALIGN, "pointers must be 16-byte aligned");
  const uint64_t elems = uint64_t(B) * uint64_t(S) * uint64_t(H) * uint64_t(dh);
  if (elems > MC_QK_STATIC_MAX_ELEMS)
    return fail(MC_ERR_NOSPC, "B*S*H*dh = " + std::to_string(elems) + " exceeds the static scratch limit of " +
                                  std::to_string(MC_QK_STATIC_MAX_ELEMS) + " elements; use mc_qk_max_logit");
  if (H > MC_QK_STATIC_MAX_HEADS)
    return fail(MC_ERR_NOSPC, "H = " + std::to_string(H) + " exceeds the static scratch limit of " +
                                  std::to_string(MC_QK_STATIC_MAX_HEADS) + " heads");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* st = nullptr;
  if ((rc = device_state(&st)) != MC_OK) return rc;
  void* scratch = nullptr;
  if ((rc = qk_static_scratch(&scratch)) != MC_OK) return rc;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  uint8_t* q = base;
  uint8_t* k = base + 2ull * MC_QK_STATIC_MAX_ELEMS;
  int* keys = reinterpret_cast<int*>(base + 4ull * MC_QK_STATIC_MAX_ELEMS);
  const int HD = H * dh;
  const int64_t BS = int64_t(B) * S;

  // The keys carry the previous call's maxima: reset them first.
  qk_keys_init_kernel<<<(H + 255) / 256, 256, 0, s>>>(keys, H);
  MC_CUDA(cudaGetLastError());

  GemmParams proj;
  std::memset(&proj, 0, sizeof(proj));
  proj.err = st->err_ptr;
  for (int which = 0; which < 2; ++which) {
    if ((rc = map_batched(&proj.map_a[which], x, 1, BS, D, D, HALF)) != MC_OK) return rc;
    if ((rc = map_batched(&proj.map_b[which], which == 0 ? wq : wk, 1, HD, D, D, HALF)) != MC_OK) return rc;
    GemmGroup G;
    std::memset(&G, 0, sizeof(G));
    G.M = static_cast<int>(BS);
    G.N = HD;
    G.K = D;
    G.count = 1;
    G.sched = SCHED_DENSE;
    G.layout = LAYOUT_BATCHED;
    G.heads = 1;
    G.band = 8;
    G.d = which == 0 ? q : k;
    G.d_ld = HD;
    // the projection's full 32 x 64 output blocks leave by tensor stores
    bool e_ok = false;
    if ((rc = map_epilogue(&proj.map_eo[which], &e_ok, G.d, 1, BS, HD, HD, false)) != MC_OK) return rc;
    G.tma_epi = e_ok ? 1 : 0;
    finish_group(proj, which, G, 1);
  }
  if ((rc = launch_gemm_unprofiled<EPI_STORE, 1>(proj, *st, s)) != MC_OK) return rc;

  GemmParams cm;
  std::memset(&cm, 0, sizeof(cm));
  cm.err = st->err_ptr;
  const uint64_t dims[4] = {uint64_t(dh), uint64_t(H), uint64_t(S), uint64_t(B)};
  const uint64_t strides[3] = {uint64_t(dh) * 2, uint64_t(HD) * 2, uint64_t(S) * uint64_t(HD) * 2};
  const uint32_t box_q[4] = {64, 1, HALF, 1};
  const uint32_t box_k[4] = {64, 1, HALF, 1};
  if ((rc = make_map(&cm.map_a[0], q, 4, dims, strides, box_q)) != MC_OK) return rc;
  if ((rc = make_map(&cm.map_b[0], k, 4, dims, strides, box_k)) != MC_OK) return rc;
  GemmGroup G;
  std::memset(&G, 0, sizeof(G));
  G.M = G.N = S;
  G.K = dh;
  G.count = B * H;
  G.heads = H;
  G.layout = LAYOUT_HEADS;
  G.sched = causal ? SCHED_CAUSAL : SCHED_DENSE;
  G.band = 8;
  G.mask_causal = causal ? 1 : 0;
  G.keys = keys;
  G.out_scale = 1.f / std::sqrt(static_cast<float>(dh));
  finish_group(cm, 0, G, 0);
  if ((rc = launch_causal_max(cm, *st, s, -1, 0, false)) != MC_OK) return rc;

  qk_keys_decode_kernel<<<(H + 255) / 256, 256, 0, s>>>(keys, smax_out, H);
  MC_CUDA(cudaGetLastError());
  return MC_OK;
}
