/*
 * muonclip.h -- C ABI of the B200 (sm_100a) MuonClip step library.
 *
 * The three operations of the MuonClip training step ("MuonClip: speed, then
 * stability", §07 "One complete training step"):
 *
 *   mc_muon_step     the Muon update of a list of hidden 2D weights
 *   mc_qk_max_logit  per-head causal max of the pre-softmax logit (S_max)
 *   mc_qk_clip       QK-Clip: rescale the W_q / W_k rows of heads with S_max > tau
 *
 * and their widenings:
 *
 *   mc_muon_step_host_grads  mc_muon_step with the gradient upload overlapped
 *   mc_normuon_step          the Muon update with NorMuon's per-row normalisation
 *   mc_mla_max_logit         S_max of multi-head latent attention (content + rotary)
 *   mc_qk_clip_slices        QK-Clip over an explicit slice map (MLA, fused layouts)
 *   mc_qk_max_logit_static   mc_qk_max_logit without a workspace or any allocation
 *   mc_polar_express_coeffs  host: a Polar Express coefficient table for mc_hparams
 *   mc_shard_plan            host: whole-matrix ownership for a sharded step
 *
 * Conventions for every call
 *   - All pointers named "device" are CUDA device pointers on the current
 *     device; they must be 16-byte aligned.  The library never frees or
 *     retains caller memory beyond the call (the call is asynchronous, so the
 *     buffers must stay valid until the stream reaches that point).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls
 *     enqueue work and return without waiting for the device.  A Muon-type
 *     call's parameter tables travel inside the parameters of its first
 *     launches, so no host buffer outlives the call.  The one exception: with
 *     a NULL workspace a call waits for the device to go idle when the
 *     engine-owned workspace has to grow.  mc_device_status synchronises.
 *   - CUDA graphs: a call with a workspace of its own may be captured into a
 *     graph once an earlier, uncaptured call has set the library up on the
 *     device; each replay repeats the captured call (same buffers,
 *     hyper-parameters and workspace).  mc_muon_step_host_grads, calls with a
 *     NULL workspace and calls made while profiling is on are not capturable.
 *   - Host-side state is guarded by one mutex, so calls may come from several
 *     threads.  GPU work of calls that share the engine-owned workspace (NULL
 *     workspace) or, for mc_muon_step_host_grads, the library's copy stream on
 *     one device must be ordered by the caller (one stream, or events).
 *   - Matrices are row-major and contiguous.  A weight of shape rows x cols
 *     uses the nn.Linear layout: rows = out-features.
 *   - Return value: MC_OK (0) or a negative MC_ERR_* code.  On an argument
 *     error nothing is enqueued and no memory is touched.  The text of the last
 *     error of the calling thread is available from mc_last_error().
 *   - Requires a compute capability 10.0 device (B200); otherwise
 *     MC_ERR_UNSUPPORTED.
 */
#ifndef MUONCLIP_H_
#define MUONCLIP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  MC_OK = 0,
  MC_ERR_INVAL = -1,       /* null pointer, bad shape, bad hyper-parameter */
  MC_ERR_ALIGN = -2,       /* a pointer is not 16-byte aligned */
  MC_ERR_NOSPC = -3,       /* workspace smaller than the *_workspace_size query */
  MC_ERR_CUDA = -4,        /* a CUDA runtime call failed (message in mc_last_error) */
  MC_ERR_UNSUPPORTED = -5, /* not a compute capability 10.0 device */
  MC_ERR_DEVICE = -6,      /* mc_device_status: a kernel gave up on a bounded wait */
  MC_ERR_NONFINITE = -7    /* mc_device_status: a Muon step met a NaN/Inf NS input */
};

enum { MC_F32 = 0, MC_BF16 = 1 };

/* One hidden 2D weight, its gradient and its momentum buffer. */
typedef struct {
  void* w;            /* device, rows x cols, dtype w_dtype; updated in place      */
  const void* g;      /* device, rows x cols, dtype g_dtype; read only (only
                         mc_muon_step_host_grads writes it, from host memory)    */
  float* m;           /* device, rows x cols fp32 momentum; updated in place        */
  int64_t rows;       /* >= 1 */
  int64_t cols;       /* >= 1 */
  int32_t w_dtype;    /* MC_F32 or MC_BF16 */
  int32_t g_dtype;    /* MC_F32 or MC_BF16 */
  float* update_out;  /* optional device fp32 rows x cols: receives the applied
                         update 0.2*sqrt(max(rows,cols))*NS(.) (diagnostics);
                         NULL = not written */
} mc_param;

/* Hyper-parameters of the Muon step. */
typedef struct {
  float mu;           /* momentum coefficient (0.95) */
  int32_t nesterov;   /* 1: NS input U = G + mu*M_t; 0: U = M_t */
  float lr;           /* learning rate eta */
  float wd;           /* decoupled weight decay lambda */
  int32_t ns_steps;   /* Newton-Schulz iterations, 1 <= ns_steps < 100 (5) */
  float a, b, c;      /* quintic coefficients (3.4445, -4.7750, 2.0315) */
  float eps;          /* normalisation floor: X0 = U / max(||U||_F, eps) (1e-7) */
  float rms_scale;    /* update scale factor: rms_scale*sqrt(max(rows,cols)) (0.2) */
  const float* coeffs; /* optional host array of 3*ns_steps floats: (a_k, b_k, c_k)
                          for iteration k, e.g. the classic cubic (1.5, -0.5, 0) or
                          the simple quintic (2, -1.5, 0.5) of "Muon and MuonClip:
                          orthogonalised updates for LLM training" §2, or a
                          per-step schedule; NULL = (a, b, c) in every iteration */
  const float* lr_wd; /* optional device fp32 [2]: (lr, wd) read by the kernels when
                         they run, in place of lr and wd above (which are then not
                         used), so that a step captured into a CUDA graph can follow
                         a learning-rate schedule: write the next values before each
                         replay.  Finite values are the caller's responsibility.
                         NULL = lr and wd above */
} mc_hparams;

/*
 * mc_muon_step -- one Muon step on every matrix of `params`.
 *
 * Per matrix, following "MuonClip: speed, then stability" §02-§03 and
 * "Muon and MuonClip: orthogonalised updates for LLM training" §2:
 *   M <- mu*M + G
 *   U <- G + mu*M  (nesterov) or M
 *   X0 <- U / max(||U||_F, eps), with the short side first (U^T when rows > cols)
 *   ns_steps times:  A = X X^T;  B = b*A + c*A*A;  X <- a*X + B*X
 *                    (with (a, b, c) taken from hp->coeffs per iteration if set)
 *   O <- X in the weight's orientation
 *   W <- W - lr*(rms_scale*sqrt(max(rows,cols))*O + wd*W)
 * The Newton-Schulz products run on tcgen05 tensor cores with bf16 operands
 * and fp32 accumulation.  In the first two iterations the a*X term is taken
 * from a two-part copy of the iterate (bf16 hi + bf16 lo, about 16
 * significant bits); from the third on, a*I is folded into B
 * (X <- (aI + B) X), which amplifies the bf16 rounding of X less once the
 * singular values have entered the polynomial's band.  The last iteration
 * applies the update to W straight from the fp32 accumulator.  Matrices whose
 * short side is at most 32 are no tensor-core contraction (A is at most
 * 32 x 32): they run the same iteration in fp32 on CUDA cores, streaming the
 * long side.
 * The list is processed in consecutive pieces of at most 2^29 elements (at
 * least one matrix each), all reusing one workspace; inside a piece, matrices
 * of equal shape and weight dtype are batched into one problem group.  The
 * parameter tables of every piece go to the device in one copy at the start
 * of the call.  A matrix's result does not depend on the other matrices of
 * the call.
 *
 * params/n      host array of n >= 0 entries (n == 0 is a no-op).  W, G, M of
 *               one entry must not alias; G is left unchanged.
 * hp            host pointer.
 * workspace     device scratch of at least mc_muon_workspace_size(...) bytes
 *               (what the largest piece needs, plus every piece's tables), or
 *               NULL to let the library allocate (and keep) its own.
 *               Must not be used by anything else until the step completes.
 * norms_out     optional device fp32 [n]: ||U||_F of each matrix (NULL = skip);
 *               NaN or Inf exactly when that matrix's U has a non-finite element.
 * Errors        MC_ERR_INVAL, MC_ERR_ALIGN, MC_ERR_NOSPC, MC_ERR_CUDA,
 *               MC_ERR_UNSUPPORTED.
 * Non-finite input ("MuonClip: speed, then stability" §12 lists overflow
 * events among what a run should watch): a matrix whose U holds a NaN or Inf
 * (from its gradient or momentum) gets a zero orthogonalised update, so its
 * W only decays; its momentum keeps the non-finite values (reset it before
 * the next step); its norms_out entry is not finite, and the next
 * mc_device_status returns MC_ERR_NONFINITE.  The other matrices of the call
 * are not affected.
 */
size_t mc_muon_workspace_size(const mc_param* params, int n, const mc_hparams* hp);
int mc_muon_step(const mc_param* params, int n, const mc_hparams* hp, void* workspace,
                 size_t workspace_bytes, float* norms_out, void* stream);

/*
 * mc_muon_step_host_grads -- mc_muon_step for gradients that still sit in
 * host memory.  g_host[i] (HOST, page-locked for the copies to overlap,
 * rows*cols elements of params[i].g_dtype) is copied into params[i].g
 * (device) on the library's own copy stream.  The list is split in order into
 * pieces: the first ones grow geometrically (from 1/256 of the gradient bytes,
 * x1.75 each) up to 1/chunks of the bytes, the size the rest keep (chunks = 1:
 * one piece).  The step of piece k runs on `stream` once piece k has landed,
 * so the transfer of later pieces runs under the Newton-Schulz GEMMs of
 * earlier ones and only the small first upload is exposed.  Every result is bit-for-bit that of
 * mc_muon_step (a matrix's update does not depend on the other matrices of a
 * call).  The copies start after the work already queued on `stream`, and
 * everything this call enqueues is ordered before later work on `stream`.
 * Workspace: >= mc_muon_host_grads_workspace_size(...) (the largest piece's
 * mc_muon_workspace_size), or NULL for an engine-owned buffer.
 * Errors: as mc_muon_step, plus MC_ERR_INVAL for chunks < 1 or a NULL host
 * pointer.
 */
size_t mc_muon_host_grads_workspace_size(const mc_param* params, int n, const mc_hparams* hp, int chunks);
int mc_muon_step_host_grads(const mc_param* params, const void* const* g_host, int n, const mc_hparams* hp,
                            int chunks, void* workspace, size_t workspace_bytes, float* norms_out, void* stream);

/*
 * mc_qk_max_logit -- S_max[h] = max over b, i and j (j <= i when causal) of
 * (q_{b,i,h} . k_{b,j,h}) / sqrt(dh), with Q = X W_q^T and K = X W_k^T.
 * Definition: "Muon and MuonClip: orthogonalised updates for LLM training",
 * "The exploding-logit problem"; "MuonClip: speed, then stability" §05.
 * Q and K are formed on tensor cores (bf16 in, fp32 accumulate) and stored as
 * bf16 in the workspace; the S x S score matrix is never stored.
 *
 * x             device bf16 [B][S][D]
 * wq, wk        device bf16 [H*dh][D]; head h owns rows [h*dh, (h+1)*dh)
 * causal        1: causal mask j <= i (diagonal included); 0: all pairs
 * smax_out      device fp32 [H]
 * workspace     device scratch of at least mc_qk_workspace_size(...) bytes, or NULL.
 * Constraints   B, S, D, H, dh >= 1; D and dh multiples of 8.
 */
size_t mc_qk_workspace_size(int B, int S, int D, int H, int dh);
int mc_qk_max_logit(const void* x, const void* wq, const void* wk, int B, int S, int D, int H, int dh,
                    int causal, float* smax_out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * mc_qk_clip -- QK-Clip for multi-head attention ("MuonClip: speed, then
 * stability" §05; "About Muon: Muon At Scale", "When Softmax Collapses"):
 *   gamma_h = tau / S_max[h] if S_max[h] > tau, else 1
 *   rows [h*dh, (h+1)*dh) of W_q  *= gamma_h^alpha
 *   rows [h*dh, (h+1)*dh) of W_k  *= gamma_h^(1-alpha)
 * computed on the device from `smax` (no host round trip); rows of heads that
 * are not clipped are left bit-for-bit unchanged.  The momentum buffers are
 * never touched (§07).
 *
 * wq, wk        device bf16 [H*dh][D], updated in place
 * smax          device fp32 [H] (e.g. from mc_qk_max_logit)
 * gamma_out     optional device fp32 [H] (NULL = skip)
 * mask_out      optional device int32 [H]: 1 where clipped (NULL = skip)
 */
int mc_qk_clip(void* wq, void* wk, int H, int dh, int D, const float* smax, float tau, float alpha,
               float* gamma_out, int32_t* mask_out, void* stream);

/*
 * mc_normuon -- the per-row state and constants of NorMuon ("About Muon: Muon
 * At Scale", "Certain Neurons Still Dominate").
 */
typedef struct mc_normuon {
  float beta2;       /* exponential-average factor of the row second moment, in [0, 1) */
  float eps;         /* added to sqrt(v) before dividing, finite and >= 0 */
  float* const* v;   /* HOST array of n device pointers; v[i] is fp32 [params[i].rows],
                        16-byte aligned, updated in place (start from zeros) */
} mc_normuon;

/*
 * mc_normuon_step -- the Muon step of mc_muon_step with NorMuon's per-row
 * normalisation between Newton-Schulz and the scale.  With O the un-oriented
 * NS output of a rows x cols weight:
 *   v_i   <- beta2 v_i + (1 - beta2) mean_j O_ij^2          (row = out-feature)
 *   Ohat_i = O_i / (sqrt(v_i) + eps)
 *   Ohat  <- Ohat * ||O||_F / ||Ohat||_F                     (0 if ||Ohat||_F = 0)
 *   W     <- (1 - lr wd) W - lr * rms_scale * sqrt(max(rows, cols)) * Ohat
 * update_out (if set) receives rms_scale * sqrt(max(rows, cols)) * Ohat.
 * Everything else (arguments, momentum, workspace ownership, errors) is as
 * for mc_muon_step; the workspace is larger (mc_normuon_workspace_size).
 * Errors also: MC_ERR_INVAL for a NULL nm or v, beta2 outside [0, 1), a
 * negative or non-finite eps, or a v that aliases w, g or m; MC_ERR_ALIGN.
 */
size_t mc_normuon_workspace_size(const mc_param* params, int n, const mc_hparams* hp);
int mc_normuon_step(const mc_param* params, int n, const mc_hparams* hp, const mc_normuon* nm, void* workspace,
                    size_t workspace_bytes, float* norms_out, void* stream);

/*
 * mc_clip_slice -- one block of weight rows that QK-Clip rescales with the
 * factor of one head.  Rows [row_begin, row_end) of the row-major matrix at
 * `w` (`cols` elements per row, dtype MC_BF16 or MC_F32) are multiplied by
 * gamma_head ^ exponent when head `head` clips.
 */
typedef struct mc_clip_slice {
  void* w;            /* device, 16-byte aligned base of the matrix */
  int64_t row_begin;  /* first row, >= 0 */
  int64_t row_end;    /* one past the last row, > row_begin */
  int64_t cols;       /* elements per row (the row stride), >= 1 */
  int32_t dtype;      /* MC_BF16 or MC_F32 */
  int32_t head;       /* index into smax, in [0, H) */
  float exponent;     /* in [0, 1] */
  int32_t reserved;   /* set to 0 */
} mc_clip_slice;

/*
 * mc_qk_clip_slices -- QK-Clip where the rescaled tensors are named by an
 * explicit map ("MuonClip: speed, then stability" §06, and its §12 item on
 * identifying the physical slices; "Muon and MuonClip: orthogonalised updates
 * for LLM training", "MuonClip: QK-clip, per head, adapted to MLA"):
 *   gamma_h = tau / S_max[h] if S_max[h] > tau, else 1
 *   for every slice: its rows *= gamma_head ^ exponent
 * For multi-head latent attention the map holds, per head h, the rows of the
 * head-specific content query q^C_h and content key k^C_h with exponent 1/2
 * and the rows of the head-specific rotary query q^R_h with exponent 1; the
 * rotary key that every head shares is not in the map and is never written.
 * Plain MHA is the map {W_q rows of h: alpha, W_k rows of h: 1 - alpha}.
 * Slices may live in different matrices, in one fused projection matrix
 * (e.g. per-head [content | rotary] row blocks) or in both; rows outside
 * every slice and rows of heads that do not clip are left bit-for-bit
 * unchanged.  Computed on the device from `smax`; rows are rescaled in fp32
 * and rounded to nearest-even into their dtype.
 *
 * slices     HOST array of n entries (read during the call only); no two
 *            slices may overlap in memory (MC_ERR_INVAL otherwise)
 * smax       device fp32 [H]
 * gamma_out  optional device fp32 [H] (NULL = skip)
 * mask_out   optional device int32 [H]: 1 where clipped (NULL = skip)
 * Errors: MC_ERR_INVAL (bad slice, head out of range, exponent outside
 * [0, 1], overlap, tau not finite and > 0), MC_ERR_ALIGN.
 */
int mc_qk_clip_slices(const mc_clip_slice* slices, int n, const float* smax, int H, float tau,
                      float* gamma_out, int32_t* mask_out, void* stream);

/*
 * mc_mla_max_logit -- per-head max pre-softmax logit of multi-head latent
 * attention, whose score splits into a content part with a head-specific
 * query and key and a rotary part whose key is shared by all heads
 * ("MuonClip: speed, then stability" §06):
 *   s_h(b, i, j) = (q^C_{b,i,h} . k^C_{b,j,h} + q^R_{b,i,h} . k^R_{b,j}) / sqrt(dc + dr)
 *   q^C = X W_qC^T, k^C = X W_kC^T, q^R = X W_qR^T, k^R = X W_kR^T
 *   S_max[h] = max over b, i and j <= i (all j when causal == 0)
 * Position rotation is not applied (it does not change how the clip factors
 * enter the score); pass already-rotated projections' weights if needed.
 * The score matrix is never stored: the two parts are one tensor-core
 * contraction of length dc + dr.  q^C, k^C, q^R and k^R are kept in bf16.
 *
 * x         device bf16 [B][S][D]
 * wqc, wkc  device bf16 [H*dc][D]     (head h owns rows [h*dc, (h+1)*dc))
 * wqr       device bf16 [H*dr][D]     (head h owns rows [h*dr, (h+1)*dr))
 * wkr       device bf16 [dr][D]       (shared by every head)
 * smax_out  device fp32 [H]
 * workspace device, >= mc_mla_workspace_size(...) bytes, or NULL for an
 *           engine-owned buffer
 * Requirements: D and dr multiples of 8, dc a multiple of 64.
 */
size_t mc_mla_workspace_size(int B, int S, int D, int H, int dc, int dr);
int mc_mla_max_logit(const void* x, const void* wqc, const void* wkc, const void* wqr, const void* wkr, int B,
                     int S, int D, int H, int dc, int dr, int causal, float* smax_out, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * mc_qk_max_logit_static -- the same S_max as mc_qk_max_logit, but without a
 * workspace argument and without allocating anything.  The pages have no
 * counterpart: this exists for callers that cannot call cudaMalloc, e.g. a
 * process whose device memory is entirely owned by another allocator's
 * pre-reserved pool (so a cudaMalloc would fail or fragment it), or a code
 * path that must not risk the implicit device synchronisation a cudaMalloc
 * or cudaFree may perform.
 *
 * The Q and K projections live in one file-scope device array of
 * MC_QK_STATIC_SCRATCH_BYTES (64 MiB + 16 KiB) that every GPU which loads this
 * library holds until the process exits.  Limits: B*S*H*dh <= MC_QK_STATIC_MAX_ELEMS
 * (2^24) and H <= MC_QK_STATIC_MAX_HEADS (4096); larger problems return
 * MC_ERR_NOSPC before anything is enqueued.  The first call on a device looks
 * up that device's address of the array (cudaGetSymbolAddress) and caches it,
 * so make that first call before any stream capture.  All calls share the one
 * array and it keeps the last call's contents (each call resets what must
 * start fresh), so calls that can overlap on the GPU -- on different streams,
 * or from different threads -- race and must be ordered by the caller.
 * Arguments, layouts and the other errors are as for mc_qk_max_logit.  The
 * measurement support below does not record this call's launches (it would
 * have to create CUDA events).
 */
#define MC_QK_STATIC_MAX_ELEMS (1u << 24)
#define MC_QK_STATIC_MAX_HEADS 4096
#define MC_QK_STATIC_SCRATCH_BYTES (4ull * MC_QK_STATIC_MAX_ELEMS + 4ull * MC_QK_STATIC_MAX_HEADS)
int mc_qk_max_logit_static(const void* x, const void* wq, const void* wk, int B, int S, int D, int H, int dh,
                           int causal, float* smax_out, void* stream);

/*
 * mc_polar_express_coeffs -- host-only: a per-iteration coefficient table
 * (for mc_hparams.coeffs) built the Polar Express way.  "About Muon: Muon At
 * Scale" ("Which Norm for Which Layer") cites it as a better polynomial for
 * UV^T, whose ten steps take a singular value of 1e-4 to 0.994, but does not
 * print the coefficients.  This restates the published construction (Amsel,
 * Persson, Musco and Gower, "The Polar Express", 2025):
 *   l_0 = l0, u_0 = 1; step t uses the odd quintic p_t closest to 1 in the
 *   max norm on [l_t, u_t] (found by the Remez exchange), then
 *   l_{t+1} = p_t(l_t), u_{t+1} = 2 - l_{t+1}; once u_t - l_t < 1e-3 the step
 *   is the limit 15/8 x - 5/4 x^3 + 3/8 x^5; finally every polynomial but the
 *   last is replaced by p(x / (1 + safety)).
 * With steps = 10, l0 = 1e-3 and safety = 0.01 the composed map takes 1e-4 to
 * 0.9942.
 *
 * coeffs_out  HOST float [3 * steps]: (a_t, b_t, c_t) for t = 0 .. steps-1
 * Errors: MC_ERR_INVAL (steps outside [1, 100), l0 outside (0, 1), safety
 * negative or not finite, NULL coeffs_out), MC_ERR_UNSUPPORTED if the
 * exchange does not converge.  Touches no device.
 */
int mc_polar_express_coeffs(int steps, double l0, double safety, float* coeffs_out);

/*
 * mc_shard_plan -- host-only: assign whole matrices to the ranks of an
 * ownership-sharded data-parallel step ("MuonClip: speed, then stability" §08:
 * orthogonalising a shard of a matrix is not orthogonalising the matrix, so
 * the unit of work is a whole matrix).  Each matrix costs its Newton-Schulz
 * work ns_steps * (4 m^2 n + 2 m^3), m = min(rows, cols), n = max(rows, cols).
 * Matrices are taken in decreasing cost (ties: lower index first) and each is
 * given to the rank with the least cost so far (ties: lower rank): the
 * longest-processing-time rule, whose largest load is within
 * 4/3 - 1/(3 world) of the best possible.  The result depends only on the
 * arguments, so every rank computes the same plan.
 *
 * rows, cols  HOST int64 [n], each >= 1
 * owner_out   HOST int32 [n]: rank in [0, world)
 * load_out    optional HOST double [world]: summed cost per rank
 * Errors: MC_ERR_INVAL (NULL arrays with n > 0, n < 0, world < 1,
 * ns_steps < 1, a dimension < 1).  Touches no device.
 */
int mc_shard_plan(const int64_t* rows, const int64_t* cols, int n, int ns_steps, int world, int32_t* owner_out,
                  double* load_out);

/* Text of the last error returned on the calling thread ("" if none). */
const char* mc_last_error(void);

/*
 * mc_device_status -- synchronises the current device, then reads and clears
 * the library's device error word.  Returns MC_OK; MC_ERR_DEVICE when a kernel
 * abandoned a bounded wait (its outputs are then invalid); MC_ERR_NONFINITE
 * when a Muon step since the last call met a non-finite Newton-Schulz input
 * (see mc_muon_step); or MC_ERR_CUDA.
 */
int mc_device_status(void);

/*
 * mc_selftest_bounded_wait -- test support with no counterpart on the pages:
 * launches one small kernel whose single wait (on an mbarrier that expects an
 * arrival nothing makes) runs out after limit_cycles SM cycles, the way every
 * wait in the library's kernels gives up instead of hanging.  The kernel then
 * returns normally, and the next mc_device_status returns MC_ERR_DEVICE (and
 * clears the word).  Lets a test check the timeout path and that the context
 * stays usable, without breaking a real kernel.
 * limit_cycles in [1000, 2^32]; MC_ERR_INVAL otherwise.
 */
int mc_selftest_bounded_wait(long long limit_cycles, void* stream);

/*
 * Measurement support.  Between mc_profile_begin() and mc_profile_end(), every
 * kernel this thread's calls enqueue is bracketed by two CUDA events recorded
 * on the launch stream, and its algorithmic work is computed from the shapes.
 * mc_profile_end() waits for those events and reports one row per kernel kind:
 *
 *   momentum        bytes = the momentum kernel's DRAM traffic by design:
 *                   G (2 or 4) + M read/write (8) + the iterate's two bf16
 *                   halves, hi and lo (4) bytes per element
 *   ns_gram         A = X X^T: flops = m (m+1) n (the entries on and above the
 *                   diagonal, 2n each), flops_dense_equiv = 2 m^2 n
 *   ns_poly         B = bA + cA^2: flops = m^2 (m+1), flops_dense_equiv = 2 m^3
 *   ns_apply_mixed  X <- s(aX + BX), iterations that read the iterate's hi + lo halves
 *   ns_apply        X <- (aI + B) X, later iterations
 *   ns_apply_final  last iteration fused with the weight update
 *                   (apply rows: flops = flops_dense_equiv = 2 m^2 n.  Per
 *                   iteration the dense-equivalent figures add up to the
 *                   2(2nm^2 + m^3) of "Muon and MuonClip: orthogonalised updates
 *                   for LLM training", §2.)
 *                   flops_executed = 2*256*N_tile*K_padded per tile the tensor
 *                   cores actually ran
 *   qk_proj         flops = 2 * B*S * H*dh * D * 2 (Q and K)
 *   qk_causal_max   flops = 2 * dh * (score pairs inside the causal mask)
 *   norm_finalize, qk_keys, qk_clip   (small kernels; counted, no work figure)
 *   table_upload    the launches that carry a call's parameter tables in
 *                   their parameters to device memory (bytes = the table
 *                   bytes); one launch per 32704 bytes of tables, per
 *                   mc_muon_step, mc_normuon_step or mc_muon_step_host_grads
 *
 * The rows are written to `out` (up to `max_rows`), `*rows` receives the count.
 * Recording events adds no synchronisation; the durations are device time.
 */
typedef struct {
  char name[32];
  int32_t launches;
  double total_ms;
  double flops;
  double flops_executed;
  double flops_dense_equiv;
  double bytes;
} mc_kernel_stat;

int mc_profile_begin(void);
int mc_profile_end(mc_kernel_stat* out, int max_rows, int* rows);

/*
 * mc_struct_size -- host-only: sizeof of this header's structures as the
 * library was built, for bindings that lay the structures out themselves:
 * 0 mc_param, 1 mc_hparams, 2 mc_normuon, 3 mc_clip_slice, 4 mc_kernel_stat;
 * 0 for any other index.
 */
size_t mc_struct_size(int which);

#ifdef __cplusplus
}
#endif

#endif /* MUONCLIP_H_ */
