/*
 * am_b200.h — C ABI of the B200 (sm_100a) Attention-Matching KV compaction
 * library (AM-OMP).
 *
 * The operation ("Fast KV Compaction via Attention Matching"):
 *   zhichai.net deep dive §1.3-§1.6 — attention mass, the per-token scalar
 *     bias β, the mass-feature matrix Φ_ij = exp(q_i·k_j), target mass
 *     m = Φ·1, greedy OMP key selection with an NNLS refit after each pick,
 *     and β = log w;
 *   xinfinite.net article §2 (steps 2 and 3, Fig. 1 and Fig. 2) — NNLS bias
 *     fit (projected gradient on the GPU in the authors' version), value fit
 *     by ordinary least squares; §3 and Table 1 — top-k batched selection
 *     with lazy refit ("OMP-fast");
 *   zhichai.net/en summary, "The Three-Step Closed-Form Pipeline" and
 *     "Engineering Practicality" (varlen per-head packing).
 *
 * For every head h independently, with s_ij = (q_i·k_j)·scale + b_j:
 *   Φ_ij = exp(s_ij − c_h),  m_i = Σ_j Φ_ij,
 *   S  = t_h keys chosen greedily: each round appends the kk = min(k, t−|S|)
 *        unselected keys with the largest c_j = Σ_i r_i Φ_ij (ties → lowest
 *        index); on every R-th round and the last, w = NNLS(Φ_S, m) and
 *        r = m − Φ_S w,
 *   β_l = b_{S_l} + log max(w_l, w_floor_rel·max w),
 *   Y_i = Σ_j Φ_ij V_j / m_i,  A_il = softmax_l(Q C_kᵀ·scale + β)_i,
 *   C_v = (AᵀA + λI)⁻¹ AᵀY with λ = ridge·tr(AᵀA)/t_h.
 *
 * Status codes 8 and 10 are warnings (the results are valid as described);
 * the others above 0 are errors.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers unless marked "host".
 *   - The caller owns every buffer; nothing is allocated inside a call.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream); the call returns before it finishes.
 *   - Argument errors are returned synchronously and nothing is enqueued.
 *     Device-side per-head conditions (NNLS iteration limit, a Cholesky
 *     pivot that is not positive, non-finite features) are written to status
 *     words inside the workspace; read them with am_get_status().
 *   - No entry point calls exit(), throws, or falls back to the CPU.
 */
#ifndef AM_B200_H
#define AM_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum am_status {
  AM_OK = 0,
  AM_ERR_INVALID_ARG = 1,     /* null pointer, bad size or option          */
  AM_ERR_BUDGET = 2,          /* a budget outside [1, T]                   */
  AM_ERR_WORKSPACE = 3,       /* workspace missing, misaligned or too small */
  AM_ERR_NONFINITE = 4,       /* (device) a non-finite feature or solution  */
  AM_ERR_CUDA = 5,            /* a CUDA runtime call failed                 */
  AM_ERR_TIMEOUT = 6,         /* (device) a bounded wait ran out            */
  AM_ERR_UNSUPPORTED = 7,     /* shape or dtype this build does not handle  */
  AM_WARN_NOT_CONVERGED = 8,  /* (device) NNLS stopped at its iteration cap */
  AM_ERR_NOT_SPD = 9,         /* (device) value-fit matrix not positive definite */
  AM_WARN_MASS_UNDERFLOW = 10 /* (device) every fp32 feature of some reference
                                 query underflowed to 0 (its best logit lies more
                                 than ~87 below the head's shift): that query has
                                 no mass, and it drops out of the NNLS and the
                                 value fit (zero target, zero design row) */
} am_status_t;

typedef enum am_dtype { AM_BF16 = 0, AM_FP32 = 1 } am_dtype_t;

/* Where the correlation pass c = Φᵀ r reads the features from.  The mass,
 * Gram, residual and value fit always use the stored fp32 Φ. */
typedef enum am_corr_mode {
  AM_CORR_AUTO = 0,         /* BOUNDED                                           */
  AM_CORR_STORED_FP32 = 1,  /* stream the stored fp32 Φᵀ (4 bytes per feature)    */
  AM_CORR_STORED_BF16 = 2,  /* stream a bf16 copy of Φᵀ written by the feature
                               pass (2 bytes per feature; picks may differ from
                               exact arithmetic where correlations are closer
                               than bf16 rounding)                                 */
  AM_CORR_RECOMPUTE = 3,    /* recompute Φ from Q and K on the tensor cores in
                               every pass (no feature reads; bf16 inputs only)     */
  AM_CORR_BOUNDED = 4       /* exact fp64 correlations, from the stored fp32 Φᵀ,
                               for only the keys that can reach the pass's top
                               k·R: |c_j| <= ‖r‖·‖Φ_{:,j}‖ (Cauchy-Schwarz) rules
                               out every other key once k·R computed values exceed
                               its bound; the picks are those of a full pass      */
} am_corr_mode_t;

/* How the t keys of each head are chosen.  Either way β is fit by NNLS on
 * the chosen keys and C_v by the ridge least-squares fit.
 *   AM_SELECT_OMP      greedy Orthogonal Matching Pursuit on the attention
 *                      mass ("Fast KV Compaction via Attention Matching":
 *                      zhichai.net deep dive §1.6; top-k batching with lazy
 *                      refit, xinfinite.net article §3)
 *   AM_SELECT_HIGHEST  the t keys with the largest total attention over the
 *                      reference queries, score_j = Σ_i Φ_ij / m_i (each
 *                      query's softmax probability of key j), ties to the
 *                      lower key (AM-Highest: zhichai.net/en summary, "Method
 *                      Family and Trade-offs"; the youleyou.com rewrite's
 *                      highest-attention keys).  topk, refit_every and
 *                      corr_mode are ignored; requires T <= 16384. */
typedef enum am_select_mode { AM_SELECT_OMP = 0, AM_SELECT_HIGHEST = 1 } am_select_mode_t;

/* Options.  Fill with am_default_opts() and override fields. */
typedef struct am_opts {
  int32_t in_dtype;        /* am_dtype_t of Q_ref, K, V and of the C_k output   */
  int32_t topk;            /* k: keys appended per OMP round (1 = plain OMP)     */
  int32_t refit_every;     /* R: rounds between NNLS refits (1 = every round)    */
  int32_t nnls_max_iter;   /* active-set iteration cap per refit (0 = 3·t + 50)  */
  float scale;             /* logit scale; <= 0 selects 1/sqrt(d)                */
  float ridge;             /* λ = ridge·tr(AᵀA)/t (default 1e-6); must be >= 0   */
  float w_floor_rel;       /* β floor: w >= w_floor_rel·max(w) (default 1e-12)   */
  int32_t corr_mode;       /* am_corr_mode_t: how the correlation pass gets Φ      */
  /* Optional device inputs */
  const float* shift;      /* [H] per-head shift c_h, or NULL: c_h = max_ij s_ij
                              computed on the device                              */
  const float* key_bias;   /* [H][T] prior per-key bias b (an already compacted
                              block's β), or NULL for b = 0                       */
  /* Optional device outputs (NULL = not written) */
  int32_t* pick_order;     /* [Σt] keys in greedy pick order, packed like indices */
  float* pick_corr;        /* [Σt] correlation c_j of each pick when it was made
                              (AM_SELECT_HIGHEST: its score)                     */
  float* shift_out;        /* [H] shift used                                     */
  double* residual_out;    /* [H] ‖m − Φ_S w‖ / ‖m‖ after the last refit          */
  float* w_out;            /* [Σt] NNLS weights, aligned with indices            */
  int32_t select_mode;     /* am_select_mode_t (default AM_SELECT_OMP)           */
  int32_t reserved0;       /* must be 0                                          */
  /* Optional HOST input: variable key counts per head (KV-based chunking of a
   * long context, "Fast KV Compaction via Attention Matching": xinfinite.net
   * article §3, where each chunk is compacted independently and the last
   * chunk is shorter; per-head varlen segments, zhichai.net deep dive §4.2).
   * NULL: every head has T keys, K/V are [H][T][d] and key_bias [H][T].
   * Otherwise int64 [H+1], key_offsets[0] = 0, T_h = key_offsets[h+1] −
   * key_offsets[h] >= 1, and max_h T_h must equal the T argument: K and V
   * are packed [Σ T_h][d] (head h's keys are rows key_offsets[h] ..
   * key_offsets[h+1] − 1), key_bias is packed [Σ T_h], and each budget
   * satisfies 1 <= t_h <= T_h.  Read during the call only. */
  const int64_t* key_offsets;
  /* Clock-cycle budget of each bounded device wait on an asynchronous copy
   * or tensor-core step (0: 4e9 cycles, about 2 s).  A wait that runs out
   * records AM_ERR_TIMEOUT for its head; the kernel then stops issuing
   * work, waits (with the full budget) for what it already issued, releases
   * its tensor memory and returns, so the context stays usable.  >= 0. */
  int64_t wait_cycles;
} am_opts_t;

/* Fill *opts with defaults: bf16 inputs, k = 1, R = 1, scale = 1/sqrt(d),
 * ridge = 1e-6, w_floor_rel = 1e-12, corr_mode = AM_CORR_AUTO, every
 * optional pointer NULL (key_offsets NULL: T keys per head),
 * select_mode = AM_SELECT_OMP. */
am_status_t am_default_opts(am_opts_t* opts);

/* Device workspace needed by am_compact_heads for this problem.
 *   n, T, d          reference queries, keys per head, head dim (d in {64, 128}
 *                    for bf16 inputs; any d in [1, 256] for fp32 inputs)
 *   num_heads        H
 *   budgets          host int32 [H], 1 <= t_h <= T, and t_h <= 2048
 *                    (larger budgets return AM_ERR_UNSUPPORTED)
 *   opts             as passed to am_compact_heads
 *   bytes            host out
 * The dominant term is H·T·round_up(n, 32)·4 bytes of stored features
 * (·6 with AM_CORR_STORED_BF16). */
am_status_t am_workspace_size(int32_t n, int32_t T, int32_t d, int32_t num_heads,
                              const int32_t* budgets, const am_opts_t* opts,
                              size_t* bytes);

/* Workspace with which am_compact_heads processes the heads in waves of at
 * most `wave_heads` consecutive heads (head order), one wave after the other
 * through the same memory.  Problems whose stored features do not fit in
 * HBM at once (2048 chunk-heads of 8192 keys × 8192 queries hold 512 GiB of
 * fp32 Φᵀ) run this way.  wave_heads >= 1; values >= num_heads give
 * am_workspace_size().  Same argument rules otherwise. */
am_status_t am_workspace_size_waves(int32_t n, int32_t T, int32_t d, int32_t num_heads,
                                    const int32_t* budgets, const am_opts_t* opts,
                                    int32_t wave_heads, size_t* bytes);

/* Compact H independent heads.
 *   Q_ref   [H][n][d], K [H][T][d], V [H][T][d], row-major, dtype opts->in_dtype
 *           (K, V packed [Σ T_h][d] when opts->key_offsets is set)
 *   budgets host int32 [H]
 *   out_offsets host int64 [H+1]: out_offsets[0] = 0,
 *           out_offsets[h+1] = out_offsets[h] + budgets[h] (checked)
 *   workspace   device, 256-byte aligned.  With >= am_workspace_size() bytes
 *               all heads run in one wave; with less, the call runs the heads
 *               in waves of consecutive heads, each as many as the workspace
 *               holds (am_workspace_size_waves() gives the size for a chosen
 *               wave size).  AM_ERR_WORKSPACE if one head does not fit.
 *   Outputs, packed per head at out_offsets[h] (the varlen layout), rows in
 *   ascending original key position:
 *     C_k      [Σt][d]  dtype opts->in_dtype (exact copies of the chosen keys)
 *     beta     [Σt]     fp32
 *     C_v      [Σt][d]  fp32
 *     indices  [Σt]     int32, position of each kept key within its head
 *   stream  cudaStream_t as void*
 * Inputs must not alias outputs or the workspace.  The workspace must not be
 * shared by two calls in flight at once. */
am_status_t am_compact_heads(const void* Q_ref, const void* K, const void* V,
                             int32_t n, int32_t T, int32_t d, int32_t num_heads,
                             const int32_t* budgets, const am_opts_t* opts,
                             void* workspace, size_t workspace_bytes,
                             const int64_t* out_offsets,
                             void* C_k, float* beta, float* C_v, int32_t* indices,
                             void* stream);

/* Where am_compact_heads leaves its intermediate features inside the
 * caller's workspace (byte offsets from the workspace base), valid once a
 * call that ran all heads in one wave (workspace >= am_workspace_size())
 * has completed, and until the workspace is reused:
 *   phiT    fp32 [H][T][ldn]  Φᵀ_ji = exp(s_ij − c_h), key-major, rows padded
 *                             with zeros from n to ldn (with key_offsets:
 *                             rows T_h .. T−1 of head h are not written)
 *   mass    fp64 [H][ldn]     m_i = Σ_j Φ_ij (exact sum of the stored fp32 Φ)
 *   target  fp32 [H][n][d]    Y_i = Σ_j Φ_ij V_j / m_i
 *   shift   fp32 [H]          c_h used
 *   ldn     n rounded up to a multiple of 32
 *   weights fp64 [Σt]         the last NNLS refit's w, packed per head at
 *                             out_offsets[h] in PICK order (zero where w_l = 0)
 *   resid   fp32 [H][ldn]     r = m − Φ_S w after the last refit
 *   rows_evaluated            see the field below
 * rows_evaluated, nnls_refits and nnls_solves are per-head call statistics
 * kept in the workspace's prefix: valid after any completed call, whether or
 * not it ran in one wave.
 * Same argument rules as am_workspace_size. */
typedef struct am_workspace_view {
  size_t phiT, mass, target, shift;
  int32_t ldn;
  int32_t reserved;
  size_t weights, resid;
  size_t rows_evaluated;   /* int64 [H]: keys whose correlation the bounded
                              passes evaluated, summed over the call's passes */
  size_t column_norms;     /* fp64 [H][T]: the bounded pass's ‖Φ_{:,j}‖₂, an upper
                              bound within a relative 2e-6 of the exact norm
                              (AM_SELECT_HIGHEST: each key's total-attention
                              score Σ_i Φ_ij / m_i instead) */
  size_t nnls_refits;      /* int32 [H]: NNLS refits of the call (one per pass) */
  size_t nnls_solves;      /* int32 [H]: inner least-squares solves of those
                              refits (each at most nnls_max_iter per refit) */
} am_workspace_view_t;

am_status_t am_workspace_view(int32_t n, int32_t T, int32_t d, int32_t num_heads,
                              const int32_t* budgets, const am_opts_t* opts,
                              am_workspace_view_t* view);

/* Size of the fixed device scratch area behind am_compact_heads_noalloc. */
#define AM_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* am_compact_heads without any device allocation (the paper has no
 * counterpart; this is a library convenience).
 *
 * For callers that cannot call cudaMalloc: code running inside a runtime
 * that owns every device allocation through its own pool and forbids
 * others, code on a latency-critical path where an allocation would
 * synchronise the device, or plugins handed only input and output buffers.
 * The scratch memory this call needs lives in one file-scope device array of
 * AM_NOALLOC_SCRATCH_BYTES (16 MiB) inside this library; every GPU that loads
 * the library keeps that array until the process exits.
 *
 *   Arguments as for am_compact_heads, without workspace and size.
 *   status_out  optional device int32 [H]: per-head status codes as
 *               am_get_status reports them (AM_OK, AM_WARN_NOT_CONVERGED, ...),
 *               written on `stream` when the call completes; NULL to skip.
 * Returns AM_ERR_WORKSPACE, before touching the GPU, when the problem's
 * workspace (am_workspace_size) exceeds AM_NOALLOC_SCRATCH_BYTES.
 *
 * The first call on a device looks up the array's device address with the
 * CUDA runtime.  Every call also copies a small header and the per-head
 * tables from pageable host memory with cudaMemcpyAsync, so the call cannot
 * be recorded into a CUDA graph: make every call outside stream capture.
 * All calls share the one array and leave their contents in it: calls whose
 * work overlaps on the GPU (on different streams, or from different threads)
 * race on it and must be serialised by the caller.  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.  It
 * creates no stream or event, except that while stage timing is switched on
 * (am_profile_enable) each launch is bracketed by CUDA events as described
 * there. */
am_status_t am_compact_heads_noalloc(const void* Q_ref, const void* K, const void* V,
                                     int32_t n, int32_t T, int32_t d, int32_t num_heads,
                                     const int32_t* budgets, const am_opts_t* opts,
                                     const int64_t* out_offsets,
                                     void* C_k, float* beta, float* C_v, int32_t* indices,
                                     int32_t* status_out, void* stream);

/* Attention that consumes a compacted cache: for head h and query i,
 *   out[h][i] = Σ_j softmax_j(q_i·k_j·scale + b_j) v_j
 * over head h's compacted segment (k = C_k, v = C_v, b = β, rows cu_t[h] ..
 * cu_t[h+1] of the packed outputs of am_compact_heads) followed by T_new
 * fresh keys (k = K_new, v = V_new, b = 0).  The compacted block stands in
 * for the keys it replaced through its additive per-key bias, and the
 * result equals the mass-weighted mixture of the two blocks' local outputs
 * (the attention mixing identity: "Fast KV Compaction via Attention
 * Matching", zhichai.net deep dive §4.1-4.2 on bias-capable attention
 * kernels and varlen per-head segments; zhichai.net/en summary,
 * "Engineering Practicality").
 *   Q            device [H][nq][d], dtype in_dtype
 *   C_k          device [Σt][d], dtype in_dtype; beta device [Σt] fp32;
 *   C_v          device [Σt][d] fp32 (as am_compact_heads writes them)
 *   cu_t         device int64 [H+1], the segment offsets
 *   K_new, V_new device [H][T_new][d], dtype in_dtype (NULL when T_new = 0)
 *   scale        logit scale; <= 0 selects 1/sqrt(d)
 *   out          device [H][nq][d] fp32
 * fp32 arithmetic with an online softmax; 1 <= d <= 256, num_heads <= 65535.
 * Asynchronous on stream; argument errors return synchronously. */
am_status_t am_attend_packed(const void* Q, int32_t nq, int32_t d, int32_t num_heads, int32_t in_dtype,
                             const void* C_k, const float* beta, const float* C_v, const int64_t* cu_t,
                             const void* K_new, const void* V_new, int32_t T_new, float scale,
                             float* out, void* stream);

/* Non-uniform per-head budgets from sensitivity curves by greedy swaps
 * ("Fast KV Compaction via Attention Matching": zhichai.net/en summary,
 * "Engineering Practicality"; zhichai.net deep dive §4.2).  Host-only: no
 * GPU work, every pointer is a host pointer.
 *   loss        [num_heads][levels]: head h's loss at budget t_min + g·quantum
 *   total       Σ budgets; total − num_heads·t_min must be a multiple of
 *               quantum and at most num_heads·(levels − 1)·quantum
 *               (otherwise AM_ERR_BUDGET)
 *   max_swaps   cap on swaps, < 0 for none
 *   budgets_out [num_heads]; swaps_out (optional) the swaps made
 * The levels start as even as the total allows (the first heads take the
 * remainder); each swap moves one quantum to the head whose loss falls most
 * from the head, other than that one, whose loss rises least, ties to the
 * lower head, while the fall exceeds the rise.  Non-finite losses return
 * AM_ERR_NONFINITE. */
am_status_t am_assign_budgets(const double* loss, int32_t num_heads, int32_t levels, int32_t t_min,
                              int32_t quantum, int64_t total, int32_t max_swaps,
                              int32_t* budgets_out, int32_t* swaps_out);

/* Synchronise `stream`, then copy the per-head device status words of the last
 * call that used `workspace` into host per_head[H] (may be NULL) and return the
 * most severe one (AM_OK if all heads succeeded). */
am_status_t am_get_status(const void* workspace, int32_t num_heads,
                          int32_t* per_head, void* stream);

/* Stage timing.  While enabled, every kernel launch made by
 * am_compact_heads (and am_compact_heads_noalloc) is bracketed by CUDA events
 * that the library creates and records on the launch's stream (event
 * creation is the only host-side cost; no device memory is used).
 * am_profile_collect() waits for the recorded events, adds up the device time
 * and the launch count per stage into ms[AM_STAGE_COUNT] and
 * launches[AM_STAGE_COUNT] (host arrays, either may be NULL), and clears the
 * record.  Process-wide; not meant for concurrent calls from several threads. */
typedef enum am_stage {
  AM_STAGE_SHIFT = 0,    /* c_h = max logit                         */
  AM_STAGE_PHI = 1,      /* Φᵀ = exp(s − c_h)                        */
  AM_STAGE_TARGET = 2,   /* Y = ΦV/m and m                           */
  AM_STAGE_INIT = 3,     /* ‖m‖², selection flags                    */
  AM_STAGE_CORR = 4,     /* c = Φᵀ r (full-pass modes)                */
  AM_STAGE_SELECT = 5,   /* top-k·R unselected keys                  */
  AM_STAGE_GRAM = 6,     /* Φ_SᵀΦ_S, Φ_Sᵀm updates                   */
  AM_STAGE_NNLS = 7,     /* active-set NNLS refit                    */
  AM_STAGE_RESID = 8,    /* r = m − Φ_S w                            */
  AM_STAGE_FINALIZE = 9, /* sort, β, C_k, indices                    */
  AM_STAGE_DESIGN = 10,  /* A = rownorm(Φ_S diag w)                  */
  AM_STAGE_NORMAL = 11,  /* AᵀA, AᵀY                                 */
  AM_STAGE_SOLVE = 12,   /* ridge Cholesky, C_v                      */
  AM_STAGE_NORMS = 13,   /* bounded mode: column and group norms   */
  AM_STAGE_ROWS = 14,    /* bounded mode: exact c_j of listed keys,
                            threshold and picks                      */
  AM_STAGE_ATTEND = 15,  /* am_attend_packed                         */
  AM_STAGE_COUNT = 16
} am_stage_t;

am_status_t am_profile_enable(int32_t on);
am_status_t am_profile_collect(double* ms, int64_t* launches);

/* Total number of kernels this library has launched in the process. */
int64_t am_kernel_launches(void);

/* Static description of a status code. */
const char* am_status_string(am_status_t status);

/* Library version, major·10000 + minor·100 + patch. */
int32_t am_version(void);

#ifdef __cplusplus
}
#endif
#endif /* AM_B200_H */
