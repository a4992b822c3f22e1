// Internal declarations shared by the library's translation units.
// Nothing here is part of the C ABI (include/am_b200.h is).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "am_b200.h"

namespace am {

constexpr int kWsHeaderBytes = 256;      // magic + head count, then status words
constexpr uint32_t kWsMagic = 0x414d4232u;  // "AMB2"
constexpr int kMaxPicksPerPass = 64;     // k·R upper bound handled per pass
constexpr int kHighestChunk = 8;         // pre-selected keys appended per refit (AM_SELECT_HIGHEST)
constexpr int kMaxBudget = 2048;         // largest t_h the per-head solvers are sized for
constexpr int kNnlsThreads = 256;
constexpr int kCholThreads = 256;

// Problem-wide constants, passed by value to every kernel.
struct Problem {
  int H, n, T, d;     // T: the largest key count of a head (the padded per-head stride)
  int ldn;            // leading dimension of per-query rows, n rounded up to 32
  int in_dtype;       // AM_BF16 / AM_FP32
  float scale;        // logit scale
  int topk, refit_every, kR;
  int nnls_max_iter;  // 0 → 3·t + 50
  float ridge, w_floor_rel;
  int max_t;          // max_h t_h
  int has_bias;
  int corr_bf16;      // the correlation pass streams a bf16 copy of Φᵀ
  int corr_recompute; // the correlation pass recomputes Φ on the tensor cores
  int corr_bounded;   // the correlation pass computes only keys its bound cannot exclude
  int select_highest; // keys chosen up front by total attention, fed to the refits kR at a time
  int64_t key_rows;   // rows of K and V (and entries of key_bias) this launch reads: Σ_h Th[h]
  long long wait_cycles;   // budget of a bounded device wait that does not drain issued work
};

constexpr long long kDefaultWaitCycles = 4000000000ll;   // ~2 s at 2 GHz

// Device pointers into the caller's workspace (see plan_workspace()).
struct Work {
  int32_t* status;      // [H]
  int32_t* t;           // [H] budgets
  int64_t* cu_t;        // [H+1] packed output offsets
  int64_t* cu_t2;       // [H+1] offsets of per-head t×t blocks
  int32_t* order;       // [H] heads sorted by pass count, descending
  int64_t* koff;        // [H+1] first input key row of each head (K, V, key_bias rows)
  int32_t* Th;          // [H] key count of each head (<= T); keys j >= Th[h] do not exist
  float* shift;         // [H]
  float* phiT;          // [H][T][ldn] key-major features Φᵀ
  __nv_bfloat16* phiT16; // [H][T][ldn] bf16 copy for the correlation pass (or null)
  double* m;            // [H][ldn] mass: fp64 sum of the stored fp32 features
  float* Y;             // [H][n][d]
  float* r;             // [H][ldn] residual (fp32 copy read by the correlation pass)
  float* corr;          // [H][T]
  double* inv_m;        // [H][ldn] 1 / m_i (0 for a query without mass), highest-attention scores
  uint8_t* sel;         // [H][T] selected flags
  int32_t* picks;       // [Σt] pick order
  float* pick_corr;     // [Σt]
  double* G;            // [Σt²] Gram of the picks (pick-order indexing)
  double* bvec;         // [Σt] Φ_Sᵀ m
  double* w;            // [Σt] NNLS weights (pick order)
  double* L;            // [Σt²] Cholesky factor scratch (global fallback)
  int32_t* plist;       // [Σt] NNLS passive list (factor order)
  int32_t* np;          // [H] passive count
  int32_t* ylen;        // [H] leading length of ycache that is valid
  double* mm;           // [H] ‖m‖²
  double* rr_part;      // [H][kRedBlocks] partial ‖r‖²
  int32_t* sorted_slot; // [Σt] pick slot of each ascending-position output row
  double* w_eff;        // [Σt] floored weights, ascending-position order
  double* ycache;       // [Σt] forward solve L⁻¹ b_P (factor order), kept across refits
  float* A;             // [Σt][ldn] design matrix, key-major (CUDA-core normal equations)
  __nv_bfloat16* Apl;   // [3][Σt][ldn] the design matrix as bf16 planes hi, mid, lo (tensor-core path)
  __nv_bfloat16* Ypl;   // [3][H][n][d] the targets Y as bf16 planes hi, mid, lo (tensor-core path)
  double* AtA;          // [Σt²]
  double* AtY;          // [Σt][d]
  double* nrm_part;     // [kNormalMaxSplits][Σt² + Σt·d] split partials of AᵀA, AᵀY
  // bounded correlation pass
  double* cnorm;        // [H][T] ‖Φ_{:,j}‖₂ (fp64, an upper bound within 1e-6 when from cnpart)
  float* cnpart;        // [H][⌈n/128⌉][4][T] per-warp partial Σ_i Φ_ij² from the feature pass, or null
  double* rnorm;        // [H] ‖r‖₂ of the stored fp32 residual, this pass
  uint64_t* clist;      // [H][T] this pass's evaluated keys: order keys of their exact c_j
  int32_t* clj;         // [H][T] and the key indices, in completion order
  int32_t* ccount;      // [H] entries in that list
  float* gb;            // [H][T] this pass's group bound b_j of every key (−1: selected or past T_h)
  int32_t* ghist;       // [H][1024] histogram of the positive bounds (cleared after each use)
  float* gtau;          // [H] this pass's probe threshold τ
  int32_t* gcnt;        // [H] group-bound blocks finished this pass
  int32_t* cdone;       // [H] 1 when the probe step already made this pass's picks
  float* cnblk;         // [H][64][T] per residual query group g, an upper bound of ‖Φ_{i∈g, j}‖₂
                        // (group g: queries i with (i / 128) mod resid_blocks == g)
  double* ctheta;       // [H] this pass's threshold θ, the kk-th largest value the probe found
  unsigned long long* rows_eval;   // [H] keys evaluated, summed over the passes
  int32_t* nnls_refits;            // [H] NNLS refits of the call
  int32_t* nnls_solves;            // [H] inner solves of those refits
  double* gpart;        // [kGramMaxSlices·(Σt + H)·kR] Gram partial sums per query slice
  int32_t* gcount;      // [Σt + H] Gram blocks finished this pass, per head and row group
  int32_t* rcount;      // [H] bounded-correlation row blocks finished this launch
  double* dinv;         // per head at 32·(cu_t[h] + 32h): inverses of the value-fit factor's 32×32 diagonal tiles
  double* vinv;         // per head at 64·(cu_t[h] + 64h): inverses of the 64×64 diagonal tiles (tiled solve)
  double* ndinv;        // per head at 64·(cu_t[h] + 32h): the NNLS factor's diagonal-tile inverses and their transposes
  int32_t* dvalid;      // [H] leading row blocks of the NNLS factor whose cached inverse is valid
  int64_t nrm_ata;      // Σt²
  int64_t nrm_stride;   // Σt² + Σt·d
  int64_t sum_t;        // Σt
};

constexpr int kRedBlocks = 64;   // partial-sum slots per head for ‖r‖²
constexpr int kResidPos = 32;    // float4 query positions per residual block

// Blocks per head of the residual update, each leaving one partial ‖r‖².
inline __host__ __device__ int resid_blocks(const Problem& p) {
  const int b = (p.ldn / 4 + kResidPos - 1) / kResidPos;
  return b < kRedBlocks ? b : kRedBlocks;
}
constexpr int kSortSmemKeys = 16384;  // key counts the highest-attention sort handles in shared memory
constexpr int kGramMaxSlices = 32;    // query slices of the tiled Gram update
constexpr int kGramMaxNew = 16;       // picks per pass the tiled Gram update takes
constexpr int kNormalMaxSplits = 8;   // query splits of the normal-equation products
constexpr int kQuerySplit = 2048;     // queries one tensor-core normal-equation CTA sums in fp32

// ---- launchers (each file defines its own) ----
// feature pass (am_phi_simt.cu)
cudaError_t launch_shift_max(const Problem& p, const Work& w, const void* Q, const void* K, const float* key_bias,
                             float* shift, cudaStream_t s);
cudaError_t launch_phi(const Problem& p, const void* Q, const void* K, const float* key_bias,
                       const Work& w, cudaStream_t s);
cudaError_t launch_y_m(const Problem& p, const void* V, const Work& w, cudaStream_t s);
cudaError_t launch_shift_copy(const float* src, float* dst, int H, cudaStream_t s);
cudaError_t launch_shift_init(float* shift, int H, cudaStream_t s);
cudaError_t launch_shift_decode(float* shift, int H, cudaStream_t s);
// tensor-core feature pass (am_phi_tc.cu): bf16 inputs, d in {64, 128}
bool phi_tc_supported(const Problem& p);
cudaError_t launch_shift_max_tc(const Problem& p, const void* Q, const void* K, const float* key_bias,
                                const Work& w, uint32_t* shift_ord, cudaStream_t s);
cudaError_t launch_phi_tc(const Problem& p, const void* Q, const void* K, const void* V, const float* key_bias,
                          const Work& w, cudaStream_t s);
cudaError_t launch_corr_tc(const Problem& p, const void* Q, const void* K, const float* key_bias, const Work& w,
                           int pass, int active, cudaStream_t s);
// OMP engine (am_omp.cu)
cudaError_t launch_omp_init(const Problem& p, const Work& w, cudaStream_t s);
// inputs the recomputing correlation pass needs
struct CorrInputs {
  const void* Q;
  const void* K;
  const float* key_bias;
};
// big_heads: how many of the first active heads of w.order keep their NNLS
// factor in the workspace (budget above nnls_smem_cap(max_t)); small_tmax:
// the largest budget among the other active heads
cudaError_t launch_omp_pass(const Problem& p, const Work& w, int pass, int active_heads, int big_heads,
                            int small_tmax, const CorrInputs& in, cudaStream_t s);
int nnls_smem_cap(int max_t);
// bounded correlation pass (am_bounded.cu): column norms once, then per pass
// probe, exact rows, extension, exact rows, selection
cudaError_t launch_column_norms(const Problem& p, const Work& w, cudaStream_t s);
cudaError_t launch_corr_bounded(const Problem& p, const Work& w, int pass, int active, cudaStream_t s);
// highest-attention selection: scores, then each head's t best keys as its picks (am_bounded.cu)
cudaError_t launch_select_highest(const Problem& p, const Work& w, cudaStream_t s);
cudaError_t launch_residual_norm(const Problem& p, const Work& w, double* residual_out,
                                 cudaStream_t s);
// value fit and packing (am_valfit.cu)
cudaError_t launch_finalize(const Problem& p, const Work& w, const void* K, const float* key_bias,
                            void* C_k, float* beta, int32_t* indices, float* w_out,
                            int32_t* pick_order, float* pick_corr, cudaStream_t s);
cudaError_t launch_value_fit(const Problem& p, const Work& w, float* C_v, cudaStream_t s);
cudaError_t launch_normal_reduce(const Work& w, int splits, cudaStream_t s);
// the value-fit solve for large budgets, tiled over many CTAs (am_valsolve.cu)
cudaError_t launch_value_solve_tiled(const Problem& p, const Work& w, float* C_v, cudaStream_t s);
constexpr int kTiledSolveMinT = 97;   // budgets from which a call uses the tiled solve
// tensor-core normal equations (am_normal_tc.cu): bf16 inputs, d in {64, 128}
bool normal_tc_supported(const Problem& p);
cudaError_t launch_normal_tc(const Problem& p, const Work& w, cudaStream_t s);

// The body of am_compact_heads; OMP passes of up to max_groups head groups run
// concurrently on internal streams (1: everything on the caller's stream).
am_status_t compact_heads_impl(const void* Q, const void* K, const void* V, int32_t n, int32_t T, int32_t d,
                               int32_t H, const int32_t* budgets, const am_opts_t* opts, void* workspace,
                               size_t workspace_bytes, const int64_t* out_offsets, void* C_k, float* beta,
                               float* C_v, int32_t* indices, void* stream, int max_groups);

// ---- small device helpers ----
__host__ __device__ inline int round_up(int x, int a) { return (x + a - 1) / a * a; }

__device__ __forceinline__ float load_in(const void* base, int64_t idx, int dtype) {
  if (dtype == AM_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  return reinterpret_cast<const float*>(base)[idx];
}

// Severity of a device condition: a head keeps the most severe one it met.
// A timeout leaves the head's work unfinished; non-finite values are the
// cause of whatever else failed downstream (a value-fit matrix that is not
// positive definite, an iteration cap); warnings rank below every error.
__device__ __forceinline__ int severity(int code) {
  switch (code) {
    case AM_WARN_NOT_CONVERGED: return 1;
    case AM_WARN_MASS_UNDERFLOW: return 2;
    case AM_ERR_NOT_SPD: return 3;
    case AM_ERR_NONFINITE: return 4;
    default: return 5;   // AM_ERR_TIMEOUT
  }
}

// Status words hold 1000·severity + code (0 for none), so the largest word is
// the most severe condition and word % 1000 its code.
__device__ __forceinline__ void record_status(int32_t* status, int code) {
  atomicMax(status, 1000 * severity(code) + code);
}

// Number of OMP passes for budget t: one correlation pass per refit interval.
__host__ __device__ inline int num_passes(int t, int kR) { return (t + kR - 1) / kR; }

// Pick slots [s0, s1) that pass `pass` appends for a head of budget t.
__device__ __forceinline__ void pass_range(const Problem& p, int t, int pass, int& s0, int& s1) {
  s0 = min(pass * p.kR, t);
  s1 = min(s0 + p.kR, t);
}

// ---- programmatic dependent launch (the per-pass kernel chain) ----
// A kernel launched with launch_chained may start while its stream
// predecessor drains: it must call chain_wait() before touching anything,
// which returns once the predecessor grid has completed and its writes are
// visible (a no-op for an ordinary launch).  chain_release() lets the next
// chained kernel begin launching; a kernel calls it once its block is past
// the main parallel work.
__device__ __forceinline__ void chain_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void chain_release() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace am
