// Ridge value-fit solve for large budgets, batched over heads and spread
// over many CTAs: C_v = (AᵀA + λI)⁻¹ AᵀY with λ = ridge·tr(AᵀA)/t
// ("Fast KV Compaction via Attention Matching": with C_k and β fixed, C_v is
// the least-squares fit of the original attention outputs, xinfinite.net
// article §2 step 3; the youleyou.com rewrite, the OLS step).
//
// A right-looking blocked Cholesky on 64 × 64 tiles, in fp64, in place on
// each head's AᵀA (row-major t × t in the workspace), then blocked forward
// and backward solves on AᵀY (row-major t × d).  Every step is one launch
// over all heads' tiles at once, so a head with a budget near 1000 keeps the
// whole GPU busy instead of one SM:
//   k_vs_ridge          λ on the diagonal (one CTA per head)
//   k_vs_diag(kb)       factor diagonal tile kb in shared memory, store its
//                       inverse (one CTA per head)
//   k_vs_panel(kb)      L_ik = M_ik L_kk⁻ᵀ for the tiles below it
//   k_vs_update(kb)     M_ij −= L_ik L_jkᵀ for the trailing tile pairs
//   k_vs_fwd(kb) / k_vs_bwd(kb)   X_kb ← L_kk⁻¹ X_kb (L_kk⁻ᵀ X_kb), then the
//                       other row tiles take X_kb's contribution
//   k_vs_out            C_v = X in fp32
// A pivot that is not positive marks the head AM_ERR_NOT_SPD; its later
// steps are skipped and its C_v is zero.
#include "am_internal.cuh"
#include "am_profile.cuh"
#include "am_linalg.cuh"

namespace am {
namespace {

constexpr int VB = 64;               // tile edge
constexpr int kVsThreads = 256;      // 16 × 16 threads, 4 × 4 outputs each
typedef double Tile[VB][VB + 1];     // shared-memory tile (odd row stride)
constexpr size_t kTileBytes = sizeof(Tile);

// The i-th tile of the kernel's dynamic shared memory.
__device__ __forceinline__ Tile& smem_tile(int i) {
  extern __shared__ __align__(16) double vs_smem[];
  return *reinterpret_cast<Tile*>(vs_smem + (size_t)i * VB * (VB + 1));
}

__device__ __forceinline__ bool head_failed(const Work& w, int h) {
  return (w.status[h] / 1000) >= 3;   // an error at or above AM_ERR_NOT_SPD's severity
}

// Loads the (rows × cols) block at M + r0·ld + c0 into T (zero padded to 64 × 64).
__device__ __forceinline__ void load_tile(Tile& T, const double* M, int64_t ld, int r0, int c0, int rows, int cols) {
  for (int e = threadIdx.x; e < VB * VB; e += blockDim.x) {
    const int r = e / VB, c = e % VB;
    T[r][c] = (r < rows && c < cols) ? M[(int64_t)(r0 + r) * ld + c0 + c] : 0.0;
  }
}

// acc[u][v] = Σ_k A(tr+u, k)·B(k, tc+v) for 64 × 64 tiles, where A(r, k) is
// At[r][k] (or At[k][r] when ta) and B(k, c) is Bt[k][c] (or Bt[c][k] when tb).
template <bool TA, bool TB>
__device__ __forceinline__ void tile_mm(const Tile& At, const Tile& Bt, double (&acc)[4][4]) {
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.0;
#pragma unroll 4
  for (int k = 0; k < VB; ++k) {
    double a[4], b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      a[u] = TA ? At[k][tr + u] : At[tr + u][k];
      b[u] = TB ? Bt[tc + u][k] : Bt[k][tc + u];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
  }
}

__global__ void __launch_bounds__(kVsThreads) k_vs_ridge(Problem p, Work w) {
  const int h = blockIdx.x;
  const int t = w.t[h];
  __shared__ double scratch[33];
  double* M = w.AtA + w.cu_t2[h];
  double tr = 0.0;
  for (int a = threadIdx.x; a < t; a += blockDim.x) tr += M[(int64_t)a * t + a];
  tr = block_sum(tr, scratch);
  const double lam = (double)p.ridge * tr / t;
  for (int a = threadIdx.x; a < t; a += blockDim.x) M[(int64_t)a * t + a] += lam;
}

// Diagonal tile kb: Cholesky in shared memory (one column step per
// iteration), written back, and its inverse (lower triangular) stored at
// w.vinv + (cu_t[h] + 64h)·64 + kb·4096 as a zero-padded 64 × 64 block.
__global__ void __launch_bounds__(kVsThreads) k_vs_diag(Problem p, Work w, int kb) {
  const int h = blockIdx.x;
  const int t = w.t[h];
  const int k0 = kb * VB;
  if (k0 >= t || head_failed(w, h)) return;
  const int kw = min(VB, t - k0);
  Tile& D = smem_tile(0);
  double* M = w.AtA + w.cu_t2[h];
  load_tile(D, M, t, k0, k0, kw, kw);
  __syncthreads();
  bool bad = false;
  for (int k = 0; k < kw; ++k) {
    const double dkk = D[k][k];
    if (!(dkk > 0.0)) {   // every thread reads the same pivot and leaves together
      bad = true;
      break;
    }
    const double lkk = sqrt(dkk), il = 1.0 / lkk;
    __syncthreads();   // all have read D[k][k]
    for (int r = k + 1 + threadIdx.x; r < kw; r += blockDim.x) D[r][k] *= il;
    if (threadIdx.x == 0) D[k][k] = lkk;
    __syncthreads();
    // trailing lower triangle of the tile: D[r][c] −= D[r][k]·D[c][k], k < c <= r < kw
    const int m = kw - 1 - k;
    for (int e = threadIdx.x; e < m * m; e += blockDim.x) {
      const int r = k + 1 + e / m, c = k + 1 + e % m;
      if (c <= r) D[r][c] -= D[r][k] * D[c][k];
    }
    __syncthreads();
  }
  if (bad) {
    if (threadIdx.x == 0) record_status(w.status + h, AM_ERR_NOT_SPD);
    return;
  }
  for (int e = threadIdx.x; e < kw * kw; e += blockDim.x) {
    const int r = e / kw, c = e % kw;
    if (c <= r) M[(int64_t)(k0 + r) * t + k0 + c] = D[r][c];
  }
  // inverse: thread c < 64 solves L x = e_c by forward substitution (column c)
  double* inv = w.vinv + (w.cu_t[h] + (int64_t)VB * h) * VB + (int64_t)kb * VB * VB;
  if (threadIdx.x < VB) {
    const int c = threadIdx.x;
    double x[VB];
#pragma unroll
    for (int r = 0; r < VB; ++r) {
      double acc = r == c ? 1.0 : 0.0;
#pragma unroll
      for (int j = 0; j < r; ++j) acc -= D[r][j] * x[j];
      x[r] = (r < kw && r >= c) ? acc / D[r][r] : 0.0;
    }
#pragma unroll
    for (int r = 0; r < VB; ++r) inv[r * VB + c] = x[r];
  }
}

__device__ __forceinline__ const double* tile_inv(const Work& w, int h, int kb) {
  return w.vinv + (w.cu_t[h] + (int64_t)VB * h) * VB + (int64_t)kb * VB * VB;
}

// Panel: for row tile i = kb + 1 + blockIdx.x, M_ik ← M_ik · L_kk⁻ᵀ.
__global__ void __launch_bounds__(kVsThreads) k_vs_panel(Problem p, Work w, int kb) {
  const int h = blockIdx.y;
  const int t = w.t[h];
  const int i = kb + 1 + blockIdx.x;
  const int k0 = kb * VB, i0 = i * VB;
  if (i0 >= t || head_failed(w, h)) return;
  const int kw = min(VB, t - k0), iw = min(VB, t - i0);
  Tile& A = smem_tile(0);
  Tile& Inv = smem_tile(1);
  double* M = w.AtA + w.cu_t2[h];
  load_tile(A, M, t, i0, k0, iw, kw);
  load_tile(Inv, tile_inv(w, h, kb), VB, 0, 0, VB, VB);
  __syncthreads();
  double acc[4][4];
  tile_mm<false, true>(A, Inv, acc);   // Σ_j A[r][j] Inv[c][j]
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v)
      if (tr + u < iw && tc + v < kw) M[(int64_t)(i0 + tr + u) * t + k0 + tc + v] = acc[u][v];
}

// Trailing update: tile pair (i, j), kb < j <= i, M_ij −= L_ik L_jkᵀ.
__global__ void __launch_bounds__(kVsThreads) k_vs_update(Problem p, Work w, int kb) {
  const int h = blockIdx.y;
  const int t = w.t[h];
  const int nb = (t + VB - 1) / VB;
  const int m = nb - 1 - kb;
  int pr = blockIdx.x;
  if (pr >= m * (m + 1) / 2 || head_failed(w, h)) return;
  int a = 0;
  while ((a + 1) * (a + 2) / 2 <= pr) ++a;
  const int i = kb + 1 + a, j = kb + 1 + (pr - a * (a + 1) / 2);
  const int k0 = kb * VB, i0 = i * VB, j0 = j * VB;
  const int kw = min(VB, t - k0), iw = min(VB, t - i0), jw = min(VB, t - j0);
  Tile& Li = smem_tile(0);
  Tile& Lj = smem_tile(1);
  double* M = w.AtA + w.cu_t2[h];
  load_tile(Li, M, t, i0, k0, iw, kw);
  load_tile(Lj, M, t, j0, k0, jw, kw);
  __syncthreads();
  double acc[4][4];
  tile_mm<false, true>(Li, Lj, acc);   // Σ_k Li[r][k] Lj[c][k]
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int r = i0 + tr + u, c = j0 + tc + v;
      if (tr + u < iw && tc + v < jw && c <= r) M[(int64_t)r * t + c] -= acc[u][v];
    }
}

// Forward step kb over the 64-column slice blockIdx.y of X = AᵀY.
// DIAG: row tile kb ← L_kk⁻¹ X_kb (backward: L_kk⁻ᵀ X_kb), one CTA per slice.
// Otherwise, with X_kb already solved by the DIAG launch: row tile
// i = kb + 1 + blockIdx.x takes X_i −= L_ik X_kb (backward: i = kb − 1 −
// blockIdx.x takes X_i −= L_kiᵀ X_kb).
template <bool BWD, bool DIAG>
__global__ void __launch_bounds__(kVsThreads) k_vs_solve(Problem p, Work w, int kb) {
  const int h = blockIdx.z;
  const int t = w.t[h];
  const int k0 = kb * VB;
  if (k0 >= t || head_failed(w, h)) return;
  const int i = DIAG ? kb : (BWD ? kb - 1 - (int)blockIdx.x : kb + 1 + (int)blockIdx.x);
  if (i < 0 || i * VB >= t) return;
  const int c0 = blockIdx.y * VB;
  if (c0 >= p.d) return;
  const int kw = min(VB, t - k0), cw = min(VB, p.d - c0);
  Tile& Lt = smem_tile(0);
  Tile& Xk = smem_tile(1);
  double* X = w.AtY + w.cu_t[h] * p.d;
  const double* M = w.AtA + w.cu_t2[h];
  const int i0 = i * VB, iw = min(VB, t - i0);
  if (DIAG) load_tile(Lt, tile_inv(w, h, kb), VB, 0, 0, VB, VB);
  else if (BWD) load_tile(Lt, M, t, k0, i0, kw, iw);   // L_ki: rows k0.., cols i0..
  else load_tile(Lt, M, t, i0, k0, iw, kw);            // L_ik: rows i0.., cols k0..
  load_tile(Xk, X, p.d, k0, c0, kw, cw);
  __syncthreads();
  double acc[4][4];
  if (BWD) tile_mm<true, false>(Lt, Xk, acc);    // Σ_j Lt[j][r] Xk[j][c]
  else tile_mm<false, false>(Lt, Xk, acc);      // Σ_j Lt[r][j] Xk[j][c]
  const int tr = (threadIdx.x / 16) * 4, tc = (threadIdx.x % 16) * 4;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      if (tr + u >= iw || tc + v >= cw) continue;
      double& x = X[(int64_t)(i0 + tr + u) * p.d + c0 + tc + v];
      if (DIAG) x = acc[u][v];
      else x -= acc[u][v];
    }
}

// C_v (fp32, packed) from the solved X; zero for a head whose factor failed.
__global__ void k_vs_out(Problem p, Work w, float* C_v) {
  const int h = blockIdx.y;
  const int t = w.t[h];
  const bool bad = head_failed(w, h);
  const int64_t base = w.cu_t[h];
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)t * p.d;
       e += (int64_t)gridDim.x * blockDim.x)
    C_v[base * p.d + e] = bad ? 0.f : (float)w.AtY[base * p.d + e];
}

}  // namespace

cudaError_t launch_value_solve_tiled(const Problem& p, const Work& w, float* C_v, cudaStream_t s) {
  const int nb = (p.max_t + VB - 1) / VB;
  const int ncs = (p.d + VB - 1) / VB;
  const int two = (int)(2 * kTileBytes);
  cudaFuncSetAttribute(k_vs_panel, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
  cudaFuncSetAttribute(k_vs_update, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
  cudaFuncSetAttribute(k_vs_solve<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
  cudaFuncSetAttribute(k_vs_solve<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
  cudaFuncSetAttribute(k_vs_solve<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
  cudaFuncSetAttribute(k_vs_solve<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, two);
  AM_LAUNCH(AM_STAGE_SOLVE, s, k_vs_ridge<<<p.H, kVsThreads, 0, s>>>(p, w));
  for (int kb = 0; kb < nb; ++kb) {
    AM_LAUNCH(AM_STAGE_SOLVE, s, k_vs_diag<<<p.H, kVsThreads, kTileBytes, s>>>(p, w, kb));
    const int below = nb - 1 - kb;
    if (below > 0) {
      AM_LAUNCH(AM_STAGE_SOLVE, s, k_vs_panel<<<dim3(below, p.H), kVsThreads, two, s>>>(p, w, kb));
      AM_LAUNCH(AM_STAGE_SOLVE, s,
                k_vs_update<<<dim3(below * (below + 1) / 2, p.H), kVsThreads, two, s>>>(p, w, kb));
    }
  }
  for (int kb = 0; kb < nb; ++kb) {
    AM_LAUNCH(AM_STAGE_SOLVE, s, (k_vs_solve<false, true><<<dim3(1, ncs, p.H), kVsThreads, two, s>>>(p, w, kb)));
    if (nb - 1 - kb > 0)
      AM_LAUNCH(AM_STAGE_SOLVE, s,
                (k_vs_solve<false, false><<<dim3(nb - 1 - kb, ncs, p.H), kVsThreads, two, s>>>(p, w, kb)));
  }
  for (int kb = nb - 1; kb >= 0; --kb) {
    AM_LAUNCH(AM_STAGE_SOLVE, s, (k_vs_solve<true, true><<<dim3(1, ncs, p.H), kVsThreads, two, s>>>(p, w, kb)));
    if (kb > 0)
      AM_LAUNCH(AM_STAGE_SOLVE, s, (k_vs_solve<true, false><<<dim3(kb, ncs, p.H), kVsThreads, two, s>>>(p, w, kb)));
  }
  AM_LAUNCH(AM_STAGE_SOLVE, s, k_vs_out<<<dim3(64, p.H), 256, 0, s>>>(p, w, C_v));
  return cudaGetLastError();
}

}  // namespace am
