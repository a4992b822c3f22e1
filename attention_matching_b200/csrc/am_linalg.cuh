// Small dense float64 linear algebra for one thread block: a packed
// lower-triangular Cholesky factor and its triangular solves.  Used by the
// per-head NNLS refit and the per-head ridge value fit.
//
// Packed storage: row i of the lower triangle holds entries (i, 0..i) at
// tri(i, 0) .. tri(i, i).  The pointer may be shared or global memory.
#pragma once

#include "am_internal.cuh"

namespace am {

__device__ __forceinline__ int64_t tri(int i, int j) { return (int64_t)i * (i + 1) / 2 + j; }

// In-place Cholesky of the packed symmetric matrix M (n×n): M = L Lᵀ.
// Pivot k must exceed pivot_floor(k) (a caller-supplied functor); returns the
// first failing index, or -1 on success.  All threads of the block must call.
template <class Floor>
__device__ int block_cholesky_packed(double* M, int n, Floor pivot_floor, int* s_flag) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  for (int k = 0; k < n; ++k) {
    if (tid == 0) {
      double dkk = M[tri(k, k)];
      if (!(dkk > pivot_floor(k))) {
        *s_flag = k;
      } else {
        M[tri(k, k)] = sqrt(dkk);
        *s_flag = -1;
      }
    }
    __syncthreads();
    int bad = *s_flag;
    if (bad >= 0) return bad;
    const double lkk = M[tri(k, k)];
    for (int i = k + 1 + tid; i < n; i += blockDim.x) M[tri(i, k)] /= lkk;
    __syncthreads();
    // trailing update: rows to warps, columns to lanes
    for (int i = k + 1 + warp; i < n; i += nw) {
      const double lik = M[tri(i, k)];
      for (int j = k + 1 + lane; j <= i; j += 32) M[tri(i, j)] -= lik * M[tri(j, k)];
    }
    __syncthreads();
  }
  return -1;
}

// Warp-level solves on one right-hand side v (length n, shared memory),
// overwritten with the solution.  Called by exactly one full warp.
__device__ __forceinline__ void warp_forward_solve(const double* L, double* v, int n) {
  const int lane = threadIdx.x & 31;
  for (int k = 0; k < n; ++k) {
    const double yk = v[k] / L[tri(k, k)];
    __syncwarp();
    if (lane == 0) v[k] = yk;
    for (int i = k + 1 + lane; i < n; i += 32) v[i] -= L[tri(i, k)] * yk;
    __syncwarp();
  }
}

__device__ __forceinline__ void warp_backward_solve(const double* L, double* v, int n) {
  const int lane = threadIdx.x & 31;
  for (int k = n - 1; k >= 0; --k) {
    const double zk = v[k] / L[tri(k, k)];
    __syncwarp();
    if (lane == 0) v[k] = zk;
    const double* row = L + tri(k, 0);
    for (int i = lane; i < k; i += 32) v[i] -= row[i] * zk;
    __syncwarp();
  }
}

__device__ __forceinline__ double warp_sum(double v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide sum of one double; all threads get the result.  scratch >= 33.
__device__ __forceinline__ double block_sum(double v, double* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    double x = lane < nw ? scratch[lane] : 0.0;
    x = warp_sum(x);
    if (lane == 0) scratch[32] = x;
  }
  __syncthreads();
  return scratch[32];
}

}  // namespace am
