// Small dense float64 linear algebra for one thread block: packed
// lower-triangular indexing, warp and block sums, and the tiled Cholesky of
// the ridge value fit (the NNLS refit keeps its own blocked solves).
//
// Packed storage: row i of the lower triangle holds entries (i, 0..i) at
// tri(i, 0) .. tri(i, i).  The pointer may be shared or global memory.
#pragma once

#include "am_internal.cuh"

namespace am {

__device__ __forceinline__ int64_t tri(int i, int j) { return (int64_t)i * (i + 1) / 2 + j; }

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

namespace am {

// Blocked Cholesky of a packed lower-triangular matrix that lives in global
// memory (too large for shared memory): 32×32 tiles, right-looking.
//   1. the diagonal tile is factored in shared memory (pivot k must exceed
//      pivot_floor(k), else the index is returned);
//   2. the panel of tiles below it is solved row by row (X = M L_Dᵀ⁻¹);
//   3. the trailing lower triangle is updated tile by tile, M_ij −= X_i X_jᵀ,
//      four 64-thread groups each taking one tile, 4×4 outputs per thread.
// Each tile row is 32 consecutive doubles of the packed storage, so every
// global access is coalesced.  Needs 4·3·32·33 + 32·33 doubles of shared
// scratch (≈ 110 KB); all threads of the block (256) must call.  When dinv
// is given, the inverse of each factored diagonal tile is stored there as a
// zero-padded row-major 32×32 block (tile kb at dinv + kb·1024): one warp,
// lane c solving D x = e_c by forward substitution.
constexpr int kTile = 32;
constexpr size_t kTiledScratchDoubles = 4 * 3 * kTile * (kTile + 1) + kTile * (kTile + 1);

template <class Floor>
__device__ int block_cholesky_tiled(double* M, int n, Floor pivot_floor, double* scratch, int* s_flag,
                                    double* dinv = nullptr) {
  const int tid = threadIdx.x;
  double (*D)[kTile + 1] = reinterpret_cast<double (*)[kTile + 1]>(scratch);
  double* grp_base = scratch + kTile * (kTile + 1);
  const int nb = (n + kTile - 1) / kTile;
  for (int kb = 0; kb < nb; ++kb) {
    const int k0 = kb * kTile, kw = min(kTile, n - k0);
    // 1. diagonal tile
    for (int e = tid; e < kTile * kTile; e += blockDim.x) {
      const int r = e / kTile, c = e % kTile;
      D[r][c] = (r < kw && c <= r) ? M[tri(k0 + r, k0 + c)] : 0.0;
    }
    __syncthreads();
    if (tid < 32) {
      const int lane = tid;
      int bad = -1;
      for (int k = 0; k < kw; ++k) {
        const double dkk = D[k][k];
        if (!(dkk > pivot_floor(k0 + k))) { bad = k0 + k; break; }
        const double lkk = sqrt(dkk);
        __syncwarp();
        if (lane == 0) D[k][k] = lkk;
        if (lane > k && lane < kw) D[lane][k] /= lkk;
        __syncwarp();
        if (lane > k && lane < kw)
          for (int c = k + 1; c <= lane; ++c) D[lane][c] -= D[lane][k] * D[c][k];
        __syncwarp();
      }
      if (lane == 0) *s_flag = bad;
    }
    __syncthreads();
    if (*s_flag >= 0) return *s_flag;
    for (int e = tid; e < kTile * kTile; e += blockDim.x) {
      const int r = e / kTile, c = e % kTile;
      if (r < kw && c <= r) M[tri(k0 + r, k0 + c)] = D[r][c];
    }
    if (dinv && tid < 32) {   // lane c: column c of D⁻¹
      const int c = tid;
      double x[kTile];
#pragma unroll
      for (int r = 0; r < kTile; ++r) {
        double acc = r == c ? 1.0 : 0.0;
#pragma unroll
        for (int j = 0; j < r; ++j) acc -= D[r][j] * x[j];
        x[r] = (r < kw && r >= c) ? acc / D[r][r] : 0.0;
      }
      double* out = dinv + (int64_t)kb * kTile * kTile;
#pragma unroll
      for (int r = 0; r < kTile; ++r) out[r * kTile + c] = x[r];
    }
    // 2. panel: rows below the diagonal tile, X_r = M_r L_Dᵀ⁻¹ (one thread per row)
    for (int r = k0 + kw + tid; r < n; r += blockDim.x) {
      double* row = M + tri(r, k0);
      double x[kTile];
#pragma unroll
      for (int c = 0; c < kTile; ++c) x[c] = c < kw ? row[c] : 0.0;
#pragma unroll
      for (int c = 0; c < kTile; ++c) {
        if (c < kw) {
          double s = x[c];
          for (int c2 = 0; c2 < c; ++c2) s -= x[c2] * D[c][c2];
          x[c] = s / D[c][c];
        }
      }
#pragma unroll
      for (int c = 0; c < kTile; ++c)
        if (c < kw) row[c] = x[c];
    }
    __syncthreads();
    // 3. trailing update over tile pairs (ib >= jb > kb)
    const int m = nb - kb - 1;
    const int npairs = m * (m + 1) / 2;
    const int grp = tid >> 6, gt = tid & 63;
    double (*Xi)[kTile + 1] = reinterpret_cast<double (*)[kTile + 1]>(grp_base + grp * 3 * kTile * (kTile + 1));
    double (*Xj)[kTile + 1] = Xi + kTile;
    const int tr = (gt >> 3) * 4, tc = (gt & 7) * 4;   // this thread's 4×4 outputs
    for (int pb = 0; pb < npairs; pb += 4) {
      const int pr = pb + grp;
      const bool live = pr < npairs;
      int ib = 0, jb = 0;
      if (live) {
        int a = 0;
        while ((a + 1) * (a + 2) / 2 <= pr) ++a;
        ib = kb + 1 + a;
        jb = kb + 1 + (pr - a * (a + 1) / 2);
      }
      const int i0 = ib * kTile, j0 = jb * kTile;
      if (live) {
        for (int e = gt; e < kTile * kTile; e += 64) {
          const int r = e / kTile, c = e % kTile;
          Xi[r][c] = (i0 + r < n && c < kw) ? M[tri(i0 + r, k0 + c)] : 0.0;
          Xj[r][c] = (j0 + r < n && c < kw) ? M[tri(j0 + r, k0 + c)] : 0.0;
        }
      }
      __syncthreads();
      if (live) {
        double acc[4][4] = {};
        for (int c = 0; c < kw; ++c) {
          double xi[4], xj[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) { xi[u] = Xi[tr + u][c]; xj[u] = Xj[tc + u][c]; }
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[u][v] = fma(xi[u], xj[v], acc[u][v]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int r = i0 + tr + u, c = j0 + tc + v;
            if (r < n && c <= r) M[tri(r, c)] -= acc[u][v];
          }
      }
      __syncthreads();
    }
  }
  return -1;
}

}  // namespace am
