// OMP key selection with NNLS refits, batched over heads.
//
// "Fast KV Compaction via Attention Matching": zhichai.net deep dive §1.6
// (r = m; repeat: j* = argmax_{j∉S} rᵀΦ_{:,j}, S ∪= {j*}, refit w ≥ 0 by
// NNLS, r = m − Φ_S w); xinfinite.net article §2 step 2 (Fig. 1, Fig. 2:
// NNLS solved on the GPU) and §3 (top-k batched selection with lazy refit,
// Table 1).
//
// One "pass" covers R rounds of k picks: the residual does not change
// between refits, so those R rounds take the next k·R keys of one
// correlation vector.  A pass is four or five launches over the active heads:
//   correlation and selection of the top-(k·R) unselected keys (ties to the
//             lowest index): k_rows twice (the default bounded mode,
//             am_bounded.cu), or k_corr / k_corr_tc (c = Φᵀ r streamed or
//             recomputed) then k_select
//   k_gram_tile (k_gram past 16 picks per pass)  new rows/columns of
//             G = Φ_SᵀΦ_S and b = Φ_Sᵀm (fp64 sums)
//   k_nnls    active-set NNLS on (G, b), warm-started from the last refit
//   k_resid   r = m − Φ_S w (fp64 sums, stored fp32) and partials of ‖r‖²
// The pass kernels are chained with programmatic dependent launch.
#include "am_internal.cuh"
#include "am_async.cuh"
#include "am_profile.cuh"
#include "am_linalg.cuh"

#include <float.h>

namespace am {
namespace {


// ---------------------------------------------------------------- init ----
__global__ void k_init(Problem p, Work w) {
  const int h = blockIdx.x;
  __shared__ double scratch[33];
  const double* m = w.m + (int64_t)h * p.ldn;
  double acc = 0.0;
  for (int i = threadIdx.x; i < p.n; i += blockDim.x) acc += m[i] * m[i];
  acc = block_sum(acc, scratch);
  // Σ m² per residual query group (the groups of k_resid's ‖r‖² partials):
  // r = m until the first refit; warp w takes groups w, w + 8, ...
  {
    const int G = resid_blocks(p), lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int nseg = p.ldn / 128 + (p.ldn % 128 ? 1 : 0);
    for (int g = threadIdx.x >> 5; g < G; g += nw) {
      double sg = 0.0;
      for (int seg = g; seg < nseg; seg += G)
        for (int i = seg * 128 + lane; i < min(p.ldn, seg * 128 + 128); i += 32) sg += m[i] * m[i];
      sg = warp_sum(sg);
      if (lane == 0) w.rr_part[(int64_t)h * kRedBlocks + g] = sg;
    }
  }
  if (threadIdx.x == 0) {
    w.mm[h] = acc;
    w.np[h] = 0;
    w.ylen[h] = 0;
    w.dvalid[h] = 0;
    if (!(acc > 0.0) || !isfinite(acc)) record_status(w.status + h, AM_ERR_NONFINITE);
  }
  // keys past the head's own count are marked as taken: never candidates
  uint8_t* sel = w.sel + (int64_t)h * p.T;
  const int Th = w.Th[h];
  for (int j = threadIdx.x; j < p.T; j += blockDim.x) sel[j] = j >= Th;
}

// ----------------------------------------------------------- correlation --
// One warp per 4 key rows; 128-bit streaming loads of Φᵀ (4 fp32 or 8 bf16
// features per load), r from L1.
constexpr int kCorrRowsPerWarp = 4;
constexpr int kCorrWarps = 8;
constexpr int kCorrRowsPerBlock = kCorrRowsPerWarp * kCorrWarps;

__device__ __forceinline__ float dot8_bf16(uint4 x, float4 ra, float4 rb, float acc) {
  const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&x);
  float2 f0 = __bfloat1622float2(e[0]), f1 = __bfloat1622float2(e[1]);
  float2 f2 = __bfloat1622float2(e[2]), f3 = __bfloat1622float2(e[3]);
  acc = fmaf(f0.x, ra.x, acc); acc = fmaf(f0.y, ra.y, acc);
  acc = fmaf(f1.x, ra.z, acc); acc = fmaf(f1.y, ra.w, acc);
  acc = fmaf(f2.x, rb.x, acc); acc = fmaf(f2.y, rb.y, acc);
  acc = fmaf(f3.x, rb.z, acc); acc = fmaf(f3.y, rb.w, acc);
  return acc;
}

__global__ void __launch_bounds__(256) k_corr(Problem p, Work w, int pass) {
  const int h = w.order[blockIdx.y];
  const int t = w.t[h];
  if (pass * p.kR >= t) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int j0 = blockIdx.x * kCorrRowsPerBlock + warp * kCorrRowsPerWarp;
  const int Th = w.Th[h];   // rows past the head's keys are never read
  if (j0 >= Th) return;
  const float4* r4 = reinterpret_cast<const float4*>(w.r + (int64_t)h * p.ldn);
  float acc[kCorrRowsPerWarp] = {0.f, 0.f, 0.f, 0.f};
  if (w.phiT16) {
    const uint4* rows[kCorrRowsPerWarp];
#pragma unroll
    for (int q = 0; q < kCorrRowsPerWarp; ++q) {
      const int j = min(j0 + q, Th - 1);
      rows[q] = reinterpret_cast<const uint4*>(w.phiT16 + ((int64_t)h * p.T + j) * p.ldn);
    }
    const int n8 = p.ldn >> 3;
    int i = lane;
    for (; i + 32 < n8; i += 64) {
      const float4 ra0 = __ldg(r4 + 2 * i), rb0 = __ldg(r4 + 2 * i + 1);
      const float4 ra1 = __ldg(r4 + 2 * (i + 32)), rb1 = __ldg(r4 + 2 * (i + 32) + 1);
      uint4 xa[kCorrRowsPerWarp], xb[kCorrRowsPerWarp];
#pragma unroll
      for (int q = 0; q < kCorrRowsPerWarp; ++q) {
        xa[q] = __ldcs(rows[q] + i);
        xb[q] = __ldcs(rows[q] + i + 32);
      }
#pragma unroll
      for (int q = 0; q < kCorrRowsPerWarp; ++q) {
        acc[q] = dot8_bf16(xa[q], ra0, rb0, acc[q]);
        acc[q] = dot8_bf16(xb[q], ra1, rb1, acc[q]);
      }
    }
    for (; i < n8; i += 32) {
      const float4 ra = __ldg(r4 + 2 * i), rb = __ldg(r4 + 2 * i + 1);
#pragma unroll
      for (int q = 0; q < kCorrRowsPerWarp; ++q) acc[q] = dot8_bf16(__ldcs(rows[q] + i), ra, rb, acc[q]);
    }
  } else {
    const float4* rows[kCorrRowsPerWarp];
#pragma unroll
    for (int q = 0; q < kCorrRowsPerWarp; ++q) {
      const int j = min(j0 + q, Th - 1);
      rows[q] = reinterpret_cast<const float4*>(w.phiT + ((int64_t)h * p.T + j) * p.ldn);
    }
    const int n4 = p.ldn >> 2;
    int i = lane;
    for (; i + 32 < n4; i += 64) {
      const float4 ra = __ldg(r4 + i), rb = __ldg(r4 + i + 32);
      float4 xa[kCorrRowsPerWarp], xb[kCorrRowsPerWarp];
#pragma unroll
      for (int q = 0; q < kCorrRowsPerWarp; ++q) {
        xa[q] = __ldcs(rows[q] + i);
        xb[q] = __ldcs(rows[q] + i + 32);
      }
#pragma unroll
      for (int q = 0; q < kCorrRowsPerWarp; ++q) {
        acc[q] = fmaf(xa[q].x, ra.x, acc[q]); acc[q] = fmaf(xa[q].y, ra.y, acc[q]);
        acc[q] = fmaf(xa[q].z, ra.z, acc[q]); acc[q] = fmaf(xa[q].w, ra.w, acc[q]);
        acc[q] = fmaf(xb[q].x, rb.x, acc[q]); acc[q] = fmaf(xb[q].y, rb.y, acc[q]);
        acc[q] = fmaf(xb[q].z, rb.z, acc[q]); acc[q] = fmaf(xb[q].w, rb.w, acc[q]);
      }
    }
    for (; i < n4; i += 32) {
      const float4 ra = __ldg(r4 + i);
#pragma unroll
      for (int q = 0; q < kCorrRowsPerWarp; ++q) {
        const float4 x = __ldcs(rows[q] + i);
        acc[q] = fmaf(x.x, ra.x, acc[q]); acc[q] = fmaf(x.y, ra.y, acc[q]);
        acc[q] = fmaf(x.z, ra.z, acc[q]); acc[q] = fmaf(x.w, ra.w, acc[q]);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kCorrRowsPerWarp; ++q) {
    float v = acc[q];
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && j0 + q < Th) w.corr[(int64_t)h * p.T + j0 + q] = v;
  }
}

// -------------------------------------------------------------- select ----
__global__ void __launch_bounds__(1024) k_select(Problem p, Work w, int pass) {
  const int h = w.order[blockIdx.x];
  const int t = w.t[h];
  int s0, s1;
  pass_range(p, t, pass, s0, s1);
  if (s0 >= s1) return;
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ int bad;
  const float* c = w.corr + (int64_t)h * p.T;
  uint8_t* sel = w.sel + (int64_t)h * p.T;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int q = s0; q < s1; ++q) {
    float bv = -INFINITY;
    int bi = INT_MAX;
    for (int j = threadIdx.x; j < p.T; j += blockDim.x) {
      if (sel[j]) continue;
      float v = c[j];
      if (v != v) { v = -INFINITY; bad = 1; }
      if (v > bv || (v == bv && j < bi)) { bv = v; bi = j; }
    }
    for (int o = 16; o; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
    }
    if (lane == 0) { sv[warp] = bv; si[warp] = bi; }
    __syncthreads();
    if (warp == 0) {
      bv = lane < (int)(blockDim.x >> 5) ? sv[lane] : -INFINITY;
      bi = lane < (int)(blockDim.x >> 5) ? si[lane] : INT_MAX;
      for (int o = 16; o; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (lane == 0) {
        if (bi == INT_MAX) {  // everything left is -inf: take the lowest free key
          for (int j = 0; j < p.T; ++j)
            if (!sel[j]) { bi = j; break; }
          bad = 1;
        }
        const int64_t o = w.cu_t[h] + q;
        w.picks[o] = bi;
        w.pick_corr[o] = bv;
        sel[bi] = 1;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0 && bad) record_status(w.status + h, AM_ERR_NONFINITE);
}

// ---------------------------------------------------------------- gram ----
// Block (a, head): G[a][b] for the new picks b ∈ [s0, s1) (and the mirror
// G[b][a] when a is an old pick); b_vec[a] = φ_aᵀm when a is new.
constexpr int kGramGroup = 8;

// Dot products (fp64 sums of fp32 products) of one row with nb <= 8 rows.
__device__ __forceinline__ void block_dots(const float4* ra, const float4* const* rb, int nb, int n4,
                                           double (*red)[kGramGroup + 1], double* out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double acc[kGramGroup];
#pragma unroll
  for (int bb = 0; bb < kGramGroup; ++bb) acc[bb] = 0.0;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 x = ra[i];
#pragma unroll
    for (int bb = 0; bb < kGramGroup; ++bb) {
      if (bb < nb) {
        const float4 y = rb[bb][i];
        acc[bb] += (double)x.x * y.x + (double)x.y * y.y + (double)x.z * y.z + (double)x.w * y.w;
      }
    }
  }
#pragma unroll
  for (int bb = 0; bb < kGramGroup; ++bb) {
    const double v = warp_sum(acc[bb]);
    if (lane == 0) red[warp][bb] = v;
  }
  __syncthreads();
  if (threadIdx.x < nb) {
    double v = 0.0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) v += red[k][threadIdx.x];
    out[threadIdx.x] = v;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256) k_gram(Problem p, Work w, int pass) {
  const int h = w.order[blockIdx.y];
  const int t = w.t[h];
  int s0, s1;
  pass_range(p, t, pass, s0, s1);
  const int a = blockIdx.x;
  if (s0 >= s1 || a >= s1) return;
  __shared__ double red[8][kGramGroup + 1];
  __shared__ double res[kGramGroup];
  const int64_t base = w.cu_t[h];
  const int64_t gbase = w.cu_t2[h];
  const int n4 = p.ldn >> 2;
  const float* P0 = w.phiT + (int64_t)h * p.T * p.ldn;
  const float4* ra = reinterpret_cast<const float4*>(P0 + (int64_t)w.picks[base + a] * p.ldn);
  const float4* rb[kGramGroup];
  for (int g0 = s0; g0 < s1; g0 += kGramGroup) {
    const int nb = min(kGramGroup, s1 - g0);
#pragma unroll
    for (int bb = 0; bb < kGramGroup; ++bb)
      rb[bb] = reinterpret_cast<const float4*>(P0 + (int64_t)w.picks[base + min(g0 + bb, s1 - 1)] * p.ldn);
    block_dots(ra, rb, nb, n4, red, res);
    if (threadIdx.x < nb) {
      const int b = g0 + threadIdx.x;
      w.G[gbase + (int64_t)a * t + b] = res[threadIdx.x];
      if (a < s0) w.G[gbase + (int64_t)b * t + a] = res[threadIdx.x];
    }
    __syncthreads();
  }
  if (a >= s0) {   // b_a = φ_aᵀ m with the fp64 mass
    const double2* m2 = reinterpret_cast<const double2*>(w.m + (int64_t)h * p.ldn);
    double acc = 0.0;
    for (int i = threadIdx.x; i < n4; i += blockDim.x) {
      const float4 x = ra[i];
      const double2 u = m2[2 * i], v = m2[2 * i + 1];
      acc += (double)x.x * u.x + (double)x.y * u.y + (double)x.z * v.x + (double)x.w * v.y;
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    acc = warp_sum(acc);
    if (lane == 0) red[warp][0] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      double v = 0.0;
      for (int k = 0; k < (int)(blockDim.x >> 5); ++k) v += red[k][0];
      w.bvec[base + a] = v;
    }
  }
}

// Sums 32 per-lane values across the warp: afterwards lane l holds the
// total of value l (31 shuffles: each step halves the values a lane keeps).
__device__ __forceinline__ double warp_reduce32(double (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const double send = upper ? v[i] : v[i + s];
      const double keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

// Sums N per-lane values (N a power of two, at most 32) across the warp:
// afterwards lane l holds the total of value l mod N (N − 1 halving shuffles,
// then one per remaining lane bit).
template <int N>
__device__ __forceinline__ double warp_reduce_n(double (&v)[N]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = N / 2; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const double send = upper ? v[i] : v[i + s];
      const double keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  double r = v[0];
#pragma unroll
  for (int s = N; s < 32; s <<= 1) r += __shfl_xor_sync(0xffffffffu, r, s);
  return r;
}

// Tiled form for passes of at most kGramMaxNew picks, NB >= the pass's new
// picks.  Block (row group, query slice, head): warp k takes row a0 + k of
// the rows 0 .. s1 (rows below s1 are the picks' feature columns, row s1 is
// m, giving b_new = Σ_i m_i Φ_{i,new}) against the new picks over one slice of
// 512 queries (grid-stride over slices when there are more than gridDim.y).
// The new picks' slice is staged in shared memory and every lane loads its
// row's 16 queries before any is used; lane l then holds the partial of new
// pick l mod NB after one butterfly across the warp.  Products of features
// are exact (fp32 × fp32 in fp64).  The last block of a (head, row group) to
// finish (counted with an atomic) adds the slices' partials in a fixed order
// and writes each unordered pair of G once into both triangles, so G is
// exactly symmetric and the result does not depend on block timing.
constexpr int kGramWarps = 8;        // rows per block
constexpr int kGramSlice4 = 128;     // float4 positions per query slice
constexpr int kGramPos = kGramSlice4 / 32;   // float4 positions per lane

template <int NB>
__global__ void __launch_bounds__(kGramWarps * 32, 2) k_gram_tile(Problem p, Work w, int pass) {
  chain_wait();
  __shared__ __align__(16) float4 stage[NB][kGramSlice4];
  __shared__ const float4* newrow[NB];
  __shared__ int s_last;
  const int h = w.order[blockIdx.z];
  const int t = w.t[h];
  int s0, s1;
  pass_range(p, t, pass, s0, s1);
  const int a0 = blockIdx.x * kGramWarps;
  if (s0 >= s1 || a0 > s1) return;
  const int nb = s1 - s0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int a = a0 + warp;                     // warp-uniform
  const bool is_m = a == s1, live = a <= s1;
  const int64_t base = w.cu_t[h];
  const int64_t gbase = w.cu_t2[h];
  const int n4 = p.ldn >> 2;
  const int nslices = (n4 + kGramSlice4 - 1) / kGramSlice4;
  const float* P0 = w.phiT + (int64_t)h * p.T * p.ldn;
  const double2* m2 = reinterpret_cast<const double2*>(w.m + (int64_t)h * p.ldn);
  if (threadIdx.x < NB)
    newrow[threadIdx.x] = reinterpret_cast<const float4*>(
        P0 + (int64_t)w.picks[base + s0 + min((int)threadIdx.x, nb - 1)] * p.ldn);
  const float4* row = reinterpret_cast<const float4*>(P0 + (int64_t)w.picks[base + min(a, s1 - 1)] * p.ldn);
  __syncthreads();
  double acc[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = 0.0;
  for (int sl = blockIdx.y; sl < nslices; sl += gridDim.y) {
    const int c0 = sl * kGramSlice4;
    const int cw = min(kGramSlice4, n4 - c0);
    // the new picks' columns go straight to shared memory (asynchronous 16-byte
    // copies, zeros past the picks and the slice), in flight with this warp's row
    constexpr int kStage = (NB * kGramSlice4 + kGramWarps * 32 - 1) / (kGramWarps * 32);
#pragma unroll
    for (int u = 0; u < kStage; ++u) {
      const int e = threadIdx.x + u * kGramWarps * 32, b = e / kGramSlice4, i = e % kGramSlice4;
      if (e < NB * kGramSlice4) {
        if (b < nb && i < cw)
          cp_async16(&stage[b][i], &newrow[b][c0 + i]);
        else
          stage[b][i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    cp_async_commit();
    float4 xf[kGramPos];
    double2 xm[kGramPos][2];
    if (is_m) {
#pragma unroll
      for (int k = 0; k < kGramPos; ++k) {
        const int i = lane + 32 * k;
        xm[k][0] = i < cw ? m2[2 * (c0 + i)] : make_double2(0.0, 0.0);
        xm[k][1] = i < cw ? m2[2 * (c0 + i) + 1] : make_double2(0.0, 0.0);
      }
    } else {
#pragma unroll
      for (int k = 0; k < kGramPos; ++k) {
        const int i = lane + 32 * k;
        xf[k] = live && i < cw ? row[c0 + i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    cp_async_wait<0>();
    __syncthreads();
    if (is_m) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
#pragma unroll
        for (int k = 0; k < kGramPos; ++k) {
          const float4 y = stage[b][lane + 32 * k];
          acc[b] = fma(xm[k][0].x, (double)y.x, acc[b]);
          acc[b] = fma(xm[k][0].y, (double)y.y, acc[b]);
          acc[b] = fma(xm[k][1].x, (double)y.z, acc[b]);
          acc[b] = fma(xm[k][1].y, (double)y.w, acc[b]);
        }
      }
    } else {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
#pragma unroll
        for (int k = 0; k < kGramPos; ++k) {
          const float4 y = stage[b][lane + 32 * k];
          acc[b] = fma((double)xf[k].x, (double)y.x, acc[b]);
          acc[b] = fma((double)xf[k].y, (double)y.y, acc[b]);
          acc[b] = fma((double)xf[k].z, (double)y.z, acc[b]);
          acc[b] = fma((double)xf[k].w, (double)y.w, acc[b]);
        }
      }
    }
    __syncthreads();
  }
  // partials: [slice][row 0..t (row t: b_new)][kR]
  double* part = w.gpart + (int64_t)kGramMaxSlices * (base + h) * p.kR;
  const int64_t zstride = (int64_t)(t + 1) * p.kR;
  {
    const double tot = warp_reduce_n<NB>(acc);
    const int prow = is_m ? t : a;
    if (live && lane < nb) part[blockIdx.y * zstride + (int64_t)prow * p.kR + lane] = tot;
  }
  chain_release();
  __threadfence();
  __syncthreads();
  int32_t* counter = w.gcount + base + h + blockIdx.x;
  if (threadIdx.x == 0) s_last = atomicAdd(counter, 1) == (int)gridDim.y - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int rows_here = min(kGramWarps, s1 + 1 - a0);
  for (int e = threadIdx.x; e < rows_here * nb; e += blockDim.x) {
    const int ri = e / nb, b = e - ri * nb;
    const int r = a0 + ri;
    const int prow = r == s1 ? t : r;
    double v = 0.0;
    for (int q0 = 0; q0 < (int)gridDim.y; q0 += 8) {   // eight slices' partials in flight
      double z[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        z[q] = q0 + q < (int)gridDim.y ? __ldcg(part + (q0 + q) * zstride + (int64_t)prow * p.kR + b) : 0.0;
#pragma unroll
      for (int q = 0; q < 8; ++q) v += z[q];
    }
    if (r == s1) {
      w.bvec[base + s0 + b] = v;
    } else if (r < s0 || s0 + b <= r) {   // each unordered pair once, both triangles
      w.G[gbase + (int64_t)r * t + s0 + b] = v;
      w.G[gbase + (int64_t)(s0 + b) * t + r] = v;
    }
  }
  if (threadIdx.x == 0) *counter = 0;   // ready for the next pass
}

// ---------------------------------------------------------------- NNLS ----
// Lawson-Hanson active set on the normal equations G w = b in fp64, with
// the Cholesky factor of G restricted to the passive set kept across refits.
// Entering variables are appended as a block: their rows are forward-solved
// against the current factor as several right-hand sides at once, then a
// small Cholesky of their Schur complement finishes the new rows.  If an
// entering block holds a variable that will not grow, the refit continues one
// variable at a time.  A variable that leaves the passive set is deleted from
// the factor by a rank-one update of the rows below it (no refactorisation),
// and the forward solve y = L⁻¹ b_P is kept (also across refits) for every
// factor row above the first one that changed, so each solve only extends it.
// The factor is packed by rows (in shared memory while the kernel runs, for
// small budgets), or kept in the workspace as 32×32 tiles with cached
// inverses of its diagonal tiles (larger budgets; see the tiled solves
// below).  Triangular solves multiply by stored reciprocal diagonals.
constexpr int kSB = 32;        // rows per block of the blocked triangular solves
constexpr int kMaxRhs = 8;     // vectors one blocked forward solve carries
constexpr size_t kDiagTileBytes = kSB * (kSB + 1) * sizeof(double);

__host__ __device__ inline size_t nnls_vec_bytes(int t) {
  // x, z, g, invd, y: 5t doubles; red: 64 doubles; diagonal tile: 32×33 doubles;
  // ctl: 16 ints; the factor copy's barrier: 16 bytes; P, inP, blocked, add, cand: 5t ints
  size_t b = (size_t)t * 5 * sizeof(double) + 64 * sizeof(double) + kDiagTileBytes + 16 * sizeof(int) + 16 +
             (size_t)t * 5 * sizeof(int);
  return (b + 15) & ~size_t(15);
}
__host__ __device__ inline size_t nnls_tri_bytes(int t) { return (size_t)t * (t + 1) / 2 * sizeof(double); }
constexpr size_t kSmemCap = 227 * 1024;
constexpr uint32_t kBulkChunk = 32768;               // bytes per bulk copy instruction
constexpr long long kBulkWaitCycles = 4000000000ll;  // ~2 s at 2 GHz

// Blocked triangular solves with the packed factor (shared or global
// memory), run by all threads of the block, 32 rows at a time.  Each block of
// rows takes the products with every solved entry in one parallel pass whose
// factor reads are coalesced (lanes run along a factor row), then one warp per
// vector sweeps the 32×32 diagonal block, staged in shared memory.
typedef double DiagTile[kSB + 1];

// dst[0..n) = src[0..n) by all threads, four loads per thread in flight.
__device__ __forceinline__ void copy_doubles(double* dst, const double* src, int64_t n) {
  for (int64_t e0 = threadIdx.x; e0 < n; e0 += 4 * (int64_t)blockDim.x) {
    double v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = e0 + (int64_t)u * blockDim.x;
      v[u] = e < n ? src[e] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t e = e0 + (int64_t)u * blockDim.x;
      if (e < n) dst[e] = v[u];
    }
  }
}

// D[r][c] = L[r0 + r][r0 + c] for c <= r < bw, zero elsewhere (all loads
// of a thread issued before its stores).
__device__ __forceinline__ void load_diag_tile(const double* L, int r0, int bw, DiagTile* D) {
  for (int e0 = threadIdx.x; e0 < kSB * kSB; e0 += 4 * blockDim.x) {
    double v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * blockDim.x, r = e >> 5, c = e & 31;
      v[u] = (e < kSB * kSB && r < bw && c <= r) ? L[tri(r0 + r, r0 + c)] : 0.0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * blockDim.x;
      if (e < kSB * kSB) D[e >> 5][e & 31] = v[u];
    }
  }
}

// u_e ← L⁻¹ u_e on rows [k0, n) for the R <= 8 vectors U[0..R); entries
// below k0 are already final.  Products: warp w takes rows r0 + 4w .. +3,
// its lanes run across the solved columns.
__device__ void block_forward(const double* L, const double* invd, double* const* U, int R, int k0, int n,
                              DiagTile* D) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r0 = k0; r0 < n; r0 += kSB) {
    const int bw = min(kSB, n - r0);
    load_diag_tile(L, r0, bw, D);
    const int rb = r0 + 4 * warp;
    if (4 * warp < bw && r0 > 0) {
      const double* lr[4];
      bool live[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        live[i] = 4 * warp + i < bw;
        lr[i] = L + tri(live[i] ? rb + i : rb, 0);
      }
      double acc[4][kMaxRhs];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < kMaxRhs; ++e) acc[i][e] = 0.0;
      for (int j0 = lane; j0 < r0; j0 += 32 * 4) {   // four columns per lane in flight
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int j = j0 + 32 * s;
          if (j < r0) {
            double uj[kMaxRhs];
#pragma unroll
            for (int e = 0; e < kMaxRhs; ++e) uj[e] = e < R ? U[e][j] : 0.0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const double l = live[i] ? lr[i][j] : 0.0;
#pragma unroll
              for (int e = 0; e < kMaxRhs; ++e) acc[i][e] = fma(l, uj[e], acc[i][e]);
            }
          }
        }
      }
      double flat[32];   // value i·8 + e: row rb + i, vector e
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < kMaxRhs; ++e) flat[i * kMaxRhs + e] = acc[i][e];
      const double sum = warp_reduce32(flat);
      const int li = lane / kMaxRhs, le = lane % kMaxRhs;
      if (le < R && 4 * warp + li < bw) U[le][rb + li] -= sum;
    }
    __syncthreads();
    if (warp < R) {
      double* u = U[warp];
      double v = lane < bw ? u[r0 + lane] : 0.0;
      for (int c = 0; c < bw; ++c) {
        if (lane == c) v *= invd[r0 + c];
        const double vc = __shfl_sync(0xffffffffu, v, c);
        if (lane > c) v -= D[lane][c] * vc;
      }
      if (lane < bw) u[r0 + lane] = v;
    }
    __syncthreads();
  }
}

// v ← L⁻ᵀ v on rows [0, n).  Blocks from the bottom: one warp sweeps the
// diagonal block, then every row above takes that block's contribution
// (threads across columns, each summing over the block's 32 factor rows).
__device__ void block_backward(const double* L, const double* invd, double* v, int n, DiagTile* D) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int b = (n + kSB - 1) / kSB - 1; b >= 0; --b) {
    const int r0 = b * kSB, bw = min(kSB, n - r0);
    load_diag_tile(L, r0, bw, D);
    __syncthreads();
    if (warp == 0) {
      double x = lane < bw ? v[r0 + lane] : 0.0;
      for (int c = bw - 1; c >= 0; --c) {
        if (lane == c) x *= invd[r0 + c];
        const double xc = __shfl_sync(0xffffffffu, x, c);
        if (lane < c) x -= D[c][lane] * xc;
      }
      if (lane < bw) v[r0 + lane] = x;
    }
    __syncthreads();
    for (int j = tid; j < r0; j += blockDim.x) {
      const double* col = L + tri(r0, 0) + j;   // L[r0 + r][j] = col[r·r0 + r(r+1)/2]
      double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int r = 0; r < kSB; ++r)
        if (r < bw) acc[r & 3] = fma(col[(int64_t)r * r0 + r * (r + 1) / 2], v[r0 + r], acc[r & 3]);
      v[j] -= (acc[0] + acc[1]) + (acc[2] + acc[3]);
    }
    __syncthreads();
  }
}

// ------------------------------------------------- tiled factor solves ----
// A head whose factor lives in the workspace keeps it in 32×32 tiles: tile
// (I, J), J <= I, holds rows 32I .. 32I+31 and columns 32J .. 32J+31
// row-major at offset (I(I+1)/2 + J)·1024, so the off-diagonal tiles of a
// row block are one contiguous range.  Beside the factor the head keeps the
// inverses of its diagonal tiles, D_I = L_II⁻¹ and D_Iᵀ, valid for its first
// `dvalid` row blocks; a triangular solve then takes each diagonal block as
// one 32×32 matrix-vector product instead of 32 dependent steps, and a block
// whose inverse is stale is inverted (one warp, a column per lane) when the
// solve reaches it.  A solve reads the factor once, in order: steps of up to
// kSlotTiles tiles go through a ring of kSlots shared-memory slots filled by
// 16-byte asynchronous copies (cp.async) one step ahead of their use.
constexpr int kTileElems = kSB * kSB;
constexpr int kSlotTiles = 3;
constexpr int kSlots = 3;
constexpr int kSlotDoubles = kSlotTiles * kTileElems;
constexpr size_t kRingBytes = (size_t)kSlots * kSlotDoubles * sizeof(double);
constexpr int kStreamRhs = 8;    // vectors one forward solve carries
constexpr int kAppendRows = 32;  // most new rows the append keeps in shared memory

__host__ __device__ __forceinline__ int64_t tile_at(int I, int J) {
  return ((int64_t)I * (I + 1) / 2 + J) * kTileElems;
}
// element (r, c), c <= r, of a tiled factor
__device__ __forceinline__ int64_t tl(int r, int c) { return tile_at(r >> 5, c >> 5) + (r & 31) * kSB + (c & 31); }
// doubles a tiled factor of order t takes, plus one for the 16-byte alignment
__host__ __device__ inline int64_t tiled_doubles(int t) { return tile_at((t + kSB - 1) / kSB, 0) + 1; }
// the cached inverses of head h: block I at 2·1024·I (D_I) and + 1024 (D_Iᵀ)
__device__ __forceinline__ double* dinv_cache(const Work& w, int h) {
  return w.ndinv + 64 * (w.cu_t[h] + 32 * (int64_t)h);
}

struct Step {
  int I, J0, nt;
  bool diag;
};

// Forward order over row blocks I0 .. I1: each block's off-diagonal tiles in
// steps of up to kSlotTiles, then its diagonal step.
struct ForwardSteps {
  int I, J, I1;
  __device__ bool done() const { return I > I1; }
  __device__ Step step() const {
    Step s;
    s.I = I;
    s.diag = J >= I;
    s.J0 = s.diag ? I : J;
    s.nt = s.diag ? 1 : min(kSlotTiles, I - J);
    return s;
  }
  __device__ void next() {
    if (J >= I) { ++I; J = 0; } else { J += kSlotTiles; }
  }
};

// Backward order over row blocks I1 .. 0: each block's diagonal step, then
// its off-diagonal tiles in steps of up to kSlotTiles.
struct BackwardSteps {
  int I, J;   // J < 0: the diagonal step
  __device__ bool done() const { return I < 0; }
  __device__ Step step() const {
    Step s;
    s.I = I;
    s.diag = J < 0;
    s.J0 = s.diag ? I : J;
    s.nt = s.diag ? 1 : min(kSlotTiles, I - J);
    return s;
  }
  __device__ void next() {
    J = J < 0 ? 0 : J + kSlotTiles;
    if (J >= I) { --I; J = -1; }
  }
};

// Copies step s into a slot and commits the copies as one group: its
// off-diagonal tiles, or for a diagonal step the cached inverse (D_Iᵀ for a
// forward solve, D_I for a backward one) when block I is below dvalid, else
// the factor's diagonal tile.
__device__ __forceinline__ void issue_step(const double* Lt, const double* dc, int dvalid, bool fwd, double* slot,
                                           const Step& s) {
  const double* src = s.diag ? (s.I < dvalid ? dc + (int64_t)s.I * 2 * kTileElems + (fwd ? kTileElems : 0)
                                             : Lt + tile_at(s.I, s.I))
                             : Lt + tile_at(s.I, s.J0);
  const int chunks = s.nt * kTileElems / 2;   // 16-byte chunks
#pragma unroll
  for (int u = 0; u < kSlotDoubles / 2 / kNnlsThreads; ++u) {
    const int e = threadIdx.x + u * kNnlsThreads;
    if (e < chunks) cp_async16(slot + 2 * e, src + 2 * e);
  }
  cp_async_commit();
}

// Runs consume(step, slot) over the steps of `it` in order, with the next
// kSlots − 1 steps' copies in flight.  Every thread of the block calls it;
// consume may synchronise the block.  Ends with the block synchronised.
template <class Steps, class Consume>
__device__ __forceinline__ void stream_steps(const double* Lt, const double* dc, int dvalid, bool fwd, double* ring,
                                             Steps it, Consume&& consume) {
  Steps ahead = it;
#pragma unroll
  for (int s = 0; s < kSlots - 1; ++s) {
    if (!ahead.done()) {
      issue_step(Lt, dc, dvalid, fwd, ring + s * kSlotDoubles, ahead.step());
      ahead.next();
    } else {
      cp_async_commit();
    }
  }
  for (int p = 0; !it.done(); ++p) {
    cp_async_wait<kSlots - 2>();
    __syncthreads();   // step p is in; the slot of step p − 1 is free
    if (!ahead.done()) {
      issue_step(Lt, dc, dvalid, fwd, ring + ((p + kSlots - 1) % kSlots) * kSlotDoubles, ahead.step());
      ahead.next();
    } else {
      cp_async_commit();
    }
    consume(it.step(), static_cast<const double*>(ring + (p % kSlots) * kSlotDoubles));
    it.next();
  }
  cp_async_wait<0>();
  __syncthreads();
}

// X = S⁻¹ for the 32×32 lower-triangular tile S (row-major) with reciprocal
// diagonal id[0..32), by one warp: lane c computes column c, each entry as
// soon as its sum is complete, then adds its terms to every later row's sum
// (independent products, not one chain); rows past the block's last hold
// whatever their entries give.  X goes to D with zeros above the diagonal.
__device__ __noinline__ void invert_tile(const double* S, const double* id, DiagTile* D) {
  const int c = threadIdx.x & 31;
  double a[kSB];
#pragma unroll
  for (int r = 0; r < kSB; ++r) a[r] = 0.0;
#pragma unroll
  for (int m = 0; m < kSB; ++m) {
    const double d = id[m];
    a[m] = m < c ? 0.0 : (m == c ? d : -a[m] * d);
#pragma unroll
    for (int r = m + 1; r < kSB; ++r) a[r] = fma(S[r * kSB + m], a[m], a[r]);
  }
#pragma unroll
  for (int r = 0; r < kSB; ++r) D[r][c] = a[r];
}

// After invert_tile and a block barrier: D_I and D_Iᵀ of block I into the cache.
__device__ __forceinline__ void store_inverse(const DiagTile* D, double* dc, int I) {
  double* di = dc + (int64_t)I * 2 * kTileElems;
  for (int e = threadIdx.x; e < kTileElems; e += blockDim.x) {
    const int a = e >> 5, b = e & 31;
    di[e] = D[a][b];                // D_I[a][b]
    di[kTileElems + e] = D[b][a];   // D_Iᵀ[a][b]
  }
}

// u_e ← L⁻¹ u_e on rows [32·I0, n) for the R <= RMAX vectors u_e = U0 + e·ldu
// (shared memory); entries below 32·I0 are final.  Products: warp w takes
// rows 4w .. 4w+3 of the row block, its lanes a column of each tile; the sums
// close at the diagonal step, which multiplies by D_I, one warp per vector.
// *dvalid is raised past the blocks this solve inverted.
template <int RMAX>
__device__ void stream_forward(const double* Lt, double* dc, int* dvalid, const double* invd, double* U0, int ldu,
                               int R, int I0, int n, double* ring, DiagTile* D) {
  if (32 * I0 >= n) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, rl = 4 * warp;
  const int dv = *dvalid;
  double acc[4][RMAX];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < RMAX; ++e) acc[i][e] = 0.0;
  stream_steps(Lt, dc, dv, true, ring, ForwardSteps{I0, 0, (n - 1) / kSB}, [&](const Step& st, const double* S) {
    const int r0 = kSB * st.I, bw = min(kSB, n - r0);
    if (!st.diag) {
      if (rl < bw) {
        for (int j = 0; j < st.nt; ++j) {
          const int col = kSB * (st.J0 + j) + lane;
          double u[RMAX];
#pragma unroll
          for (int e = 0; e < RMAX; ++e) u[e] = e < R ? U0[e * ldu + col] : 0.0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const double l = rl + i < bw ? S[j * kTileElems + (rl + i) * kSB + lane] : 0.0;
#pragma unroll
            for (int e = 0; e < RMAX; ++e) acc[i][e] = fma(l, u[e], acc[i][e]);
          }
        }
      }
      return;
    }
    if (st.I > 0 && rl < bw) {
      if constexpr (RMAX == 1) {
        double flat[4] = {acc[0][0], acc[1][0], acc[2][0], acc[3][0]};
        const double sum = warp_reduce_n<4>(flat);   // lane l: row rl + l mod 4
        if (lane < 4 && rl + lane < bw) U0[r0 + rl + lane] -= sum;
      } else {
        static_assert(RMAX == 8, "four rows × eight vectors fill the 32 lanes");
        double flat[32];   // value i·8 + e: row rl + i, vector e
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int e = 0; e < 8; ++e) flat[i * 8 + e] = acc[i][e];
        const double sum = warp_reduce32(flat);
        const int li = lane / 8, le = lane % 8;
        if (le < R && rl + li < bw) U0[le * ldu + r0 + rl + li] -= sum;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < RMAX; ++e) acc[i][e] = 0.0;
    const bool cached = st.I < dv;
    if (!cached && warp == 0) invert_tile(S, invd + r0, D);
    __syncthreads();
    if (!cached) store_inverse(D, dc, st.I);
    if (warp < R) {   // u ← D_I w, lane r one row (D_I[r][c] from D_Iᵀ or D)
      double* u = U0 + warp * ldu + r0;
      double a[4] = {0.0, 0.0, 0.0, 0.0};
      if (cached) {
#pragma unroll
        for (int c = 0; c < kSB; ++c)
          if (c < bw) a[c & 3] = fma(S[c * kSB + lane], u[c], a[c & 3]);
      } else {
#pragma unroll
        for (int c = 0; c < kSB; ++c)
          if (c < bw) a[c & 3] = fma(D[lane][c], u[c], a[c & 3]);
      }
      __syncwarp();
      if (lane < bw) u[lane] = (a[0] + a[1]) + (a[2] + a[3]);
    }
  });
  if (threadIdx.x == 0 && dv >= I0) *dvalid = max(dv, (n - 1) / kSB + 1);
  __syncthreads();
}

// v ← L⁻ᵀ v on rows [0, n), v in shared memory.  Per row block from the
// bottom: warp 0 multiplies the block by D_Iᵀ, then each off-diagonal tile
// takes the block's contribution, two warps per tile (sixteen columns each,
// the lane halves on sixteen rows each, added by one shuffle).  Every block
// inverse is valid afterwards.
__device__ void stream_backward(const double* Lt, double* dc, int* dvalid, const double* invd, double* v, int n,
                                double* ring, DiagTile* D) {
  if (n <= 0) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int dv = *dvalid;
  const int I1 = (n - 1) / kSB;
  stream_steps(Lt, dc, dv, false, ring, BackwardSteps{I1, -1}, [&](const Step& st, const double* S) {
    const int r0 = kSB * st.I, bw = min(kSB, n - r0);
    if (st.diag) {
      const bool cached = st.I < dv;
      if (!cached) {
        if (warp == 0) invert_tile(S, invd + r0, D);
        __syncthreads();
        store_inverse(D, dc, st.I);
      }
      if (warp == 0) {   // x = D_Iᵀ v_I, lane c one entry
        double a[4] = {0.0, 0.0, 0.0, 0.0};
        if (cached) {
#pragma unroll
          for (int r = 0; r < kSB; ++r)
            if (r < bw) a[r & 3] = fma(S[r * kSB + lane], v[r0 + r], a[r & 3]);
        } else {
#pragma unroll
          for (int r = 0; r < kSB; ++r)
            if (r < bw) a[r & 3] = fma(D[r][lane], v[r0 + r], a[r & 3]);
        }
        __syncwarp();
        if (lane < bw) v[r0 + lane] = (a[0] + a[1]) + (a[2] + a[3]);
      }
      return;
    }
    const int j = warp >> 1;
    if (j < st.nt) {
      const int c = 16 * (warp & 1) + (lane & 15), rh = 16 * (lane >> 4);
      const double* T = S + j * kTileElems;
      double a[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = rh + i;
        if (r < bw) a[i & 3] = fma(T[r * kSB + c], v[r0 + r], a[i & 3]);
      }
      double s = (a[0] + a[1]) + (a[2] + a[3]);
      s += __shfl_xor_sync(0xffffffffu, s, 16);
      if (lane < 16) v[kSB * (st.J0 + j) + c] -= s;
    }
  });
  if (threadIdx.x == 0) *dvalid = max(dv, I1 + 1);
  __syncthreads();
}

// Us[e·ldu + q] = G[add_e, P_q] for e < R, q < np (all loads of a thread
// issued before its stores, eight at a time).
__device__ __forceinline__ void gather_new_rows(double* Us, int ldu, const double* G, int t, const int* addl, int R,
                                                const int* P, int np) {
  const int total = R * np;
  for (int i0 = threadIdx.x; i0 < total; i0 += 8 * blockDim.x) {
    double v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < total) {
        const int e = i / np, q = i - e * np;
        v[u] = G[(int64_t)addl[e] * t + P[q]];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < total) {
        const int e = i / np, q = i - e * np;
        Us[e * ldu + q] = v[u];
      }
    }
  }
}

// Deletes position q from the packed factor L of an np×np matrix (all
// threads of the block).  Writing L = [L11 · ·; l21ᵀ l22 ·; L31 l32 L33],
// the matrix without row and column q has the factor [L11 ·; L31 L̃33] with
// L̃33 L̃33ᵀ = L33 L33ᵀ + l32 l32ᵀ: the classic rank-one Cholesky update,
// one plane rotation per column of L33.  The rotations are formed sixteen
// columns at a time by one warp on the diagonal block, then applied by every
// thread to one trailing row at a time.  Last, the rows below q move up one
// slot and lose column q.  xv (m doubles) and rot (48 doubles) are scratch.
constexpr int kRotBlock = 16;
constexpr int kMoveRegs = 8;

__device__ __forceinline__ int tri_row(int64_t e) {
  // row of packed index e (e < 2^23: exact in fp32, then corrected)
  int r = (int)((sqrtf(8.0f * (float)e + 1.0f) - 1.0f) * 0.5f);
  while (tri(r + 1, 0) <= e) ++r;
  while (tri(r, 0) > e) --r;
  return r;
}

__device__ void factor_remove(double* L, double* invd, double* xv, double* rot, int q, int np) {
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int m = np - 1 - q;   // trailing rows: old indices o .. np-1
  const int o = q + 1;
  for (int a = tid; a < m; a += nthr) xv[a] = L[tri(o + a, q)];
  __syncthreads();
  for (int J = 0; J < m; J += kRotBlock) {
    const int jw = min(kRotBlock, m - J);
    if (warp == 0) {
      // lane e holds trailing row J+e, columns J .. J+e
      const bool mine = lane < jw;
      double* row = L + tri(o + J + (mine ? lane : 0), o + J);
      double v[kRotBlock];
#pragma unroll
      for (int c = 0; c < kRotBlock; ++c) v[c] = (mine && c <= lane) ? row[c] : 0.0;
      double xr = mine ? xv[J + lane] : 0.0;
#pragma unroll
      for (int k = 0; k < kRotBlock; ++k) {
        if (k < jw) {
          const double lkk = __shfl_sync(0xffffffffu, v[k], k);
          const double xk = __shfl_sync(0xffffffffu, xr, k);
          // r = sqrt(lkk² + xk²) through one reciprocal square root and one
          // reciprocal (entries of a Cholesky factor of a Gram matrix of
          // features in [0, 1]: no overflow); c = r/lkk, sn = xk/lkk, ic = lkk/r
          const double rr = fma(lkk, lkk, xk * xk);
          const double irr = rsqrt(rr), il = 1.0 / lkk;
          const double r = rr * irr;
          const double c = r * il, sn = xk * il, ic = lkk * irr;
          if (lane == k) v[k] = r;
          if (mine && lane > k) {
            v[k] = (v[k] + sn * xr) * ic;
            xr = c * xr - sn * v[k];
          }
          if (lane == 0) { rot[3 * k] = c; rot[3 * k + 1] = sn; rot[3 * k + 2] = ic; }
        }
      }
      if (mine) {
#pragma unroll
        for (int c = 0; c < kRotBlock; ++c)
          if (c <= lane) row[c] = v[c];
      }
    }
    __syncthreads();
    for (int a = J + jw + tid; a < m; a += nthr) {
      double* row = L + tri(o + a, o + J);
      double v[kRotBlock];
#pragma unroll
      for (int c = 0; c < kRotBlock; ++c) v[c] = c < jw ? row[c] : 0.0;
      double xa = xv[a];
#pragma unroll
      for (int k = 0; k < kRotBlock; ++k) {
        if (k < jw) {
          v[k] = (v[k] + rot[3 * k + 1] * xa) * rot[3 * k + 2];
          xa = rot[3 * k] * xa - rot[3 * k + 1] * v[k];
        }
      }
#pragma unroll
      for (int c = 0; c < kRotBlock; ++c)
        if (c < jw) row[c] = v[c];
      xv[a] = xa;
    }
    __syncthreads();
  }
  // New row r >= q is old row r+1 without column q; it fills exactly the
  // slot of old row r, so the move runs in chunks, each read before written.
  const int64_t f0 = tri(q, 0), f1 = tri(np - 1, 0);
  for (int64_t e0 = f0; e0 < f1; e0 += (int64_t)nthr * kMoveRegs) {
    double v[kMoveRegs];
#pragma unroll
    for (int u = 0; u < kMoveRegs; ++u) {
      const int64_t e = e0 + (int64_t)u * nthr + tid;
      if (e < f1) {
        const int r = tri_row(e);
        const int c = (int)(e - tri(r, 0));
        v[u] = L[tri(r + 1, c + (c >= q))];
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kMoveRegs; ++u) {
      const int64_t e = e0 + (int64_t)u * nthr + tid;
      if (e < f1) L[e] = v[u];
    }
    __syncthreads();
  }
  for (int r = q + tid; r < np - 1; r += nthr) invd[r] = 1.0 / L[tri(r, r)];
  __syncthreads();
}

// factor_remove for a tiled factor (same steps; elements addressed by tile).
// The move runs over the new factor's tiles from row block q/32 on, in
// storage order: every moved element's source lies after its destination,
// and the sources of later chunks after every destination of earlier ones,
// so each chunk is read before it is written.
__device__ void factor_remove_tiled(double* L, double* invd, double* xv, double* rot, int q, int np) {
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int m = np - 1 - q;
  const int o = q + 1;
  for (int a = tid; a < m; a += nthr) xv[a] = L[tl(o + a, q)];
  __syncthreads();
  for (int J = 0; J < m; J += kRotBlock) {
    const int jw = min(kRotBlock, m - J);
    if (warp == 0) {
      const bool mine = lane < jw;
      const int rr = o + J + (mine ? lane : 0);
      double v[kRotBlock];
#pragma unroll
      for (int c = 0; c < kRotBlock; ++c) v[c] = (mine && c <= lane) ? L[tl(rr, o + J + c)] : 0.0;
      double xr = mine ? xv[J + lane] : 0.0;
#pragma unroll
      for (int k = 0; k < kRotBlock; ++k) {
        if (k < jw) {
          const double lkk = __shfl_sync(0xffffffffu, v[k], k);
          const double xk = __shfl_sync(0xffffffffu, xr, k);
          // r = sqrt(lkk² + xk²) through one reciprocal square root and one
          // reciprocal (entries of a Cholesky factor of a Gram matrix of
          // features in [0, 1]: no overflow); c = r/lkk, sn = xk/lkk, ic = lkk/r
          const double rr = fma(lkk, lkk, xk * xk);
          const double irr = rsqrt(rr), il = 1.0 / lkk;
          const double r = rr * irr;
          const double c = r * il, sn = xk * il, ic = lkk * irr;
          if (lane == k) v[k] = r;
          if (mine && lane > k) {
            v[k] = (v[k] + sn * xr) * ic;
            xr = c * xr - sn * v[k];
          }
          if (lane == 0) { rot[3 * k] = c; rot[3 * k + 1] = sn; rot[3 * k + 2] = ic; }
        }
      }
      if (mine) {
#pragma unroll
        for (int c = 0; c < kRotBlock; ++c)
          if (c <= lane) L[tl(rr, o + J + c)] = v[c];
      }
    }
    __syncthreads();
    for (int a = J + jw + tid; a < m; a += nthr) {
      const int rr = o + a;
      double v[kRotBlock];
#pragma unroll
      for (int c = 0; c < kRotBlock; ++c) v[c] = c < jw ? L[tl(rr, o + J + c)] : 0.0;
      double xa = xv[a];
#pragma unroll
      for (int k = 0; k < kRotBlock; ++k) {
        if (k < jw) {
          v[k] = (v[k] + rot[3 * k + 1] * xa) * rot[3 * k + 2];
          xa = rot[3 * k] * xa - rot[3 * k + 1] * v[k];
        }
      }
#pragma unroll
      for (int c = 0; c < kRotBlock; ++c)
        if (c < jw) L[tl(rr, o + J + c)] = v[c];
      xv[a] = xa;
    }
    __syncthreads();
  }
  // new (r, c) = old (r + 1, c + [c >= q]) for q <= r < np − 1, c <= r: the
  // new factor's tiles from row block q/32 on, two per chunk, in storage order
  const int nbn = (np - 1 + kSB - 1) / kSB;
  int I = q >> 5, J = 0;
  while (I < nbn) {
    int ti[2], tj[2];
    ti[0] = I;
    tj[0] = J;
    if (++J > I) { ++I; J = 0; }
    const bool two = I < nbn;
    ti[1] = I;
    tj[1] = J;
    if (two && ++J > I) { ++I; J = 0; }
    double v[2][kTileElems / kNnlsThreads];
    bool live[2][kTileElems / kNnlsThreads];
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int u = 0; u < kTileElems / kNnlsThreads; ++u) {
        const int l = tid + u * kNnlsThreads;
        const int r = kSB * ti[k] + (l >> 5), c = kSB * tj[k] + (l & 31);
        live[k][u] = (k == 0 || two) && r >= q && r < np - 1 && c <= r;
        v[k][u] = live[k][u] ? L[tl(r + 1, c + (c >= q))] : 0.0;
      }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int u = 0; u < kTileElems / kNnlsThreads; ++u)
        if (live[k][u]) L[tile_at(ti[k], tj[k]) + tid + u * kNnlsThreads] = v[k][u];
    __syncthreads();
  }
  for (int r = q + tid; r < np - 1; r += nthr) invd[r] = 1.0 / L[tl(r, r)];
  __syncthreads();
}

// l_in_smem_max: heads with t at or below it keep the factor in shared
// memory.  ucap > 0: the others stream their solves (ring and up to ucap new
// rows of t doubles in shared memory after the vectors); 0: they read the
// factor in place.
__global__ void __launch_bounds__(kNnlsThreads) k_nnls(Problem p, Work w, int pass, int l_in_smem_max, int ucap) {
  chain_wait();
  extern __shared__ __align__(16) unsigned char smem[];
  const int h = w.order[blockIdx.x];
  const int t = w.t[h];
  int s0, s1;
  pass_range(p, t, pass, s0, s1);
  if (s0 >= s1) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int np_old = w.np[h];
  const int64_t base = w.cu_t[h];
  const int64_t gbase = w.cu_t2[h];
  const double* G = w.G + gbase;
  const double* b = w.bvec + base;

  double* x = reinterpret_cast<double*>(smem);   // pick-slot indexed weights
  double* z = x + t;                             // factor-position indexed solve buffer
  double* g = z + t;                             // scaled gradient
  double* invd = g + t;                          // 1 / L_qq
  double* yv = invd + t;                         // forward solve L⁻¹ b_P, valid below ctl[10]
  double* red = yv + t;                          // 64 doubles
  DiagTile* D = reinterpret_cast<DiagTile*>(red + 64);              // solve scratch
  int* ctl = reinterpret_cast<int*>(red + 64 + kSB * (kSB + 1));    // 16 ints
  uint64_t* lbar = reinterpret_cast<uint64_t*>(ctl + 16);            // 16 bytes
  int* P = ctl + 20;
  int* inP = P + t;
  int* blocked = inP + t;
  int* add = blocked + t;
  int* cand = add + t;
  const bool l_smem = t <= l_in_smem_max;
  double* Lg = w.L + gbase;
  double* L = l_smem ? reinterpret_cast<double*>(smem + nnls_vec_bytes(t)) : Lg;
  const bool streamed = !l_smem && ucap > 0;
  // streamed heads: the tiled factor (16-byte aligned inside the head's t×t
  // region), its cached block inverses, the copy ring and ucap new rows of t
  double* Lt = w.L + ((gbase + 1) & ~(int64_t)1);
  double* dc = dinv_cache(w, h);
  double* ring = reinterpret_cast<double*>(smem + nnls_vec_bytes(t));
  double* Us = ring + kSlots * kSlotDoubles;
  // the factor kept in shared memory arrives by one bulk copy (16-byte
  // aligned at both ends; rounding the size up reads at most one double past
  // the factor, still inside the head's t×t region and the shared buffer)
  const uint32_t lbytes = l_smem ? (uint32_t)((tri(np_old, 0) * 8 + 15) & ~(int64_t)15) : 0u;
  // ctl: 0 np, 1 nadd, 2 single mode, 4 argmin, 5 nneg, 7 ncand, 9 removed count, 10 valid y rows,
  //      11 first factor row that differs from the stored factor, 12 leading row blocks whose
  //      cached inverse is valid (streamed heads)
  const int maxit = p.nnls_max_iter > 0 ? p.nnls_max_iter : 3 * t + 50;
  const double mnorm = sqrt(w.mm[h]);
  auto diag = [&](int l) { return G[(int64_t)l * t + l]; };

  for (int l = tid; l < s1; l += blockDim.x) {
    x[l] = l < s0 ? w.w[base + l] : 0.0;
    inP[l] = 0;
    blocked[l] = 0;
  }
  if (lbytes > 0 && tid == 0) {
    mbar_init(lbar, 1);
    mbar_init_fence();
    mbar_expect_tx(lbar, lbytes);
    for (uint32_t o = 0; o < lbytes; o += kBulkChunk)
      bulk_load(reinterpret_cast<char*>(L) + o, reinterpret_cast<const char*>(Lg) + o,
                lbytes - o < kBulkChunk ? lbytes - o : kBulkChunk, lbar);
  }
  for (int q = tid; q < np_old; q += blockDim.x) P[q] = w.plist[base + q];
  const int ylen0 = min(w.ylen[h], np_old);
  for (int q = tid; q < ylen0; q += blockDim.x) yv[q] = w.ycache[base + q];
  if (tid == 0) { ctl[0] = np_old; ctl[2] = 0; ctl[10] = ylen0; ctl[11] = np_old; ctl[12] = w.dvalid[h]; }
  __syncthreads();   // the barrier is initialised before anyone waits on it
  const bool landed = lbytes == 0 || mbar_wait_bounded(lbar, 0, p.wait_cycles);
  if (__syncthreads_or(!landed)) {
    // the copy did not land: flag the head, let it drain (full budget), leave
    // everything as it was; the head's outputs are not valid (AM_ERR_TIMEOUT)
    if (tid == 0) record_status(w.status + h, AM_ERR_TIMEOUT);
    mbar_wait_bounded(lbar, 0, kBulkWaitCycles);
    return;
  }
  for (int q = tid; q < np_old; q += blockDim.x) {
    inP[P[q]] = 1;
    invd[q] = 1.0 / (streamed ? Lt[tl(q, q)] : L[tri(q, q)]);
  }
  __syncthreads();

  // Append add[0..nadd) to the factor as a block; variables whose Schur
  // pivot is too small are blocked and the block is redone without them.
  auto block_append = [&]() {
    for (;;) {
      const int np = ctl[0], k = ctl[1];
      if (k == 0) return;
      // right-hand sides G[add_e, P] into the new packed rows
      for (int e = warp; e < k; e += nw) {
        double* row = L + tri(np + e, 0);
        const double* Ge = G + (int64_t)add[e] * t;
        for (int q = lane; q < np; q += 32) row[q] = Ge[P[q]];
      }
      __syncthreads();
      for (int e0 = 0; e0 < k; e0 += kMaxRhs) {
        const int R = min(kMaxRhs, k - e0);
        double* U[kMaxRhs];
#pragma unroll
        for (int e = 0; e < kMaxRhs; ++e) U[e] = L + tri(np + e0 + min(e, R - 1), 0);
        block_forward(L, invd, U, R, 0, np, D);
      }
      // Schur complement of the new block (lower triangle)
      for (int pr = warp; pr < k * (k + 1) / 2; pr += nw) {
        int e = 0;
        while ((e + 1) * (e + 2) / 2 <= pr) ++e;
        const int f = pr - e * (e + 1) / 2;
        const double* re = L + tri(np + e, 0);
        const double* rf = L + tri(np + f, 0);
        double acc = 0.0;
        for (int q = lane; q < np; q += 32) acc += re[q] * rf[q];
        acc = warp_sum(acc);
        if (lane == 0) L[tri(np + e, np + f)] = G[(int64_t)add[e] * t + add[f]] - acc;
      }
      __syncthreads();
      // Cholesky of the k×k Schur block: lane e owns new row e (lane 0 alone
      // for k > 32); a pivot at or below 1e-13·G_ll blocks that variable
      if (warp == 0) {
        int failed = 0;
        const bool wide = k <= 32;
        const double dg = wide && lane < k ? diag(add[lane]) : 0.0;   // G_ll of new row `lane`
        for (int f = 0; f < k; ++f) {
          const double piv = L[tri(np + f, np + f)];
          const double gff = wide ? __shfl_sync(0xffffffffu, dg, f) : diag(add[f]);
          if (!(piv > 1e-13 * gff)) {
            if (lane == 0) blocked[add[f]] = 1;
            failed = 1;
            break;
          }
          const double lff = sqrt(piv), il = 1.0 / lff;
          __syncwarp();
          if (lane == 0) { L[tri(np + f, np + f)] = lff; invd[np + f] = il; }
          if (wide) {
            const int e = lane;
            if (e > f && e < k) L[tri(np + e, np + f)] *= il;
            __syncwarp();
            if (e > f && e < k) {
              const double lef = L[tri(np + e, np + f)];
              for (int q = f + 1; q <= e; ++q) L[tri(np + e, np + q)] -= lef * L[tri(np + q, np + f)];
            }
          } else if (lane == 0) {
            for (int e = f + 1; e < k; ++e) L[tri(np + e, np + f)] *= il;
            for (int e = f + 1; e < k; ++e) {
              const double lef = L[tri(np + e, np + f)];
              for (int q = f + 1; q <= e; ++q) L[tri(np + e, np + q)] -= lef * L[tri(np + q, np + f)];
            }
          }
          __syncwarp();
        }
        if (lane == 0) {
          if (failed) {
            int kk = 0;
            for (int e = 0; e < k; ++e)
              if (!blocked[add[e]]) add[kk++] = add[e];
            ctl[1] = kk;
          } else {
            for (int e = 0; e < k; ++e) {
              P[np + e] = add[e];
              inP[add[e]] = 1;
            }
            ctl[0] = np + k;
            ctl[1] = 0;
          }
        }
      }
      __syncthreads();
      if (ctl[1] == 0) return;
    }
  };

  // Streamed heads: the same block append on the tiled factor, with the
  // forward solves of the new rows streamed (kStreamRhs vectors per read of
  // the factor) and, for at most ucap new rows, the rows, their Schur block
  // and its Cholesky in shared memory until the block is accepted.
  auto append_streamed = [&]() {
    for (;;) {
      const int np = ctl[0], k = ctl[1];
      if (k == 0) return;
      const bool one = k <= ucap;
      const int chunk = one ? k : ucap;
      for (int e0 = 0; e0 < k; e0 += chunk) {
        const int rows = min(chunk, k - e0);
        gather_new_rows(Us, t, G, t, add + e0, rows, P, np);
        __syncthreads();
        for (int c0 = 0; c0 < rows; c0 += kStreamRhs) {
          const int R = min(kStreamRhs, rows - c0);
          if (R == 1)
            stream_forward<1>(Lt, dc, &ctl[12], invd, Us + c0 * t, t, 1, 0, np, ring, D);
          else
            stream_forward<kStreamRhs>(Lt, dc, &ctl[12], invd, Us + c0 * t, t, R, 0, np, ring, D);
        }
        if (!one) {
          for (int i = tid; i < rows * np; i += blockDim.x) {
            const int e = i / np, q = i - e * np;
            Lt[tl(np + e0 + e, q)] = Us[e * t + q];
          }
          __syncthreads();
        }
      }
      // Schur complement of the new block: in the diagonal tile for k <= 32,
      // else in the factor
      const bool small = k <= kSB;
      for (int pr = warp; pr < k * (k + 1) / 2; pr += nw) {
        int e = 0;
        while ((e + 1) * (e + 2) / 2 <= pr) ++e;
        const int f = pr - e * (e + 1) / 2;
        double a4[4] = {0.0, 0.0, 0.0, 0.0};
        for (int q0 = lane; q0 < np; q0 += 128) {
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const int q = q0 + 32 * s;
            if (q < np) {
              const double xe = one ? Us[e * t + q] : Lt[tl(np + e, q)];
              const double xf = one ? Us[f * t + q] : Lt[tl(np + f, q)];
              a4[s] = fma(xe, xf, a4[s]);
            }
          }
        }
        const double acc = warp_sum((a4[0] + a4[1]) + (a4[2] + a4[3]));
        if (lane == 0) {
          const double sv = G[(int64_t)add[e] * t + add[f]] - acc;
          if (small)
            D[e][f] = sv;
          else
            Lt[tl(np + e, np + f)] = sv;
        }
      }
      __syncthreads();
      // Cholesky of the Schur block (lane e owns new row e; lane 0 alone past
      // 32 rows); a pivot at or below 1e-13·G_ll blocks that variable
      if (warp == 0) {
        int failed = 0;
        if (small) {
          const double dg = lane < k ? diag(add[lane]) : 0.0;
          for (int f = 0; f < k; ++f) {
            const double piv = D[f][f];
            const double gff = __shfl_sync(0xffffffffu, dg, f);
            if (!(piv > 1e-13 * gff)) {
              if (lane == 0) blocked[add[f]] = 1;
              failed = 1;
              break;
            }
            const double lff = sqrt(piv), il = 1.0 / lff;
            __syncwarp();
            if (lane == f) D[f][f] = lff;
            if (lane > f && lane < k) D[lane][f] *= il;
            __syncwarp();
            if (lane > f && lane < k) {
              const double lef = D[lane][f];
              for (int q = f + 1; q <= lane; ++q) D[lane][q] -= lef * D[q][f];
            }
            __syncwarp();
          }
        } else if (lane == 0) {
          for (int f = 0; f < k; ++f) {
            const double piv = Lt[tl(np + f, np + f)];
            if (!(piv > 1e-13 * diag(add[f]))) {
              blocked[add[f]] = 1;
              failed = 1;
              break;
            }
            const double lff = sqrt(piv), il = 1.0 / lff;
            Lt[tl(np + f, np + f)] = lff;
            invd[np + f] = il;
            for (int e = f + 1; e < k; ++e) Lt[tl(np + e, np + f)] *= il;
            for (int e = f + 1; e < k; ++e) {
              const double lef = Lt[tl(np + e, np + f)];
              for (int q = f + 1; q <= e; ++q) Lt[tl(np + e, np + q)] -= lef * Lt[tl(np + q, np + f)];
            }
          }
        }
        failed = __shfl_sync(0xffffffffu, failed, 0);
        if (lane == 0) {
          if (failed) {
            int kk = 0;
            for (int e = 0; e < k; ++e)
              if (!blocked[add[e]]) add[kk++] = add[e];
            ctl[1] = kk;
          } else {
            for (int e = 0; e < k; ++e) {
              P[np + e] = add[e];
              inP[add[e]] = 1;
            }
            ctl[0] = np + k;
            ctl[1] = 0;
            ctl[12] = min(ctl[12], np / kSB);   // the block holding row np changed
          }
        }
      }
      __syncthreads();
      const bool ok = ctl[0] != np;
      if (ok && small) {   // the accepted block goes into the factor
        if (one)
          for (int i = tid; i < k * np; i += blockDim.x) {
            const int e = i / np, q = i - e * np;
            Lt[tl(np + e, q)] = Us[e * t + q];
          }
        for (int i = tid; i < k * k; i += blockDim.x) {
          const int e = i / k, f = i - e * k;
          if (f <= e) Lt[tl(np + e, np + f)] = D[e][f];
        }
        for (int e = tid; e < k; e += blockDim.x) invd[np + e] = 1.0 / D[e][e];
      }
      __syncthreads();
      if (ok || ctl[1] == 0) return;
    }
  };

  int iter = 0;
  bool converged = false;
  for (int outer = 0; outer <= maxit; ++outer) {
    // ---- candidates and their scaled gradients b_l − G[l, P] x_P ----
    const int np = ctl[0];
    for (int q = tid; q < np; q += blockDim.x) z[q] = x[P[q]];
    if (warp == 0) {
      int nc = 0;
      for (int l0 = 0; l0 < s1; l0 += 32) {
        const int l = l0 + lane;
        const bool c = l < s1 && !inP[l] && !blocked[l];
        const unsigned msk = __ballot_sync(0xffffffffu, c);
        if (c) cand[nc + __popc(msk & ((1u << lane) - 1))] = l;
        nc += __popc(msk);
      }
      if (lane == 0) ctl[7] = nc;
    }
    __syncthreads();
    const int nc = ctl[7];
    for (int ci = warp; ci < nc; ci += nw) {
      const int l = cand[ci];
      const double* Gl = G + (int64_t)l * t;
      const double dl = lane == 0 ? diag(l) : 0.0, bl = lane == 0 ? b[l] : 0.0;   // in flight with the row
      double a4[4] = {0.0, 0.0, 0.0, 0.0};
      for (int q0 = lane; q0 < np; q0 += 128) {
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int q = q0 + 32 * s;
          if (q < np) a4[s] = fma(Gl[P[q]], z[q], a4[s]);
        }
      }
      const double acc = warp_sum((a4[0] + a4[1]) + (a4[2] + a4[3]));
      if (lane == 0) g[l] = dl > 0.0 ? (bl - acc) / (sqrt(dl) * mnorm) : -INFINITY;
    }
    __syncthreads();
    if (warp == 0) {
      // enter while g_l / (‖φ_l‖·‖m‖) > 1e-12; the rounding of b_l − G_l x
      // in fp64 stays near 1e-14 on this scale
      const double tol = 1e-12;
      int nadd = 0;
      if (ctl[2]) {                                    // single mode: argmax only
        double bv = tol;
        int bi = -1;
        for (int ci = lane; ci < nc; ci += 32) {
          const int l = cand[ci];
          if (g[l] > bv || (g[l] == bv && bi >= 0 && l < bi)) { bv = g[l]; bi = l; }
        }
        for (int o = 16; o; o >>= 1) {
          const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
          const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (ov > bv || (ov == bv && oi >= 0 && (bi < 0 || oi < bi))) { bv = ov; bi = oi; }
        }
        if (lane == 0 && bi >= 0) { add[0] = bi; nadd = 1; }
        nadd = __shfl_sync(0xffffffffu, nadd, 0);
      } else {
        for (int c0 = 0; c0 < nc; c0 += 32) {
          const int ci = c0 + lane;
          const bool c = ci < nc && g[cand[ci]] > tol;
          const unsigned msk = __ballot_sync(0xffffffffu, c);
          if (c) add[nadd + __popc(msk & ((1u << lane) - 1))] = cand[ci];
          nadd += __popc(msk);
        }
      }
      if (lane == 0) ctl[1] = nadd;
    }
    __syncthreads();
    if (ctl[1] == 0) { converged = true; break; }
    if (streamed)
      append_streamed();
    else
      block_append();

    // ---- inner loop: solve on P, step back toward feasibility ----
    bool abort = false;
    for (;;) {
      if (++iter > maxit) { abort = true; break; }
      // streamed heads restart the extension at a row-block boundary
      const int npc = ctl[0], y0 = streamed ? ctl[10] / kSB * kSB : ctl[10];
      // z = y on the cached rows; the forward solve extends it over the rest
      for (int q = tid; q < npc; q += blockDim.x) z[q] = q < y0 ? yv[q] : b[P[q]];
      __syncthreads();
      if (streamed) {
        stream_forward<1>(Lt, dc, &ctl[12], invd, z, 0, 1, y0 / kSB, npc, ring, D);
      } else {
        double* U[kMaxRhs] = {z, z, z, z, z, z, z, z};
        block_forward(L, invd, U, 1, y0, npc, D);
      }
      for (int q = y0 + tid; q < npc; q += blockDim.x) yv[q] = z[q];
      if (tid == 0) ctl[10] = npc;
      if (streamed)
        stream_backward(Lt, dc, &ctl[12], invd, z, npc, ring, D);
      else
        block_backward(L, invd, z, npc, D);
      double best = INFINITY;
      int bq = -1, nneg = 0;
      for (int q = tid; q < npc; q += blockDim.x) {
        const double zq = z[q];
        if (!(zq > 0.0)) {
          ++nneg;
          const double xq = x[P[q]];
          const double den = xq - zq;
          const double ratio = den > 0.0 ? xq / den : 0.0;
          if (ratio < best || (ratio == best && q < bq)) { best = ratio; bq = q; }
        }
      }
      for (int o = 16; o; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int oq = __shfl_xor_sync(0xffffffffu, bq, o);
        nneg += __shfl_xor_sync(0xffffffffu, nneg, o);
        if (ov < best || (ov == best && oq >= 0 && (bq < 0 || oq < bq))) { best = ov; bq = oq; }
      }
      if (tid == 0) ctl[5] = 0;
      __syncthreads();
      if (lane == 0) {
        red[warp] = best;
        reinterpret_cast<int*>(red + 16)[warp] = bq;
        atomicAdd(&ctl[5], nneg);
      }
      __syncthreads();
      if (tid == 0) {
        double bv = INFINITY;
        int bi = -1;
        for (int k = 0; k < nw; ++k) {
          const double v = red[k];
          const int qi = reinterpret_cast<int*>(red + 16)[k];
          if (qi >= 0 && (v < bv || (v == bv && qi < bi))) { bv = v; bi = qi; }
        }
        red[32] = bv;
        ctl[4] = bi;
      }
      __syncthreads();
      if (ctl[5] == 0) {   // all positive: accept
        for (int q = tid; q < npc; q += blockDim.x) x[P[q]] = z[q];
        __syncthreads();
        break;
      }
      const double alpha = red[32];
      if (alpha == 0.0) {
        // entering variables that will not grow: drop them
        if (tid == 0) {
          int kk = 0, nrm = 0;
          const bool single = ctl[2];
          for (int q = 0; q < npc; ++q) {
            const int l = P[q];
            if (!(z[q] > 0.0) && x[l] == 0.0) {
              inP[l] = 0;
              if (single) blocked[l] = 1;
              cand[nrm++] = q;
            } else {
              P[kk++] = l;
            }
          }
          ctl[0] = kk;
          ctl[2] = 1;
          ctl[9] = nrm;
        }
      } else {
        const int qmin = ctl[4];
        for (int q = tid; q < npc; q += blockDim.x) {
          const int l = P[q];
          double v = x[l] + alpha * (z[q] - x[l]);
          if (q == qmin) v = 0.0;
          x[l] = v;
        }
        __syncthreads();
        if (tid == 0) {
          int kk = 0, nrm = 0;
          for (int q = 0; q < npc; ++q) {
            const int l = P[q];
            if (x[l] <= 0.0) { inP[l] = 0; x[l] = 0.0; cand[nrm++] = q; }
            else P[kk++] = l;
          }
          ctl[0] = kk;
          ctl[9] = nrm;
        }
      }
      __syncthreads();
      // delete the leavers from the factor, last position first
      const int nrm = ctl[9];
      for (int i = nrm - 1, npr = ctl[0] + nrm; i >= 0; --i, --npr) {
        if (streamed)
          factor_remove_tiled(Lt, invd, g, red, cand[i], npr);
        else
          factor_remove(L, invd, g, red, cand[i], npr);
      }
      if (tid == 0 && nrm > 0) {
        ctl[10] = min(ctl[10], cand[0]);
        ctl[11] = min(ctl[11], cand[0]);
        ctl[12] = min(ctl[12], cand[0] / kSB);
      }
      __syncthreads();
    }
    if (abort) break;
  }
  __syncthreads();

  // ---- write back ----
  chain_release();
  const int npf = ctl[0];
  for (int l = tid; l < s1; l += blockDim.x) w.w[base + l] = inP[l] ? x[l] : 0.0;
  for (int q = tid; q < npf; q += blockDim.x) w.plist[base + q] = P[q];
  const int yl = ctl[10];
  for (int q = tid; q < yl; q += blockDim.x) w.ycache[base + q] = yv[q];
  if (l_smem) {   // rows above ctl[11] are unchanged since the load
    const int64_t e0 = tri(ctl[11], 0);
    copy_doubles(Lg + e0, L + e0, tri(npf, 0) - e0);
  }
  if (tid == 0) {
    w.np[h] = npf;
    w.ylen[h] = yl;
    w.dvalid[h] = ctl[12];
    w.nnls_refits[h] += 1;
    w.nnls_solves[h] += min(iter, maxit);
    if (!converged) record_status(w.status + h, AM_WARN_NOT_CONVERGED);
  }
}

// ------------------------------------------------------------ residual ----
// r = m − Φ_S w over all current picks; fp64 sums, fp32 store; partial ‖r‖².
// A block covers 32 float4 positions (128 queries) with sixteen thread
// groups, group g taking picks g, g + 16, ... (eight in flight); the groups'
// sums are combined in a fixed order, so the result is deterministic.
constexpr int kResidGroups = 16;   // pick groups per position
constexpr int kResidThreads = kResidPos * kResidGroups;
constexpr int kResidChunk = 512;   // picks staged in shared memory at a time

__global__ void __launch_bounds__(kResidThreads) k_resid(Problem p, Work w, int pass) {
  chain_wait();
  const int h = w.order[blockIdx.y];
  const int t = w.t[h];
  int s0, s1;
  pass_range(p, t, pass, s0, s1);
  if (s0 >= s1) return;
  __shared__ int sj[kResidChunk];
  __shared__ double sw[kResidChunk];
  __shared__ double4 part[kResidGroups - 1][kResidPos];
  __shared__ double scratch[33];
  const int64_t base = w.cu_t[h];
  const float* P0 = w.phiT + (int64_t)h * p.T * p.ldn;
  const int n4 = p.ldn >> 2;
  const int g = threadIdx.x / kResidPos, li = threadIdx.x % kResidPos;
  double rr = 0.0;
  for (int b4 = blockIdx.x * kResidPos; b4 < n4; b4 += gridDim.x * kResidPos) {
    const int i4 = b4 + li;
    const bool live = i4 < n4;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    if (live && g == 0) {
      const double2* m2 = reinterpret_cast<const double2*>(w.m + (int64_t)h * p.ldn);
      const double2 u = m2[2 * i4], v = m2[2 * i4 + 1];
      acc[0] = u.x; acc[1] = u.y; acc[2] = v.x; acc[3] = v.y;
    }
    for (int c0 = 0; c0 < s1; c0 += kResidChunk) {
      const int cn = min(kResidChunk, s1 - c0);
      __syncthreads();
      for (int q = threadIdx.x; q < cn; q += blockDim.x) {
        sj[q] = w.picks[base + c0 + q];
        sw[q] = w.w[base + c0 + q];
      }
      __syncthreads();
      if (live) {
        for (int q0 = g; q0 < cn; q0 += 8 * kResidGroups) {   // eight picks in flight
          float4 x[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * kResidGroups;
            x[u] = q < cn ? reinterpret_cast<const float4*>(P0 + (int64_t)sj[q] * p.ldn)[i4]
                          : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int q = q0 + u * kResidGroups;
            const double wl = q < cn ? sw[q] : 0.0;
            acc[0] -= x[u].x * wl; acc[1] -= x[u].y * wl; acc[2] -= x[u].z * wl; acc[3] -= x[u].w * wl;
          }
        }
      }
    }
    if (g > 0) part[g - 1][li] = make_double4(acc[0], acc[1], acc[2], acc[3]);
    __syncthreads();
    if (g == 0 && live) {
#pragma unroll
      for (int k = 0; k < kResidGroups - 1; ++k) {
        const double4 o = part[k][li];
        acc[0] += o.x; acc[1] += o.y; acc[2] += o.z; acc[3] += o.w;
      }
      float4 o = make_float4((float)acc[0], (float)acc[1], (float)acc[2], (float)acc[3]);
      reinterpret_cast<float4*>(w.r + (int64_t)h * p.ldn)[i4] = o;
      rr += acc[0] * acc[0] + acc[1] * acc[1] + acc[2] * acc[2] + acc[3] * acc[3];
    }
  }
  chain_release();
  rr = block_sum(rr, scratch);
  if (threadIdx.x == 0) w.rr_part[(int64_t)h * kRedBlocks + blockIdx.x] = rr;
}

__global__ void k_residual_norm(Problem p, Work w, int nblk, double* out) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= p.H) return;
  double s = 0.0;
  for (int k = 0; k < nblk; ++k) s += w.rr_part[(int64_t)h * kRedBlocks + k];
  out[h] = sqrt(s / w.mm[h]);
}


}  // namespace

// Dynamic shared memory of k_nnls: the vectors for max_t, plus the packed
// factor for the largest tl <= max_t that still fits; heads with t <= tl keep
// their factor in shared memory, larger ones in the workspace.
size_t nnls_smem_bytes(int max_t, int* l_in_smem_max) {
  const size_t vec = nnls_vec_bytes(max_t);
  int tl = 0;
  while (tl < max_t && vec + nnls_tri_bytes(tl + 1) <= kSmemCap) ++tl;
  *l_in_smem_max = tl;
  return vec + nnls_tri_bytes(tl);
}

cudaError_t launch_omp_init(const Problem& p, const Work& w, cudaStream_t s) {
  AM_LAUNCH(AM_STAGE_INIT, s, k_init<<<p.H, 256, 0, s>>>(p, w));
  return cudaGetLastError();
}

// New rows the streamed append keeps in shared memory next to the vectors
// for max_t and the ring (0: the factor does not stream).
int nnls_stream_rows(int max_t) {
  const size_t fixed = nnls_vec_bytes(max_t) + kRingBytes, row = (size_t)max_t * sizeof(double);
  if (fixed + row > kSmemCap) return 0;
  // the tiled factor must fit every streamed head's t×t region (t above the
  // shared-memory cap; it does for every t >= 102)
  int lcap = 0;
  nnls_smem_bytes(max_t, &lcap);
  for (int t = lcap + 1; t <= max_t; ++t)
    if (tiled_doubles(t) > (int64_t)t * t) return 0;
  const size_t r = (kSmemCap - fixed) / row;
  return r < (size_t)kAppendRows ? (int)r : kAppendRows;
}

int nnls_smem_cap(int max_t) {
  int lcap = 0;
  nnls_smem_bytes(max_t, &lcap);
  return lcap;
}

cudaError_t launch_omp_pass(const Problem& p, const Work& w, int pass, int active, int big, int small_tmax,
                            const CorrInputs& in, cudaStream_t s) {
  if (active <= 0) return cudaSuccess;
  if (p.select_highest) {
    // the picks were made up front; this pass feeds the next kR of them to the refit
  } else if (p.corr_bounded) {
    cudaError_t e = launch_corr_bounded(p, w, pass, active, s);   // selects too
    if (e != cudaSuccess) return e;
  } else {
    if (p.corr_recompute) {
      cudaError_t e = launch_corr_tc(p, in.Q, in.K, in.key_bias, w, pass, active, s);
      if (e != cudaSuccess) return e;
    } else {
      dim3 gc((p.T + kCorrRowsPerBlock - 1) / kCorrRowsPerBlock, active);
      AM_LAUNCH(AM_STAGE_CORR, s, k_corr<<<gc, 256, 0, s>>>(p, w, pass));
    }
    AM_LAUNCH(AM_STAGE_SELECT, s, k_select<<<active, 1024, 0, s>>>(p, w, pass));
  }
  const int s1max = (pass + 1) * p.kR < p.max_t ? (pass + 1) * p.kR : p.max_t;
  if (p.kR <= kGramMaxNew) {
    const int nslices = (p.ldn / 4 + kGramSlice4 - 1) / kGramSlice4;
    const int Z = nslices < kGramMaxSlices ? nslices : kGramMaxSlices;
    const int nb = p.kR <= 1 ? 1 : p.kR <= 2 ? 2 : p.kR <= 4 ? 4 : p.kR <= 8 ? 8 : 16;
    dim3 gg((s1max + 1 + kGramWarps - 1) / kGramWarps, Z, active);
    const int th = kGramWarps * 32;
    switch (nb) {
      case 1: AM_LAUNCH(AM_STAGE_GRAM, s, launch_chained(k_gram_tile<1>, gg, dim3(th), 0, s, p, w, pass)); break;
      case 2: AM_LAUNCH(AM_STAGE_GRAM, s, launch_chained(k_gram_tile<2>, gg, dim3(th), 0, s, p, w, pass)); break;
      case 4: AM_LAUNCH(AM_STAGE_GRAM, s, launch_chained(k_gram_tile<4>, gg, dim3(th), 0, s, p, w, pass)); break;
      case 8: AM_LAUNCH(AM_STAGE_GRAM, s, launch_chained(k_gram_tile<8>, gg, dim3(th), 0, s, p, w, pass)); break;
      default: AM_LAUNCH(AM_STAGE_GRAM, s, launch_chained(k_gram_tile<16>, gg, dim3(th), 0, s, p, w, pass)); break;
    }
  } else {
    dim3 gg(s1max, active);
    AM_LAUNCH(AM_STAGE_GRAM, s, k_gram<<<gg, 256, 0, s>>>(p, w, pass));
  }
  int lcap;
  size_t sm = nnls_smem_bytes(p.max_t, &lcap);
  cudaFuncSetAttribute(k_nnls, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemCap);
  // heads whose factor lives in the workspace (the vectors, the copy ring and
  // the new rows in shared memory); then the others with the factor
  if (big > 0) {
    const int ucap = nnls_stream_rows(p.max_t);
    const size_t sm_big =
        nnls_vec_bytes(p.max_t) + (ucap > 0 ? kRingBytes + (size_t)ucap * p.max_t * sizeof(double) : 0);
    AM_LAUNCH(AM_STAGE_NNLS, s,
              launch_chained(k_nnls, dim3(big), dim3(kNnlsThreads), sm_big, s, p, w, pass, 0, ucap));
  }
  if (active > big) {
    Work ws = w;
    ws.order = w.order + big;
    // shared memory for the largest factor of this launch, not of the whole call
    const size_t sm_small = nnls_vec_bytes(p.max_t) + nnls_tri_bytes(small_tmax < lcap ? small_tmax : lcap);
    AM_LAUNCH(AM_STAGE_NNLS, s,
              launch_chained(k_nnls, dim3(active - big), dim3(kNnlsThreads), sm_small < sm ? sm_small : sm, s, p,
                             ws, pass, lcap, 0));
  }
  dim3 gr(resid_blocks(p), active);
  AM_LAUNCH(AM_STAGE_RESID, s, launch_chained(k_resid, gr, dim3(kResidThreads), 0, s, p, w, pass));
  return cudaGetLastError();
}

cudaError_t launch_residual_norm(const Problem& p, const Work& w, double* out, cudaStream_t s) {
  AM_LAUNCH(AM_STAGE_RESID, s, k_residual_norm<<<(p.H + 127) / 128, 128, 0, s>>>(p, w, resid_blocks(p), out));
  return cudaGetLastError();
}

}  // namespace am
