// Bounded correlation pass: the OMP selection step j* = argmax_{j∉S} rᵀΦ_{:,j}
// ("Fast KV Compaction via Attention Matching": zhichai.net deep dive §1.6;
// k·R keys per pass under top-k batching with lazy refit, xinfinite.net
// article §3), evaluated exactly for only the keys that can win.
//
// For every key |c_j| = |rᵀΦ_{:,j}| <= ‖r‖₂·‖Φ_{:,j}‖₂ = B_j (Cauchy-Schwarz).
// One pass of kk = s1 − s0 picks per head:
//   1. k_probe   lists the unselected keys of largest bound: a histogram of B
//                over 1/16-octave bins, cut where at least kProbe keys lie at
//                or above;
//   2. k_rows    computes their c_j exactly: fp64 sums of the stored fp32
//                features times the stored fp32 residual;
//   3. k_extend  takes θ = the kk-th largest of those values and lists every
//                other unselected key with B_j·(1 + 1e-9) >= θ;
//   4. k_rows    computes those;
//   5. k_pick    appends the kk largest listed values (ties to the lower key).
// A key left off the list has c_j < θ while kk listed keys reach θ, so it is
// not among the kk largest: the picks are those of a full pass over all keys.
// The margin 1e-9 covers the rounding of the fp64 sums and norms (relative
// error below n·2^-53 for the sums, a few ulp for the norms).
//
// The column norms ‖Φ_{:,j}‖₂ are computed once per call (k_colnorm).
#include "am_internal.cuh"
#include "am_profile.cuh"
#include "am_linalg.cuh"

#include <float.h>

namespace am {
namespace {

constexpr int kProbe = 256;        // keys whose exact values set the first threshold
constexpr int kHistBins = 4096;    // float bits 30..19 of the bound: 1/16 octave
constexpr int kBoundThreads = 1024;
constexpr int kStage = 4096;       // listed values staged in shared memory
constexpr int kMaxKK = kMaxPicksPerPass;
constexpr double kBoundMargin = 1e-9;

__device__ __forceinline__ int bound_bin(double b) {
  return (int)(__float_as_uint((float)b) >> 19);   // b >= 0: monotone in b, < 4096
}

// (v, j) precedes (v', j') in pick order: larger value first, then lower key.
// A NaN value ranks below every number.
__device__ __forceinline__ bool ahead(double v, int j, double v2, int j2) {
  const bool n1 = v != v, n2 = v2 != v2;
  if (n1 || n2) return !n1 && n2 ? true : (n1 && !n2 ? false : j < j2);
  return v > v2 || (v == v2 && j < j2);
}

// ---------------------------------------------------------- column norms --
__global__ void __launch_bounds__(256) k_colnorm(Problem p, Work w) {
  const int h = blockIdx.y;
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= p.T) return;
  const float4* row = reinterpret_cast<const float4*>(w.phiT + ((int64_t)h * p.T + j) * p.ldn);
  const int n4 = p.ldn >> 2;
  double a0 = 0.0, a1 = 0.0;
  for (int i = lane; i < n4; i += 32) {
    const float4 x = __ldcs(row + i);
    a0 = fma((double)x.x, (double)x.x, a0);
    a1 = fma((double)x.y, (double)x.y, a1);
    a0 = fma((double)x.z, (double)x.z, a0);
    a1 = fma((double)x.w, (double)x.w, a1);
  }
  const double s = warp_sum(a0 + a1);
  if (lane == 0) w.cnorm[(int64_t)h * p.T + j] = sqrt(s);
}

// ----------------------------------------------------------------- probe --
__global__ void __launch_bounds__(kBoundThreads) k_probe(Problem p, Work w, int pass) {
  const int h = w.order[blockIdx.x];
  int s0, s1;
  pass_range(p, w.t[h], pass, s0, s1);
  if (s0 >= s1) return;
  __shared__ int hist[kHistBins];
  __shared__ int wsum[32];
  __shared__ double red[33];
  __shared__ int s_cut, s_n;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* r = w.r + (int64_t)h * p.ldn;
  double a = 0.0;
  for (int i = tid; i < p.ldn; i += blockDim.x) {
    const double v = r[i];
    a = fma(v, v, a);
  }
  const double rn = sqrt(block_sum(a, red));
  for (int b = tid; b < kHistBins; b += blockDim.x) hist[b] = 0;
  if (tid == 0) {
    w.rnorm[h] = rn;
    s_n = 0;
  }
  __syncthreads();
  const double* cn = w.cnorm + (int64_t)h * p.T;
  const uint8_t* sel = w.sel + (int64_t)h * p.T;
  for (int j = tid; j < p.T; j += blockDim.x)
    if (!sel[j]) atomicAdd(&hist[bound_bin(rn * cn[j])], 1);
  __syncthreads();
  // warp q sums bins [128q, 128q + 128); the cut is the highest bin with at
  // least kProbe keys at or above it (bin 0 when fewer keys are left)
  int cnt = 0;
  for (int b = warp * 128 + lane; b < warp * 128 + 128; b += 32) cnt += hist[b];
  for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) wsum[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int above = 0, cut = 0;
    for (int q = 31; q >= 0; --q) {
      if (above + wsum[q] >= kProbe) {
        for (int b = q * 128 + 127; b >= q * 128; --b) {
          above += hist[b];
          if (above >= kProbe) { cut = b; break; }
        }
        break;
      }
      above += wsum[q];
    }
    s_cut = cut;
  }
  __syncthreads();
  const int cut = s_cut;
  int32_t* list = w.clist + (int64_t)h * p.T;
  int32_t* stamp = w.cstamp + (int64_t)h * p.T;
  for (int j = tid; j < p.T; j += blockDim.x)
    if (!sel[j] && bound_bin(rn * cn[j]) >= cut) {
      list[atomicAdd(&s_n, 1)] = j;
      stamp[j] = pass + 1;
    }
  __syncthreads();
  if (tid == 0) {
    w.ccount[2 * h] = s_n;
    w.ccount[2 * h + 1] = s_n;
  }
}

// ------------------------------------------------------------ exact rows --
// c_j = Σ_i r_i Φ_ij for the listed keys [lo, hi) of each head (probe list
// when which = 0, its extension when which = 1): one warp per key, fp64 sums
// of exact fp32 products, four float4 loads per lane in flight.
__global__ void __launch_bounds__(256) k_rows(Problem p, Work w, int pass, int which) {
  const int h = w.order[blockIdx.y];
  int s0, s1;
  pass_range(p, w.t[h], pass, s0, s1);
  if (s0 >= s1) return;
  const int lo = which ? w.ccount[2 * h] : 0;
  const int hi = which ? w.ccount[2 * h + 1] : w.ccount[2 * h];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float4* r4 = reinterpret_cast<const float4*>(w.r + (int64_t)h * p.ldn);
  const int n4 = p.ldn >> 2;
  for (int q = lo + blockIdx.x * 8 + warp; q < hi; q += gridDim.x * 8) {
    const int j = w.clist[(int64_t)h * p.T + q];
    const float4* row = reinterpret_cast<const float4*>(w.phiT + ((int64_t)h * p.T + j) * p.ldn);
    double a[4] = {0.0, 0.0, 0.0, 0.0};
    for (int i0 = lane; i0 < n4; i0 += 32 * 4) {
      float4 x[4], y[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + 32 * u;
        x[u] = i < n4 ? __ldcs(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        y[u] = i < n4 ? __ldg(r4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[0] = fma((double)x[u].x, (double)y[u].x, a[0]);
        a[1] = fma((double)x[u].y, (double)y[u].y, a[1]);
        a[2] = fma((double)x[u].z, (double)y[u].z, a[2]);
        a[3] = fma((double)x[u].w, (double)y[u].w, a[3]);
      }
    }
    const double c = warp_sum((a[0] + a[1]) + (a[2] + a[3]));
    if (lane == 0) w.corrd[(int64_t)h * p.T + j] = c;
  }
}

// ------------------------------------------------------------ top-kk -----
// The kk <= 64 listed entries first in pick order, into ov/oi (shared).  Each
// warp finds the top kk of its share by kk rounds of "best entry after the
// previous one", then warp 0 does the same over the 32·kk warp winners.
// Values of the first kStage entries are staged in shared memory.
struct TopScratch {
  double v[kStage];
  int j[kStage];
  double cv[32 * kMaxKK];
  int cj[32 * kMaxKK];
};

__device__ void block_topk(const Problem& p, const Work& w, int h, int cnt, int kk, TopScratch& S, double* ov,
                           int* oi) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int32_t* list = w.clist + (int64_t)h * p.T;
  const double* cd = w.corrd + (int64_t)h * p.T;
  for (int q = tid; q < min(cnt, kStage); q += blockDim.x) {
    const int j = list[q];
    S.j[q] = j;
    S.v[q] = cd[j];
  }
  __syncthreads();
  auto entry = [&](int q, double& v, int& j) {
    if (q < kStage) { v = S.v[q]; j = S.j[q]; }
    else { j = list[q]; v = cd[j]; }
  };
  // per-warp winners over positions q ≡ warp (mod nw) ... strided by lanes
  const int per = (cnt + nw - 1) / nw;
  const int q0 = warp * per, q1 = min(cnt, q0 + per);
  double pv = INFINITY;
  int pj = -1;
  for (int k = 0; k < kk; ++k) {
    double bv = -INFINITY;
    int bj = INT_MAX;
    bool have = false;
    for (int q = q0 + lane; q < q1; q += 32) {
      double v;
      int j;
      entry(q, v, j);
      const bool after = pj < 0 || ahead(pv, pj, v, j);
      if (after && (!have || ahead(v, j, bv, bj))) { bv = v; bj = j; have = true; }
    }
    for (int o = 16; o; o >>= 1) {
      const double v2 = __shfl_xor_sync(0xffffffffu, bv, o);
      const int j2 = __shfl_xor_sync(0xffffffffu, bj, o);
      const int h2 = __shfl_xor_sync(0xffffffffu, (int)have, o);
      if (h2 && (!have || ahead(v2, j2, bv, bj))) { bv = v2; bj = j2; have = true; }
    }
    if (lane == 0) {
      S.cv[warp * kMaxKK + k] = have ? bv : -INFINITY;
      S.cj[warp * kMaxKK + k] = have ? bj : INT_MAX;
    }
    pv = bv;
    pj = have ? bj : INT_MAX;
  }
  __syncthreads();
  if (warp == 0) {
    pv = INFINITY;
    pj = -1;
    for (int k = 0; k < kk; ++k) {
      double bv = -INFINITY;
      int bj = INT_MAX;
      for (int e = lane; e < nw * kk; e += 32) {
        const double v = S.cv[(e / kk) * kMaxKK + e % kk];
        const int j = S.cj[(e / kk) * kMaxKK + e % kk];
        if (j == INT_MAX) continue;
        const bool after = pj < 0 || ahead(pv, pj, v, j);
        if (after && (bj == INT_MAX || ahead(v, j, bv, bj))) { bv = v; bj = j; }
      }
      for (int o = 16; o; o >>= 1) {
        const double v2 = __shfl_xor_sync(0xffffffffu, bv, o);
        const int j2 = __shfl_xor_sync(0xffffffffu, bj, o);
        if (j2 != INT_MAX && (bj == INT_MAX || ahead(v2, j2, bv, bj))) { bv = v2; bj = j2; }
      }
      if (lane == 0) { ov[k] = bv; oi[k] = bj; }
      pv = bv;
      pj = bj;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------- extension --
__global__ void __launch_bounds__(kBoundThreads) k_extend(Problem p, Work w, int pass) {
  extern __shared__ __align__(16) unsigned char smem[];
  TopScratch& S = *reinterpret_cast<TopScratch*>(smem);
  __shared__ double ov[kMaxKK];
  __shared__ int oi[kMaxKK];
  __shared__ int s_n;
  const int h = w.order[blockIdx.x];
  int s0, s1;
  pass_range(p, w.t[h], pass, s0, s1);
  if (s0 >= s1) return;
  const int kk = s1 - s0;
  const int c0 = w.ccount[2 * h];
  if (threadIdx.x == 0) s_n = 0;
  block_topk(p, w, h, c0, kk, S, ov, oi);
  const double theta = ov[kk - 1];
  if (!(theta == theta)) return;   // NaN correlations: the pick stage reports them
  const double rn = w.rnorm[h];
  const double* cn = w.cnorm + (int64_t)h * p.T;
  const uint8_t* sel = w.sel + (int64_t)h * p.T;
  int32_t* list = w.clist + (int64_t)h * p.T;
  int32_t* stamp = w.cstamp + (int64_t)h * p.T;
  for (int j = threadIdx.x; j < p.T; j += blockDim.x)
    if (!sel[j] && stamp[j] != pass + 1 && rn * cn[j] * (1.0 + kBoundMargin) >= theta) {
      list[c0 + atomicAdd(&s_n, 1)] = j;
      stamp[j] = pass + 1;
    }
  __syncthreads();
  if (threadIdx.x == 0) w.ccount[2 * h + 1] = c0 + s_n;
}

// ------------------------------------------------------------------ pick --
__global__ void __launch_bounds__(kBoundThreads) k_pick(Problem p, Work w, int pass) {
  extern __shared__ __align__(16) unsigned char smem[];
  TopScratch& S = *reinterpret_cast<TopScratch*>(smem);
  __shared__ double ov[kMaxKK];
  __shared__ int oi[kMaxKK];
  const int h = w.order[blockIdx.x];
  int s0, s1;
  pass_range(p, w.t[h], pass, s0, s1);
  if (s0 >= s1) return;
  const int kk = s1 - s0;
  block_topk(p, w, h, w.ccount[2 * h + 1], kk, S, ov, oi);
  if (threadIdx.x == 0) {
    uint8_t* sel = w.sel + (int64_t)h * p.T;
    bool bad = false;
    for (int k = 0; k < kk; ++k) {
      int j = oi[k];
      double v = ov[k];
      if (j == INT_MAX || !(v == v)) {   // no finite value left: lowest free key
        bad = true;
        for (j = 0; j < p.T && sel[j]; ++j) {}
        v = -INFINITY;
      }
      const int64_t o = w.cu_t[h] + s0 + k;
      w.picks[o] = j;
      w.pick_corr[o] = (float)v;
      sel[j] = 1;
    }
    if (bad) record_status(w.status + h, AM_ERR_NONFINITE);
  }
}

int rows_ctas_per_head(int active) {
  const int c = (2 * 148 + active - 1) / active;
  return c < 1 ? 1 : (c > 64 ? 64 : c);
}

}  // namespace

cudaError_t launch_column_norms(const Problem& p, const Work& w, cudaStream_t s) {
  dim3 g((p.T + 7) / 8, p.H);
  AM_LAUNCH(AM_STAGE_PHI, s, k_colnorm<<<g, 256, 0, s>>>(p, w));
  return cudaGetLastError();
}

cudaError_t launch_corr_bounded(const Problem& p, const Work& w, int pass, int active, cudaStream_t s) {
  const int top_smem = (int)sizeof(TopScratch);
  cudaFuncSetAttribute(k_extend, cudaFuncAttributeMaxDynamicSharedMemorySize, top_smem);
  cudaFuncSetAttribute(k_pick, cudaFuncAttributeMaxDynamicSharedMemorySize, top_smem);
  dim3 gr(rows_ctas_per_head(active), active);
  AM_LAUNCH(AM_STAGE_CORR, s, k_probe<<<active, kBoundThreads, 0, s>>>(p, w, pass));
  AM_LAUNCH(AM_STAGE_CORR, s, k_rows<<<gr, 256, 0, s>>>(p, w, pass, 0));
  AM_LAUNCH(AM_STAGE_CORR, s, k_extend<<<active, kBoundThreads, top_smem, s>>>(p, w, pass));
  AM_LAUNCH(AM_STAGE_CORR, s, k_rows<<<gr, 256, 0, s>>>(p, w, pass, 1));
  AM_LAUNCH(AM_STAGE_SELECT, s, k_pick<<<active, kBoundThreads, top_smem, s>>>(p, w, pass));
  return cudaGetLastError();
}

}  // namespace am
