// Bounded correlation pass: the OMP selection step j* = argmax_{j∉S} rᵀΦ_{:,j}
// ("Fast KV Compaction via Attention Matching": zhichai.net deep dive §1.6;
// k·R keys per pass under top-k batching with lazy refit, xinfinite.net
// article §3), evaluated exactly for only the keys that can win.
//
// For every key |c_j| = |rᵀΦ_{:,j}| <= ‖r‖₂·‖Φ_{:,j}‖₂ (Cauchy-Schwarz).  The
// column norms do not depend on r, so once per call the keys are sorted by
// norm (k_colnorm, k_sortnorm); in every pass the keys a bound cannot exclude
// then form a prefix of that order.  One pass of kk = s1 − s0 picks per head
// is two launches of k_rows:
//   1. exact c_j for the unselected keys among the first P0 sorted positions,
//      P0 = max(kProbe + s0, the previous pass's L) (so at least kProbe keys;
//      L moves little from pass to pass): fp64 sums of the stored fp32
//      features times the stored fp32 residual; then the last block of the
//      head takes θ = the kk-th largest of those values and the prefix length
//      L: every key with ‖Φ_{:,j}‖ >= θ / (‖r‖(1 + 1e-9)) lies in [0, L) (a
//      count over the sorted norms).  When L <= P0 the kk largest values found
//      are already the picks, and it appends them;
//   2. otherwise exact c_j for the unselected keys in [P0, L); then the last
//      block appends the kk largest values of [0, L) (ties to the lower key).
// A key beyond L has c_j < θ while kk keys in the prefix reach θ, so it is not
// among the kk largest: the picks are those of a full pass over all keys.
// The margin 1e-9 covers the rounding of the fp64 sums and norms (relative
// error below n·2^-53 for the sums, a few ulp for the norms); the fp32 copies
// of the norms only move the cut outward (rounding to nearest is monotone).
// The selections take kk rounds of a block-wide argmax over candidates staged
// in shared memory.
#include "am_internal.cuh"
#include "am_profile.cuh"
#include "am_linalg.cuh"

#include <float.h>

namespace am {
namespace {

constexpr int kProbe = 256;        // unselected keys whose exact values set the threshold
constexpr int kBoundThreads = 1024;
constexpr int kSelCap = 2304;      // candidates one selection holds (>= kProbe + 2048)
constexpr double kBoundMargin = 1e-9;

// Order-preserving map of a double to uint64 (NaN ranks lowest).
__device__ __forceinline__ uint64_t order_key(double v) {
  if (v != v) return 0ull;
  const uint64_t u = (uint64_t)__double_as_longlong(v);
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// (a, ja) before (b, jb) in pick order: larger key first, then lower index.
__device__ __forceinline__ bool before(uint64_t a, int ja, uint64_t b, int jb) {
  return a > b || (a == b && ja < jb);
}

// ---------------------------------------------------------- column norms --
// ‖Φ_{:,j}‖₂ in fp64 from the stored fp32 features: one warp per key.
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

// ‖Φ_{:,j}‖₂ from the feature pass's per-warp partial sums (fp32 sums of 32
// fp32 squares, relative error below 4e-7): their fp64 total, raised by the
// factor 1 + 1e-6 so the result stays an upper bound of the exact norm.
__global__ void __launch_bounds__(256) k_normsum(Problem p, Work w) {
  const int h = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= p.T) return;
  const int parts = 4 * ((p.n + 127) / 128);
  const float* src = w.cnpart + (int64_t)h * parts * p.T + j;
  double s = 0.0;
  for (int k = 0; k < parts; ++k) s += (double)src[(int64_t)k * p.T];
  w.cnorm[(int64_t)h * p.T + j] = sqrt(s) * (1.0 + 1e-6);
}

// Keys of each head by descending fp32 norm (ties: lower key first): one
// block per head; 64-bit sort keys (norm bits, inverted key index) in shared
// memory, or in the workspace when T exceeds kSortSmemKeys.
__global__ void __launch_bounds__(kBoundThreads) k_sortnorm(Problem p, Work w) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int h = blockIdx.x;
  int n2 = 1;
  while (n2 < p.T) n2 <<= 1;
  uint64_t* key = p.T > kSortSmemKeys ? w.ksort + (int64_t)h * n2 : reinterpret_cast<uint64_t*>(smem);
  const double* cn = w.cnorm + (int64_t)h * p.T;
  for (int i = threadIdx.x; i < n2; i += blockDim.x)
    key[i] = i < p.T ? ((uint64_t)__float_as_uint((float)cn[i]) << 32) | (uint32_t)(0xFFFFFFFFu - (uint32_t)i)
                     : 0ull;
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int l = i ^ jj;
        if (l > i) {
          const bool desc = (i & k) == 0;
          const uint64_t a = key[i], b = key[l];
          if (desc ? a < b : a > b) { key[i] = b; key[l] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < p.T; i += blockDim.x) {
    const uint64_t k = key[i];
    w.korder[(int64_t)h * p.T + i] = (int32_t)(0xFFFFFFFFu - (uint32_t)k);
    w.knorm[(int64_t)h * p.T + i] = __uint_as_float((uint32_t)(k >> 32));
  }
}

// ------------------------------------------------------------ selection --
constexpr int kSelThreads = 256;

struct SelScratch {
  uint64_t key[kSelCap];
  int idx[kSelCap];
  uint64_t wk[kSelThreads / 32];
  int wj[kSelThreads / 32], wp[kSelThreads / 32];
  uint64_t outk[kMaxPicksPerPass];
  int outj[kMaxPicksPerPass];
  double red[33];
  int cnt;
};

// Appends the unselected keys at sorted positions [lo, hi) to the candidate
// slots from S.cnt on (at most kSelCap in all); all threads.
__device__ void stage_candidates(const Problem& p, const Work& w, int h, int lo, int hi, SelScratch& S) {
  const int32_t* ord = w.korder + (int64_t)h * p.T;
  const uint8_t* sel = w.sel + (int64_t)h * p.T;
  const double* cd = w.corrd + (int64_t)h * p.T;
  for (int q0 = lo + threadIdx.x; q0 < hi; q0 += 4 * blockDim.x) {   // four keys in flight
    int j[4];
    bool s[4];
    double v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = q0 + u * blockDim.x;
      j[u] = q < hi ? ord[q] : -1;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      s[u] = j[u] < 0 || sel[j[u] < 0 ? 0 : j[u]];
      v[u] = cd[j[u] < 0 ? 0 : j[u]];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (s[u]) continue;
      const int pos = atomicAdd(&S.cnt, 1);
      if (pos < kSelCap) {
        S.key[pos] = order_key(v[u]);
        S.idx[pos] = j[u];
      }
    }
  }
  __syncthreads();
}

// Keeps the better of (k, j, pos) and the lane `o` away, in pick order.
__device__ __forceinline__ void shfl_best(uint64_t& k, int& j, int& pos, int o) {
  const uint64_t k2 = __shfl_xor_sync(0xffffffffu, k, o);
  const int j2 = __shfl_xor_sync(0xffffffffu, j, o);
  const int p2 = __shfl_xor_sync(0xffffffffu, pos, o);
  if (p2 >= 0 && (pos < 0 || before(k2, j2, k, j))) { k = k2; j = j2; pos = p2; }
}

// The kk candidates first in pick order, by kk rounds of a block-wide argmax
// over slots [0, n): into S.outk / S.outj (index INT_MAX when none is left);
// each winner's slot is cleared.  All threads.
__device__ void select_rounds(SelScratch& S, int n, int kk) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  for (int k = 0; k < kk; ++k) {
    uint64_t bk = 0ull;
    int bj = INT_MAX, bp = -1;
    for (int e = tid; e < n; e += blockDim.x) {
      const int jv = S.idx[e];
      if (jv == INT_MAX) continue;
      const uint64_t kv = S.key[e];
      if (bp < 0 || before(kv, jv, bk, bj)) { bk = kv; bj = jv; bp = e; }
    }
    for (int o = 16; o; o >>= 1) shfl_best(bk, bj, bp, o);
    if (lane == 0) { S.wk[warp] = bk; S.wj[warp] = bj; S.wp[warp] = bp; }
    __syncthreads();
    if (warp == 0) {
      bk = lane < nw ? S.wk[lane] : 0ull;
      bj = lane < nw ? S.wj[lane] : INT_MAX;
      bp = lane < nw ? S.wp[lane] : -1;
      for (int o = 16; o; o >>= 1) shfl_best(bk, bj, bp, o);
      if (lane == 0) {
        S.outk[k] = bk;
        S.outj[k] = bp >= 0 ? bj : INT_MAX;
        if (bp >= 0) { S.key[bp] = 0ull; S.idx[bp] = INT_MAX; }
      }
    }
    __syncthreads();
  }
}

// Σ r_i² over [0, n) by all threads, eight loads per thread in flight.
__device__ __forceinline__ double sum_squares(const float* r, int n) {
  double a = 0.0;
  for (int i0 = threadIdx.x; i0 < n; i0 += 8 * blockDim.x) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      v[u] = i < n ? r[i] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) a = fma((double)v[u], (double)v[u], a);
  }
  return a;
}

// Number of entries of kn[0, n) not below thr, by all threads (per-thread part).
__device__ __forceinline__ int count_not_below(const float* kn, int n, float thr) {
  int c = 0;
  for (int i0 = threadIdx.x; i0 < n; i0 += 8 * blockDim.x) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * blockDim.x;
      v[u] = i < n ? kn[i] : thr;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) c += (i0 + u * (int)blockDim.x < n) && !(v[u] < thr);
  }
  return c;
}

__device__ void append_picks(const Problem& p, const Work& w, int h, int s0, int kk, SelScratch& S);

// θ and the prefix L (the last block of a head, after the probe rows); the
// picks too when the probe already covers L.
__device__ void theta_and_prefix(const Problem& p, const Work& w, int h, int s0, int p0, int kk, SelScratch& S) {
  const double rn = sqrt(block_sum(sum_squares(w.r + (int64_t)h * p.ldn, p.ldn), S.red));
  if (threadIdx.x == 0) S.cnt = 0;
  __syncthreads();
  stage_candidates(p, w, h, 0, p0, S);   // p0 <= kSelCap
  const int staged = min(S.cnt, kSelCap);
  select_rounds(S, staged, kk);
  const int jt = S.outj[kk - 1];
  const double theta = jt != INT_MAX ? w.corrd[(int64_t)h * p.T + jt] : -INFINITY;
  // L = number of sorted norms not below θ / (‖r‖(1 + margin)); every key when
  // the bound cannot help (θ <= 0, a zero or non-finite residual)
  const bool useful = theta > 0.0 && rn > 0.0 && rn < INFINITY;
  const float thr = useful ? (float)(theta / (rn * (1.0 + kBoundMargin))) : 0.f;
  const int count = useful ? count_not_below(w.knorm + (int64_t)h * p.T, p.T, thr) : 0;
  const double tot = block_sum((double)count, S.red);
  const int L = useful ? (int)tot : p.T;
  const bool done = L <= p0;
  if (threadIdx.x == 0) {
    w.cprefix[h] = L;   // the next pass sizes its probe by it
    w.cprobe[h] = p0;
    w.cdone[h] = done;
    w.rnorm[h] = rn;
    if (done) w.rows_eval[h] += (unsigned long long)staged;
  }
  if (done) append_picks(p, w, h, s0, kk, S);
}

// Appends S.outj[0, kk) as this pass's picks (thread 0).
__device__ void append_picks(const Problem& p, const Work& w, int h, int s0, int kk, SelScratch& S) {
  if (threadIdx.x != 0) return;
  uint8_t* sel = w.sel + (int64_t)h * p.T;
  const double* cd = w.corrd + (int64_t)h * p.T;
  bool bad = false;
  for (int k = 0; k < kk; ++k) {
    int j = S.outj[k];
    double v = j != INT_MAX ? cd[j] : -INFINITY;
    if (j == INT_MAX || !(v == v)) {   // no finite value: lowest free key
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

// The kk largest values among the unselected keys of [0, L), in chunks that
// carry the best kk of what came before (the last block of a head, after the
// remaining rows).
__device__ void pick_from_prefix(const Problem& p, const Work& w, int h, int s0, int kk, SelScratch& S) {
  const int L = w.cprefix[h];
  const int chunk = kSelCap - kMaxPicksPerPass;
  int kept = 0;
  unsigned long long evaluated = 0;
  for (int c = 0; c < L; c += chunk) {
    if (threadIdx.x < kept) {   // winners so far lead the next chunk
      S.key[threadIdx.x] = S.outk[threadIdx.x];
      S.idx[threadIdx.x] = S.outj[threadIdx.x];
    }
    if (threadIdx.x == 0) S.cnt = kept;
    __syncthreads();
    stage_candidates(p, w, h, c, min(L, c + chunk), S);
    const int n = min(S.cnt, kSelCap);
    evaluated += (unsigned long long)(n - kept);
    select_rounds(S, n, kk);
    kept = 0;
    for (int k = 0; k < kk; ++k) kept += S.outj[k] != INT_MAX;
  }
  if (threadIdx.x == 0) w.rows_eval[h] += evaluated;
  append_picks(p, w, h, s0, kk, S);
}

// ------------------------------------------------------------ exact rows --
// c_j = Σ_i r_i Φ_ij for the unselected keys at sorted positions [0, P0)
// (which = 0) or [P0, L) (which = 1), in fp64 sums of exact fp32 products.
// Four warps share a key, each summing a quarter of the queries with four
// columns per lane in flight; the quarters are added in a fixed order.  The
// last block of a head to finish (counted with an atomic) then takes the
// selection step: θ and L after the probe rows, the picks after the rest.
constexpr int kRowSplit = 4;                           // warps per key
constexpr int kRowsPerBlock = kSelThreads / 32 / kRowSplit;   // keys per block

__global__ void __launch_bounds__(kSelThreads) k_rows(Problem p, Work w, int pass, int which) {
  extern __shared__ __align__(16) unsigned char smem[];
  SelScratch& S = *reinterpret_cast<SelScratch*>(smem);
  __shared__ double part[kRowsPerBlock][kRowSplit];
  __shared__ int s_last;
  const int h = w.order[blockIdx.y];
  int s0, s1;
  pass_range(p, w.t[h], pass, s0, s1);
  if (s0 >= s1) return;
  const int kk = s1 - s0;
  if (which && w.cdone[h]) return;                     // the probe step made the picks
  // the probe reaches the previous pass's prefix (kept in cprefix until the
  // probe's last block replaces it), at most kSelCap positions
  const int p0 = which ? w.cprobe[h] : min(min(p.T, kSelCap), max(kProbe + s0, w.cprefix[h]));
  const int lo = which ? p0 : 0;
  const int hi = which ? w.cprefix[h] : p0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slot = warp / kRowSplit, quarter = warp % kRowSplit;
  const int32_t* ord = w.korder + (int64_t)h * p.T;
  const uint8_t* sel = w.sel + (int64_t)h * p.T;
  const float4* r4 = reinterpret_cast<const float4*>(w.r + (int64_t)h * p.ldn);
  const int n4 = p.ldn >> 2;
  const int per = (n4 + kRowSplit - 1) / kRowSplit;
  const int c0 = quarter * per, c1 = min(n4, c0 + per);
  for (int q0 = lo + blockIdx.x * kRowsPerBlock; q0 < hi; q0 += gridDim.x * kRowsPerBlock) {
    const int q = q0 + slot;
    const int j = q < hi ? ord[q] : 0;
    const bool on = q < hi && !sel[j];
    double a[4] = {0.0, 0.0, 0.0, 0.0};
    if (on) {
      const float4* row = reinterpret_cast<const float4*>(w.phiT + ((int64_t)h * p.T + j) * p.ldn);
      for (int i0 = c0 + lane; i0 < c1; i0 += 32 * 4) {
        float4 x[4], y[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = i0 + 32 * u;
          x[u] = i < c1 ? __ldcs(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
          y[u] = i < c1 ? __ldg(r4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          a[0] = fma((double)x[u].x, (double)y[u].x, a[0]);
          a[1] = fma((double)x[u].y, (double)y[u].y, a[1]);
          a[2] = fma((double)x[u].z, (double)y[u].z, a[2]);
          a[3] = fma((double)x[u].w, (double)y[u].w, a[3]);
        }
      }
    }
    const double c = warp_sum((a[0] + a[1]) + (a[2] + a[3]));
    if (lane == 0) part[slot][quarter] = c;
    __syncthreads();
    if (on && quarter == 0 && lane == 0)
      w.corrd[(int64_t)h * p.T + j] = (part[slot][0] + part[slot][1]) + (part[slot][2] + part[slot][3]);
    __syncthreads();
  }
  // the last block of this head to get here takes the selection step
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(w.rcount + h, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (which == 0) theta_and_prefix(p, w, h, s0, p0, kk, S);
  else pick_from_prefix(p, w, h, s0, kk, S);
  if (threadIdx.x == 0) w.rcount[h] = 0;
}

int rows_ctas_per_head(int active) {
  const int c = (8 * 148 + active - 1) / active;
  return c < 1 ? 1 : (c > 256 ? 256 : c);
}

}  // namespace

cudaError_t launch_column_norms(const Problem& p, const Work& w, cudaStream_t s) {
  if (w.cnpart) {   // partial sums left by the tensor-core feature pass
    dim3 g((p.T + 255) / 256, p.H);
    AM_LAUNCH(AM_STAGE_NORMS, s, k_normsum<<<g, 256, 0, s>>>(p, w));
  } else {
    dim3 g((p.T + 7) / 8, p.H);
    AM_LAUNCH(AM_STAGE_NORMS, s, k_colnorm<<<g, 256, 0, s>>>(p, w));
  }
  const int sort_smem = p.T > kSortSmemKeys ? 0 : (int)(sizeof(uint64_t) * kSortSmemKeys);
  cudaFuncSetAttribute(k_sortnorm, cudaFuncAttributeMaxDynamicSharedMemorySize, sort_smem);
  AM_LAUNCH(AM_STAGE_NORMS, s, k_sortnorm<<<p.H, kBoundThreads, sort_smem, s>>>(p, w));
  return cudaGetLastError();
}

cudaError_t launch_corr_bounded(const Problem& p, const Work& w, int pass, int active, cudaStream_t s) {
  const int sel_smem = (int)sizeof(SelScratch);
  cudaFuncSetAttribute(k_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, sel_smem);
  dim3 gr(rows_ctas_per_head(active), active);
  AM_LAUNCH(AM_STAGE_ROWS, s, k_rows<<<gr, kSelThreads, sel_smem, s>>>(p, w, pass, 0));
  AM_LAUNCH(AM_STAGE_ROWS, s, k_rows<<<gr, kSelThreads, sel_smem, s>>>(p, w, pass, 1));
  return cudaGetLastError();
}

}  // namespace am
