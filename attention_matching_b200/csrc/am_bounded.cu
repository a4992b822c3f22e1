// Bounded correlation pass: the OMP selection step j* = argmax_{j∉S} rᵀΦ_{:,j}
// ("Fast KV Compaction via Attention Matching": zhichai.net deep dive §1.6;
// k·R keys per pass under top-k batching with lazy refit, xinfinite.net
// article §3), evaluated exactly for only the keys that can win.
//
// Split the queries into the residual update's groups g (queries i with
// (i / 128) mod G == g).  For every key, by Cauchy-Schwarz on each group,
//   |c_j| = |Σ_i r_i Φ_ij| <= Σ_g ‖r_g‖·‖Φ_{g,j}‖ =: b_j.
// The group norms ‖Φ_{g,j}‖ do not depend on r: they come once per call from
// the feature pass's partial sums (k_normsum, or k_colnorm from the stored
// features).  One pass of kk = s1 − s0 picks per head is three launches:
//   1. k_gbound: b_j for every unselected key (fp64 sum of the group terms,
//      stored fp32) and a histogram of the bounds; the head's last block sets
//      τ, the lower edge of the histogram bin at which 2·kk + 32 keys are
//      reached counting from the top;
//   2. k_rows (probe): exact c_j (fp64 sums of the stored fp32 features times
//      the stored fp32 residual) for the keys with b_j >= τ; the head's last
//      block takes θ = the kk-th largest value; when θ >= τ·(1 + 1e-6) every
//      key left out has c_j <= b_j < θ, and it appends the kk largest as the
//      picks (ties to the lower key);
//   3. k_rows (rest): otherwise exact c_j for the keys with b_j < τ and
//      b_j·(1 + 1e-6) >= θ; then the kk largest of everything evaluated.
// A key left out has c_j < θ while kk evaluated keys reach θ, so the picks are
// those of a full pass over all keys.  The margins cover the rounding of the
// fp64 sums, the fp32 store of b_j (both below 1e-7 relative), the group
// norms (raised by 2e-6 over their fp32 partial sums) and ‖r_g‖ being taken
// from the fp64 residual while the rows are correlated with its fp32 copy
// (larger by at most 2^-24 relative).  The row blocks append every evaluated
// key (order key of c_j, key index) to a per-head list; a selection stages
// that list in shared memory and takes a warp-level top-kk (kk rounds of
// three warp reductions per warp) followed by the same over the warps'
// winners.  The global column norms ‖Φ_{:,j}‖ are kept as well (the
// workspace view reports them).
#include "am_internal.cuh"
#include "am_profile.cuh"
#include "am_linalg.cuh"

#include <float.h>

namespace am {
namespace {

constexpr int kBoundThreads = 1024;
constexpr int kSelCap = 2304;      // list entries one selection stage holds

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
// Besides ‖Φ_{:,j}‖₂, every key gets an upper bound of its norm over each
// residual query group g (the queries i with (i / 128) mod G == g, G =
// resid_blocks(p): the groups whose ‖r_g‖² the residual update leaves), so
// that |c_j| <= Σ_g ‖r_g‖·‖Φ_{g,j}‖ (Cauchy-Schwarz on each group) can skip
// keys the global bound ‖r‖·‖Φ_{:,j}‖ keeps.  Group norms are raised by the
// factor 1 + 2e-6 (covering fp32 partial sums and the fp32 store).
constexpr double kBlockNormInflate = 1.0 + 2e-6;

// ‖Φ_{:,j}‖₂ in fp64 from the stored fp32 features, and the group norms: one
// warp per key; lane l takes float4 l of each 128-query segment.
__global__ void __launch_bounds__(256) k_colnorm(Problem p, Work w) {
  __shared__ double gsum[8][kRedBlocks];
  const int h = blockIdx.y;
  const int wib = threadIdx.x >> 5;
  const int j = blockIdx.x * 8 + wib;
  const int lane = threadIdx.x & 31;
  if (j >= p.T) return;
  if (j >= w.Th[h]) {   // no such key in this head: norm 0, never evaluated
    if (lane == 0) w.cnorm[(int64_t)h * p.T + j] = 0.0;
    for (int g = lane; g < kRedBlocks; g += 32) w.cnblk[((int64_t)h * kRedBlocks + g) * p.T + j] = 0.f;
    return;
  }
  const int G = resid_blocks(p);
  for (int g = lane; g < kRedBlocks; g += 32) gsum[wib][g] = 0.0;
  __syncwarp();
  const float4* row = reinterpret_cast<const float4*>(w.phiT + ((int64_t)h * p.T + j) * p.ldn);
  const int n4 = p.ldn >> 2;
  double tot = 0.0;
  for (int seg = 0; seg * 32 < n4; ++seg) {
    const int i = seg * 32 + lane;
    double a = 0.0;
    if (i < n4) {
      const float4 x = __ldcs(row + i);
      a = fma((double)x.x, (double)x.x, a);
      a = fma((double)x.y, (double)x.y, a);
      a = fma((double)x.z, (double)x.z, a);
      a = fma((double)x.w, (double)x.w, a);
    }
    a = warp_sum(a);
    tot += a;
    if (lane == 0) gsum[wib][seg % G] += a;
  }
  __syncwarp();
  if (lane == 0) w.cnorm[(int64_t)h * p.T + j] = sqrt(tot);
  for (int g = lane; g < kRedBlocks; g += 32)
    w.cnblk[((int64_t)h * kRedBlocks + g) * p.T + j] = g < G ? (float)(sqrt(gsum[wib][g]) * kBlockNormInflate) : 0.f;
}

// ‖Φ_{:,j}‖₂ from the feature pass's per-warp partial sums (fp32 sums of 32
// fp32 squares, relative error below 4e-7): their fp64 total, raised by the
// factor 1 + 1e-6 so the result stays an upper bound of the exact norm; and
// the group norms from the same partials (a 128-query block is one segment).
__global__ void __launch_bounds__(256) k_normsum(Problem p, Work w) {
  const int h = blockIdx.y;
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= p.T) return;
  float* blk = w.cnblk + (int64_t)h * kRedBlocks * p.T + j;   // group g at blk[g·T]
  if (j >= w.Th[h]) {   // no such key in this head: norm 0, never evaluated
    w.cnorm[(int64_t)h * p.T + j] = 0.0;
    for (int g = 0; g < kRedBlocks; ++g) blk[(int64_t)g * p.T] = 0.f;
    return;
  }
  const int nqb = (p.n + 127) / 128;
  const int G = resid_blocks(p);
  const float* src = w.cnpart + (int64_t)h * 4 * nqb * p.T + j;
  double s = 0.0;
  for (int g = 0; g < kRedBlocks; ++g) {
    double sg = 0.0;
    if (g < G)
      for (int qb = g; qb < nqb; qb += G)
        for (int k = 0; k < 4; ++k) sg += (double)src[(int64_t)(qb * 4 + k) * p.T];
    s += sg;
    blk[(int64_t)g * p.T] = g < G ? (float)(sqrt(sg) * kBlockNormInflate) : 0.f;
  }
  w.cnorm[(int64_t)h * p.T + j] = sqrt(s) * (1.0 + 1e-6);
}

// ------------------------------------------------------------ selection --
constexpr int kSelThreads = 256;

struct SelScratch {
  uint64_t key[kSelCap];
  int idx[kSelCap];
  uint64_t ck[kSelThreads / 32 * kMaxPicksPerPass];   // warp w's kk best at [w·kk, (w+1)·kk)
  int cj[kSelThreads / 32 * kMaxPicksPerPass];
  uint64_t outk[kMaxPicksPerPass];
  int outj[kMaxPicksPerPass];
  double red[33];
};

// Copies entries [lo, hi) of the head's list of evaluated keys (order key of
// c_j, key index) to candidate slots from `at` on; all threads, four loads
// per thread in flight.
__device__ void stage_list(const Problem& p, const Work& w, int h, int lo, int hi, int at, SelScratch& S) {
  const uint64_t* lk = w.clist + (int64_t)h * p.T;
  const int32_t* lj = w.clj + (int64_t)h * p.T;
  for (int q0 = lo + threadIdx.x; q0 < hi; q0 += 4 * blockDim.x) {
    uint64_t k[4];
    int j[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = q0 + u * blockDim.x;
      k[u] = q < hi ? __ldcg(lk + q) : 0ull;
      j[u] = q < hi ? __ldcg(lj + q) : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int q = q0 + u * blockDim.x;
      if (q < hi) {
        S.key[at + q - lo] = k[u];
        S.idx[at + q - lo] = j[u];
      }
    }
  }
  __syncthreads();
}

// The best live entry (index not INT_MAX) of keys/idx at e = first, first +
// stride, ... below n: (key, index, position), position -1 when none.
__device__ __forceinline__ void lane_best(const uint64_t* keys, const int* idx, int first, int stride, int n,
                                          uint64_t& bk, int& bj, int& bp) {
  bk = 0ull; bj = INT_MAX; bp = -1;
  for (int e = first; e < n; e += stride) {
    const int jv = idx[e];
    if (jv == INT_MAX) continue;
    const uint64_t kv = keys[e];
    if (bp < 0 || before(kv, jv, bk, bj)) { bk = kv; bj = jv; bp = e; }
  }
}

// kk rounds of a warp argmax over one warp's entries (lane l owns positions
// first + l·… as laid out by lane_best): round k's winner goes to outk[k] /
// outj[k] (index INT_MAX once nothing is left) and its entry is marked used;
// only the winning lane rescans.  A round is three warp reductions in pick
// order: the largest high word of the key, the largest low word among those,
// the lowest key index among those (entries carry distinct indices).  One warp.
__device__ __forceinline__ void warp_top(uint64_t* keys, int* idx, int first, int stride, int n, int kk,
                                         uint64_t* outk, int* outj) {
  const int lane = threadIdx.x & 31;
  uint64_t bk;
  int bj, bp;
  lane_best(keys, idx, first, stride, n, bk, bj, bp);
  for (int k = 0; k < kk; ++k) {
    const bool live = bp >= 0;
    const unsigned kh = live ? (unsigned)(bk >> 32) : 0u;
    const unsigned kl = live ? (unsigned)bk : 0u;
    const unsigned jj = live ? (unsigned)bj : 0x7fffffffu;
    const unsigned m1 = __reduce_max_sync(0xffffffffu, kh);
    const unsigned m2 = __reduce_max_sync(0xffffffffu, kh == m1 ? kl : 0u);
    const bool top = kh == m1 && kl == m2;
    const unsigned m3 = __reduce_min_sync(0xffffffffu, top ? jj : 0xffffffffu);
    if (lane == 0) {
      outk[k] = ((uint64_t)m1 << 32) | m2;
      outj[k] = (int)m3;   // INT_MAX when no lane had an entry left
    }
    if (live && top && jj == m3) {   // the owner of the winning entry takes its next best
      idx[bp] = INT_MAX;
      lane_best(keys, idx, first, stride, n, bk, bj, bp);
    }
  }
  __syncwarp();
}

// The kk candidates first in pick order among slots [0, n) (ties to the
// lower key) into S.outk / S.outj, index INT_MAX when fewer are left: each
// warp takes the kk best of its slots, then warp 0 the kk best of those.
// The slots are consumed.  All threads.
__device__ void select_top(SelScratch& S, int n, int kk) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  warp_top(S.key, S.idx, warp * 32 + lane, blockDim.x, n, kk, S.ck + warp * kk, S.cj + warp * kk);
  __syncthreads();
  if (warp == 0) warp_top(S.ck, S.cj, lane, 32, nw * kk, kk, S.outk, S.outj);
  __syncthreads();
}

// The value behind an order key (NaN for key 0).
__device__ __forceinline__ double key_value(uint64_t k) {
  if (k == 0ull) return __longlong_as_double(0x7ff8000000000000ll);
  return __longlong_as_double((long long)((k & 0x8000000000000000ull) ? (k & 0x7fffffffffffffffull) : ~k));
}

__device__ void append_picks(const Problem& p, const Work& w, int h, int s0, int kk, SelScratch& S);

// Appends S.outj[0, kk) as this pass's picks, one thread each; a slot with no
// finite value takes the lowest free key instead (thread 0, after the
// others are marked) and flags the head.  All threads.
__device__ void append_picks(const Problem& p, const Work& w, int h, int s0, int kk, SelScratch& S) {
  uint8_t* sel = w.sel + (int64_t)h * p.T;
  const int64_t o = w.cu_t[h] + s0;
  const int k = threadIdx.x;
  bool bad = false;
  if (k < kk) {
    const int j = S.outj[k];
    const double v = j != INT_MAX ? key_value(S.outk[k]) : 0.0;
    bad = j == INT_MAX || !(v == v);
    if (!bad) {
      w.picks[o + k] = j;
      w.pick_corr[o + k] = (float)v;
      sel[j] = 1;
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) {
    for (int q = 0; q < kk; ++q) {
      const double v = S.outj[q] != INT_MAX ? key_value(S.outk[q]) : 0.0;
      if (S.outj[q] != INT_MAX && v == v) continue;
      int j = 0;
      while (j < p.T && sel[j]) ++j;
      if (j >= p.T) break;   // cannot happen: t <= T leaves a free key per pick
      w.picks[o + q] = j;
      w.pick_corr[o + q] = -INFINITY;
      sel[j] = 1;
    }
    record_status(w.status + h, AM_ERR_NONFINITE);
  }
}

// The kk largest values in the head's list of evaluated keys into
// S.outk / S.outj (index INT_MAX when fewer), in chunks that carry the best kk
// of what came before; returns the list length.  All threads.
__device__ int top_of_list(const Problem& p, const Work& w, int h, int kk, SelScratch& S) {
  const int n = __ldcg(w.ccount + h);
  const int chunk = kSelCap - kMaxPicksPerPass;
  int kept = 0;
  if (n == 0) {
    if (threadIdx.x < kk) { S.outk[threadIdx.x] = 0ull; S.outj[threadIdx.x] = INT_MAX; }
    __syncthreads();
  }
  for (int c = 0; c < n; c += chunk) {
    if (threadIdx.x < kept) {   // winners so far lead the next chunk
      S.key[threadIdx.x] = S.outk[threadIdx.x];
      S.idx[threadIdx.x] = S.outj[threadIdx.x];
    }
    const int m = min(n, c + chunk) - c;
    stage_list(p, w, h, c, c + m, kept, S);
    select_top(S, kept + m, kk);
    kept = 0;
    for (int k = 0; k < kk; ++k) kept += S.outj[k] != INT_MAX;
  }
  return n;
}

// The picks from everything evaluated this pass (the last block of a head).
__device__ void pick_from_list(const Problem& p, const Work& w, int h, int s0, int kk, SelScratch& S) {
  const int n = top_of_list(p, w, h, kk, S);
  if (threadIdx.x == 0) {
    w.rows_eval[h] += (unsigned long long)n;
    w.ccount[h] = 0;
  }
  append_picks(p, w, h, s0, kk, S);
}

// ------------------------------------------------------------ group bound --
constexpr int kHistBins = 1024;   // bins of positive fp32 bounds: exponent and two mantissa bits
constexpr int kProbeExtra = 32;   // the probe aims at 2·kk + 32 keys
constexpr double kBoundMargin = 1.0 + 1e-6;

__device__ __forceinline__ int bound_bin(float b) { return (int)(__float_as_uint(b) >> 21); }   // b > 0
__device__ __forceinline__ float bin_floor(int bin) { return __uint_as_float((uint32_t)bin << 21); }

// b_j for every key of the head (−1 for a selected key or one past T_h), and
// the histogram of the positive ones; the head's last block turns the
// histogram into τ and clears it for the next pass.
__global__ void __launch_bounds__(256) k_gbound(Problem p, Work w, int pass) {
  chain_wait();
  __shared__ double rg[kRedBlocks];
  __shared__ int hist[kHistBins];
  __shared__ int s_last;
  __shared__ int csum[32];
  const int h = w.order[blockIdx.y];
  int s0, s1;
  pass_range(p, w.t[h], pass, s0, s1);
  if (s0 >= s1) return;
  const int kk = s1 - s0;
  const int G = resid_blocks(p);
  for (int g = threadIdx.x; g < kRedBlocks; g += blockDim.x)
    rg[g] = g < G ? sqrt(w.rr_part[(int64_t)h * kRedBlocks + g]) : 0.0;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j < p.T) {
    float b = -1.f;
    if (!w.sel[(int64_t)h * p.T + j]) {
      const float* cb = w.cnblk + (int64_t)h * kRedBlocks * p.T + j;
      double acc = 0.0;
      for (int g = 0; g < G; ++g) acc = fma(rg[g], (double)__ldg(cb + (int64_t)g * p.T), acc);
      b = (float)acc;
      if (b > 0.f) atomicAdd(&hist[bound_bin(b)], 1);
    }
    w.gb[(int64_t)h * p.T + j] = b;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (hist[i]) atomicAdd(w.ghist + (int64_t)h * kHistBins + i, hist[i]);
  chain_release();
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(w.gcnt + h, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // τ: counting bins from the top, the first at which 2·kk + 32 keys are reached
  int* gh = w.ghist + (int64_t)h * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
    hist[i] = __ldcg(gh + i);
    gh[i] = 0;   // ready for the next pass
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int top = kHistBins - 1 - 32 * lane;   // this lane's bins: top .. top − 31
    int sum = 0;
    for (int k = 0; k < 32; ++k) sum += hist[top - k];
    int incl = sum;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    csum[lane] = incl;
    __syncwarp();
    const int target = 2 * kk + kProbeExtra;
    const unsigned reach = __ballot_sync(0xffffffffu, incl >= target);
    float tau = 0.f;   // fewer keys than the target: the probe takes every unselected key
    if (reach) {
      const int l = __ffs(reach) - 1;
      if (lane == l) {
        int cum = l > 0 ? csum[l - 1] : 0;
        int bin = top;
        for (int k = 0; k < 32; ++k) {
          cum += hist[top - k];
          if (cum >= target) { bin = top - k; break; }
        }
        w.gtau[h] = bin_floor(bin);
      }
    } else if (lane == 0) {
      w.gtau[h] = tau;
    }
    if (lane == 0) w.gcnt[h] = 0;
  }
}

// ------------------------------------------------------------ exact rows --
// c_j = Σ_i r_i Φ_ij in fp64 sums of exact fp32 products for the keys the
// launch takes: b_j >= τ (which = 0, the probe) or b_j < τ with
// b_j·(1 + 1e-6) >= θ (which = 1, the rest).  Each CTA scans every
// gridDim.x-th key of the head in chunks, gathers the keys it takes in shared memory, and
// evaluates them two at a time: four warps share a key, each summing a
// quarter of the queries with eight columns per lane in flight; the quarters
// are added in a fixed order.  The last block of a head to finish (counted
// with an atomic) then takes the selection step.
constexpr int kRowSplit = 4;                           // warps per key
constexpr int kRowsPerBlock = kSelThreads / 32 / kRowSplit;   // keys per block
constexpr int kRowLoads = 8;                           // float4 columns per lane in flight
constexpr int kScanChunk = 2048;                       // keys scanned per chunk of a CTA's slice

__global__ void __launch_bounds__(kSelThreads) k_rows(Problem p, Work w, int pass, int which) {
  chain_wait();
  extern __shared__ __align__(16) unsigned char smem[];
  SelScratch& S = *reinterpret_cast<SelScratch*>(smem);
  __shared__ double part[kRowsPerBlock][kRowSplit];
  __shared__ int s_last;
  __shared__ int cand[kScanChunk];
  __shared__ int ncand;
  const int h = w.order[blockIdx.y];
  int s0, s1;
  pass_range(p, w.t[h], pass, s0, s1);
  if (s0 >= s1) return;
  const int kk = s1 - s0;
  if (which && w.cdone[h]) return;                     // the probe step made the picks
  const float tau = w.gtau[h];
  const double theta = which ? w.ctheta[h] : 0.0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slot = warp / kRowSplit, quarter = warp % kRowSplit;
  const uint8_t* sel = w.sel + (int64_t)h * p.T;
  const float* gb = w.gb + (int64_t)h * p.T;
  const float4* r4 = reinterpret_cast<const float4*>(w.r + (int64_t)h * p.ldn);
  const int n4 = p.ldn >> 2;
  const int per = (n4 + kRowSplit - 1) / kRowSplit;
  const int c0 = quarter * per, c1 = min(n4, c0 + per);
  // this CTA's keys: j ≡ blockIdx.x (mod gridDim.x), so keys the bound keeps,
  // which cluster by index, spread evenly over the head's CTAs
  const int nkeys = (p.T - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
  for (int i0 = 0; i0 < nkeys; i0 += kScanChunk) {
    const int i1 = min(nkeys, i0 + kScanChunk);
    if (threadIdx.x == 0) ncand = 0;
    __syncthreads();
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
      const int j = (int)blockIdx.x + i * (int)gridDim.x;
      const float b = gb[j];
      bool take = false;
      if (!sel[j]) take = which == 0 ? b >= tau : (b < tau && (double)b * kBoundMargin >= theta);
      if (take) cand[atomicAdd(&ncand, 1)] = j;
    }
    __syncthreads();
    const int nc = ncand;
    for (int q0 = 0; q0 < nc; q0 += kRowsPerBlock) {
      const int q = q0 + slot;
      const bool on = q < nc;
      const int j = on ? cand[q] : 0;
      double a[4] = {0.0, 0.0, 0.0, 0.0};
      if (on) {
        const float4* row = reinterpret_cast<const float4*>(w.phiT + ((int64_t)h * p.T + j) * p.ldn);
        for (int i0 = c0 + lane; i0 < c1; i0 += 32 * kRowLoads) {
          float4 x[kRowLoads], y[kRowLoads];
#pragma unroll
          for (int u = 0; u < kRowLoads; ++u) {
            const int i = i0 + 32 * u;
            x[u] = i < c1 ? __ldcs(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
            y[u] = i < c1 ? __ldg(r4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < kRowLoads; ++u) {
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
      if (on && quarter == 0 && lane == 0) {   // onto the head's list of evaluated keys
        const double cj = (part[slot][0] + part[slot][1]) + (part[slot][2] + part[slot][3]);
        const int at = atomicAdd(w.ccount + h, 1);
        w.clist[(int64_t)h * p.T + at] = order_key(cj);
        w.clj[(int64_t)h * p.T + at] = j;
      }
      __syncthreads();
    }
  }
  chain_release();
  // the last block of this head to get here takes the selection step
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(w.rcount + h, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (which == 0) {
    // θ from the probe; done when every key left out is below it
    const int n = top_of_list(p, w, h, kk, S);
    const int jt = S.outj[kk - 1];
    const double th = jt != INT_MAX ? key_value(S.outk[kk - 1]) : -INFINITY;
    const bool done = !(tau > 0.f) || (jt != INT_MAX && th >= (double)tau * kBoundMargin);
    if (threadIdx.x == 0) {
      w.cdone[h] = done;
      w.ctheta[h] = th;
      if (done) {
        w.rows_eval[h] += (unsigned long long)n;
        w.ccount[h] = 0;   // the list is consumed; otherwise the second launch extends it
      }
    }
    if (done) append_picks(p, w, h, s0, kk, S);
  } else {
    pick_from_list(p, w, h, s0, kk, S);
  }
  if (threadIdx.x == 0) w.rcount[h] = 0;
}

// ------------------------------------------------- highest attention --
// AM-Highest ("Fast KV Compaction via Attention Matching": zhichai.net/en
// summary, "Method Family and Trade-offs"; youleyou.com rewrite, the
// highest-attention keys): each head keeps the t keys with the largest total
// attention over its reference queries, score_j = Σ_i Φ_ij / m_i (query i's
// softmax probability of key j; the shift cancels), ties to the lower key.

// 1 / m_i per query in fp64, 0 for a query without mass or past n.
__global__ void __launch_bounds__(256) k_inv_m(Problem p, Work w) {
  const int h = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= p.ldn) return;
  const double m = w.m[(int64_t)h * p.ldn + i];
  w.inv_m[(int64_t)h * p.ldn + i] = (i < p.n && m > 0.0) ? 1.0 / m : 0.0;
}

// score_j for every key, into w.cnorm [H][T]: fp64 sums of the stored fp32
// features times 1 / m_i; four warps per key, a quarter of the queries each,
// eight float4 columns per lane in flight, the quarters added in a fixed order.
__global__ void __launch_bounds__(kSelThreads) k_score(Problem p, Work w) {
  __shared__ double part[kRowsPerBlock][kRowSplit];
  const int h = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slot = warp / kRowSplit, quarter = warp % kRowSplit;
  const double2* im2 = reinterpret_cast<const double2*>(w.inv_m + (int64_t)h * p.ldn);
  const int n4 = p.ldn >> 2;
  const int per = (n4 + kRowSplit - 1) / kRowSplit;
  const int c0 = quarter * per, c1 = min(n4, c0 + per);
  const int Th = w.Th[h];
  for (int j0 = blockIdx.x * kRowsPerBlock; j0 < p.T; j0 += gridDim.x * kRowsPerBlock) {
    const int j = j0 + slot;
    const bool on = j < Th;
    double a[4] = {0.0, 0.0, 0.0, 0.0};
    if (on) {
      const float4* row = reinterpret_cast<const float4*>(w.phiT + ((int64_t)h * p.T + j) * p.ldn);
      for (int i0 = c0 + lane; i0 < c1; i0 += 32 * kRowLoads) {
        float4 x[kRowLoads];
#pragma unroll
        for (int u = 0; u < kRowLoads; ++u) {
          const int i = i0 + 32 * u;
          x[u] = i < c1 ? __ldcs(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kRowLoads; ++u) {
          const int i = i0 + 32 * u;
          if (i < c1) {
            const double2 lo = __ldg(im2 + 2 * i), hi = __ldg(im2 + 2 * i + 1);
            a[0] = fma((double)x[u].x, lo.x, a[0]);
            a[1] = fma((double)x[u].y, lo.y, a[1]);
            a[2] = fma((double)x[u].z, hi.x, a[2]);
            a[3] = fma((double)x[u].w, hi.y, a[3]);
          }
        }
      }
    }
    const double c = warp_sum((a[0] + a[1]) + (a[2] + a[3]));
    if (lane == 0) part[slot][quarter] = c;
    __syncthreads();
    // a key past the head's own (j >= Th) scores −1, below every real key's score
    if (j < p.T && quarter == 0 && lane == 0)
      w.cnorm[(int64_t)h * p.T + j] = on ? (part[slot][0] + part[slot][1]) + (part[slot][2] + part[slot][3]) : -1.0;
    __syncthreads();
  }
}

// Each head's keys in pick order (larger score first, ties to the lower key):
// a bitonic sort of (order key, key index) pairs in shared memory, one block
// per head; the first t become the head's picks, in that order.
__global__ void __launch_bounds__(kBoundThreads) k_pick_highest(Problem p, Work w) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int h = blockIdx.x;
  int n2 = 1;
  while (n2 < p.T) n2 <<= 1;
  uint64_t* key = reinterpret_cast<uint64_t*>(smem);
  int* idx = reinterpret_cast<int*>(key + n2);
  const double* sc = w.cnorm + (int64_t)h * p.T;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    key[i] = i < p.T ? order_key(sc[i]) : 0ull;
    idx[i] = i < p.T ? i : INT_MAX;
  }
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int l = i ^ jj;
        if (l > i) {
          const uint64_t a = key[i], b = key[l];
          const int ja = idx[i], jb = idx[l];
          // segments with bit k clear end in pick order, the others reversed
          const bool swap = (i & k) == 0 ? before(b, jb, a, ja) : before(a, ja, b, jb);
          if (swap) {
            key[i] = b; key[l] = a;
            idx[i] = jb; idx[l] = ja;
          }
        }
      }
      __syncthreads();
    }
  }
  const int t = w.t[h];
  const int64_t base = w.cu_t[h];
  uint8_t* sel = w.sel + (int64_t)h * p.T;
  for (int l = threadIdx.x; l < t; l += blockDim.x) {
    const int j = idx[l];   // t <= T: a real key
    w.picks[base + l] = j;
    w.pick_corr[base + l] = (float)key_value(key[l]);
    sel[j] = 1;
  }
  if (threadIdx.x == 0) w.rows_eval[h] = (unsigned long long)w.Th[h];
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
  return cudaGetLastError();
}

cudaError_t launch_corr_bounded(const Problem& p, const Work& w, int pass, int active, cudaStream_t s) {
  dim3 gb((p.T + 255) / 256, active);
  AM_LAUNCH(AM_STAGE_ROWS, s, launch_chained(k_gbound, gb, dim3(256), 0, s, p, w, pass));
  const int sel_smem = (int)sizeof(SelScratch);
  cudaFuncSetAttribute(k_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, sel_smem);
  dim3 gr(rows_ctas_per_head(active), active);
  AM_LAUNCH(AM_STAGE_ROWS, s, launch_chained(k_rows, gr, dim3(kSelThreads), sel_smem, s, p, w, pass, 0));
  AM_LAUNCH(AM_STAGE_ROWS, s, launch_chained(k_rows, gr, dim3(kSelThreads), sel_smem, s, p, w, pass, 1));
  return cudaGetLastError();
}

cudaError_t launch_select_highest(const Problem& p, const Work& w, cudaStream_t s) {
  dim3 gi((p.ldn + 255) / 256, p.H);
  AM_LAUNCH(AM_STAGE_CORR, s, k_inv_m<<<gi, 256, 0, s>>>(p, w));
  const int per_head = (8 * 148 + p.H - 1) / p.H;
  dim3 gs(min((p.T + kRowsPerBlock - 1) / kRowsPerBlock, per_head < 1 ? 1 : per_head), p.H);
  AM_LAUNCH(AM_STAGE_CORR, s, k_score<<<gs, kSelThreads, 0, s>>>(p, w));
  int n2 = 1;
  while (n2 < p.T) n2 <<= 1;
  const int sm = n2 * (int)(sizeof(uint64_t) + sizeof(int));   // T <= kSortSmemKeys: at most 192 KiB
  cudaFuncSetAttribute(k_pick_highest, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
  AM_LAUNCH(AM_STAGE_SELECT, s, k_pick_highest<<<p.H, kBoundThreads, sm, s>>>(p, w));
  return cudaGetLastError();
}

}  // namespace am
