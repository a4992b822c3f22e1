// Attention over a compacted cache: the consumer of the packed output.
//
// "Fast KV Compaction via Attention Matching": zhichai.net deep dive §4.1
// (the compacted block plugs into attention kernels that take an additive
// per-key bias) and §4.2 (per-head varlen segments, no padding);
// zhichai.net/en summary, "Engineering Practicality".  Head h's compacted
// keys C_k carry the bias β that makes their attention mass match the keys
// they replaced, so attention over [compacted block, fresh keys] is the
// mass-weighted mixture of the two blocks' local outputs.
//
//   k_attend   one block per (head, 8 queries), up to four key splits of 8
//              warps: split s takes every nsplit-th 32-key tile of the concatenated key
//              list (the compacted segment with bias β, then the fresh keys
//              with bias 0), staged in its own shared memory and shared by its
//              8 warps; in a warp, lane r scores key r of the tile against the
//              warp's query, and each lane keeps d/32 output dimensions of the
//              online-softmax value sum, in fp32.  The four splits' partial
//              softmaxes (running maximum, weight sum, weighted values) are
//              merged in shared memory at the end (split-key decoding inside
//              one block: no global scratch).
#include "am_internal.cuh"
#include "am_profile.cuh"

#include <math.h>

namespace am {
namespace {

constexpr int kAttWarps = 8;       // queries per block
constexpr int kAttMaxSplit = 4;    // key splits per block (fewer when shared memory is short)
constexpr int kAttTile = 32;       // keys per staged tile (one per lane)
constexpr int kAttPerLane = 8;     // d <= 32·8

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

// Shared memory of one key split for head dim d: K tile [32][d + 1], V tile
// [32][d], tile biases [32], warps' weights [8][32]; then the block's queries
// [8][d].  The merge reuses the splits' tiles.
__host__ __device__ inline size_t attend_split_floats(int d) {
  return (size_t)kAttTile * (d + 1) + (size_t)kAttTile * d + kAttTile + (size_t)kAttWarps * kAttTile;
}
__host__ __device__ inline size_t attend_smem_bytes(int d, int nsplit) {
  return sizeof(float) * (nsplit * attend_split_floats(d) + (size_t)kAttWarps * d);
}

template <typename TK>
__global__ void __launch_bounds__(kAttWarps * kAttMaxSplit * 32) k_attend(const TK* Q, int nq, int d, const TK* Ck,
                                                                          const float* beta, const float* Cv,
                                                                          const int64_t* cu_t, const TK* Kn,
                                                                          const TK* Vn, int Tn, float scale,
                                                                          float* out, int nsplit) {
  extern __shared__ __align__(16) float sm[];
  const int lane = threadIdx.x & 31;
  const int warp_all = threadIdx.x >> 5;
  const int split = warp_all / kAttWarps, warp = warp_all % kAttWarps;
  const int sthreads = kAttWarps * 32, stid = threadIdx.x % sthreads;   // threads of this split
  float* Ks = sm + split * attend_split_floats(d);   // [32][d + 1]
  float* Vs = Ks + kAttTile * (d + 1);               // [32][d]
  float* bs = Vs + kAttTile * d;                     // [32]
  float* ps = bs + kAttTile;                         // [8][32]
  float* qs = sm + nsplit * attend_split_floats(d);   // [8][d], shared by the splits
  const int h = blockIdx.y;
  const int i = blockIdx.x * kAttWarps + warp;
  const bool qlive = i < nq;
  if (split == 0)
    for (int e = lane; e < d; e += 32) qs[warp * d + e] = qlive ? to_f(Q[((int64_t)h * nq + i) * d + e]) : 0.f;
  __syncthreads();
  const int64_t c0 = cu_t[h];
  const int nc = (int)(cu_t[h + 1] - c0);
  const int ntot = nc + Tn;
  float acc[kAttPerLane];
#pragma unroll
  for (int u = 0; u < kAttPerLane; ++u) acc[u] = 0.f;
  float mrun = -INFINITY, l = 0.f;
  const int ntiles = (ntot + kAttTile - 1) / kAttTile;
  // every split runs the same number of iterations (barriers are block-wide)
  for (int it = 0; it < (ntiles + nsplit - 1) / nsplit; ++it) {
    const int k0 = (it * nsplit + split) * kAttTile;
    __syncthreads();   // the previous tile is no longer read
    for (int f = stid; f < kAttTile * d; f += sthreads) {
      const int r = f / d, e = f - r * d, g = k0 + r;
      float kv = 0.f, vv = 0.f;
      if (g < nc) {
        kv = to_f(Ck[(c0 + g) * d + e]);
        vv = Cv[(c0 + g) * d + e];
      } else if (g < ntot) {
        const int64_t o = ((int64_t)h * Tn + (g - nc)) * d + e;
        kv = to_f(Kn[o]);
        vv = to_f(Vn[o]);
      }
      Ks[r * (d + 1) + e] = kv;
      Vs[r * d + e] = vv;
    }
    if (stid < kAttTile) {
      const int g = k0 + stid;
      bs[stid] = g < nc ? beta[c0 + g] : (g < ntot ? 0.f : -INFINITY);
    }
    __syncthreads();
    // lane r: the logit of key r of the tile for this warp's query
    float dot = 0.f;
    const float* kr = Ks + lane * (d + 1);
    const float* qw = qs + warp * d;
    for (int e = 0; e < d; ++e) dot = fmaf(qw[e], kr[e], dot);
    const float b = bs[lane];
    const float sc = b == -INFINITY ? -INFINITY : fmaf(dot, scale, b);
    float mt = sc;
#pragma unroll
    for (int o = 16; o; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
    const float mnew = fmaxf(mrun, mt);
    if (mnew == -INFINITY) continue;   // warp-uniform: nothing finite yet
    const float a = expf(mrun - mnew);
    const float pj = sc == -INFINITY ? 0.f : expf(sc - mnew);
    float psum = pj;
#pragma unroll
    for (int o = 16; o; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    l = fmaf(l, a, psum);
    ps[warp * kAttTile + lane] = pj;
    __syncwarp();
#pragma unroll
    for (int u = 0; u < kAttPerLane; ++u) acc[u] *= a;
    for (int r = 0; r < kAttTile; ++r) {
      const float pr = ps[warp * kAttTile + r];
#pragma unroll
      for (int u = 0; u < kAttPerLane; ++u) {
        const int e = lane + 32 * u;
        if (e < d) acc[u] = fmaf(pr, Vs[r * d + e], acc[u]);
      }
    }
    __syncwarp();
    mrun = mnew;
  }
  // merge the splits' partial softmaxes: o = Σ_s e^{m_s − M} acc_s / Σ_s e^{m_s − M} l_s
  __syncthreads();   // the tiles are free
  float* part = sm;                                       // [split][warp][d] weighted values
  float* pm = sm + (size_t)nsplit * kAttWarps * d;     // [split][warp] running maxima
  float* pl = pm + nsplit * kAttWarps;                 // [split][warp] weight sums
#pragma unroll
  for (int u = 0; u < kAttPerLane; ++u) {
    const int e = lane + 32 * u;
    if (e < d) part[(split * kAttWarps + warp) * d + e] = acc[u];
  }
  if (lane == 0) {
    pm[split * kAttWarps + warp] = mrun;
    pl[split * kAttWarps + warp] = l;
  }
  __syncthreads();
  if (split != 0 || !qlive) return;
  float M = -INFINITY;
  for (int q = 0; q < nsplit; ++q) M = fmaxf(M, pm[q * kAttWarps + warp]);
  float wsum = 0.f, wq[kAttMaxSplit];
#pragma unroll
  for (int q = 0; q < kAttMaxSplit; ++q) {
    const float mq = q < nsplit ? pm[q * kAttWarps + warp] : -INFINITY;
    wq[q] = mq == -INFINITY ? 0.f : expf(mq - M);
    if (q < nsplit) wsum = fmaf(wq[q], pl[q * kAttWarps + warp], wsum);
  }
  const float il = wsum > 0.f ? 1.f / wsum : 0.f;
  float* orow = out + ((int64_t)h * nq + i) * d;
  for (int e = lane; e < d; e += 32) {
    float o = 0.f;
#pragma unroll
    for (int q = 0; q < kAttMaxSplit; ++q)
      if (q < nsplit) o = fmaf(wq[q], part[(q * kAttWarps + warp) * d + e], o);
    orow[e] = o * il;
  }
}

}  // namespace
}  // namespace am

using namespace am;

extern "C" am_status_t am_attend_packed(const void* Q, int32_t nq, int32_t d, int32_t num_heads, int32_t in_dtype,
                                        const void* C_k, const float* beta, const float* C_v,
                                        const int64_t* cu_t, const void* K_new, const void* V_new,
                                        int32_t T_new, float scale, float* out, void* stream) {
  if (!Q || !C_k || !beta || !C_v || !cu_t || !out) return AM_ERR_INVALID_ARG;
  if (nq < 1 || d < 1 || num_heads < 1 || T_new < 0) return AM_ERR_INVALID_ARG;
  if (T_new > 0 && (!K_new || !V_new)) return AM_ERR_INVALID_ARG;
  if (in_dtype != AM_BF16 && in_dtype != AM_FP32) return AM_ERR_INVALID_ARG;
  if (!isfinite(scale)) return AM_ERR_INVALID_ARG;
  if (d > 32 * kAttPerLane || num_heads > 65535) return AM_ERR_UNSUPPORTED;
  const float sc = scale > 0.f ? scale : (float)(1.0 / sqrt((double)d));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  dim3 grid((nq + kAttWarps - 1) / kAttWarps, num_heads);
  int nsplit = kAttMaxSplit;   // d <= 256: two splits always fit (at most 139 KiB)
  while (nsplit > 1 && attend_smem_bytes(d, nsplit) > 227 * 1024) nsplit >>= 1;
  const size_t sm = attend_smem_bytes(d, nsplit);
  const int threads = kAttWarps * 32 * nsplit;
  if (in_dtype == AM_BF16) {
    cudaFuncSetAttribute(k_attend<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    AM_LAUNCH(AM_STAGE_ATTEND, s,
              k_attend<__nv_bfloat16><<<grid, threads, sm, s>>>(
                  static_cast<const __nv_bfloat16*>(Q), nq, d, static_cast<const __nv_bfloat16*>(C_k), beta, C_v,
                  cu_t, static_cast<const __nv_bfloat16*>(K_new), static_cast<const __nv_bfloat16*>(V_new), T_new,
                  sc, out, nsplit));
  } else {
    cudaFuncSetAttribute(k_attend<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    AM_LAUNCH(AM_STAGE_ATTEND, s,
              k_attend<float><<<grid, threads, sm, s>>>(
                  static_cast<const float*>(Q), nq, d, static_cast<const float*>(C_k), beta, C_v, cu_t,
                  static_cast<const float*>(K_new), static_cast<const float*>(V_new), T_new, sc, out, nsplit));
  }
  return cudaGetLastError() == cudaSuccess ? AM_OK : AM_ERR_CUDA;
}
