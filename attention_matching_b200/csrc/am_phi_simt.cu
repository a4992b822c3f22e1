// Feature pass on CUDA cores: shift c_h = max s_ij, Φᵀ = exp(s − c_h) in the
// key-major layout, then Y = ΦV/m and m = Φ·1.
//
// "Fast KV Compaction via Attention Matching", zhichai.net deep dive §1.6:
// Φ_ij = exp(q_i·k_j) and m_i = Σ_j Φ_ij (here with the 1/√d scale, an
// optional prior key bias and one per-head shift); xinfinite.net article §2
// step 3: the value fit matches the original local attention output Y.
//
// fp32 inputs always take this path: the tensor-core kinds available for fp32
// operands (tf32) would round the logits to 10 mantissa bits.
#include "am_internal.cuh"
#include "am_profile.cuh"

#include <float.h>

namespace am {
namespace {

constexpr int TQ = 64, TK = 64, DK = 32;   // query tile, key tile, d chunk

// Order-preserving float <-> uint32 map for atomicMax on floats.
__device__ __forceinline__ uint32_t f2ord(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord2f(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}

// Loads a [64 × 32] slab (rows r0.., cols k0..) of a row-major [rows][d] input
// into smem transposed as dst[k][row], zero-filling out-of-range entries.
__device__ __forceinline__ void load_tile_T(float (*dst)[TQ + 4], const void* src, int64_t base,
                                            int rows, int r0, int k0, int d, int dtype) {
  for (int e = threadIdx.x; e < TQ * DK; e += blockDim.x) {
    int row = e / DK, k = e % DK;
    int gr = r0 + row, gk = k0 + k;
    float v = 0.f;
    if (gr < rows && gk < d) v = load_in(src, base + (int64_t)gr * d + gk, dtype);
    dst[k][row] = v;
  }
}

// One 64×64 tile of s = Q Kᵀ·scale (+ bias): thread (tx, ty) owns queries
// i0 + 4tx .. +3 and keys j0 + 4ty .. +3.
__device__ __forceinline__ void tile_logits(const Problem& p, const void* Q, const void* K, int h,
                                            int64_t krow0, int Th, int i0, int j0, float (*Qs)[TQ + 4],
                                            float (*Ks)[TK + 4], float acc[4][4]) {
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
  const int64_t qbase = (int64_t)h * p.n * p.d, kbase = krow0 * p.d;
  for (int k0 = 0; k0 < p.d; k0 += DK) {
    __syncthreads();
    load_tile_T(Qs, Q, qbase, p.n, i0, k0, p.d, p.in_dtype);
    load_tile_T(Ks, K, kbase, Th, j0, k0, p.d, p.in_dtype);
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < DK; ++k) {
      float4 qa = *reinterpret_cast<const float4*>(&Qs[k][tx * 4]);
      float4 kb = *reinterpret_cast<const float4*>(&Ks[k][ty * 4]);
      float qv[4] = {qa.x, qa.y, qa.z, qa.w}, kv[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(qv[a], kv[b], acc[a][b]);
    }
  }
}

__global__ void __launch_bounds__(256) k_shift_max(Problem p, Work w, const void* Q, const void* K,
                                                   const float* key_bias, uint32_t* out) {
  __shared__ __align__(16) float Qs[DK][TQ + 4];
  __shared__ __align__(16) float Ks[DK][TK + 4];
  __shared__ float red[8];
  const int h = blockIdx.z, i0 = blockIdx.x * TQ, j0 = blockIdx.y * TK;
  const int Th = w.Th[h];
  const int64_t krow0 = w.koff[h];
  if (j0 >= Th) return;   // the whole block: no key of this head here
  float acc[4][4];
  tile_logits(p, Q, K, h, krow0, Th, i0, j0, Qs, Ks, acc);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float mx = -FLT_MAX;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    int j = j0 + ty * 4 + b;
    if (j >= Th) continue;
    float bj = p.has_bias ? key_bias[krow0 + j] : 0.f;
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      int i = i0 + tx * 4 + a;
      if (i < p.n) mx = fmaxf(mx, fmaf(acc[a][b], p.scale, bj));
    }
  }
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = red[0];
    for (int k = 1; k < 8; ++k) v = fmaxf(v, red[k]);
    atomicMax(out + h, f2ord(v));
  }
}

__global__ void k_shift_init(uint32_t* out, int H) {
  int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) out[h] = f2ord(-FLT_MAX);
}

__global__ void k_shift_decode(uint32_t* io, int H) {
  int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) reinterpret_cast<float*>(io)[h] = ord2f(io[h]);
}

__global__ void k_shift_copy(const float* src, float* dst, int H) {
  int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) dst[h] = src[h];
}

// Φᵀ[h][j][i] = exp(s_ij − c_h) for i < n, 0 in the padding n <= i < ldn.
__global__ void __launch_bounds__(256) k_phi(Problem p, Work w, const void* Q, const void* K,
                                             const float* key_bias, const float* shift,
                                             float* phiT, __nv_bfloat16* phiT16) {
  __shared__ __align__(16) float Qs[DK][TQ + 4];
  __shared__ __align__(16) float Ks[DK][TK + 4];
  const int h = blockIdx.z, i0 = blockIdx.x * TQ, j0 = blockIdx.y * TK;
  const int Th = w.Th[h];
  const int64_t krow0 = w.koff[h];
  if (j0 >= Th) return;   // the whole block: keys past the head's own are never read
  float acc[4][4];
  tile_logits(p, Q, K, h, krow0, Th, i0, j0, Qs, Ks, acc);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const float c = shift[h];
  const int ibase = i0 + tx * 4;
  if (ibase >= p.ldn) return;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    int j = j0 + ty * 4 + b;
    if (j >= Th) continue;
    // one rounding of s·scale + b − c (no intermediate rounding of s, |s| ≈ c)
    const float bmc = p.has_bias ? key_bias[krow0 + j] - c : -c;
    float v[4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
      v[a] = (ibase + a < p.n) ? expf(fmaf(acc[a][b], p.scale, bmc)) : 0.f;
    *reinterpret_cast<float4*>(phiT + ((int64_t)h * p.T + j) * p.ldn + ibase) =
        make_float4(v[0], v[1], v[2], v[3]);
    if (phiT16) {   // bf16 copy streamed by the correlation pass
      __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
      uint2 pk = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
      *reinterpret_cast<uint2*>(phiT16 + ((int64_t)h * p.T + j) * p.ldn + ibase) = pk;
    }
  }
}

// Y[i][:] = Σ_j Φᵀ[j][i] V[j][:] / m_i and m_i = Σ_j Φᵀ[j][i]; also r = m.
// Thread (tx, ty): queries i0 + 4tx .. +3, value dims ty·DPT .. +DPT-1.
template <int DPT>
__global__ void __launch_bounds__(256) k_y_m(Problem p, Work w, const void* V, const float* phiT,
                                             float* Y, double* m, float* r) {
  constexpr int DT = 16 * DPT;
  __shared__ __align__(16) float Ps[DK][TQ + 4];
  __shared__ float Vs[DK][DT + 1];
  __shared__ double msum[TQ];
  const int h = blockIdx.y, i0 = blockIdx.x * TQ;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][DPT];
  double ms[4] = {0.0, 0.0, 0.0, 0.0};   // m is the exact sum of the stored values
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < DPT; ++c) acc[a][c] = 0.f;
  const float* P = phiT + (int64_t)h * p.T * p.ldn;
  const int Th = w.Th[h];
  const int64_t vbase = w.koff[h] * p.d;
  for (int j0 = 0; j0 < Th; j0 += DK) {
    __syncthreads();
    for (int e = threadIdx.x; e < DK * TQ; e += blockDim.x) {
      int jj = e / TQ, ii = e % TQ;
      int j = j0 + jj, i = i0 + ii;
      Ps[jj][ii] = (j < Th && i < p.ldn) ? P[(int64_t)j * p.ldn + i] : 0.f;
    }
    for (int e = threadIdx.x; e < DK * DT; e += blockDim.x) {
      int jj = e / DT, c = e % DT;
      int j = j0 + jj;
      Vs[jj][c] = (j < Th && c < p.d) ? load_in(V, vbase + (int64_t)j * p.d + c, p.in_dtype) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < DK; ++jj) {
      float4 pa = *reinterpret_cast<const float4*>(&Ps[jj][tx * 4]);
      float pv[4] = {pa.x, pa.y, pa.z, pa.w};
#pragma unroll
      for (int a = 0; a < 4; ++a) ms[a] += (double)pv[a];
#pragma unroll
      for (int c = 0; c < DPT; ++c) {
        float vv = Vs[jj][ty * DPT + c];
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[a][c] = fmaf(pv[a], vv, acc[a][c]);
      }
    }
  }
  // every ty holds the same m partial; keep ty == 0's
  if (ty == 0) {
#pragma unroll
    for (int a = 0; a < 4; ++a) msum[tx * 4 + a] = ms[a];
  }
  __syncthreads();
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    int i = i0 + tx * 4 + a;
    const double mi = msum[tx * 4 + a];
    const double im = mi > 0.0 ? 1.0 / mi : 0.0;   // no mass (all features underflowed): zero target
    if (i < p.n) {
#pragma unroll
      for (int c = 0; c < DPT; ++c) {
        int cc = ty * DPT + c;
        if (cc < p.d) Y[((int64_t)h * p.n + i) * p.d + cc] = (float)((double)acc[a][c] * im);
      }
    }
    // every feature of this reference query underflowed: it carries no mass
    if (ty == 0 && i < p.n && !(mi > 0.0)) record_status(w.status + h, AM_WARN_MASS_UNDERFLOW);
    if (ty == 0 && i < p.ldn) {
      const double v = (i < p.n) ? mi : 0.0;
      m[(int64_t)h * p.ldn + i] = v;
      r[(int64_t)h * p.ldn + i] = (float)v;
    }
  }
}

}  // namespace

cudaError_t launch_shift_max(const Problem& p, const Work& w, const void* Q, const void* K, const float* key_bias,
                             float* shift, cudaStream_t s) {
  uint32_t* u = reinterpret_cast<uint32_t*>(shift);
  AM_LAUNCH(AM_STAGE_SHIFT, s, k_shift_init<<<(p.H + 127) / 128, 128, 0, s>>>(u, p.H));
  dim3 grid((p.n + TQ - 1) / TQ, (p.T + TK - 1) / TK, p.H);
  AM_LAUNCH(AM_STAGE_SHIFT, s, k_shift_max<<<grid, 256, 0, s>>>(p, w, Q, K, key_bias, u));
  AM_LAUNCH(AM_STAGE_SHIFT, s, k_shift_decode<<<(p.H + 127) / 128, 128, 0, s>>>(u, p.H));
  return cudaGetLastError();
}

cudaError_t launch_phi(const Problem& p, const void* Q, const void* K, const float* key_bias,
                       const Work& w, cudaStream_t s) {
  dim3 grid((p.ldn + TQ - 1) / TQ, (p.T + TK - 1) / TK, p.H);
  AM_LAUNCH(AM_STAGE_PHI, s, k_phi<<<grid, 256, 0, s>>>(p, w, Q, K, key_bias, w.shift, w.phiT, w.phiT16));
  return cudaGetLastError();
}

cudaError_t launch_y_m(const Problem& p, const void* V, const Work& w, cudaStream_t s) {
  dim3 grid((p.ldn + TQ - 1) / TQ, p.H);
  if (p.d <= 16) AM_LAUNCH(AM_STAGE_TARGET, s, k_y_m<1><<<grid, 256, 0, s>>>(p, w, V, w.phiT, w.Y, w.m, w.r));
  else if (p.d <= 32) AM_LAUNCH(AM_STAGE_TARGET, s, k_y_m<2><<<grid, 256, 0, s>>>(p, w, V, w.phiT, w.Y, w.m, w.r));
  else if (p.d <= 64) AM_LAUNCH(AM_STAGE_TARGET, s, k_y_m<4><<<grid, 256, 0, s>>>(p, w, V, w.phiT, w.Y, w.m, w.r));
  else if (p.d <= 128) AM_LAUNCH(AM_STAGE_TARGET, s, k_y_m<8><<<grid, 256, 0, s>>>(p, w, V, w.phiT, w.Y, w.m, w.r));
  else AM_LAUNCH(AM_STAGE_TARGET, s, k_y_m<16><<<grid, 256, 0, s>>>(p, w, V, w.phiT, w.Y, w.m, w.r));
  return cudaGetLastError();
}

cudaError_t launch_shift_init(float* shift, int H, cudaStream_t s) {
  AM_LAUNCH(AM_STAGE_SHIFT, s, k_shift_init<<<(H + 127) / 128, 128, 0, s>>>(reinterpret_cast<uint32_t*>(shift), H));
  return cudaGetLastError();
}

cudaError_t launch_shift_decode(float* shift, int H, cudaStream_t s) {
  AM_LAUNCH(AM_STAGE_SHIFT, s, k_shift_decode<<<(H + 127) / 128, 128, 0, s>>>(reinterpret_cast<uint32_t*>(shift), H));
  return cudaGetLastError();
}

// exposed for the orchestrator: copy a caller-supplied shift into the workspace
cudaError_t launch_shift_copy(const float* src, float* dst, int H, cudaStream_t s) {
  AM_LAUNCH(AM_STAGE_SHIFT, s, k_shift_copy<<<(H + 127) / 128, 128, 0, s>>>(src, dst, H));
  return cudaGetLastError();
}

}  // namespace am
