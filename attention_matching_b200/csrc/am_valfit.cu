// Bias, packing and value fit, batched over heads.
//
// "Fast KV Compaction via Attention Matching": zhichai.net deep dive §1.6
// (β = log w); xinfinite.net article §2 step 3 and the youleyou.com rewrite
// (with C_k and β fixed, C_v is an ordinary least-squares fit of the local
// attention output); zhichai.net/en summary, "Engineering Practicality"
// (varlen per-head packing of the compacted cache).
//
//   k_finalize  rank picks by key position; β = b_S + log max(w, floor);
//               packed indices, β and C_k = K[S]
//   k_design    A_il = Φ_{i,S_l} w_l / Σ_l' Φ_{i,S_l'} w_l'  (key-major [t][ldn])
//   k_normal    AᵀA and AᵀY with fp64 sums of fp32 products
//   k_chol      λ = ridge·tr(AᵀA)/t, tiled Cholesky of AᵀA + λI (inverses of the
//               32×32 diagonal tiles kept)
//   k_trsm      C_v = (AᵀA + λI)⁻¹AᵀY by blocked forward and backward solves
#include "am_internal.cuh"
#include "am_profile.cuh"
#include "am_linalg.cuh"

namespace am {
namespace {

__global__ void __launch_bounds__(256) k_finalize(Problem p, Work w, const void* K,
                                                  const float* key_bias, void* C_k, float* beta,
                                                  int32_t* indices, float* w_out,
                                                  int32_t* pick_order, float* pick_corr) {
  const int h = blockIdx.x;
  const int t = w.t[h];
  const int64_t base = w.cu_t[h];
  __shared__ double scratch[33];
  // rank of each pick by key position (keys are distinct)
  for (int l = threadIdx.x; l < t; l += blockDim.x) {
    const int j = w.picks[base + l];
    int rank = 0;
    for (int q = 0; q < t; ++q) rank += w.picks[base + q] < j;
    w.sorted_slot[base + rank] = l;
    indices[base + rank] = j;
  }
  double wmax = 0.0;
  for (int l = threadIdx.x; l < t; l += blockDim.x) wmax = fmax(wmax, w.w[base + l]);
  for (int o = 16; o; o >>= 1) wmax = fmax(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = wmax;
  __syncthreads();
  if (threadIdx.x == 0) {
    double v = 0.0;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) v = fmax(v, scratch[k]);
    scratch[32] = v;
  }
  __syncthreads();
  wmax = scratch[32];
  const double floor_w = wmax > 0.0 ? (double)p.w_floor_rel * wmax : (double)p.w_floor_rel;
  for (int q = threadIdx.x; q < t; q += blockDim.x) {
    const int l = w.sorted_slot[base + q];
    const int j = w.picks[base + l];
    const double wl = w.w[base + l];
    const double we = fmax(wl, floor_w);
    w.w_eff[base + q] = we;
    const double bj = p.has_bias ? (double)key_bias[w.koff[h] + j] : 0.0;
    beta[base + q] = (float)(bj + log(we));
    if (w_out) w_out[base + q] = (float)wl;
    if (pick_order) pick_order[base + l] = j;
    if (pick_corr) pick_corr[base + l] = w.pick_corr[base + l];
  }
  __syncthreads();
  // C_k rows: exact copies of the chosen keys in the input dtype
  const int64_t total = (int64_t)t * p.d;
  for (int64_t e = threadIdx.x; e < total; e += blockDim.x) {
    const int q = (int)(e / p.d), c = (int)(e % p.d);
    const int j = indices[base + q];
    const int64_t src = (w.koff[h] + j) * p.d + c;
    const int64_t dst = (base + q) * p.d + c;
    if (p.in_dtype == AM_BF16)
      reinterpret_cast<__nv_bfloat16*>(C_k)[dst] = reinterpret_cast<const __nv_bfloat16*>(K)[src];
    else
      reinterpret_cast<float*>(C_k)[dst] = reinterpret_cast<const float*>(K)[src];
  }
}

constexpr int kDesignThreads = 256;
constexpr int kDesignChunk = 256;

__global__ void __launch_bounds__(kDesignThreads) k_design(Problem p, Work w) {
  const int h = blockIdx.y;
  const int t = w.t[h];
  const int64_t base = w.cu_t[h];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  __shared__ int sj[kDesignChunk];
  __shared__ double sw[kDesignChunk];
  const float* P0 = w.phiT + (int64_t)h * p.T * p.ldn;
  const bool live = i < p.n;
  double D = 0.0;
  for (int c0 = 0; c0 < t; c0 += kDesignChunk) {
    const int cn = min(kDesignChunk, t - c0);
    __syncthreads();
    for (int q = threadIdx.x; q < cn; q += blockDim.x) {
      sj[q] = w.picks[base + w.sorted_slot[base + c0 + q]];
      sw[q] = w.w_eff[base + c0 + q];
    }
    __syncthreads();
    if (live)
      for (int q = 0; q < cn; ++q) D += (double)P0[(int64_t)sj[q] * p.ldn + i] * sw[q];
  }
  const double invD = (live && D > 0.0) ? 1.0 / D : 0.0;
  for (int c0 = 0; c0 < t; c0 += kDesignChunk) {
    const int cn = min(kDesignChunk, t - c0);
    __syncthreads();
    for (int q = threadIdx.x; q < cn; q += blockDim.x) {
      sj[q] = w.picks[base + w.sorted_slot[base + c0 + q]];
      sw[q] = w.w_eff[base + c0 + q];
    }
    __syncthreads();
    if (i < p.ldn)
      for (int q = 0; q < cn; ++q) {
        const double a = live ? (double)P0[(int64_t)sj[q] * p.ldn + i] * sw[q] * invD : 0.0;
        const int64_t at = (base + c0 + q) * p.ldn + i;
        if (w.Apl) {
          // fp32 value as three bf16 planes, af = hi + mid + lo exactly
          const float af = (float)a;
          const __nv_bfloat16 hi = __float2bfloat16_rn(af);
          const float r1 = af - __bfloat162float(hi);
          const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
          const int64_t plane = w.cu_t[p.H] * p.ldn;
          w.Apl[at] = hi;
          w.Apl[plane + at] = mid;
          w.Apl[2 * plane + at] = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        } else {
          w.A[at] = (float)a;
        }
      }
  }
}

// AᵀA (upper tile triangle, mirrored) and AᵀY; one 64×64 output tile per
// block, 4×4 outputs per thread.  Operand tiles are converted to fp64 once,
// when staged in shared memory, so the inner loop is pure fp64 FMA.
constexpr int NT_ = 64;   // output tile edge
constexpr int NK_ = 16;   // query chunk

__global__ void __launch_bounds__(256) k_normal(Problem p, Work w, int splits, int64_t part_stride) {
  const int h = blockIdx.y;
  const int z = blockIdx.z;   // query split: rows [i_begin, i_end)
  const int chunk = ((p.n + splits - 1) / splits + NK_ - 1) / NK_ * NK_;
  const int i_begin = z * chunk, i_end = min(p.n, i_begin + chunk);
  const int t = w.t[h];
  const int ta = (t + NT_ - 1) / NT_, td = (p.d + NT_ - 1) / NT_;
  const int ntri = ta * (ta + 1) / 2;
  int tile = blockIdx.x;
  if (tile >= ntri + ta * td) return;
  const bool gram = tile < ntri;
  int ta0, tb0;
  if (gram) {
    int r = 0;
    while (tile >= ta - r) { tile -= ta - r; ++r; }
    ta0 = r;
    tb0 = r + tile;
  } else {
    tile -= ntri;
    ta0 = tile / td;
    tb0 = tile % td;
  }
  const int a0 = ta0 * NT_, b0 = tb0 * NT_;
  const int64_t base = w.cu_t[h];
  __shared__ double As[NK_][NT_ + 1];
  __shared__ double Bs[NK_][NT_ + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4] = {};
  const float* Yh = w.Y + (int64_t)h * p.n * p.d;
  // the next chunk's operands travel in registers while this one is multiplied
  constexpr int kPer = NK_ * NT_ / 256;   // elements per operand per thread (blockDim 256)
  float ra[kPer], rb[kPer];
  auto fetch = [&](int i0) {
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = threadIdx.x + u * 256;
      const int rr = e / NK_, ii = e % NK_;          // A rows are contiguous along queries
      const int a = a0 + rr, i = i0 + ii;
      ra[u] = (a < t && i < i_end) ? w.A[(base + a) * p.ldn + i] : 0.f;
      if (gram) {
        const int bb = b0 + rr;
        rb[u] = (bb < t && i < i_end) ? w.A[(base + bb) * p.ldn + i] : 0.f;
      } else {
        const int i2 = i0 + e / NT_, c = b0 + e % NT_;   // Y rows are contiguous along dims
        rb[u] = (i2 < i_end && c < p.d) ? Yh[(int64_t)i2 * p.d + c] : 0.f;
      }
    }
  };
  fetch(i_begin);
  for (int i0 = i_begin; i0 < i_end; i0 += NK_) {
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int e = threadIdx.x + u * 256;
      As[e % NK_][e / NK_] = (double)ra[u];
      if (gram) Bs[e % NK_][e / NK_] = (double)rb[u];
      else Bs[e / NT_][e % NT_] = (double)rb[u];
    }
    __syncthreads();
    if (i0 + NK_ < i_end) fetch(i0 + NK_);
#pragma unroll 4
    for (int ii = 0; ii < NK_; ++ii) {
      double x[4], y[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { x[u] = As[ii][ty + 16 * u]; y[u] = Bs[ii][tx + 16 * u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(x[u], y[v], acc[u][v]);
    }
  }
  // one split writes AᵀA / AᵀY directly; several write partials (reduced in order below)
  double* AtA = splits == 1 ? w.AtA : w.nrm_part + z * part_stride;
  double* AtY = splits == 1 ? w.AtY : w.nrm_part + z * part_stride + w.cu_t2[p.H];
  const int64_t gbase = w.cu_t2[h];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int a = a0 + ty + 16 * u, bb = b0 + tx + 16 * v;
      if (gram) {
        if (a < t && bb < t) {
          AtA[gbase + (int64_t)a * t + bb] = acc[u][v];
          AtA[gbase + (int64_t)bb * t + a] = acc[u][v];
        }
      } else if (a < t && bb < p.d) {
        AtY[(base + a) * p.d + bb] = acc[u][v];
      }
    }
}

// AᵀA and AᵀY = Σ over the query splits, added in split order.
__global__ void k_normal_reduce(int64_t n_ata, int64_t n_aty, int splits, int64_t part_stride, Work w) {
  const int64_t total = n_ata + n_aty;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    double acc = 0.0;
    for (int z = 0; z < splits; ++z) acc += w.nrm_part[z * part_stride + e];
    if (e < n_ata) w.AtA[e] = acc;
    else w.AtY[e - n_ata] = acc;
  }
}

// λ = ridge·tr(AᵀA)/t; packed Cholesky factor of AᵀA + λI and its
// reciprocal diagonal, written to the workspace (one CTA per head).
__global__ void __launch_bounds__(kCholThreads) k_chol(Problem p, Work w, int l_smem_max) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int h = blockIdx.x;
  const int t = w.t[h];
  const int64_t base = w.cu_t[h];
  const int64_t gbase = w.cu_t2[h];
  __shared__ double scratch[33];
  __shared__ int flag;
  const double* M = w.AtA + gbase;
  double tr = 0.0;
  for (int a = threadIdx.x; a < t; a += blockDim.x) tr += M[(int64_t)a * t + a];
  tr = block_sum(tr, scratch);
  const double lam = (double)p.ridge * tr / t;
  double* Lg = w.L + gbase;
  // tile scratch first, then (when it fits) the packed matrix
  double* scratch_t = reinterpret_cast<double*>(smem);
  double* L = t <= l_smem_max ? scratch_t + kTiledScratchDoubles : Lg;
  for (int a = threadIdx.x >> 5; a < t; a += blockDim.x >> 5)
    for (int c = threadIdx.x & 31; c <= a; c += 32) L[tri(a, c)] = M[(int64_t)a * t + c] + (a == c ? lam : 0.0);
  __syncthreads();
  // tiled factorization (32×32 tiles), of the shared-memory copy or in the workspace
  const int bad = block_cholesky_tiled(L, t, [](int) { return 0.0; }, scratch_t, &flag,
                                       w.dinv + (int64_t)32 * (base + 32 * h));
  if (bad >= 0) {
    if (threadIdx.x == 0) record_status(w.status + h, AM_ERR_NOT_SPD);
    for (int a = threadIdx.x; a < t; a += blockDim.x) w.w_eff[base + a] = 0.0;   // marks the head for k_trsm
    return;
  }
  if (L != Lg)
    for (int64_t e = threadIdx.x; e < tri(t, 0); e += blockDim.x) Lg[e] = L[e];
  // reciprocal diagonal in the NNLS vector slot (free after the bias is packed)
  for (int a = threadIdx.x; a < t; a += blockDim.x) w.bvec[base + a] = 1.0 / L[tri(a, a)];
}

// C_v[:, c0:c0+CW] = L⁻ᵀ L⁻¹ AᵀY[:, c0:c0+CW] (CW = 32, or 8 when 32 columns of
// a large head do not fit in shared memory) for one head per block, by 32-row
// blocks.  Forward, block [r0, r0+32): every row of the block takes its
// products with the solved rows above (thread = one row × four columns,
// factor rows read along their length), then the block is multiplied by the
// inverse of its diagonal tile (stored by the factorization).  Backward
// mirrors it from the bottom with the transposed tile inverse, then every
// row above takes the block's contribution.  No step is a sequential sweep.
// X is [t][CW + 1] in shared memory (odd row stride: a warp's lanes and the
// four-column groups land on distinct banks).
template <int CW>
__global__ void __launch_bounds__(256) k_trsm(Problem p, Work w, float* C_v, int l_smem_max) {
  extern __shared__ __align__(16) unsigned char smem[];
  constexpr int kTrsmCols = CW, kXs = CW + 1;
  constexpr int kGroups = CW / 4;                 // four-column groups per row
  const int h = blockIdx.x;
  const int c0 = blockIdx.y * kTrsmCols;
  const int t = w.t[h];
  const int64_t base = w.cu_t[h];
  const int64_t gbase = w.cu_t2[h];
  if (c0 >= p.d) return;
  const bool l_smem = t <= l_smem_max;
  double (*Dt)[33] = reinterpret_cast<double (*)[33]>(smem);   // a diagonal tile inverse
  double* X = reinterpret_cast<double*>(smem) + 32 * 33;        // [t][kXs]
  double* Ls = X + (size_t)t * kXs;
  const double* Dinv = w.dinv + (int64_t)32 * (base + 32 * h);
  const double* L = l_smem ? Ls : w.L + gbase;
  if (w.w_eff[base] == 0.0 && w.status[h] != 0) {           // factorization failed
    for (int e = threadIdx.x; e < t * kTrsmCols; e += blockDim.x) {
      const int r = e / kTrsmCols, c = c0 + e % kTrsmCols;
      if (c < p.d) C_v[(base + r) * p.d + c] = 0.f;
    }
    return;
  }
  if (l_smem)
    for (int64_t e = threadIdx.x; e < tri(t, 0); e += blockDim.x) Ls[e] = w.L[gbase + e];
  for (int e = threadIdx.x; e < t * kTrsmCols; e += blockDim.x) {
    const int r = e / kTrsmCols, cc = e % kTrsmCols, c = c0 + cc;
    X[r * kXs + cc] = c < p.d ? w.AtY[(base + r) * p.d + c] : 0.0;
  }
  __syncthreads();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // products: row r0 + rr, columns cg .. cg+3, kKs threads splitting the sum
  constexpr int kKs = 32 / CW;
  const int ks = tid % kKs, rr = tid / kKs / kGroups, cg = (tid / kKs % kGroups) * 4;
  const int nb = (t + 31) / 32;
  // Xb[0..bw) ← D⁻¹ Xb (or D⁻ᵀ Xb), D⁻¹ in Dt; all threads, two barriers
  auto diag_product = [&](double (*Di)[33], double* Xb, int bw, bool transposed, int rr, int cg, int ks) {
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    if (rr < bw) {
      const int j0 = transposed ? rr : 0, j1 = transposed ? bw : rr + 1;
      for (int j = j0 + ks; j < j1; j += kKs) {
        const double dij = transposed ? Di[j][rr] : Di[rr][j];
        const double* xj = Xb + j * kXs + cg;
        a0 = fma(dij, xj[0], a0); a1 = fma(dij, xj[1], a1); a2 = fma(dij, xj[2], a2); a3 = fma(dij, xj[3], a3);
      }
    }
#pragma unroll
    for (int o = 1; o < kKs; o <<= 1) {
      a0 += __shfl_xor_sync(0xffffffffu, a0, o);
      a1 += __shfl_xor_sync(0xffffffffu, a1, o);
      a2 += __shfl_xor_sync(0xffffffffu, a2, o);
      a3 += __shfl_xor_sync(0xffffffffu, a3, o);
    }
    __syncthreads();
    if (rr < bw && ks == 0) {
      double* xr = Xb + rr * kXs + cg;
      xr[0] = a0; xr[1] = a1; xr[2] = a2; xr[3] = a3;
    }
    __syncthreads();
  };
  // forward: y = L⁻¹ x
  for (int b = 0; b < nb; ++b) {
    const int r0 = b * 32, bw = min(32, t - r0);
    if (r0 > 0) {
      const bool live = rr < bw;
      const double* Lr = L + tri(r0 + (live ? rr : 0), 0);
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      if (live)
        for (int j = ks; j < r0; j += kKs) {
          const double l = Lr[j];
          const double* xj = X + j * kXs + cg;
          a0 = fma(l, xj[0], a0); a1 = fma(l, xj[1], a1); a2 = fma(l, xj[2], a2); a3 = fma(l, xj[3], a3);
        }
#pragma unroll
      for (int o = 1; o < kKs; o <<= 1) {   // the kKs partial sums are adjacent lanes
        a0 += __shfl_xor_sync(0xffffffffu, a0, o);
        a1 += __shfl_xor_sync(0xffffffffu, a1, o);
        a2 += __shfl_xor_sync(0xffffffffu, a2, o);
        a3 += __shfl_xor_sync(0xffffffffu, a3, o);
      }
      if (live && ks == 0) {
        double* xr = X + (r0 + rr) * kXs + cg;
        xr[0] -= a0; xr[1] -= a1; xr[2] -= a2; xr[3] -= a3;
      }
    }
    for (int e = tid; e < 32 * 32; e += blockDim.x) Dt[e >> 5][e & 31] = Dinv[(int64_t)b * 1024 + e];
    __syncthreads();
    diag_product(Dt, X + r0 * kXs, bw, false, rr, cg, ks);
  }
  // backward: z = L⁻ᵀ y
  for (int b = nb - 1; b >= 0; --b) {
    const int r0 = b * 32, bw = min(32, t - r0);
    for (int e = tid; e < 32 * 32; e += blockDim.x) Dt[e >> 5][e & 31] = Dinv[(int64_t)b * 1024 + e];
    __syncthreads();
    diag_product(Dt, X + r0 * kXs, bw, true, rr, cg, ks);
    // rows above the block: x_j −= Σ_{r in block} L[r][j] z_r (thread = row j × four
    // columns: thread tid takes row tid / kGroups and column group tid % kGroups,
    // so every (row, column group) pair above the block has exactly one owner)
    const int cga = (tid % kGroups) * 4;
    for (int j = tid / kGroups; j < r0; j += 256 / kGroups) {
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      for (int r = r0; r < r0 + bw; ++r) {
        const double l = L[tri(r, j)];
        const double* zr = X + r * kXs + cga;
        a0 = fma(l, zr[0], a0); a1 = fma(l, zr[1], a1); a2 = fma(l, zr[2], a2); a3 = fma(l, zr[3], a3);
      }
      double* xj = X + j * kXs + cga;
      xj[0] -= a0; xj[1] -= a1; xj[2] -= a2; xj[3] -= a3;
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < t * kTrsmCols; e += blockDim.x) {
    const int r = e / kTrsmCols, cc = e % kTrsmCols, c = c0 + cc;
    if (c < p.d) C_v[(base + r) * p.d + c] = (float)X[r * kXs + cc];
  }
}

}  // namespace

cudaError_t launch_finalize(const Problem& p, const Work& w, const void* K, const float* key_bias,
                            void* C_k, float* beta, int32_t* indices, float* w_out,
                            int32_t* pick_order, float* pick_corr, cudaStream_t s) {
  AM_LAUNCH(AM_STAGE_FINALIZE, s, k_finalize<<<p.H, 256, 0, s>>>(p, w, K, key_bias, C_k, beta, indices, w_out, pick_order, pick_corr));
  return cudaGetLastError();
}

cudaError_t launch_normal_reduce(const Work& w, int splits, cudaStream_t s) {
  AM_LAUNCH(AM_STAGE_NORMAL, s,
            k_normal_reduce<<<296, 256, 0, s>>>(w.nrm_ata, w.nrm_stride - w.nrm_ata, splits, w.nrm_stride, w));
  return cudaGetLastError();
}

cudaError_t launch_value_fit(const Problem& p, const Work& w, float* C_v, cudaStream_t s) {
  dim3 gd((p.ldn + kDesignThreads - 1) / kDesignThreads, p.H);
  AM_LAUNCH(AM_STAGE_DESIGN, s, k_design<<<gd, kDesignThreads, 0, s>>>(p, w));
  const int ta = (p.max_t + NT_ - 1) / NT_, td = (p.d + NT_ - 1) / NT_;
  const int blocks = (ta * (ta + 1) / 2 + ta * td) * p.H;
  int splits = (2 * 148 + blocks - 1) / blocks;
  splits = splits < 1 ? 1 : (splits > kNormalMaxSplits ? kNormalMaxSplits : splits);
  if (splits > (p.n + NK_ - 1) / NK_) splits = (p.n + NK_ - 1) / NK_;
  const int64_t part_stride = w.nrm_stride;
  if (w.Apl) {
    cudaError_t e = launch_normal_tc(p, w, s);
    if (e != cudaSuccess) return e;
  } else {
    dim3 gn(ta * (ta + 1) / 2 + ta * td, p.H, splits);
    AM_LAUNCH(AM_STAGE_NORMAL, s, k_normal<<<gn, 256, 0, s>>>(p, w, splits, part_stride));
    if (splits > 1) launch_normal_reduce(w, splits, s);
  }
  if (p.max_t >= kTiledSolveMinT) return launch_value_solve_tiled(p, w, C_v, s);
  // factor: heads with t <= tl keep it in shared memory (beside the tile scratch) while factoring
  const size_t cap = 226 * 1024;
  const size_t scr = kTiledScratchDoubles * sizeof(double);
  int tl = 0;
  while (tl < p.max_t && scr + (size_t)(tl + 1) * (tl + 2) / 2 * sizeof(double) <= cap) ++tl;
  const size_t sm = scr + (size_t)tl * (tl + 1) / 2 * sizeof(double);
  cudaFuncSetAttribute(k_chol, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cap);
  AM_LAUNCH(AM_STAGE_SOLVE, s, k_chol<<<p.H, kCholThreads, sm, s>>>(p, w, tl));
  // solves: a column slice of AᵀY plus (when it fits) the factor in shared memory
  const bool wide = (size_t)p.max_t * 33 * 8 <= 120 * 1024;
  const int CW = wide ? 32 : 8;
  const size_t xbytes = (size_t)p.max_t * (CW + 1) * 8 + 32 * 33 * 8;   // X and one tile inverse
  int tl2 = 0;
  while (tl2 < p.max_t && xbytes + (size_t)(tl2 + 1) * (tl2 + 2) / 2 * sizeof(double) <= cap) ++tl2;
  const size_t sm2 = xbytes + (size_t)tl2 * (tl2 + 1) / 2 * sizeof(double);
  dim3 g2(p.H, (p.d + CW - 1) / CW);
  if (wide) {
    cudaFuncSetAttribute(k_trsm<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cap);
    AM_LAUNCH(AM_STAGE_SOLVE, s, k_trsm<32><<<g2, 256, sm2, s>>>(p, w, C_v, tl2));
  } else {
    cudaFuncSetAttribute(k_trsm<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cap);
    AM_LAUNCH(AM_STAGE_SOLVE, s, k_trsm<8><<<g2, 256, sm2, s>>>(p, w, C_v, tl2));
  }
  return cudaGetLastError();
}

}  // namespace am
