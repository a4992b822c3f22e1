// Value-fit normal equations AᵀA and AᵀY on the 5th-generation tensor cores
// (tcgen05, TMEM, TMA) for bf16 problems with d in {64, 128}.
//
// "Fast KV Compaction via Attention Matching": with C_k and β fixed, C_v is
// the ordinary least-squares fit of the original attention outputs
// (xinfinite.net article §2 step 3; the youleyou.com rewrite, the OLS step),
// here through the ridge normal equations (AᵀA + λI) C_v = AᵀY.
//
// Operands.  A (key-major, [t][ldn] per head, each entry an fp32 value) and
// Y ([n][d] fp32) are each stored as three bf16 planes with
// x = hi + mid + lo exactly (bf16 keeps 8 significant bits, fp32 24).  The
// products of x·y kept are hi·hi, hi·mid, mid·hi, hi·lo, lo·hi and mid·mid
// (the dropped terms are below 2^-24 relative), each an exact bf16 product
// accumulated in fp32 by the tensor core over at most kQuerySplit queries;
// those partial sums are added in fp64 (by the query-split reduction).
// Measured on the CPU for the pages' workloads (emulating this arithmetic):
// the value fit's output moves by at most 1e-5 relative against the float64
// reference, far inside the 2e-3 acceptance.
//
// One CTA per (output tile, head, query split).  Gram tiles are 128 × 128
// blocks of AᵀA on or above the diagonal (a diagonal tile reuses its A tile
// as the B operand); a target tile is 128 × d of AᵀY with Y as an MN-major B
// operand.  Warp roles: warp 0 TMA producer (64-query stages, two-deep ring),
// warp 1 MMA issuer (one thread, M = 128, K = 16 per instruction), warp 2
// TMEM allocation, warps 4-7 the epilogue (thread r owns output row r, TMEM
// lane r).  Every wait is bounded as in the feature pass.  No cluster
// multicast.
#include "am_internal.cuh"
#include "am_tcgen05.cuh"
#include "am_profile.cuh"

#include <algorithm>

namespace am {
namespace {

constexpr int NM = 128;            // output rows per tile (TMEM lanes)
constexpr int NG = 128;            // output columns of a Gram tile
constexpr int KC = 64;             // queries per stage: one 128-byte bf16 row
constexpr int NSTAGES = 2;
constexpr int kNtThreads = 256;    // 4 control warps + one epilogue warpgroup
constexpr uint32_t kNtTmemCols = 128;
constexpr int kNPairs = 6;         // (hi,hi) (hi,mid) (mid,hi) (hi,lo) (lo,hi) (mid,mid)

struct NtPlan {
  uint32_t a_bytes, b_bytes, off_a, off_b, off_bar, total;
};

__host__ __device__ inline NtPlan nt_plan(int D) {
  NtPlan P{};
  P.a_bytes = 3 * NM * KC * 2;                 // three planes of [128 picks][64 queries]
  const uint32_t bg = 3 * NG * KC * 2;         // three planes of [128 picks][64 queries]
  const uint32_t by = 3 * KC * D * 2;          // three planes of [64 queries][d]
  P.b_bytes = bg > by ? bg : by;
  P.off_a = 0;
  P.off_b = NSTAGES * P.a_bytes;
  P.off_bar = P.off_b + NSTAGES * P.b_bytes;
  P.total = P.off_bar + 16 * 8 + 1024;         // barriers, slack to align the base to 1024
  return P;
}

__device__ __forceinline__ void pair_planes(int k, int& qa, int& qb) {
  // (0,0) (0,1) (1,0) (0,2) (2,0) (1,1)
  qa = k == 2 ? 1 : k == 4 ? 2 : k == 5 ? 1 : 0;
  qb = k == 1 ? 1 : k == 3 ? 2 : k == 5 ? 1 : 0;
}

template <int D>
__global__ void __launch_bounds__(kNtThreads, 1)
k_normal_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmY, Problem p, Work w,
            int splits, int kchunk, int64_t part_stride) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int h = blockIdx.y, z = blockIdx.z;
  const int t = w.t[h];
  const int ta = (t + NM - 1) / NM;
  const int ntri = ta * (ta + 1) / 2;
  int tile = blockIdx.x;
  if (tile >= ntri + ta) return;                 // the whole CTA leaves
  const bool gram = tile < ntri;
  int ta0, tb0 = 0;
  if (gram) {
    int r = 0;
    while (tile >= ta - r) { tile -= ta - r; ++r; }
    ta0 = r;
    tb0 = r + tile;
  } else {
    ta0 = tile - ntri;
  }
  const bool diag = gram && ta0 == tb0;
  const int a0 = ta0 * NM, b0 = tb0 * NG;
  const int64_t base = w.cu_t[h];
  const int64_t sum_t = w.cu_t[p.H];
  // queries [q0, q1) of this split, whole 64-query stages (past ldn the map reads zeros)
  const int q0 = z * kchunk, q1 = min(p.ldn, q0 + kchunk);
  const int nchunk = q1 > q0 ? (q1 - q0 + KC - 1) / KC : 0;

  const NtPlan P = nt_plan(D);
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = sm + P.off_a;
  unsigned char* sB = sm + P.off_b;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P.off_bar);
  uint64_t* full = bars;                 // [NSTAGES]
  uint64_t* empty = bars + NSTAGES;      // [NSTAGES]
  uint64_t* acc_full = bars + 2 * NSTAGES;
  uint64_t* drain = acc_full + 1;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_stop;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* status = w.status + h;
  volatile int* abort_flag = &s_abort;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < NSTAGES; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init_fence();
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kNtTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tacc = s_tmem;
  const uint32_t b_plane = gram ? NG * KC * 2 : KC * D * 2;   // bytes of one B plane tile
  const uint32_t tx_bytes = P.a_bytes + (diag ? 0u : 3 * b_plane);

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      int issued[NSTAGES] = {};
      for (int c = 0; c < nchunk; ++c) {
        const int s = c % NSTAGES, use = c / NSTAGES;
        if (use > 0 && !mbar_wait(empty + s, (use - 1) & 1, abort_flag, status, p.wait_cycles)) break;
        mbar_expect_tx(full + s, tx_bytes);
        const int qx = q0 + c * KC;
        unsigned char* dA = sA + s * P.a_bytes;
        unsigned char* dB = sB + s * P.b_bytes;
        for (int q = 0; q < 3; ++q)
          tma_load_2d(dA + q * NM * KC * 2, &tmA, full + s, qx, (int)(q * sum_t + base + a0));
        if (gram && !diag) {
          for (int q = 0; q < 3; ++q)
            tma_load_2d(dB + q * b_plane, &tmA, full + s, qx, (int)(q * sum_t + base + b0));
        } else if (!gram) {
          for (int q = 0; q < 3; ++q)
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(dB + q * b_plane + kb * KC * 128, &tmY, full + s, kb * 64, qx, q * p.H + h);
        }
        issued[s] = use + 1;
      }
      // copies still in flight must land before the CTA releases its memory
      for (int s = 0; s < NSTAGES; ++s)
        if (issued[s] > 0) {
          const long long t0 = clock64();
          while (!mbar_try_wait(full + s, (issued[s] - 1) & 1) && clock64() - t0 < kDrainCycles) {}
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc = gram ? instr_desc(NG, false) : instr_desc(D, true);
      bool ok = true;
      for (int c = 0; ok && c < nchunk; ++c) {
        const int s = c % NSTAGES, use = c / NSTAGES;
        if (!mbar_wait(full + s, use & 1, abort_flag, status, p.wait_cycles)) { ok = false; break; }
        tc_fence_after();
        const uint32_t abase = smem_u32(sA + s * P.a_bytes);
        const uint32_t bbase = diag ? abase : smem_u32(sB + s * P.b_bytes);
#pragma unroll
        for (int kk = 0; kk < KC / 16; ++kk) {
#pragma unroll
          for (int k = 0; k < kNPairs; ++k) {
            int qa, qb;
            pair_planes(k, qa, qb);
            const uint64_t ad = smem_desc(abase + qa * NM * KC * 2 + kk * 32, 16, 1024);
            const uint64_t bd = gram ? smem_desc(bbase + qb * b_plane + kk * 32, 16, 1024)
                                     : smem_desc(bbase + qb * b_plane + kk * 16 * 128, KC * 128, 1024);
            tc_mma(tacc, ad, bd, idesc, (c > 0 || kk > 0 || k > 0) ? 1u : 0u);
          }
        }
        tc_commit(empty + s);
      }
      tc_commit(acc_full);
      // drain: every MMA this thread issued has completed before TMEM is freed
      tc_commit(drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kDrainCycles) {}
    }
  } else if (warp >= 4) {
    // --------------------------------------------------- epilogue ----
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const int a = a0 + r;
    if (threadIdx.x == 128) s_stop = mbar_wait(acc_full, 0, abort_flag, status, p.wait_cycles) ? 0 : 1;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    tc_fence_after();
    double* AtA = (splits == 1 ? w.AtA : w.nrm_part + z * part_stride) + w.cu_t2[h];
    double* AtY = (splits == 1 ? w.AtY : w.nrm_part + z * part_stride + w.cu_t2[p.H]) + base * p.d;
    const int ncol = gram ? NG : D;
    if (!s_stop) {
      for (int c0 = 0; c0 < ncol; c0 += 32) {
        float v[32];
        if (nchunk > 0) {
          tmem_ld32(tacc + lane_addr_base(qd) + c0, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = 0.f;
        }
        if (a < t) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int col = c0 + k;
            if (gram) {
              // one writer per element: on a diagonal tile row a takes b >= a
              // (the two triangles of a tile round differently in fp32)
              const int b = b0 + col;
              if (b < t && (!diag || b >= a)) {
                AtA[(int64_t)a * t + b] = (double)v[k];
                AtA[(int64_t)b * t + a] = (double)v[k];
              }
            } else if (col < p.d) {
              AtY[(int64_t)a * p.d + col] = (double)v[k];
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tacc), "r"(kNtTmemCols));
}

// Y [H][n][d] fp32 → three bf16 planes [3][H][n][d] with y = hi + mid + lo.
__global__ void k_split_y(const float* __restrict__ Y, __nv_bfloat16* __restrict__ planes, int64_t count) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x) {
    const float y = Y[e];
    const __nv_bfloat16 hi = __float2bfloat16_rn(y);
    const float r1 = y - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    planes[e] = hi;
    planes[count + e] = mid;
    planes[2 * count + e] = __float2bfloat16_rn(r2);
  }
}

template <int D>
cudaError_t launch_normal_tc_d(const Problem& p, const Work& w, cudaStream_t s) {
  const int64_t sum_t = w.sum_t;
  const int64_t ycount = (int64_t)p.H * p.n * p.d;
  AM_LAUNCH(AM_STAGE_NORMAL, s, k_split_y<<<4 * 148, 256, 0, s>>>(w.Y, w.Ypl, ycount));
  CUtensorMap mA, mY;
  if (!make_map_2d(&mA, w.Apl, 3 * sum_t, p.ldn, NM) || !make_map(&mY, w.Ypl, 3 * p.H, p.n, D, KC))
    return cudaErrorInvalidValue;
  const int ta = (p.max_t + NM - 1) / NM;
  const int tiles = ta * (ta + 1) / 2 + ta;
  const int nchunks = (p.ldn + KC - 1) / KC;
  // query splits: enough CTAs to fill the GPU, and at most kQuerySplit
  // queries summed in fp32 by one CTA
  int splits = (2 * 148 + tiles * p.H - 1) / (tiles * p.H);
  splits = std::max(splits, (p.ldn + kQuerySplit - 1) / kQuerySplit);
  splits = std::min(std::min(splits, kNormalMaxSplits), nchunks);
  const int kchunk = (nchunks + splits - 1) / splits * KC;
  const NtPlan P = nt_plan(D);
  auto kern = k_normal_tc<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.total);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles, p.H, splits);
  AM_LAUNCH(AM_STAGE_NORMAL, s, kern<<<grid, kNtThreads, P.total, s>>>(mA, mY, p, w, splits, kchunk, w.nrm_stride));
  if (splits > 1) launch_normal_reduce(w, splits, s);
  return cudaGetLastError();
}

}  // namespace

bool normal_tc_supported(const Problem& p) { return p.in_dtype == AM_BF16 && (p.d == 64 || p.d == 128); }

cudaError_t launch_normal_tc(const Problem& p, const Work& w, cudaStream_t s) {
  return p.d == 64 ? launch_normal_tc_d<64>(p, w, s) : launch_normal_tc_d<128>(p, w, s);
}

}  // namespace am
