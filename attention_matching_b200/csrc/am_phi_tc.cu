// Feature pass on the 5th-generation tensor cores (tcgen05, TMEM, TMA) for
// bf16 inputs with d in {64, 128}.
//
// "Fast KV Compaction via Attention Matching", zhichai.net deep dive §1.6:
// Φ_ij = exp(q_i·k_j) and m_i = Σ_j Φ_ij (with the 1/√d scale, an optional
// prior key bias and one per-head shift); xinfinite.net article §2 step 3:
// the value fit targets the original local attention output Y = ΦV/m.
//
// One CTA per (head, 128-query block), 20 warps:
//   warp 0   TMA producer: the query block once, then (key, value) tiles of
//            64 keys through a 3-stage ring
//   warp 1   MMA issuer (one thread): S = Q·Kᵀ into one of two TMEM
//            accumulators (kind::f16, bf16 in, fp32 out), then Y += P·V
//            from the epilogue's P tiles (PHI mode)
//   warp 2   TMEM allocation and release
//   warps 4-19 epilogue, four warpgroups: thread (g, r) owns query row r
//            (TMEM lane r) and 16 of each tile's 64 keys; it reads its logits,
//            forms p = exp(s·scale + b − c), adds p to the fp64 mass, writes Φᵀ
//            (a warp writes 32 consecutive queries of one key: 128-byte
//            coalesced), and stores p split as bf16 hi + lo (p = hi + lo to 16
//            bits) into a swizzled K-major operand for Y.
// MAX mode computes only max_ij (s·scale + b) per head (the shift).
//
// Every mbarrier wait is bounded by a clock budget; on expiry the CTA records
// AM_ERR_TIMEOUT, stops issuing work, drains what it issued and releases TMEM.
#include "am_internal.cuh"
#include "am_async.cuh"
#include "am_tcgen05.cuh"
#include "am_profile.cuh"

#include <float.h>

namespace am {
namespace {

constexpr int BM = 128;        // queries per CTA (TMEM lanes)
constexpr int BN = 64;         // keys per tile
constexpr int STAGES = 3;      // key/value ring depth
constexpr int kEpiGroups = 4;  // epilogue warpgroups; each takes BN / 4 columns of a tile
constexpr int kEpiThreads = 128 * kEpiGroups;
constexpr int kThreads = 128 + kEpiThreads;   // 4 control warps + the epilogue
constexpr int kEpiWarp0 = 4;   // first epilogue warp
constexpr uint32_t kTmemCols = 256;

enum Mode { MODE_MAX = 0, MODE_PHI = 1 };

// ---- shared-memory plan (bytes); operand tiles 1024-aligned for SW128 ----
struct Plan {
  int d;
  uint32_t q_bytes, k_bytes, v_bytes, p_bytes;
  uint32_t off_q, off_k, off_v, off_p, off_bar, total;
};

__host__ __device__ inline Plan make_plan(int d, int mode) {
  Plan P{};
  P.d = d;
  P.q_bytes = BM * d * 2;
  P.k_bytes = BN * d * 2;
  P.v_bytes = mode == MODE_PHI ? BN * d * 2 : 0;
  P.p_bytes = mode == MODE_PHI ? BM * BN * 2 : 0;   // one of hi / lo
  uint32_t o = 0;
  P.off_q = o; o += P.q_bytes;
  P.off_k = o; o += STAGES * P.k_bytes;
  P.off_v = o; o += STAGES * P.v_bytes;
  P.off_p = o; o += 2 * 2 * P.p_bytes;               // 2 buffers × (hi, lo)
  P.off_bar = o; o += 32 * 8;
  P.total = o + 1024;                                 // slack to align the base
  return P;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t f2ord(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
k_phi_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
         const __grid_constant__ CUtensorMap tmV, Problem p, Work w, const float* __restrict__ key_bias,
         uint32_t* __restrict__ shift_ord) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  constexpr int KB = D / 64;                       // 128-byte K-blocks per row
  const Plan P = make_plan(D, MODE);
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = sm + P.off_q;
  unsigned char* sK = sm + P.off_k;
  unsigned char* sV = sm + P.off_v;
  unsigned char* sP = sm + P.off_p;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P.off_bar);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;             // [STAGES]
  uint64_t* kv_empty = bars + 1 + STAGES;   // [STAGES]
  uint64_t* s_full = bars + 1 + 2 * STAGES; // [2]
  uint64_t* s_empty = s_full + 2;           // [2]
  uint64_t* p_full = s_full + 4;            // [2]
  uint64_t* p_empty = s_full + 6;           // [2]
  uint64_t* y_full = s_full + 8;
  uint64_t* drain = s_full + 9;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ float s_red[4 * kEpiGroups];
  __shared__ double s_mass[kEpiGroups + 1][BM];
  __shared__ int s_stop_y;
  __shared__ int s_stopm[2];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (p.n + BM - 1) / BM;
  const int h = blockIdx.x / nqb;
  const int q0 = (blockIdx.x % nqb) * BM;
  // this head's keys are rows krow0 .. krow0 + Th − 1 of the packed K and V
  // (the 2-D tensor maps): a tile reaching past Th reads the next head's
  // rows (or zeros past the end), and the epilogue masks those columns
  const int Th = w.Th[h];
  const int krow0 = (int)w.koff[h];
  const int NT = (Th + BN - 1) / BN;
  int32_t* status = w.status + h;
  volatile int* abort_flag = &s_abort;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(q_full, 1);
    for (int s = 0; s < STAGES; ++s) { mbar_init(kv_full + s, 1); mbar_init(kv_empty + s, 1); }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, kEpiThreads);
      mbar_init(p_full + b, kEpiThreads);
      mbar_init(p_empty + b, 1);
    }
    mbar_init(y_full, 1);
    mbar_init(drain, 1);
    mbar_init_fence();
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tS[2] = {tmem, tmem + BN};
  const uint32_t tY = tmem + 2 * BN;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ----
    if (lane == 0) {
      mbar_expect_tx(q_full, P.q_bytes);
      for (int kb = 0; kb < KB; ++kb) tma_load_3d(sQ + kb * BM * 128, &tmQ, q_full, kb * 64, q0, h);
      int issued[STAGES] = {};
      for (int j = 0; j < NT; ++j) {
        const int s = j % STAGES, use = j / STAGES;
        if (use > 0 && !mbar_wait(kv_empty + s, (use - 1) & 1, abort_flag, status, p.wait_cycles)) break;
        mbar_expect_tx(kv_full + s, P.k_bytes + P.v_bytes);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(sK + s * P.k_bytes + kb * BN * 128, &tmK, kv_full + s, kb * 64, krow0 + j * BN);
        if (MODE == MODE_PHI)
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sV + s * P.v_bytes + kb * BN * 128, &tmV, kv_full + s, kb * 64, krow0 + j * BN);
        issued[s] = use + 1;
      }
      // copies still in flight must land before the CTA releases its memory
      {
        const long long t0 = clock64();
        while (!mbar_try_wait(q_full, 0) && clock64() - t0 < kDrainCycles) {}
      }
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] > 0) {
          const long long t0 = clock64();
          while (!mbar_try_wait(kv_full + s, (issued[s] - 1) & 1) && clock64() - t0 < kDrainCycles) {}
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ----
    if (lane == 0) {
      const uint32_t idesc1 = instr_desc(BN, false);
      const uint32_t idesc2 = instr_desc(D, true);
      bool ok = mbar_wait(q_full, 0, abort_flag, status, p.wait_cycles);
      tc_fence_after();
      auto gemm2 = [&](int jj) -> bool {
        const int b = jj & 1, bu = jj >> 1, s = jj % STAGES;
        if (!mbar_wait(p_full + b, bu & 1, abort_flag, status, p.wait_cycles)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(sV + s * P.v_bytes);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t pbase = smem_u32(sP + (b * 2 + half) * P.p_bytes);
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            const uint64_t ad = smem_desc(pbase + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc(vbase + kk * 16 * 128, BN * 128, 1024);
            tc_mma(tY, ad, bd, idesc2, (jj > 0 || half > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(p_empty + b);
        tc_commit(kv_empty + s);
        return true;
      };
      int j = 0;
      for (; ok && j < NT; ++j) {
        const int s = j % STAGES, use = j / STAGES, b = j & 1, bu = j >> 1;
        if (!mbar_wait(kv_full + s, use & 1, abort_flag, status, p.wait_cycles)) { ok = false; break; }
        if (bu > 0 && !mbar_wait(s_empty + b, (bu - 1) & 1, abort_flag, status, p.wait_cycles)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qbase = smem_u32(sQ), kbase = smem_u32(sK + s * P.k_bytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = kk >> 2;   // 128-byte K-block
          const uint64_t ad = smem_desc(qbase + koff * BM * 128 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(kbase + koff * BN * 128 + (kk & 3) * 32, 16, 1024);
          tc_mma(tS[b], ad, bd, idesc1, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full + b);
        if (MODE == MODE_MAX) tc_commit(kv_empty + s);
        if (MODE == MODE_PHI && j > 0 && !gemm2(j - 1)) { ok = false; break; }
      }
      if (MODE == MODE_PHI && ok && NT > 0) ok = gemm2(NT - 1);
      if (MODE == MODE_PHI) tc_commit(y_full);
      // drain: every MMA this thread issued has completed before TMEM is freed
      tc_commit(drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kDrainCycles) {}
    }
  } else if (warp >= kEpiWarp0) {
    // --------------------------------------------------- epilogue ----
    // Four warpgroups: thread (grp, et) owns query row et (TMEM lane et) and
    // columns [16·grp, 16·grp + 16) of every 64-key tile.
    const int ep = threadIdx.x - kEpiWarp0 * 32;     // 0..511
    const int grp = ep >> 7;
    const int et = ep & 127;
    const int qd = warp & 3;                         // TMEM lane quadrant of this warp
    constexpr int HC = BN / kEpiGroups;
    const int i = q0 + et;
    const bool row_live = i < p.n;
    const float c = MODE == MODE_PHI ? w.shift[h] : 0.f;
    // PHI: p = 2^(s·scale·log2e + (b − c)·log2e); any rounding of log2e or of
    // c·log2e multiplies every feature of the head by one common factor,
    // which no result depends on (the shift invariance).
    const float kLog2e = 1.4426950408889634f;
    const float scale = MODE == MODE_PHI ? p.scale * kLog2e : p.scale;
    const float bias_const = MODE == MODE_PHI ? -c * kLog2e : 0.f;
    double mrow = 0.0;
    float mx = -FLT_MAX;
    const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
    float* phi_base = w.phiT + (int64_t)h * p.T * p.ldn;
    bool ok = true;
    for (int j = 0; j < NT; ++j) {
      const int b = j & 1, bu = j >> 1;
      if constexpr (MODE == MODE_MAX) {
        // light per-tile work: one thread waits and the group follows it
        if (ep == 0) s_stopm[b] = mbar_wait(s_full + b, bu & 1, abort_flag, status, p.wait_cycles) ? 0 : 1;
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
        if (s_stopm[b]) { ok = false; break; }
      } else {
        // each epilogue thread waits for the tile itself; no named barrier in the
        // loop, but a warp leaves together (the loads and shuffles below are
        // warp-collective)
        const bool got = mbar_wait(s_full + b, bu & 1, abort_flag, status, p.wait_cycles);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      tc_fence_after();
      float v[HC];
      tmem_ld16(tS[b] + lane_addr + grp * HC, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_empty + b);
      const int kvalid = min(BN, Th - j * BN) - grp * HC;    // valid columns of this group
      // per-key additive term: (b_j − c)·log2e (PHI) or b_j (MAX); a constant without a prior bias
      const int jb = j * BN + grp * HC;
      auto bias_at = [&](int cc) -> float {
        const int jg = jb + cc;
        const float bj = jg < Th ? __ldg(key_bias + krow0 + jg) : 0.f;
        return MODE == MODE_PHI ? (bj - c) * kLog2e : bj;
      };
      const bool full = row_live && kvalid >= HC;
      if constexpr (MODE == MODE_MAX) {
        if (full && !p.has_bias) {
#pragma unroll
          for (int cc = 0; cc < HC; ++cc) mx = fmaxf(mx, v[cc] * scale);
        } else if (row_live) {
#pragma unroll
          for (int cc = 0; cc < HC; ++cc)
            if (cc < kvalid) mx = fmaxf(mx, fmaf(v[cc], scale, p.has_bias ? bias_at(cc) : 0.f));
        }
        continue;
      } else {
      if (full && !p.has_bias) {   // common case: whole tile, no prior bias
#pragma unroll
        for (int cc = 0; cc < HC; ++cc) v[cc] = ex2_approx(fmaf(v[cc], scale, bias_const));
      } else {
#pragma unroll
        for (int cc = 0; cc < HC; ++cc) {
          const float x = fmaf(v[cc], scale, p.has_bias ? bias_at(cc) : bias_const);
          v[cc] = (row_live && cc < kvalid) ? ex2_approx(x) : 0.f;
        }
      }
      double a4[4] = {0.0, 0.0, 0.0, 0.0};   // mass partials: short dependency chains
#pragma unroll
      for (int cc = 0; cc < HC; ++cc) a4[cc & 3] += (double)v[cc];
      mrow += (a4[0] + a4[1]) + (a4[2] + a4[3]);
      if (w.cnpart) {
        // this warp's 32 rows of Σ_i Φ_ij² for its 16 keys: a butterfly leaves
        // key (lane >> 1) on lanes lane, lane ^ 1; even lanes store it
        float q2[HC];
#pragma unroll
        for (int cc = 0; cc < HC; ++cc) q2[cc] = v[cc] * v[cc];
#pragma unroll
        for (int s = HC / 2, o = 16; s >= 1; s >>= 1, o >>= 1) {
          const bool upper = (lane & o) != 0;
#pragma unroll
          for (int k = 0; k < s; ++k) {
            const float send = upper ? q2[k] : q2[k + s];
            const float keep = upper ? q2[k + s] : q2[k];
            q2[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
        q2[0] += __shfl_xor_sync(0xffffffffu, q2[0], 1);
        const int key = jb + ((lane >> 1) & (HC - 1));
        if (!(lane & 1) && key < Th)
          w.cnpart[(((int64_t)h * nqb + blockIdx.x % nqb) * 4 + qd) * p.T + key] = q2[0];
      }
      if (i < p.ldn) {
        float* col = phi_base + (int64_t)(j * BN + grp * HC) * p.ldn + i;
        if (kvalid >= HC) {
#pragma unroll
          for (int cc = 0; cc < HC; ++cc) col[(int64_t)cc * p.ldn] = v[cc];
        } else {
#pragma unroll
          for (int cc = 0; cc < HC; ++cc)
            if (cc < kvalid) col[(int64_t)cc * p.ldn] = v[cc];
        }
        if (w.phiT16) {   // bf16 copy streamed by the correlation pass
          __nv_bfloat16* col16 = w.phiT16 + ((int64_t)h * p.T + j * BN + grp * HC) * p.ldn + i;
#pragma unroll
          for (int cc = 0; cc < HC; ++cc)
            if (cc < kvalid) col16[(int64_t)cc * p.ldn] = __float2bfloat16_rn(v[cc]);
        }
      }
      // P tile for Y += P·V: K-major, 128-byte rows, 16-byte chunks XOR-swizzled by row;
      // the buffer is free once the MMA that read it two tiles ago has completed
      if (bu > 0 && !mbar_wait(p_empty + b, (bu - 1) & 1, abort_flag, status, p.wait_cycles)) { ok = false; break; }
      unsigned char* hi_row = sP + (b * 2 + 0) * P.p_bytes + et * 128;
      unsigned char* lo_row = sP + (b * 2 + 1) * P.p_bytes + et * 128;
#pragma unroll
      for (int c4 = 0; c4 < HC / 8; ++c4) {
        uint32_t hv[4], lv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a0 = v[c4 * 8 + 2 * e], a1 = v[c4 * 8 + 2 * e + 1];
          const __nv_bfloat162 hb = __floats2bfloat162_rn(a0, a1);
          const float2 hf = __bfloat1622float2(hb);
          hv[e] = *reinterpret_cast<const uint32_t*>(&hb);
          lv[e] = pack_bf16x2(a0 - hf.x, a1 - hf.y);
        }
        const int pc = (grp * (HC / 8) + c4) ^ (et & 7);
        *reinterpret_cast<uint4*>(hi_row + pc * 16) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
        *reinterpret_cast<uint4*>(lo_row + pc * 16) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(p_full + b);
      }
    }
    if (MODE == MODE_MAX) {
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) s_red[warp - kEpiWarp0] = mx;
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      if (ep == 0) {
        float v = s_red[0];
        for (int k = 1; k < 4 * kEpiGroups; ++k) v = fmaxf(v, s_red[k]);
        atomicMax(shift_ord + h, f2ord(v));
      }
    } else {
      // combine the groups' mass partials in a fixed order: (0 + 1) + (2 + 3)
      s_mass[grp][et] = mrow;
      if (ep == 0) s_stop_y = (ok && mbar_wait(y_full, 0, abort_flag, status, p.wait_cycles)) ? 0 : 1;
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      if (grp == 0) s_mass[kEpiGroups][et] = (s_mass[0][et] + s_mass[1][et]) + (s_mass[2][et] + s_mass[3][et]);
      asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      const double mtot = s_mass[kEpiGroups][et];
      if (!s_stop_y) {
        tc_fence_after();
        float* yrow = w.Y + ((int64_t)h * p.n + i) * p.d;
        constexpr int YC = D / kEpiGroups;   // target columns of this group
#pragma unroll
        for (int c0 = 0; c0 < YC; c0 += 16) {
          const int cb = grp * YC + c0;
          float y[16];
          tmem_ld16(tY + lane_addr + cb, y);
          tmem_wait_ld();
          if (row_live) {
            // a query whose every feature underflowed has no mass: zero target
            const double im = mtot > 0.0 ? 1.0 / mtot : 0.0;
#pragma unroll
            for (int cc = 0; cc < 16; cc += 4)
              *reinterpret_cast<float4*>(yrow + cb + cc) =
                  make_float4((float)(y[cc] * im), (float)(y[cc + 1] * im), (float)(y[cc + 2] * im),
                              (float)(y[cc + 3] * im));
          }
        }
        // every feature of this reference query underflowed: it carries no mass
        if (grp == 0 && row_live && !(mtot > 0.0)) record_status(status, AM_WARN_MASS_UNDERFLOW);
        if (grp == 0 && i < p.ldn) {
          const double mv = row_live ? mtot : 0.0;
          w.m[(int64_t)h * p.ldn + i] = mv;
          w.r[(int64_t)h * p.ldn + i] = (float)mv;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// ---------------------------------------------------------------------------
// Correlation by recomputation: c_j = Σ_i r_i exp(s_ij·scale + b_j − c_h) for
// a block of 128 keys, with Φ recomputed from Q and K on the tensor cores
// instead of re-read from HBM (the OMP correlation step, zhichai.net deep
// dive §1.6: j* = argmax rᵀΦ_{:,j}).  Keys sit on the TMEM lanes (M = 128),
// query tiles of 128 stream through a 3-stage ring (N = 128); four epilogue
// warpgroups each fold 32 queries of every tile into their key's sum.  Each
// epilogue thread waits on the tile's barrier itself (no named barrier in
// the loop) and reads the residual with broadcast vector loads.
constexpr int CQ = 128;         // queries per tile
constexpr int CSTAGES = 3;
constexpr int kCorrThreads = 640;   // 4 control warps + 4 epilogue warpgroups
constexpr uint32_t kCorrTmemCols = 256;

__host__ __device__ inline uint32_t corr_smem_bytes(int d) {
  return (uint32_t)(BM * d * 2 + CSTAGES * CQ * d * 2 + 32 * 8 + 1024);
}

template <int D>
__global__ void __launch_bounds__(kCorrThreads, 1)
k_corr_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, Problem p, Work w,
          const float* __restrict__ key_bias, int pass) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  constexpr int KB = D / 64;
  const int h = w.order[blockIdx.y];
  const int Th = w.Th[h];
  // the whole CTA leaves when the head is finished or has no key in this block
  if (pass * p.kR >= w.t[h] || (int)blockIdx.x * BM >= Th) return;
  const int krow0 = (int)w.koff[h];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t k_bytes = BM * D * 2, q_bytes = CQ * D * 2;
  unsigned char* sK = sm;
  unsigned char* sQ = sm + k_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sQ + CSTAGES * q_bytes);
  uint64_t* k_full = bars + 0;
  uint64_t* q_full = bars + 1;                  // [CSTAGES]
  uint64_t* q_empty = bars + 1 + CSTAGES;       // [CSTAGES]
  uint64_t* s_full = bars + 1 + 2 * CSTAGES;    // [2]
  uint64_t* s_empty = s_full + 2;               // [2]
  uint64_t* drain = s_full + 4;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ float s_part[4][128];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = blockIdx.x * BM;
  const int NQ = (p.n + CQ - 1) / CQ;
  int32_t* status = w.status + h;
  volatile int* abort_flag = &s_abort;

  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(k_full, 1);
    for (int s = 0; s < CSTAGES; ++s) { mbar_init(q_full + s, 1); mbar_init(q_empty + s, 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(s_full + b, 1); mbar_init(s_empty + b, 512); }
    mbar_init(drain, 1);
    mbar_init_fence();
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                 "r"(kCorrTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tS[2] = {tmem, tmem + CQ};

  if (warp == 0) {
    if (lane == 0) {
      mbar_expect_tx(k_full, k_bytes);
      for (int kb = 0; kb < KB; ++kb) tma_load_2d(sK + kb * BM * 128, &tmK, k_full, kb * 64, krow0 + j0);
      int issued[CSTAGES] = {};
      for (int j = 0; j < NQ; ++j) {
        const int s = j % CSTAGES, use = j / CSTAGES;
        if (use > 0 && !mbar_wait(q_empty + s, (use - 1) & 1, abort_flag, status, p.wait_cycles)) break;
        mbar_expect_tx(q_full + s, q_bytes);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_3d(sQ + s * q_bytes + kb * CQ * 128, &tmQ, q_full + s, kb * 64, j * CQ, h);
        issued[s] = use + 1;
      }
      {   // the key block's copy must land before the CTA releases its memory
        const long long t0 = clock64();
        while (!mbar_try_wait(k_full, 0) && clock64() - t0 < kDrainCycles) {}
      }
      for (int s = 0; s < CSTAGES; ++s)
        if (issued[s] > 0) {
          const long long t0 = clock64();
          while (!mbar_try_wait(q_full + s, (issued[s] - 1) & 1) && clock64() - t0 < kDrainCycles) {}
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = instr_desc(CQ, false);
      bool ok = mbar_wait(k_full, 0, abort_flag, status, p.wait_cycles);
      tc_fence_after();
      for (int j = 0; ok && j < NQ; ++j) {
        const int s = j % CSTAGES, use = j / CSTAGES, b = j & 1, bu = j >> 1;
        if (!mbar_wait(q_full + s, use & 1, abort_flag, status, p.wait_cycles)) break;
        if (bu > 0 && !mbar_wait(s_empty + b, (bu - 1) & 1, abort_flag, status, p.wait_cycles)) break;
        tc_fence_after();
        const uint32_t kbase = smem_u32(sK), qbase = smem_u32(sQ + s * q_bytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t kblk = kk >> 2;
          const uint64_t ad = smem_desc(kbase + kblk * BM * 128 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc(qbase + kblk * CQ * 128 + (kk & 3) * 32, 16, 1024);
          tc_mma(tS[b], ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full + b);
        tc_commit(q_empty + s);
      }
      tc_commit(drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kDrainCycles) {}
    }
  } else if (warp >= kEpiWarp0) {
    const int wg = (warp - kEpiWarp0) >> 2;     // 32-query column group of each tile
    const int qd = warp & 3;                    // TMEM lane quadrant
    const int et = qd * 32 + lane;              // key row within the block
    const int j = j0 + et;
    const bool key_live = j < Th;
    const float kLog2e = 1.4426950408889634f;
    const float scale = p.scale * kLog2e;
    const float c = w.shift[h];
    const float bj = (p.has_bias && key_live) ? key_bias[krow0 + j] : 0.f;
    const float bias2 = (bj - c) * kLog2e;
    const float* rh = w.r + (int64_t)h * p.ldn;
    const uint32_t tcol = lane_addr_base(qd) + wg * 32;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int t = 0; t < NQ; ++t) {
      const int b = t & 1, bu = t >> 1;
      if (!mbar_wait(s_full + b, bu & 1, abort_flag, status, p.wait_cycles)) break;
      tc_fence_after();
      float v[32];
      tmem_ld32(tS[b] + tcol, v);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(s_empty + b);
      const int q0 = t * CQ + wg * 32;
      if (q0 < p.ldn) {   // r is zero from n to ldn; chunks of 32 lie wholly inside or outside
        const float4* r4 = reinterpret_cast<const float4*>(rh + q0);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 rr = __ldg(r4 + k);
          acc[0] = fmaf(ex2_approx(fmaf(v[4 * k + 0], scale, bias2)), rr.x, acc[0]);
          acc[1] = fmaf(ex2_approx(fmaf(v[4 * k + 1], scale, bias2)), rr.y, acc[1]);
          acc[2] = fmaf(ex2_approx(fmaf(v[4 * k + 2], scale, bias2)), rr.z, acc[2]);
          acc[3] = fmaf(ex2_approx(fmaf(v[4 * k + 3], scale, bias2)), rr.w, acc[3]);
        }
      }
    }
    s_part[wg][et] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    asm volatile("bar.sync 1, 512;" ::: "memory");
    if (wg == 0 && key_live && !s_abort)
      w.corr[(int64_t)h * p.T + j] = ((s_part[0][et] + s_part[1][et]) + s_part[2][et]) + s_part[3][et];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCorrTmemCols));
}

template <int D, int MODE>
cudaError_t launch_tc(const Problem& p, const void* Q, const void* K, const void* V, const float* key_bias,
                      const Work& w, uint32_t* shift_ord, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, p.H, p.n, D, BM) || !make_map_2d(&mk, K, p.key_rows, D, BN) ||
      !make_map_2d(&mv, MODE == MODE_PHI ? V : K, p.key_rows, D, BN))
    return cudaErrorInvalidValue;
  const Plan P = make_plan(D, MODE);
  auto kern = k_phi_tc<D, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)P.total);
  if (e != cudaSuccess) return e;
  const int grid = p.H * ((p.n + BM - 1) / BM);
  AM_LAUNCH(MODE == MODE_PHI ? AM_STAGE_PHI : AM_STAGE_SHIFT, s,
            kern<<<grid, kThreads, P.total, s>>>(mq, mk, mv, p, w, key_bias, shift_ord));
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_corr_tc_d(const Problem& p, const void* Q, const void* K, const float* key_bias, const Work& w,
                             int pass, int active, cudaStream_t s) {
  CUtensorMap mq, mk;
  if (!make_map(&mq, Q, p.H, p.n, D, CQ) || !make_map_2d(&mk, K, p.key_rows, D, BM)) return cudaErrorInvalidValue;
  const uint32_t bytes = corr_smem_bytes(D);
  auto kern = k_corr_tc<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  dim3 grid((p.T + BM - 1) / BM, active);
  AM_LAUNCH(AM_STAGE_CORR, s, kern<<<grid, kCorrThreads, bytes, s>>>(mq, mk, p, w, key_bias, pass));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_corr_tc(const Problem& p, const void* Q, const void* K, const float* key_bias, const Work& w,
                           int pass, int active, cudaStream_t s) {
  return p.d == 64 ? launch_corr_tc_d<64>(p, Q, K, key_bias, w, pass, active, s)
                   : launch_corr_tc_d<128>(p, Q, K, key_bias, w, pass, active, s);
}

bool phi_tc_supported(const Problem& p) { return p.in_dtype == AM_BF16 && (p.d == 64 || p.d == 128); }

cudaError_t launch_shift_max_tc(const Problem& p, const void* Q, const void* K, const float* key_bias,
                                const Work& w, uint32_t* shift_ord, cudaStream_t s) {
  return p.d == 64 ? launch_tc<64, MODE_MAX>(p, Q, K, nullptr, key_bias, w, shift_ord, s)
                   : launch_tc<128, MODE_MAX>(p, Q, K, nullptr, key_bias, w, shift_ord, s);
}

cudaError_t launch_phi_tc(const Problem& p, const void* Q, const void* K, const void* V, const float* key_bias,
                          const Work& w, cudaStream_t s) {
  return p.d == 64 ? launch_tc<64, MODE_PHI>(p, Q, K, V, key_bias, w, nullptr, s)
                   : launch_tc<128, MODE_PHI>(p, Q, K, V, key_bias, w, nullptr, s);
}

}  // namespace am
