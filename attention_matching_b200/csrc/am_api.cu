// C ABI entry points: argument checks, workspace plan, launch sequence.
//
// One call compacts H independent heads (the per-(layer, KV-head) problems of
// "Fast KV Compaction via Attention Matching", zhichai.net deep dive §1.6;
// varlen packing of non-uniform budgets per the zhichai.net/en summary,
// "Engineering Practicality"; per-head key counts for KV-based chunking of a
// long context, xinfinite.net article §3).  All work is ordered after the
// caller's stream and the caller's stream waits for all of it; no device
// memory is allocated here.  The OMP passes of different head groups run on
// internal streams of their own (the heads are independent), so one group's
// latency-bound refits overlap another group's bandwidth-bound passes.
//
// Workspace: a prefix (header, every head's status word, the device tables
// of every wave), then one wave's region.  When the caller's workspace holds
// fewer heads than the call has, the heads run in waves of consecutive heads
// through that one region, each wave as many heads as fit.
#include "am_internal.cuh"

#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

namespace am {
namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
  // byte offsets from the workspace base
  size_t tables, status, shift, np, ylen, mm, rr_part;
  size_t phiT, phiT16, m, Y, r, corr, sel;
  size_t picks, pick_corr, plist, sorted_slot;
  size_t bvec, w, w_eff, ycache;
  size_t G, L, AtA, A, Apl, Ypl, AtY, nrm_part;
  size_t cnorm, cnpart, rnorm, clist, clj, ccount, inv_m, gb, ghist, gtau, gcnt, cdone, cnblk, ctheta, gpart, gcount,
      rcount,
      dinv, vinv, ndinv, dvalid;
  size_t total;
  size_t tables_bytes;
  bool tc_normal;   // the value fit's normal equations run on the tensor cores (bf16 planes)
};

struct Tables {
  std::vector<int32_t> t;
  std::vector<int32_t> Th;        // key count per head
  std::vector<int64_t> koff;      // [H+1] first key row per head (relative to the first head's)
  std::vector<int64_t> cu_t, cu_t2;
  std::vector<int32_t> order;
  std::vector<int> active;   // active heads per pass
  // head groups for concurrent pass chains: group g holds order[g], order[g + G], ...
  std::vector<int32_t> gorder;                // groups' orders, concatenated
  std::vector<int> gstart;                    // [G + 1] offsets into gorder
  std::vector<std::vector<int>> gactive;      // per group: active heads per pass
  std::vector<int> passes;                    // OMP passes per head
  int max_t = 0;
  int64_t sum_t = 0, sum_t2 = 0;
};

// The feature pass also writes a bf16 copy of Φᵀ for the bf16 correlation mode.
bool bf16_copy(const am_opts_t* o) {
  return o->corr_mode == AM_CORR_STORED_BF16 && o->select_mode == AM_SELECT_OMP;
}

// The value fit forms its normal equations on the tensor cores (bf16 inputs,
// d in {64, 128}); otherwise on CUDA cores in fp64.
bool tc_normal(const am_opts_t* o, int d) { return o->in_dtype == AM_BF16 && (d == 64 || d == 128); }

// Bytes of one wave's device tables: cu_t, cu_t2, koff [H+1] int64 and
// t, Th, order, group order [H] int32 (a multiple of 8).
size_t table_bytes(int H) { return (size_t)(H + 1) * 8 * 3 + (size_t)H * 4 * 4; }

// The workspace prefix for a call of H heads: header, H status words, a
// tables region that holds every wave's tables (Σ over waves of
// table_bytes(H_w) <= 64·H bytes for any split into waves), and per-head call
// statistics that outlive the waves: keys evaluated (int64 [H]), then NNLS
// refits and their inner solves (int32 [H] each).
// (each statistic's array starts 16-byte aligned)
size_t round16(size_t x) { return (x + 15) & ~(size_t)15; }
size_t stats_offset(int H) { return align_up(kWsHeaderBytes + (size_t)H * 4) + align_up((size_t)H * 64 + 256); }
size_t refits_offset(int H) { return stats_offset(H) + round16((size_t)H * 8); }
size_t solves_offset(int H) { return refits_offset(H) + round16((size_t)H * 4); }
size_t prefix_bytes(int H) { return align_up(solves_offset(H) + (size_t)H * 4); }

// One wave's region, from byte `o0` (the end of the prefix) on.
Layout plan(int n, int T, int d, int H, int64_t sum_t, int64_t sum_t2, bool corr_bf16, size_t o0, bool tc_normal) {
  Layout L{};
  const size_t ldn = (size_t)round_up(n, 32);
  size_t o = o0;
  auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes); return at; };
  L.tables_bytes = table_bytes(H);
  L.tc_normal = tc_normal;
  L.shift = take((size_t)H * 4);
  L.np = take((size_t)H * 4);
  L.ylen = take((size_t)H * 4);
  L.mm = take((size_t)H * 8);
  L.rr_part = take((size_t)H * kRedBlocks * 8);
  L.phiT = take((size_t)H * T * ldn * 4);
  L.phiT16 = take(corr_bf16 ? (size_t)H * T * ldn * 2 : 0);
  L.m = take((size_t)H * ldn * 8);
  L.r = take((size_t)H * ldn * 4);
  L.Y = take((size_t)H * n * d * 4);
  L.corr = take((size_t)H * T * 4);
  L.sel = take((size_t)H * T);
  L.picks = take((size_t)sum_t * 4);
  L.pick_corr = take((size_t)sum_t * 4);
  L.plist = take((size_t)sum_t * 4);
  L.sorted_slot = take((size_t)sum_t * 4);
  L.bvec = take((size_t)sum_t * 8);
  L.w = take((size_t)sum_t * 8);
  L.w_eff = take((size_t)sum_t * 8);
  L.ycache = take((size_t)sum_t * 8);
  L.G = take((size_t)sum_t2 * 8);
  L.L = take((size_t)sum_t2 * 8);
  L.AtA = take((size_t)sum_t2 * 8);
  // the design matrix: fp32 for the CUDA-core normal equations, or three bf16
  // planes (and the targets' planes) for the tensor-core ones
  L.A = take(tc_normal ? 0 : (size_t)sum_t * ldn * 4);
  L.Apl = take(tc_normal ? (size_t)3 * sum_t * ldn * 2 : 0);
  L.Ypl = take(tc_normal ? (size_t)3 * H * n * d * 2 : 0);
  L.AtY = take((size_t)sum_t * d * 8);
  L.nrm_part = take((size_t)kNormalMaxSplits * ((size_t)sum_t2 + (size_t)sum_t * d) * 8);
  L.cnorm = take((size_t)H * T * 8);
  L.cnpart = take((size_t)H * 4 * ((n + 127) / 128) * T * 4);
  L.rnorm = take((size_t)H * 8);
  L.clist = take((size_t)H * T * 8);
  L.clj = take((size_t)H * T * 4);
  L.ccount = take((size_t)H * 4);
  L.inv_m = take((size_t)H * ldn * 8);
  L.gb = take((size_t)H * T * 4);
  L.ghist = take((size_t)H * 1024 * 4);
  L.gtau = take((size_t)H * 4);
  L.gcnt = take((size_t)H * 4);
  L.cdone = take((size_t)H * 4);
  L.cnblk = take((size_t)H * T * kRedBlocks * 4);
  L.ctheta = take((size_t)H * 8);
  L.gpart = take((size_t)kGramMaxSlices * ((size_t)sum_t + H) * kGramMaxNew * 8);
  L.gcount = take(((size_t)sum_t + H) * 4);
  L.rcount = take((size_t)H * 4);
  L.dinv = take(((size_t)sum_t + 32 * (size_t)H) * 32 * 8);
  L.vinv = take(((size_t)sum_t + 64 * (size_t)H) * 64 * 8);
  L.ndinv = take(((size_t)sum_t + 32 * (size_t)H) * 64 * 8);
  L.dvalid = take((size_t)H * 4);
  L.total = o;
  return L;
}

void set_groups(Tables* tb, const std::vector<int>& passes, int G);
void finish_tables(Tables* tb, int kR);

// Key rows per pass of greedy selection (or per refit of pre-selected keys).
int picks_per_pass(const am_opts_t* o) {
  return o->select_mode == AM_SELECT_HIGHEST ? kHighestChunk : o->topk * o->refit_every;
}

am_status_t check_shape(int n, int T, int d, int H, const int32_t* budgets, const am_opts_t* opts,
                        Tables* tb) {
  if (!budgets || !opts) return AM_ERR_INVALID_ARG;
  if (n < 1 || T < 1 || d < 1 || H < 1) return AM_ERR_INVALID_ARG;
  if (opts->in_dtype != AM_BF16 && opts->in_dtype != AM_FP32) return AM_ERR_INVALID_ARG;
  if (d > 256) return AM_ERR_UNSUPPORTED;
  if (opts->select_mode != AM_SELECT_OMP && opts->select_mode != AM_SELECT_HIGHEST) return AM_ERR_INVALID_ARG;
  const bool highest = opts->select_mode == AM_SELECT_HIGHEST;
  if (!highest && (opts->topk < 1 || opts->refit_every < 1)) return AM_ERR_INVALID_ARG;
  if (!highest && (int64_t)opts->topk * opts->refit_every > kMaxPicksPerPass) return AM_ERR_UNSUPPORTED;
  if (highest && T > kSortSmemKeys) return AM_ERR_UNSUPPORTED;
  if (opts->nnls_max_iter < 0) return AM_ERR_INVALID_ARG;
  if (!(opts->ridge >= 0.f) || !isfinite(opts->ridge)) return AM_ERR_INVALID_ARG;
  if (!(opts->w_floor_rel > 0.f) || !(opts->w_floor_rel < 1.f)) return AM_ERR_INVALID_ARG;
  if (!isfinite(opts->scale)) return AM_ERR_INVALID_ARG;
  if (opts->corr_mode < AM_CORR_AUTO || opts->corr_mode > AM_CORR_BOUNDED) return AM_ERR_INVALID_ARG;
  if (!highest && opts->corr_mode == AM_CORR_RECOMPUTE && !(opts->in_dtype == AM_BF16 && (d == 64 || d == 128)))
    return AM_ERR_UNSUPPORTED;
  if ((int64_t)n * d > (1ll << 31) || (int64_t)T * round_up(n, 32) > (1ll << 40))
    return AM_ERR_UNSUPPORTED;
  if (opts->reserved0 != 0 || opts->wait_cycles < 0) return AM_ERR_INVALID_ARG;
  const int kR = highest ? kHighestChunk : opts->topk * opts->refit_every;
  tb->t.assign(budgets, budgets + H);
  tb->Th.assign(H, T);
  tb->koff.assign(H + 1, 0);
  if (opts->key_offsets) {
    const int64_t* ko = opts->key_offsets;
    if (ko[0] != 0) return AM_ERR_INVALID_ARG;
    int tmax = 0;
    for (int h = 0; h < H; ++h) {
      const int64_t th = ko[h + 1] - ko[h];
      if (th < 1 || th > T) return AM_ERR_INVALID_ARG;
      tb->Th[h] = (int)th;
      tmax = std::max(tmax, (int)th);
    }
    if (tmax != T) return AM_ERR_INVALID_ARG;
    for (int h = 0; h <= H; ++h) tb->koff[h] = ko[h];
  } else {
    for (int h = 0; h <= H; ++h) tb->koff[h] = (int64_t)h * T;
  }
  // the feature passes address key rows with 32-bit tensor-map coordinates
  if (tb->koff[H] > (int64_t)INT32_MAX - 256) return AM_ERR_UNSUPPORTED;
  for (int h = 0; h < H; ++h) {
    const int t = budgets[h];
    if (t < 1 || t > tb->Th[h]) return AM_ERR_BUDGET;
    if (t > kMaxBudget) return AM_ERR_UNSUPPORTED;
  }
  finish_tables(tb, kR);
  return AM_OK;
}

// From t, Th and koff: the packed offsets, pass counts, the pass order of the
// heads and the active heads per pass (one group).
void finish_tables(Tables* tb, int kR) {
  const int H = (int)tb->t.size();
  tb->cu_t.assign(H + 1, 0);
  tb->cu_t2.assign(H + 1, 0);
  tb->max_t = 0;
  std::vector<int> passes(H);
  for (int h = 0; h < H; ++h) {
    const int t = tb->t[h];
    tb->cu_t[h + 1] = tb->cu_t[h] + t;
    // t² rounded up to even: every head's t×t regions start 16-byte aligned
    tb->cu_t2[h + 1] = tb->cu_t2[h] + (((int64_t)t * t + 1) & ~(int64_t)1);
    tb->max_t = std::max(tb->max_t, t);
    passes[h] = num_passes(t, kR);
  }
  tb->sum_t = tb->cu_t[H];
  tb->sum_t2 = tb->cu_t2[H];
  tb->order.resize(H);
  for (int h = 0; h < H; ++h) tb->order[h] = h;
  // by pass count, then budget, descending: the heads whose NNLS factor
  // lives in the workspace (the largest budgets) lead every group's order
  std::stable_sort(tb->order.begin(), tb->order.end(), [&](int a, int b) {
    return passes[a] != passes[b] ? passes[a] > passes[b] : tb->t[a] > tb->t[b];
  });
  const int maxp = passes[tb->order[0]];
  tb->active.assign(maxp, 0);
  for (int q = 0; q < maxp; ++q)
    for (int h = 0; h < H; ++h) tb->active[q] += passes[h] > q;
  tb->passes = passes;
  set_groups(tb, passes, 1);
}

// Heads [h0, h1) of `all` as a problem of their own (key rows relative to
// head h0's first row).
void sub_tables(const Tables& all, int h0, int h1, int kR, Tables* tw) {
  tw->t.assign(all.t.begin() + h0, all.t.begin() + h1);
  tw->Th.assign(all.Th.begin() + h0, all.Th.begin() + h1);
  tw->koff.resize(h1 - h0 + 1);
  for (int h = h0; h <= h1; ++h) tw->koff[h - h0] = all.koff[h] - all.koff[h0];
  finish_tables(tw, kR);
}

// Splits the pass-ordered heads round-robin into G groups (each group's list
// stays sorted by pass count, so a group's active heads are a prefix).
void set_groups(Tables* tb, const std::vector<int>& passes, int G) {
  const int H = (int)tb->order.size();
  G = std::max(1, std::min(G, H));
  tb->gorder.clear();
  tb->gstart.assign(1, 0);
  tb->gactive.assign(G, {});
  for (int g = 0; g < G; ++g) {
    for (int k = g; k < H; k += G) tb->gorder.push_back(tb->order[k]);
    tb->gstart.push_back((int)tb->gorder.size());
    const int maxp = passes[tb->gorder[tb->gstart[g]]];
    tb->gactive[g].assign(maxp, 0);
    for (int q = 0; q < maxp; ++q)
      for (int k = tb->gstart[g]; k < tb->gstart[g + 1]; ++k) tb->gactive[g][q] += passes[tb->gorder[k]] > q;
  }
}

Work bind(const Layout& L, char* base, bool corr_bf16) {
  Work w{};
  w.phiT16 = corr_bf16 ? reinterpret_cast<__nv_bfloat16*>(base + L.phiT16) : nullptr;
  w.shift = reinterpret_cast<float*>(base + L.shift);
  w.np = reinterpret_cast<int32_t*>(base + L.np);
  w.ylen = reinterpret_cast<int32_t*>(base + L.ylen);
  w.mm = reinterpret_cast<double*>(base + L.mm);
  w.rr_part = reinterpret_cast<double*>(base + L.rr_part);
  w.phiT = reinterpret_cast<float*>(base + L.phiT);
  w.m = reinterpret_cast<double*>(base + L.m);
  w.r = reinterpret_cast<float*>(base + L.r);
  w.Y = reinterpret_cast<float*>(base + L.Y);
  w.corr = reinterpret_cast<float*>(base + L.corr);
  w.sel = reinterpret_cast<uint8_t*>(base + L.sel);
  w.picks = reinterpret_cast<int32_t*>(base + L.picks);
  w.pick_corr = reinterpret_cast<float*>(base + L.pick_corr);
  w.plist = reinterpret_cast<int32_t*>(base + L.plist);
  w.sorted_slot = reinterpret_cast<int32_t*>(base + L.sorted_slot);
  w.bvec = reinterpret_cast<double*>(base + L.bvec);
  w.w = reinterpret_cast<double*>(base + L.w);
  w.w_eff = reinterpret_cast<double*>(base + L.w_eff);
  w.ycache = reinterpret_cast<double*>(base + L.ycache);
  w.G = reinterpret_cast<double*>(base + L.G);
  w.L = reinterpret_cast<double*>(base + L.L);
  w.AtA = reinterpret_cast<double*>(base + L.AtA);
  w.A = reinterpret_cast<float*>(base + L.A);
  w.Apl = L.tc_normal ? reinterpret_cast<__nv_bfloat16*>(base + L.Apl) : nullptr;
  w.Ypl = L.tc_normal ? reinterpret_cast<__nv_bfloat16*>(base + L.Ypl) : nullptr;
  w.AtY = reinterpret_cast<double*>(base + L.AtY);
  w.nrm_part = reinterpret_cast<double*>(base + L.nrm_part);
  w.cnorm = reinterpret_cast<double*>(base + L.cnorm);
  w.cnpart = reinterpret_cast<float*>(base + L.cnpart);
  w.rnorm = reinterpret_cast<double*>(base + L.rnorm);
  w.clist = reinterpret_cast<uint64_t*>(base + L.clist);
  w.clj = reinterpret_cast<int32_t*>(base + L.clj);
  w.ccount = reinterpret_cast<int32_t*>(base + L.ccount);
  w.inv_m = reinterpret_cast<double*>(base + L.inv_m);
  w.gb = reinterpret_cast<float*>(base + L.gb);
  w.ghist = reinterpret_cast<int32_t*>(base + L.ghist);
  w.gtau = reinterpret_cast<float*>(base + L.gtau);
  w.gcnt = reinterpret_cast<int32_t*>(base + L.gcnt);
  w.cdone = reinterpret_cast<int32_t*>(base + L.cdone);
  w.cnblk = reinterpret_cast<float*>(base + L.cnblk);
  w.ctheta = reinterpret_cast<double*>(base + L.ctheta);
  w.gpart = reinterpret_cast<double*>(base + L.gpart);
  w.gcount = reinterpret_cast<int32_t*>(base + L.gcount);
  w.rcount = reinterpret_cast<int32_t*>(base + L.rcount);
  w.dinv = reinterpret_cast<double*>(base + L.dinv);
  w.vinv = reinterpret_cast<double*>(base + L.vinv);
  w.ndinv = reinterpret_cast<double*>(base + L.ndinv);
  w.dvalid = reinterpret_cast<int32_t*>(base + L.dvalid);
  return w;
}

// Appends one wave's tables to `out` in the device order
// cu_t | cu_t2 | koff | t | Th | order | group order, and points the Work
// (and *gorder_dev) at where they will sit on the device: `dev` is the
// device address of the block's first byte.
void pack_tables(const Tables& tb, int H, std::vector<unsigned char>* out, Work* w, char* dev,
                 int32_t** gorder_dev) {
  const size_t b_cu = (size_t)(H + 1) * 8, b_h = (size_t)H * 4;
  const size_t at = out->size();
  out->resize(at + table_bytes(H));
  unsigned char* o = out->data() + at;
  memcpy(o, tb.cu_t.data(), b_cu);
  memcpy(o + b_cu, tb.cu_t2.data(), b_cu);
  memcpy(o + 2 * b_cu, tb.koff.data(), b_cu);
  memcpy(o + 3 * b_cu, tb.t.data(), b_h);
  memcpy(o + 3 * b_cu + b_h, tb.Th.data(), b_h);
  memcpy(o + 3 * b_cu + 2 * b_h, tb.order.data(), b_h);
  memcpy(o + 3 * b_cu + 3 * b_h, tb.gorder.data(), b_h);
  w->cu_t = reinterpret_cast<int64_t*>(dev);
  w->cu_t2 = reinterpret_cast<int64_t*>(dev + b_cu);
  w->koff = reinterpret_cast<int64_t*>(dev + 2 * b_cu);
  w->t = reinterpret_cast<int32_t*>(dev + 3 * b_cu);
  w->Th = reinterpret_cast<int32_t*>(dev + 3 * b_cu + b_h);
  w->order = reinterpret_cast<int32_t*>(dev + 3 * b_cu + 2 * b_h);
  *gorder_dev = reinterpret_cast<int32_t*>(dev + 3 * b_cu + 3 * b_h);
}

// Internal streams for the head groups, created once per device.
constexpr int kMaxGroups = 4;
constexpr int kMaxDevices = 64;
cudaStream_t group_stream(int g) {
  static std::mutex mu;
  static cudaStream_t streams[kMaxDevices][kMaxGroups] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!streams[dev][g] && cudaStreamCreateWithFlags(&streams[dev][g], cudaStreamNonBlocking) != cudaSuccess)
    streams[dev][g] = nullptr;
  return streams[dev][g];
}

Problem make_problem(int n, int T, int d, int H, const am_opts_t* o, const Tables& tb) {
  Problem p{};
  p.H = H; p.n = n; p.T = T; p.d = d;
  p.ldn = round_up(n, 32);
  p.in_dtype = o->in_dtype;
  p.scale = o->scale > 0.f ? o->scale : (float)(1.0 / sqrt((double)d));
  p.select_highest = o->select_mode == AM_SELECT_HIGHEST;
  p.topk = p.select_highest ? kHighestChunk : o->topk;
  p.refit_every = p.select_highest ? 1 : o->refit_every;
  p.kR = p.topk * p.refit_every;
  p.nnls_max_iter = o->nnls_max_iter;
  p.ridge = o->ridge;
  p.w_floor_rel = o->w_floor_rel;
  p.max_t = tb.max_t;
  p.has_bias = o->key_bias != nullptr;
  p.corr_bf16 = bf16_copy(o);
  p.corr_recompute = o->corr_mode == AM_CORR_RECOMPUTE;
  p.corr_bounded = !p.select_highest && (o->corr_mode == AM_CORR_BOUNDED || o->corr_mode == AM_CORR_AUTO);
  if (p.select_highest) p.corr_recompute = false;
  p.key_rows = tb.koff[H];
  p.wait_cycles = o->wait_cycles > 0 ? (long long)o->wait_cycles : kDefaultWaitCycles;
  return p;
}

struct WsHeader {
  uint32_t magic;
  int32_t H;
};

// Size of the wave region for heads [h0, h1) of `tb`.
size_t wave_bytes(const Tables& tb, int n, int T, int d, int h0, int h1, bool corr_bf16, bool tcn) {
  const int64_t st = tb.cu_t[h1] - tb.cu_t[h0], st2 = tb.cu_t2[h1] - tb.cu_t2[h0];
  return plan(n, T, d, h1 - h0, st, st2, corr_bf16, 0, tcn).total;
}

// Waves of consecutive heads: each takes as many heads as fit in `region`
// bytes.  Empty when one head does not fit.
std::vector<std::pair<int, int>> plan_waves(const Tables& tb, int n, int T, int d, bool corr_bf16, bool tcn,
                                            size_t region) {
  const int H = (int)tb.t.size();
  std::vector<std::pair<int, int>> waves;
  int h0 = 0;
  while (h0 < H) {
    int h1 = h0;
    while (h1 < H && wave_bytes(tb, n, T, d, h0, h1 + 1, corr_bf16, tcn) <= region) ++h1;
    if (h1 == h0) return {};
    waves.emplace_back(h0, h1);
    h0 = h1;
  }
  return waves;
}

const char* cbyte(const void* p, int64_t off) { return reinterpret_cast<const char*>(p) + off; }
char* mbyte(void* p, int64_t off) { return reinterpret_cast<char*>(p) + off; }

}  // namespace
}  // namespace am

using namespace am;

extern "C" {

am_status_t am_default_opts(am_opts_t* opts) {
  if (!opts) return AM_ERR_INVALID_ARG;
  memset(opts, 0, sizeof(*opts));
  opts->in_dtype = AM_BF16;
  opts->topk = 1;
  opts->refit_every = 1;
  opts->scale = 0.f;
  opts->ridge = 1e-6f;
  opts->w_floor_rel = 1e-12f;
  opts->corr_mode = AM_CORR_AUTO;
  return AM_OK;
}

am_status_t am_workspace_size(int32_t n, int32_t T, int32_t d, int32_t num_heads,
                              const int32_t* budgets, const am_opts_t* opts, size_t* bytes) {
  return am_workspace_size_waves(n, T, d, num_heads, budgets, opts, num_heads, bytes);
}

am_status_t am_workspace_size_waves(int32_t n, int32_t T, int32_t d, int32_t num_heads,
                                    const int32_t* budgets, const am_opts_t* opts, int32_t wave_heads,
                                    size_t* bytes) {
  if (!bytes || wave_heads < 1) return AM_ERR_INVALID_ARG;
  Tables tb;
  am_status_t st = check_shape(n, T, d, num_heads, budgets, opts, &tb);
  if (st != AM_OK) return st;
  // the largest region over every window of wave_heads consecutive heads, so
  // that the call's waves (each as many heads as fit) hold wave_heads heads
  const int W = std::min(wave_heads, num_heads);
  size_t region = 0;
  for (int h0 = 0; h0 + W <= num_heads; ++h0)
    region = std::max(region, wave_bytes(tb, n, T, d, h0, h0 + W, bf16_copy(opts), tc_normal(opts, d)));
  *bytes = prefix_bytes(num_heads) + region;
  return AM_OK;
}

am_status_t am_workspace_view(int32_t n, int32_t T, int32_t d, int32_t num_heads, const int32_t* budgets,
                              const am_opts_t* opts, am_workspace_view_t* view) {
  if (!view) return AM_ERR_INVALID_ARG;
  Tables tb;
  am_status_t st = check_shape(n, T, d, num_heads, budgets, opts, &tb);
  if (st != AM_OK) return st;
  const Layout L = plan(n, T, d, num_heads, tb.sum_t, tb.sum_t2, bf16_copy(opts), prefix_bytes(num_heads),
                        tc_normal(opts, d));
  view->phiT = L.phiT;
  view->mass = L.m;
  view->target = L.Y;
  view->shift = L.shift;
  view->ldn = round_up(n, 32);
  view->reserved = 0;
  view->weights = L.w;
  view->resid = L.r;
  view->rows_evaluated = stats_offset(num_heads);
  view->column_norms = L.cnorm;
  view->nnls_refits = refits_offset(num_heads);
  view->nnls_solves = solves_offset(num_heads);
  return AM_OK;
}

am_status_t am_compact_heads(const void* Q, const void* K, const void* V, int32_t n, int32_t T,
                             int32_t d, int32_t H, const int32_t* budgets, const am_opts_t* opts,
                             void* workspace, size_t workspace_bytes, const int64_t* out_offsets,
                             void* C_k, float* beta, float* C_v, int32_t* indices, void* stream) {
  return am::compact_heads_impl(Q, K, V, n, T, d, H, budgets, opts, workspace, workspace_bytes, out_offsets, C_k,
                                beta, C_v, indices, stream, am::kMaxGroups);
}

}  // extern "C"

namespace am {

#define AM_TRY(x)                      \
  do {                                 \
    if ((x) != cudaSuccess) return AM_ERR_CUDA; \
  } while (0)

// Outputs and optional inputs of one wave, already offset to its first head.
struct WaveIO {
  const void *Q, *K, *V;
  const float* key_bias;
  const float* shift_in;
  void* C_k;
  float *beta, *C_v;
  int32_t* indices;
  int32_t* pick_order;
  float *pick_corr, *w_out, *shift_out;
  double* residual_out;
};

// The compaction of one wave of heads, on stream s (internal group streams
// forked from and joined back into s).
am_status_t run_wave(const Problem& p, Work w, const Tables& tb, int G, int32_t* gorder, const WaveIO& io,
                     cudaStream_t s) {
  const int H = p.H;
  const bool tc = phi_tc_supported(p);
  if (!tc || !p.corr_bounded) w.cnpart = nullptr;   // column norms from the features instead
  if (io.shift_in) {
    AM_TRY(launch_shift_copy(io.shift_in, w.shift, H, s));
  } else if (tc) {
    AM_TRY(launch_shift_init(w.shift, H, s));
    AM_TRY(launch_shift_max_tc(p, io.Q, io.K, io.key_bias, w, reinterpret_cast<uint32_t*>(w.shift), s));
    AM_TRY(launch_shift_decode(w.shift, H, s));
  } else {
    AM_TRY(launch_shift_max(p, w, io.Q, io.K, io.key_bias, w.shift, s));
  }
  if (tc) {
    AM_TRY(launch_phi_tc(p, io.Q, io.K, io.V, io.key_bias, w, s));
  } else {
    AM_TRY(launch_phi(p, io.Q, io.K, io.key_bias, w, s));
    AM_TRY(launch_y_m(p, io.V, w, s));
  }
  AM_TRY(launch_omp_init(p, w, s));
  if (p.corr_bounded) AM_TRY(launch_column_norms(p, w, s));
  AM_TRY(cudaMemsetAsync(w.gcount, 0, ((size_t)tb.sum_t + H) * 4, s));
  AM_TRY(cudaMemsetAsync(w.rcount, 0, (size_t)H * 4, s));
  AM_TRY(cudaMemsetAsync(w.ghist, 0, (size_t)H * 1024 * 4, s));
  AM_TRY(cudaMemsetAsync(w.gcnt, 0, (size_t)H * 4, s));
  AM_TRY(cudaMemsetAsync(w.ccount, 0, (size_t)H * 4, s));
  if (p.select_highest) AM_TRY(launch_select_highest(p, w, s));
  const CorrInputs cin{io.Q, io.K, io.key_bias};
  // the NNLS refit keeps a head's factor in shared memory when its budget is
  // at most lcap; per pass, the active heads above it (a prefix of the order)
  // get a launch of their own with a small shared-memory footprint
  const int lcap = nnls_smem_cap(p.max_t);
  // (count of those, largest budget among the rest)
  auto big_heads = [&](const int32_t* ord, int active) {
    int nb = 0;
    while (nb < active && tb.t[ord[nb]] > lcap) ++nb;
    return std::make_pair(nb, nb < active ? (int)tb.t[ord[nb]] : 0);
  };
  if (G == 1) {
    for (int pass = 0; pass < (int)tb.active.size(); ++pass) {
      const auto bh = big_heads(tb.order.data(), tb.active[pass]);
      AM_TRY(launch_omp_pass(p, w, pass, tb.active[pass], bh.first, bh.second, cin, s));
    }
  } else {
    // fork the groups off the caller's stream, issue their passes interleaved,
    // and make the caller's stream wait for every group
    cudaEvent_t fork, join[kMaxGroups];
    AM_TRY(cudaEventCreateWithFlags(&fork, cudaEventDisableTiming));
    AM_TRY(cudaEventRecord(fork, s));
    std::vector<Work> wg(G, w);
    for (int g = 0; g < G; ++g) {
      wg[g].order = gorder + tb.gstart[g];
      AM_TRY(cudaStreamWaitEvent(group_stream(g), fork, 0));
    }
    const int maxp = (int)tb.active.size();
    for (int pass = 0; pass < maxp; ++pass)
      for (int g = 0; g < G; ++g)
        if (pass < (int)tb.gactive[g].size()) {
          const auto bh = big_heads(tb.gorder.data() + tb.gstart[g], tb.gactive[g][pass]);
          AM_TRY(launch_omp_pass(p, wg[g], pass, tb.gactive[g][pass], bh.first, bh.second, cin, group_stream(g)));
        }
    for (int g = 0; g < G; ++g) {
      AM_TRY(cudaEventCreateWithFlags(&join[g], cudaEventDisableTiming));
      AM_TRY(cudaEventRecord(join[g], group_stream(g)));
      AM_TRY(cudaStreamWaitEvent(s, join[g], 0));
      cudaEventDestroy(join[g]);   // released once the work it marks completes
    }
    cudaEventDestroy(fork);
  }
  if (io.residual_out) AM_TRY(launch_residual_norm(p, w, io.residual_out, s));
  AM_TRY(launch_finalize(p, w, io.K, io.key_bias, io.C_k, io.beta, io.indices, io.w_out, io.pick_order,
                         io.pick_corr, s));
  AM_TRY(launch_value_fit(p, w, io.C_v, s));
  if (io.shift_out) AM_TRY(launch_shift_copy(w.shift, io.shift_out, H, s));
  return AM_OK;
}

am_status_t compact_heads_impl(const void* Q, const void* K, const void* V, int32_t n, int32_t T, int32_t d,
                               int32_t H, const int32_t* budgets, const am_opts_t* opts, void* workspace,
                               size_t workspace_bytes, const int64_t* out_offsets, void* C_k, float* beta,
                               float* C_v, int32_t* indices, void* stream, int max_groups) {
  if (!Q || !K || !V || !C_k || !beta || !C_v || !indices || !out_offsets) return AM_ERR_INVALID_ARG;
  Tables tb;
  am_status_t st = check_shape(n, T, d, H, budgets, opts, &tb);
  if (st != AM_OK) return st;
  for (int h = 0; h <= H; ++h)
    if (out_offsets[h] != tb.cu_t[h]) return AM_ERR_INVALID_ARG;
  if (!workspace || ((uintptr_t)workspace % kAlign) != 0) return AM_ERR_WORKSPACE;
  const bool bf16 = bf16_copy(opts);
  const size_t pre = prefix_bytes(H);
  if (workspace_bytes <= pre) return AM_ERR_WORKSPACE;
  const bool tcn = tc_normal(opts, d);
  const std::vector<std::pair<int, int>> waves = plan_waves(tb, n, T, d, bf16, tcn, workspace_bytes - pre);
  if (waves.empty()) return AM_ERR_WORKSPACE;
  // head groups on internal streams (one group: everything on the caller's stream)
  int G = std::max(1, std::min(max_groups, H));
  for (int g = 0; g < G && G > 1; ++g)
    if (!group_stream(g)) G = 1;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* base = reinterpret_cast<char*>(workspace);
  const int kR = picks_per_pass(opts);
  const size_t esz = opts->in_dtype == AM_BF16 ? 2 : 4;
  // every wave's tables, packed into one host block and copied once
  const size_t tables_at = align_up(kWsHeaderBytes + (size_t)H * 4);
  std::vector<unsigned char> host_tables;
  std::vector<Tables> wt(waves.size());
  std::vector<Work> ww(waves.size());
  std::vector<int32_t*> wgorder(waves.size());
  for (size_t k = 0; k < waves.size(); ++k) {
    const int h0 = waves[k].first, h1 = waves[k].second, Hw = h1 - h0;
    sub_tables(tb, h0, h1, kR, &wt[k]);
    set_groups(&wt[k], wt[k].passes, std::min(G, Hw));
    const Layout L = plan(n, T, d, Hw, wt[k].sum_t, wt[k].sum_t2, bf16, pre, tcn);
    ww[k] = bind(L, base, bf16);
    ww[k].status = reinterpret_cast<int32_t*>(base + kWsHeaderBytes) + h0;
    ww[k].rows_eval = reinterpret_cast<unsigned long long*>(base + stats_offset(H)) + h0;
    ww[k].nnls_refits = reinterpret_cast<int32_t*>(base + refits_offset(H)) + h0;
    ww[k].nnls_solves = reinterpret_cast<int32_t*>(base + solves_offset(H)) + h0;
    ww[k].nrm_ata = wt[k].sum_t2;
    ww[k].nrm_stride = wt[k].sum_t2 + wt[k].sum_t * d;
    ww[k].sum_t = wt[k].sum_t;
    pack_tables(wt[k], Hw, &host_tables, &ww[k], base + tables_at + host_tables.size(), &wgorder[k]);
  }
  if (host_tables.size() > stats_offset(H) - tables_at) return AM_ERR_WORKSPACE;   // cannot happen: 64 bytes per head

  WsHeader hdr{kWsMagic, H};
  // Pageable sources: both copies are staged before cudaMemcpyAsync returns.
  AM_TRY(cudaMemcpyAsync(base, &hdr, sizeof(hdr), cudaMemcpyHostToDevice, s));
  AM_TRY(cudaMemcpyAsync(base + tables_at, host_tables.data(), host_tables.size(), cudaMemcpyHostToDevice, s));
  AM_TRY(cudaMemsetAsync(base + kWsHeaderBytes, 0, (size_t)H * 4, s));
  AM_TRY(cudaMemsetAsync(base + stats_offset(H), 0, solves_offset(H) + (size_t)H * 4 - stats_offset(H), s));

  for (size_t k = 0; k < waves.size(); ++k) {
    const int h0 = waves[k].first, h1 = waves[k].second, Hw = h1 - h0;
    const Problem p = make_problem(n, T, d, Hw, opts, wt[k]);
    const int64_t krow = tb.koff[h0], orow = tb.cu_t[h0];
    WaveIO io{};
    io.Q = cbyte(Q, (int64_t)h0 * n * d * (int64_t)esz);
    io.K = cbyte(K, krow * d * (int64_t)esz);
    io.V = cbyte(V, krow * d * (int64_t)esz);
    io.key_bias = opts->key_bias ? opts->key_bias + krow : nullptr;
    io.shift_in = opts->shift ? opts->shift + h0 : nullptr;
    io.C_k = mbyte(C_k, orow * d * (int64_t)esz);
    io.beta = beta + orow;
    io.C_v = C_v + orow * d;
    io.indices = indices + orow;
    io.pick_order = opts->pick_order ? opts->pick_order + orow : nullptr;
    io.pick_corr = opts->pick_corr ? opts->pick_corr + orow : nullptr;
    io.w_out = opts->w_out ? opts->w_out + orow : nullptr;
    io.shift_out = opts->shift_out ? opts->shift_out + h0 : nullptr;
    io.residual_out = opts->residual_out ? opts->residual_out + h0 : nullptr;
    st = run_wave(p, ww[k], wt[k], std::min(G, Hw), wgorder[k], io, s);
    if (st != AM_OK) return st;
  }
  return AM_OK;
}
#undef AM_TRY
}  // namespace am

extern "C" {

am_status_t am_get_status(const void* workspace, int32_t H, int32_t* per_head, void* stream) {
  if (!workspace || H < 1) return AM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return AM_ERR_CUDA;
  WsHeader hdr{};
  if (cudaMemcpy(&hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost) != cudaSuccess) return AM_ERR_CUDA;
  if (hdr.magic != kWsMagic || hdr.H != H) return AM_ERR_WORKSPACE;
  std::vector<int32_t> raw(H);
  if (cudaMemcpy(raw.data(), reinterpret_cast<const char*>(workspace) + kWsHeaderBytes, (size_t)H * 4,
                 cudaMemcpyDeviceToHost) != cudaSuccess)
    return AM_ERR_CUDA;
  int worst = 0;
  for (int h = 0; h < H; ++h) {
    const int code = raw[h] % 1000;
    if (per_head) per_head[h] = code;
    if (raw[h] > worst) worst = raw[h];
  }
  return (am_status_t)(worst % 1000);
}

const char* am_status_string(am_status_t s) {
  switch (s) {
    case AM_OK: return "ok";
    case AM_ERR_INVALID_ARG: return "invalid argument";
    case AM_ERR_BUDGET: return "budget outside [1, T]";
    case AM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case AM_ERR_NONFINITE: return "non-finite feature or solution";
    case AM_ERR_CUDA: return "CUDA runtime error";
    case AM_ERR_TIMEOUT: return "bounded device wait ran out";
    case AM_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case AM_WARN_NOT_CONVERGED: return "NNLS stopped at its iteration cap";
    case AM_ERR_NOT_SPD: return "value-fit matrix not positive definite";
    case AM_WARN_MASS_UNDERFLOW: return "a reference query's features all underflowed in fp32";
  }
  return "unknown status";
}

int32_t am_version(void) { return 100; }

}  // extern "C"
