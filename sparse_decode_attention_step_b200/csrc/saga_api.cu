// C ABI of the SAGA + Atop-N decode step: argument checks, the work plan
// (split of l_kv across CTAs, workspace carve-up) and the kernel launches.
// Nothing here allocates device memory or synchronises, except
// saga_read_device_error, which synchronises by contract.
#include <cmath>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "saga.h"

namespace saga {
namespace {

constexpr int64_t kSms = 148;              // B200 SMs: the persistent grid
constexpr int64_t kTileKeys = 128;         // split lengths are multiples of a K tile
constexpr int64_t kUnitTiles = 32;         // grid-per-split kernels: at most about this many tiles per split
constexpr int64_t kPersistTiles = 128;     // persistent kernel: at most about this many tiles per unit
constexpr int64_t kGridCtasPerSm = 4;      // grid-per-split kernels: at least this many units per SM
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Plan {
  int S;                    // scan / split-kernel units per (b, key head)
  int64_t split_len;        // positions per unit
  // tensor-core path: the gather kernel's own splits of a row
  bool lists;               // the scan writes per-head kept lists
  int SB;                   // gather splits per (b, query head)
  int64_t blk_per_split;    // 32-position blocks per gather split
  int64_t nblk;             // 32-position blocks per row
  // the records the combine merges: comb_S per (b, j), comb_split_len positions each
  int comb_S;
  int64_t comb_split_len;
  // radix select: per row, the list of the top-byte bucket (gcap keys at most)
  int gcap;
  size_t off_partials, off_lmask, off_lscore, off_scores, off_hist, off_gcount, off_hist1,
      off_gcand, off_tau, off_tie, total;
};

// Keys per row in the radix select's bucket list: half the row (the top-byte
// bucket of a score row can hold a third of it), at least 16384, a multiple
// of 4.
int select_list_cap(int64_t max_l_kv) {
  const int64_t c = std::max<int64_t>(16384, (max_l_kv / 2 + 3) / 4 * 4);
  return static_cast<int>(c);
}

bool use_tc(const saga_shape &s);

// Splits of equal length, a multiple of the K tile.
// Grid-per-split kernels (SIMT, dense): the (b, kh, split) units number about a
// whole multiple of the SM count, with at most about kUnitTiles tiles each and,
// where the sequence is long enough, at least as many per SM as fit on one
// (`ctas_per_sm`, at most kGridCtasPerSm, which sizes the workspace): those
// kernels hide their load latency only with every resident slot filled, and
// more splits than slots only add waves and combine work.
// Persistent tensor-core scan: at most one unit per SM and wave, units of up
// to about kPersistTiles tiles. Its gather kernel splits each (b, query head)
// row on its own, into at most kGatherCtas CTAs in all (about four waves of
// eight resident per SM, so that heads that keep more rows than others are
// balanced out by the block scheduler) where the rows allow, each at least
// kGatherMinBlocks blocks of 32 positions long; the combine merges the
// gather's records.
constexpr int64_t kGatherCtas = 32 * kSms;
constexpr int64_t kGatherMinBlocks = 64;

Plan make_plan(const saga_shape &s, bool persistent, int64_t ctas_per_sm = kGridCtasPerSm) {
  Plan p{};
  const int64_t rows = static_cast<int64_t>(s.B) * s.h_k;
  const int64_t L = std::max<int64_t>(1, s.max_l_kv);
  const int64_t tiles = rows * ceil_div(L, kTileKeys);
  int64_t s_target;
  if (persistent) {
    const int64_t waves = std::max<int64_t>(1, ceil_div(tiles, kSms * kPersistTiles));
    s_target = std::max<int64_t>(1, kSms * waves / rows);
  } else {
    const int64_t waves = std::max<int64_t>(1, ceil_div(tiles, kSms * kUnitTiles));
    const int64_t slots = std::min(std::max<int64_t>(1, ctas_per_sm), kGridCtasPerSm);
    s_target = std::max<int64_t>(1, ceil_div(kSms * std::max(waves, slots), rows));
  }
  p.split_len = ceil_div(ceil_div(L, s_target), kTileKeys) * kTileKeys;
  p.S = static_cast<int>(ceil_div(L, p.split_len));
  p.comb_S = p.S;
  p.comb_split_len = p.split_len;
  p.nblk = ceil_div(L, 32);
  if (persistent && saga_tc_supports(s.dtype, s.d, s.h_q, s.h_k, s.h_v)) {
    p.lists = true;
    const int64_t items = static_cast<int64_t>(s.B) * s.h_q;
    const int64_t max_sb = std::max<int64_t>(1, p.nblk / kGatherMinBlocks);
    const int64_t sb = std::min(max_sb, std::max<int64_t>(1, kGatherCtas / items));
    p.blk_per_split = ceil_div(p.nblk, sb);
    p.SB = static_cast<int>(ceil_div(p.nblk, p.blk_per_split));
    p.comb_S = p.SB;
    p.comb_split_len = p.blk_per_split * 32;
  }
  const size_t rec = static_cast<size_t>(s.d + kRecPad) * sizeof(float);
  const size_t lists = p.lists ? static_cast<size_t>(s.B) * s.h_q * p.nblk : 0;
  p.off_partials = kAlign;   // [0, 256): device error word, then the step's abort word
  p.off_lmask = align_up(p.off_partials + static_cast<size_t>(s.B) * s.h_q * p.comb_S * rec);
  p.off_lscore = align_up(p.off_lmask + lists * sizeof(uint32_t));
  p.off_scores = align_up(p.off_lscore + lists * 32 * sizeof(float));
  p.off_hist = align_up(p.off_scores + static_cast<size_t>(s.B) * s.h_q * s.max_l_kv * sizeof(float));
  // the bucket counts and digit-1 histograms follow the top-byte histograms
  // directly: one memset clears all three
  p.gcap = select_list_cap(s.max_l_kv);
  p.off_gcount = p.off_hist + static_cast<size_t>(s.B) * s.h_q * 256 * sizeof(uint32_t);
  p.off_hist1 = p.off_gcount + static_cast<size_t>(s.B) * s.h_q * sizeof(uint32_t);
  p.off_gcand = align_up(p.off_hist1 + static_cast<size_t>(s.B) * s.h_q * 256 * sizeof(uint32_t));
  p.off_tau = align_up(p.off_gcand + static_cast<size_t>(s.B) * s.h_q * p.gcap * sizeof(uint32_t));
  p.off_tie = align_up(p.off_tau + static_cast<size_t>(s.B) * s.h_q * sizeof(float));
  p.total = align_up(p.off_tie + static_cast<size_t>(s.B) * s.h_q * sizeof(int32_t));
  return p;
}

// The plan of the SAGA calls (step, refresh, debug scores) of a shape.
Plan saga_plan(const saga_shape &s) { return make_plan(s, use_tc(s)); }

// One workspace serves every call of a shape: the larger of the step's plan
// and the grid-per-split plan (dense calls, at most kGridCtasPerSm units per SM).
size_t workspace_bytes(const saga_shape &s) {
  return std::max(saga_plan(s).total, make_plan(s, false).total);
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

saga_status check_shape(const saga_shape *s) {
  if (s == nullptr) return SAGA_ERR_INVALID_ARG;
  if (s->B < 1 || s->h_q < 1 || s->h_k < 1 || s->h_v < 1 || s->d < 1) return SAGA_ERR_INVALID_ARG;
  if (s->h_k > s->h_v || s->h_v > s->h_q) return SAGA_ERR_INVALID_ARG;
  if (s->dtype != SAGA_F32 && s->dtype != SAGA_BF16) return SAGA_ERR_INVALID_ARG;
  if (s->max_l_kv < 0 || s->cap < s->max_l_kv) return SAGA_ERR_INVALID_ARG;
  if (s->h_q % s->h_v != 0 || s->h_v % s->h_k != 0) return SAGA_ERR_UNSUPPORTED;
  if (s->h_q / s->h_k > kMaxGroup) return SAGA_ERR_UNSUPPORTED;
  if (s->d != 64 && s->d != 128) return SAGA_ERR_UNSUPPORTED;
  if (s->max_l_kv > INT32_MAX) return SAGA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->B) * s->h_k > 65535) return SAGA_ERR_UNSUPPORTED;
  const int64_t esz = s->dtype == SAGA_F32 ? 4 : 2;
  const int64_t st[6] = {s->q_stride_b, s->q_stride_h, s->k_stride_b,
                         s->k_stride_h, s->v_stride_b, s->v_stride_h};
  for (int64_t x : st)
    if (x <= 0 || (x * esz) % 16 != 0) return SAGA_ERR_INVALID_ARG;
  if (s->q_stride_h < s->d || s->k_stride_h < s->cap * s->d || s->v_stride_h < s->cap * s->d)
    return SAGA_ERR_INVALID_ARG;
  return SAGA_OK;
}

saga_status check_ws(const saga_shape &s, void *ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned(ws, kAlign)) return SAGA_ERR_WORKSPACE;
  if (ws_bytes < workspace_bytes(s)) return SAGA_ERR_WORKSPACE;
  return SAGA_OK;
}

saga_status check_inputs(const saga_shape &s, const void *q, const void *K, const int32_t *l_kv) {
  if (q == nullptr || K == nullptr || l_kv == nullptr) return SAGA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(K, 16) || !aligned(l_kv, 4)) return SAGA_ERR_INVALID_ARG;
  (void)s;
  return SAGA_OK;
}

StepParams base_params(const saga_shape &s, const Plan &pl, const void *q, const void *K,
                       const void *V, const int32_t *l_kv, void *ws) {
  StepParams p{};
  char *wsb = static_cast<char *>(ws);
  p.q = q; p.K = K; p.V = V; p.l_kv = l_kv;
  p.err = static_cast<int32_t *>(ws);
  p.abort = static_cast<int32_t *>(ws) + 1;
  p.partials = reinterpret_cast<float *>(wsb + pl.off_partials);
  if (pl.lists) {
    p.lmask = reinterpret_cast<uint32_t *>(wsb + pl.off_lmask);
    p.lscore = reinterpret_cast<float *>(wsb + pl.off_lscore);
    p.nblk = pl.nblk;
  }
  p.q_sb = s.q_stride_b; p.q_sh = s.q_stride_h;
  p.k_sb = s.k_stride_b; p.k_sh = s.k_stride_h;
  p.v_sb = s.v_stride_b; p.v_sh = s.v_stride_h;
  p.cap = s.cap; p.max_l_kv = s.max_l_kv; p.row_stride = s.max_l_kv;
  p.split_len = pl.split_len;
  p.B = s.B; p.h_q = s.h_q; p.h_k = s.h_k; p.h_v = s.h_v; p.S = pl.S;
  p.scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(s.d)));
  return p;
}

int group_pad(const saga_shape &s) { return ((s.h_q / s.h_k) + 3) / 4 * 4; }


// The tensor-core kernel takes the score-producing modes (dump, step) of the
// shapes it supports (a failure there is reported, never replaced by another
// path); every other shape, and the from-scores mode, runs on the SIMT split
// kernel. The choice depends on the shape alone, so a refresh and the steps
// that follow it always see scores from the same kernel.
bool use_tc(const saga_shape &s) {
  return saga_tc_supports(s.dtype, s.d, s.h_q, s.h_k, s.h_v);
}

cudaError_t launch_split(const saga_shape &s, const StepParams &p, int mode, cudaStream_t st) {
  if (mode != kModeFromScores && use_tc(s)) return launch_saga_tc(p, mode, s.d, st);
  return launch_saga_split(p, mode, s.dtype, s.d, group_pad(s), st);
}

// Select + PV over the stored thresholds, then the combine. Tensor-core
// shapes: the scan kernel writes the kept lists, the gather kernel the
// records; other shapes: the SIMT split kernel does both.
saga_status run_step(const saga_shape &s, const Plan &pl, StepParams p, int mode,
                     float *out, int32_t *sel_count, cudaStream_t st) {
  const bool tc = mode != kModeFromScores && use_tc(s);
  cudaError_t e = launch_split(s, p, mode, st);
  if (e != cudaSuccess)
    return cuda_fail(e, !tc ? "split kernel" : (p.scores_in ? "scan kernel (stored scores)" : "scan kernel"));
  if (tc) {
    GatherParams g{};
    g.V = static_cast<const uint16_t *>(p.V);
    g.v_sb = p.v_sb; g.v_sh = p.v_sh;
    g.l_kv = p.l_kv; g.cap = p.cap; g.max_l_kv = p.max_l_kv;
    g.lmask = p.lmask; g.lscore = p.lscore; g.nblk = p.nblk;
    g.partials = p.partials; g.abort = p.abort; g.err = p.err;
    g.B = s.B; g.h_q = s.h_q; g.SB = pl.SB; g.hpv = s.h_q / s.h_v;
    g.blk_per_split = pl.blk_per_split;
    if ((e = launch_gather(g, s.d, st)) != cudaSuccess) return cuda_fail(e, "gather kernel");
  }
  return cuda_check(launch_combine(p.partials, p.l_kv, tc ? p.abort : nullptr, out, sel_count, s.B,
                                   s.h_q, s.d, pl.comb_S, pl.comb_split_len, s.cap, s.max_l_kv, st),
                    "combine kernel");
}

// Full attention (Eq. 2-4) with the shape's key and value head maps: the
// dense kernel, then the combine.
saga_status run_dense(const saga_shape &s, const void *q, const void *K, const void *V,
                      const int32_t *l_kv, float *out, void *ws, size_t ws_bytes,
                      cudaStream_t st) {
  if (!dense_supports(s.h_q, s.h_k, s.h_v)) return SAGA_ERR_UNSUPPORTED;
  saga_status r = check_inputs(s, q, K, l_kv);
  if (r != SAGA_OK) return r;
  if (V == nullptr || !aligned(V, 16) || out == nullptr || !aligned(out, 16))
    return SAGA_ERR_INVALID_ARG;
  if ((r = check_ws(s, ws, ws_bytes)) != SAGA_OK) return r;
  const Plan pl = make_plan(s, false, dense_ctas_per_sm(s.dtype, s.d, s.h_q, s.h_k, s.h_v));
  StepParams p = base_params(s, pl, q, K, V, l_kv, ws);
  cudaError_t e = launch_dense_split(p, s.dtype, s.d, st);
  if (e != cudaSuccess) return cuda_fail(e, "dense kernel");
  return cuda_check(launch_combine(p.partials, l_kv, nullptr, out, nullptr, s.B, s.h_q, s.d, pl.S,
                                   pl.split_len, s.cap, s.max_l_kv, st),
                    "combine kernel");
}

thread_local char g_last_error[256] = "";

// The top-byte histograms the score pass fills, and the bucket counts and
// digit-1 histograms of the radix select, cleared together (they are
// adjacent in the workspace).
struct SelectBufs {
  uint32_t *hist = nullptr, *gcount = nullptr, *hist1 = nullptr, *gcand = nullptr;
};
cudaError_t clear_select_counts(const saga_shape &s, const Plan &pl, void *ws, SelectBufs *b,
                                cudaStream_t st) {
  char *wsb = static_cast<char *>(ws);
  b->hist = reinterpret_cast<uint32_t *>(wsb + pl.off_hist);
  b->gcount = reinterpret_cast<uint32_t *>(wsb + pl.off_gcount);
  b->hist1 = reinterpret_cast<uint32_t *>(wsb + pl.off_hist1);
  b->gcand = reinterpret_cast<uint32_t *>(wsb + pl.off_gcand);
  const size_t rows = static_cast<size_t>(s.B) * s.h_q;
  return cudaMemsetAsync(b->hist, 0, rows * (256 + 1 + 256) * sizeof(uint32_t), st);
}

}  // namespace

saga_status cuda_fail(cudaError_t e, const char *where) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e),
                cudaGetErrorString(e));
  cudaGetLastError();   // a failed launch's error is not sticky: clear it for the next call
  return SAGA_ERR_CUDA;
}

// Scratch a plain step needs (error word + per-split states; no score rows).
size_t plain_step_scratch_bytes(const saga_shape &s) { return saga_plan(s).off_scores; }

// saga_decode_step's checks and launches with a caller-chosen scratch buffer
// in place of the workspace (sel_mask not supported).
saga_status plain_step_with_scratch(const saga_shape *shape, const void *q, const void *K,
                                    const void *V, const int32_t *l_kv, const float *tau,
                                    float *out, int32_t *sel_count, void *scratch,
                                    size_t scratch_bytes, cudaStream_t st) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  const saga_shape &s = *shape;
  if ((r = check_inputs(s, q, K, l_kv)) != SAGA_OK) return r;
  if (V == nullptr || !aligned(V, 16) || tau == nullptr || out == nullptr ||
      !aligned(tau, 4) || !aligned(out, 16) || (sel_count && !aligned(sel_count, 4)))
    return SAGA_ERR_INVALID_ARG;
  if (scratch == nullptr || !aligned(scratch, kAlign) || scratch_bytes < plain_step_scratch_bytes(s))
    return SAGA_ERR_WORKSPACE;
  const Plan pl = saga_plan(s);
  StepParams p = base_params(s, pl, q, K, V, l_kv, scratch);
  p.tau = tau;
  return run_step(s, pl, p, kModeStep, out, sel_count, st);
}

}  // namespace saga

using namespace saga;

extern "C" {

void saga_shape_contiguous(saga_shape *s, int32_t B, int32_t h_q, int32_t h_k, int32_t h_v,
                           int32_t d, int32_t dtype, int64_t cap, int64_t max_l_kv) {
  if (s == nullptr) return;
  std::memset(s, 0, sizeof(*s));
  s->B = B; s->h_q = h_q; s->h_k = h_k; s->h_v = h_v; s->d = d; s->dtype = dtype;
  s->cap = cap; s->max_l_kv = max_l_kv;
  s->q_stride_h = d; s->q_stride_b = static_cast<int64_t>(h_q) * d;
  s->k_stride_h = cap * d; s->k_stride_b = static_cast<int64_t>(h_k) * cap * d;
  s->v_stride_h = cap * d; s->v_stride_b = static_cast<int64_t>(h_v) * cap * d;
}

size_t saga_workspace_size(const saga_shape *shape, int32_t N) {
  (void)N;
  if (check_shape(shape) != SAGA_OK) return 0;
  return workspace_bytes(*shape);
}

saga_status saga_workspace_init(void *ws, size_t ws_bytes, saga_stream_t stream) {
  if (ws == nullptr || !aligned(ws, kAlign) || ws_bytes < kAlign) return SAGA_ERR_WORKSPACE;
  return cuda_check(cudaMemsetAsync(ws, 0, kAlign, reinterpret_cast<cudaStream_t>(stream)),
                    "cudaMemsetAsync (error word)");
}

saga_status saga_decode_step(const saga_shape *shape, const void *q, const void *K,
                             const void *V, const int32_t *l_kv, const float *tau, float *out,
                             int32_t *sel_count, uint8_t *sel_mask, void *ws, size_t ws_bytes,
                             saga_stream_t stream) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  const saga_shape &s = *shape;
  if ((r = check_inputs(s, q, K, l_kv)) != SAGA_OK) return r;
  if (V == nullptr || !aligned(V, 16) || tau == nullptr || out == nullptr ||
      !aligned(tau, 4) || !aligned(out, 16) || (sel_count && !aligned(sel_count, 4)))
    return SAGA_ERR_INVALID_ARG;
  if ((r = check_ws(s, ws, ws_bytes)) != SAGA_OK) return r;
  const Plan pl = saga_plan(s);
  StepParams p = base_params(s, pl, q, K, V, l_kv, ws);
  p.tau = tau;
  p.sel_mask = sel_mask;
  return run_step(s, pl, p, kModeStep, out, sel_count, reinterpret_cast<cudaStream_t>(stream));
}

saga_status saga_refresh_threshold(const saga_shape *shape, const void *q, const void *K,
                                   const void *V, const int32_t *l_kv, int32_t N, float *tau,
                                   float *out, int32_t *sel_count, uint8_t *sel_mask,
                                   float *scores, void *ws, size_t ws_bytes,
                                   saga_stream_t stream) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  const saga_shape &s = *shape;
  if ((r = check_inputs(s, q, K, l_kv)) != SAGA_OK) return r;
  if (N < 1 || tau == nullptr || !aligned(tau, 4)) return SAGA_ERR_INVALID_ARG;
  if ((V == nullptr) != (out == nullptr)) return SAGA_ERR_INVALID_ARG;
  if (V != nullptr && (!aligned(V, 16) || !aligned(out, 16))) return SAGA_ERR_INVALID_ARG;
  if ((scores && !aligned(scores, 4)) || (sel_count && !aligned(sel_count, 4)))
    return SAGA_ERR_INVALID_ARG;
  if ((r = check_ws(s, ws, ws_bytes)) != SAGA_OK) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Plan pl = saga_plan(s);
  StepParams p = base_params(s, pl, q, K, V, l_kv, ws);
  float *rows = scores != nullptr
                    ? scores
                    : reinterpret_cast<float *>(static_cast<char *>(ws) + pl.off_scores);
  // 1. score rows (tensor-core kernel: with the top-byte histogram of every row)
  SelectBufs sb;
  if (use_tc(s)) {
    const cudaError_t me = clear_select_counts(s, pl, ws, &sb, st);
    if (me != cudaSuccess) return cuda_fail(me, "cudaMemsetAsync (histograms)");
  }
  uint32_t *hist = sb.hist;
  p.scores_out = rows;
  p.hist = hist;
  cudaError_t e = launch_split(s, p, kModeDump, st);
  if (e != cudaSuccess) return cuda_fail(e, "score dump kernel");
  // 2. exact N-th largest per row
  e = launch_radix_select(rows, s.max_l_kv, l_kv, N, tau, s.B, s.h_q, s.cap, s.max_l_kv, hist,
                          nullptr, sb.gcand, sb.gcount, sb.hist1, pl.gcap, static_cast<int>(kSms),
                          st);
  if (e != cudaSuccess) return cuda_fail(e, "radix select kernel");
  if (V == nullptr) return SAGA_OK;
  // 3. this step's select + PV with the fresh tau, over the very rows tau
  // came from: streamed back from memory (K is not read again), or, on the
  // tensor-core path when the rows cannot be streamed (a caller's buffer
  // with an odd stride), recomputed from K with the same MMAs, which gives
  // the same scores bit for bit.
  p.scores_out = nullptr;
  p.hist = nullptr;
  p.tau = tau;
  p.sel_mask = sel_mask;
  if (use_tc(s)) {
    if (saga_tc_scores_streamable(rows, s.max_l_kv)) p.scores_in = rows;
    return run_step(s, pl, p, kModeStep, out, sel_count, st);
  }
  p.scores_in = rows;
  return run_step(s, pl, p, kModeFromScores, out, sel_count, st);
}

saga_status saga_topn_step(const saga_shape *shape, const void *q, const void *K,
                           const void *V, const int32_t *l_kv, int32_t N, float *out,
                           int32_t *sel_count, uint8_t *sel_mask, float *scores, void *ws,
                           size_t ws_bytes, saga_stream_t stream) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  const saga_shape &s = *shape;
  if ((r = check_inputs(s, q, K, l_kv)) != SAGA_OK) return r;
  if (N < 1 || V == nullptr || out == nullptr || !aligned(V, 16) || !aligned(out, 16))
    return SAGA_ERR_INVALID_ARG;
  if ((scores && !aligned(scores, 4)) || (sel_count && !aligned(sel_count, 4)))
    return SAGA_ERR_INVALID_ARG;
  if ((r = check_ws(s, ws, ws_bytes)) != SAGA_OK) return r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const Plan pl = saga_plan(s);
  StepParams p = base_params(s, pl, q, K, V, l_kv, ws);
  char *wsb = static_cast<char *>(ws);
  float *rows = scores != nullptr ? scores : reinterpret_cast<float *>(wsb + pl.off_scores);
  float *tau = reinterpret_cast<float *>(wsb + pl.off_tau);
  int32_t *tie = reinterpret_cast<int32_t *>(wsb + pl.off_tie);
  // 1. score rows (tensor-core kernel: with the top-byte histogram of every row)
  SelectBufs sb;
  if (use_tc(s)) {
    const cudaError_t me = clear_select_counts(s, pl, ws, &sb, st);
    if (me != cudaSuccess) return cuda_fail(me, "cudaMemsetAsync (histograms)");
  }
  uint32_t *hist = sb.hist;
  p.scores_out = rows;
  p.hist = hist;
  cudaError_t e = launch_split(s, p, kModeDump, st);
  if (e != cudaSuccess) return cuda_fail(e, "score dump kernel");
  // 2. the N-th largest and, when it is tied, the last tied position taken
  e = launch_radix_select(rows, s.max_l_kv, l_kv, N, tau, s.B, s.h_q, s.cap, s.max_l_kv, hist,
                          tie, sb.gcand, sb.gcount, sb.hist1, pl.gcap, static_cast<int>(kSms),
                          st);
  if (e != cudaSuccess) return cuda_fail(e, "radix select kernel");
  // 3. the step over exactly those positions, from the stored rows (or, on
  // the tensor-core path when they cannot be streamed, from bit-identical
  // scores recomputed from K)
  p.scores_out = nullptr;
  p.hist = nullptr;
  p.tau = tau;
  p.tie = tie;
  p.sel_mask = sel_mask;
  if (use_tc(s)) {
    if (saga_tc_scores_streamable(rows, s.max_l_kv)) p.scores_in = rows;
    return run_step(s, pl, p, kModeStepTies, out, sel_count, st);
  }
  p.scores_in = rows;
  return run_step(s, pl, p, kModeFromScores, out, sel_count, st);
}

saga_status gqa_dense_decode(const saga_shape *shape, const void *q, const void *K,
                             const void *V, const int32_t *l_kv, float *out, void *ws,
                             size_t ws_bytes, saga_stream_t stream) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  if (shape->h_k != shape->h_v) return SAGA_ERR_INVALID_ARG;
  return run_dense(*shape, q, K, V, l_kv, out, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

saga_status saga_dense_decode(const saga_shape *shape, const void *q, const void *K,
                              const void *V, const int32_t *l_kv, float *out, void *ws,
                              size_t ws_bytes, saga_stream_t stream) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  return run_dense(*shape, q, K, V, l_kv, out, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

saga_status saga_append_kv(const saga_shape *shape, const void *k_new, const void *v_new,
                           void *K, void *V, int32_t *l_kv, void *ws, size_t ws_bytes,
                           saga_stream_t stream) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  const saga_shape &s = *shape;
  if (k_new == nullptr || v_new == nullptr || K == nullptr || V == nullptr || l_kv == nullptr)
    return SAGA_ERR_INVALID_ARG;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(K, 16) || !aligned(V, 16) ||
      !aligned(l_kv, 4))
    return SAGA_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, kAlign) || ws_bytes < kAlign) return SAGA_ERR_WORKSPACE;
  const int esz = s.dtype == SAGA_F32 ? 4 : 2;
  return cuda_check(launch_append(k_new, v_new, K, V, l_kv, static_cast<int32_t *>(ws), s.B, s.h_k,
                                   s.h_v, s.d, esz, s.k_stride_b, s.k_stride_h, s.v_stride_b,
                                   s.v_stride_h, s.cap, reinterpret_cast<cudaStream_t>(stream)),
                    "append kernel");
}

saga_status saga_debug_scores(const saga_shape *shape, const void *q, const void *K,
                              const int32_t *l_kv, float *scores, void *ws, size_t ws_bytes,
                              saga_stream_t stream) {
  saga_status r = check_shape(shape);
  if (r != SAGA_OK) return r;
  const saga_shape &s = *shape;
  if ((r = check_inputs(s, q, K, l_kv)) != SAGA_OK) return r;
  if (scores == nullptr || !aligned(scores, 4)) return SAGA_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned(ws, kAlign) || ws_bytes < kAlign) return SAGA_ERR_WORKSPACE;
  const Plan pl = saga_plan(s);
  StepParams p = base_params(s, pl, q, K, nullptr, l_kv, ws);
  p.partials = nullptr;
  p.scores_out = scores;
  return cuda_check(launch_split(s, p, kModeDump, reinterpret_cast<cudaStream_t>(stream)),
                    "score dump kernel");
}

saga_status saga_read_device_error(void *ws, saga_stream_t stream, int32_t *flags) {
  if (ws == nullptr || !aligned(ws, kAlign) || flags == nullptr) return SAGA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync (error word)");
  if ((e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st)) != cudaSuccess)
    return cuda_fail(e, "cudaMemsetAsync (error word)");
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  *flags = h;
  return h != 0 ? SAGA_ERR_DEVICE : SAGA_OK;
}

const char *saga_last_error(void) { return g_last_error; }

const char *saga_status_string(saga_status status) {
  switch (status) {
    case SAGA_OK: return "ok";
    case SAGA_ERR_INVALID_ARG: return "invalid argument";
    case SAGA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case SAGA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SAGA_ERR_CUDA: return "CUDA runtime or launch failure";
    case SAGA_ERR_DEVICE: return "device error word set (out-of-contract input)";
  }
  return "unknown status";
}

}  // extern "C"
