// C-ABI entry points: argument checks, workspace layout, TMA descriptors,
// work partitioning and the launch sequence of a decode step.
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include <float.h>

#include <chrono>
#include <thread>

#include "../../include/dllm.h"
#include "kernels.cuh"

namespace dllm {
unsigned long long launch_count();
void add_launches(long long n);
}

using namespace dllm;

namespace {

// ------------------------------------------------------------------ helpers
size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int cdiv(int a, int b) { return (a + b - 1) / b; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D bf16 tensor map: dims {d0 (innermost), d1, d2}, box {b0, b1, 1}.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
              uint32_t b1, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn || !ptr) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ shapes
struct Shape {
  int b, L, d, Hq, Hkv, D, V, P, G, B, S, W, mode, wfmt, commit_mode, spb;
  int qkv_rows, Kw, Ko;
  float tau, theta, exit_tau;
  int mask_id;
};

dllm_status check_cfg(const dllm_config* c, Shape* s) {
  if (!c) return DLLM_ERR_INVALID;
  if (c->batch < 1 || c->n_layers < 1 || c->hidden < 1 || c->n_q_heads < 1 ||
      c->n_kv_heads < 1 || c->head_dim < 1 || c->vocab < 2 || c->prompt_len < 0 ||
      c->gen_len < 1 || c->block < 1)
    return DLLM_ERR_INVALID;
  if (c->mode < DLLM_CACHE_NONE || c->mode > DLLM_CACHE_PREFIX_SUFFIXQ) return DLLM_ERR_INVALID;
  if (c->weight_format != DLLM_W_BF16 && c->weight_format != DLLM_W_F32_SPLIT)
    return DLLM_ERR_INVALID;
  if (c->n_q_heads % c->n_kv_heads) return DLLM_ERR_INVALID;
  if (c->gen_len % c->block) return DLLM_ERR_INVALID;
  if (c->mode == DLLM_CACHE_DUAL_PRUNED && c->window < 0) return DLLM_ERR_INVALID;
  if (c->mask_id < 0 || c->mask_id >= c->vocab) return DLLM_ERR_INVALID;
  if (c->commit_mode != DLLM_COMMIT_THRESHOLD && c->commit_mode != DLLM_COMMIT_TOPK &&
      c->commit_mode != DLLM_COMMIT_EARLY_EXIT)
    return DLLM_ERR_INVALID;
  if (c->commit_mode == DLLM_COMMIT_EARLY_EXIT &&
      !(c->exit_tau >= 0.f && c->exit_tau <= FLT_MAX))  // NaN, inf, negative
    return DLLM_ERR_INVALID;
  if (c->commit_mode == DLLM_COMMIT_TOPK &&
      (c->steps_per_block < 1 || c->steps_per_block > c->block))
    return DLLM_ERR_INVALID;
  if (!(c->tau == c->tau)) return DLLM_ERR_INVALID;
  if (!(c->rope_theta >= 0.f && c->rope_theta <= FLT_MAX)) return DLLM_ERR_INVALID;  // NaN, inf
  // Positions are int32 on the device, and cache and query rows are addressed
  // with 32-bit offsets in units of head_dim.
  const long long seq = (long long)c->prompt_len + c->gen_len;
  if (seq > (1ll << 24)) return DLLM_ERR_UNSUPPORTED;
  if ((long long)c->n_layers * c->batch * c->n_kv_heads * seq >= (1ll << 31) ||
      (long long)c->batch * seq * c->n_q_heads >= (1ll << 31))
    return DLLM_ERR_UNSUPPORTED;
  if (c->head_dim != 32 && c->head_dim != 128) return DLLM_ERR_UNSUPPORTED;
  const int qkv = (c->n_q_heads + 2 * c->n_kv_heads) * c->head_dim;
  if (c->hidden % 128 || (c->n_q_heads * c->head_dim) % 128 || qkv % 128 || c->vocab % 128)
    return DLLM_ERR_UNSUPPORTED;
  if (c->block > 64 || c->batch > 1024) return DLLM_ERR_UNSUPPORTED;
  s->b = c->batch;
  s->L = c->n_layers;
  s->d = c->hidden;
  s->Hq = c->n_q_heads;
  s->Hkv = c->n_kv_heads;
  s->D = c->head_dim;
  s->V = c->vocab;
  s->P = c->prompt_len;
  s->G = c->gen_len;
  s->B = c->block;
  s->S = c->prompt_len + c->gen_len;
  s->W = c->window;
  s->mode = c->mode;
  s->wfmt = c->weight_format;
  s->commit_mode = c->commit_mode;
  s->spb = c->steps_per_block > 0 ? c->steps_per_block : 0;
  s->qkv_rows = qkv;
  const int f = c->weight_format == DLLM_W_F32_SPLIT ? 2 : 1;
  s->Kw = f * c->hidden;
  s->Ko = f * c->n_q_heads * c->head_dim;
  s->tau = c->tau;
  s->theta = c->rope_theta;
  s->exit_tau = c->exit_tau;
  s->mask_id = c->mask_id;
  return DLLM_OK;
}

// ------------------------------------------------------------------ partitioning
struct GemmPlan {
  int nt, m_tiles, n_tiles, splits, kbps, units, grid;
};

// Split K only for decode tiles (NT <= 64): the splits of a tile run as one
// cluster (at most 4 CTAs for NT 32, 3 for NT 64) whose ranks exchange their
// fp32 partials through distributed shared memory.  The cost model counts
// k-blocks per CTA, one per unit, and one for a split's reduction.
GemmPlan plan_gemm(int M, int R, int K, bool allow_split) {
  GemmPlan g;
  g.nt = R <= 32 ? 32 : R <= 64 ? 64 : R <= 128 ? 128 : 256;
  g.n_tiles = cdiv(R, g.nt);
  g.m_tiles = M / 128;
  const int tiles = g.m_tiles * g.n_tiles;
  const int kbt = K / 64;
  int best_s = 1, best_kbps = kbt;
  double best_cost = 1e30;
  const int cluster_max = g.nt == 32 ? 4 : g.nt == 64 ? 3 : 1;
  const int max_s = allow_split ? std::min(cluster_max, kbt) : 1;
  for (int s = 1; s <= max_s; ++s) {
    const int kbps = cdiv(kbt, s);
    const int se = cdiv(kbt, kbps);
    if (se != s) continue;
    const int units = tiles * se;
    const int per_cta = cdiv(units, kNumSMs);
    const double cost = (double)per_cta * kbps + 1.0 * per_cta + (se > 1 ? 1.0 : 0.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best_s = se;
      best_kbps = kbps;
    }
  }
  g.splits = best_s;
  g.kbps = best_kbps;
  g.units = tiles * best_s;
  // split tiles: one unit per CTA (clusters); otherwise persistent CTAs
  g.grid = best_s > 1 ? g.units : std::min(g.units, kNumSMs);
  return g;
}

// The same GEMM with K split into exactly sp parts (one unit per CTA).
GemmPlan plan_gemm_splits(int M, int R, int K, int sp) {
  GemmPlan g = plan_gemm(M, R, K, false);
  const int kbt = K / 64;
  g.kbps = cdiv(kbt, sp);
  g.splits = cdiv(kbt, g.kbps);
  g.units = g.m_tiles * g.n_tiles * g.splits;
  g.grid = g.splits > 1 ? g.units : std::min(g.units, kNumSMs);
  return g;
}

// The LM head streams whole vocabulary tiles on persistent CTAs.  Its grid
// is the fewest CTAs (at most one per SM, a multiple of the row tiles) that
// keep the tiles per CTA at their minimum, so no last round runs on a few
// SMs alone: 1188 tiles take 132 CTAs x 9 rather than 148 CTAs with 4 of
// them streaming a ninth tile after the others are done.
GemmPlan plan_lmhead(int V, int R, int K) {
  GemmPlan g = plan_gemm(V, R, K, false);
  const int rounds = cdiv(g.units, kNumSMs);
  int grid = cdiv(cdiv(g.units, rounds), g.n_tiles) * g.n_tiles;
  if (grid > kNumSMs) grid = kNumSMs / g.n_tiles * g.n_tiles;
  g.grid = std::max(g.n_tiles, grid);
  return g;
}

// Extra plan cost (in key tiles) that 32-row attention tiles may have over
// 128-row tiles and still be chosen for groups of more than 32 rows.
constexpr int kAttnSgSlack = 1;
// SMs a key-chunk plan counts as one wave.  Fewer than the 148 SMs: the
// O-projection that follows starts its CTAs on the SMs that attention leaves
// free and streams its weights before its dependency wait.  Measured on the
// Dream-7B-shaped first block: 7 x 4 row tiles x 5 chunks (140 CTAs) 1171 us
// per step, x 3 chunks of 2 tiles (84 CTAs) 1026 us.
constexpr int kAttnSMs = 128;

struct AttnPlan {
  int row_tiles, chunks, tpc;
  bool sg;  // row tiles of 32 rows (the attention kernel's small-group mode)
};

// Key chunks per row tile for `base` row tiles: the chunks form one cluster
// and merge on chip.  At most 8 for head_dim 128 and 6 for head_dim 32 (the
// merge buffer must fit in the K/V/P region).  Seven head_dim-128 chunks would
// not fit either, so they run as eight, the last one without keys.
// While the row tiles alone leave SMs idle, the chunk count minimises
// waves x key tiles per chunk (one CTA per SM: the K/V ring and P take most
// of the shared memory), counting each merge as one more tile, so a second
// wave of CTAs costs as much as the first.  Once the row tiles fill the SMs,
// splitting the keys only adds merges (measured +15 % on a 16-sequence batch).
AttnPlan plan_chunks(const Shape& s, int base, int ntile_bound, long long* cost_out) {
  AttnPlan a{};
  const int cap = base >= kNumSMs ? 1 : s.D == 128 ? 8 : 6;
  int chunks = 1;
  long long best = 1ll << 62;
  for (int c = 1; c <= std::min(ntile_bound, cap); ++c) {
    const long long waves = cdiv((long long)base * c, kAttnSMs);
    const long long cost = waves * cdiv(ntile_bound, c) + (c > 1 ? 1 : 0);
    if (cost < best) {
      best = cost;
      chunks = c;
    }
  }
  a.tpc = cdiv(ntile_bound, chunks);
  a.chunks = cdiv(ntile_bound, a.tpc);
  if (a.chunks == 7) a.chunks = 8;
  *cost_out = best;
  return a;
}

AttnPlan plan_attn(const Shape& s, int n_rows, int ntile_bound) {
  const int g = s.Hq / s.Hkv;
  const int gr = g * n_rows;
  long long cost128 = 0, cost32 = 0;
  AttnPlan a = plan_chunks(s, s.b * s.Hkv * cdiv(gr, 128), ntile_bound, &cost128);
  a.row_tiles = cdiv(gr, 128);
  a.sg = false;
  if (s.D != 128) return a;
  // Row tiles of 32 rows, each loaded four times so that every warp takes a
  // quarter of the keys and of the output columns: always for groups of at
  // most 32 rows (same grid, a quarter of the softmax per thread); for larger
  // groups while their plan costs at most one tile more than 128-row tiles
  // (its tiles and merges are the cheaper ones).
  const int rt32 = cdiv(gr, 32);
  const AttnPlan b = plan_chunks(s, s.b * s.Hkv * rt32, ntile_bound, &cost32);
  if (gr <= 32 || cost32 <= cost128 + kAttnSgSlack) {
    a = b;
    a.row_tiles = rt32;
    a.sg = true;
  }
  return a;
}

constexpr int kKeyTile = 128;  // keys per attention tile

// Upper bound of key tiles of a sequence for a block at blk (first valid
// position 0), or for a plain range [0, seg_end) when seg_end > 0.
int key_tiles_bound(const Shape& s, int blk, int seg_end) {
  if (seg_end > 0) return cdiv(seg_end, kKeyTile);
  const int end = blk + s.B;
  switch (s.mode) {
    case DLLM_CACHE_DUAL:
    case DLLM_CACHE_PREFIX_SUFFIXQ: return cdiv(s.S, kKeyTile);
    case DLLM_CACHE_DUAL_PRUNED: {
      const int wend = std::min(end + s.W, s.S);
      return cdiv(wend, kKeyTile) + ((end < s.S && s.S - 1 >= wend) ? 1 : 0);
    }
    default: return cdiv(end, kKeyTile);
  }
}

// ------------------------------------------------------------------ layer stack
// Plan of the persistent layer-stack kernel (csrc/stack.cu) for a step or a
// refresh of n_rows rows per sequence at block blk.  Shape conditions only;
// whether the kernel is used at run time also depends on the device and on
// dllm_set_layer_stack.
struct StackPlan {
  bool ok = false;
  int nt = 0, grid = 0, qt = 0, ot = 0, qkbt = 0, okbt = 0, qn = 0, on = 0, qmaxc = 0, omaxc = 0;
  int rt = 0, chunks = 0, tpc = 0, units = 0, fs = 0;
};
constexpr int kStackMinSeg = 2;  // k-blocks a CTA's share holds at least

// 64-key attention tiles of the widest sequence (sequence start 0).
int stack_key_tiles(const Shape& s, int blk) {
  const int end = blk + s.B;
  if (s.mode == DLLM_CACHE_DUAL) return cdiv(s.S, 64);
  if (s.mode == DLLM_CACHE_DUAL_PRUNED) {
    const int wend = std::min(end + s.W, s.S);
    return cdiv(wend, 64) + ((end < s.S && s.S - 1 >= wend) ? 1 : 0);
  }
  return cdiv(end, 64);
}

// Largest number of contributors (CTA shares) of one tile.
int stack_maxc(int tiles, int kbt, int n) {
  const long long T = (long long)tiles * kbt;
  int mx = 0;
  for (int t = 0; t < tiles; ++t) {
    const int ca = stack_owner((long long)t * kbt, n, T);
    const int cb = stack_owner((long long)t * kbt + kbt - 1, n, T);
    mx = std::max(mx, cb - ca + 1);
  }
  return mx;
}

StackPlan plan_stack(const Shape& s, int n_rows, int blk, int grid) {
  StackPlan P;
  if (grid < 1 || s.D != 128 || s.wfmt != DLLM_W_BF16) return P;
  if (s.mode != DLLM_CACHE_PREFIX && s.mode != DLLM_CACHE_DUAL && s.mode != DLLM_CACHE_DUAL_PRUNED)
    return P;
  const int R = s.b * n_rows;
  if (R < 1 || R > 64) return P;
  P.nt = R <= 32 ? 32 : 64;
  P.grid = grid;
  P.qt = s.qkv_rows / 128;
  P.ot = s.d / 128;
  P.qkbt = s.Kw / 64;
  P.okbt = s.Ko / 64;
  P.qn = std::min(grid, std::max(1, P.qt * P.qkbt / kStackMinSeg));
  P.on = std::min(grid, std::max(1, P.ot * P.okbt / kStackMinSeg));
  StackSeg tmp[kStackMaxSeg];
  for (int c = 0; c < P.qn; ++c)
    if (stack_segments(c, P.qt, P.qkbt, P.qn, tmp, kStackMaxSeg) < 0) return P;
  for (int c = 0; c < P.on; ++c)
    if (stack_segments(c, P.ot, P.okbt, P.on, tmp, kStackMaxSeg) < 0) return P;
  P.qmaxc = stack_maxc(P.qt, P.qkbt, P.qn);
  P.omaxc = stack_maxc(P.ot, P.okbt, P.on);
  const int g = s.Hq / s.Hkv;
  P.rt = cdiv(g * n_rows, 128);
  // key chunks of a row tile: a power of two (each finishes D/chunks columns
  // of the merge) that keeps at most two 64-key tiles per chunk, fewer when
  // the units would outnumber the CTAs (one unit per CTA and layer)
  const int nt64 = stack_key_tiles(s, blk);
  int chunks = 1;
  while (chunks < 16 && cdiv(nt64, chunks) > 2) chunks *= 2;
  while (chunks > 1 && s.b * s.Hkv * P.rt * chunks > grid) chunks /= 2;
  P.chunks = chunks;
  P.tpc = cdiv(nt64, chunks);
  P.units = s.b * s.Hkv * P.rt * chunks;
  if (P.units > grid) return P;
  // counters of one layer, each on its own 128-byte line (32 ints)
  P.fs = 32 * (2 * P.qt + 2 * P.ot + s.b * s.Hkv * P.rt + s.Hkv);
  P.ok = true;
  return P;
}

// ------------------------------------------------------------------ workspace
struct Layout {
  size_t status, stepc, seqblk, seqdone, exitst, x, xb, sumsq, q, attn, h, stats, conf, tok, gap, commit,
      remaining, blkdone, refresh, segs, rope, total;
  int rmax, lm_slots;
  // layer-stack kernel: flags, split-K partials, attention chunk partials
  size_t stk_flags, stk_qpart, stk_opart, stk_apart, stk_aml;
  long long stk_nflags;  // ints of flags reserved (0: the shape never uses the kernel)
  int stk_chunks;        // key chunks the attention partials are sized for
};

// Row counts (per sequence) a configuration uses: decode steps and prefill.
std::vector<int> row_counts(const Shape& s) {
  std::vector<int> r;
  if (s.mode == DLLM_CACHE_NONE) {
    for (int blk = s.P; blk < s.S; blk += s.B) r.push_back(blk + s.B);
  } else if (s.mode == DLLM_CACHE_PREFIX_SUFFIXQ) {
    r.push_back(s.G);  // the first block's step: block and whole suffix
    r.push_back(std::max(s.P, 1));
  } else {
    r.push_back(s.B);
    r.push_back(s.mode == DLLM_CACHE_PREFIX ? std::max(s.P, 1) : s.S);
  }
  return r;
}

Layout compute_layout(const Shape& s);

// The workspace layout of a shape, computed once and then looked up: every
// entry point needs it, and planning the layer-stack partition for every block
// costs more host time than a projection kernel takes on the GPU.
Layout layout(const Shape& s) {
  static std::mutex mu;
  static std::vector<std::pair<Shape, Layout>> memo;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& e : memo)
    if (memcmp(&e.first, &s, sizeof(Shape)) == 0) return e.second;
  const Layout l = compute_layout(s);
  if (memo.size() >= 64) memo.erase(memo.begin());
  memo.emplace_back(s, l);
  return l;
}

Layout compute_layout(const Shape& s) {
  Layout l{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const std::vector<int> rows = row_counts(s);
  int max_rows = 0;
  for (int n : rows) max_rows = std::max(max_rows, n);
  l.rmax = s.b * max_rows;
  const GemmPlan gl = plan_lmhead(s.V, s.b * s.B, s.Kw);
  l.lm_slots = gl.grid / gl.n_tiles;
  l.status = take(256);
  l.stepc = take((size_t)s.b * 2 * 4);  // per sequence: steps in the block, block start
  l.seqblk = take((size_t)s.b * 4);     // per sequence: current block (dllm_decode_all)
  l.seqdone = take((size_t)s.b * 4);    // per sequence: every block done
  // early exit: per sequence the block start + 1 of the previous step (0:
  // none), then every row's argmax at that step; zeroed with the counters
  l.exitst = take((size_t)s.b * (1 + s.B) * 4);
  l.x = take((size_t)l.rmax * s.d * 4);
  l.xb = take((size_t)l.rmax * s.d * 2);
  l.sumsq = take((size_t)l.rmax * (s.d / 128) * 4);
  l.q = take((size_t)l.rmax * s.Hq * s.D * 2);
  l.attn = take((size_t)l.rmax * s.Hq * s.D * 2);
  l.h = take((size_t)s.b * s.B * s.d * 2);
  l.stats = take((size_t)s.b * s.B * l.lm_slots * sizeof(LmStat));
  l.conf = take((size_t)s.b * s.B * 4);
  l.tok = take((size_t)s.b * s.B * 4);
  l.gap = take((size_t)s.b * s.B * 4);
  l.commit = take((size_t)s.b * s.B);
  l.remaining = take((size_t)s.b * 4);
  l.blkdone = take((size_t)s.b * 4);
  l.refresh = take((size_t)s.b * 4);
  l.segs = take((size_t)s.b * 16);
  l.rope = take(s.theta > 0.f ? (size_t)s.S * (s.D / 2) * 8 : 256);
  // the layer-stack kernel runs steps and refreshes of b*B rows; its scratch
  // is sized for the widest key set over the blocks
  StackPlan sp{};
  for (int blk = s.P; blk < s.S; blk += s.B) {
    const StackPlan q = plan_stack(s, s.B, blk, kNumSMs);
    if (q.ok && (!sp.ok || q.chunks > sp.chunks)) sp = q;
  }
  if (sp.ok) {
    l.stk_nflags = (long long)s.L * sp.fs + 32;  // then the abort word
    l.stk_chunks = sp.chunks;
    l.stk_flags = take((size_t)l.stk_nflags * 4);
    l.stk_qpart = take((size_t)sp.qt * sp.qmaxc * sp.nt * 128 * 4);
    l.stk_opart = take((size_t)sp.ot * sp.omaxc * sp.nt * 128 * 4);
    const size_t slots = (size_t)s.b * s.Hkv * sp.rt * sp.chunks;
    l.stk_apart = take(slots * 128 * 128 * 4);
    l.stk_aml = take(slots * 128 * 8);
  }
  l.total = off;
  return l;
}

// ------------------------------------------------------------------ context
struct Ctx {
  Shape s{};
  Layout l{};
  uint8_t* ws = nullptr;  // null for entry points that take no workspace
  cudaStream_t st = nullptr;
  // per-sequence block starts in the workspace (dllm_decode_all), or null:
  // every sequence is at the block the call names
  int* seq_blk = nullptr;
  template <class T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
};

// Process-wide switches of the layer-stack kernel (dllm_set_layer_stack).
struct StackTune {
  bool enable = false;  // measured slower than the per-projection kernels (see the header)
  int lookahead = 16;   // weight k-blocks prefetched into L2 beyond the ring
};
StackTune g_stack_tune;
bool g_stack_dev_ok[64] = {};

// One-time per-device setup that must not run inside a graph capture:
// kernel shared-memory attributes and the tensor-map encoder entry point.
dllm_status prepare_device() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DLLM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return DLLM_OK;
  if (!encode_fn() || gemm_prepare() != cudaSuccess || attn_prepare() != cudaSuccess ||
      stack_prepare() != cudaSuccess)
    return DLLM_ERR_CUDA;
  // The layer-stack kernel's CTAs wait on one another, so all of them must be
  // resident at once: one CTA on each of kNumSMs SMs.
  int sms = 0, per_sm32 = 0, per_sm64 = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      stack_occupancy(32, &per_sm32) != cudaSuccess || stack_occupancy(64, &per_sm64) != cudaSuccess)
    return DLLM_ERR_CUDA;
  g_stack_dev_ok[dev] = sms >= kNumSMs && per_sm32 >= 1 && per_sm64 >= 1;
  done[dev] = true;
  return DLLM_OK;
}

// The layer-stack kernel runs on the current device (prepared above) and is
// switched on (dllm_set_layer_stack).
bool stack_usable() {
  int dev = 0;
  if (!g_stack_tune.enable || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return false;
  return g_stack_dev_ok[dev];
}

dllm_status make_ctx(const dllm_config* cfg, void* ws, size_t ws_bytes, dllm_stream stream,
                     Ctx* c) {
  dllm_status e = check_cfg(cfg, &c->s);
  if (e != DLLM_OK) return e;
  if (!ws) return DLLM_ERR_INVALID;
  c->l = layout(c->s);
  if (ws_bytes < c->l.total) return DLLM_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % 256) return DLLM_ERR_INVALID;
  c->ws = static_cast<uint8_t*>(ws);
  c->st = reinterpret_cast<cudaStream_t>(stream);
  return DLLM_OK;  // validation only: nothing here touches the device
}

dllm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA; }

#define DLLM_TRY(x)                       \
  do {                                    \
    dllm_status _e = (x);                 \
    if (_e != DLLM_OK) return _e;         \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// NVTX range over an entry point (free when no profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// Wait for the work queued on st so far, giving up after deadline_s: the
// kernels bound their own waits, this bounds the host side as well.
dllm_status wait_stream(cudaStream_t st, double deadline_s) {
  thread_local cudaEvent_t ev = nullptr;
  if (!ev && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess)
    return DLLM_ERR_CUDA;
  if (cudaEventRecord(ev, st) != cudaSuccess) return DLLM_ERR_CUDA;
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    const cudaError_t q = cudaEventQuery(ev);
    if (q == cudaSuccess) return DLLM_OK;
    if (q != cudaErrorNotReady) return DLLM_ERR_CUDA;
    const double el = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
    if (el > deadline_s) return DLLM_ERR_TIMEOUT;
    if (el > 2e-3) std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}
constexpr double kHostDeadlineS = 60.0;

// ------------------------------------------------------------------ launches
// Q/K/V projection plan for R activation rows.  More split CTAs than SMs
// start partly late (beside the O-projection still running); two splits on a
// deeper ring measured faster than three.
GemmPlan plan_qkv(const Shape& s, int R, int* epi) {
  GemmPlan g = plan_gemm(s.qkv_rows, R, s.Kw, true);
  *epi = EPI_QKV;
  if (g.nt <= 64 && g.splits > 2 && g.grid > kNumSMs) {
    g = plan_gemm_splits(s.qkv_rows, R, s.Kw, 2);
    *epi = EPI_QKV_DEEP;
  }
  return g;
}

dllm_status run_qkv(const Ctx& c, const void* wqkv, int layer, const void* xb,
                    const float* sumsq, int row0, int n_rows, const int* seq_start, void* q_out,
                    void* kc, void* vc, bool pdl, const L2Prefetch& pf = L2Prefetch{}) {
  const Shape& s = c.s;
  const int R = s.b * n_rows;
  int epi;
  const GemmPlan g = plan_qkv(s, R, &epi);
  CUtensorMap wm, xm;
  if (!make_map(&wm, wqkv, s.Kw, s.qkv_rows, s.L, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&xm, xb, s.d, R, 1, 64, g.nt, CU_TENSOR_MAP_SWIZZLE_128B))
    return DLLM_ERR_CUDA;
  GemmParams p{};
  p.M = s.qkv_rows;
  p.R = R;
  p.K = s.Kw;
  p.kx_blocks = s.d / 64;
  p.m_tiles = g.m_tiles;
  p.n_tiles = g.n_tiles;
  p.splits = g.splits;
  p.kb_per_split = g.kbps;
  p.units = g.units;
  p.layer = layer;
  p.seq_blk = c.seq_blk;
  p.status = c.at<int>(c.l.status);
  p.n_rows = n_rows;
  p.row0 = row0;
  p.seq_start = seq_start;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.D = s.D;
  p.S = s.S;
  p.batch = s.b;
  p.rope_tab = s.theta > 0.f ? c.at<float2>(c.l.rope) : nullptr;
  p.sumsq_in = sumsq;
  p.npart = s.d / 128;
  p.d_norm = s.d;
  p.rms_eps = kRmsEps;
  p.q_out = static_cast<__nv_bfloat16*>(q_out);
  p.k_cache = static_cast<__nv_bfloat16*>(kc);
  p.v_cache = static_cast<__nv_bfloat16*>(vc);
  p.pf = pf;
  p.recv_in_ring = g.grid > kNumSMs;
  return cuda_status(launch_gemm(epi, g.nt, wm, xm, p, g.grid, pdl, c.st));
}

dllm_status run_oproj(const Ctx& c, const void* wo, int layer, const void* attn, int row0,
                      int n_rows, float* x, void* xb, float* sumsq, bool pdl,
                      const L2Prefetch& pf = L2Prefetch{}) {
  const Shape& s = c.s;
  const int R = s.b * n_rows;
  const GemmPlan g = plan_gemm(s.d, R, s.Ko, true);
  CUtensorMap wm, xm;
  if (!make_map(&wm, wo, s.Ko, s.d, s.L, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&xm, attn, s.Hq * s.D, R, 1, 64, g.nt, CU_TENSOR_MAP_SWIZZLE_128B))
    return DLLM_ERR_CUDA;
  GemmParams p{};
  p.M = s.d;
  p.R = R;
  p.K = s.Ko;
  p.kx_blocks = s.Hq * s.D / 64;
  p.m_tiles = g.m_tiles;
  p.n_tiles = g.n_tiles;
  p.splits = g.splits;
  p.kb_per_split = g.kbps;
  p.units = g.units;
  p.layer = layer;
  p.status = c.at<int>(c.l.status);
  p.n_rows = n_rows;
  p.row0 = row0;
  p.x = x;
  p.xb = static_cast<__nv_bfloat16*>(xb);
  p.d_model = s.d;
  p.sumsq_out = sumsq;
  p.npart = s.d / 128;
  p.d_norm = s.d;
  p.pf = pf;
  p.recv_in_ring = g.grid > kNumSMs;
  return cuda_status(launch_gemm(EPI_OPROJ, g.nt, wm, xm, p, g.grid, pdl, c.st));
}

struct AttnKeys {
  const int* segs;  // explicit segments, or null to derive them in the kernel
  const int* seq_start;
  int blk_start, seg_end, dep_lo, dep_hi;
};

dllm_status run_attn(const Ctx& c, int layer, int n_rows, const void* q, const void* kc,
                     const void* vc, const AttnKeys& keys, void* out, int ntile_bound,
                     bool pdl, const L2Prefetch& pf = L2Prefetch{}) {
  const Shape& s = c.s;
  const int g = s.Hq / s.Hkv;
  const AttnPlan a = plan_attn(s, n_rows, ntile_bound);
  const int box_d = s.D >= 64 ? 64 : s.D;
  const CUtensorMapSwizzle sw = s.D >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap qm, km, vm;
  const uint32_t q_box = a.sg ? 32 : 128;
  if (!make_map(&qm, q, s.D, (uint64_t)g * n_rows, (uint64_t)s.b * s.Hkv, box_d, q_box, sw) ||
      !make_map(&km, kc, s.D, s.S, (uint64_t)s.L * s.b * s.Hkv, box_d, kKeyTile, sw) ||
      !make_map(&vm, vc, s.D, s.S, (uint64_t)s.L * s.b * s.Hkv, box_d, kKeyTile, sw))
    return DLLM_ERR_CUDA;
  AttnParams p{};
  p.batch = s.b;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.D = s.D;
  p.S = s.S;
  p.layer = layer;
  p.n_rows = n_rows;
  p.group_rows = g * n_rows;
  p.row_tiles = a.row_tiles;
  p.small_group = a.sg ? 1 : 0;
  p.chunks = a.chunks;
  p.tiles_per_chunk = a.tpc;
  p.segs = keys.segs;
  p.mode = s.mode;
  p.blk_start = keys.blk_start;
  p.blk_len = s.B;
  p.window = s.W;
  p.seg_end = keys.seg_end;
  p.seq_start = keys.seq_start;
  p.dep_lo = keys.dep_lo;
  p.dep_hi = keys.dep_hi;
  p.seq_blk = c.seq_blk;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = c.at<int>(c.l.status);
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)s.D);
  p.pf = pf;
  return cuda_status(launch_attn(s.D, qm, km, vm, p, pdl, c.st));
}

dllm_status run_embed(const Ctx& c, const dllm_weights* w, const dllm_state* stt, int row0,
                      int n_rows, int blk_start, int seg_end, bool pdl, int* zero = nullptr,
                      long long nzero = 0) {
  const Shape& s = c.s;
  EmbedParams e{};
  e.batch = s.b;
  e.S = s.S;
  e.d = s.d;
  e.n_rows = n_rows;
  e.row0 = row0;
  e.blk_start = blk_start;
  e.blk_len = s.B;
  e.embed_f32 = s.wfmt == DLLM_W_F32_SPLIT;
  e.vocab = s.V;
  e.mask_id = s.mask_id;
  e.npart = s.d / 128;
  e.status = c.at<int>(c.l.status);
  e.seq_blk = c.seq_blk;
  e.tokens = stt->tokens;
  e.masked = stt->masked;
  e.embed = w->embed;
  e.x = c.at<float>(c.l.x);
  e.xb = c.at<__nv_bfloat16>(c.l.xb);
  e.sumsq = c.at<float>(c.l.sumsq);
  e.segs = c.at<int>(c.l.segs);
  e.seq_start = stt->seq_start;
  e.mode = s.mode;
  e.window = s.W;
  e.seg_end = seg_end;
  e.zero = zero;
  e.nzero = (int)nzero;
  return cuda_status(launch_embed(e, pdl, c.st));
}

// How much of the weights that come next the layer stack pulls into L2 ahead
// of use.  The attention kernel moves little data, so while it runs HBM
// would idle: it can prefetch its own layer's W_o and the start of the next
// weights (the next layer's W_qkv, or the LM head after the last layer);
// the O-projection can prefetch a further part.  Off by default: on the
// 8B-shaped stacks the projections' time goes to their ramp-up and tail, not
// to the weight stream, and the extra traffic cost more than it saved.
struct PrefetchTune {
  // 8 MB of the next layer's W_qkv while attention runs: -1.7 % step time on
  // the LLaDA-8B shape, neutral on Dream-7B (4-12 MB swept; W_o during
  // attention and prefetches from the O-projection were slower).
  long long attn_next = 8ll << 20;
  long long oproj_next = 0;
  bool attn_wo = false;
};
PrefetchTune g_pf_tune;

long long round16(long long v) { return v < 0 ? 0 : v & ~15ll; }

// All L layers of n_rows rows per sequence at row0 (the block) in one
// launch of the layer-stack kernel.  The embedding kernel before it clears
// the kernel's flags.
dllm_status run_stack(const Ctx& c, const dllm_weights* w, const dllm_state* stt, int row0,
                      int n_rows, int blk_start, const StackPlan& P) {
  const Shape& s = c.s;
  const int R = s.b * n_rows;
  const int g = s.Hq / s.Hkv;
  void* xb = c.at<void>(c.l.xb);
  void* q = c.at<void>(c.l.q);
  void* attn = c.at<void>(c.l.attn);
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap m[7];
  if (!make_map(&m[0], w->wqkv, s.Kw, s.qkv_rows, s.L, 64, 128, sw) ||
      !make_map(&m[1], w->wo, s.Ko, s.d, s.L, 64, 128, sw) ||
      !make_map(&m[2], xb, s.d, R, 1, 64, P.nt, sw) ||
      !make_map(&m[3], attn, s.Hq * s.D, R, 1, 64, P.nt, sw) ||
      !make_map(&m[4], q, s.D, (uint64_t)g * n_rows, (uint64_t)s.b * s.Hkv, 64, 128, sw) ||
      !make_map(&m[5], stt->k_cache, s.D, s.S, (uint64_t)s.L * s.b * s.Hkv, 64, 64, sw) ||
      !make_map(&m[6], stt->v_cache, s.D, s.S, (uint64_t)s.L * s.b * s.Hkv, 64, 64, sw))
    return DLLM_ERR_CUDA;
  StackParams p{};
  p.L = s.L;
  p.R = R;
  p.n_rows = n_rows;
  p.batch = s.b;
  p.Hq = s.Hq;
  p.Hkv = s.Hkv;
  p.S = s.S;
  p.d = s.d;
  p.g = g;
  p.qt = P.qt;
  p.ot = P.ot;
  p.qkbt = P.qkbt;
  p.okbt = P.okbt;
  p.qn = P.qn;
  p.on = P.on;
  p.qmaxc = P.qmaxc;
  p.omaxc = P.omaxc;
  p.rt = P.rt;
  p.chunks = P.chunks;
  p.tpc = P.tpc;
  p.units = P.units;
  p.mode = s.mode;
  p.blk_start = blk_start;
  p.blk_len = s.B;
  p.window = s.W;
  p.seg_end = 0;
  p.dep_lo = row0;
  p.dep_hi = row0 + n_rows;
  p.lookahead = g_stack_tune.lookahead;
  p.seq_start = stt->seq_start;
  p.q = static_cast<__nv_bfloat16*>(q);
  p.attn = static_cast<__nv_bfloat16*>(attn);
  p.qpart = c.at<float>(c.l.stk_qpart);
  p.opart = c.at<float>(c.l.stk_opart);
  p.apart = c.at<float>(c.l.stk_apart);
  p.aml = c.at<float2>(c.l.stk_aml);
  p.flags = c.at<int>(c.l.stk_flags);
  p.fs = P.fs;
  p.status = c.at<int>(c.l.status);
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)s.D);
  // epilogue of the Q/K/V projection: RMS scale, RoPE, q and the cache rows
  GemmParams& gq = p.gq;
  gq.M = s.qkv_rows;
  gq.R = R;
  gq.K = s.Kw;
  gq.layer = 0;
  gq.status = p.status;
  gq.n_rows = n_rows;
  gq.row0 = row0;
  gq.seq_start = stt->seq_start;
  gq.Hq = s.Hq;
  gq.Hkv = s.Hkv;
  gq.D = s.D;
  gq.S = s.S;
  gq.batch = s.b;
  gq.rope_tab = s.theta > 0.f ? c.at<float2>(c.l.rope) : nullptr;
  gq.q_out = p.q;
  gq.k_cache = static_cast<__nv_bfloat16*>(stt->k_cache);
  gq.v_cache = static_cast<__nv_bfloat16*>(stt->v_cache);
  gq.sumsq_in = c.at<float>(c.l.sumsq);
  gq.npart = s.d / 128;
  gq.d_norm = s.d;
  gq.rms_eps = kRmsEps;
  // epilogue of the O-projection: residual, its bf16 copy, sums of squares
  GemmParams& go = p.go;
  go.M = s.d;
  go.R = R;
  go.K = s.Ko;
  go.status = p.status;
  go.n_rows = n_rows;
  go.row0 = row0;
  go.x = c.at<float>(c.l.x);
  go.xb = static_cast<__nv_bfloat16*>(xb);
  go.d_model = s.d;
  go.sumsq_out = c.at<float>(c.l.sumsq);
  go.npart = s.d / 128;
  go.d_norm = s.d;
  return cuda_status(launch_stack(P.nt, m, p, P.grid, true, c.st));
}

// Embed + L pre-norm layers for n_rows rows per sequence at row0.  lm_next:
// the LM head follows the last layer.
dllm_status run_forward(const Ctx& c, const dllm_weights* w, const dllm_state* stt, int row0,
                        int n_rows, int blk_start, int seg_end, bool lm_next) {
  const Shape& s = c.s;
  if (c.seq_blk == nullptr && seg_end == 0 && row0 == blk_start && c.l.stk_nflags > 0 &&
      stack_usable()) {
    const StackPlan P = plan_stack(s, n_rows, blk_start, kNumSMs);
    if (P.ok && (long long)s.L * P.fs + 32 <= c.l.stk_nflags && P.chunks <= c.l.stk_chunks) {
      DLLM_TRY(run_embed(c, w, stt, row0, n_rows, blk_start, seg_end, true,
                         c.at<int>(c.l.stk_flags), (long long)s.L * P.fs + 32));
      return run_stack(c, w, stt, row0, n_rows, blk_start, P);
    }
  }
  DLLM_TRY(run_embed(c, w, stt, row0, n_rows, blk_start, seg_end, true));
  int ntb = key_tiles_bound(s, blk_start, seg_end);
  if (c.seq_blk)  // each sequence at its own block: plan for the widest key set
    for (int blk = s.P; blk < s.S; blk += s.B) ntb = std::max(ntb, key_tiles_bound(s, blk, seg_end));
  const long long qkv_bytes = (long long)s.qkv_rows * s.Kw * 2;
  const long long wo_bytes = (long long)s.d * s.Ko * 2;
  const auto* wqkv = static_cast<const uint8_t*>(w->wqkv);
  const auto* wo = static_cast<const uint8_t*>(w->wo);
  const PrefetchTune tune = g_pf_tune;
  for (int l = 0; l < s.L; ++l) {
    const uint8_t* next = nullptr;
    long long next_bytes = 0;
    if (l + 1 < s.L) {
      next = wqkv + (l + 1) * qkv_bytes;
      next_bytes = qkv_bytes;
    } else if (lm_next) {
      next = static_cast<const uint8_t*>(w->w_lm);
      next_bytes = (long long)s.V * s.Kw * 2;
    }
    const long long a = round16(std::min(tune.attn_next, next_bytes));
    const long long o = round16(std::min(tune.oproj_next, next_bytes - a));
    L2Prefetch pf_attn{}, pf_oproj{};
    if (tune.attn_wo) {
      pf_attn.ptr[0] = wo + l * wo_bytes;
      pf_attn.bytes[0] = wo_bytes;
    }
    if (next && a > 0) {
      pf_attn.ptr[1] = next;
      pf_attn.bytes[1] = a;
    }
    if (next && o > 0) {
      pf_oproj.ptr[0] = next + a;
      pf_oproj.bytes[0] = o;
    }
    DLLM_TRY(run_qkv(c, w->wqkv, l, c.at<void>(c.l.xb), c.at<float>(c.l.sumsq), row0, n_rows,
                     stt->seq_start, c.at<void>(c.l.q), stt->k_cache, stt->v_cache, true));
    const AttnKeys keys{nullptr, stt->seq_start, blk_start, seg_end, row0, row0 + n_rows};
    DLLM_TRY(run_attn(c, l, n_rows, c.at<void>(c.l.q), stt->k_cache, stt->v_cache, keys,
                      c.at<void>(c.l.attn), ntb, true, pf_attn));
    DLLM_TRY(run_oproj(c, w->wo, l, c.at<void>(c.l.attn), row0, n_rows, c.at<float>(c.l.x),
                       c.at<void>(c.l.xb), c.at<float>(c.l.sumsq), true, pf_oproj));
  }
  return DLLM_OK;
}

dllm_status run_final_norm(const Ctx& c, const float* x, int row0, int n_rows, int blk_start,
                           const uint8_t* masked, const void* plants, void* h, bool pdl) {
  const Shape& s = c.s;
  FinalNormParams f{};
  f.batch = s.b;
  f.B = s.B;
  f.d = s.d;
  f.n_rows = n_rows;
  f.row0 = row0;
  f.blk_start = blk_start;
  f.S = s.S;
  f.P = s.P;
  f.G = s.G;
  f.eps = kRmsEps;
  f.x = x;
  f.masked = masked;
  f.plants = static_cast<const __nv_bfloat16*>(plants);
  f.h = static_cast<__nv_bfloat16*>(h);
  f.seq_blk = c.seq_blk;
  f.status = c.ws ? c.at<int>(c.l.status) : nullptr;
  return cuda_status(launch_final_norm(f, pdl, c.st));
}

dllm_status run_lmhead(const Ctx& c, const void* w_lm, const void* h, int n_rows, bool pdl) {
  const Shape& s = c.s;
  const GemmPlan g = plan_lmhead(s.V, n_rows, s.Kw);
  if (g.grid / g.n_tiles > c.l.lm_slots) return DLLM_ERR_WORKSPACE;
  CUtensorMap wm, xm;
  if (!make_map(&wm, w_lm, s.Kw, s.V, 1, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&xm, h, s.d, n_rows, 1, 64, g.nt, CU_TENSOR_MAP_SWIZZLE_128B))
    return DLLM_ERR_CUDA;
  GemmParams p{};
  p.M = s.V;
  p.R = n_rows;
  p.K = s.Kw;
  p.kx_blocks = s.d / 64;
  p.m_tiles = g.m_tiles;
  p.n_tiles = g.n_tiles;
  p.splits = 1;
  p.kb_per_split = g.kbps;
  p.units = g.units;
  p.layer = 0;
  p.status = c.at<int>(c.l.status);
  p.stats = c.at<LmStat>(c.l.stats);
  p.stat_slots = g.grid / g.n_tiles;
  return cuda_status(launch_gemm(EPI_LMHEAD, g.nt, wm, xm, p, g.grid, pdl, c.st));
}

dllm_status run_commit(const Ctx& c, const dllm_state* stt, int blk_start, bool from_stats,
                       const float* conf_in, const int* tok_in, bool pdl) {
  const Shape& s = c.s;
  const GemmPlan g = plan_lmhead(s.V, s.b * s.B, s.Kw);
  CommitParams p{};
  p.batch = s.b;
  p.S = s.S;
  p.B = s.B;
  p.blk_start = blk_start;
  p.stat_slots = g.grid / g.n_tiles;
  p.vocab = s.V;
  p.tau = s.tau;
  p.stats = from_stats ? c.at<LmStat>(c.l.stats) : nullptr;
  p.conf = from_stats ? c.at<float>(c.l.conf) : const_cast<float*>(conf_in);
  p.tok = from_stats ? c.at<int>(c.l.tok) : const_cast<int*>(tok_in);
  p.gap = from_stats ? c.at<float>(c.l.gap) : nullptr;
  p.tokens = stt->tokens;
  p.masked = stt->masked;
  p.commit = c.at<uint8_t>(c.l.commit);
  p.remaining = c.at<int>(c.l.remaining);
  p.block_done = c.at<int>(c.l.blkdone);
  p.refresh = c.at<int>(c.l.refresh);
  p.do_commit = 1;
  p.topk = s.commit_mode == DLLM_COMMIT_TOPK;
  p.steps_per_block = s.spb;
  p.step_ctr = c.at<int>(c.l.stepc);
  p.exit_state = s.commit_mode == DLLM_COMMIT_EARLY_EXIT ? c.at<int>(c.l.exitst) : nullptr;
  p.exit_tau = s.exit_tau;
  p.tau_seq = stt->tau;
  p.seq_blk = c.seq_blk;
  p.seq_done = c.seq_blk ? c.at<int>(c.l.seqdone) : nullptr;
  p.status = c.ws ? c.at<int>(c.l.status) : nullptr;
  return cuda_status(launch_commit(p, pdl, c.st));
}

dllm_status check_state(const Shape& s, const dllm_weights* w, const dllm_state* st) {
  if (!w || !st || !w->wqkv || !w->wo || !w->w_lm || !w->embed || !st->tokens || !st->masked ||
      !st->seq_start || !st->k_cache || !st->v_cache)
    return DLLM_ERR_INVALID;
  if (!aligned16(w->wqkv) || !aligned16(w->wo) || !aligned16(w->w_lm) || !aligned16(w->embed) ||
      !aligned16(st->k_cache) || !aligned16(st->v_cache))
    return DLLM_ERR_INVALID;
  (void)s;
  return DLLM_OK;
}

// [start, start + len) inside [0, limit), in 64-bit so that no int32
// argument can wrap the test.
bool rows_ok(long long start, long long len, long long limit) {
  return start >= 0 && len >= 1 && start + len <= limit;
}

dllm_status check_block(const Shape& s, int blk) {
  if (blk < s.P || !rows_ok(blk, s.B, s.S) || (blk - s.P) % s.B) return DLLM_ERR_INVALID;
  return DLLM_OK;
}

dllm_status step(const Ctx& c, const dllm_weights* w, const dllm_state* st, int blk) {
  const Shape& s = c.s;
  if (!st->plants || !aligned16(st->plants)) return DLLM_ERR_INVALID;
  const bool none = s.mode == DLLM_CACHE_NONE;
  const bool sufq = s.mode == DLLM_CACHE_PREFIX_SUFFIXQ;
  const int row0 = none ? 0 : blk;
  const int n_rows = none ? blk + s.B : sufq ? s.S - blk : s.B;
  DLLM_TRY(run_forward(c, w, st, row0, n_rows, blk, none ? blk + s.B : sufq ? s.S : 0,
                       true));
  DLLM_TRY(run_final_norm(c, c.at<float>(c.l.x), row0, n_rows, blk, st->masked, st->plants,
                          c.at<void>(c.l.h), true));
  DLLM_TRY(run_lmhead(c, w->w_lm, c.at<void>(c.l.h), s.b * s.B, true));
  return run_commit(c, st, blk, true, nullptr, nullptr, true);
}

// ------------------------------------------------------------------ graphs
// The launch sequence of a step, a refresh or a prefill is captured once per
// (configuration, weight / state / workspace pointers, block) into a CUDA
// graph and replayed with a single launch afterwards.  Capture runs on a
// library-owned stream; the graph is launched on the caller's stream.
struct GraphKey {
  dllm_config cfg;
  dllm_weights w;
  dllm_state st;
  const void* ws;
  size_t ws_bytes;
  int kind, blk, device;
};

struct GraphEntry {
  GraphKey key;
  cudaGraphExec_t exec;
  long long kernels;
};

std::mutex g_graph_mu;
std::vector<GraphEntry> g_graphs;
constexpr size_t kMaxGraphs = 256;

GraphKey make_key(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                  const void* ws, size_t ws_bytes, int kind, int blk) {
  GraphKey k;
  memset(&k, 0, sizeof(k));
  k.cfg = *cfg;
  k.w = *w;
  k.st = *st;
  k.ws = ws;
  k.ws_bytes = ws_bytes;
  k.kind = kind;
  k.blk = blk;
  cudaGetDevice(&k.device);
  return k;
}

cudaStream_t capture_stream(int device) {
  static cudaStream_t streams[64] = {};
  if (device < 0 || device >= 64) return nullptr;
  if (!streams[device]) cudaStreamCreateWithFlags(&streams[device], cudaStreamNonBlocking);
  return streams[device];
}

template <class F>
dllm_status run_graph(const Ctx& c, const GraphKey& key, F&& body) {
  DLLM_TRY(prepare_device());  // attribute calls may not run inside the capture below
  std::lock_guard<std::mutex> lock(g_graph_mu);
  for (const GraphEntry& e : g_graphs) {
    if (memcmp(&e.key, &key, sizeof(GraphKey)) == 0) {
      add_launches(e.kernels);
      return cuda_status(cudaGraphLaunch(e.exec, c.st));
    }
  }
  cudaStream_t cs = capture_stream(key.device);
  if (!cs) return DLLM_ERR_CUDA;
  Ctx cc = c;
  cc.st = cs;
  const unsigned long long n0 = launch_count();
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
    return DLLM_ERR_CUDA;
  const dllm_status e = body(cc);
  cudaGraph_t g = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(cs, &g);
  const long long kernels = (long long)(launch_count() - n0);
  add_launches(-kernels);  // captured, not executed
  if (e != DLLM_OK || ce != cudaSuccess || !g) {
    if (g) cudaGraphDestroy(g);
    return e != DLLM_OK ? e : DLLM_ERR_CUDA;
  }
  cudaGraphExec_t exec = nullptr;
  const cudaError_t ie = cudaGraphInstantiate(&exec, g, 0);
  cudaGraphDestroy(g);
  if (ie != cudaSuccess) return DLLM_ERR_CUDA;
  if (g_graphs.size() >= kMaxGraphs) {
    cudaGraphExecDestroy(g_graphs.front().exec);
    g_graphs.erase(g_graphs.begin());
  }
  g_graphs.push_back({key, exec, kernels});
  add_launches(kernels);
  return cuda_status(cudaGraphLaunch(exec, c.st));
}

enum GraphKind { kGraphStep = 1, kGraphRefresh = 2, kGraphPrefill = 3, kGraphSeqPass = 4 };

dllm_status step_graph(const Ctx& c, const dllm_config* cfg, const dllm_weights* w,
                       const dllm_state* st, void* ws, size_t ws_bytes, int blk) {
  const GraphKey key = make_key(cfg, w, st, ws, ws_bytes, kGraphStep, blk);
  return run_graph(c, key, [&](const Ctx& cc) { return step(cc, w, st, blk); });
}

dllm_status refresh_graph(const Ctx& c, const dllm_config* cfg, const dllm_weights* w,
                          const dllm_state* st, void* ws, size_t ws_bytes, int blk) {
  if (c.s.mode == DLLM_CACHE_NONE) return DLLM_OK;
  const GraphKey key = make_key(cfg, w, st, ws, ws_bytes, kGraphRefresh, blk);
  return run_graph(c, key, [&](const Ctx& cc) {
    return run_forward(cc, w, st, blk, cc.s.B, blk, 0, false);
  });
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

dllm_status dllm_workspace_size(const dllm_config* cfg, size_t* bytes) {
  Shape s;
  DLLM_TRY(check_cfg(cfg, &s));
  if (!bytes) return DLLM_ERR_INVALID;
  *bytes = layout(s).total;
  return DLLM_OK;
}

dllm_status dllm_workspace_init(const dllm_config* cfg, void* ws, size_t ws_bytes,
                                dllm_stream stream) {
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  // status word: zero
  if (cudaMemsetAsync(c.ws, 0, c.l.x, c.st) != cudaSuccess) return DLLM_ERR_CUDA;
  if (c.s.theta > 0.f)
    return cuda_status(launch_rope_table(c.at<float2>(c.l.rope), c.s.S, c.s.D, c.s.theta, c.st));
  return DLLM_OK;
}

dllm_status dllm_split_f32_weights(const float* src, void* dst, int64_t rows, int64_t cols,
                                   dllm_stream stream) {
  if (!src || !dst || rows < 1 || cols < 1) return DLLM_ERR_INVALID;
  return cuda_status(launch_split_f32(src, static_cast<__nv_bfloat16*>(dst), rows, cols,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

dllm_status dllm_embed_rows(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                            int32_t row0, int32_t n_rows, float* x, void* xb, float* row_sumsq,
                            dllm_stream stream) {
  Shape s;
  DLLM_TRY(check_cfg(cfg, &s));
  if (!w || !w->embed || !st || !st->tokens || !st->masked || !x || !xb) return DLLM_ERR_INVALID;
  if (!rows_ok(row0, n_rows, s.S)) return DLLM_ERR_INVALID;
  EmbedParams e{};
  e.batch = s.b;
  e.S = s.S;
  e.d = s.d;
  e.n_rows = n_rows;
  e.row0 = row0;
  e.embed_f32 = s.wfmt == DLLM_W_F32_SPLIT;
  e.vocab = s.V;
  e.mask_id = s.mask_id;
  e.npart = s.d / 128;
  e.status = nullptr;
  e.tokens = st->tokens;
  e.masked = st->masked;
  e.embed = w->embed;
  e.x = x;
  e.xb = static_cast<__nv_bfloat16*>(xb);
  e.sumsq = row_sumsq;
  e.segs = nullptr;
  return cuda_status(launch_embed(e, false, reinterpret_cast<cudaStream_t>(stream)));
}

dllm_status dllm_final_norm(const dllm_config* cfg, const float* x, int32_t row0, int32_t n_rows,
                            int32_t block_start, const uint8_t* masked, const void* plants,
                            void* h, dllm_stream stream) {
  Shape s;
  DLLM_TRY(check_cfg(cfg, &s));
  if (!x || !masked || !plants || !h) return DLLM_ERR_INVALID;
  DLLM_TRY(check_block(s, block_start));
  if (!rows_ok(row0, n_rows, s.S) || block_start < row0 ||
      (long long)block_start + s.B > (long long)row0 + n_rows)
    return DLLM_ERR_INVALID;
  Ctx c;
  c.s = s;
  c.st = reinterpret_cast<cudaStream_t>(stream);
  return run_final_norm(c, x, row0, n_rows, block_start, masked, plants, h, false);
}

dllm_status dllm_qkv_proj(const dllm_config* cfg, const dllm_weights* w, int32_t layer,
                          const void* xb, const float* row_sumsq, int32_t row0, int32_t n_rows,
                          const int32_t* seq_start, void* q_out, void* k_cache, void* v_cache,
                          void* ws, size_t ws_bytes, dllm_stream stream) {
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  if (!w || !w->wqkv || !xb || !seq_start || !q_out || !k_cache || !v_cache)
    return DLLM_ERR_INVALID;
  if (layer < 0 || layer >= c.s.L || !rows_ok(row0, n_rows, c.s.S))
    return DLLM_ERR_INVALID;
  DLLM_TRY(prepare_device());
  return run_qkv(c, w->wqkv, layer, xb, row_sumsq, row0, n_rows, seq_start, q_out, k_cache,
                 v_cache, false);
}

dllm_status dllm_block_attn(const dllm_config* cfg, int32_t layer, int32_t n_rows, const void* q,
                            const void* k_cache, const void* v_cache, const int32_t* segs,
                            void* out, void* ws, size_t ws_bytes, dllm_stream stream) {
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  if (!q || !k_cache || !v_cache || !segs || !out) return DLLM_ERR_INVALID;
  if (layer < 0 || layer >= c.s.L || n_rows < 1 || n_rows > c.s.S) return DLLM_ERR_INVALID;
  const int ntb = cdiv(c.s.S, kKeyTile) + 1;
  const AttnKeys keys{segs, nullptr, 0, 0, 0, c.s.S};
  DLLM_TRY(prepare_device());
  return run_attn(c, layer, n_rows, q, k_cache, v_cache, keys, out, ntb, false);
}

dllm_status dllm_o_proj(const dllm_config* cfg, const dllm_weights* w, int32_t layer,
                        const void* attn, int32_t row0, int32_t n_rows, float* x, void* xb,
                        float* row_sumsq, void* ws, size_t ws_bytes, dllm_stream stream) {
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  if (!w || !w->wo || !attn || !x || !xb) return DLLM_ERR_INVALID;
  if (layer < 0 || layer >= c.s.L || !rows_ok(row0, n_rows, c.s.S))
    return DLLM_ERR_INVALID;
  DLLM_TRY(prepare_device());
  return run_oproj(c, w->wo, layer, attn, row0, n_rows, x, xb, row_sumsq, false);
}

dllm_status dllm_lmhead_confidence(const dllm_config* cfg, const dllm_weights* w, const void* h,
                                   int32_t n_rows, float* conf, int32_t* tok, float* gap,
                                   void* ws, size_t ws_bytes, dllm_stream stream) {
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  if (!w || !w->w_lm || !h || !conf || !tok) return DLLM_ERR_INVALID;
  if (n_rows < 1 || n_rows > c.s.b * c.s.B) return DLLM_ERR_INVALID;
  DLLM_TRY(prepare_device());
  DLLM_TRY(run_lmhead(c, w->w_lm, h, n_rows, false));
  // reduce the per-CTA statistics (one "sequence" of n_rows rows, no commit)
  const GemmPlan g = plan_lmhead(c.s.V, n_rows, c.s.Kw);
  CommitParams p{};
  p.batch = 1;
  p.S = 0;
  p.B = n_rows;
  p.stat_slots = g.grid / g.n_tiles;
  p.vocab = c.s.V;
  p.tau = c.s.tau;
  p.stats = c.at<LmStat>(c.l.stats);
  p.conf = conf;
  p.tok = tok;
  p.gap = gap;
  p.do_commit = 0;
  if (n_rows > 64) {
    // the reduce kernel handles up to 64 rows per CTA: run it per 64-row group
    for (int r0 = 0; r0 < n_rows; r0 += 64) {
      CommitParams q = p;
      q.B = std::min(64, n_rows - r0);
      q.stats = p.stats + (size_t)r0 * p.stat_slots;
      q.conf = conf + r0;
      q.tok = tok + r0;
      q.gap = gap ? gap + r0 : nullptr;
      DLLM_TRY(cuda_status(launch_commit(q, false, c.st)));
    }
    return DLLM_OK;
  }
  return cuda_status(launch_commit(p, false, c.st));
}

dllm_status dllm_threshold_commit(const dllm_config* cfg, int32_t block_start, const float* conf,
                                  const int32_t* tok, int32_t* tokens, uint8_t* masked,
                                  uint8_t* commit, int32_t* remaining, int32_t* block_done,
                                  int32_t* refresh_list, dllm_stream stream) {
  Shape s;
  DLLM_TRY(check_cfg(cfg, &s));
  if (!conf || !tok || !tokens || !masked) return DLLM_ERR_INVALID;
  DLLM_TRY(check_block(s, block_start));
  CommitParams p{};
  p.batch = s.b;
  p.S = s.S;
  p.B = s.B;
  p.blk_start = block_start;
  p.tau = s.tau;
  p.vocab = s.V;
  p.stats = nullptr;
  p.conf = const_cast<float*>(conf);
  p.tok = const_cast<int*>(tok);
  p.tokens = tokens;
  p.masked = masked;
  p.commit = commit;
  p.remaining = remaining;
  p.block_done = block_done;
  p.refresh = refresh_list;
  p.do_commit = 1;
  p.topk = s.commit_mode == DLLM_COMMIT_TOPK;
  p.steps_per_block = s.spb;
  return cuda_status(launch_commit(p, false, reinterpret_cast<cudaStream_t>(stream)));
}

dllm_status dllm_prefill(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                         void* ws, size_t ws_bytes, dllm_stream stream) {
  NvtxRange nv("dllm_prefill");
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  DLLM_TRY(check_state(c.s, w, st));
  if (c.s.mode == DLLM_CACHE_NONE) return DLLM_OK;
  const int end =
      (c.s.mode == DLLM_CACHE_PREFIX || c.s.mode == DLLM_CACHE_PREFIX_SUFFIXQ) ? c.s.P : c.s.S;
  if (end < 1) return DLLM_OK;
  const GraphKey key = make_key(cfg, w, st, ws, ws_bytes, kGraphPrefill, 0);
  return run_graph(c, key,
                   [&](const Ctx& cc) { return run_forward(cc, w, st, 0, end, -1, end, false); });
}

dllm_status dllm_decode_step(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                             int32_t block_start, void* ws, size_t ws_bytes,
                             dllm_stream stream) {
  NvtxRange nv("dllm_decode_step");
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  DLLM_TRY(check_state(c.s, w, st));
  DLLM_TRY(check_block(c.s, block_start));
  if (!st->plants || !aligned16(st->plants)) return DLLM_ERR_INVALID;
  return step_graph(c, cfg, w, st, ws, ws_bytes, block_start);
}

dllm_status dllm_kv_cache_refresh(const dllm_config* cfg, const dllm_weights* w,
                                  const dllm_state* st, int32_t block_start, void* ws,
                                  size_t ws_bytes, dllm_stream stream) {
  NvtxRange nv("dllm_kv_cache_refresh");
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  DLLM_TRY(check_state(c.s, w, st));
  DLLM_TRY(check_block(c.s, block_start));
  return refresh_graph(c, cfg, w, st, ws, ws_bytes, block_start);
}

dllm_status dllm_decode_block(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                              int32_t block_start, int32_t max_steps, int32_t* steps_taken,
                              void* ws, size_t ws_bytes, dllm_stream stream) {
  NvtxRange nv("dllm_decode_block");
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  DLLM_TRY(check_state(c.s, w, st));
  DLLM_TRY(check_block(c.s, block_start));
  if (max_steps < 1) max_steps = c.s.B;
  if (!st->plants || !aligned16(st->plants)) return DLLM_ERR_INVALID;
  // steps until the commit step reports the block done in every sequence
  std::vector<int> done(c.s.b + 1);
  int n = 0;
  for (; n < max_steps;) {
    DLLM_TRY(step_graph(c, cfg, w, st, ws, ws_bytes, block_start));
    ++n;
    if (cudaMemcpyAsync(done.data(), c.at<int>(c.l.blkdone), sizeof(int) * c.s.b,
                        cudaMemcpyDeviceToHost, c.st) != cudaSuccess ||
        cudaMemcpyAsync(done.data() + c.s.b, c.at<int>(c.l.status), sizeof(int),
                        cudaMemcpyDeviceToHost, c.st) != cudaSuccess)
      return DLLM_ERR_CUDA;
    DLLM_TRY(wait_stream(c.st, kHostDeadlineS));
    if (done[c.s.b] != 0) return DLLM_ERR_TIMEOUT;
    int all = 1;
    for (int i = 0; i < c.s.b; ++i) all &= done[i] != 0;
    if (all) break;
  }
  if (steps_taken) *steps_taken = n;
  return refresh_graph(c, cfg, w, st, ws, ws_bytes, block_start);
}

dllm_status dllm_decode_all(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                            int32_t* passes, void* ws, size_t ws_bytes, dllm_stream stream) {
  NvtxRange nv("dllm_decode_all");
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, stream, &c));
  DLLM_TRY(check_state(c.s, w, st));
  if (c.s.mode == DLLM_CACHE_NONE || c.s.mode == DLLM_CACHE_PREFIX_SUFFIXQ)
    return DLLM_ERR_UNSUPPORTED;
  if (!st->plants || !aligned16(st->plants)) return DLLM_ERR_INVALID;
  const Shape& s = c.s;
  // every sequence starts at the first generated block
  std::vector<int> init(s.b, s.P);
  if (cudaMemcpyAsync(c.at<int>(c.l.seqblk), init.data(), sizeof(int) * s.b,
                      cudaMemcpyHostToDevice, c.st) != cudaSuccess ||
      cudaMemsetAsync(c.at<int>(c.l.seqdone), 0, sizeof(int) * s.b, c.st) != cudaSuccess ||
      cudaMemsetAsync(c.at<int>(c.l.stepc), 0, sizeof(int) * 2 * s.b, c.st) != cudaSuccess)
    return DLLM_ERR_CUDA;
  Ctx cs = c;
  cs.seq_blk = c.at<int>(c.l.seqblk);
  const GraphKey key = make_key(cfg, w, st, ws, ws_bytes, kGraphSeqPass, 0);
  // a block takes at most B steps and one refresh pass
  const int max_passes = (s.G / s.B) * (s.B + 1) + 1;
  std::vector<int> rem(s.b + 1);
  int n = 0;
  for (; n < max_passes;) {
    DLLM_TRY(run_graph(cs, key, [&](const Ctx& cc) { return step(cc, w, st, s.P); }));
    ++n;
    if (cudaMemcpyAsync(rem.data(), c.at<int>(c.l.remaining), sizeof(int) * s.b,
                        cudaMemcpyDeviceToHost, c.st) != cudaSuccess ||
        cudaMemcpyAsync(rem.data() + s.b, c.at<int>(c.l.status), sizeof(int),
                        cudaMemcpyDeviceToHost, c.st) != cudaSuccess)
      return DLLM_ERR_CUDA;
    DLLM_TRY(wait_stream(c.st, kHostDeadlineS));
    if (rem[s.b] != 0) return DLLM_ERR_TIMEOUT;
    int left = 0;
    for (int i = 0; i < s.b; ++i) left += rem[i];
    if (left == 0) break;
  }
  if (passes) *passes = n;
  return n < max_passes ? DLLM_OK : DLLM_ERR_INVALID;
}

dllm_status dllm_selftest_wait_timeout(int32_t* status, int32_t limit_us, dllm_stream stream) {
  if (!status) return DLLM_ERR_INVALID;
  DLLM_TRY(prepare_device());
  const long long us = std::min<long long>(std::max<long long>(limit_us, 1), 2000000);
  return cuda_status(launch_wait_timeout(status, us * 1000, reinterpret_cast<cudaStream_t>(stream)));
}

dllm_status dllm_set_l2_prefetch(int64_t attn_next_bytes, int64_t oproj_next_bytes,
                                 int32_t attn_prefetch_wo) {
  if (attn_next_bytes < 0 || oproj_next_bytes < 0) return DLLM_ERR_INVALID;
  g_pf_tune.attn_next = attn_next_bytes;
  g_pf_tune.oproj_next = oproj_next_bytes;
  g_pf_tune.attn_wo = attn_prefetch_wo != 0;
  dllm_graph_cache_clear();  // cached graphs hold the old prefetch ranges
  return DLLM_OK;
}

dllm_status dllm_set_layer_stack(int32_t enable, int32_t l2_lookahead) {
  if (l2_lookahead < 0 || l2_lookahead > 4096) return DLLM_ERR_INVALID;
  g_stack_tune.enable = enable != 0;
  g_stack_tune.lookahead = l2_lookahead;
  dllm_graph_cache_clear();
  return DLLM_OK;
}

dllm_status dllm_attention_plan(const dllm_config* cfg, int32_t block_start, int32_t* info) {
  Shape s;
  DLLM_TRY(check_cfg(cfg, &s));
  if (!info) return DLLM_ERR_INVALID;
  int n_rows, blk, seg_end;
  if (block_start < 0) {  // the prefill
    if (s.mode == DLLM_CACHE_NONE) return DLLM_ERR_INVALID;
    n_rows = (s.mode == DLLM_CACHE_PREFIX || s.mode == DLLM_CACHE_PREFIX_SUFFIXQ) ? s.P : s.S;
    if (n_rows < 1) return DLLM_ERR_INVALID;
    blk = -1;
    seg_end = n_rows;
  } else {  // the rows and key range a decode step uses
    DLLM_TRY(check_block(s, block_start));
    const bool none = s.mode == DLLM_CACHE_NONE;
    const bool sufq = s.mode == DLLM_CACHE_PREFIX_SUFFIXQ;
    n_rows = none ? block_start + s.B : sufq ? s.S - block_start : s.B;
    blk = block_start;
    seg_end = none ? block_start + s.B : sufq ? s.S : 0;
  }
  const int ntb = key_tiles_bound(s, blk, seg_end);
  const AttnPlan a = plan_attn(s, n_rows, ntb);
  info[0] = a.sg ? 32 : 128;
  info[1] = a.row_tiles;
  info[2] = a.chunks;
  info[3] = a.tpc;
  info[4] = (int32_t)std::min<long long>((long long)s.b * s.Hkv * a.row_tiles * a.chunks, INT32_MAX);
  info[5] = ntb;
  info[6] = a.sg ? 128 : 256;
  info[7] = a.tpc <= 1 ? 1 : 2;
  return DLLM_OK;
}

dllm_status dllm_layer_stack_plan(const dllm_config* cfg, int32_t block_start, int32_t* info) {
  Shape s;
  DLLM_TRY(check_cfg(cfg, &s));
  if (!info) return DLLM_ERR_INVALID;
  DLLM_TRY(check_block(s, block_start));
  const StackPlan P = plan_stack(s, s.B, block_start, kNumSMs);
  for (int i = 0; i < 8; ++i) info[i] = 0;
  if (!P.ok) return DLLM_OK;
  info[0] = 1;
  info[1] = P.nt;
  info[2] = P.qn;
  info[3] = P.on;
  info[4] = P.chunks;
  info[5] = P.tpc;
  info[6] = P.units;
  // every k-block of every tile belongs to exactly one segment, and the
  // segments of a tile are numbered 0..nc-1 in k order
  bool good = true;
  for (int ph = 0; ph < 2 && good; ++ph) {
    const int tiles = ph ? P.ot : P.qt, kbt = ph ? P.okbt : P.qkbt, n = ph ? P.on : P.qn;
    const int maxc = ph ? P.omaxc : P.qmaxc;
    std::vector<int> owner((size_t)tiles * kbt, -1), nc(tiles, -1), next(tiles, 0);
    for (int c = 0; c < n && good; ++c) {
      StackSeg sg[kStackMaxSeg];
      const int k = stack_segments(c, tiles, kbt, n, sg, kStackMaxSeg);
      if (k < 1) good = false;
      for (int i = 0; i < k && good; ++i) {
        const StackSeg& g = sg[i];
        if (g.tile < 0 || g.tile >= tiles || g.kb0 < 0 || g.kb1 > kbt || g.kb0 >= g.kb1 ||
            g.nc < 1 || g.nc > maxc || g.ci != next[g.tile] || (nc[g.tile] >= 0 && nc[g.tile] != g.nc))
          good = false;
        if (!good) break;
        nc[g.tile] = g.nc;
        ++next[g.tile];
        for (int kb = g.kb0; kb < g.kb1; ++kb) {
          int& o = owner[(size_t)g.tile * kbt + kb];
          if (o >= 0) good = false;
          o = c;
        }
      }
    }
    for (int t = 0; t < tiles && good; ++t) {
      if (next[t] != nc[t]) good = false;
      for (int kb = 0; kb < kbt; ++kb)
        if (owner[(size_t)t * kbt + kb] < 0) good = false;
    }
  }
  info[7] = good ? 1 : 0;
  return DLLM_OK;
}

void dllm_graph_cache_clear(void) {
  std::lock_guard<std::mutex> lock(g_graph_mu);
  for (GraphEntry& e : g_graphs) cudaGraphExecDestroy(e.exec);
  g_graphs.clear();
}

dllm_status dllm_step_outputs(const dllm_config* cfg, void* ws, size_t ws_bytes, float** conf,
                              int32_t** tok, float** gap, uint8_t** commit, int32_t** block_done,
                              int32_t** refresh_list) {
  Ctx c;
  DLLM_TRY(make_ctx(cfg, ws, ws_bytes, nullptr, &c));
  if (conf) *conf = c.at<float>(c.l.conf);
  if (tok) *tok = c.at<int>(c.l.tok);
  if (gap) *gap = c.at<float>(c.l.gap);
  if (commit) *commit = c.at<uint8_t>(c.l.commit);
  if (block_done) *block_done = c.at<int>(c.l.blkdone);
  if (refresh_list) *refresh_list = c.at<int>(c.l.refresh);
  return DLLM_OK;
}

dllm_status dllm_device_status(void* ws, int32_t* code, dllm_stream stream) {
  if (!ws || !code) return DLLM_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(code, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DLLM_ERR_CUDA;
  return DLLM_OK;
}

// ---------------------------------------------------------------------------
// LM head + confidence without a caller workspace.
//
// Some callers cannot hand this library device memory: they run under an
// inference server or plugin host whose allocator owns the whole device pool
// and forbids cudaMalloc on the request path, or they sit behind a binding
// that can pass tensors but not an extra workspace buffer.  This entry point
// serves them: its only scratch, the per-CTA vocabulary statistics, lives in
// the fixed-size array below, which every GPU that loads the library keeps
// until the process exits.  Nothing here allocates.
// ---------------------------------------------------------------------------
namespace {
constexpr int kNoAllocMaxSlots = 160;  // persistent LM-head CTAs per row tile (<= SM count)
}
static __device__ __align__(256) dllm::LmStat
    g_noalloc_stats[DLLM_NOALLOC_MAX_ROWS * kNoAllocMaxSlots];
// Status word of the call in flight: a bounded device wait that gives up sets
// a bit here, and the reduce kernel then marks every row of the call invalid.
static __device__ __align__(256) int g_noalloc_status;

namespace {
// Device addresses of g_noalloc_stats and g_noalloc_status on the current
// device, looked up once per device (host code may not use the symbols
// themselves as device addresses).
bool noalloc_scratch(dllm::LmStat** stats, int** status) {
  static std::mutex mu;
  static dllm::LmStat* addr[64] = {};
  static int* st_addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* ptr = nullptr;
    void* sp = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_stats) != cudaSuccess ||
        cudaGetSymbolAddress(&sp, g_noalloc_status) != cudaSuccess)
      return false;
    addr[dev] = static_cast<dllm::LmStat*>(ptr);
    st_addr[dev] = static_cast<int*>(sp);
  }
  *stats = addr[dev];
  *status = st_addr[dev];
  return true;
}
}  // namespace

dllm_status dllm_lmhead_confidence_noalloc(const dllm_config* cfg, const dllm_weights* w,
                                           const void* h, int32_t n_rows, float* conf,
                                           int32_t* tok, float* gap, dllm_stream stream) {
  Shape s;
  DLLM_TRY(check_cfg(cfg, &s));
  if (!w || !w->w_lm || !h || !conf || !tok) return DLLM_ERR_INVALID;
  if (n_rows < 1) return DLLM_ERR_INVALID;
  if (n_rows > DLLM_NOALLOC_MAX_ROWS) return DLLM_ERR_UNSUPPORTED;  // scratch holds 256 rows
  DLLM_TRY(prepare_device());
  const GemmPlan g = plan_lmhead(s.V, n_rows, s.Kw);
  const int slots = g.grid / g.n_tiles;
  if (slots > kNoAllocMaxSlots) return DLLM_ERR_UNSUPPORTED;
  LmStat* scratch = nullptr;
  int* dstatus = nullptr;
  if (!noalloc_scratch(&scratch, &dstatus)) return DLLM_ERR_CUDA;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap wm, xm;
  if (!make_map(&wm, w->w_lm, s.Kw, s.V, 1, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&xm, h, s.d, n_rows, 1, 64, g.nt, CU_TENSOR_MAP_SWIZZLE_128B))
    return DLLM_ERR_CUDA;
  GemmParams p{};
  p.M = s.V;
  p.R = n_rows;
  p.K = s.Kw;
  p.kx_blocks = s.d / 64;
  p.m_tiles = g.m_tiles;
  p.n_tiles = g.n_tiles;
  p.splits = 1;
  p.kb_per_split = g.kbps;
  p.units = g.units;
  p.layer = 0;
  p.status = dstatus;
  p.stats = scratch;  // every slot a later read needs is written by this launch
  p.stat_slots = slots;
  DLLM_TRY(cuda_status(cudaMemsetAsync(dstatus, 0, sizeof(int), st)));
  DLLM_TRY(cuda_status(launch_gemm(EPI_LMHEAD, g.nt, wm, xm, p, g.grid, false, st)));
  for (int r0 = 0; r0 < n_rows; r0 += 64) {  // the reduce kernel takes 64 rows per CTA
    CommitParams q{};
    q.batch = 1;
    q.B = std::min(64, n_rows - r0);
    q.stat_slots = slots;
    q.vocab = s.V;
    q.tau = s.tau;
    q.stats = scratch + (size_t)r0 * slots;
    q.conf = conf + r0;
    q.tok = tok + r0;
    q.gap = gap ? gap + r0 : nullptr;
    q.do_commit = 0;
    q.status = dstatus;
    q.invalid_on_status = 1;
    DLLM_TRY(cuda_status(launch_commit(q, false, st)));
  }
  return DLLM_OK;
}

uint64_t dllm_launch_count(void) { return dllm::launch_count(); }

const char* dllm_status_string(dllm_status s) {
  switch (s) {
    case DLLM_OK: return "ok";
    case DLLM_ERR_INVALID: return "invalid argument";
    case DLLM_ERR_UNSUPPORTED: return "unsupported shape";
    case DLLM_ERR_CUDA: return "CUDA error";
    case DLLM_ERR_TIMEOUT: return "device wait timed out";
    case DLLM_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

}  // extern "C"
