// Persistent layer-stack kernel: every layer of a decode step (or of a block
// refresh) in one launch, one CTA per SM.
//
// In a decode step each projection reads a large weight matrix once for only
// b*B activation rows, so the step is a weight stream; what costs time is
// every place where that stream stops: kernel boundaries, split-K tails and
// the attention's dependent chain, during which HBM has nothing to do.  Here
// the weight stream never waits for activations.  Every CTA owns a fixed,
// equal share of every layer's Q/K/V and O-projection weights (stream-K:
// contiguous runs of (tile, 64-wide k-block) pairs) and one thread streams
// them, layer after layer, through a shared-memory ring, while a second
// thread keeps an L2 prefetch a fixed number of k-blocks ahead of it.  The
// activations are loaded only once the CTAs that produce them have published
// them, through counters in global memory (release / acquire), so a weight
// stage waits in shared memory (or L2) for its activations instead of the
// other way round.
//
// Warp roles (384 threads):
//   warp 0      weight producer (TMA, ring of kWStages stages, L2 lookahead)
//   warp 1      activation producer: waits for the columns a k-block reads
//               (the previous O-projection's tiles, or this layer's
//               attention of the heads it covers), then loads them by TMA
//   warp 2      UMMA issuer (tcgen05, fp32 accumulators double-buffered in TMEM)
//   warps 4-7   GEMM epilogue: a segment's fp32 partial goes to global memory
//               (L2); the tile's last contributor (arrival counter) adds the
//               partials in contributor order, runs the fused epilogue (RMS
//               scale + RoPE + cache store, or residual add + bf16 copy + sums
//               of squares) and publishes the tile
//   warps 8-11  attention: at most one (sequence, kv head, row tile, key
//               chunk) unit per CTA and layer, on tcgen05 with 64-key tiles.
//               Cache tiles outside the step's rows are requested as soon as
//               the previous layer's unit is done; the key chunks of a row
//               tile merge through global memory, each chunk finishing a slice
//               of head_dim columns.
// Every wait is bounded: a wait that gives up sets the timeout bit of the
// status word and the launch-wide abort word, and every role then stops.
// The sum order of split-K partials and key chunks is fixed, so results do
// not depend on timing.
#include <float.h>
#include <limits.h>

#include "gemm_epi.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace dllm {

constexpr int kStackThreads = 384;

// Timeline probe: with DLLM_STACK_TRACE defined, STACK_STAMP(l, k) records
// %globaltimer for event k of layer l of this CTA into a buffer set with
// dllm_stack_trace_set; other builds compile it to nothing.
#ifdef DLLM_STACK_TRACE
__device__ unsigned long long* g_stack_trace = nullptr;
#define STACK_STAMP(l, k)                                                                 \
  do {                                                                                    \
    if (g_stack_trace) g_stack_trace[((size_t)blockIdx.x * p.L + (l)) * 32 + (k)] = global_ns(); \
  } while (0)
// time spent in a wait, added to slot k of layer l
#define STACK_T0 const unsigned long long _t0 = g_stack_trace ? global_ns() : 0
#define STACK_ACC(l, k)                                                                        \
  do {                                                                                         \
    if (g_stack_trace)                                                                         \
      g_stack_trace[((size_t)blockIdx.x * p.L + (l)) * 32 + (k)] += global_ns() - _t0;         \
  } while (0)
#else
#define STACK_STAMP(l, k) \
  do {                    \
  } while (0)
#define STACK_T0 \
  do {           \
  } while (0)
#define STACK_ACC(l, k) \
  do {                  \
  } while (0)
#endif
constexpr int kAttKeys = 64;  // keys per attention tile

#ifndef DLLM_STACK_WSTAGES
#define DLLM_STACK_WSTAGES 5
#endif
#ifndef DLLM_STACK_ASTAGES
#define DLLM_STACK_ASTAGES 4
#endif

template <int NT>
struct StackCfg {
  static constexpr int kWStages = NT <= 32 ? DLLM_STACK_WSTAGES : DLLM_STACK_WSTAGES - 1;
  static constexpr int kAStages = NT <= 32 ? DLLM_STACK_ASTAGES : (DLLM_STACK_ASTAGES + 1) / 2;
  static constexpr int kAttStages = 2;
  static constexpr int kWBytes = 128 * 64 * 2;
  static constexpr int kXBytes = NT * 64 * 2;
  static constexpr int kQBytes = 128 * 128 * 2;         // 128 query rows x head_dim 128
  static constexpr int kKVBytes = kAttKeys * 128 * 2;   // one K or V tile
  static constexpr int kPBytes = 128 * kAttKeys * 2;
  static constexpr int oW = 0;
  static constexpr int oX = oW + kWStages * kWBytes;
  static constexpr int oQ = oX + kAStages * kXBytes;
  static constexpr int oK = oQ + kQBytes;
  static constexpr int oV = oK + kAttStages * kKVBytes;
  static constexpr int oP = oV + kAttStages * kKVBytes;
  static constexpr int oStage = oP + kPBytes;            // epilogue staging, 16 x 128 fp32
  static constexpr int oRun = oStage + 16 * 128 * 4;     // epilogue per-column arrays
  static constexpr int oBar = oRun + NT * 16;
  static constexpr int kBars = 2 * kWStages + 2 * kAStages + 4 + 3 + kAttStages + 2;
  static constexpr int oMisc = oBar + kBars * 8;
  static constexpr int kMisc = 256;
  static constexpr size_t kSmem = 1024 + oMisc + kMisc;
  static_assert(kSmem <= 227 * 1024, "layer-stack shared memory");
  static constexpr int kTmemCols = 512;  // GEMM accumulators [0, 2 NT), S [256, 320), O [384, 512)
};

// Flag layout of one layer (ints).
struct StackFlags {
  int qarr, qdone, oarr, odone, amerge, adone;
};
// Offsets are in counters; counter i of a layer is the int at i * kFlagStride.
__device__ __forceinline__ StackFlags stack_flags(const StackParams& p) {
  StackFlags f;
  f.qarr = 0;
  f.qdone = p.qt;
  f.oarr = 2 * p.qt;
  f.odone = 2 * p.qt + p.ot;
  f.amerge = 2 * p.qt + 2 * p.ot;
  f.adone = f.amerge + p.batch * p.Hkv * p.rt;
  return f;
}

// Counters sit one per 128-byte line, so that CTAs polling different
// counters load different L2 lines.
constexpr int kFlagStride = 32;  // ints

// Poll n counters (n <= 32, kFlagStride apart) until each reaches target.
// The loads of one round are issued together and are relaxed; the thread
// sleeps a little between rounds (every poller shares the L2 with the weight
// stream), and one acquire fence follows success.  Gives up after the wait
// limit or when another role has aborted the launch.
__device__ __noinline__ bool poll_range(const int* f, int n, int target, int* abort_w,
                                        int* status) {
  const unsigned long long t0 = global_ns();
  uint32_t nap = 32;
  for (uint32_t i = 0;; ++i) {
    int v[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = k < n ? ld_relaxed_gpu(f + k * kFlagStride) : target;
    bool all = true;
#pragma unroll
    for (int k = 0; k < 32; ++k) all = all && v[k] >= target;
    if (all) {
      fence_acq_rel_gpu();
      return true;
    }
    __nanosleep(nap);
    if (nap < 256) nap <<= 1;
    if ((i & 15u) == 15u) {
      if (ld_relaxed_gpu(abort_w) != 0) return false;
      if (global_ns() - t0 > kWaitLimitNs) {
        if (status) atomicOr(status, kErrTimeout);
        atomicExch(abort_w, 1);
        return false;
      }
    }
  }
}
__device__ __forceinline__ bool poll_flag(const int* f, int target, int* abort_w, int* status) {
  return poll_range(f, 1, target, abort_w, status);
}

// Key segments (start, len) x 2 of sequence b (the same rule as the attention
// kernel): prefix + block (PREFIX), the whole valid range (DUAL), or the
// window after the block plus the trailing position (DUAL_PRUNED).
__device__ __forceinline__ void stack_key_segments(const StackParams& p, int b, int* sg) {
  const int st = p.seq_start[b];
  const int end = p.blk_start + p.blk_len;
  int l0, s1 = 0, l1 = 0;
  if (p.seg_end > 0) {
    l0 = p.seg_end - st;
  } else if (p.mode == 2) {  // DUAL
    l0 = p.S - st;
  } else if (p.mode == 3) {  // DUAL_PRUNED
    const int wend = min(end + p.window, p.S);
    l0 = wend - st;
    if (end < p.S && p.S - 1 >= wend) {
      s1 = p.S - 1;
      l1 = 1;
    }
  } else {  // PREFIX
    l0 = end - st;
  }
  sg[0] = st;
  sg[1] = l0 > 0 ? l0 : 0;
  sg[2] = s1;
  sg[3] = l1;
}

__device__ __forceinline__ void key_tile64(const int* sg, int t, int& start, int& nvalid) {
  const int n0 = (sg[1] + kAttKeys - 1) / kAttKeys;
  if (t < n0) {
    start = sg[0] + t * kAttKeys;
    nvalid = min(kAttKeys, sg[1] - t * kAttKeys);
  } else {
    const int tt = t - n0;
    start = sg[2] + tt * kAttKeys;
    nvalid = min(kAttKeys, sg[3] - tt * kAttKeys);
  }
}

template <int NT>
__global__ void __launch_bounds__(kStackThreads, 1)
    stack_kernel(const __grid_constant__ CUtensorMap wq_map,
                 const __grid_constant__ CUtensorMap wo_map,
                 const __grid_constant__ CUtensorMap xb_map,
                 const __grid_constant__ CUtensorMap at_map,
                 const __grid_constant__ CUtensorMap q_map,
                 const __grid_constant__ CUtensorMap k_map,
                 const __grid_constant__ CUtensorMap v_map, const __grid_constant__ StackParams p) {
  using C = StackCfg<NT>;
  constexpr int WS = C::kWStages, AS = C::kAStages, STA = C::kAttStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* w_ring = base + C::oW;
  uint8_t* x_ring = base + C::oX;
  uint8_t* q_s = base + C::oQ;
  uint8_t* k_s = base + C::oK;
  uint8_t* v_s = base + C::oV;
  uint8_t* p_s = base + C::oP;
  float* stage = reinterpret_cast<float*>(base + C::oStage);
  LmStat* run = reinterpret_cast<LmStat*>(base + C::oRun);
  uint64_t* w_full = reinterpret_cast<uint64_t*>(base + C::oBar);
  uint64_t* w_empty = w_full + WS;
  uint64_t* a_full = w_empty + WS;
  uint64_t* a_empty = a_full + AS;
  uint64_t* tfull = a_empty + AS;
  uint64_t* tempty = tfull + 2;
  uint64_t* bar_q = tempty + 2;
  uint64_t* bar_s = bar_q + 1;
  uint64_t* bar_o = bar_s + 1;
  uint64_t* bar_kv = bar_o + 1;      // [STA]
  uint64_t* fin_mma = bar_kv + STA;  // the GEMM issuer's last UMMAs
  uint64_t* fin_att = fin_mma + 1;   // the attention issuer's last UMMAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + C::oMisc);
  volatile int* bcast = reinterpret_cast<volatile int*>(tmem_slot + 1);  // [0] epilogue, [1] attention
  int* nseg = reinterpret_cast<int*>(tmem_slot + 4);                    // [2]
  StackSeg* segs = reinterpret_cast<StackSeg*>(tmem_slot + 8);          // [2][kStackMaxSeg]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  int* abort_w = p.flags + (size_t)p.L * p.fs;
  const StackFlags F = stack_flags(p);

  if (threadIdx.x == 0) {
    bcast[0] = 0;
    bcast[1] = 0;
    for (int s = 0; s < WS; ++s) {
      mbar_init(&w_full[s], 1);
      mbar_init(&w_empty[s], 1);
    }
    for (int s = 0; s < AS; ++s) {
      mbar_init(&a_full[s], 1);
      mbar_init(&a_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(bar_q, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    for (int s = 0; s < STA; ++s) mbar_init(&bar_kv[s], 1);
    mbar_init(fin_mma, 1);
    mbar_init(fin_att, 1);
    // this CTA's segments of both projections (the same for every layer); the
    // host has checked that none needs more than kStackMaxSeg
    nseg[0] = max(0, stack_segments(cta, p.qt, p.qkbt, p.qn, segs, kStackMaxSeg));
    nseg[1] = max(0, stack_segments(cta, p.ot, p.okbt, p.on, segs + kStackMaxSeg, kStackMaxSeg));
    fence_barrier_init();
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&wq_map);
    prefetch_tmap(&wo_map);
    prefetch_tmap(&xb_map);
    prefetch_tmap(&at_map);
    prefetch_tmap(&q_map);
    prefetch_tmap(&k_map);
    prefetch_tmap(&v_map);
  }
  if (warp == 2) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nq = nseg[0], no = nseg[1];
  int nqk = 0, nok = 0;  // weight k-blocks per layer of each phase
  for (int s = 0; s < nq; ++s) nqk += segs[s].kb1 - segs[s].kb0;
  for (int s = 0; s < no; ++s) nok += segs[kStackMaxSeg + s].kb1 - segs[kStackMaxSeg + s].kb0;
  const int per_layer = nqk + nok;

  // i-th weight k-block of this CTA's stream: layer, projection, tile, k-block
  auto wblock = [&](int i, const CUtensorMap*& m, int& x, int& y, int& z) {
    const int l = i / per_layer;
    int r = i - l * per_layer;
    z = l;
    const bool o = r >= nqk;
    if (o) r -= nqk;
    m = o ? &wo_map : &wq_map;
    const StackSeg* sp = segs + (o ? kStackMaxSeg : 0);
    const int n = o ? no : nq;
    for (int s = 0; s < n; ++s) {
      const int len = sp[s].kb1 - sp[s].kb0;
      if (r < len) {
        x = (sp[s].kb0 + r) * 64;
        y = sp[s].tile * 128;
        return;
      }
      r -= len;
    }
    x = 0;
    y = 0;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ weights
    // (The weight stream reads nothing the previous kernel writes, so it
    // starts before the dependency wait; it never reads the flags, which that
    // kernel clears.  After an abort its ring waits run out and it stops.)
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const int total = p.L * per_layer;
      int pf = WS;  // next k-block to prefetch into L2 (the first WS load directly)
      int i = 0;
      bool ok = true;
      for (; i < total; ++i) {
        const int lim = min(total, i + p.lookahead);
        for (; pf < lim; ++pf) {
          const CUtensorMap* m;
          int x, y, z;
          wblock(pf, m, x, y, z);
          tma_prefetch_3d(m, x, y, z);
        }
        const int s = i % WS;
        {
          STACK_T0;
          if (!mbar_wait(&w_empty[s], ((i / WS) & 1) ^ 1, p.status)) {
            atomicExch(abort_w, 1);
            ok = false;
            break;
          }
          STACK_ACC(i / per_layer, 19);
        }
        const CUtensorMap* m;
        int x, y, z;
        wblock(i, m, x, y, z);
#ifdef DLLM_STACK_TRACE
        {
          const int r = i % per_layer;
          if (r == 0) STACK_STAMP(z, 12);
          if (r == nqk) STACK_STAMP(z, 13);
          if (r == per_layer - 1) STACK_STAMP(z, 14);
        }
#endif
        mbar_arrive_expect_tx(&w_full[s], C::kWBytes);
        tma_load_3d_hint(w_ring + s * C::kWBytes, m, &w_full[s], x, y, z, pol);
      }
      if (!ok) {  // let the loads in flight land before the CTA can exit
        for (int k = 0; k < WS && i - 1 - k >= 0; ++k) {
          const int j = i - 1 - k;
          mbar_wait(&w_full[j % WS], (j / WS) & 1, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ activations
    if (lane == 0) {
      grid_dep_wait();
      int i = 0;
      bool ok = true;
      for (int l = 0; l < p.L && ok; ++l) {
        for (int ph = 0; ph < 2 && ok; ++ph) {
          const StackSeg* sp = segs + (ph ? kStackMaxSeg : 0);
          const int n = ph ? no : nq;
          int* lf = p.flags + (size_t)l * p.fs;
          for (int s = 0; s < n && ok; ++s) {
            // the columns the segment reads: residual columns [64 kb0, 64 kb1)
            // come from O-projection tiles kb0/2 .. (kb1-1)/2 of the previous
            // layer; attention columns from the kv heads of heads kb0/2 ..
            // (kb1-1)/2 (head_dim 128) of this layer
            const int* f = nullptr;
            int nf = 0, target = 1;
            if (ph == 0) {
              if (l > 0) {
                f = lf - p.fs + (size_t)(F.odone + (sp[s].kb0 >> 1)) * kFlagStride;
                nf = ((sp[s].kb1 - 1) >> 1) - (sp[s].kb0 >> 1) + 1;
              }
            } else {
              const int v0 = (sp[s].kb0 >> 1) / p.g, v1 = ((sp[s].kb1 - 1) >> 1) / p.g;
              f = lf + (size_t)(F.adone + v0) * kFlagStride;
              nf = v1 - v0 + 1;
              target = p.batch * p.rt * p.chunks;
            }
            {
              STACK_T0;
              for (int k0 = 0; k0 < nf && ok; k0 += 32)
                ok = poll_range(f + (size_t)k0 * kFlagStride, min(32, nf - k0), target, abort_w,
                                p.status);
              STACK_ACC(l, 21);
            }
            if (!ok) break;
            if (nf > 0) fence_proxy_async_global();
            if (s == 0) STACK_STAMP(l, ph ? 4 : 0);
            for (int kb = sp[s].kb0; kb < sp[s].kb1; ++kb) {
              const int st = i % AS;
              {
                STACK_T0;
                if (!mbar_wait(&a_empty[st], ((i / AS) & 1) ^ 1, p.status)) {
                  atomicExch(abort_w, 1);
                  ok = false;
                  break;
                }
                STACK_ACC(l, 20);
              }
              mbar_arrive_expect_tx(&a_full[st], C::kXBytes);
              tma_load_3d(x_ring + st * C::kXBytes, ph ? &at_map : &xb_map, &a_full[st], kb * 64,
                          0, 0);
              ++i;
            }
          }
        }
      }
      if (!ok) {
        for (int k = 0; k < AS && i - 1 - k >= 0; ++k) {
          const int j = i - 1 - k;
          mbar_wait(&a_full[j % AS], (j / AS) & 1, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16(128, NT, 0, 0);
      int wi = 0, ai = 0, j = 0;
      bool ok = true;
      for (int l = 0; l < p.L && ok; ++l) {
        for (int ph = 0; ph < 2 && ok; ++ph) {
          const StackSeg* sp = segs + (ph ? kStackMaxSeg : 0);
          const int n = ph ? no : nq;
          for (int s = 0; s < n && ok; ++s, ++j) {
            const int acc = j & 1;
            {
              STACK_T0;
              if (!mbar_wait(&tempty[acc], ((j >> 1) & 1) ^ 1, p.status)) {
                atomicExch(abort_w, 1);
                ok = false;
                break;
              }
              STACK_ACC(l, 18);
            }
            tc_fence_after();
            const uint32_t d_tmem = tmem + acc * NT;
            for (int kb = sp[s].kb0; kb < sp[s].kb1; ++kb, ++wi, ++ai) {
              const int ws = wi % WS, as = ai % AS;
              bool got;
              {
                STACK_T0;
                got = mbar_wait(&w_full[ws], (wi / WS) & 1, p.status);
                STACK_ACC(l, 16 + 8 * ph);
              }
              {
                STACK_T0;
                got = got && mbar_wait(&a_full[as], (ai / AS) & 1, p.status);
                STACK_ACC(l, 17 + 8 * ph);
              }
              if (!got) {
                atomicExch(abort_w, 1);
                ok = false;
                break;
              }
              tc_fence_after();
              if (s == 0 && kb == sp[s].kb0) STACK_STAMP(l, ph ? 5 : 1);
              const uint32_t wa = smem_u32(w_ring + ws * C::kWBytes);
              const uint32_t xa = smem_u32(x_ring + as * C::kXBytes);
#pragma unroll
              for (int k = 0; k < 4; ++k)
                umma_bf16(d_tmem, smem_desc(wa + k * 32, 16, 1024, 2),
                          smem_desc(xa + k * 32, 16, 1024, 2), kIdesc,
                          (kb > sp[s].kb0 || k > 0) ? 1u : 0u);
              umma_commit(&w_empty[ws]);
              umma_commit(&a_empty[as]);
            }
            if (!ok) break;
            umma_commit(&tfull[acc]);
            if (s == n - 1) STACK_STAMP(l, ph ? 6 : 2);
          }
        }
      }
      // no UMMA may still be writing TMEM when it is released
      umma_commit(fin_mma);
      mbar_wait(fin_mma, 0, nullptr);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ GEMM epilogue
    grid_dep_wait();
    const int et = threadIdx.x - 128;
    const int lane_base = 32 * (warp & 3);
    const int wl = lane_base + lane;
    int j = 0;
    bool ok = true;
    for (int l = 0; l < p.L && ok; ++l) {
      int* lf = p.flags + (size_t)l * p.fs;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const StackSeg* sp = segs + (ph ? kStackMaxSeg : 0);
        const int n = ph ? no : nq;
        const GemmParams& gp = ph ? p.go : p.gq;
        const int maxc = ph ? p.omaxc : p.qmaxc;
        for (int s = 0; s < n; ++s, ++j) {
          const StackSeg sg = sp[s];
          const int acc = j & 1;
          const bool bad = !mbar_wait(&tfull[acc], (j >> 1) & 1, p.status);
          if (named_bar_or(1, 128, bad)) {
            atomicExch(abort_w, 1);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tbase = tmem + ((uint32_t)lane_base << 16) + acc * NT;
          float* part = (ph ? p.opart : p.qpart) + (size_t)sg.tile * maxc * NT * 128;
          bool last = true;
          if (sg.nc > 1) {
            // this contributor's partial, [128 weight rows][NT] fp32: each
            // thread writes its row with 16-byte stores
            float4* mine = reinterpret_cast<float4*>(part + ((size_t)sg.ci * 128 + wl) * NT);
#pragma unroll
            for (int c0 = 0; c0 < NT; c0 += 16) {
              float v[16];
              tmem_ld16(tbase + c0, v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 4; ++j)
                __stcg(mine + c0 / 4 + j,
                       make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
            }
            fence_acq_rel_gpu();
            named_bar_sync(1, 128);
            if (et == 0)
              bcast[0] = atom_acq_rel_add(lf + (size_t)((ph ? F.oarr : F.qarr) + sg.tile) * kFlagStride, 1) ==
                          sg.nc - 1;
            named_bar_sync(1, 128);
            last = bcast[0] != 0;
            if (last) fence_acq_rel_gpu();
          }
          if (last) {
            // the tile is complete: add the contributors' partials in k order
            float* inv = reinterpret_cast<float*>(run);
            if (ph == 0)
              epi_prepare<NT, EPI_QKV, true>(gp, l, 0, et, inv, reinterpret_cast<int*>(inv + NT));
#pragma unroll 1
            for (int c0 = 0; c0 < NT; c0 += 16) {
              float own[16], v[16], xo[16];
              tmem_ld16(tbase + c0, own);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = 0.f;
              // the other contributors' partials, three at a time with all
              // loads issued before the adds; the sum runs in contributor order
              for (int cb = 0; cb < sg.nc; cb += 3) {
                float4 buf[3][4];
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                  const int c = cb + q;
                  if (c < sg.nc && c != sg.ci) {
                    const float4* src = reinterpret_cast<const float4*>(
                                            part + ((size_t)c * 128 + wl) * NT + c0);
#pragma unroll
                    for (int j = 0; j < 4; ++j) buf[q][j] = __ldcg(src + j);
                  }
                }
#pragma unroll
                for (int q = 0; q < 3; ++q) {
                  const int c = cb + q;
                  if (c >= sg.nc) break;
                  if (c == sg.ci) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] += own[i];
                  } else {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                      v[4 * j] += buf[q][j].x;
                      v[4 * j + 1] += buf[q][j].y;
                      v[4 * j + 2] += buf[q][j].z;
                      v[4 * j + 3] += buf[q][j].w;
                    }
                  }
                }
              }
              if (ph == 0) {
                epi_chunk<NT, EPI_QKV>(gp, sg.tile, 0, c0, wl, et, v, xo, stage, run);
              } else {
                oproj_load_x<NT, true>(gp, sg.tile, 0, c0, wl, xo);
                epi_chunk<NT, EPI_OPROJ>(gp, sg.tile, 0, c0, wl, et, v, xo, stage, run);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
          if (last) {
            fence_acq_rel_gpu();
            fence_proxy_async_global();
            named_bar_sync(1, 128);
            if (et == 0) red_release_add(lf + (size_t)((ph ? F.odone : F.qdone) + sg.tile) * kFlagStride, 1);
            if (et == 0 && ph == 0) STACK_STAMP(l, 15);
          }
          if (et == 0 && s == n - 1) STACK_STAMP(l, ph ? 7 : 3);
        }
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ attention
    const int at = threadIdx.x - 256;  // query row of the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t s_tmem = tmem + 256;
    const uint32_t o_tmem = tmem + 384;
    constexpr uint32_t kIdescS = idesc_bf16(128, kAttKeys, 0, 0);
    constexpr uint32_t kIdescO = idesc_bf16(128, 128, 0, 1);
    const int G = (int)gridDim.x;
    // this CTA's attention unit (units are spread over the grid, one per CTA at most)
    int u = (int)(((long long)cta * p.units + G - 1) / G);
    if (u >= p.units || (int)((long long)u * G / p.units) != cta) u = -1;
    bool ok = true;
    if (u < 0) {
      grid_dep_wait();
    } else {
      const int chunk = u % p.chunks;
      int r = u / p.chunks;
      const int rti = r % p.rt;
      r /= p.rt;
      const int kvh = r % p.Hkv;
      const int b = r / p.Hkv;
      const int zq = b * p.Hkv + kvh;
      const int slot = (b * p.Hkv + kvh) * p.rt + rti;
      int sg[4];
      stack_key_segments(p, b, sg);
      const int n_tiles = (sg[1] + kAttKeys - 1) / kAttKeys + (sg[3] + kAttKeys - 1) / kAttKeys;
      const int first = chunk * p.tpc;
      const int my = max(0, min(n_tiles, first + p.tpc) - first);
      const int group_rows = p.g * p.n_rows;
      const int row = rti * 128 + at;
      const bool row_ok = row < group_rows;
      const int hl = row / p.n_rows;
      const int ii = row - hl * p.n_rows;
      const int h = kvh * p.g + hl;
      __nv_bfloat16* dst = p.attn + ((size_t)(b * p.n_rows + ii) * p.Hq + h) * 128;
      // heads of this row tile, whose q rows it reads
      const int hl0 = rti * 128 / p.n_rows;
      const int hl1 = (min(group_rows, rti * 128 + 128) - 1) / p.n_rows;
      // running counts of the single-thread issuer's barrier phases
      int kv_issued[STA], kv_done[STA];
      for (int s = 0; s < STA; ++s) kv_issued[s] = kv_done[s] = 0;
      int q_issued = 0, q_done = 0, s_cnt = 0, o_cnt = 0;
      bool gdw = false;
      for (int l = 0; l < p.L && ok; ++l) {
        int* lf = p.flags + (size_t)l * p.fs;
        const int zc = (l * p.batch + b) * p.Hkv + kvh;
        auto issue_kv = [&](int j, int start) {
          const int st = j % STA;
          mbar_arrive_expect_tx(&bar_kv[st], 2 * C::kKVBytes);
#pragma unroll
          for (int bx = 0; bx < 2; ++bx) {
            tma_load_3d(k_s + st * C::kKVBytes + bx * (kAttKeys * 128), &k_map, &bar_kv[st],
                        bx * 64, start, zc);
            tma_load_3d(v_s + st * C::kKVBytes + bx * (kAttKeys * 128), &v_map, &bar_kv[st],
                        bx * 64, start, zc);
          }
          ++kv_issued[st];
        };
        unsigned pre = 0;
        if (at == 0) {  // cache tiles this launch does not write: request them now
          for (int j = 0; j < min(my, STA); ++j) {
            int start, nv;
            key_tile64(sg, first + j, start, nv);
            if (start + kAttKeys <= p.dep_lo || start >= p.dep_hi) {
              issue_kv(j, start);
              pre |= 1u << j;
            }
          }
        }
        if (!gdw) {
          grid_dep_wait();
          gdw = true;
        }
        bool bad = false;
        if (at == 0 && my > 0) {
          // q tiles of the row tile's heads, then the k and v tiles of the kv head
          bad = !poll_range(lf + (size_t)(F.qdone + kvh * p.g + hl0) * kFlagStride, hl1 - hl0 + 1,
                            1, abort_w, p.status);
          if (!bad)
            bad = !poll_flag(lf + (size_t)(F.qdone + p.Hq + kvh) * kFlagStride, 1, abort_w,
                             p.status);
          if (!bad)
            bad = !poll_flag(lf + (size_t)(F.qdone + p.Hq + p.Hkv + kvh) * kFlagStride, 1,
                             abort_w, p.status);
          fence_proxy_async_global();
          if (!bad) {
            mbar_arrive_expect_tx(bar_q, C::kQBytes);
#pragma unroll
            for (int bx = 0; bx < 2; ++bx)
              tma_load_3d(q_s + bx * (128 * 128), &q_map, bar_q, bx * 64, rti * 128, zq);
            ++q_issued;
            for (int j = 0; j < min(my, STA); ++j) {
              if (pre & (1u << j)) continue;
              int start, nv;
              key_tile64(sg, first + j, start, nv);
              issue_kv(j, start);
            }
          }
        }
        if (named_bar_or(2, 128, bad)) {
          ok = false;
          break;
        }
        if (at == 0) STACK_STAMP(l, 8);
        // ---- key tiles of the chunk: S = Q K^T, softmax, O += P V
        float m_run = -FLT_MAX, l_run = 0.f;
        for (int j = 0; j < my; ++j) {
          const int st = j % STA;
          int kstart, nvalid;
          key_tile64(sg, first + j, kstart, nvalid);
          if (at == 0) {
            bool good = true;
            if (j == 0) {
              good = mbar_wait(bar_q, q_done & 1, p.status);
              ++q_done;
            }
            good = good && mbar_wait(&bar_kv[st], kv_done[st] & 1, p.status);
            ++kv_done[st];
            if (good) {
              tc_fence_after();
              const uint32_t qa = smem_u32(q_s);
              const uint32_t ka = smem_u32(k_s + st * C::kKVBytes);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t qo = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
                const uint32_t ko = (kk >> 2) * (kAttKeys * 128) + (kk & 3) * 32;
                umma_bf16(s_tmem, smem_desc(qa + qo, 16, 1024, 2),
                          smem_desc(ka + ko, 16, 1024, 2), kIdescS, kk > 0 ? 1u : 0u);
              }
              umma_commit(bar_s);
            } else {
              bcast[1] = 1;
            }
          }
          named_bar_sync(2, 128);
          const bool bad_s = bcast[1] != 0 || !mbar_wait(bar_s, s_cnt & 1, p.status);
          ++s_cnt;
          if (named_bar_or(2, 128, bad_s)) {
            ok = false;
            break;
          }
          tc_fence_after();
          float s[kAttKeys];
          tmem_ld32(s_tmem + lane_off, s);
          tmem_ld32(s_tmem + lane_off + 32, s + 32);
          tmem_ld_wait();
          float tm[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
          for (int i = 0; i < kAttKeys; ++i)
            if (i < nvalid) tm[i & 3] = fmaxf(tm[i & 3], s[i]);
          const float tmax = fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3]));
          const float m_new = fmaxf(m_run, tmax * p.scale_log2);
          const float alpha = fast_exp2(m_run - m_new);
          float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < kAttKeys / 8; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              const int k0 = c * 8 + i;
              const float p0 = k0 < nvalid ? fast_exp2(s[k0] * p.scale_log2 - m_new) : 0.f;
              const float p1 = k0 + 1 < nvalid ? fast_exp2(s[k0 + 1] * p.scale_log2 - m_new) : 0.f;
              const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
              ls[c & 3] += __low2float(h2) + __high2float(h2);
              pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            // row `at` of P: 64 keys = one 128-byte swizzled row
            *reinterpret_cast<uint4*>(p_s + at * 128 + (((c ^ (at & 7))) << 4)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          // O of earlier tiles is rescaled in TMEM when the running max grew
          // (the previous P V finished before this tile's S completed)
          if (j > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              float v[16];
              tmem_ld16(o_tmem + lane_off + c * 16, v);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] *= alpha;
              tmem_st16(o_tmem + lane_off + c * 16, v);
            }
            tmem_st_wait();
          }
          l_run = l_run * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
          m_run = m_new;
          fence_proxy_async_smem();
          tc_fence_before();
          named_bar_sync(2, 128);
          if (at == 0) {
            tc_fence_after();
            const uint32_t pa = smem_u32(p_s);
            const uint32_t va = smem_u32(v_s + st * C::kKVBytes);
#pragma unroll
            for (int kk = 0; kk < kAttKeys / 16; ++kk)
              umma_bf16(o_tmem, smem_desc(pa + kk * 32, 16, 1024, 2),
                        smem_desc(va + kk * 16 * 128, kAttKeys * 128, 1024, 2), kIdescO,
                        (j > 0 || kk > 0) ? 1u : 0u);
            umma_commit(bar_o);
            if (j + STA < my) {  // the stage is free once this P V has read V
              if (mbar_wait(bar_o, (o_cnt + j) & 1, p.status)) {
                int start, nv;
                key_tile64(sg, first + j + STA, start, nv);
                issue_kv(j + STA, start);
              } else {
                bcast[1] = 1;
              }
            }
          }
        }
        if (ok && my > 0) {
          const bool bad_o = !mbar_wait(bar_o, (o_cnt + my - 1) & 1, p.status);
          ok = !named_bar_or(2, 128, bad_o || bcast[1] != 0);
        }
        o_cnt += my;
        if (!ok) break;
        if (at == 0) STACK_STAMP(l, 9);
        tc_fence_after();
        // ---- output: the whole row tile, or this chunk's share of the merge
        if (p.chunks == 1) {
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            float v[16];
            tmem_ld16(o_tmem + lane_off + c * 16, v);
            tmem_ld_wait();
            if (row_ok && my > 0) {
#pragma unroll
              for (int q = 0; q < 16; q += 8) {
                uint4 w;
                __nv_bfloat162 a0 = __floats2bfloat162_rn(v[q] * inv, v[q + 1] * inv);
                __nv_bfloat162 a1 = __floats2bfloat162_rn(v[q + 2] * inv, v[q + 3] * inv);
                __nv_bfloat162 a2 = __floats2bfloat162_rn(v[q + 4] * inv, v[q + 5] * inv);
                __nv_bfloat162 a3 = __floats2bfloat162_rn(v[q + 6] * inv, v[q + 7] * inv);
                w.x = *reinterpret_cast<uint32_t*>(&a0);
                w.y = *reinterpret_cast<uint32_t*>(&a1);
                w.z = *reinterpret_cast<uint32_t*>(&a2);
                w.w = *reinterpret_cast<uint32_t*>(&a3);
                *reinterpret_cast<uint4*>(dst + c * 16 + q) = w;
              }
            }
          }
        } else {
          // unnormalised O and (max, sum) of this chunk, then the merge of
          // this chunk's columns once every chunk of the row tile has written
          const int pc = slot * p.chunks + chunk;
          const bool have = my > 0 && l_run > 0.f;
          __stcg(p.aml + (size_t)pc * 128 + at,
                 have ? make_float2(m_run, l_run) : make_float2(-FLT_MAX, 0.f));
          if (have) {  // [128 rows][128 columns] fp32, each thread its own row
            float4* ap = reinterpret_cast<float4*>(p.apart + ((size_t)pc * 128 + at) * 128);
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              float o[32];
              tmem_ld32(o_tmem + lane_off + c * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 8; ++j)
                __stcg(ap + c * 8 + j,
                       make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]));
            }
          }
          fence_acq_rel_gpu();
          named_bar_sync(2, 128);
          if (at == 0) {
            int* mf = lf + (size_t)(F.amerge + slot) * kFlagStride;
            atom_acq_rel_add(mf, 1);
            bcast[1] = poll_flag(mf, p.chunks, abort_w, p.status) ? 0 : 1;
          }
          named_bar_sync(2, 128);
          if (bcast[1] != 0) {
            ok = false;
            break;
          }
          if (at == 0) STACK_STAMP(l, 10);
          fence_acq_rel_gpu();
          // merged row = sum_c 2^(m_c - mx) O_c / sum_c 2^(m_c - mx) l_c, over
          // the chunks that saw keys, in chunk order; this chunk finishes
          // columns [d0, d0 + ds)
          const float2* ml = p.aml + (size_t)slot * p.chunks * 128 + at;
          float2 e[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            e[c] = c < p.chunks ? __ldcg(ml + c * 128) : make_float2(-FLT_MAX, 0.f);
          float mx = -FLT_MAX;
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (e[c].y > 0.f) mx = fmaxf(mx, e[c].x);
          float lt = 0.f;
#pragma unroll
          for (int c = 0; c < 16; ++c)
            if (e[c].y > 0.f) lt += fast_exp2(e[c].x - mx) * e[c].y;
          const float rl = lt > 0.f ? 1.f / lt : 0.f;
          float wgt[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) wgt[c] = e[c].y > 0.f ? fast_exp2(e[c].x - mx) * rl : 0.f;
          const int ds = 128 / p.chunks;
          constexpr int pw = 8;  // columns per pass (ds is a multiple of 8)
          const int d0 = chunk * ds;
          const float4* a0 = reinterpret_cast<const float4*>(
              p.apart + ((size_t)slot * p.chunks * 128 + at) * 128);
#pragma unroll 1
          for (int d = d0; d < d0 + ds; d += pw) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
            for (int cb = 0; cb < 16; cb += 4) {
              if (cb >= p.chunks) break;
              float4 buf[4][2];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int c = cb + q;
#pragma unroll
                for (int j = 0; j < 2; ++j)
                  if (c < p.chunks && wgt[c] > 0.f)
                    buf[q][j] = __ldcg(a0 + (size_t)c * 128 * 32 + d / 4 + j);
              }
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int c = cb + q;
                const float wc = c < p.chunks ? wgt[c] : 0.f;
                if (wc > 0.f) {
#pragma unroll
                  for (int j = 0; j < 2; ++j) {
                    acc[4 * j] += wc * buf[q][j].x;
                    acc[4 * j + 1] += wc * buf[q][j].y;
                    acc[4 * j + 2] += wc * buf[q][j].z;
                    acc[4 * j + 3] += wc * buf[q][j].w;
                  }
                }
              }
            }
            if (row_ok) {
#pragma unroll
              for (int q = 0; q < pw; q += 8) {
                uint4 w;
                __nv_bfloat162 b0 = __floats2bfloat162_rn(acc[q], acc[q + 1]);
                __nv_bfloat162 b1 = __floats2bfloat162_rn(acc[q + 2], acc[q + 3]);
                __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[q + 4], acc[q + 5]);
                __nv_bfloat162 b3 = __floats2bfloat162_rn(acc[q + 6], acc[q + 7]);
                w.x = *reinterpret_cast<uint32_t*>(&b0);
                w.y = *reinterpret_cast<uint32_t*>(&b1);
                w.z = *reinterpret_cast<uint32_t*>(&b2);
                w.w = *reinterpret_cast<uint32_t*>(&b3);
                *reinterpret_cast<uint4*>(dst + d + q) = w;
              }
            }
          }
        }
        fence_acq_rel_gpu();
        fence_proxy_async_global();
        tc_fence_before();
        named_bar_sync(2, 128);
        if (at == 0) red_release_add(lf + (size_t)(F.adone + kvh) * kFlagStride, 1);
        if (at == 0) STACK_STAMP(l, 11);
      }
      if (at == 0) {
        // after an abort: loads in flight land and UMMAs finish before exit
        for (int s = 0; s < STA; ++s)
          while (kv_done[s] < kv_issued[s]) {
            mbar_wait(&bar_kv[s], kv_done[s] & 1, nullptr);
            ++kv_done[s];
          }
        if (q_done < q_issued) mbar_wait(bar_q, q_done & 1, nullptr);
        umma_commit(fin_att);
        mbar_wait(fin_att, 0, nullptr);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  grid_dep_launch();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

#ifdef DLLM_STACK_TRACE
extern "C" int dllm_stack_trace_set(void* buf) {
  return (int)cudaMemcpyToSymbol(g_stack_trace, &buf, sizeof(buf));
}
#endif

template <int NT>
static cudaError_t launch_stack_t(const CUtensorMap* m, const StackParams& p, int grid, bool pdl,
                                  cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kStackThreads);
  cfg.dynamicSmemBytes = StackCfg<NT>::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  count_launch();
  return cudaLaunchKernelEx(&cfg, stack_kernel<NT>, m[0], m[1], m[2], m[3], m[4], m[5], m[6], p);
}

cudaError_t stack_prepare() {
  cudaError_t e = cudaFuncSetAttribute(stack_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)StackCfg<32>::kSmem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(stack_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)StackCfg<64>::kSmem);
  return e;
}

size_t stack_smem_bytes(int nt) { return nt <= 32 ? StackCfg<32>::kSmem : StackCfg<64>::kSmem; }

cudaError_t stack_occupancy(int nt, int* blocks_per_sm) {
  if (nt == 32)
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, stack_kernel<32>,
                                                         kStackThreads, StackCfg<32>::kSmem);
  return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, stack_kernel<64>,
                                                       kStackThreads, StackCfg<64>::kSmem);
}

cudaError_t launch_stack(int nt, const CUtensorMap* maps, const StackParams& p, int grid, bool pdl,
                         cudaStream_t s) {
  if (nt == 32) return launch_stack_t<32>(maps, p, grid, pdl, s);
  if (nt == 64) return launch_stack_t<64>(maps, p, grid, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace dllm
