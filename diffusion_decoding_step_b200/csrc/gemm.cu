// Weight-streaming GEMM on tcgen05 for the decode step's projections and LM head.
//
// Every projection of the step has few activation rows (b*B = 32..512) and a
// large weight matrix, so the weights are the UMMA "A" operand (M = 128 weight
// rows per tile) and the activations the "B" operand (N = NT rows):
//     D^T[wrow][xrow] = sum_k W[wrow][k] * X[xrow][k]
// with both operands K-major in shared memory (128-byte swizzle, staged by
// TMA) and the fp32 accumulator in TMEM.  A CTA (persistent over units when
// K is not split) runs three warp roles: warp 0 issues TMA loads through a
// ring of stages,
// warp 1 issues the UMMAs, warps 2-5 drain TMEM (double-buffered
// accumulator) and run one of three fused epilogues:
//   EPI_QKV    RoPE on q/k, bf16 store of q and of k/v into the cache slots
//   EPI_OPROJ  residual add in fp32, bf16 copy for the next projection
//   EPI_LMHEAD per-row running max / sum-exp / argmax / second max over the
//              CTA's vocabulary tiles; logits never leave the SM
// When (weight tiles x row tiles) would leave SMs idle, K is split: the
// splits of a tile run as one thread-block cluster, one unit per CTA.  The
// tile's 16-column chunks are dealt round robin to the ranks; each rank stages
// its fp32 partials of the chunks it does not own in its idle ring and sends
// each to its owner with one bulk copy (completing on the owner's mbarrier),
// and every owner adds the partials in rank order and runs the epilogue of
// its chunks.  The result
// does not depend on timing and no partial goes through global memory.
#include <float.h>
#include <limits.h>

#include "gemm_epi.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace dllm {

template <int NT, int EPI>
struct GemmCfg {
  // Bytes in flight per SM bound a weight stream: the LM head runs alone with
  // one CTA per SM and a deep ring.  The O-projection (one CTA per SM) takes
  // four stages (about 90 KB), which still fits beside the attention kernel
  // before it; the Q/K/V projection keeps about 70 KB per CTA so that it runs
  // two or three CTAs per SM; split across more CTAs than SMs it takes five
  // stages (about 110 KB with the receive buffer in the ring), which still fit
  // beside the O-projection and measured 1.4 % faster per LLaDA-8B-shaped step
  // than four.  (Three O-projection stages, which would let two Q/K/V CTAs
  // start beside it, measured slower; six Q/K/V stages no longer fit beside
  // it and measured 20 % slower.)
  static constexpr int kStages = EPI == EPI_LMHEAD     ? (NT <= 64 ? 8 : NT <= 128 ? 6 : 4)
                                 : EPI == EPI_OPROJ   ? 4
                                 : EPI == EPI_QKV_DEEP ? (NT <= 64 ? 5 : 4)
                                                      : (NT <= 64 ? 3 : 4);
  static constexpr int kWBytes = 128 * 64 * 2;
  static constexpr int kXBytes = NT * 64 * 2;
  static constexpr int kTmemCols = 2 * NT;
  static constexpr int kChunk = 16;
  // Split-K partials received from the other ranks of a cluster: [src slot
  // (splits - 1)][owned chunk][128 lanes][16 fp32]; splits <= 4 for NT 32 and
  // <= 3 for NT 64 (two owned chunks at most).
  static constexpr int kRecvSlots = NT <= 32 ? 3 : 2;
  static constexpr int kRecvOwn = NT <= 32 ? 1 : 2;
  static constexpr int kRecvBytes =
      (NT <= 64 && EPI != EPI_LMHEAD) ? kRecvSlots * kRecvOwn * 128 * 64 : 0;
  // the receive buffer sits last, so a launch that keeps it in the (then
  // idle) weight ring simply asks for kSmemBase bytes
  static constexpr size_t kSmemBase = 1024 + (size_t)kStages * (kWBytes + kXBytes) +
                                      kChunk * 128 * 4 + NT * sizeof(LmStat) +
                                      (2 * kStages + 4) * 8 + 64;
  static constexpr size_t kSmem = kSmemBase + kRecvBytes;
  static_assert(kSmem <= 227 * 1024, "GEMM shared memory");
  // split-K staging of the chunks a rank sends, after the receive buffer when
  // that sits in the ring
  static_assert(NT > 64 || EPI == EPI_LMHEAD ||
                    kRecvBytes + (NT / 16) * 128 * 16 * 4 <= kStages * (kWBytes + kXBytes),
                "split-K staging must fit in the ring");
};

__device__ __forceinline__ void decode_unit(const GemmParams& p, int u, int& m, int& n, int& tile,
                                            int& kb0, int& kb1) {
  tile = u / p.splits;
  const int sp = u - tile * p.splits;
  m = tile / p.n_tiles;
  n = tile - m * p.n_tiles;
  kb0 = sp * p.kb_per_split;
  kb1 = min(p.K / 64, kb0 + p.kb_per_split);
}

// CTAs per SM the register budget is sized for.  The O-projection runs one
// CTA per SM (its ring and receive buffer), so its NT = 32 variant may take
// the registers of two; the Q/K/V projection runs two or three per SM.
template <int NT, int EPI>
constexpr int gemm_min_blocks() {
  return (EPI == EPI_OPROJ && NT <= 32) ? 2 : NT <= 32 ? 3 : NT <= 64 ? 2 : 1;
}

// CW: width of the split-K chunks dealt to a cluster's ranks (16 columns,
// or 8 so that all ranks of a 3- or 4-way split of a 32-column tile own one).
template <int NT, int EPI, int CW>
__global__ void __launch_bounds__(192, gemm_min_blocks<NT, EPI>())
    gemm_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap,
                const GemmParams p) {
  using C = GemmCfg<NT, EPI>;
  static_assert(CW == 16 || (CW == 8 && NT == 32 && EPI != EPI_LMHEAD), "chunk width");
  constexpr int ST = C::kStages;
  constexpr int kEpi = EPI == EPI_QKV_DEEP ? EPI_QKV : EPI;  // epilogue kind
  constexpr uint32_t kIdesc = idesc_bf16(128, NT, 0, 0);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* w_st = base;
  uint8_t* x_st = w_st + ST * C::kWBytes;
  float* stage = reinterpret_cast<float*>(x_st + ST * C::kXBytes);
  LmStat* run = reinterpret_cast<LmStat*>(stage + C::kChunk * 128);
  uint64_t* full = reinterpret_cast<uint64_t*>(run + NT);
  uint64_t* empty = full + ST;
  uint64_t* tfull = empty + ST;
  uint64_t* tempty = tfull + 2;
  // dep_bar: one thread passes the programmatic-dependency wait and releases
  // the others through it (they sleep instead of polling beside the kernel
  // still running on this SM)
  uint64_t* dep_bar = tempty + 2;
  uint64_t* red_bar = dep_bar + 1;  // split-K partials received from the cluster
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(red_bar + 1);
  // split-K receive buffer: its own region when the launch has one CTA per SM
  // at most, else the weight ring once every mainloop of the cluster is done
  float* recv = p.recv_in_ring ? reinterpret_cast<float*>(w_st)
                               : reinterpret_cast<float*>(base + C::kSmemBase - 1024);
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [0] abort, [1] last

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Split K is reduced inside a thread-block cluster for decode tiles.
  constexpr bool kClusterSplit = NT <= 64;
  float part[kClusterSplit ? NT : 1];
  // CW-column chunks of a split tile are dealt round robin to the cluster's
  // ranks; at most kOwnMax per rank (splits >= 2)
  constexpr int kNChunk = NT / CW;
  constexpr int kOwnMax = kClusterSplit ? (kNChunk + 1) / 2 : 1;
  float xpre[kOwnMax][CW];
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(dep_bar, 1);
    mbar_init(red_bar, 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
  }
  for (int c = threadIdx.x; c < NT; c += blockDim.x) {
    run[c].m = -FLT_MAX;
    run[c].s = 0.f;
    run[c].m2 = -FLT_MAX;
    run[c].idx = INT_MAX;
  }
  if (threadIdx.x == 32) {
    prefetch_tmap(&wmap);
    prefetch_tmap(&xmap);
  }
  __syncthreads();
  if constexpr (kClusterSplit) {
    if (p.splits > 1) {
      // Owners of split-K chunks expect the other ranks' partials; the
      // cluster barrier (waited for in the tail) publishes the armed barriers.
      const int rank = (int)cluster_ctarank();
      const int owned = (kNChunk - rank + p.splits - 1) / p.splits;
      if (threadIdx.x == 0 && owned > 0)
        mbar_arrive_expect_tx(red_bar, (uint32_t)((p.splits - 1) * owned * 128 * CW * 4));
      cluster_arrive_relaxed();
    }
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      // The weights do not depend on the previous kernel: the first stages of
      // the first unit are requested before waiting for it to finish.
      int pre = 0, pre_kb0 = 0, pre_n = 0;
      if ((int)blockIdx.x < p.units) {
        int m, n, tile, kb0, kb1;
        decode_unit(p, blockIdx.x, m, n, tile, kb0, kb1);
        pre = min(ST, kb1 - kb0);
        pre_kb0 = kb0;
        pre_n = n;
        for (int i = 0; i < pre; ++i) {
          mbar_arrive_expect_tx(&full[i], C::kWBytes + C::kXBytes);
          tma_load_3d_hint(w_st + i * C::kWBytes, &wmap, &full[i], (kb0 + i) * 64, m * 128,
                           p.layer, pol_w);
        }
      }
      grid_dep_wait();
      mbar_arrive(dep_bar);
      for (int i = 0; i < pre; ++i)
        tma_load_3d(x_st + i * C::kXBytes, &xmap, &full[i], ((pre_kb0 + i) % p.kx_blocks) * 64,
                    pre_n * NT, 0);
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        int m, n, tile, kb0, kb1;
        decode_unit(p, u, m, n, tile, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          if (it < pre) continue;  // issued before the dependency wait
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.status) || flags[0]) {
            flags[0] = 1;
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], C::kWBytes + C::kXBytes);
          tma_load_3d_hint(w_st + s * C::kWBytes, &wmap, &full[s], kb * 64, m * 128, p.layer,
                           pol_w);
          tma_load_3d(x_st + s * C::kXBytes, &xmap, &full[s], (kb % p.kx_blocks) * 64, n * NT,
                      0);
        }
      }
      // Before leaving after an abort, let loads already in flight land.
      if (!ok) {
        for (int k = 0; k < ST && it - 1 - k >= 0; ++k) {
          const int j = it - 1 - k;
          mbar_wait(&full[j % ST], (j / ST) & 1, nullptr);
        }
      }
    } else {
      // lanes 1..31 warm L2 for a later kernel while the weights stream
      l2_prefetch_share(p.pf, blockIdx.x, gridDim.x, lane - 1, 31);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    mbar_wait_sleep(dep_bar, 0, p.status);
    tmem_alloc(tmem_slot, C::kTmemCols);
    tc_fence_before();
    named_bar_sync(2, 160);
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (lane == 0) {
      int it = 0, j = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++j) {
        int m, n, tile, kb0, kb1;
        decode_unit(p, u, m, n, tile, kb0, kb1);
        const int acc = j & 1;
        const uint32_t aph = (j >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1, p.status) || flags[0]) {
          flags[0] = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * NT;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % ST;
          const uint32_t ph = (it / ST) & 1;
          if (!mbar_wait(&full[s], ph, p.status) || flags[0]) {
            flags[0] = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t wa = smem_u32(w_st + s * C::kWBytes);
          const uint32_t xa = smem_u32(x_st + s * C::kXBytes);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            umma_bf16(d_tmem, smem_desc(wa + k * 32, 16, 1024, 2),
                      smem_desc(xa + k * 32, 16, 1024, 2), kIdesc,
                      (kb > kb0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    mbar_wait_sleep(dep_bar, 0, p.status);
    named_bar_sync(2, 160);
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int et = threadIdx.x - 64;         // 0..127
    const int lane_base = 32 * (warp & 3);   // TMEM lanes this warp may access
    const int wl = lane_base + lane;         // weight row within the tile
    int j = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++j) {
      int m, n, tile, kb0, kb1;
      decode_unit(p, u, m, n, tile, kb0, kb1);
      const int acc = j & 1;
      const uint32_t aph = (j >> 1) & 1;
      float* inv = reinterpret_cast<float*>(run);
      epi_prepare<NT, kEpi>(p, p.layer, n, et, inv, reinterpret_cast<int*>(inv + NT));
      if constexpr (kClusterSplit && kEpi == EPI_OPROJ) {
        if (p.splits > 1) {  // residual rows of the chunks this rank will finish
          const int rank = (int)cluster_ctarank();
#pragma unroll
          for (int lq = 0; lq < kOwnMax; ++lq) {
            const int q = lq * p.splits + rank;
            if (q < kNChunk) oproj_load_x<NT, false, CW>(p, m, n, q * CW, wl, xpre[lq]);
          }
        }
      }
      const bool bad = !mbar_wait(&tfull[acc], aph, p.status) || flags[0];
      if (named_bar_or(1, 128, bad)) {
        flags[0] = 1;
        break;
      }
      tc_fence_after();
      if constexpr (kClusterSplit) {
        if (p.splits > 1) {
          // cluster split-K: keep this CTA's partial for the reduction below
#pragma unroll
          for (int c0 = 0; c0 < NT; c0 += 16) {
            float v[16];
            tmem_ld16(tmem + ((uint32_t)lane_base << 16) + acc * NT + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) part[c0 + i] = v[i];
          }
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
          continue;
        }
      }
      for (int c0 = 0; c0 < NT; c0 += 16) {
        float v[16], xo[16];
        if constexpr (kEpi == EPI_OPROJ) oproj_load_x<NT>(p, m, n, c0, wl, xo);
        tmem_ld16(tmem + ((uint32_t)lane_base << 16) + acc * NT + c0, v);
        tmem_ld_wait();
        epi_chunk<NT, kEpi, 16>(p, m, n, c0, wl, et, v, xo, stage, run);
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
    if constexpr (kEpi == EPI_LMHEAD) {
      named_bar_sync(1, 128);
      const int n = blockIdx.x % p.n_tiles;
      const int slot = blockIdx.x / p.n_tiles;
      for (int c = et; c < NT; c += 128) {
        const int xrow = n * NT + c;
        if (xrow < p.R) p.stats[(size_t)xrow * p.stat_slots + slot] = run[c];
      }
    }
  }
  __syncthreads();
  // Every mainloop of this CTA is done: the next kernel may start loading
  // its weights during the reduction and epilogue below.
  grid_dep_launch();
  if constexpr (kClusterSplit) {
    if (p.splits > 1) {
      // The splits of a tile form one cluster (one unit per CTA).  The tile's
      // CW-column chunks are dealt round robin to the ranks; every rank sends
      // its partial of each chunk it does not own to the owner's receive
      // buffer with a bulk copy (the bytes complete on the owner's red_bar), and
      // each owner adds the partials of its chunks in rank order and runs
      // their epilogue.  The final cluster barrier keeps every CTA alive
      // until the transfers into it have landed.
      cluster_wait();
      if (p.recv_in_ring) {  // the owners' rings must be idle before they receive
        cluster_arrive();
        cluster_wait();
      }
      const int rank = (int)cluster_ctarank();
      const bool epi = warp >= 2;
      const int et = threadIdx.x - 64;
      const int wl = 32 * (warp & 3) + (threadIdx.x & 31);
      const int sp = p.splits;
      const int own = (kNChunk + sp - 1) / sp;  // chunk slots per owner
      // float4 j of a lane's chunk row sits at j ^ sw (bank spread of the staging stores)
      const int sw = CW == 16 ? (wl >> 1) & 3 : (wl >> 2) & 1;
      if (epi) {
        // Each chunk this rank does not own is staged in the (idle) ring in
        // the owner's layout, then sent with one bulk copy.
        float* stg = reinterpret_cast<float*>(w_st + (p.recv_in_ring ? C::kRecvBytes : 0));
        int k = 0;
#pragma unroll
        for (int q = 0; q < kNChunk; ++q) {
          if (q % sp == rank) continue;
          float4* row = reinterpret_cast<float4*>(stg + ((size_t)k * 128 + wl) * CW);
#pragma unroll
          for (int j = 0; j < CW / 4; ++j)
            row[j ^ sw] = make_float4(part[q * CW + 4 * j], part[q * CW + 4 * j + 1],
                                      part[q * CW + 4 * j + 2], part[q * CW + 4 * j + 3]);
          ++k;
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (et == 0) {
          k = 0;
#pragma unroll
          for (int q = 0; q < kNChunk; ++q) {
            const int owner = q % sp;
            if (owner == rank) continue;
            const int slot = rank < owner ? rank : rank - 1;
            const uint32_t dst = map_to_rank(
                smem_u32(recv + (size_t)(slot * own + q / sp) * 128 * CW), (uint32_t)owner);
            bulk_copy_to_cluster(dst, smem_u32(stg + (size_t)k * 128 * CW), 128 * CW * 4,
                                 map_to_rank(smem_u32(red_bar), (uint32_t)owner));
            ++k;
          }
        }
      }
      // The closing cluster barrier only keeps every CTA alive until the
      // partials sent to it have landed; the partials themselves are ordered
      // by red_bar, so the arrivals need no release.
      if (epi && rank < kNChunk) {
        const bool got = mbar_wait_cluster(red_bar, 0, p.status);
        cluster_arrive_relaxed();
        if (got && !flags[0]) {
          int m, n, tile, kb0, kb1;
          decode_unit(p, blockIdx.x, m, n, tile, kb0, kb1);
#pragma unroll
          for (int lq = 0; lq < kOwnMax; ++lq) {
            const int q = lq * sp + rank;
            if (q >= kNChunk) break;
            float mine[CW];
#pragma unroll
            for (int qq = 0; qq < kNChunk; ++qq)
              if (qq == q) {
#pragma unroll
                for (int i = 0; i < CW; ++i) mine[i] = part[qq * CW + i];
              }
            float v[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) v[i] = 0.f;
            for (int r = 0; r < sp; ++r) {
              if (r == rank) {
#pragma unroll
                for (int i = 0; i < CW; ++i) v[i] += mine[i];
                continue;
              }
              const int slot = r < rank ? r : r - 1;
              const float4* src = reinterpret_cast<const float4*>(
                  recv + ((size_t)(slot * own + lq) * 128 + wl) * CW);
#pragma unroll
              for (int j = 0; j < CW / 4; ++j) {
                const float4 x = src[j ^ sw];
                v[4 * j] += x.x;
                v[4 * j + 1] += x.y;
                v[4 * j + 2] += x.z;
                v[4 * j + 3] += x.w;
              }
            }
            epi_chunk<NT, kEpi, CW>(p, m, n, q * CW, wl, et, v, xpre[lq], stage, run);
          }
        }
      } else {
        cluster_arrive_relaxed();
      }
      cluster_wait();
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, C::kTmemCols);
  }
}

template <int NT, int EPI, int CW = 16>
static cudaError_t launch_t(const CUtensorMap& wmap, const CUtensorMap& xmap, const GemmParams& p,
                            int grid, bool pdl, cudaStream_t s) {
  auto kern = gemm_kernel<NT, EPI, CW>;
  const size_t smem = p.recv_in_ring ? GemmCfg<NT, EPI>::kSmemBase : GemmCfg<NT, EPI>::kSmem;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (p.splits > 1) {
    if (NT > 64 || grid != p.units) return cudaErrorInvalidValue;
    if (p.recv_in_ring &&
        (size_t)GemmCfg<NT, EPI>::kStages * GemmCfg<NT, EPI>::kWBytes < GemmCfg<NT, EPI>::kRecvBytes)
      return cudaErrorInvalidValue;
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.splits;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, wmap, xmap, p);
}

// Opt every kernel variant into its dynamic shared memory size up front, so
// that no attribute call happens while a launch sequence is being captured.
cudaError_t gemm_prepare() {
  cudaError_t e = cudaSuccess;
#define DLLM_SET(NT, EPI, CW)                                             \
  if (e == cudaSuccess)                                                  \
    e = cudaFuncSetAttribute(gemm_kernel<NT, EPI, CW>,                   \
                             cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             (int)GemmCfg<NT, EPI>::kSmem);
  DLLM_SET(32, 0, 16) DLLM_SET(32, 1, 16) DLLM_SET(32, 2, 16) DLLM_SET(32, 3, 16)
  DLLM_SET(32, 0, 8) DLLM_SET(32, 1, 8) DLLM_SET(32, 3, 8)
  DLLM_SET(64, 0, 16) DLLM_SET(64, 1, 16) DLLM_SET(64, 2, 16) DLLM_SET(64, 3, 16)
  DLLM_SET(128, 0, 16) DLLM_SET(128, 1, 16) DLLM_SET(128, 2, 16)
  DLLM_SET(256, 0, 16) DLLM_SET(256, 1, 16) DLLM_SET(256, 2, 16)
#undef DLLM_SET
  return e;
}


template <int EPI>
static cudaError_t launch_e(int nt, const CUtensorMap& wmap, const CUtensorMap& xmap,
                            const GemmParams& p, int grid, bool pdl, cudaStream_t s) {
  // 3- and 4-way splits of a 32-column tile deal 8-column chunks, so that
  // every rank owns part of the reduction and the epilogue
  if constexpr (EPI != EPI_LMHEAD)
    if (nt == 32 && p.splits >= 3) return launch_t<32, EPI, 8>(wmap, xmap, p, grid, pdl, s);
  if constexpr (EPI == EPI_QKV_DEEP) {
    switch (nt) {
      case 32: return launch_t<32, EPI>(wmap, xmap, p, grid, pdl, s);
      case 64: return launch_t<64, EPI>(wmap, xmap, p, grid, pdl, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (nt) {
    case 32: return launch_t<32, EPI>(wmap, xmap, p, grid, pdl, s);
    case 64: return launch_t<64, EPI>(wmap, xmap, p, grid, pdl, s);
    case 128: return launch_t<128, EPI>(wmap, xmap, p, grid, pdl, s);
    case 256: return launch_t<256, EPI>(wmap, xmap, p, grid, pdl, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(int epi, int nt, const CUtensorMap& wmap, const CUtensorMap& xmap,
                        const GemmParams& p, int grid, bool pdl, cudaStream_t s) {
  switch (epi) {
    case EPI_QKV: return launch_e<EPI_QKV>(nt, wmap, xmap, p, grid, pdl, s);
    case EPI_OPROJ: return launch_e<EPI_OPROJ>(nt, wmap, xmap, p, grid, pdl, s);
    case EPI_LMHEAD: return launch_e<EPI_LMHEAD>(nt, wmap, xmap, p, grid, pdl, s);
    case EPI_QKV_DEEP: return launch_e<EPI_QKV_DEEP>(nt, wmap, xmap, p, grid, pdl, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dllm
