// Non-causal GQA block attention on tcgen05.
//
// One CTA = (sequence b, kv head, tile of 128 query rows of that kv head's
// group, chunk of key tiles).  The query rows of a kv head's group are the
// g = Hq/Hkv heads x n_rows block rows, contiguous in the q buffer
// [b][Hq][n_rows][D], so a row tile is one TMA box (rows past the group are
// zero-filled).  Key/value tiles of 128 positions stream from the bf16 cache
// [L][b][Hkv][S][D] through a 2-stage TMA ring.  Per key tile:
//   S = Q K^T           UMMA M=128 (rows) N=128 (keys) into TMEM columns [0,128)
//   softmax             thread t owns query row t (TMEM lane t): running max
//                       and sum in registers, exp2 in the log2 domain, P in bf16
//                       written to shared memory in the UMMA K-major layout
//   O_tile = P V        UMMA M=128 N=D, V read MN-major straight from the TMA
//                       tile; O accumulates in registers with the usual
//                       rescaling by exp2(m_old - m_new)
// Keys outside the sequence's segments are masked inside the tile.  When a
// (row tile) is split over several key chunks, each chunk writes an
// unnormalised partial (O, max, sum) and the last chunk to finish merges them.
#include <float.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dllm {

template <int D>
struct AttnCfg {
  static constexpr int kBoxD = D >= 64 ? 64 : D;      // elements per swizzled row
  static constexpr int kRowBytes = kBoxD * 2;         // 128 or 64
  static constexpr int kSwCode = kRowBytes == 128 ? 2 : 4;
  static constexpr int kNBox = D / kBoxD;
  static constexpr int kBoxBytes = 128 * kRowBytes;   // one box of 128 rows
  static constexpr int kTileBytes = 128 * D * 2;      // Q, K or V tile of 128 rows
  static constexpr int kPBytes = 128 * 128 * 2;
  static constexpr int kStages = 2;
  static constexpr int kTmemCols = 256;
  static constexpr size_t kSmem =
      1024 + kTileBytes /*Q*/ + kStages * 2 * kTileBytes /*K,V*/ + kPBytes + 16 * 8 + 64;
};

__device__ __forceinline__ void tile_of(const int* sg, int t, int& start, int& nvalid) {
  const int n0 = (sg[1] + 127) >> 7;
  if (t < n0) {
    start = sg[0] + t * 128;
    nvalid = min(128, sg[1] - t * 128);
  } else {
    const int tt = t - n0;
    start = sg[2] + tt * 128;
    nvalid = min(128, sg[3] - tt * 128);
  }
}

template <int D>
__global__ void __launch_bounds__(128, 1)
    attn_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const AttnParams p) {
  using C = AttnCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = base;
  uint8_t* k_s = q_s + C::kTileBytes;                    // [stage]
  uint8_t* v_s = k_s + C::kStages * C::kTileBytes;       // [stage]
  uint8_t* p_s = v_s + C::kStages * C::kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p_s + C::kPBytes);
  uint64_t* bar_q = bars;
  uint64_t* bar_kv = bars + 1;  // [2]
  uint64_t* bar_s = bars + 3;
  uint64_t* bar_o = bars + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 6);
  volatile int* flags = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int t = threadIdx.x;
  const int warp = t >> 5;
  int idx = blockIdx.x;
  const int chunk = idx % p.chunks;
  idx /= p.chunks;
  const int rt = idx % p.row_tiles;
  idx /= p.row_tiles;
  const int kvh = idx % p.Hkv;
  const int b = idx / p.Hkv;

  if (t == 0) {
    mbar_init(bar_q, 1);
    mbar_init(&bar_kv[0], 1);
    mbar_init(&bar_kv[1], 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
    prefetch_tmap(&qmap);
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
  }
  __syncthreads();
  grid_dep_launch();
  grid_dep_wait();
  if (warp == 0) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t s_tmem = tmem;
  const uint32_t o_tmem = tmem + 128;

  const int* sg = p.segs + b * 4;
  const int n_tiles = ((sg[1] + 127) >> 7) + ((sg[3] + 127) >> 7);
  const int t0 = chunk * p.tiles_per_chunk;
  const int t1 = min(n_tiles, t0 + p.tiles_per_chunk);
  const int my_tiles = t1 > t0 ? t1 - t0 : 0;
  const int zc = (p.layer * p.batch + b) * p.Hkv + kvh;   // cache plane
  const int zq = b * p.Hkv + kvh;                          // q plane

  constexpr uint32_t kIdescS = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t kIdescO = idesc_bf16(128, D, 0, 1);

  auto issue_kv = [&](int j) {  // load key tile t0 + j into stage j & 1
    int start, nv;
    tile_of(sg, t0 + j, start, nv);
    const int st = j & 1;
    mbar_arrive_expect_tx(&bar_kv[st], 2 * C::kTileBytes);
#pragma unroll
    for (int bx = 0; bx < C::kNBox; ++bx) {
      tma_load_3d(k_s + st * C::kTileBytes + bx * C::kBoxBytes, &kmap, &bar_kv[st],
                  bx * C::kBoxD, start, zc);
      tma_load_3d(v_s + st * C::kTileBytes + bx * C::kBoxBytes, &vmap, &bar_kv[st],
                  bx * C::kBoxD, start, zc);
    }
  };

  if (t == 0 && my_tiles > 0) {
    mbar_arrive_expect_tx(bar_q, C::kTileBytes);
#pragma unroll
    for (int bx = 0; bx < C::kNBox; ++bx)
      tma_load_3d(q_s + bx * C::kBoxBytes, &qmap, bar_q, bx * C::kBoxD, rt * 128, zq);
    issue_kv(0);
    if (my_tiles > 1) issue_kv(1);
  }

  float o[D];
#pragma unroll
  for (int i = 0; i < D; ++i) o[i] = 0.f;
  float m_run = -FLT_MAX, l_run = 0.f;
  bool ok = true;

  for (int j = 0; j < my_tiles && ok; ++j) {
    const int st = j & 1;
    int kstart, nvalid;
    tile_of(sg, t0 + j, kstart, nvalid);
    // ---- S = Q K^T
    if (t == 0) {
      bool good = (j > 0 || mbar_wait(bar_q, 0, p.status)) &&
                  mbar_wait(&bar_kv[st], (j >> 1) & 1, p.status);
      if (good) {
        tc_fence_after();
        const uint32_t qa = smem_u32(q_s);
        const uint32_t ka = smem_u32(k_s + st * C::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk * 16 / C::kBoxD) * C::kBoxBytes + ((kk * 16) % C::kBoxD) * 2;
          umma_bf16(s_tmem, smem_desc(qa + off, 16, 8 * C::kRowBytes, C::kSwCode),
                    smem_desc(ka + off, 16, 8 * C::kRowBytes, C::kSwCode), kIdescS,
                    kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_s);
      } else {
        flags[0] = 1;
      }
    }
    const bool bad_s = !mbar_wait(bar_s, j & 1, p.status) || flags[0];
    if (__syncthreads_or(bad_s)) {
      ok = false;
      break;
    }
    tc_fence_after();
    // ---- softmax over the tile (log2 domain)
    const uint32_t lane_addr = s_tmem + ((uint32_t)(warp * 32) << 16);
    float tmax = -FLT_MAX;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float v[16];
      tmem_ld16(lane_addr + c * 16, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (c * 16 + i < nvalid) tmax = fmaxf(tmax, v[i]);
    }
    const float m_new = fmaxf(m_run, tmax * p.scale_log2);
    const float alpha = exp2f(m_run - m_new);
    float lsum = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float v[16];
      tmem_ld16(lane_addr + c * 16, v);
      tmem_ld_wait();
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const float p0 = (c * 16 + i < nvalid) ? exp2f(v[i] * p.scale_log2 - m_new) : 0.f;
        const float p1 = (c * 16 + i + 1 < nvalid) ? exp2f(v[i + 1] * p.scale_log2 - m_new) : 0.f;
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        lsum += __low2float(h2) + __high2float(h2);
        pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      // keys c*16 .. c*16+15: half (c / 4), 16-byte chunks 2*(c%4) and 2*(c%4)+1
      uint8_t* prow = p_s + (c >> 2) * (128 * 128) + t * 128;
      const int ch0 = 2 * (c & 3);
      *reinterpret_cast<uint4*>(prow + (((ch0) ^ (t & 7)) << 4)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(prow + (((ch0 + 1) ^ (t & 7)) << 4)) =
          make_uint4(pk[4], pk[5], pk[6], pk[7]);
    }
    l_run = l_run * alpha + lsum;
    m_run = m_new;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- O_tile = P V
    if (t == 0) {
      tc_fence_after();
      const uint32_t pa = smem_u32(p_s);
      const uint32_t va = smem_u32(v_s + st * C::kTileBytes);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
        const uint32_t boff = kk * 16 * C::kRowBytes;
        umma_bf16(o_tmem, smem_desc(pa + aoff, 16, 1024, 2),
                  smem_desc(va + boff, C::kBoxBytes, 8 * C::kRowBytes, C::kSwCode), kIdescO,
                  kk > 0 ? 1u : 0u);
      }
      umma_commit(bar_o);
    }
    const bool bad_o = !mbar_wait(bar_o, j & 1, p.status);
    if (__syncthreads_or(bad_o)) {
      ok = false;
      break;
    }
    tc_fence_after();
    // stage st is free again: prefetch tile j + 2 into it
    if (t == 0 && j + 2 < my_tiles) issue_kv(j + 2);
    const uint32_t o_addr = o_tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll
    for (int c = 0; c < D / 16; ++c) {
      float v[16];
      tmem_ld16(o_addr + c * 16, v);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 16; ++i) o[c * 16 + i] = o[c * 16 + i] * alpha + v[i];
    }
    tc_fence_before();
    __syncthreads();
  }

  // ---- output
  const int g = p.Hq / p.Hkv;
  const int r = rt * 128 + t;
  const bool row_ok = r < p.group_rows;
  const int hl = r / p.n_rows;
  const int ii = r - hl * p.n_rows;
  const int h = kvh * g + hl;
  auto store_row = [&](const float* vals, float inv) {
    __nv_bfloat16* dst = p.out + ((size_t)(b * p.n_rows + ii) * p.Hq + h) * D;
#pragma unroll
    for (int d0 = 0; d0 < D; d0 += 8) {
      __nv_bfloat162 q0 = __floats2bfloat162_rn(vals[d0] * inv, vals[d0 + 1] * inv);
      __nv_bfloat162 q1 = __floats2bfloat162_rn(vals[d0 + 2] * inv, vals[d0 + 3] * inv);
      __nv_bfloat162 q2 = __floats2bfloat162_rn(vals[d0 + 4] * inv, vals[d0 + 5] * inv);
      __nv_bfloat162 q3 = __floats2bfloat162_rn(vals[d0 + 6] * inv, vals[d0 + 7] * inv);
      uint4 w;
      w.x = *reinterpret_cast<uint32_t*>(&q0);
      w.y = *reinterpret_cast<uint32_t*>(&q1);
      w.z = *reinterpret_cast<uint32_t*>(&q2);
      w.w = *reinterpret_cast<uint32_t*>(&q3);
      *reinterpret_cast<uint4*>(dst + d0) = w;
    }
  };

  if (ok) {
    if (p.chunks == 1) {
      if (row_ok && l_run > 0.f) store_row(o, 1.f / l_run);
    } else {
      const size_t grp = ((size_t)(b * p.Hkv + kvh) * p.row_tiles + rt);
      const size_t prow = (grp * p.chunks + chunk) * 128 + t;
      if (row_ok) {
        float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D);
#pragma unroll
        for (int d0 = 0; d0 < D; d0 += 4)
          dst[d0 >> 2] = make_float4(o[d0], o[d0 + 1], o[d0 + 2], o[d0 + 3]);
        p.part_ml[prow] = make_float2(m_run, l_run);
      }
      __threadfence();
      __syncthreads();
      if (t == 0) {
        const int old = atomicAdd(&p.counters[grp], 1);
        const int last = old == p.chunks - 1;
        if (last) p.counters[grp] = 0;
        flags[1] = last;
      }
      __syncthreads();
      if (flags[1]) {
        __threadfence();
        if (row_ok) {
          float mx = -FLT_MAX;
          for (int c = 0; c < p.chunks; ++c) {
            const float2 ml = __ldcg(&p.part_ml[(grp * p.chunks + c) * 128 + t]);
            if (ml.y > 0.f) mx = fmaxf(mx, ml.x);
          }
          float lt = 0.f;
#pragma unroll
          for (int i = 0; i < D; ++i) o[i] = 0.f;
          for (int c = 0; c < p.chunks; ++c) {
            const size_t cr = (grp * p.chunks + c) * 128 + t;
            const float2 ml = __ldcg(&p.part_ml[cr]);
            if (!(ml.y > 0.f)) continue;
            const float w = exp2f(ml.x - mx);
            lt += w * ml.y;
            const float4* src = reinterpret_cast<const float4*>(p.part_o + cr * D);
#pragma unroll
            for (int d0 = 0; d0 < D; d0 += 4) {
              const float4 x = __ldcg(src + (d0 >> 2));
              o[d0] += w * x.x;
              o[d0 + 1] += w * x.y;
              o[d0 + 2] += w * x.z;
              o[d0 + 3] += w * x.w;
            }
          }
          if (lt > 0.f) store_row(o, 1.f / lt);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
static cudaError_t launch_attn_t(const CUtensorMap& qmap, const CUtensorMap& kmap,
                                 const CUtensorMap& vmap, const AttnParams& p, bool pdl,
                                 cudaStream_t s) {
  auto kern = attn_kernel<D>;
  const size_t smem = AttnCfg<D>::kSmem;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.batch * p.Hkv * p.row_tiles * p.chunks);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, qmap, kmap, vmap, p);
}

size_t attn_smem_bytes(int head_dim) {
  return head_dim == 128 ? AttnCfg<128>::kSmem : AttnCfg<32>::kSmem;
}

cudaError_t launch_attn(int head_dim, const CUtensorMap& qmap, const CUtensorMap& kmap,
                        const CUtensorMap& vmap, const AttnParams& p, bool pdl,
                        cudaStream_t s) {
  if (head_dim == 128) return launch_attn_t<128>(qmap, kmap, vmap, p, pdl, s);
  if (head_dim == 32) return launch_attn_t<32>(qmap, kmap, vmap, p, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace dllm
