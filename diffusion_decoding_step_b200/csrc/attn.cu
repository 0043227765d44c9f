// Non-causal GQA block attention on tcgen05.
//
// One CTA = (sequence b, kv head, tile of query rows of that kv head's
// group, chunk of key tiles).  The query rows of a kv head's group are the
// g = Hq/Hkv heads x n_rows block rows, contiguous in the q buffer
// [b][Hq][n_rows][D], so a row tile is one TMA box (rows past the group are
// zero-filled).  Key/value tiles of 128 positions stream from the bf16 cache
// [L][b][Hkv][S][D] through a TMA ring of ST stages.  Per key tile:
//   S = Q K^T      UMMA M=128 (rows) x N=128 (keys) into TMEM columns [0,128)
//   softmax        the row is read from TMEM once, max and sum run in
//                  registers in the log2 domain, P goes to shared memory in
//                  bf16 in the UMMA K-major layout
//   O += P V       UMMA M=128 x N=D into TMEM columns [128,128+D); V is read
//                  MN-major straight from its TMA tile.  O stays in TMEM; a
//                  row is rescaled there only when its running max grows.
// Key tiles that the preceding kernel does not write (everything outside
// [dep_lo, dep_hi)) are requested before the programmatic-dependency wait,
// so for a decode step the prefix/suffix cache is already in flight while the
// Q/K/V projection finishes.  Keys outside the sequence's segments are
// masked inside the tile.  When a row tile is split over several key
// chunks, the chunks run as one thread-block cluster: every CTA sends its
// rows' (max, sum) to all others through distributed shared memory, scales
// its O by its share of the merged softmax and sends each 16-column group to
// the CTA that owns the group, which adds the chunks' contributions in chunk
// order and writes the bf16 output.  No partial goes through global memory.
//
// Two row-tile shapes:
// - 128 rows, 8 warps: threads t and t+128 share TMEM lane t % 128 (a warp
//   reaches lanes 32(w % 4)..); each takes one 64-key half of the row in the
//   softmax (the row max crosses the halves through shared memory) and the
//   same half of the output columns.  K and V complete on separate barriers,
//   and S of the next key tile is issued at the row-max barrier, once every
//   thread holds this tile's S in registers, so it overlaps the softmax.
// - 32 rows (SG, head_dim 128, 4 warps): the 32 rows are loaded four times
//   into the 128-row Q tile, so S holds each row in four TMEM lanes 32w + i,
//   one per warp w.  Warp w takes keys [32w, 32w+32) of every row in the
//   softmax (the row max is exchanged once per tile through shared memory)
//   and writes its quarter of P into all four copies of the row, so every
//   lane of O = P V holds its full row and warp w reads, scales and stores
//   output columns [32w, 32w+32).
#include <float.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dllm {

constexpr int kKeys = 128;     // keys per tile
constexpr int kMaxMerge = 8;   // key chunks (cluster size) per row tile

template <int D, int ST>
struct AttnCfg {
  static constexpr int kBoxD = D >= 64 ? 64 : D;      // elements per swizzled row
  static constexpr int kRowBytes = kBoxD * 2;         // 128 or 64
  static constexpr int kSwCode = kRowBytes == 128 ? 2 : 4;
  static constexpr int kNBox = D / kBoxD;
  static constexpr int kBoxBytes = 128 * kRowBytes;   // one box of 128 rows (Q or keys)
  static constexpr int kQBytes = 128 * D * 2;
  static constexpr int kKVBytes = kKeys * D * 2;      // K or V tile
  static constexpr int kPBytes = 128 * kKeys * 2;     // two 128B-swizzle atom columns
  static constexpr int kTmemCols = 256;               // S [0,128), O [128,128+D)
  static constexpr int kMlBytes = kMaxMerge * 128 * 8;  // (max, sum) of every chunk's rows
  static constexpr int kXBytes = 2 * 128 * 4;  // small groups: quarter maxima and sums
  static constexpr size_t kSmem =
      1024 + kQBytes + ST * 2 * kKVBytes + kPBytes + kMlBytes + kXBytes + 128 + 64;
  // The merge reuses the K/V/P region once every chunk's last P V is done:
  // [src chunk][owned group][4 float4][128 rows] fp32 for up to kMaxMerge chunks.
  static constexpr int kGroups = D / 16;
  static constexpr int kRegion = ST * 2 * kKVBytes + kPBytes;
};

template <int D>
constexpr int merge_bytes(int n) {
  return n * ((D / 16 + n - 1) / n) * 4 * 128 * 16;
}
static_assert(merge_bytes<128>(2) <= AttnCfg<128, 1>::kRegion &&
                  merge_bytes<128>(3) <= AttnCfg<128, 1>::kRegion &&
                  merge_bytes<128>(4) <= AttnCfg<128, 1>::kRegion &&
                  merge_bytes<128>(5) <= AttnCfg<128, 1>::kRegion &&
                  merge_bytes<128>(6) <= AttnCfg<128, 1>::kRegion &&
                  merge_bytes<128>(8) <= AttnCfg<128, 1>::kRegion &&
                  merge_bytes<32>(2) <= AttnCfg<32, 1>::kRegion &&
                  merge_bytes<32>(3) <= AttnCfg<32, 1>::kRegion &&
                  merge_bytes<32>(4) <= AttnCfg<32, 1>::kRegion &&
                  merge_bytes<32>(5) <= AttnCfg<32, 1>::kRegion &&
                  merge_bytes<32>(6) <= AttnCfg<32, 1>::kRegion,
              "the chunk merge buffer must fit in the K/V/P region");

// Key segments (start, len) x 2 of sequence b: given explicitly, or derived
// from the cache mode, the block and the sequence start.
__device__ __forceinline__ void seq_segments(const AttnParams& p, int b, int* sg) {
  if (p.segs != nullptr) {
#pragma unroll
    for (int i = 0; i < 4; ++i) sg[i] = p.segs[b * 4 + i];
    return;
  }
  const int st = p.seq_start[b];
  const int end = (p.seq_blk ? p.seq_blk[b] : p.blk_start) + p.blk_len;
  int l0, s1 = 0, l1 = 0;
  if (p.seg_end > 0) {
    l0 = p.seg_end - st;
  } else if (p.mode == 2 || p.mode == 4) {  // DUAL, PREFIX_SUFFIXQ
    l0 = p.S - st;
  } else if (p.mode == 3) {  // DUAL_PRUNED
    const int wend = min(end + p.window, p.S);
    l0 = wend - st;
    if (end < p.S && p.S - 1 >= wend) {
      s1 = p.S - 1;
      l1 = 1;
    }
  } else {  // NONE, PREFIX
    l0 = end - st;
  }
  sg[0] = st;
  sg[1] = l0 > 0 ? l0 : 0;
  sg[2] = s1;
  sg[3] = l1;
}

__device__ __forceinline__ void tile_of(const int* sg, int t, int& start, int& nvalid) {
  const int n0 = (sg[1] + kKeys - 1) / kKeys;
  if (t < n0) {
    start = sg[0] + t * kKeys;
    nvalid = min(kKeys, sg[1] - t * kKeys);
  } else {
    const int tt = t - n0;
    start = sg[2] + tt * kKeys;
    nvalid = min(kKeys, sg[3] - tt * kKeys);
  }
}

template <int D, int ST, bool SG>
__global__ void __launch_bounds__(SG ? 128 : 256, 1)
    attn_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const AttnParams p) {
  using C = AttnCfg<D, ST>;
  static_assert(!SG || D == 128, "small groups: one 32-key quarter and 32 columns per warp");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_s = base;
  uint8_t* k_s = q_s + C::kQBytes;                 // [ST]
  uint8_t* v_s = k_s + ST * C::kKVBytes;           // [ST]
  uint8_t* p_s = v_s + ST * C::kKVBytes;
  float2* ml_s = reinterpret_cast<float2*>(p_s + C::kPBytes);  // [kMaxMerge][128]
  float* x_s = reinterpret_cast<float*>(p_s + C::kPBytes + C::kMlBytes);  // [2][4 warps][32]
  uint64_t* bars = reinterpret_cast<uint64_t*>(p_s + C::kPBytes + C::kMlBytes + C::kXBytes);
  uint64_t* bar_q = bars;
  uint64_t* bar_s = bars + 1;
  uint64_t* bar_o = bars + 2;
  uint64_t* bar_k = bars + 3;       // [ST]
  uint64_t* bar_v = bars + 3 + ST;  // [ST]
  uint64_t* dep_bar = bars + 3 + 2 * ST;  // thread 0 passes the dependency wait, the rest sleep
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 + 2 * ST);
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
  const int zc = (p.layer * p.batch + b) * p.Hkv + kvh;  // cache plane
  const int zq = b * p.Hkv + kvh;                         // q plane

  if (t == 0) {
    mbar_init(bar_q, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(&bar_k[s], 1);
      mbar_init(&bar_v[s], 1);
    }
    mbar_init(dep_bar, 1);
    flags[0] = 0;
    flags[1] = 0;
    fence_barrier_init();
    prefetch_tmap(&qmap);
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
  }
  __syncthreads();

  // Segments come from the sequence start (an input of the step) unless an
  // explicit list is given, which may be produced by earlier kernels.
  int sg[4] = {0, 0, 0, 0};
  if (p.segs == nullptr) seq_segments(p, b, sg);

  // Key tile t0 + j into stage j % ST.  On 128-row tiles K and V complete
  // on separate barriers: a K stage is refilled as soon as its S = Q K^T is
  // done, its V stage once P V is done.  32-row tiles load both on bar_k and
  // refill the stage once P V is done.
  constexpr bool kSplitKV = !SG;
  auto issue_k = [&](int j, int start) {
    const int st = j % ST;
    mbar_arrive_expect_tx(&bar_k[st], C::kKVBytes);
#pragma unroll
    for (int bx = 0; bx < C::kNBox; ++bx)
      tma_load_3d(k_s + st * C::kKVBytes + bx * C::kBoxBytes, &kmap, &bar_k[st],
                  bx * C::kBoxD, start, zc);
  };
  auto issue_v = [&](int j, int start) {
    const int st = j % ST;
    mbar_arrive_expect_tx(&bar_v[st], C::kKVBytes);
#pragma unroll
    for (int bx = 0; bx < C::kNBox; ++bx)
      tma_load_3d(v_s + st * C::kKVBytes + bx * C::kBoxBytes, &vmap, &bar_v[st],
                  bx * C::kBoxD, start, zc);
  };
  auto issue_kv = [&](int j, int start) {
    if constexpr (kSplitKV) {
      issue_k(j, start);
      issue_v(j, start);
    } else {
      const int st = j % ST;
      mbar_arrive_expect_tx(&bar_k[st], 2 * C::kKVBytes);
#pragma unroll
      for (int bx = 0; bx < C::kNBox; ++bx) {
        tma_load_3d(k_s + st * C::kKVBytes + bx * C::kBoxBytes, &kmap, &bar_k[st],
                    bx * C::kBoxD, start, zc);
        tma_load_3d(v_s + st * C::kKVBytes + bx * C::kBoxBytes, &vmap, &bar_k[st],
                    bx * C::kBoxD, start, zc);
      }
    }
  };
  auto chunk_range = [&](int& first, int& n) {
    const int n_tiles = (sg[1] + kKeys - 1) / kKeys + (sg[3] + kKeys - 1) / kKeys;
    first = chunk * p.tiles_per_chunk;
    const int last = min(n_tiles, first + p.tiles_per_chunk);
    n = last > first ? last - first : 0;
  };

  unsigned pre = 0;  // stages requested before the dependency wait
  // key positions the preceding kernel writes: this sequence's query rows
  const int dep_lo = p.seq_blk ? p.seq_blk[b] : p.dep_lo;
  const int dep_hi = p.seq_blk ? p.seq_blk[b] + p.n_rows : p.dep_hi;
  if (t == 0 && p.segs == nullptr) {
    int first, n;
    chunk_range(first, n);
    for (int j = 0; j < min(n, ST); ++j) {
      int start, nv;
      tile_of(sg, first + j, start, nv);
      if (start + kKeys <= dep_lo || start >= dep_hi) {
        issue_kv(j, start);
        pre |= 1u << j;
      }
    }
  }
  if (warp == 3) l2_prefetch_share(p.pf, blockIdx.x, gridDim.x, t - 96, 32);
  if (t == 0) {
    grid_dep_wait();
    mbar_arrive(dep_bar);
  } else {
    mbar_wait_sleep(dep_bar, 0, p.status);
  }
  if (p.segs != nullptr) seq_segments(p, b, sg);
  int t0, my_tiles;
  chunk_range(t0, my_tiles);

  if (warp == 0) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t s_tmem = tmem;
  const uint32_t o_tmem = tmem + 128;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;  // a warp reads lanes 32(w%4)..
  // 128-row tiles run 8 warps: thread t holds row t % 128 and key half
  // t / 128 in the softmax, and the same half of the output columns.
  const int half = SG ? 0 : t >> 7;
  const int trow = t & 127;

  constexpr uint32_t kIdescS = idesc_bf16(128, kKeys, 0, 0);
  constexpr uint32_t kIdescO = idesc_bf16(128, D, 0, 1);

  if (t == 0 && my_tiles > 0) {
    mbar_arrive_expect_tx(bar_q, C::kQBytes);
#pragma unroll
    for (int bx = 0; bx < C::kNBox; ++bx) {
      if constexpr (SG) {  // four copies of the (at most) 32 rows; the map's box is 32 rows
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tma_load_3d(q_s + bx * C::kBoxBytes + c * 32 * C::kRowBytes, &qmap, bar_q,
                      bx * C::kBoxD, rt * 32, zq);
      } else {
        tma_load_3d(q_s + bx * C::kBoxBytes, &qmap, bar_q, bx * C::kBoxD, rt * 128, zq);
      }
    }
    for (int j = 0; j < min(my_tiles, ST); ++j) {
      if (pre & (1u << j)) continue;
      int start, nv;
      tile_of(sg, t0 + j, start, nv);
      issue_kv(j, start);
    }
  }

  auto issue_s = [&](int j) {  // S = Q K^T of tile t0 + j (thread 0; Q and K are in)
    tc_fence_after();
    const uint32_t qa = smem_u32(q_s);
    const uint32_t ka = smem_u32(k_s + (j % ST) * C::kKVBytes);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk * 16 / C::kBoxD) * C::kBoxBytes + ((kk * 16) % C::kBoxD) * 2;
      umma_bf16(s_tmem, smem_desc(qa + off, 16, 8 * C::kRowBytes, C::kSwCode),
                smem_desc(ka + off, 16, 8 * C::kRowBytes, C::kSwCode), kIdescS,
                kk > 0 ? 1u : 0u);
    }
    umma_commit(bar_s);
  };
  // 128-row tiles: once every thread holds tile j's S in registers (the
  // row-max barrier), S of tile j+1 is issued at once if its K has landed,
  // so that it runs during the rest of the softmax.  Its completion then no
  // longer implies that P V of tile j is done: the P writes and O rescales of
  // tile j+1 wait for that explicitly.  (On the 32-row shapes, one or two key
  // tiles per CTA, this measured slower.)
  bool s_next = false;  // thread 0: S of the next tile already issued
  auto early_s = [&](int j) {
    if (!SG && t == 0) {
      s_next = j + 1 < my_tiles && mbar_try_wait(&bar_k[(j + 1) % ST], ((j + 1) / ST) & 1);
      if (s_next) issue_s(j + 1);
    }
  };

  float m_run = -FLT_MAX, l_run = 0.f;
  bool ok = true;
  for (int j = 0; j < my_tiles; ++j) {
    const int st = j % ST;
    int kstart, nvalid;
    tile_of(sg, t0 + j, kstart, nvalid);
    // ---- S = Q K^T (unless issued early during the previous tile)
    if (t == 0 && !s_next) {
      const bool good = (j > 0 || mbar_wait(bar_q, 0, p.status)) &&
                        mbar_wait(&bar_k[st], (j / ST) & 1, p.status);
      if (good)
        issue_s(j);
      else
        flags[0] = 1;
    }
    const bool bad_s = !mbar_wait(bar_s, j & 1, p.status) || flags[0];
    if (__syncthreads_or(bad_s)) {
      ok = false;
      break;
    }
    tc_fence_after();
    if (kSplitKV && t == 0 && j + ST < my_tiles) {  // S has read this K stage
      int start, nv;
      tile_of(sg, t0 + j + ST, start, nv);
      issue_k(j + ST, start);
    }
    if constexpr (SG) {
      // ---- softmax of row (t & 31) over keys [32w, 32w+32) of the tile
      const int kq = warp * 32;
      float s[32];
      tmem_ld32(s_tmem + lane_off + kq, s);
      tmem_ld_wait();
      float tm[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (kq + i < nvalid) tm[i & 3] = fmaxf(tm[i & 3], s[i]);
      x_s[t] = fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3]));
      __syncthreads();
      const int i0 = t & 31;
      const float tmax = fmaxf(fmaxf(x_s[i0], x_s[32 + i0]), fmaxf(x_s[64 + i0], x_s[96 + i0]));
      const float m_new = fmaxf(m_run, tmax * p.scale_log2);
      const float alpha = fast_exp2(m_run - m_new);
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 8 keys = one 16-byte chunk of P
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const int k0 = c * 8 + i;
          const float p0 = kq + k0 < nvalid ? fast_exp2(s[k0] * p.scale_log2 - m_new) : 0.f;
          const float p1 =
              kq + k0 + 1 < nvalid ? fast_exp2(s[k0 + 1] * p.scale_log2 - m_new) : 0.f;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          ls[c] += __low2float(h2) + __high2float(h2);
          pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        // the chunk goes into all four copies 32r + i0 of the row (same swizzle phase)
        const int key = kq + c * 8;
        uint8_t* pcol = p_s + (key >> 6) * (128 * 128) + ((((key & 63) >> 3) ^ (i0 & 7)) << 4);
#pragma unroll
        for (int r = 0; r < 4; ++r)
          *reinterpret_cast<uint4*>(pcol + (r * 32 + i0) * 128) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      // this warp only ever reads O columns [32w, 32w+32) of its lanes
      if (j > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float v[16];
          tmem_ld16(o_tmem + lane_off + kq + c * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= alpha;
          tmem_st16(o_tmem + lane_off + kq + c * 16, v);
        }
        tmem_st_wait();
      }
      l_run = l_run * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));  // this quarter's share
      m_run = m_new;
    } else {
      // ---- softmax of row trow over key half `half` of the tile (log2
      // domain); the row max crosses the two halves through shared memory
      constexpr int kH = kKeys / 2;
      const int kb = half * kH;
      float s[kH];
#pragma unroll
      for (int c = 0; c < kH / 32; ++c) tmem_ld32(s_tmem + lane_off + kb + c * 32, s + c * 32);
      tmem_ld_wait();
      // independent partial maxima and sums: two warps per scheduler still
      // leave little other work to hide a serial dependency chain behind
      float tm[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
      for (int i = 0; i < kH; ++i)
        if (kb + i < nvalid) tm[i & 3] = fmaxf(tm[i & 3], s[i]);
      x_s[t] = fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3]));
      tc_fence_before();
      __syncthreads();
      early_s(j);
      const float tmax = fmaxf(x_s[trow], x_s[128 + trow]);
      const float m_new = fmaxf(m_run, tmax * p.scale_log2);
      const float alpha = fast_exp2(m_run - m_new);
      if (j > 0 && !mbar_wait(bar_o, (j - 1) & 1, p.status)) flags[0] = 1;  // P and O free
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < kH / 8; ++c) {  // 8 keys = one 16-byte chunk of P
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const int k0 = c * 8 + i;
          const float p0 = kb + k0 < nvalid ? fast_exp2(s[k0] * p.scale_log2 - m_new) : 0.f;
          const float p1 =
              kb + k0 + 1 < nvalid ? fast_exp2(s[k0 + 1] * p.scale_log2 - m_new) : 0.f;
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          ls[c & 3] += __low2float(h2) + __high2float(h2);
          pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&h2);
        }
        // keys 64h..64h+63 form atom column h; row trow holds 8 chunks of 16 bytes
        uint8_t* prow = p_s + half * (128 * 128) + trow * 128;
        *reinterpret_cast<uint4*>(prow + ((c ^ (trow & 7)) << 4)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      // O (from earlier tiles) is rescaled in TMEM when the running max grew
      // (the previous P V was waited for above).  Each
      // thread rescales the half of the row's columns that it later reads.
      if (j > 0 && __any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          float v[16];
          tmem_ld16(o_tmem + lane_off + half * (D / 2) + c * 16, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= alpha;
          tmem_st16(o_tmem + lane_off + half * (D / 2) + c * 16, v);
        }
        tmem_st_wait();
      }
      l_run = l_run * alpha + ((ls[0] + ls[1]) + (ls[2] + ls[3]));  // this half's share
      m_run = m_new;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- O += P V
    if (t == 0) {
      tc_fence_after();
      if (!kSplitKV || mbar_wait(&bar_v[st], (j / ST) & 1, p.status)) {
        const uint32_t pa = smem_u32(p_s);
        const uint32_t va = smem_u32(v_s + st * C::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          const uint32_t boff = kk * 16 * C::kRowBytes;
          umma_bf16(o_tmem, smem_desc(pa + aoff, 16, 1024, 2),
                    smem_desc(va + boff, C::kBoxBytes, 8 * C::kRowBytes, C::kSwCode), kIdescO,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
      } else {
        flags[0] = 1;
      }
      umma_commit(bar_o);  // arrives at once when nothing was issued
      if (j + ST < my_tiles) {
        // the V stage is free once this P V has read it
        if (mbar_wait(bar_o, j & 1, p.status)) {
          int start, nv;
          tile_of(sg, t0 + j + ST, start, nv);
          if constexpr (kSplitKV)
            issue_v(j + ST, start);
          else
            issue_kv(j + ST, start);
        } else {
          flags[0] = 1;
        }
      }
    }
  }
  if (ok && my_tiles > 0) {
    const bool bad = !mbar_wait(bar_o, (my_tiles - 1) & 1, p.status) || flags[0];
    ok = !__syncthreads_or(bad);
  }
  tc_fence_after();

  // ---- output
  // A small group's thread (w, i) holds row i and output columns [32w, 32w+32);
  // otherwise thread t holds row t of the tile and every column.
  constexpr int kCols = SG ? 32 : D / 2;
  const int lrow = SG ? (t & 31) : trow;  // row within the tile
  const int c0 = SG ? warp * 32 : half * (D / 2);
  // the row's softmax sum is split over its four quarter (or two half) threads
  if constexpr (SG) {
    x_s[128 + t] = l_run;
    __syncthreads();
    l_run = (x_s[128 + lrow] + x_s[160 + lrow]) + (x_s[192 + lrow] + x_s[224 + lrow]);
  } else {
    __syncthreads();  // the last tile's maxima have been read
    x_s[t] = l_run;
    __syncthreads();
    l_run = x_s[trow] + x_s[128 + trow];
  }
  const int g = p.Hq / p.Hkv;
  const int r = rt * (SG ? 32 : 128) + lrow;
  const bool row_ok = r < p.group_rows;
  const int hl = r / p.n_rows;
  const int ii = r - hl * p.n_rows;
  const int h = kvh * g + hl;
  __nv_bfloat16* dst = p.out + ((size_t)(b * p.n_rows + ii) * p.Hq + h) * D;
  auto store16 = [&](int d0, const float (&v)[16], float inv) {
#pragma unroll
    for (int q = 0; q < 16; q += 8) {
      __nv_bfloat162 a0 = __floats2bfloat162_rn(v[q] * inv, v[q + 1] * inv);
      __nv_bfloat162 a1 = __floats2bfloat162_rn(v[q + 2] * inv, v[q + 3] * inv);
      __nv_bfloat162 a2 = __floats2bfloat162_rn(v[q + 4] * inv, v[q + 5] * inv);
      __nv_bfloat162 a3 = __floats2bfloat162_rn(v[q + 6] * inv, v[q + 7] * inv);
      uint4 w;
      w.x = *reinterpret_cast<uint32_t*>(&a0);
      w.y = *reinterpret_cast<uint32_t*>(&a1);
      w.z = *reinterpret_cast<uint32_t*>(&a2);
      w.w = *reinterpret_cast<uint32_t*>(&a3);
      *reinterpret_cast<uint4*>(dst + d0 + q) = w;
    }
  };

  if (p.chunks == 1) {
    if (ok) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
      for (int c = 0; c < kCols / 16; ++c) {
        float v[16];
        tmem_ld16(o_tmem + lane_off + c0 + c * 16, v);
        tmem_ld_wait();
        if (row_ok && my_tiles > 0) store16(c0 + c * 16, v, inv);
      }
    }
  } else {
    // ---- merge of the key chunks inside the cluster (rank = chunk).  Every
    // CTA reaches both cluster barriers, whatever happened before.
    const int nch = p.chunks;
    const uint32_t rank = (uint32_t)chunk;
    const bool have = ok && my_tiles > 0 && l_run > 0.f;
    const float2 mine = have ? make_float2(m_run, l_run) : make_float2(-FLT_MAX, 0.f);
    const uint32_t ml_addr = smem_u32(&ml_s[rank * 128 + lrow]);
    if (SG ? warp == 0 : half == 0)
      for (int q = 0; q < nch; ++q)
        st_cluster_v2(map_to_rank(ml_addr, (uint32_t)q), mine.x, mine.y);
    cluster_sync();  // (max, sum) everywhere; every chunk's P V is done
    float mx = -FLT_MAX;
    for (int c = 0; c < nch; ++c) {
      const float2 e = ml_s[c * 128 + lrow];
      if (e.y > 0.f) mx = fmaxf(mx, e.x);
    }
    float lt = 0.f;
    for (int c = 0; c < nch; ++c) {
      const float2 e = ml_s[c * 128 + lrow];
      if (e.y > 0.f) lt += fast_exp2(e.x - mx) * e.y;
    }
    const float wmine = have && lt > 0.f ? fast_exp2(mine.x - mx) / lt : 0.f;
    // groups of 16 columns are dealt round robin to the ranks; the owner's
    // buffer is [src][owned group][4][128 rows] float4 over the K/V/P region
    const int gpo = (C::kGroups + nch - 1) / nch;
    float4* red = reinterpret_cast<float4*>(k_s);
    const uint32_t red_addr = smem_u32(red);
    // this thread's columns of the O row are read from TMEM with one wait, then sent out
    float o[kCols];
    if constexpr (kCols % 32 == 0) {
#pragma unroll
      for (int c = 0; c < kCols / 32; ++c) tmem_ld32(o_tmem + lane_off + c0 + c * 32, o + c * 32);
    } else {
      tmem_ld16(o_tmem + lane_off + c0, *reinterpret_cast<float(*)[16]>(o));
    }
    tmem_ld_wait();
    if (row_ok) {
#pragma unroll
      for (int gg = 0; gg < kCols / 16; ++gg) {
        const int gi = c0 / 16 + gg;
        const uint32_t owner = (uint32_t)(gi % nch);
        const int lg = gi / nch;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int slot = ((int)(rank * gpo + lg) * 4 + q) * 128 + lrow;
          const uint32_t dst = map_to_rank(red_addr + slot * 16, owner);
          const float* v = o + gg * 16 + 4 * q;
          if (wmine != 0.f)
            st_cluster_v4(dst, v[0] * wmine, v[1] * wmine, v[2] * wmine, v[3] * wmine);
          else
            st_cluster_v4(dst, 0.f, 0.f, 0.f, 0.f);
        }
      }
    }
    cluster_sync();  // every contribution has landed
    if (ok && row_ok) {
      // the row's four quarter (two half) threads share its owned groups
      for (int lg = SG ? warp : half; lg < gpo; lg += SG ? 4 : 2) {
        const int gi = lg * nch + (int)rank;
        if (gi >= C::kGroups) break;
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
        for (int c = 0; c < nch; ++c) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 x = red[((c * gpo + lg) * 4 + q) * 128 + lrow];
            v[4 * q] += x.x;
            v[4 * q + 1] += x.y;
            v[4 * q + 2] += x.z;
            v[4 * q + 3] += x.w;
          }
        }
        store16(gi * 16, v, 1.f);
      }
    }
  }
  // The next kernel is released only now: its CTAs, resident beside this
  // one while they wait, slowed this kernel's softmax and merge measurably.
  grid_dep_launch();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, int ST, bool SG>
static cudaError_t launch_attn_t(const CUtensorMap& qmap, const CUtensorMap& kmap,
                                 const CUtensorMap& vmap, const AttnParams& p, bool pdl,
                                 cudaStream_t s) {
  using C_ = AttnCfg<D, ST>;
  auto kern = attn_kernel<D, ST, SG>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.batch * p.Hkv * p.row_tiles * p.chunks);
  cfg.blockDim = dim3(SG ? 128 : 256);
  cfg.dynamicSmemBytes = AttnCfg<D, ST>::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (p.chunks > kMaxMerge || (p.chunks > 1 && merge_bytes<D>(p.chunks) > C_::kRegion))
    return cudaErrorInvalidValue;  // the merge buffer would not fit
  if (p.chunks > 1) {  // the chunks of a row tile merge through distributed shared memory
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.chunks;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, qmap, kmap, vmap, p);
}

cudaError_t attn_prepare() {
  cudaError_t e = cudaSuccess;
#define DLLM_SET(D, ST, SG)                                                   \
  if (e == cudaSuccess)                                                      \
    e = cudaFuncSetAttribute(attn_kernel<D, ST, SG>,                         \
                             cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                             (int)AttnCfg<D, ST>::kSmem);
  DLLM_SET(128, 1, false) DLLM_SET(128, 2, false) DLLM_SET(32, 1, false) DLLM_SET(32, 2, false)
  DLLM_SET(128, 1, true) DLLM_SET(128, 2, true)
#undef DLLM_SET
  return e;
}

size_t attn_smem_bytes(int head_dim) {
  return head_dim == 128 ? AttnCfg<128, 2>::kSmem : AttnCfg<32, 2>::kSmem;
}

// One key tile per CTA keeps a single stage; longer chunks double-buffer.
// A small group's Q map has a 32-row box (it is loaded four times).
cudaError_t launch_attn(int head_dim, const CUtensorMap& qmap, const CUtensorMap& kmap,
                        const CUtensorMap& vmap, const AttnParams& p, bool pdl,
                        cudaStream_t s) {
  const bool one = p.tiles_per_chunk <= 1;
  if (p.small_group) {
    if (head_dim != 128 || p.row_tiles * 32 < p.group_rows) return cudaErrorInvalidValue;
    return one ? launch_attn_t<128, 1, true>(qmap, kmap, vmap, p, pdl, s)
               : launch_attn_t<128, 2, true>(qmap, kmap, vmap, p, pdl, s);
  }
  if (head_dim == 128)
    return one ? launch_attn_t<128, 1, false>(qmap, kmap, vmap, p, pdl, s)
               : launch_attn_t<128, 2, false>(qmap, kmap, vmap, p, pdl, s);
  if (head_dim == 32)
    return one ? launch_attn_t<32, 1, false>(qmap, kmap, vmap, p, pdl, s)
               : launch_attn_t<32, 2, false>(qmap, kmap, vmap, p, pdl, s);
  return cudaErrorInvalidValue;
}

}  // namespace dllm
