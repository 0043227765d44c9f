// Latency-bound kernels of the step: layer-0 input (plant or embedding),
// cross-tile vocabulary reduce fused with the threshold commit, and the
// one-time tables (RoPE cos/sin, fp32 weight split).
#include <float.h>
#include <limits.h>
#include <math.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dllm {

static long long g_launches = 0;
void count_launch() { ++g_launches; }
void add_launches(long long n) { g_launches += n; }
unsigned long long launch_count() { return (unsigned long long)g_launches; }

template <class K, class... A>
static cudaError_t launch_simple(K kern, dim3 grid, dim3 block, bool pdl, cudaStream_t s,
                                 A... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ------------------------------------------------------------------ debug checks
// A DLLM_DEBUG build checks the row positions that come from device memory
// before they address a buffer.  An out-of-range position sets kErrIndex in
// the status word, and the CTA skips the access.  The per-sequence block
// starts of dllm_decode_all are written only by the commit kernel, which
// checks both what it reads and what it writes, so the projection and
// attention kernels that read them later get checked values.  Other builds
// compile the checks away.
constexpr int kErrIndex = 4;  // status bit beside kErrTimeout and kErrBadArg
#ifdef DLLM_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
// lo <= v < hi, or (DLLM_DEBUG builds only) false with kErrIndex recorded.
__device__ __forceinline__ bool dbg_in_range(int v, int lo, int hi, int* status) {
  if constexpr (kDebugChecks) {
    const bool ok = v >= lo && v < hi;
    if (!ok && status != nullptr) atomicOr(status, kErrIndex);
    return ok;
  }
  return true;
}

// ------------------------------------------------------------------ embed
// Sum of a value over the CTA (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int mask = 16; mask > 0; mask >>= 1) v += __shfl_xor_sync(0xffffffffu, v, mask);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  return t;
}

// One CTA per row: x0 = embed[masked ? mask_id : token], its bf16 copy and
// the row's sum of squares (partial slot 0; the other slots are zeroed).
// Block 0 also writes the key segments of the launch sequence.
__global__ void __launch_bounds__(256) embed_kernel(const EmbedParams p) {
  __shared__ float red[32];
  grid_dep_wait();
  grid_dep_launch();
  const int row = blockIdx.x;
  for (int i = row * blockDim.x + threadIdx.x; i < p.nzero; i += gridDim.x * blockDim.x)
    p.zero[i] = 0;
  const int b = row / p.n_rows;
  const int pos = (p.seq_blk ? p.seq_blk[b] : p.row0) + (row - b * p.n_rows);
  for (int bb = threadIdx.x; row == 0 && p.segs != nullptr && bb < p.batch; bb += blockDim.x) {
    const int st = p.seq_start[bb];
    int s0 = st, l0 = 0, s1 = 0, l1 = 0;
    const int end = (p.seq_blk ? p.seq_blk[bb] : p.blk_start) + p.blk_len;
    if (p.seg_end > 0) {
      l0 = p.seg_end - st;
    } else if (p.mode == 2 || p.mode == 4) {  // DUAL, PREFIX_SUFFIXQ
      l0 = p.S - st;
    } else if (p.mode == 3) {           // DUAL_PRUNED
      const int wend = min(end + p.window, p.S);
      l0 = wend - st;
      if (end < p.S && p.S - 1 >= wend) {
        s1 = p.S - 1;
        l1 = 1;
      }
    } else {                            // NONE, PREFIX
      l0 = end - st;
    }
    int* o = p.segs + bb * 4;
    o[0] = s0;
    o[1] = l0 > 0 ? l0 : 0;
    o[2] = s1;
    o[3] = l1;
  }
  if (!dbg_in_range(pos, 0, p.S, p.status)) return;  // uniform over the CTA
  int tok = p.masked[(size_t)b * p.S + pos] ? p.mask_id : p.tokens[(size_t)b * p.S + pos];
  if (tok < 0 || tok >= p.vocab) {  // never read outside the embedding table
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, kErrBadArg);
    tok = 0;
  }
  float* xr = p.x + (size_t)row * p.d;
  __nv_bfloat16* xbr = p.xb + (size_t)row * p.d;
  float sq = 0.f;
  if (p.embed_f32) {
    const float* src = reinterpret_cast<const float*>(p.embed) + (size_t)tok * p.d;
    for (int i = threadIdx.x * 4; i < p.d; i += blockDim.x * 4) {
      const float4 f = *reinterpret_cast<const float4*>(src + i);
      *reinterpret_cast<float4*>(xr + i) = f;
      xbr[i] = __float2bfloat16_rn(f.x);
      xbr[i + 1] = __float2bfloat16_rn(f.y);
      xbr[i + 2] = __float2bfloat16_rn(f.z);
      xbr[i + 3] = __float2bfloat16_rn(f.w);
      sq += f.x * f.x + f.y * f.y + f.z * f.z + f.w * f.w;
    }
  } else {
    const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(p.embed) + (size_t)tok * p.d;
    for (int i = threadIdx.x * 8; i < p.d; i += blockDim.x * 8) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src + i);
      *reinterpret_cast<uint4*>(xbr + i) = raw;
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(h2[k]);
        xr[i + 2 * k] = f.x;
        xr[i + 2 * k + 1] = f.y;
        sq += f.x * f.x + f.y * f.y;
      }
    }
  }
  const float tot = block_sum(sq, red);
  if (p.sumsq != nullptr)
    for (int k = threadIdx.x; k < p.npart; k += blockDim.x)
      p.sumsq[(size_t)row * p.npart + k] = k == 0 ? tot : 0.f;
}

// One CTA per block row: h = bf16(x / rms(x) + plant where the row is masked).
__global__ void __launch_bounds__(256) final_norm_kernel(const FinalNormParams p) {
  __shared__ float red[32];
  grid_dep_wait();
  grid_dep_launch();
  const int b = blockIdx.x / p.B, i = blockIdx.x - b * p.B;
  const int blk = p.seq_blk ? p.seq_blk[b] : p.blk_start;
  const int pos = blk + i;
  if (!dbg_in_range(pos, p.P, p.S, p.status)) return;  // uniform over the CTA
  const float* xr = p.x + ((size_t)b * p.n_rows + (pos - (p.seq_blk ? blk : p.row0))) * p.d;
  float sq = 0.f;
  for (int k = threadIdx.x * 4; k < p.d; k += blockDim.x * 4) {
    const float4 f = *reinterpret_cast<const float4*>(xr + k);
    sq += f.x * f.x + f.y * f.y + f.z * f.z + f.w * f.w;
  }
  const float inv = rsqrtf(block_sum(sq, red) / (float)p.d + p.eps);
  const bool planted = p.masked[(size_t)b * p.S + pos] != 0;
  const __nv_bfloat16* pl = p.plants + ((size_t)b * p.G + (pos - p.P)) * p.d;
  __nv_bfloat16* hr = p.h + ((size_t)b * p.B + i) * p.d;
  for (int k = threadIdx.x * 4; k < p.d; k += blockDim.x * 4) {
    const float4 f = *reinterpret_cast<const float4*>(xr + k);
    float a0 = f.x * inv, a1 = f.y * inv, a2 = f.z * inv, a3 = f.w * inv;
    if (planted) {
      const uint2 raw = *reinterpret_cast<const uint2*>(pl + k);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
      const float2 u = __bfloat1622float2(h2[0]), w = __bfloat1622float2(h2[1]);
      a0 += u.x;
      a1 += u.y;
      a2 += w.x;
      a3 += w.y;
    }
    __nv_bfloat162 o0 = __floats2bfloat162_rn(a0, a1), o1 = __floats2bfloat162_rn(a2, a3);
    uint2 out;
    out.x = *reinterpret_cast<uint32_t*>(&o0);
    out.y = *reinterpret_cast<uint32_t*>(&o1);
    *reinterpret_cast<uint2*>(hr + k) = out;
  }
}

cudaError_t launch_final_norm(const FinalNormParams& p, bool pdl, cudaStream_t s) {
  return launch_simple(final_norm_kernel, dim3(p.batch * p.B), dim3(256), pdl, s, p);
}

cudaError_t launch_embed(const EmbedParams& p, bool pdl, cudaStream_t s) {
  return launch_simple(embed_kernel, dim3(p.batch * p.n_rows), dim3(256), pdl, s, p);
}

// ------------------------------------------------------------------ reduce + commit
__device__ __forceinline__ LmStat merge_stat(const LmStat& a, const LmStat& b) {
  const bool b_hi = (b.m > a.m) || (b.m == a.m && b.idx < a.idx);
  const LmStat& hi = b_hi ? b : a;
  const LmStat& lo = b_hi ? a : b;
  LmStat r;
  r.m = hi.m;
  r.idx = hi.idx;
  r.m2 = fmaxf(hi.m2, lo.m);
  r.s = hi.s + (lo.s > 0.f ? lo.s * __expf(lo.m - hi.m) : 0.f);
  return r;
}

// One CTA (1024 threads) per sequence.  Phase 1: one warp per block row
// merges the per-CTA vocabulary statistics into conf = 1 / sum exp(l - max),
// tok and gap.
// Phase 2 (warp 0): commit masked rows with conf > tau, plus the most
// confident masked row (lowest position on ties).
__global__ void __launch_bounds__(1024) commit_kernel(const CommitParams p) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ float s_conf[64];
  __shared__ int s_tok[64];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (p.stats != nullptr) {
    const int nwarps = blockDim.x >> 5;
    for (int i = warp; i < p.B; i += nwarps) {
      const LmStat* src = p.stats + (size_t)(b * p.B + i) * p.stat_slots;
      LmStat st;
      st.m = -FLT_MAX;
      st.s = 0.f;
      st.m2 = -FLT_MAX;
      st.idx = INT_MAX;
      LmStat buf[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {  // issue the loads before merging
        const int k = lane + 32 * q;
        buf[q] = k < p.stat_slots ? src[k] : st;
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) st = merge_stat(st, buf[q]);
      for (int k = lane + 256; k < p.stat_slots; k += 32) st = merge_stat(st, src[k]);
#pragma unroll
      for (int mask = 16; mask > 0; mask >>= 1) {
        LmStat o;
        o.m = __shfl_xor_sync(0xffffffffu, st.m, mask);
        o.s = __shfl_xor_sync(0xffffffffu, st.s, mask);
        o.m2 = __shfl_xor_sync(0xffffffffu, st.m2, mask);
        o.idx = __shfl_xor_sync(0xffffffffu, st.idx, mask);
        st = merge_stat(st, o);
      }
      if (lane == 0) {
        float conf = 1.f / st.s, gap = st.m - st.m2;
        int tok = st.idx;
        if (p.invalid_on_status && p.status != nullptr && *p.status != 0) {
          conf = __int_as_float(0x7fc00000);  // NaN: the statistics are not this call's
          gap = conf;
          tok = -1;
        }
        s_conf[i] = conf;
        s_tok[i] = tok;
        p.conf[b * p.B + i] = conf;
        p.tok[b * p.B + i] = tok;
        if (p.gap) p.gap[b * p.B + i] = gap;
      }
    }
  } else {
    for (int i = threadIdx.x; i < p.B; i += blockDim.x) {
      s_conf[i] = p.conf[b * p.B + i];
      s_tok[i] = p.tok[b * p.B + i];
    }
  }
  __syncthreads();
  if (!p.do_commit || warp != 0) return;
  // two rows per lane (B <= 64)
  const int i0 = lane, i1 = lane + 32;
  const int blk = p.seq_blk ? p.seq_blk[b] : p.blk_start;
  if (!dbg_in_range(blk, 0, p.S - p.B + 1, p.status)) return;  // uniform over the warp
  const size_t base = (size_t)b * p.S + blk;
  const bool m0 = i0 < p.B && p.masked[base + i0];
  const bool m1 = i1 < p.B && p.masked[base + i1];
  const float c0 = m0 ? s_conf[i0] : -1.f;
  const float c1 = m1 ? s_conf[i1] : -1.f;
  // best masked row: largest conf, lowest position on ties
  float bc = c0;
  int bi = i0;
  if (c1 > bc) {
    bc = c1;
    bi = i1;
  }
#pragma unroll
  for (int mask = 16; mask > 0; mask >>= 1) {
    const float oc = __shfl_xor_sync(0xffffffffu, bc, mask);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, mask);
    if (oc > bc || (oc == bc && oi < bi)) {
      bc = oc;
      bi = oi;
    }
  }
  const bool any_masked = bc >= 0.f;
  bool k0, k1;
  if (p.topk) {
    // fixed budget: this step's share of the block, then the rows whose rank
    // (masked rows ahead of them: higher conf, or equal conf and lower
    // position) is below it
    const int nm = __popc(__ballot_sync(0xffffffffu, m0)) + __popc(__ballot_sync(0xffffffffu, m1));
    const int base = p.B / p.steps_per_block, rem = p.B % p.steps_per_block;
    const int done = p.B - nm;
    const int j = done < rem * (base + 1) ? done / (base + 1)
                                          : rem + (done - rem * (base + 1)) / max(base, 1);
    const int k = min(max(base + (j < rem ? 1 : 0), 1), nm);
    __shared__ float s_mc[64];  // conf of masked rows, -1 elsewhere
    if (i0 < p.B) s_mc[i0] = c0;
    if (i1 < p.B) s_mc[i1] = c1;
    __syncwarp();
    int r0 = 0, r1 = 0;
    for (int q = 0; q < p.B; ++q) {
      const float cq = s_mc[q];
      if (cq < 0.f) continue;
      r0 += (cq > c0 || (cq == c0 && q < i0)) ? 1 : 0;
      r1 += (cq > c1 || (cq == c1 && q < i1)) ? 1 : 0;
    }
    k0 = m0 && r0 < k;
    k1 = m1 && r1 < k;
  } else {
    // step cap: the step that reaches it commits every row still masked.
    // The counter restarts whenever the block start changes or the block is
    // untouched (every row masked).
    bool force = false;
    if (p.steps_per_block > 0 && p.step_ctr != nullptr) {
      const int nm =
          __popc(__ballot_sync(0xffffffffu, m0)) + __popc(__ballot_sync(0xffffffffu, m1));
      int n = 0;
      if (lane == 0) {
        int* ctr = p.step_ctr + 2 * b;
        n = (ctr[1] != blk || nm == p.B) ? 0 : ctr[0];
        ctr[0] = n + 1;
        ctr[1] = blk;
      }
      n = __shfl_sync(0xffffffffu, n, 0);
      force = n + 1 >= p.steps_per_block;
    }
    const float tau = p.tau_seq ? p.tau_seq[b] : p.tau;
    // early exit: a row whose argmax repeats from the previous step of this
    // block has converged and commits once conf > exit_tau
    bool e0 = false, e1 = false;
    if (p.exit_state != nullptr) {
      int* pb = p.exit_state + b;
      int* pt = p.exit_state + p.batch + (size_t)b * p.B;
      // a block with every row masked is at its first step (also after the
      // caller reset the state), so there is no previous argmax
      const int nmask =
          __popc(__ballot_sync(0xffffffffu, m0)) + __popc(__ballot_sync(0xffffffffu, m1));
      const bool same = *pb == blk + 1 && nmask < p.B;
      if (i0 < p.B) {
        e0 = same && m0 && pt[i0] == s_tok[i0] && c0 > p.exit_tau;
        pt[i0] = m0 ? s_tok[i0] : -1;
      }
      if (i1 < p.B) {
        e1 = same && m1 && pt[i1] == s_tok[i1] && c1 > p.exit_tau;
        pt[i1] = m1 ? s_tok[i1] : -1;
      }
      __syncwarp();
      if (lane == 0) *pb = blk + 1;
    }
    k0 = m0 && (force || c0 > tau || e0 || (any_masked && bi == i0));
    k1 = m1 && (force || c1 > tau || e1 || (any_masked && bi == i1));
  }
  if (k0) {
    p.tokens[base + i0] = s_tok[i0];
    p.masked[base + i0] = 0;
  }
  if (k1) {
    p.tokens[base + i1] = s_tok[i1];
    p.masked[base + i1] = 0;
  }
  if (p.commit) {
    if (i0 < p.B) p.commit[b * p.B + i0] = k0;
    if (i1 < p.B) p.commit[b * p.B + i1] = k1;
  }
  const unsigned left = __popc(__ballot_sync(0xffffffffu, m0 && !k0)) +
                        __popc(__ballot_sync(0xffffffffu, m1 && !k1));
  if (lane == 0) {
    // the block's state after this commit: done, and (when this commit
    // finished it) due for the key/value refresh from its committed tokens
    if (p.block_done) p.block_done[b] = left == 0 ? 1 : 0;
    if (p.refresh) p.refresh[b] = (left == 0 && any_masked) ? blk : -1;
  }
  if (p.seq_blk != nullptr) {
    // per-sequence blocks: a block without masked rows was refreshed by this
    // pass (the refresh list named it after the previous pass); move on.
    // remaining = 1 while the sequence has work left.
    const bool any_start = __any_sync(0xffffffffu, m0 || m1);
    if (lane == 0) {
      int done = p.seq_done[b];
      if (!done && !any_start) {
        if (blk + p.B >= p.S) p.seq_done[b] = done = 1;
        else if (dbg_in_range(blk + p.B, 0, p.S - p.B + 1, p.status)) p.seq_blk[b] = blk + p.B;
      }
      if (p.remaining) p.remaining[b] = done ? 0 : 1;
    }
    return;
  }
  if (lane == 0 && p.remaining) p.remaining[b] = (int)left;
}

cudaError_t launch_commit(const CommitParams& p, bool pdl, cudaStream_t s) {
  return launch_simple(commit_kernel, dim3(p.batch), dim3(1024), pdl, s, p);
}

// ------------------------------------------------------------------ tables
__global__ void rope_table_kernel(float2* tab, int S, int D, double theta) {
  const int half = D / 2;
  const int n = S * half;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int pos = i / half, j = i - pos * half;
    const double inv = pow(theta, -2.0 * (double)j / (double)D);
    double sn, cs;
    sincos((double)pos * inv, &sn, &cs);
    tab[i] = make_float2((float)cs, (float)sn);
  }
}

cudaError_t launch_rope_table(float2* tab, int S, int D, double theta, cudaStream_t s) {
  count_launch();
  rope_table_kernel<<<148, 256, 0, s>>>(tab, S, D, theta);
  return cudaGetLastError();
}

__global__ void split_f32_kernel(const float* src, __nv_bfloat16* dst, int64_t rows,
                                 int64_t cols) {
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cols, c = i - r * cols;
    const float w = src[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const __nv_bfloat16 lo = __float2bfloat16_rn(w - __bfloat162float(hi));
    dst[r * 2 * cols + c] = hi;
    dst[r * 2 * cols + cols + c] = lo;
  }
}

cudaError_t launch_split_f32(const float* src, __nv_bfloat16* dst, int64_t rows, int64_t cols,
                             cudaStream_t s) {
  count_launch();
  split_f32_kernel<<<4 * 148, 256, 0, s>>>(src, dst, rows, cols);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ diagnostics
// One CTA waits on an mbarrier that nothing arrives at: the bounded wait must
// give up after limit_ns and report it in *status, and the kernel returns
// normally (no trap, no fault), leaving the context usable.
__global__ void wait_timeout_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, status, limit_ns);
}

cudaError_t launch_wait_timeout(int* status, long long limit_ns, cudaStream_t s) {
  count_launch();
  wait_timeout_kernel<<<1, 32, 0, s>>>(status, (unsigned long long)limit_ns);
  return cudaGetLastError();
}

}  // namespace dllm
