// Fused epilogues of the weight-streaming GEMM (Q/K/V with RMS scale, RoPE
// and cache store; O-projection with residual add and per-slice sums of
// squares; LM head with a running max / sum-exp / argmax / second max),
// shared by the per-projection GEMM kernel and the persistent layer-stack
// kernel.  In the persistent kernel (XCTA = true) values another CTA of the
// same launch may have written (the residual, its sums of squares) are read
// with L2-only loads, so that no stale L1 line is used.
#pragma once
#include <float.h>
#include <limits.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace dllm {

__device__ __forceinline__ LmStat lm_merge(const LmStat& a, const LmStat& b) {
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

__device__ __forceinline__ LmStat lm_shfl_xor(const LmStat& a, int mask) {
  LmStat r;
  r.m = __shfl_xor_sync(0xffffffffu, a.m, mask);
  r.s = __shfl_xor_sync(0xffffffffu, a.s, mask);
  r.m2 = __shfl_xor_sync(0xffffffffu, a.m2, mask);
  r.idx = __shfl_xor_sync(0xffffffffu, a.idx, mask);
  return r;
}

// Sum over the 128 lanes of each of the chunk's CW columns staged as
// stage[col][lane]: 128 / CW threads per column, CW lanes each, then a
// shuffle tree.  Returns the column sum in the column's first thread.  Each
// thread starts its CW lanes at a rotation that puts the warp's 32 threads on
// 32 distinct banks at every step (16 columns: 4 columns x 8 subs; 8
// columns: 2 columns x 16 subs).
template <int CW>
__device__ __forceinline__ float column_sum(const float* stage, int et) {
  static_assert(CW == 16 || CW == 8, "chunk width");
  constexpr int TPC = 128 / CW;  // threads per column
  const int col = et / TPC, sub = et % TPC;
  const float* cv = stage + col * 128 + sub * CW;
  const int rot = CW == 16 ? 4 * (col & 3) + (sub >> 1) : (sub >> 2) + 4 * (col & 1);
  float s = 0.f;
#pragma unroll
  for (int q = 0; q < CW; ++q) s += cv[(q + rot) & (CW - 1)];
#pragma unroll
  for (int mask = 1; mask < TPC; mask <<= 1) s += __shfl_xor_sync(0xffffffffu, s, mask);
  return s;
}

// Per-unit preparation of the final epilogue.  The epilogue warps run it
// while the unit's mainloop is still streaming: it reads only what earlier
// kernels wrote.  QKV, per activation row c of the tile: inv[c] = RMS scale
// (from the partial sums of squares), rp[c] = rotary position, and the row
// parts of the destination offsets in units of head_dim, qoff[c] into q and
// koff[c] into the caches (the head / kv-head parts are added per weight row).
// Load of a value another CTA of the same launch may have written.
template <bool XCTA>
__device__ __forceinline__ float ld_shared_f32(const float* p) {
  if constexpr (XCTA) return __ldcg(p);
  return *p;
}

template <int NT, int EPI, bool XCTA = false>
__device__ __forceinline__ void epi_prepare(const GemmParams& p, int layer, int n, int et,
                                            float* inv, int* rp) {
  if constexpr (EPI == EPI_QKV) {
    int* qoff = rp + NT;
    int* koff = qoff + NT;
    constexpr int TPC = NT >= 128 ? 1 : 128 / NT;  // threads per column
    const int sub = et % TPC;
    for (int c = et / TPC; c < NT; c += 128 / TPC) {
      const int xrow = n * NT + c;
      float s = 0.f;
      if (p.sumsq_in != nullptr && xrow < p.R) {
        const float* src = p.sumsq_in + (size_t)xrow * p.npart;
#pragma unroll 8
        for (int k = sub; k < p.npart; k += TPC) s += ld_shared_f32<XCTA>(src + k);
      }
#pragma unroll
      for (int o = 1; o < TPC; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (sub == 0) {
        inv[c] = p.sumsq_in != nullptr ? rsqrtf(s / (float)p.d_norm + p.rms_eps) : 1.f;
        int r = 0, qo = 0, ko = 0;
        if (xrow < p.R) {
          const int b = xrow / p.n_rows;
          const int ii = xrow - b * p.n_rows;
          const int pos = (p.seq_blk ? p.seq_blk[b] : p.row0) + ii;
          if (p.rope_tab != nullptr) r = pos - p.seq_start[b];
          qo = b * p.Hq * p.n_rows + ii;                       // in units of D
          ko = (layer * p.batch + b) * p.Hkv * p.S + pos;    // in units of D
        }
        rp[c] = r < 0 ? 0 : r;
        qoff[c] = qo;
        koff[c] = ko;
      }
    }
    named_bar_sync(1, 128);
  }
}

// O-projection: the residual entries x[n*NT + c0 + i][m*128 + wl] a chunk
// adds to.  The previous kernels are complete once the dependency wait has
// returned, so these loads may run while the mainloop is still streaming.
template <int NT, bool XCTA = false, int CW = 16>
__device__ __forceinline__ void oproj_load_x(const GemmParams& p, int m, int n, int c0, int wl,
                                             float (&xo)[CW]) {
  const int wrow = m * 128 + wl;
#pragma unroll
  for (int i = 0; i < CW; ++i) {
    const int xrow = n * NT + c0 + i;
    xo[i] = xrow < p.R ? ld_shared_f32<XCTA>(p.x + (size_t)xrow * p.d_model + wrow) : 0.f;
  }
}

// Epilogue of one CW-column chunk; v[i] = D^T[m*128 + wl][n*NT + c0 + i].
// xo: the O-projection's residual entries of the chunk (oproj_load_x).
// The LM head takes 16-column chunks only.
template <int NT, int EPI, int CW = 16>
__device__ __forceinline__ void epi_chunk(const GemmParams& p, int m, int n, int c0, int wl,
                                          int et, const float (&v)[CW], const float (&xo)[CW],
                                          float* stage, LmStat* run) {
  static_assert(EPI != EPI_LMHEAD || CW == 16, "LM-head chunks are 16 columns");
  if constexpr (EPI == EPI_OPROJ) {
    const int wrow = m * 128 + wl;
#pragma unroll
    for (int i = 0; i < CW; ++i) {
      const int xrow = n * NT + c0 + i;
      float sq = 0.f;
      if (xrow < p.R) {
        const size_t off = (size_t)xrow * p.d_model + wrow;
        const float nx = xo[i] + v[i];
        p.x[off] = nx;
        p.xb[off] = __float2bfloat16_rn(nx);
        sq = nx * nx;
      }
      stage[i * 128 + wl] = sq;
    }
    if (p.sumsq_out != nullptr) {
      named_bar_sync(1, 128);
      const float s = column_sum<CW>(stage, et);
      const int xrow = n * NT + c0 + et / (128 / CW);
      if (et % (128 / CW) == 0 && xrow < p.R) p.sumsq_out[(size_t)xrow * p.npart + m] = s;
      named_bar_sync(1, 128);
    }
  } else if constexpr (EPI == EPI_QKV) {
    const float* inv = reinterpret_cast<const float*>(run);
    const int* rpos = reinterpret_cast<const int*>(inv + NT);
    const int* qoff = rpos + NT;
    const int* koff = qoff + NT;
    const int D = p.D, half = D >> 1;
    const int wrow = m * 128 + wl;
    const int head = wrow / D;
    const int dd = wrow - head * D;
    const bool is_q = head < p.Hq;
    const bool is_k = !is_q && head < p.Hq + p.Hkv;
    const bool has_rope = p.rope_tab != nullptr;  // uniform over the CTA
    float val[CW];
#pragma unroll
    for (int i = 0; i < CW; ++i) val[i] = v[i] * inv[c0 + i];
    if (has_rope) {
      // rotate-half pairs live in lanes dd and dd +- D/2 of the same tile
#pragma unroll
      for (int i = 0; i < CW; ++i) stage[i * 128 + wl] = val[i];
      named_bar_sync(1, 128);
      if (is_q || is_k) {
        const int partner = wl + (dd < half ? half : -half);
        const int j = dd < half ? dd : dd - half;
        float2 cs[CW];
#pragma unroll
        for (int i = 0; i < CW; ++i) cs[i] = p.rope_tab[(size_t)rpos[c0 + i] * half + j];
#pragma unroll
        for (int i = 0; i < CW; ++i) {
          const float o = stage[i * 128 + partner];
          val[i] = dd < half ? (val[i] * cs[i].x - o * cs[i].y) : (val[i] * cs[i].x + o * cs[i].y);
        }
      }
      named_bar_sync(1, 128);
    }
    __nv_bfloat16* dst;
    size_t hoff;
    if (is_q) {
      dst = p.q_out;
      hoff = (size_t)head * p.n_rows * D + dd;
    } else {
      const int kvh = is_k ? head - p.Hq : head - p.Hq - p.Hkv;
      dst = is_k ? p.k_cache : p.v_cache;
      hoff = (size_t)kvh * p.S * D + dd;
    }
    const int* roff = is_q ? qoff : koff;
#pragma unroll
    for (int i = 0; i < CW; ++i) {
      if (n * NT + c0 + i < p.R)
        dst[(size_t)roff[c0 + i] * D + hoff] = __float2bfloat16_rn(val[i]);
    }
  } else {  // EPI_LMHEAD
#pragma unroll
    for (int i = 0; i < 16; ++i) stage[i * 128 + wl] = v[i];
    named_bar_sync(1, 128);
    const int col = et >> 3, sub = et & 7;
    const float* cv = stage + col * 128 + sub * 16;
    const int vbase = m * 128 + sub * 16;
    LmStat st;
    st.m = -FLT_MAX;
    st.m2 = -FLT_MAX;
    st.idx = INT_MAX;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float x = cv[q];
      if (x > st.m) {
        st.m2 = st.m;
        st.m = x;
        st.idx = vbase + q;
      } else if (x > st.m2) {
        st.m2 = x;
      }
    }
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) s += __expf(cv[q] - st.m);
    st.s = s;
#pragma unroll
    for (int mask = 1; mask < 8; mask <<= 1) st = lm_merge(st, lm_shfl_xor(st, mask));
    if (sub == 0) run[c0 + col] = lm_merge(run[c0 + col], st);
    named_bar_sync(1, 128);
  }
}

}  // namespace dllm
