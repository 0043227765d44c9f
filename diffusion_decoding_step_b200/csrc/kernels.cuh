// Internal parameter blocks and launchers shared by the kernel files and the
// C-ABI layer.  Nothing here is part of the public interface.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dllm {

constexpr int kNumSMs = 148;

// EPI_QKV_DEEP: the Q/K/V epilogue on a deeper weight ring (split tiles that
// run two CTAs on some SMs)
enum EpiKind : int { EPI_QKV = 0, EPI_OPROJ = 1, EPI_LMHEAD = 2, EPI_QKV_DEEP = 3 };

// Running softmax statistics of a set of logits: max, sum of exp(l - max),
// second largest (a tied maximum counts), index of the first maximum.
struct __align__(16) LmStat {
  float m, s, m2;
  int idx;
};

// Bytes a later kernel of the sequence will read, fetched into L2 while
// this kernel runs: ranges [ptr[i], ptr[i] + bytes[i]), split over the CTAs.
// Nothing waits for them; a prefetch only warms the cache.
struct L2Prefetch {
  const uint8_t* ptr[2];
  long long bytes[2];
};

struct GemmParams {
  // D^T[wrow][xrow] = sum_k W[layer][wrow][k] * X[xrow][k mod kx]
  int M;          // weight rows (multiple of 128)
  int R;          // activation rows
  int K;          // weight K extent (multiple of 64)
  int kx_blocks;  // X operand K extent / 64 (k-block kb reads X block kb % kx_blocks)
  int m_tiles, n_tiles, splits, kb_per_split, units;
  int layer;
  int* status;
  // rows are (sequence, i) with position row0 + i, n_rows per sequence
  int n_rows, row0;
  const int* seq_start;
  // QKV epilogue
  int Hq, Hkv, D, S, batch;
  const float2* rope_tab;  // [S][D/2] (cos, sin) or null
  __nv_bfloat16* q_out;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  // row norms: sumsq[xrow][npart] partial sums of x^2 over 128-column slices
  const float* sumsq_in;   // QKV: scale each row by 1/sqrt(sum/d_norm + eps)
  float* sumsq_out;        // O-proj: this tile's slice sum of the new residual
  int npart, d_norm;
  float rms_eps;
  // O-proj epilogue
  float* x;
  __nv_bfloat16* xb;
  int d_model;
  // LM-head epilogue: stats[xrow][slot]
  LmStat* stats;
  int stat_slots;
  int recv_in_ring;  // split K: partials go into the weight ring (grid > SM count)
  const int* seq_blk;  // QKV: per-sequence first row position, or null: row0
  L2Prefetch pf;
};

struct AttnParams {
  int batch, Hq, Hkv, D, S, layer;
  int n_rows;       // query rows per sequence and head
  int group_rows;   // (Hq/Hkv) * n_rows
  int row_tiles;    // ceil(group_rows / 128), or ceil(group_rows / 32) with small_group
  int small_group;  // 1: row tiles of 32 rows, loaded four times (Q map box of 32 rows)
  int chunks;       // key chunks per (sequence, kv head, row tile) = cluster size
  int tiles_per_chunk;
  const int* segs;  // [b][2][2] (start, len), or null: derived from the fields below
  int mode, blk_start, blk_len, window, seg_end;
  const int* seq_start;
  int dep_lo, dep_hi;  // key positions the preceding kernel writes (load after the wait)
  __nv_bfloat16* out;  // [b*n_rows][Hq*D]
  int* status;
  const int* seq_blk;  // per-sequence block starts (query rows and dep range), or null
  float scale_log2;    // log2(e) / sqrt(D)
  L2Prefetch pf;
};

#ifdef __CUDACC__
// This CTA's share of a prefetch: the ranges are cut into 32 KB chunks, dealt
// round robin over the CTAs and issued by `lanes` threads of the CTA.
__device__ __forceinline__ void l2_prefetch_share(const L2Prefetch& pf, int cta, int ctas,
                                                  int lane, int lanes) {
  constexpr long long kChunk = 32768;
  long long c0 = 0;  // chunks of the earlier ranges
  for (int r = 0; r < 2; ++r) {
    const long long nb = pf.bytes[r];
    if (pf.ptr[r] == nullptr || nb <= 0) continue;
    const long long nc = (nb + kChunk - 1) / kChunk;
    const long long first = ((cta - c0) % ctas + ctas) % ctas;
    for (long long i = first + (long long)lane * ctas; i < nc; i += (long long)lanes * ctas) {
      const long long off = i * kChunk;
      const long long n = nb - off < kChunk ? nb - off : kChunk;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(pf.ptr[r] + off),
                   "r"((uint32_t)n)
                   : "memory");
    }
    c0 += nc;
  }
}
#endif

// ---------------------------------------------------------------- layer stack
// The persistent layer-stack kernel runs every layer of a step (or of a
// refresh) in one launch, one CTA per SM.  Each GEMM phase (Q/K/V, O-proj)
// flattens its (weight tile, 64-wide k-block) space and gives each of `n`
// CTAs one contiguous, equal share (stream-K); a share that crosses a tile
// boundary is cut into one segment per tile.  The segments of a tile are its
// contributors, numbered in k order.
struct StackSeg {
  int tile, kb0, kb1, ci, nc;  // tile, k-block range, contributor index, contributors
};
constexpr int kStackMaxSeg = 4;  // segments per CTA and phase

__host__ __device__ inline long long stack_lo(int c, int n, long long T) {
  return (long long)c * T / n;
}
// The CTA whose share holds k-block kb (0 <= kb < T).
__host__ __device__ inline int stack_owner(long long kb, int n, long long T) {
  return (int)(((kb + 1) * n + T - 1) / T) - 1;
}
// Segments of CTA c; returns their count, or -1 if more than maxs are needed.
__host__ __device__ inline int stack_segments(int c, int tiles, int kbt, int n, StackSeg* out,
                                              int maxs) {
  if (c >= n) return 0;
  const long long T = (long long)tiles * kbt;
  long long a = stack_lo(c, n, T);
  const long long e = stack_lo(c + 1, n, T);
  int k = 0;
  while (a < e) {
    if (k == maxs) return -1;
    const int t = (int)(a / kbt);
    const long long tb = (long long)t * kbt;
    const long long b = e < tb + kbt ? e : tb + kbt;
    const int ca = stack_owner(tb, n, T);
    const int cb = stack_owner(tb + kbt - 1, n, T);
    out[k].tile = t;
    out[k].kb0 = (int)(a - tb);
    out[k].kb1 = (int)(b - tb);
    out[k].ci = c - ca;
    out[k].nc = cb - ca + 1;
    ++k;
    a = b;
  }
  return k;
}

struct StackParams {
  int L, R, n_rows, batch, Hq, Hkv, S, d, g;
  int qt, ot;      // weight tiles of the Q/K/V and O-projection GEMMs
  int qkbt, okbt;  // k-blocks (64 wide) per tile
  int qn, on;      // CTAs sharing each phase
  int qmaxc, omaxc;  // contributor slots per tile in the partial buffers
  // attention: row tiles and key chunks per (sequence, kv head), 64-key
  // tiles per chunk, units per layer
  int rt, chunks, tpc, units;
  int mode, blk_start, blk_len, window, seg_end, dep_lo, dep_hi;
  int lookahead;   // weight k-blocks prefetched into L2 beyond the ring
  const int* seq_start;
  __nv_bfloat16* q;     // [b][Hq][n_rows][D]
  __nv_bfloat16* attn;  // [b*n_rows][Hq*D]
  float* qpart;         // [qt][qmaxc][NT][128] fp32 split-K partials
  float* opart;         // [ot][omaxc][NT][128]
  float* apart;         // [b*Hkv*rt][chunks][D][128] unnormalised attention outputs
  float2* aml;          // [b*Hkv*rt][chunks][128] (running max in log2 units, sum)
  int* flags;           // fs ints per layer, then the abort word
  int fs;
  int* status;
  float scale_log2;
  GemmParams gq, go;    // epilogue parameters of the two projections
};

// Launch helpers (return cudaError_t of the launch).
cudaError_t launch_gemm(int epi, int nt, const CUtensorMap& wmap, const CUtensorMap& xmap,
                        const GemmParams& p, int grid, bool pdl, cudaStream_t s);
cudaError_t gemm_prepare();
cudaError_t attn_prepare();
cudaError_t launch_wait_timeout(int* status, long long limit_ns, cudaStream_t s);

// Layer-stack kernel (csrc/stack.cu): maps for W_qkv, W_o, xb, the attention
// output, q, and the K/V caches (64-key boxes).
cudaError_t stack_prepare();
size_t stack_smem_bytes(int nt);
cudaError_t stack_occupancy(int nt, int* blocks_per_sm);
cudaError_t launch_stack(int nt, const CUtensorMap* maps, const StackParams& p, int grid,
                         bool pdl, cudaStream_t s);

cudaError_t launch_attn(int head_dim, const CUtensorMap& qmap, const CUtensorMap& kmap,
                        const CUtensorMap& vmap, const AttnParams& p, bool pdl,
                        cudaStream_t s);
size_t attn_smem_bytes(int head_dim);

struct EmbedParams {
  int batch, S, d, n_rows, row0, embed_f32, vocab, mask_id, npart, blk_start, blk_len;
  int* status;
  const int* tokens;
  const uint8_t* masked;
  const void* embed;
  float* x;
  __nv_bfloat16* xb;
  float* sumsq;
  // optional: key segments of the step, written by block 0 thread 0
  int* segs;
  const int* seq_start;
  int mode, window, seg_end;  // seg_end: end of the key range for prefill/none
  const int* seq_blk;  // per-sequence block starts (rows start there), or null: row0 / blk_start
  // optional: ints cleared before the next kernel (the layer-stack kernel's flags)
  int* zero;
  int nzero;
};
cudaError_t launch_embed(const EmbedParams& p, bool pdl, cudaStream_t s);

// LM-head input of the block rows: h = bf16(x / rms(x) + plant where masked).
struct FinalNormParams {
  int batch, B, d, n_rows, row0, blk_start, S, P, G;
  float eps;
  const float* x;
  const uint8_t* masked;
  const __nv_bfloat16* plants;
  __nv_bfloat16* h;
  const int* seq_blk;  // per-sequence block starts, or null: blk_start (= row0)
  int* status;         // device status word, or null
};
cudaError_t launch_final_norm(const FinalNormParams& p, bool pdl, cudaStream_t s);

constexpr float kRmsEps = 1e-6f;

struct CommitParams {
  int batch, S, B, blk_start, stat_slots, vocab;
  float tau;
  const LmStat* stats;  // [b*B][stat_slots] or null when conf/tok are given
  float* conf;          // [b][B]
  int* tok;
  float* gap;
  int* tokens;
  uint8_t* masked;
  uint8_t* commit;
  int* remaining;
  // optional: block_done[b] = 1 when no row of the block is left masked;
  // refresh[b] = the block start this commit finished (its keys/values are to
  // be recomputed from the committed tokens), else -1
  int* block_done;
  int* refresh;
  int do_commit;
  int topk;             // fixed-budget rule instead of the threshold
  int steps_per_block;  // topk: steps a block takes; threshold: step cap (0 = none)
  int* step_ctr;        // [b][2] steps taken in the current block, its start (null: no cap)
  // early exit (null: off): [b] block start + 1 of the previous step (0: none),
  // then [b][B] each row's argmax at that step (-1: not masked then)
  int* exit_state;
  float exit_tau;
  // per-sequence blocks (null: blk_start for every sequence): a pass that
  // finds no masked row in a sequence's block was that block's refresh, and
  // the sequence moves on to its next block (or is done after the last)
  int* seq_blk;
  int* seq_done;
  const float* tau_seq;  // [b] per-sequence threshold, or null: tau
  int* status;           // device status word, or null
  // reduce only: when the status word is nonzero (a wait of the LM head gave
  // up), write conf = gap = NaN and tok = -1 instead of the merged statistics
  int invalid_on_status;
};
cudaError_t launch_commit(const CommitParams& p, bool pdl, cudaStream_t s);

cudaError_t launch_rope_table(float2* tab, int S, int D, double theta, cudaStream_t s);
cudaError_t launch_split_f32(const float* src, __nv_bfloat16* dst, int64_t rows, int64_t cols,
                             cudaStream_t s);

// Count of kernels launched by this library.
void count_launch();

}  // namespace dllm
