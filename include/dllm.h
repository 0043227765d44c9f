/*
 * dllm.h - C ABI of the B200 (sm_100a) block-decode step of a masked-diffusion LLM.
 *
 * The method (Fast-dLLM v1): a block of masked positions is denoised in
 * parallel; each step every masked position gets the max-softmax confidence
 * and argmax token of the LM head, and every position whose confidence
 * exceeds the threshold tau is committed ("Fast-dLLM: Four Acceleration Tracks
 * for Diffusion Language Models...", section "The v1 Mechanism: KV Cache Plus
 * Confidence-Threshold Parallel Decoding").  A key/value cache holds the
 * attention state of settled positions (same section; Fast-dLLM README,
 * project table, "KV Cache + Parallel Decoding"); the suffix may be pruned to
 * a window after the block plus the trailing position (Streaming-dLLM README,
 * figure "Illustration of approximated suffix pruning").
 *
 * The model is a pre-norm transformer with the MLP dropped: per layer
 * x <- x + Wo . attn(W_qkv . x / rms(x)) with a weightless RMSNorm
 * (rms(x) = sqrt(mean(x^2) + 1e-6)); the LM head reads x_L / rms(x_L) plus,
 * for a masked row, its planted hidden state.  A masked row enters layer 0 as
 * the embedding of mask_id.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller unless a
 *    parameter says "host".  The library allocates no device memory; scratch
 *    comes from the caller's workspace (dllm_workspace_size bytes, prepared
 *    once with dllm_workspace_init), except for dllm_lmhead_confidence_noalloc,
 *    which keeps a fixed scratch array in the library's device image.
 *  - Calls are asynchronous on `stream` unless documented otherwise; nothing
 *    prints, nothing aborts.  Invalid arguments return DLLM_ERR_INVALID or
 *    DLLM_ERR_UNSUPPORTED before anything is launched.
 *  - Layouts are row-major, innermost index last.  bf16 = IEEE bfloat16.
 *    b = batch, L = layers, d = hidden, Hq/Hkv = query/kv heads, D = head_dim,
 *    V = vocab, P = prompt_len, G = gen_len, B = block, S = P + G.
 *  - Supported: D in {32, 128}; d, Hq*D and (Hq+2Hkv)*D multiples of 128;
 *    V a multiple of 128; Hq a multiple of Hkv; B <= 64; b <= 1024;
 *    S <= 2^24; L*b*Hkv*S < 2^31 and b*S*Hq < 2^31 (the device addresses cache
 *    and query rows with 32-bit offsets in units of D).  rope_theta must be
 *    finite and >= 0 (0: no RoPE); tau must not be NaN.
 *  - Device-side waits are bounded (about 2 s); a wait that gives up sets a bit
 *    in the workspace status word, read with dllm_device_status (calls
 *    without a workspace report it in their outputs; see
 *    dllm_lmhead_confidence_noalloc).
 */
#ifndef DLLM_H_
#define DLLM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dllm_stream; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  DLLM_OK = 0,
  DLLM_ERR_INVALID = -1,     /* bad pointer, size or configuration */
  DLLM_ERR_UNSUPPORTED = -2, /* valid but not implemented shape */
  DLLM_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed */
  DLLM_ERR_TIMEOUT = -4,     /* a device wait gave up (status word set) */
  DLLM_ERR_WORKSPACE = -5    /* workspace too small */
} dllm_status;

/* Which keys a block row attends to (block at [s, s+B), sequence start st):
 *   NONE        [st, s+B), every position recomputed each step (no cache)
 *   PREFIX      [st, s+B), prefix keys/values from the cache
 *   DUAL        [st, S),   prefix and suffix from the cache
 *   DUAL_PRUNED [st, min(s+B+window, S)) plus S-1 when the suffix is not empty
 *   PREFIX_SUFFIXQ [st, S), prefix from the cache; the block and every later
 *               position run through the layers as queries each step (their
 *               keys/values are recomputed), only the block reaches the LM
 *               head.  The prefill covers the prompt, as for PREFIX. */
typedef enum {
  DLLM_CACHE_NONE = 0,
  DLLM_CACHE_PREFIX = 1,
  DLLM_CACHE_DUAL = 2,
  DLLM_CACHE_DUAL_PRUNED = 3,
  DLLM_CACHE_PREFIX_SUFFIXQ = 4
} dllm_cache_mode;

/* Weight storage.  BF16: bf16 weights, K extent = the input width.
 * F32_SPLIT: fp32 weights stored as two bf16 halves [hi | lo] along K
 * (made by dllm_split_f32_weights); hi + lo equals the fp32 value to about
 * 2^-17 relative, and the embedding stays fp32. */
typedef enum { DLLM_W_BF16 = 0, DLLM_W_F32_SPLIT = 1 } dllm_weight_format;

/* Commit rule of a step (Fast-dLLM overview page, "The v1 Mechanism": the
 * confidence-threshold rule; Fast-dLLM README, "Quick Start": the sampler's
 * --steps knob next to the block length).
 *   THRESHOLD  every masked row with conf > tau, and at least the most
 *              confident masked row (lowest position on ties).
 *   TOPK       a fixed budget: a block is decoded in exactly steps_per_block
 *              steps; step j commits floor(B/steps) + [j < B mod steps] of
 *              the most confident masked rows (lower position first on
 *              equal confidence), j being inferred from the rows already
 *              committed.  tau is not used.
 *   EARLY_EXIT a dynamic threshold, reading Streaming-dLLM's confidence-aware
 *              early exit for converged tokens (thelatestinai listing page,
 *              Streaming-dLLM abstract): a masked row whose argmax equals
 *              its argmax at the previous step of the same block has
 *              converged and commits once conf > exit_tau (<= tau); other
 *              rows as THRESHOLD (conf > tau, plus the most confident masked
 *              row).  At a block's first step it is THRESHOLD.  The previous
 *              argmax per row is kept in the workspace by dllm_decode_step /
 *              dllm_decode_block / dllm_decode_all; dllm_threshold_commit,
 *              which has no workspace, applies the first-step rule. */
typedef enum {
  DLLM_COMMIT_THRESHOLD = 0,
  DLLM_COMMIT_TOPK = 1,
  DLLM_COMMIT_EARLY_EXIT = 2
} dllm_commit_mode;

typedef struct {
  int32_t batch, n_layers, hidden, n_q_heads, n_kv_heads, head_dim, vocab;
  int32_t prompt_len; /* P: longest prompt; shorter prompts are left-padded */
  int32_t gen_len, block, window, mask_id;
  float tau;        /* commit threshold, strict conf > tau */
  float rope_theta; /* rotate-half RoPE base; 0 disables RoPE */
  int32_t mode;          /* dllm_cache_mode */
  int32_t weight_format; /* dllm_weight_format */
  int32_t commit_mode;   /* dllm_commit_mode */
  int32_t steps_per_block; /* TOPK: 1 <= steps_per_block <= block.  THRESHOLD: a step cap
                            * per block when > 0 (the step that reaches it commits every
                            * row still masked; counted per sequence in the workspace by
                            * dllm_decode_step / dllm_decode_block), none when <= 0.
                            * EARLY_EXIT: the same step cap */
  float exit_tau;          /* EARLY_EXIT: confidence bound of converged rows, finite, >= 0
                            * (>= tau: the THRESHOLD rule).  Unused otherwise. */
} dllm_config;

/* Kw = hidden (BF16) or 2*hidden (F32_SPLIT); Ko = Hq*D or 2*Hq*D. */
typedef struct {
  const void* wqkv;  /* bf16 [L][(Hq+2Hkv)*D][Kw]; rows: q heads, k heads, v heads */
  const void* wo;    /* bf16 [L][hidden][Ko] */
  const void* w_lm;  /* bf16 [V][Kw] */
  const void* embed; /* [V][hidden]; bf16 (BF16) or fp32 (F32_SPLIT); tied to w_lm */
} dllm_weights;

typedef struct {
  int32_t* tokens;          /* [b][S] token ids */
  uint8_t* masked;          /* [b][S] 1 = still masked; only ever goes 1 -> 0 */
  const int32_t* seq_start; /* [b] first valid position (left padding before it) */
  void* k_cache;            /* bf16 [L][b][Hkv][S][D]; must hold finite values */
  void* v_cache;            /* bf16 [L][b][Hkv][S][D] */
  const void* plants;       /* bf16 [b][G][hidden] planted LM-head offsets of generated rows */
  const float* tau;         /* [b] per-sequence commit threshold (device), read by every step,
                             * so a policy may change it between steps; NULL: cfg->tau */
} dllm_state;

/* Bytes of workspace a configuration needs (host call, no GPU work).  Library
 * plumbing, no counterpart on the pages. */
dllm_status dllm_workspace_size(const dllm_config* cfg, size_t* bytes);

/* Zero the workspace's counters and status word and build the RoPE table.
 * Call once per workspace before any other call that takes it.  Library
 * plumbing, no counterpart on the pages. */
dllm_status dllm_workspace_init(const dllm_config* cfg, void* ws, size_t ws_bytes,
                                dllm_stream stream);

/* fp32 [rows][cols] -> bf16 [rows][2*cols] with hi = bf16(w), lo = bf16(w - hi).
 * Storage of fp32 weights for the GEMM; no counterpart on the pages. */
dllm_status dllm_split_f32_weights(const float* src, void* dst, int64_t rows, int64_t cols,
                                   dllm_stream stream);

/* Per-row sums of squares of the residual are kept as row_sumsq
 * [rows][hidden/128] fp32: entry j is the sum of x^2 over columns
 * [128j, 128j+128) (a row's total is the sum of its entries). */

/* Step a1.  Layer-0 input of the rows a step evaluates: a masked position is
 * evaluated as the mask token, a settled one as its token (the masked
 * positions of the block are evaluated in parallel: "Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism").
 * Layer-0 input of n_rows rows per sequence starting at position row0:
 * x[b*n_rows+i] = embed[masked[b][p] ? mask_id : tokens[b][p]], p = row0+i.
 * x fp32 [b*n_rows][hidden]; xb its bf16 copy; row_sumsq (may be NULL) gets
 * each row's sum of squares in entry 0 and zeros elsewhere. */
dllm_status dllm_embed_rows(const dllm_config* cfg, const dllm_weights* w,
                            const dllm_state* st, int32_t row0, int32_t n_rows, float* x,
                            void* xb, float* row_sumsq, dllm_stream stream);

/* Step a2.  The keys/values written here are the cache the v1 mechanism
 * keeps for settled positions ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism"); RoPE
 * is the Qwen2.5-shaped workload's rotary embedding.
 * Q/K/V projection of layer `layer` (GEMM on tcgen05, fp32 accumulate) for
 * n_rows rows per sequence at positions row0..: (W_qkv . xb) / rms(x) with
 * rms from row_sumsq (NULL = no scaling), RoPE at position p-seq_start on q
 * and k, q -> q_out bf16 [b][Hq][n_rows][D], k/v -> the caches at p.
 * xb bf16 [b*n_rows][hidden]. */
dllm_status dllm_qkv_proj(const dllm_config* cfg, const dllm_weights* w, int32_t layer,
                          const void* xb, const float* row_sumsq, int32_t row0, int32_t n_rows,
                          const int32_t* seq_start, void* q_out, void* k_cache, void* v_cache,
                          void* ws, size_t ws_bytes, dllm_stream stream);

/* Step a3.  Block attention against the cached keys/values ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism"); the
 * two segments per sequence express the pruned suffix: a window after the
 * block plus the trailing position (Streaming-dLLM README, figure
 * "Illustration of approximated suffix pruning").  There is no log-sum-exp
 * output: no caller of the step needs it, and the key chunks of a row tile
 * are merged inside the kernel.
 * Non-causal GQA attention of n_rows query rows per sequence (q bf16
 * [b][Hq][n_rows][D]) against layer `layer` of the caches.  Query head h reads
 * kv head h/(Hq/Hkv).  Keys of sequence i: segs[i][j] = (start, len) for
 * j = 0,1 (device int32 [b][2][2]; len 0 = unused).  Scale 1/sqrt(D).
 * out bf16 [b*n_rows][Hq*D]. */
dllm_status dllm_block_attn(const dllm_config* cfg, int32_t layer, int32_t n_rows,
                            const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* segs, void* out, void* ws, size_t ws_bytes,
                            dllm_stream stream);

/* Step a4 (the backbone's attention output projection; the shapes are the
 * LLaDA-8B / Dream-7B-shaped workloads').
 * Output projection and residual: x += attn . Wo^T (fp32), xb = bf16(x),
 * row_sumsq (may be NULL) = the new residual's per-slice sums of squares. */
dllm_status dllm_o_proj(const dllm_config* cfg, const dllm_weights* w, int32_t layer,
                        const void* attn, int32_t row0, int32_t n_rows, float* x, void* xb,
                        float* row_sumsq, void* ws, size_t ws_bytes, dllm_stream stream);

/* LM-head input (the final norm, and the workloads' planted hidden state of a
 * masked row; no counterpart on the pages).
 * LM-head input of the block at block_start: for every sequence b and block
 * row i (position p = block_start+i, x row b*n_rows + p-row0):
 * h[b][i] = bf16(x / rms(x) + (masked[b][p] ? plants[b][p-P] : 0)).
 * x fp32 [b*n_rows][hidden]; h bf16 [b][B][hidden]. */
dllm_status dllm_final_norm(const dllm_config* cfg, const float* x, int32_t row0, int32_t n_rows,
                            int32_t block_start, const uint8_t* masked, const void* plants,
                            void* h, dllm_stream stream);

/* Step a5.  The confidence each masked position is committed on ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism").
 * The rows are given contiguous (the step's caller compacts them); there is
 * no row-index list.
 * LM head + confidence over the full vocabulary for n_rows rows of h (bf16
 * [n_rows][hidden]); no logits are written.  conf = max softmax probability,
 * tok = argmax (lowest id on ties), gap = top-1 minus top-2 logit (may be NULL). */
dllm_status dllm_lmhead_confidence(const dllm_config* cfg, const dllm_weights* w,
                                   const void* h, int32_t n_rows, float* conf, int32_t* tok,
                                   float* gap, void* ws, size_t ws_bytes, dllm_stream stream);

/* Largest n_rows dllm_lmhead_confidence_noalloc accepts. */
#define DLLM_NOALLOC_MAX_ROWS 256

/* The same computation as dllm_lmhead_confidence for callers that cannot
 * give the library any device memory (an allocator that owns the device pool
 * and forbids cudaMalloc on the request path, or a binding that passes only
 * tensors).  It allocates nothing and takes no workspace: its scratch is a
 * fixed 640 KiB array in the library's device image, held by every GPU that
 * loads the library until the process exits.  This call has no counterpart on
 * the method's pages; it only changes where the scratch lives.
 *  - n_rows must be <= DLLM_NOALLOC_MAX_ROWS; larger values return
 *    DLLM_ERR_UNSUPPORTED and launch nothing.
 *  - The first call on each device looks up the scratch's device address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *  - All calls share the one scratch array, whatever their stream: calls that
 *    overlap on the GPU race and give wrong results.  Each call writes every
 *    scratch entry it reads, so nothing needs clearing between calls.
 *  - conf/tok/gap as in dllm_lmhead_confidence (gap may be NULL).  This call
 *    has no workspace status word: if one of its bounded device waits gives
 *    up (about 2 s), every row of the call gets conf = gap = NaN and
 *    tok = -1, so the failure shows in the outputs themselves.  The call
 *    clears its own device status word first (a cudaMemsetAsync of 4 bytes of
 *    the library's static memory; nothing is allocated). */
dllm_status dllm_lmhead_confidence_noalloc(const dllm_config* cfg, const dllm_weights* w,
                                           const void* h, int32_t n_rows, float* conf,
                                           int32_t* tok, float* gap, dllm_stream stream);

/* Step a6.  The commit rule of "Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism":
 * positions whose confidence clears the threshold are committed and never
 * revised; a finished block's keys/values are then recomputed (the cache keeps
 * settled positions).
 * Commit of the block at block_start for every sequence (cfg->commit_mode;
 * THRESHOLD: masked rows with conf > tau commit, and the most confident
 * masked row always does, lowest position on ties).  conf/tok [b][B].
 * Updates tokens and masked.  Optional outputs (NULL to skip), all device:
 *  - commit [b][B] u8: 1 for the rows this call committed;
 *  - remaining [b]: rows of the block still masked;
 *  - block_done [b]: 1 when no row of the sequence's block is left masked;
 *  - refresh_list [b]: block_start when this call finished the sequence's
 *    block (some row was masked before it), so its keys/values are due for
 *    dllm_kv_cache_refresh; -1 otherwise. */
dllm_status dllm_threshold_commit(const dllm_config* cfg, int32_t block_start,
                                  const float* conf, const int32_t* tok, int32_t* tokens,
                                  uint8_t* masked, uint8_t* commit, int32_t* remaining,
                                  int32_t* block_done, int32_t* refresh_list,
                                  dllm_stream stream);

/* Step a8.  The cache a step reads from ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism";
 * Fast-dLLM README, "Quick Start": use_cache).
 * Fill the caches before decoding: PREFIX runs the prompt, DUAL and
 * DUAL_PRUNED run prompt plus mask tokens (whole sequence); NONE does nothing. */
dllm_status dllm_prefill(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                         void* ws, size_t ws_bytes, dllm_stream stream);

/* Steps a1-a6 as one denoising step ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism").
 * One denoising step of the block at block_start: embed, L layers, LM head,
 * commit.  The step's conf/tok/gap/commit, block-done flags and refresh list
 * stay in the workspace (dllm_step_outputs). */
dllm_status dllm_decode_step(const dllm_config* cfg, const dllm_weights* w,
                             const dllm_state* st, int32_t block_start, void* ws,
                             size_t ws_bytes, dllm_stream stream);

/* Step a7, the cache refresh of a finished block ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism";
 * same page, section "Fast-dLLM v1 Versus a Standard Diffusion Sampler").
 * Recompute the keys/values of a finished block from its committed tokens:
 * L layers with input embed[token], same key set as a step, no LM head. */
dllm_status dllm_kv_cache_refresh(const dllm_config* cfg, const dllm_weights* w,
                                  const dllm_state* st, int32_t block_start, void* ws,
                                  size_t ws_bytes, dllm_stream stream);

/* A block of the block schedule decoded to completion, then refreshed
 * ("Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism"; same page, section "Fast-dLLM v1
 * Versus a Standard Diffusion Sampler"; Fast-dLLM README, "Quick Start":
 * --block_size).
 * Decode one block to completion: steps until the commit step reports the
 * block done in every sequence (or max_steps), then the cache refresh.  Blocks
 * the calling host thread until the block is done; *steps_taken (host) gets
 * the count. */
dllm_status dllm_decode_block(const dllm_config* cfg, const dllm_weights* w,
                              const dllm_state* st, int32_t block_start, int32_t max_steps,
                              int32_t* steps_taken, void* ws, size_t ws_bytes,
                              dllm_stream stream);

/* The block schedule of "Fast-dLLM: Four Acceleration Tracks ...", section "The v1 Mechanism" run per
 * sequence: each sequence decodes its own blocks left to right.
 * Decode every block of every sequence, each sequence at its own block
 * (after dllm_prefill).  A pass runs one step for every sequence at its
 * current block.  The pass after the one whose commit finished a sequence's
 * block (the commit step's refresh list names that block) finds no masked
 * row in it and is that block's refresh (the rows, all committed, rewrite
 * their keys/values against the step's key set); the sequence then moves to
 * its next block.  A
 * finished sequence's passes recompute its last block (no state change).
 * Each sequence's tokens equal those of dllm_decode_block run block by block
 * with the batch in lockstep: sequences never interact.  Blocks the calling
 * host thread until done; *passes (host, may be NULL) gets the pass count.
 * NONE and PREFIX_SUFFIXQ caches return DLLM_ERR_UNSUPPORTED. */
dllm_status dllm_decode_all(const dllm_config* cfg, const dllm_weights* w, const dllm_state* st,
                            int32_t* passes, void* ws, size_t ws_bytes, dllm_stream stream);

/* Device pointers (into ws) of the last step's outputs: conf, tok, gap and
 * commit [b][B]; block_done and refresh_list [b], as dllm_threshold_commit
 * describes them.  Any output pointer may be NULL. */
dllm_status dllm_step_outputs(const dllm_config* cfg, void* ws, size_t ws_bytes, float** conf,
                              int32_t** tok, float** gap, uint8_t** commit, int32_t** block_done,
                              int32_t** refresh_list);

/* Copy the workspace's device status word to *code (host); synchronises stream.
 * The word is 0, or an OR of:
 *  - DLLM_DEVICE_TIMEOUT (1): a bounded device wait gave up (see
 *    dllm_selftest_wait_timeout); the kernel skipped the rest of its work.
 *  - DLLM_DEVICE_BAD_TOKEN (2): a token id outside [0, V) reached the
 *    embedding gather; row 0 of the table was read instead.
 *  - DLLM_DEVICE_INDEX (4): only in the DLLM_DEBUG build (libdllm_debug.so,
 *    built by build.py --debug).  A row position read from device memory (a
 *    per-sequence block start) was outside the sequence, and the access was
 *    skipped.  The other builds do not check these positions. */
#define DLLM_DEVICE_BAD_TOKEN 2
#define DLLM_DEVICE_INDEX 4
dllm_status dllm_device_status(void* ws, int32_t* code, dllm_stream stream);

/* Number of kernels this library has launched in this process (kernels run
 * by a replayed graph included). */
uint64_t dllm_launch_count(void);

/* dllm_prefill, dllm_decode_step, dllm_kv_cache_refresh and dllm_decode_block
 * record their launch sequence once per (configuration, weight, state and
 * workspace pointers, block) as a CUDA graph and replay it afterwards.  The
 * cache holds at most 256 graphs; this call destroys them all (call it before
 * freeing buffers that a cached graph references, or to bound memory). */
void dllm_graph_cache_clear(void);

/* L2 prefetch of upcoming weights inside the layer stack (a tuning knob; no
 * counterpart on the pages).  While layer l's attention runs, HBM has little
 * to do: the attention kernel asks L2 for layer l's W_o (attn_prefetch_wo != 0)
 * and the first attn_next_bytes of the weights read next (layer l+1's W_qkv,
 * or the LM head after the last layer of a step); layer l's O-projection asks
 * for the following oproj_next_bytes.  Only the cache is affected, never a
 * result.  Process-wide; clears the graph cache.  Negative sizes are
 * rejected (DLLM_ERR_INVALID).  Defaults: 8 MiB, 0, off. */
dllm_status dllm_set_l2_prefetch(int64_t attn_next_bytes, int64_t oproj_next_bytes,
                                 int32_t attn_prefetch_wo);

/* Persistent layer-stack kernel (a scheduling choice with no counterpart on
 * the pages; results follow the same definitions).  Off by default: on the
 * 8B-shaped workloads it measured 1.8-2x slower than the per-projection
 * kernels, because each hand-off between CTAs through global memory costs
 * more than a kernel boundary.  When switched on,
 * a decode step or a block refresh whose b*B rows fit 64 activation rows,
 * with head_dim 128, bf16 weights and a PREFIX, DUAL or DUAL_PRUNED cache,
 * runs all L layers in one launch with one CTA per SM (the device must have
 * at least 148 SMs; otherwise, and for every other shape, the per-projection
 * kernels run).  l2_lookahead: weight k-blocks (16 KB each) per CTA that the
 * kernel prefetches into L2 ahead of its shared-memory ring (0..4096,
 * default 16).  Process-wide; clears the graph cache.  enable = 0 restores
 * the default. */
dllm_status dllm_set_layer_stack(int32_t enable, int32_t l2_lookahead);

/* Host query (no GPU work): the layer-stack plan of a step of the block at
 * block_start.  info (host, 8 ints): [0] 1 if the shape qualifies, [1]
 * activation tile width, [2]/[3] CTAs sharing the Q/K/V / O-projection
 * weights, [4] key chunks per attention row tile, [5] 64-key tiles per chunk,
 * [6] attention units per layer, [7] 1 if every weight k-block of every
 * tile belongs to exactly one CTA share (a self-check of the partition). */
dllm_status dllm_layer_stack_plan(const dllm_config* cfg, int32_t block_start, int32_t* info);

/* Host query (no GPU work): the launch plan of the block attention
 * (dllm_block_attn's kernel as a decode step or the prefill runs it) for the
 * step of the block at block_start, or for the prefill when block_start < 0.
 * info (host, 8 ints): [0] query rows per tile (32: each row tile is loaded
 * four times and every warp takes a quarter of the keys and output columns;
 * 128: two threads per row), [1] row tiles per (sequence, kv head), [2] key
 * chunks per row tile (the cluster size), [3] 128-key tiles per chunk, [4]
 * CTAs, [5] the key-tile bound the plan is made for, [6] threads per CTA, [7]
 * K/V ring stages.  DLLM_ERR_INVALID for a block start that is not a block of
 * the generation, or a prefill of a cache mode that has none. */
dllm_status dllm_attention_plan(const dllm_config* cfg, int32_t block_start, int32_t* info);

/* Failure-detection self-test (no counterpart on the pages).  Launches one
 * CTA whose bounded device wait has nothing to wait for: after limit_us
 * microseconds (clamped to [1, 2000000]) it gives up and ORs
 * DLLM_DEVICE_TIMEOUT into *status (device int32), exactly as a wait inside
 * the decode kernels reports a stalled producer, and returns without a trap
 * or fault.  Lets tests check that a timed-out wait is reported and that the
 * context stays usable afterwards. */
#define DLLM_DEVICE_TIMEOUT 1
dllm_status dllm_selftest_wait_timeout(int32_t* status, int32_t limit_us, dllm_stream stream);

const char* dllm_status_string(dllm_status s);

#ifdef __cplusplus
}
#endif
#endif /* DLLM_H_ */
