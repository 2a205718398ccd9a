/*
 * orthrus.h -- C ABI of the B200 (sm_100a) hot path of one Orthrus
 * self-speculative decoding round.
 *
 * One round (Orthrus explainer, cjcn.com.cn, on arXiv:2605.12825, §四):
 *   1. diffusion view: the block [anchor, MASK x (blk-1)] attends to the frozen
 *      AR model's KV cache and, bidirectionally, to its own block K/V
 *      (orthrus_block_attn, ORTHRUS_BIDIR_BLOCK), per layer;
 *      LM-head logits -> orthrus_vocab_argmax -> drafts d[0..blk)
 *   2. AR view: [anchor, d0..d_{blk-2}] verified causally over the same cache
 *      (orthrus_block_attn, ORTHRUS_CAUSAL_VERIFY), per layer;
 *      logits -> orthrus_vocab_argmax -> a[0..blk)
 *   3. orthrus_consensus: accept the agreeing prefix plus one correction token
 *   4. orthrus_kv_commit: only the accepted rows' AR K/V enter the cache
 *
 * Conventions (all entry points):
 *   - Every pointer is caller-owned device memory unless stated otherwise; the
 *     library allocates nothing and keeps no state between calls other than
 *     the zero-initialised workspaces the caller passes in.
 *   - Calls are asynchronous on `stream` (NULL = legacy default stream) and
 *     never synchronise it.  Lengths (ctx_lens, n_emit) stay on the device, so
 *     a whole round can be captured in one CUDA graph.
 *   - Arguments the host can check are checked before any launch; a bad one
 *     returns a negative status and launches nothing.  Conditions only the
 *     device can see (a device-resident length out of range) set the optional
 *     device error word `err` (first error code wins) and skip the affected
 *     sequence's writes; kernels never trap.
 *   - Workspaces: query the size and allocate it once.  Workspaces hold
 *     ticket or arrival counters: zero them once (cudaMemset 0); the kernels
 *     leave the counters at zero again, so the buffer serves every later call
 *     on the same stream (zero it again after a call that reported an
 *     error).  Calls that may run at the same time (different streams) need
 *     separate workspaces.
 *   - Tensors are dense, row-major, with the layouts written next to each
 *     field.  dtype applies to every floating-point tensor of a call.
 */
#ifndef ORTHRUS_H
#define ORTHRUS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORTHRUS_VERSION 10000 /* major*10000 + minor*100 + patch */

typedef struct CUstream_st* orthrus_stream_t; /* same type as cudaStream_t */

typedef enum {
  ORTHRUS_OK = 0,
  ORTHRUS_EINVAL = -1,       /* null pointer, negative size, bad enum */
  ORTHRUS_EUNSUPPORTED = -2, /* valid but not implemented (D, G*blk, ...) */
  ORTHRUS_EWORKSPACE = -3,   /* workspace missing or too small */
  ORTHRUS_ECAPACITY = -4,    /* a length exceeds the cache capacity */
  ORTHRUS_ECUDA = -5,        /* a CUDA launch or attribute call failed */
  ORTHRUS_ETIMEOUT = -6      /* device error word only: a bounded wait inside a
                                kernel gave up; that call's outputs are not valid */
} orthrus_status;

typedef enum { ORTHRUS_F32 = 0, ORTHRUS_BF16 = 1 } orthrus_dtype;

typedef enum {
  /* Diffusion view (explainer §二 and §三): every block row sees the cache
   * rows [0, n) -- the context before the anchor -- and all blk block rows. */
  ORTHRUS_BIDIR_BLOCK = 0,
  /* AR verify view (explainer §四 step 2): block row i sees cache rows
   * [0, n) and block rows [0, i]; row i equals a single-token decode at
   * absolute position n + i. */
  ORTHRUS_CAUSAL_VERIFY = 1
} orthrus_mask_mode;

typedef enum {
  /* The kernel that immediately precedes this call on the stream does not
   * write k_cache, v_cache or ctx_lens.  BF16 calls then start streaming the
   * cache while that kernel is still finishing (programmatic dependent
   * launch); q, k_blk and v_blk are still read only after it has completed.
   * Without the flag every input is read after the preceding work finishes. */
  ORTHRUS_ATTN_EARLY_KV = 1
} orthrus_attn_flags;

/* ------------------------------------------------------------------------
 * Block attention (both views), one layer.
 *
 * For sequence b (context n = ctx_lens[b]), block row i in [0, blk) and query
 * head h, with kv-head g = h / (Hq / Hkv):
 *   out[b,i,h,:] = sum_j softmax_j(scale * q[b,i,h,:] . k_j) v_j
 * over the visible keys j of the mask mode, where key positions [0, n) come
 * from k_cache/v_cache[b,g,0:n,:] and positions n + r from k_blk/v_blk[b,r,g,:].
 *
 * Arithmetic: F32 tensors -> FP32 FMA on CUDA cores, split-KV by absolute key
 * position (fixed 256-key chunks) with a fixed-order combine, so a causal row
 * reproduces single-token decoding bit for bit.  BF16 tensors -> tcgen05
 * tensor-core tiles (bf16 products, FP32 accumulation, bf16 softmax weights),
 * FP32 online softmax, bf16 output.
 * ---------------------------------------------------------------------- */
typedef struct orthrus_attn_args {
  int32_t dtype;     /* orthrus_dtype of q, k_blk, v_blk, caches and out */
  int32_t mask_mode; /* orthrus_mask_mode */
  int32_t B;         /* sequences (0 = nothing to do) */
  int32_t Hq, Hkv;   /* query heads, kv heads; Hq % Hkv == 0 */
  int32_t D;         /* head dim: 64 or 128 */
  int32_t blk;       /* block rows, 1..32; (Hq/Hkv)*blk <= 128 */
  int32_t cap;       /* cache rows per (sequence, kv-head) */
  int32_t max_ctx;   /* host bound on every ctx_lens[b]; 0 <= max_ctx <= cap.
                        Sizes the grid; a device length above it is an error. */
  float scale;       /* softmax scale, finite and > 0; usually 1/sqrt(D) */
  int32_t flags;     /* bitwise OR of orthrus_attn_flags (0 = none) */
  const void* q;       /* [B, blk, Hq, D] */
  const void* k_blk;   /* [B, blk, Hkv, D] block K (bidir: diffusion K_diff; causal: AR K) */
  const void* v_blk;   /* [B, blk, Hkv, D] */
  const void* k_cache; /* [B, Hkv, cap, D] frozen AR K cache, rows [0, n) valid */
  const void* v_cache; /* [B, Hkv, cap, D] */
  const int32_t* ctx_lens; /* [B] device, committed context length n per sequence */
  void* out;           /* [B, blk, Hq, D], same dtype as q */
  int32_t* err;        /* optional device int32 error word (NULL = none) */
  void* workspace;     /* >= orthrus_block_attn_workspace() bytes, 256-byte aligned,
                          zeroed once (see below) */
  size_t workspace_bytes; /* size of the caller's buffer */
  /* Optional L2 warm-up for the call that follows this one on the stream
   * (the next layer of the same view, say): its K and V caches, with this
   * call's B, Hkv, cap, D and lengths.  NULL = none.  The BF16 tensor-core
   * path then prefetches, while it runs, the rows [0, ctx_lens[b]) of those
   * caches into L2 (each CTA its own tiles' rows, after issuing its last load
   * of this call's cache), so HBM keeps streaming across the boundary between
   * the two calls.  A hint only: the results of both calls are unchanged, and
   * the FP32 path ignores it.  16-byte aligned. */
  const void* next_k_cache;
  const void* next_v_cache;
} orthrus_attn_args;

/* Workspace of orthrus_block_attn: the per-split partial results of the
 * split-KV reduction (unnormalised O plus row max and row sum), written and
 * read back within the call.  The BF16 tensor-core path also keeps, in the
 * buffer's first 2048 bytes, the state of its in-launch merge (a 64-bit
 * generation and arrival count per (sequence, kv-head)): zero the buffer
 * once (cudaMemset 0); every call leaves each count at zero and moves the
 * generations it used on by one, so one buffer serves any later FP32 and
 * BF16 calls on one stream whose sizes fit it (zero it again after a call
 * that reported an error).
 * A BF16 call whose grid fits one wave (see orthrus_block_attn_plan) counts
 * on all of its CTAs being resident together: do not run it concurrently
 * with kernels (other streams) that could hold SMs until it ends -- the
 * merge's wait would give up after about a second and report
 * ORTHRUS_ETIMEOUT. */

/* Bytes of workspace orthrus_block_attn needs for these arguments (0 if none).
 * Pointers in `a` are not read.  Returns 0 for invalid shapes as well. */
size_t orthrus_block_attn_workspace(const orthrus_attn_args* a);

int orthrus_block_attn(const orthrus_attn_args* a, orthrus_stream_t stream);

/* Number of kernel launches one orthrus_block_attn call with these arguments
 * issues (for launch accounting); 0 for invalid shapes or B == 0. */
int orthrus_block_attn_launches(const orthrus_attn_args* a);

/* Launch plan of the BF16 tensor-core path for a GPU with `sms` SMs (host
 * only; pointers in `a` are not read).  The keys of each (sequence, kv-head)
 * -- cache[0, max_ctx) in 128-key tiles, then one tile of block rows -- are
 * dealt over S splits, one CTA each; the splits' partial results are merged
 * in split order.  out[0..8) = S, grid x, y, z (Hkv, B, S), threads per CTA,
 * dynamic shared memory bytes, most tiles one split streams, and 1 if the
 * merge runs inside the one launch (the grid fits one wave of one CTA per SM:
 * B * Hkv * S <= sms and B * Hkv <= 256) or 0 if a second, PDL-chained
 * kernel merges.  ORTHRUS_EUNSUPPORTED when the call would take the FP32
 * path. */
int orthrus_block_attn_plan(const orthrus_attn_args* a, int32_t sms, int32_t* out);

/* ------------------------------------------------------------------------
 * Vocab-row argmax (explainer §四: "the token that should most appear here").
 * idx[r] = smallest j with logits[r*row_stride + j] == max_k logits[r*row_stride + k];
 * NaN never wins; an all-NaN row gives 0; -0.0 and +0.0 are equal.
 * maxval (nullable) receives the winning value as float (bf16 widened exactly).
 * dtype: ORTHRUS_F32 or ORTHRUS_BF16; rows >= 0, vocab >= 1, row_stride >= vocab.
 * ---------------------------------------------------------------------- */
size_t orthrus_vocab_argmax_workspace(int32_t rows);

int orthrus_vocab_argmax(int32_t dtype, const void* logits, int32_t rows,
                         int32_t vocab, int64_t row_stride, int32_t* idx,
                         float* maxval, void* workspace, size_t workspace_bytes,
                         orthrus_stream_t stream);

/* Scratch-free variant of orthrus_vocab_argmax, for callers that cannot
 * allocate device memory (no allocator available or allowed where they run,
 * e.g. code handed only the tensors it works on, or a process whose device
 * memory is fully reserved).  The pages describe no such entry point; it is
 * a property of this library only.  Same arguments and results as
 * orthrus_vocab_argmax minus the workspace: the per-row scratch (12 bytes a
 * row) lives in a static device array of ORTHRUS_NOALLOC_ARGMAX_MAX_ROWS rows
 * that every GPU loading the library holds until the process exits.
 *   - rows > ORTHRUS_NOALLOC_ARGMAX_MAX_ROWS returns ORTHRUS_EUNSUPPORTED.
 *   - Allocates nothing (no cudaMalloc/cudaFree); each call clears the rows it
 *     uses with cudaMemsetAsync on `stream`, then launches the argmax kernel.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress); make that first call before any stream capture.
 *     The address is kept with the context it came from and looked up again
 *     when the current context differs (after a device reset, for example);
 *     that later lookup is again a call to make outside stream capture.
 *   - Every call shares the one array: calls that overlap on the GPU (other
 *     streams, other threads) race and give wrong indices; serialise them. */
#define ORTHRUS_NOALLOC_ARGMAX_MAX_ROWS 4096
int orthrus_vocab_argmax_noalloc(int32_t dtype, const void* logits, int32_t rows,
                                 int32_t vocab, int64_t row_stride, int32_t* idx,
                                 float* maxval, orthrus_stream_t stream);

/* ------------------------------------------------------------------------
 * Prefix consensus (explainer §四 step 3), per sequence b:
 *   accept_len[b]  = first j with draft[b,j] != verify[b,j], else blk
 *   n_emit[b]      = min(accept_len[b] + 1, blk)        (always >= 1)
 *   emitted[b,j]   = verify[b,j] for j < n_emit[b], else -1
 *   next_anchor[b] = verify[b, n_emit[b] - 1]
 * draft/verify [B, blk] int32 device; 1 <= blk <= 32.  Any output pointer
 * except n_emit may be NULL.
 * ---------------------------------------------------------------------- */
int orthrus_consensus(const int32_t* draft, const int32_t* verify, int32_t B,
                      int32_t blk, int32_t* accept_len, int32_t* n_emit,
                      int32_t* emitted, int32_t* next_anchor,
                      orthrus_stream_t stream);

/* ------------------------------------------------------------------------
 * KV commit / rollback for all layers in one launch (explainer §四 step 3
 * "update the notebook"; §七: the block is the only extra state).  For every
 * layer l, sequence b (n = ctx_lens[b], e = n_emit[b]) and kv-head g:
 *   cache_l[b, g, n + r, :] = blk_l[b, r, g, :]   for r in [0, e)
 * then ctx_lens[b] = n + e.  Rows r >= e are never written (that is the
 * rollback); e == 0 changes nothing.  If n + e > cap or e is outside
 * [0, blk], sequence b is skipped and `err` gets ORTHRUS_ECAPACITY.
 * ---------------------------------------------------------------------- */
typedef struct orthrus_commit_args {
  int32_t dtype;   /* element type of caches and blocks */
  int32_t layers;  /* >= 1 */
  int32_t B, Hkv, D, blk, cap;
  void* k_cache;   /* layer l at k_cache + l*cache_layer_stride: [B, Hkv, cap, D] */
  void* v_cache;
  int64_t cache_layer_stride; /* elements; >= B*Hkv*cap*D */
  const void* k_blk; /* layer l at k_blk + l*blk_layer_stride: [B, blk, Hkv, D] */
  const void* v_blk;
  int64_t blk_layer_stride;   /* elements; >= B*blk*Hkv*D */
  int32_t* ctx_lens;          /* [B] device, in/out */
  const int32_t* n_emit;      /* [B] device */
  int32_t* err;               /* optional device error word */
  void* workspace;            /* zero-initialised, orthrus_kv_commit_workspace() bytes */
  size_t workspace_bytes;
} orthrus_commit_args;

size_t orthrus_kv_commit_workspace(const orthrus_commit_args* a);

int orthrus_kv_commit(const orthrus_commit_args* a, orthrus_stream_t stream);

/* ------------------------------------------------------------------------
 * Stochastic consensus (explainer §四: for sampling with a temperature the
 * framework aligns the two views' distributions by strict rejection
 * sampling, which keeps decoding lossless).  Per sequence, with
 * q_j = softmax(z_diff[j] / T) and p_j = softmax(z_ar[j] / T):
 *   drafts      d_j ~ q_j                               (orthrus_vocab_sample)
 *   accept      d_j while u_j < p_j(d_j) / q_j(d_j), left to right
 *   correction  at the first rejected position L: c ~ normalize(max(0, p_L - q_L))
 *   emit        d_0 .. d_{L-1}, c (n_emit = L + 1), or all blk drafts when every
 *               one is accepted (n_emit = min(L + 1, blk), as in the greedy rule)
 * Sampling from a softmax uses Gumbel-max: argmax_k x_k + g_k with
 * g_k = -log(-log u_k).  Uniforms: Philox4x32-10 (Salmon et al., SC'11) with
 * key = seed (low, high 32 bits) and counter (x0, x1, purpose, step):
 * purpose 1 draft noise (x0 = vocab index / 4, x1 = row, word = index % 4),
 * purpose 2 acceptance (x0 = block position, x1 = sequence, word 0), purpose 3
 * correction noise (x0 = vocab index / 4, x1 = sequence); a word w becomes
 * u = ((w >> 9) + 1/2) 2^-23 (exact in FP32).  `step` must differ between rounds.  z / T is an
 * FP32 division; reductions are FP32.
 * ---------------------------------------------------------------------- */

/* Draft sampling, with the draft's log-probability from the same read:
 *   idx[r]     = argmax_k logits[r, k] / T + g_k (purpose 1, x1 = r), lowest
 *                index on equal keys
 *   lse[r]     = log sum_k exp(logits[r, k] / T)          (nullable)
 *   logprob[r] = logits[r, idx[r]] / T - lse[r]           (nullable)
 * temperature > 0 and finite; vocab <= 2^30.  Grid: 4096-element chunks x
 * rows; each CTA folds its best key into the row's slot with an atomic max
 * and, when lse or logprob is wanted, stores its chunk's maximum and sum of
 * exponentials; the row's last CTA writes idx and merges the chunk pairs in
 * a fixed order.  workspace: orthrus_vocab_sample_workspace(rows, vocab)
 * bytes, 16-byte aligned, zeroed once; every call leaves it all zero. */
size_t orthrus_vocab_sample_workspace(int32_t rows, int32_t vocab);
int orthrus_vocab_sample(int32_t dtype, const void* logits, int32_t rows, int32_t vocab,
                         int64_t row_stride, float temperature, uint64_t seed, uint32_t step,
                         int32_t* idx, float* logprob, float* lse, void* workspace,
                         size_t workspace_bytes, orthrus_stream_t stream);

/* Log-probability of a chosen token per row at temperature T:
 *   lse[r]     = log sum_k exp(logits[r, k] / T)
 *   logprob[r] = logits[r, idx[r]] / T - lse[r]
 * idx int32 [rows] device, each in [0, vocab) (else logprob[r] = NaN); lse
 * nullable.  Rows are cut into 4096-element chunks; each chunk's maximum and
 * sum of exp(z/T - max) are reduced in FP32 in a fixed order and the chunks
 * are merged in index order, so the result depends only on the row.  T = 1
 * gives the plain log-softmax the precision study uses (the reproduction "How
 * Lossless Is Lossless Speculative Decoding? The Role of Numerical Precision
 * in Orthrus", abstract, relates exact trajectory matching to the reference's
 * perplexity).  workspace: orthrus_token_logprob_workspace(rows, vocab) bytes,
 * 16-byte aligned, zeroed once: every call leaves it all zero, so one buffer
 * serves later calls of any shape on the same stream. */
size_t orthrus_token_logprob_workspace(int32_t rows, int32_t vocab);
int orthrus_token_logprob(int32_t dtype, const void* logits, int32_t rows, int32_t vocab,
                          int64_t row_stride, const int32_t* idx, float temperature,
                          float* logprob, float* lse, void* workspace, size_t workspace_bytes,
                          orthrus_stream_t stream);

typedef struct orthrus_sample_args {
  int32_t dtype;          /* of both logit matrices */
  int32_t B, blk, vocab;  /* 1 <= blk <= 32, B * blk <= 65535, vocab <= 2^30 */
  int64_t row_stride;     /* elements between logit rows, >= vocab */
  float temperature;      /* > 0 */
  uint32_t step;
  uint64_t seed;
  const int32_t* draft;   /* [B, blk] d_j: orthrus_vocab_sample of logits_diff ... */
  const float* logq;      /* [B*blk] log q_j(d_j): ... its logprob output */
  const float* lse_diff;  /* [B*blk] log-sum-exp of logits_diff / T: ... its lse output */
  const void* logits_ar;  /* [B*blk, vocab] row b*blk + j: AR view */
  const void* logits_diff;/* [B*blk, vocab] diffusion view */
  float* logp;            /* out [B*blk] log p_j(d_j) */
  float* lse_ar;          /* out [B*blk] log-sum-exp of logits_ar / T */
  int32_t* accept_len;    /* out [B] L */
  int32_t* n_emit;        /* out [B] */
  int32_t* emitted;       /* out [B, blk] (nullable), -1 past n_emit */
  int32_t* next_anchor;   /* out [B] (nullable) */
  void* workspace;        /* orthrus_consensus_sample_workspace(B, blk, vocab) bytes,
                             16-byte aligned, zeroed once; left all zero */
  size_t workspace_bytes;
} orthrus_sample_args;

/* Outputs as orthrus_consensus.  Two launches.  (1) Grid 4096-element chunks
 * x rows over logits_ar: log p_j(d_j) and the row's log-sum-exp (chunk pairs
 * merged in a fixed order by the row's last CTA); the CTA that completes a
 * sequence's last row then runs its acceptance test in one warp.  (2) Grid
 * chunks x sequences: Gumbel-max over the rejected row's max(0, p - q),
 * folded per sequence with an atomic max; the last CTA writes the
 * correction.  When no token has p > q at the rejected position (impossible
 * in exact arithmetic) the correction is argmax p. */
size_t orthrus_consensus_sample_workspace(int32_t B, int32_t blk, int32_t vocab);
int orthrus_consensus_sample(const orthrus_sample_args* a, orthrus_stream_t stream);

/* ------------------------------------------------------------------------
 * LM head with the argmax in its epilogue (the output projection every view
 * ends in -- explainer §二: the LM head is shared -- followed by the row
 * argmax that gives the drafts and the AR tokens, §四 steps 1-3):
 *   idx[r]    = argmax_v sum_k h[r, k] w[v, k]   lowest index among equal maxima
 *   maxval[r] = that maximum                     (nullable)
 * h [rows, d] bf16, row r at h + r * h_row_stride (elements); w [vocab, d]
 * bf16, dense (the PyTorch Linear layout of the LM head).  The logits never
 * reach memory: a tcgen05 GEMM (all hidden rows x one vocabulary tile of
 * 128-256 rows, fp32 accumulation in TMEM) reduces each tile to per-row bests
 * in its epilogue.  The dot products are fp32 sums of exact bf16 products in the
 * tensor core's order, so an argmax whose top two logits lie within fp32
 * rounding may differ from an exact evaluation; the index returned is then
 * one of the near-maxima.
 * Limits: dtype ORTHRUS_BF16 (ORTHRUS_F32: ORTHRUS_EUNSUPPORTED); 1 <= rows
 * <= 128 (0: no-op); d a multiple of 64; h_row_stride >= d and a multiple of
 * 8; vocab <= 2^30; h and w 16-byte aligned.  err (nullable) receives
 * ORTHRUS_ETIMEOUT if a bounded wait inside the kernel gave up.
 * workspace: orthrus_lm_head_argmax_workspace(rows) bytes, 16-byte aligned,
 * zeroed once; every call leaves it zero.  One launch, one CTA per SM.  w is
 * read before the wait on the preceding kernel on the stream (it may not be
 * written by the kernel right before this call); h only after it.
 * ---------------------------------------------------------------------- */
size_t orthrus_lm_head_argmax_workspace(int32_t rows);
/* The launch orthrus_lm_head_argmax would make for these sizes on a GPU with
 * `sms` SMs (host only, no device needed): out[0..8) = vocabulary rows per
 * tile, 64-column boxes per stage, stages, TMEM h slots, dynamic shared
 * memory bytes, grid, tiles, TMEM columns.  ORTHRUS_EINVAL outside the
 * limits above. */
int orthrus_lm_head_argmax_plan(int32_t rows, int32_t d, int32_t vocab, int32_t sms,
                                int32_t* out);
int orthrus_lm_head_argmax(int32_t dtype, const void* h, int32_t rows, int32_t d,
                           int64_t h_row_stride, const void* w, int32_t vocab, int32_t* idx,
                           float* maxval, int32_t* err, void* workspace,
                           size_t workspace_bytes, orthrus_stream_t stream);

/* ------------------------------------------------------------------------
 * Projection on the tensor cores: the attention block's QKV and output
 * projections around the round's attention (explainer §二: the diffusion
 * view has its own copy of the attention projections, the AR view uses the
 * frozen model's), for the few rows of a decoding block:
 *   y[r, n] = bf16( sum_k x[r, k] w[n, k] )                  residual == NULL
 *   y[r, n] = bf16( residual[r, n] + bf16(sum_k x[r, k] w[n, k]) )
 * x [rows, K] (row pitch ldx elements), w [N, K] dense (the PyTorch Linear
 * layout), residual and y [rows, N] (row pitch ldy; y may alias residual).
 * The sum is an fp32 accumulation of exact bf16 products on the tensor cores
 * (128 output features per tile; a tile's K range split over several CTAs
 * whose fp32 partials are added in a fixed order), so the result does not
 * depend on timing but may differ from an exactly rounded product by one
 * bf16 step.  w is read before the wait on the preceding kernel (it may not
 * be written by the kernel right before this call on the stream); x and the
 * residual only after it.
 * Limits: dtype ORTHRUS_BF16 (ORTHRUS_F32: ORTHRUS_EUNSUPPORTED);
 * 1 <= rows <= 128 (0: no-op); K a multiple of 64; ldx a multiple of 8;
 * x, w 16-byte aligned.  err (nullable) receives ORTHRUS_ETIMEOUT if a
 * bounded wait inside the kernel gave up.  workspace:
 * orthrus_linear_tc_workspace(rows, K, N) bytes, 256-byte aligned, zeroed
 * once; every call leaves its ticket counters zero.  One launch.
 * l2_next / l2_next_bytes (optional; NULL / 0 for none): a hint naming
 * device memory a later call reads (say the next projection's weights);
 * once its own loads are issued, each CTA prefetches its share of it into
 * L2.  It changes no result.  Address and size multiples of 16, else
 * ORTHRUS_EINVAL.
 * ---------------------------------------------------------------------- */
size_t orthrus_linear_tc_workspace(int32_t rows, int32_t K, int32_t N);
/* The launch for these sizes on a GPU with `sms` SMs (host only): out[0..8)
 * = 128-feature tiles, K splits per tile, ring stages, bytes per stage,
 * dynamic shared memory, grid, TMEM columns, rows rounded up to 16.
 * ORTHRUS_EINVAL outside the limits above. */
int orthrus_linear_tc_plan(int32_t rows, int32_t K, int32_t N, int32_t sms, int32_t* out);
int orthrus_linear_tc(int32_t dtype, const void* x, int32_t rows, int32_t K, int64_t ldx,
                      const void* w, int32_t N, const void* residual, void* y, int64_t ldy,
                      const void* l2_next, int64_t l2_next_bytes, int32_t* err,
                      void* workspace, size_t workspace_bytes, orthrus_stream_t stream);

/* RoPE cos/sin table for the rows of B blocks of blk rows (row r = b*blk + j
 * at absolute position ctx_lens[b] + j, read on the device):
 *   cos_sin[(r * hd/2 + i) * 2 + 0] = cos(pos * theta^(-2i/hd)),  [.. + 1] = sin(..)
 * for i < hd/2, the angle and its cosine and sine in double, rounded to
 * float: the values orthrus_qkv_rope (orthrus_decoder.h) uses.  cos_sin:
 * B*blk*hd floats, 8-byte aligned.  hd even, theta > 0.  One launch. */
int orthrus_rope_table(const int32_t* ctx_lens, int32_t B, int32_t blk, int32_t hd, double theta,
                       float* cos_sin, orthrus_stream_t stream);

/* The QKV projection with RoPE and the head split in its epilogue (the input
 * side of each layer's attention; explainer §二): for the rows r of x,
 *   qkv[r, :] = bf16( sum_k x[r, k] w[n, k] ),  w [(Hq + 2 Hkv) * hd, K]
 * as orthrus_linear_tc computes it, then
 *   q[r, h, :] = RoPE(qkv[r, h*hd .. h*hd + hd)),          h < Hq
 *   k[r, g, :] = RoPE(qkv[r, (Hq + g)*hd ..)),             g < Hkv
 *   v[r, g, :] =      qkv[r, (Hq + Hkv + g)*hd ..)
 * with the rotation of the pairs (i, i + hd/2) by cos_sin (orthrus_rope_table
 * for the same rows) -- the same bits as orthrus_linear_tc followed by
 * orthrus_qkv_rope, in one launch.  q [rows, Hq, hd], k and v [rows, Hkv, hd]
 * dense bf16.  Limits: dtype ORTHRUS_BF16, hd == 128 (one 128-feature tile
 * is one head; otherwise ORTHRUS_EUNSUPPORTED), the rest (the L2 hint
 * included) as orthrus_linear_tc; workspace: orthrus_linear_tc_workspace(
 * rows, K, (Hq + 2 Hkv) * hd) bytes, same rules. */
int orthrus_linear_tc_qkv_rope(int32_t dtype, const void* x, int32_t rows, int32_t K,
                               int64_t ldx, const void* w, int32_t Hq, int32_t Hkv, int32_t hd,
                               const float* cos_sin, void* q, void* k, void* v,
                               const void* l2_next, int64_t l2_next_bytes, int32_t* err,
                               void* workspace, size_t workspace_bytes,
                               orthrus_stream_t stream);

/* ------------------------------------------------------------------------
 * Self-test of the bounded waits (failure detection without a fault): one
 * launch whose single wait never completes -- which = 0: an mbarrier phase
 * nothing arrives on (the form of every TMA / MMA handshake in the kernels);
 * which = 1: a generation word at `never` (device memory, 4-byte aligned,
 * left unchanged by the caller meanwhile) that nothing advances (the form of
 * the attention kernel's split-merge barrier).  After timeout_us
 * microseconds (1 .. 10^7) the wait gives up, ORTHRUS_ETIMEOUT goes to *err
 * (device memory) and the kernel returns; the context stays usable.  Returns
 * ORTHRUS_EINVAL for other arguments.
 * ---------------------------------------------------------------------- */
int orthrus_selftest_bounded_wait(int32_t which, uint32_t timeout_us, const uint32_t* never,
                                  int32_t* err, orthrus_stream_t stream);

/* ------------------------------------------------------------------------ */
const char* orthrus_status_str(int status);
int orthrus_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ORTHRUS_H */
