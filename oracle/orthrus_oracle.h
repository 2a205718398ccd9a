/*
 * orthrus_oracle.h -- plain, slow, obviously-correct CPU oracle for one
 * Orthrus self-speculative decoding round (block attention in both mask
 * modes, vocab argmax, prefix consensus, KV commit) and for a tiny
 * Qwen3-style decoder used to check the consensus loop end to end.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or call this code: only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no source with the CUDA
 * library.
 *
 * Sources (the method has no code on its pages; every function restates a
 * passage in its own words):
 *   [EXPLAINER] news explainer of "Orthrus" (arXiv:2605.12825), cjcn.com.cn:
 *       §二 (two heads share one KV notebook; diffusion-head attention is
 *            Q_diff over concat(K_AR,V_AR cache) and (K_diff,V_diff) of the block)
 *       §三 (training masks: AR causal; a diffusion query sees the AR context
 *            before its block's anchor plus its own block, bidirectionally)
 *       §四 (inference: 32-slot draft, AR verify of 32 positions, left-to-right
 *            consensus, correction token, KV notebook update; >= 1 token/round)
 *       §七 (block state is a constant ~4.5 MiB extra KV)
 *   [REPRO] "How Lossless Is Lossless Speculative Decoding? The Role of
 *       Numerical Precision in Orthrus" (arXiv 2609.15504), abstract:
 *       FP32 gives exact trajectory match with AR greedy decoding.
 *
 * Arithmetic: every floating-point reduction accumulates in double; bf16
 * inputs are widened exactly (bits << 16).  Loops run in the order the
 * definition is written; OpenMP only splits independent (row, head) work, so
 * the per-row arithmetic does not depend on the thread count.
 *
 * Parity pins: every function here is pinned by tests in tests/test_oracle_*.py
 * (closed forms, brute force, invariants); none is "parity unpinned".
 */
#ifndef ORTHRUS_ORACLE_H
#define ORTHRUS_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F64 = 2 /* argmax only */ };
enum { ORACLE_BIDIR_BLOCK = 0, ORACLE_CAUSAL_VERIFY = 1 };

/* Block attention for one round (both views).
 * q      [B, blk, Hq, D]   (dtype)
 * k_blk  [B, blk, Hkv, D]  v_blk same
 * k_cache[B, Hkv, cap, D]  v_cache same; rows [0, ctx_lens[b]) are valid
 * out    [B, blk, Hq, D]   double
 * Query head h reads kv-head h / (Hq/Hkv).
 * bidir : row i sees cache[0,n) and block rows [0, blk)
 * causal: row i sees cache[0,n) and block rows [0, i]
 * Returns 0, or -1 on a bad argument. */
int oracle_block_attn(int dtype, int mask_mode, int B, int Hq, int Hkv, int D,
                      int blk, const void* q, const void* k_blk,
                      const void* v_blk, const void* k_cache,
                      const void* v_cache, int cap, const int32_t* ctx_lens,
                      double scale, double* out, int nthreads);

/* Row argmax with lowest-index tie-break; NaN never wins; an all-NaN row
 * gives 0.  logits row r starts at element r*row_stride.  maxval may be NULL
 * (else it receives the winning value, widened). */
int oracle_vocab_argmax(int dtype, const void* logits, int rows, int vocab,
                        int64_t row_stride, int32_t* idx, double* maxval);

/* Prefix consensus per sequence (draft, verify: [B, blk]).
 * accept_len = first j with draft[j] != verify[j], else blk
 * n_emit     = min(accept_len + 1, blk)
 * emitted[j] = verify[j] for j < n_emit, -1 otherwise
 * next_anchor= verify[n_emit - 1] */
int oracle_consensus(const int32_t* draft, const int32_t* verify, int B,
                     int blk, int32_t* accept_len, int32_t* n_emit,
                     int32_t* emitted, int32_t* next_anchor);

/* KV commit of one layer: cache rows [n, n + n_emit[b]) <- block rows
 * [0, n_emit[b]) for every kv-head, then ctx_lens[b] += n_emit[b].
 * Element size 4 (f32) or 2 (bf16); copies bytes, no arithmetic. */
int oracle_kv_commit(int dtype, void* k_cache, void* v_cache,
                     const void* k_blk, const void* v_blk, int B, int Hkv,
                     int D, int cap, int blk, int32_t* ctx_lens,
                     const int32_t* n_emit);

/* ---- tiny Qwen3-style decoder (for the end-to-end consensus check) ----
 * Weights: one flat double array, packed in this order (W[out][in], row-major):
 *   embed [V][d]
 *   per layer l in [0, L):
 *     attn_norm [d]
 *     wq [Hq*hd][d], wk [Hkv*hd][d], wv [Hkv*hd][d], wo [d][Hq*hd]   (AR view)
 *     dq [Hq*hd][d], dk [Hkv*hd][d], dv [Hkv*hd][d], do [d][Hq*hd]   (diffusion copy)
 *     ffn_norm [d]
 *     w_gate [ffn][d], w_up [ffn][d], w_down [d][ffn]
 *   final_norm [d]
 *   lm_head [V][d]
 * Cache of one sequence: k_cache/v_cache [L][Hkv][cap][hd] double (post-RoPE K). */
typedef struct {
  int V, d, L, Hq, Hkv, hd, ffn;
  double eps, rope_theta;
} oracle_model_cfg;

int64_t oracle_model_num_weights(const oracle_model_cfg* c);

/* Forward `rows` tokens at absolute positions [n, n + rows) over a sequence
 * whose cache holds rows [0, n).  view 0 = AR weights with causal mask
 * (prefill, decode, verify); view 1 = diffusion attention copy with the
 * bidirectional block mask.  Writes logits [rows][V] and, when k_blk/v_blk
 * are non-NULL, the block's K (post-RoPE) and V per layer: [L][rows][Hkv][hd].
 * Each row's arithmetic is the same routine whatever `rows` is. */
int oracle_model_forward(const oracle_model_cfg* c, const double* w, int view,
                         const int32_t* tokens, int rows,
                         const double* k_cache, const double* v_cache, int cap,
                         int n, double* logits, double* k_blk, double* v_blk,
                         int nthreads);

#ifdef __cplusplus
}
#endif
#endif
