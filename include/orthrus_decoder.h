/* orthrus_decoder.h -- C ABI of the decoder building blocks that run the
 * Orthrus consensus loop end to end on a small Qwen3-style decoder.
 *
 * The method (cjcn.com.cn explainer of "Orthrus", §二) keeps a frozen
 * autoregressive decoder and adds, per layer, a separate-weight copy of the
 * attention projections that serves the diffusion view; everything else
 * (embedding, norms, FFN, LM head, the KV cache) is shared.  The explainer
 * does not spell out the decoder itself; the layer used here is the Qwen3
 * pattern the pages' models belong to:
 *
 *   x = embed[token]
 *   per layer:  h = RMSNorm(x) ; q,k,v = h Wq/Wk/Wv (view's copy) ; RoPE(q,k)
 *               x = x + Attn(q, cache ‖ block k/v) Wo (view's copy)
 *               h = RMSNorm(x) ; x = x + (silu(h Wg) * (h Wu)) Wd
 *   logits = RMSNorm(x) Wlm
 *
 * where Attn is orthrus_block_attn (orthrus.h).  These entry points are the
 * per-row pieces of that forward pass.  Every one of them is ROW-INVARIANT:
 * a row's result depends only on that row's inputs, and every reduction runs
 * in an order fixed by the shapes (K, d), never by the number of rows.  With
 * orthrus_block_attn's FP32 path (reduction order fixed by absolute key
 * position) that makes a causal-verify row bitwise equal to a single-token
 * decode of the same position, so in FP32 the consensus loop emits exactly
 * the tokens of greedy autoregressive decoding (explainer §四: lossless).
 *
 * Conventions are those of orthrus.h: caller-owned device pointers, calls
 * asynchronous on `stream`, host-checkable errors returned before any launch,
 * no allocation, no synchronisation.  dtype ORTHRUS_F32 or ORTHRUS_BF16
 * applies to every floating-point tensor of a call; arithmetic is FP32 in
 * both cases, and BF16 calls round each result to bf16 where a BF16 decoder
 * stores it (noted per call).  A "row" is one token position; rows are dense
 * and row-major.
 */
#ifndef ORTHRUS_DECODER_H
#define ORTHRUS_DECODER_H

#include "orthrus.h"

#ifdef __cplusplus
extern "C" {
#endif

/* out[r, :] = table[tokens[r], :].  table [V, d], out [rows, d].  A token
 * outside [0, V) writes a zero row and sets *err (nullable) to ORTHRUS_EINVAL. */
int orthrus_embed(int32_t dtype, const void* table, int32_t V, int32_t d,
                  const int32_t* tokens, int32_t rows, void* out, int32_t* err,
                  orthrus_stream_t stream);

/* RMSNorm per row: out = x / sqrt(mean(x^2) + eps) * gain.
 * x, out [rows, d] (out may alias x); gain [d].  The sum of squares is
 * accumulated in FP32 in a fixed order.  BF16: the normalised row is rounded
 * to bf16 before the gain multiply, and the product is rounded again. */
int orthrus_rmsnorm(int32_t dtype, const void* x, const void* gain, int32_t rows,
                    int32_t d, float eps, void* out, orthrus_stream_t stream);

/* out[r, o] = residual[r, o] + sum_k x[r, k] * w[o, k]   (residual nullable)
 * x [rows, K], w [N, K] (PyTorch Linear layout), residual/out [rows, N].
 * Each output is one FP32 fused-multiply-add chain over k = 0..K-1 in
 * ascending order.  out may alias residual, never x or w.  BF16: the dot
 * product is rounded to bf16, then added to the residual and rounded again. */
int orthrus_linear(int32_t dtype, const void* x, const void* w, const void* residual,
                   int32_t rows, int32_t K, int32_t N, void* out, orthrus_stream_t stream);

/* Split a fused projection into q, k, v and apply the rotary embedding to q
 * and k.  qkv [B*blk, (Hq + 2*Hkv) * hd] holds, per row, q heads then k heads
 * then v heads; row b*blk + j sits at position ctx_lens[b] + j (ctx_lens
 * [B] device).  Outputs q [B, blk, Hq, hd], k/v [B, blk, Hkv, hd] -- the
 * layouts orthrus_block_attn reads.  Rotation pairs element i with i + hd/2
 * (i < hd/2) by the angle pos * theta^(-2i/hd), evaluated in double and
 * applied in FP32; hd even.  BF16: each rotated element is rounded once. */
int orthrus_qkv_rope(int32_t dtype, const void* qkv, int32_t B, int32_t blk, int32_t Hq,
                     int32_t Hkv, int32_t hd, const int32_t* ctx_lens, double theta,
                     void* q, void* k, void* v, orthrus_stream_t stream);

/* SwiGLU: out[r, i] = silu(gu[r, i]) * gu[r, F + i], silu(g) = g / (1 + e^-g).
 * gu [rows, 2F] (gate half, then up half), out [rows, F].  BF16: silu(g) is
 * rounded to bf16 before the multiply, the product rounded again. */
int orthrus_swiglu(int32_t dtype, const void* gu, int32_t rows, int32_t F, void* out,
                   orthrus_stream_t stream);

/* The block a round feeds its two views (explainer §四 steps 1-2):
 *   out[b, 0] = anchor[b];  out[b, j] = draft[b, j-1] (j >= 1)  if draft != NULL
 *                           out[b, j] = mask_id      (j >= 1)  if draft == NULL
 * i.e. [anchor, MASK x (blk-1)] for the diffusion view and
 * [anchor, d_0 .. d_{blk-2}] for verification.  anchor [B], draft and out
 * [B, blk] int32 device; 1 <= blk <= 32. */
int orthrus_block_tokens(const int32_t* anchor, const int32_t* draft, int32_t B,
                         int32_t blk, int32_t mask_id, int32_t* out,
                         orthrus_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* ORTHRUS_DECODER_H */
