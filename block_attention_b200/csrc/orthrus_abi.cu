// orthrus_abi.cu -- the extern "C" entry points declared in include/orthrus.h:
// host-side argument checks, workspace sizing and kernel dispatch.
#include <math.h>

#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "common.cuh"

namespace orthrus {
size_t argmax_workspace_bytes(int rows);
cudaError_t launch_argmax(int dtype, const void* logits, int rows, int vocab, int64_t stride,
                          int32_t* idx, float* maxval, void* ws, cudaStream_t st);
cudaError_t launch_consensus(const int32_t* draft, const int32_t* verify, int B, int blk,
                             int32_t* accept_len, int32_t* n_emit, int32_t* emitted,
                             int32_t* next_anchor, cudaStream_t st);
size_t commit_workspace_bytes(int B);
cudaError_t launch_commit(const orthrus_commit_args& a, cudaStream_t st);
}  // namespace orthrus

using namespace orthrus;

namespace {

bool dtype_ok(int32_t d) { return d == ORTHRUS_F32 || d == ORTHRUS_BF16; }

bool aligned(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

// Shape checks shared by the size query and the launch.
int check_attn_shape(const orthrus_attn_args* a) {
  if (!a) return ORTHRUS_EINVAL;
  if (!dtype_ok(a->dtype)) return ORTHRUS_EINVAL;
  if (a->mask_mode != ORTHRUS_BIDIR_BLOCK && a->mask_mode != ORTHRUS_CAUSAL_VERIFY)
    return ORTHRUS_EINVAL;
  if (a->B < 0 || a->Hq <= 0 || a->Hkv <= 0 || a->D <= 0 || a->blk <= 0 || a->cap < 0 ||
      a->max_ctx < 0)
    return ORTHRUS_EINVAL;
  if (a->Hq % a->Hkv) return ORTHRUS_EINVAL;
  if (!isfinite(a->scale) || !(a->scale > 0.f)) return ORTHRUS_EINVAL;
  if (a->max_ctx > a->cap) return ORTHRUS_ECAPACITY;
  if (a->D != 64 && a->D != 128) return ORTHRUS_EUNSUPPORTED;
  if (a->blk > 32 || (a->Hq / a->Hkv) * a->blk > 128) return ORTHRUS_EUNSUPPORTED;
  return ORTHRUS_OK;
}

bool use_tc_path(const orthrus_attn_args* a) {
  return a->dtype == ORTHRUS_BF16 && tc_supported(*a);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA; }

}  // namespace

extern "C" {

int orthrus_version(void) { return ORTHRUS_VERSION; }

const char* orthrus_status_str(int s) {
  switch (s) {
    case ORTHRUS_OK: return "ok";
    case ORTHRUS_EINVAL: return "invalid argument";
    case ORTHRUS_EUNSUPPORTED: return "unsupported shape or dtype";
    case ORTHRUS_EWORKSPACE: return "workspace missing or too small";
    case ORTHRUS_ECAPACITY: return "length exceeds cache capacity";
    case ORTHRUS_ECUDA: return "CUDA launch failed";
    case ORTHRUS_ETIMEOUT: return "bounded device wait timed out";
    default: return "unknown status";
  }
}

size_t orthrus_block_attn_workspace(const orthrus_attn_args* a) {
  if (check_attn_shape(a) != ORTHRUS_OK) return 0;
  if (use_tc_path(a)) return tc_workspace_bytes(*a);
  return simt_workspace_bytes(a->B, a->Hq, a->D, a->blk, a->max_ctx);
}

int orthrus_block_attn(const orthrus_attn_args* a, orthrus_stream_t stream) {
  int rc = check_attn_shape(a);
  if (rc != ORTHRUS_OK) return rc;
  if (a->B == 0) return ORTHRUS_OK;
  const size_t vec = 16;  // every path reads rows with 16-byte vectors
  const void* ptrs[] = {a->q, a->k_blk, a->v_blk, a->k_cache, a->v_cache, a->out};
  for (const void* p : ptrs)
    if (!p || !aligned(p, vec)) return ORTHRUS_EINVAL;
  if (!a->ctx_lens) return ORTHRUS_EINVAL;
  if ((a->next_k_cache && !aligned(a->next_k_cache, vec)) ||
      (a->next_v_cache && !aligned(a->next_v_cache, vec)))
    return ORTHRUS_EINVAL;
  const size_t need = orthrus_block_attn_workspace(a);
  if (need > 0 && (!a->workspace || a->workspace_bytes < need || !aligned(a->workspace, 256)))
    return ORTHRUS_EWORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (use_tc_path(a)) return tc_launch(*a, st);
  return cuda_status(launch_attn_simt(*a, st));
}

int orthrus_block_attn_launches(const orthrus_attn_args* a) {
  if (check_attn_shape(a) != ORTHRUS_OK || a->B == 0) return 0;
  return use_tc_path(a) ? tc_launches(*a) : 2;  // split + combine
}

int orthrus_block_attn_plan(const orthrus_attn_args* a, int32_t sms, int32_t* out) {
  if (!out || sms < 1) return ORTHRUS_EINVAL;
  const int rc = check_attn_shape(a);
  if (rc != ORTHRUS_OK) return rc;
  if (!use_tc_path(a)) return ORTHRUS_EUNSUPPORTED;
  const int S = tc_plan_splits(*a, sms);
  const int tiles = (a->max_ctx + 127) / 128 + 1;  // 128-key cache tiles + the block tile
  out[0] = S;
  out[1] = a->Hkv;
  out[2] = a->B;
  out[3] = S;
  out[4] = tc_threads();
  out[5] = tc_smem_bytes();
  out[6] = (tiles + S - 1) / S;
  out[7] = tc_plan_fused(*a, sms, S) ? 1 : 0;
  return ORTHRUS_OK;
}

size_t orthrus_vocab_argmax_workspace(int32_t rows) {
  return rows < 0 ? 0 : argmax_workspace_bytes(rows);
}

int orthrus_vocab_argmax(int32_t dtype, const void* logits, int32_t rows, int32_t vocab,
                         int64_t row_stride, int32_t* idx, float* maxval, void* workspace,
                         size_t workspace_bytes, orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || rows < 0 || vocab <= 0 || row_stride < vocab) return ORTHRUS_EINVAL;
  if (rows > 65535) return ORTHRUS_EUNSUPPORTED;
  if (rows == 0) return ORTHRUS_OK;
  if (!logits || !idx) return ORTHRUS_EINVAL;
  if (!aligned(logits, dtype == ORTHRUS_F32 ? 4 : 2)) return ORTHRUS_EINVAL;
  if (!workspace || workspace_bytes < argmax_workspace_bytes(rows) || !aligned(workspace, 16))
    return ORTHRUS_EWORKSPACE;
  return cuda_status(launch_argmax(dtype, logits, rows, vocab, row_stride, idx, maxval,
                                   workspace, reinterpret_cast<cudaStream_t>(stream)));
}

int orthrus_consensus(const int32_t* draft, const int32_t* verify, int32_t B, int32_t blk,
                      int32_t* accept_len, int32_t* n_emit, int32_t* emitted,
                      int32_t* next_anchor, orthrus_stream_t stream) {
  if (B < 0 || blk < 1) return ORTHRUS_EINVAL;
  if (blk > 32) return ORTHRUS_EUNSUPPORTED;
  if (B == 0) return ORTHRUS_OK;
  if (!draft || !verify || !n_emit) return ORTHRUS_EINVAL;
  return cuda_status(launch_consensus(draft, verify, B, blk, accept_len, n_emit, emitted,
                                      next_anchor, reinterpret_cast<cudaStream_t>(stream)));
}

size_t orthrus_kv_commit_workspace(const orthrus_commit_args* a) {
  if (!a || a->B < 0) return 0;
  return commit_workspace_bytes(a->B);
}

int orthrus_kv_commit(const orthrus_commit_args* a, orthrus_stream_t stream) {
  if (!a || !dtype_ok(a->dtype)) return ORTHRUS_EINVAL;
  if (a->layers < 1 || a->B < 0 || a->Hkv < 1 || a->D < 1 || a->blk < 1 || a->cap < 0)
    return ORTHRUS_EINVAL;
  if (a->B > 65535 || a->layers > 65535) return ORTHRUS_EUNSUPPORTED;
  if (a->B == 0) return ORTHRUS_OK;
  const int64_t cache_elems = (int64_t)a->B * a->Hkv * a->cap * a->D;
  const int64_t blk_elems = (int64_t)a->B * a->blk * a->Hkv * a->D;
  if (a->layers > 1 && (a->cache_layer_stride < cache_elems || a->blk_layer_stride < blk_elems))
    return ORTHRUS_EINVAL;
  const size_t es = a->dtype == ORTHRUS_F32 ? 4 : 2;
  const void* ptrs[] = {a->k_cache, a->v_cache, a->k_blk, a->v_blk};
  for (const void* p : ptrs)
    if (!p || !aligned(p, es)) return ORTHRUS_EINVAL;
  if (!a->ctx_lens || !a->n_emit) return ORTHRUS_EINVAL;
  if (!a->workspace || a->workspace_bytes < commit_workspace_bytes(a->B) ||
      !aligned(a->workspace, 4))
    return ORTHRUS_EWORKSPACE;
  return cuda_status(launch_commit(*a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
