// attn_simt.cuh -- parameters of the CUDA-core block-attention path.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "orthrus.h"

namespace orthrus {

constexpr int kSimtChunk = 64;   // keys per split (absolute positions)
constexpr int kSimtTile = 16;    // keys per tile (absolute positions)

struct SimtParams {
  const void *q, *k_blk, *v_blk, *k_cache, *v_cache;
  const int32_t* ctx_lens;
  void* out;
  int32_t* err;
  float *ws_o, *ws_m, *ws_l;
  int B, Hq, Hkv, blk, cap, max_ctx, mask_mode, nsplit;
  float scale_log2;  // scale * log2(e): scores live in the exp2 domain
};

size_t simt_workspace_bytes(int B, int Hq, int D, int blk, int max_ctx);
cudaError_t launch_attn_simt(const orthrus_attn_args& a, cudaStream_t st);

}  // namespace orthrus
