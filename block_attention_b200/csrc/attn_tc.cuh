// attn_tc.cuh -- tensor-core (tcgen05) block attention for bf16 tensors.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>

#include "orthrus.h"

namespace orthrus {

bool tc_supported(const orthrus_attn_args& a);
// Splits per (sequence, kv-head) for a GPU with `sms` SMs, and whether the
// split merge runs inside the one launch (the grid fits one wave).
int tc_plan_splits(const orthrus_attn_args& a, int sms);
bool tc_plan_fused(const orthrus_attn_args& a, int sms, int S);
int tc_smem_bytes();
int tc_threads();
size_t tc_workspace_bytes(const orthrus_attn_args& a);
int tc_launch(const orthrus_attn_args& a, cudaStream_t st);
int tc_launches(const orthrus_attn_args& a);

}  // namespace orthrus
