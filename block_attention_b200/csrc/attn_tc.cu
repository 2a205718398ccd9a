// attn_tc.cu -- tensor-core block attention (bf16); not enabled yet.
#include "attn_tc.cuh"

namespace orthrus {

bool tc_supported(const orthrus_attn_args&) { return false; }
size_t tc_workspace_bytes(const orthrus_attn_args&) { return 0; }
int tc_launch(const orthrus_attn_args&, cudaStream_t) { return ORTHRUS_EUNSUPPORTED; }
int tc_launches(const orthrus_attn_args&) { return 1; }

}  // namespace orthrus
