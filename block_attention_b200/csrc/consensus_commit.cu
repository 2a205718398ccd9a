// consensus_commit.cu -- prefix consensus and KV commit/rollback
// (Orthrus explainer §四 step 3: compare drafts with the AR view's tokens left
// to right, accept the agreeing prefix, emit the AR token at the first
// disagreement as the correction, drop the rest, update the KV notebook;
// §七: the block is the only extra state, so committing is a bounded copy).
#include "common.cuh"

namespace orthrus {

// One warp per sequence; lane j owns block position j (blk <= 32).
__global__ void __launch_bounds__(32)
consensus_kernel(const int32_t* __restrict__ draft, const int32_t* __restrict__ verify,
                 int blk, int32_t* accept_len, int32_t* n_emit, int32_t* emitted,
                 int32_t* next_anchor) {
  const int b = blockIdx.x, lane = threadIdx.x;
  const bool in = lane < blk;
  const int d = in ? draft[(int64_t)b * blk + lane] : 0;
  const int a = in ? verify[(int64_t)b * blk + lane] : 0;
  const unsigned miss = __ballot_sync(0xffffffffu, in && d != a);
  const int L = miss ? __ffs(miss) - 1 : blk;
  const int ne = min(L + 1, blk);
  const int anchor = __shfl_sync(0xffffffffu, a, ne - 1);
  if (in && emitted) emitted[(int64_t)b * blk + lane] = lane < ne ? a : -1;
  if (lane == 0) {
    if (accept_len) accept_len[b] = L;
    n_emit[b] = ne;
    if (next_anchor) next_anchor[b] = anchor;
  }
}

cudaError_t launch_consensus(const int32_t* draft, const int32_t* verify, int B, int blk,
                             int32_t* accept_len, int32_t* n_emit, int32_t* emitted,
                             int32_t* next_anchor, cudaStream_t st) {
  if (B == 0) return cudaSuccess;
  consensus_kernel<<<B, 32, 0, st>>>(draft, verify, blk, accept_len, n_emit, emitted,
                                     next_anchor);
  return cudaGetLastError();
}

// CTA (kv-head g, layer l, sequence b) copies the accepted rows of that
// (layer, head); the last CTA of sequence b (ticket) advances ctx_lens[b]
// after every CTA of b has read the old length.
template <typename W>
__global__ void __launch_bounds__(128)
kv_commit_kernel(const orthrus_commit_args p, int row_words, unsigned* tickets) {
  const int g = blockIdx.x, l = blockIdx.y, b = blockIdx.z;
  __shared__ int s_n, s_e, s_ok;
  if (threadIdx.x == 0) {
    const int n = p.ctx_lens[b], e = p.n_emit[b];
    const int ok = n >= 0 && e >= 0 && e <= p.blk && (int64_t)n + e <= p.cap;
    if (!ok && g == 0 && l == 0) set_err(p.err, ORTHRUS_ECAPACITY);
    s_n = n; s_e = e; s_ok = ok;
  }
  __syncthreads();
  const int n = s_n, e = s_ok ? s_e : 0;
  const size_t es = p.dtype == ORTHRUS_F32 ? 4 : 2;
  const size_t wpe = sizeof(W) / es;  // elements per word
  const W* kb = reinterpret_cast<const W*>(static_cast<const char*>(p.k_blk) +
                                           (l * p.blk_layer_stride) * es);
  const W* vb = reinterpret_cast<const W*>(static_cast<const char*>(p.v_blk) +
                                           (l * p.blk_layer_stride) * es);
  W* kc = reinterpret_cast<W*>(static_cast<char*>(p.k_cache) + (l * p.cache_layer_stride) * es);
  W* vc = reinterpret_cast<W*>(static_cast<char*>(p.v_cache) + (l * p.cache_layer_stride) * es);
  const int64_t D = p.D;
  for (int t = threadIdx.x; t < e * row_words; t += blockDim.x) {
    const int rr = t / row_words, w = t % row_words;
    const int64_t src = ((((int64_t)b * p.blk + rr) * p.Hkv + g) * D) / wpe + w;
    const int64_t dst = ((((int64_t)b * p.Hkv + g) * p.cap + n + rr) * D) / wpe + w;
    kc[dst] = kb[src];
    vc[dst] = vb[src];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned total = (unsigned)(p.Hkv * p.layers);
    if (atomicAdd(&tickets[b], 1u) == total - 1u) {
      if (s_ok) p.ctx_lens[b] = n + s_e;
      tickets[b] = 0u;
    }
  }
}

size_t commit_workspace_bytes(int B) { return (size_t)(((int64_t)B * 4 + 255) / 256 * 256); }

cudaError_t launch_commit(const orthrus_commit_args& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  const size_t es = a.dtype == ORTHRUS_F32 ? 4 : 2;
  const size_t row_bytes = (size_t)a.D * es;
  // Widest word that every row start is aligned to.
  auto fits = [&](size_t w) {
    auto al = [&](const void* p) { return reinterpret_cast<uintptr_t>(p) % w == 0; };
    return row_bytes % w == 0 && al(a.k_cache) && al(a.v_cache) && al(a.k_blk) &&
           al(a.v_blk) && (a.cache_layer_stride * (int64_t)es) % (int64_t)w == 0 &&
           (a.blk_layer_stride * (int64_t)es) % (int64_t)w == 0;
  };
  dim3 grid(a.Hkv, a.layers, a.B);
  unsigned* tickets = static_cast<unsigned*>(a.workspace);
  if (fits(16))
    kv_commit_kernel<uint4><<<grid, 128, 0, st>>>(a, (int)(row_bytes / 16), tickets);
  else if (fits(4))
    kv_commit_kernel<uint32_t><<<grid, 128, 0, st>>>(a, (int)(row_bytes / 4), tickets);
  else
    kv_commit_kernel<uint16_t><<<grid, 128, 0, st>>>(a, (int)(row_bytes / 2), tickets);
  return cudaGetLastError();
}

}  // namespace orthrus
