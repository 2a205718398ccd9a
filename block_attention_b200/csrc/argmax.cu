// argmax.cu -- vocab-row argmax with lowest-index tie-break (the per-position
// "most likely token" of both views, Orthrus explainer §四 steps 1-2).
//
// One pass over the logits, split across many CTAs per row so a 32 x 151936
// matrix spreads over every SM.  Each element maps to a 64-bit key
//     (order-preserving bits of the value) << 32 | (0xFFFFFFFF - index)
// so the unsigned maximum of the keys is the largest value and, among equal
// values, the smallest index.  NaN maps to key 0 and never wins; -0.0 is
// canonicalised to +0.0 so the two zeros tie.  Because max is associative
// and commutative, the result does not depend on how the row is split or in
// which order CTAs finish.  When a row takes at most 16 chunks, its CTAs form
// one thread-block cluster: each stores its key into the rank-0 CTA's shared
// memory, and after the cluster barrier rank 0 folds them and writes
// idx/maxval -- no global atomics, the workspace is not touched.  Longer rows
// fold each CTA's key into the row's slot with atomicMax; the last CTA of the
// row (ticket counter) decodes the key, writes idx/maxval and returns the slot
// and the ticket to zero for the next call.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace orthrus {

constexpr int kArgmaxThreads = 256;
constexpr int kArgmaxChunk = 16384;  // elements per CTA (multiple of 8)
constexpr int kArgmaxMaxCluster = 16;  // most chunks of a row one cluster takes (non-portable)

__device__ __forceinline__ unsigned long long argmax_key(float v, int j) {
  if (v != v) return 0ull;  // NaN
  if (v == 0.f) v = 0.f;    // -0.0 -> +0.0
  unsigned u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (unsigned)j);
}

__device__ __forceinline__ float key_value(unsigned long long k) {
  unsigned u = (unsigned)(k >> 32);
  u = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
  return __uint_as_float(u);
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a,
                                                     unsigned long long b) {
  return a > b ? a : b;
}

// Running (value, index) best of one thread, over elements it visits in
// increasing index order.  A group of consecutive elements is folded by its
// NaN-ignoring maximum m; only when m beats the best so far (strictly: an
// equal value keeps the earlier index) is the group searched for the first
// element equal to m.  -0.0 == +0.0, so the two zeros tie and the earlier
// one stays; NaN never wins; a group of NaNs only is skipped.
struct RunningBest {
  float v = -INFINITY;
  int j = -1;  // -1: nothing but NaN seen yet
  template <int N>
  __device__ __forceinline__ void fold(const float (&e)[N], int j0) {
    float m = e[0];
#pragma unroll
    for (int u = 1; u < N; ++u) m = fmaxf(m, e[u]);
    if (m > v || (j < 0 && m == m)) {
      int k = N - 1;
#pragma unroll
      for (int u = N - 2; u >= 0; --u) k = e[u] == m ? u : k;
      v = m;
      j = j0 + k;
    }
  }
  __device__ __forceinline__ unsigned long long key() const {
    return j < 0 ? 0ull : argmax_key(v, j);
  }
};

// The key of the best element of chunk c of `row` (elements
// [c * kArgmaxChunk, min((c + 1) * kArgmaxChunk, vocab))) seen by this thread.
template <typename T, bool kVec>
__device__ __forceinline__ unsigned long long scan_chunk(const T* __restrict__ row, int vocab,
                                                         int c) {
  const int beg = c * kArgmaxChunk;
  const int end = min(beg + kArgmaxChunk, vocab);
  RunningBest rb;
  if (kVec) {
    // 4 elements per vector load for f32 (16 B), 8 for bf16 (16 B), all of
    // the thread's loads in flight before the first is used
    constexpr int kV = 16 / sizeof(T);
    constexpr int kIters = kArgmaxChunk / (kV * kArgmaxThreads);
    uint4 buf[kIters];
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      const int j = beg + (it * kArgmaxThreads + threadIdx.x) * kV;
      if (j + kV <= end) buf[it] = __ldcs(reinterpret_cast<const uint4*>(row + j));
    }
#pragma unroll
    for (int it = 0; it < kIters; ++it) {
      const int j = beg + (it * kArgmaxThreads + threadIdx.x) * kV;
      float e[kV];
      if (j + kV <= end) {
        const T* t = reinterpret_cast<const T*>(&buf[it]);
#pragma unroll
        for (int u = 0; u < kV; ++u) e[u] = to_f32(t[u]);
        rb.fold(e, j);
      } else {
        for (int u = 0; u < kV && j + u < end; ++u) {
          const float one[1] = {to_f32(row[j + u])};
          rb.fold(one, j + u);
        }
      }
    }
  } else {
    for (int j = beg + threadIdx.x; j < end; j += kArgmaxThreads) {
      const float one[1] = {to_f32(row[j])};
      rb.fold(one, j);
    }
  }
  return rb.key();
}

// The CTA's best key (valid in thread 0).
__device__ __forceinline__ unsigned long long cta_best(unsigned long long best) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    best = umax64(best, __shfl_xor_sync(0xffffffffu, best, off));
  __shared__ unsigned long long warp_best[kArgmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_best[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0)
    for (int w = 1; w < kArgmaxThreads / 32; ++w) best = umax64(best, warp_best[w]);
  return best;
}

// One cluster of gridDim.x CTAs per row (grid (nchunks, rows), cluster
// (nchunks, 1, 1)): CTA c scans chunk c and stores its key into slot c of the
// rank-0 CTA's shared memory; after the cluster barrier rank 0 folds them.
template <typename T, bool kVec>
__global__ void __launch_bounds__(kArgmaxThreads)
argmax_cluster_kernel(const T* __restrict__ logits, int vocab, int64_t stride, int32_t* idx,
                      float* maxval) {
  __shared__ unsigned long long cta_keys[kArgmaxMaxCluster];
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int c = blockIdx.x, r = blockIdx.y;
  const T* row = logits + (int64_t)r * stride;
  const unsigned long long best = cta_best(scan_chunk<T, kVec>(row, vocab, c));
  if (threadIdx.x == 0)
    ptx::st_cluster_u64(ptx::map_rank(ptx::smem_u32(&cta_keys[c]), 0), best);
  ptx::cluster_sync();  // release / acquire: every CTA's key is in rank 0's slots
  if (c == 0 && threadIdx.x == 0) {
    unsigned long long k = 0ull;
    for (int q = 0; q < (int)gridDim.x; ++q) k = umax64(k, cta_keys[q]);
    if (k == 0ull) {  // every element was NaN
      idx[r] = 0;
      if (maxval) maxval[r] = to_f32(row[0]);
    } else {
      idx[r] = (int32_t)(0xFFFFFFFFu - (unsigned)(k & 0xFFFFFFFFull));
      if (maxval) maxval[r] = key_value(k);
    }
  }
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kArgmaxThreads)
argmax_kernel(const T* __restrict__ logits, int vocab, int64_t stride,
              int nchunks, unsigned long long* keys, unsigned* tickets,
              int32_t* idx, float* maxval) {
  const int c = blockIdx.x, r = blockIdx.y;
  // Launched with programmatic stream serialization: the launch overlaps the
  // tail of the preceding kernel; nothing is read before that kernel has
  // completed (it may be the one writing the logits).
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const T* row = logits + (int64_t)r * stride;
  const unsigned long long best = cta_best(scan_chunk<T, kVec>(row, vocab, c));
  __shared__ bool last;
  if (threadIdx.x == 0) {
    atomicMax(&keys[r], best);
    __threadfence();
    last = atomicAdd(&tickets[r], 1u) == (unsigned)nchunks - 1u;
    if (last) {
      const unsigned long long k = atomicExch(&keys[r], 0ull);
      tickets[r] = 0u;
      if (k == 0ull) {  // every element was NaN
        idx[r] = 0;
        if (maxval) maxval[r] = to_f32(row[0]);
      } else {
        idx[r] = (int32_t)(0xFFFFFFFFu - (unsigned)(k & 0xFFFFFFFFull));
        if (maxval) maxval[r] = key_value(k);
      }
    }
  }
}

size_t argmax_workspace_bytes(int rows) {
  return (size_t)(((int64_t)rows * 12 + 255) / 256 * 256);
}

cudaError_t launch_argmax(int dtype, const void* logits, int rows, int vocab,
                          int64_t stride, int32_t* idx, float* maxval, void* ws,
                          cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  unsigned long long* keys = static_cast<unsigned long long*>(ws);
  unsigned* tickets = reinterpret_cast<unsigned*>(keys + rows);
  const int nchunks = ceil_div(vocab, kArgmaxChunk);
  const size_t es = dtype == ORTHRUS_F32 ? 4 : 2;
  const bool vec = (reinterpret_cast<uintptr_t>(logits) % 16 == 0) &&
                   ((stride * (int64_t)es) % 16 == 0);
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nchunks, rows);
  cfg.blockDim = dim3(kArgmaxThreads);
  cfg.stream = st;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  if (nchunks <= kArgmaxMaxCluster) {
    attrs[1].id = cudaLaunchAttributeClusterDimension;
    attrs[1].val.clusterDim.x = (unsigned)nchunks;
    attrs[1].val.clusterDim.y = 1;
    attrs[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
    auto go = [&](auto kernel, auto p) -> cudaError_t {
      const cudaError_t e =
          cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
      return cudaLaunchKernelEx(&cfg, kernel, p, vocab, stride, idx, maxval);
    };
    if (dtype == ORTHRUS_F32) {
      auto p = static_cast<const float*>(logits);
      return vec ? go(argmax_cluster_kernel<float, true>, p)
                 : go(argmax_cluster_kernel<float, false>, p);
    }
    auto p = static_cast<const __nv_bfloat16*>(logits);
    return vec ? go(argmax_cluster_kernel<__nv_bfloat16, true>, p)
               : go(argmax_cluster_kernel<__nv_bfloat16, false>, p);
  }
  if (dtype == ORTHRUS_F32) {
    auto p = static_cast<const float*>(logits);
    return vec ? cudaLaunchKernelEx(&cfg, argmax_kernel<float, true>, p, vocab, stride, nchunks,
                                    keys, tickets, idx, maxval)
               : cudaLaunchKernelEx(&cfg, argmax_kernel<float, false>, p, vocab, stride, nchunks,
                                    keys, tickets, idx, maxval);
  }
  auto p = static_cast<const __nv_bfloat16*>(logits);
  return vec ? cudaLaunchKernelEx(&cfg, argmax_kernel<__nv_bfloat16, true>, p, vocab, stride,
                                  nchunks, keys, tickets, idx, maxval)
             : cudaLaunchKernelEx(&cfg, argmax_kernel<__nv_bfloat16, false>, p, vocab, stride,
                                  nchunks, keys, tickets, idx, maxval);
}

}  // namespace orthrus

// ---------------------------------------------------------------------------
// Scratch-free variant of the argmax entry point.
//
// Some callers cannot allocate device memory for a workspace: code that runs
// where no allocator is available or allowed (inside another library's
// fixed memory budget, from a plugin handed only the tensors it works on, or
// in a process whose device memory is already fully reserved).  For them the
// argmax keeps its per-row scratch -- one 64-bit key and one ticket counter
// per row -- in a file-scope device array that every GPU loading this
// library holds until the process exits.
namespace orthrus {
namespace {

constexpr int kNoAllocMaxRows = ORTHRUS_NOALLOC_ARGMAX_MAX_ROWS;
constexpr size_t kNoAllocBytes = (size_t)kNoAllocMaxRows * 12;

static __device__ __align__(256) unsigned char g_argmax_scratch[kNoAllocBytes];

// Device address of g_argmax_scratch per device, together with the context it
// was looked up in (in host code the symbol itself is only a host-side
// stand-in, never a device address).  A device reset or a new primary context
// reloads the module at another address, so the cached address is reused only
// while the current context is the one it came from.
std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {nullptr};
CUcontext g_scratch_ctx[64] = {nullptr};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

}  // namespace
}  // namespace orthrus

extern "C" int orthrus_vocab_argmax_noalloc(int32_t dtype, const void* logits, int32_t rows,
                                            int32_t vocab, int64_t row_stride, int32_t* idx,
                                            float* maxval, orthrus_stream_t stream) {
  using namespace orthrus;
  if (!(dtype == ORTHRUS_F32 || dtype == ORTHRUS_BF16) || rows < 0 || vocab <= 0 ||
      row_stride < vocab)
    return ORTHRUS_EINVAL;
  if (rows > kNoAllocMaxRows) return ORTHRUS_EUNSUPPORTED;  // beyond the static scratch
  if (rows == 0) return ORTHRUS_OK;
  if (!logits || !idx) return ORTHRUS_EINVAL;
  if (reinterpret_cast<uintptr_t>(logits) % (dtype == ORTHRUS_F32 ? 4 : 2)) return ORTHRUS_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ORTHRUS_ECUDA;
  void* ws = nullptr;
  {
    CtxGetCurrentFn get_ctx = ctx_get_current();
    CUcontext ctx = nullptr;
    if (!get_ctx || get_ctx(&ctx) != CUDA_SUCCESS) return ORTHRUS_ECUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_argmax_scratch) != cudaSuccess || !ptr)
        return ORTHRUS_ECUDA;
      if (!ctx && (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)) return ORTHRUS_ECUDA;
      g_scratch_ptr[dev] = ptr;
      g_scratch_ctx[dev] = ctx;
    }
    ws = g_scratch_ptr[dev];
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the rows' keys and tickets must start at zero (the kernel also leaves them zero)
  if (cudaMemsetAsync(ws, 0, (size_t)rows * 12, st) != cudaSuccess) return ORTHRUS_ECUDA;
  return launch_argmax(dtype, logits, rows, vocab, row_stride, idx, maxval, ws, st) ==
                 cudaSuccess
             ? ORTHRUS_OK
             : ORTHRUS_ECUDA;
}
