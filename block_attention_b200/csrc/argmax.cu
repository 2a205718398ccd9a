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
// which order CTAs finish.  Each CTA folds its key into the row's slot with
// atomicMax; the last CTA of the row (ticket counter) decodes the key, writes
// idx/maxval and returns the slot and the ticket to zero for the next call.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace orthrus {

constexpr int kArgmaxThreads = 256;
constexpr int kArgmaxChunk = 16384;  // elements per CTA (multiple of 8)

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
  const int beg = c * kArgmaxChunk;
  const int end = min(beg + kArgmaxChunk, vocab);
  unsigned long long best = 0ull;
  if (kVec) {
    // 4 elements per vector load for f32 (16 B), 8 for bf16 (16 B)
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
      if (j + kV <= end) {
        const T* e = reinterpret_cast<const T*>(&buf[it]);
#pragma unroll
        for (int u = 0; u < kV; ++u) best = umax64(best, argmax_key(to_f32(e[u]), j + u));
      } else {
        for (int u = 0; u < kV && j + u < end; ++u)
          best = umax64(best, argmax_key(to_f32(row[j + u]), j + u));
      }
    }
  } else {
    for (int j = beg + threadIdx.x; j < end; j += kArgmaxThreads)
      best = umax64(best, argmax_key(to_f32(row[j]), j));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
    best = umax64(best, __shfl_xor_sync(0xffffffffu, best, off));
  __shared__ unsigned long long warp_best[kArgmaxThreads / 32];
  __shared__ bool last;
  if ((threadIdx.x & 31) == 0) warp_best[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < kArgmaxThreads / 32; ++w) best = umax64(best, warp_best[w]);
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
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nchunks, rows);
  cfg.blockDim = dim3(kArgmaxThreads);
  cfg.stream = st;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
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
