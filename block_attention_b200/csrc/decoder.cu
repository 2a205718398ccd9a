// decoder.cu -- row-invariant building blocks of a Qwen3-style decoder, used
// to run the Orthrus consensus loop end to end (cjcn.com.cn explainer of
// "Orthrus", §二: a frozen AR decoder plus a per-layer diffusion copy of the
// attention projections; §四: the round).  Declared in orthrus_decoder.h.
//
// Every kernel computes each row from that row's inputs alone, with its
// reductions in an order fixed by the shapes: the FP32 linear layer is one
// fused-multiply-add chain over k = 0..K-1 per output however the rows are
// tiled, RMSNorm sums squares in a fixed lane order, RoPE depends only on the
// absolute position.  Together with the FP32 block attention (split by
// absolute key position) this makes a verify row bitwise equal to a
// one-token decode of the same position.
#include <algorithm>

#include "common.cuh"
#include "orthrus_decoder.h"
#include "tc_ptx.cuh"

namespace orthrus {
namespace {

bool dtype_ok(int32_t t) { return t == ORTHRUS_F32 || t == ORTHRUS_BF16; }
size_t esize(int32_t t) { return t == ORTHRUS_F32 ? 4 : 2; }
bool aligned_to(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }
int status(cudaError_t e) { return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA; }

__device__ __forceinline__ float round_to(float x, float*) { return x; }
__device__ __forceinline__ float round_to(float x, __nv_bfloat16*) {
  return __bfloat162float(__float2bfloat16_rn(x));
}
// x rounded to T's precision and widened back (a no-op for float)
template <typename T> __device__ __forceinline__ float rnd(float x) {
  return round_to(x, static_cast<T*>(nullptr));
}

// ------------------------------------------------ 16-byte chunk helpers
// A row is read and written in 16-byte chunks of kW<T> elements; chunk c of a
// row is elements c*kW .. c*kW+kW-1.  kVec: the row is 16-byte aligned and a
// whole number of chunks (one vector access per chunk); otherwise element by
// element, elements past the row's end reading as zero.
template <typename T> constexpr int kW = 16 / sizeof(T);

template <typename T, bool kVec>
__device__ __forceinline__ void load_chunk(const T* row, int c, int n, float (&v)[kW<T>]) {
  if (kVec) {
    const uint4 u = *reinterpret_cast<const uint4*>(row + c * kW<T>);
    if constexpr (sizeof(T) == 4) {
      v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
      v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    } else {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < kW<T>; ++i) {
      const int e = c * kW<T> + i;
      v[i] = e < n ? to_f32(row[e]) : 0.f;
    }
  }
}

template <typename T, bool kVec>
__device__ __forceinline__ void store_chunk(T* row, int c, int n, const float (&v)[kW<T>]) {
  if (kVec) {
    uint4 u;
    if constexpr (sizeof(T) == 4) {
      u = make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                     __float_as_uint(v[3]));
    } else {
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
      }
      u = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4*>(row + c * kW<T>) = u;
  } else {
#pragma unroll
    for (int i = 0; i < kW<T>; ++i) {
      const int e = c * kW<T> + i;
      if (e < n) row[e] = from_f32<T>(v[i]);
    }
  }
}

// Launch with programmatic stream serialization: the grid may start while
// the preceding kernel finishes; each of these kernels lets its own
// dependents start at once and waits for its predecessor before reading.
template <typename... KA, typename... A>
cudaError_t launch_pdl(void (*kernel)(KA...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, A... args) {
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KA>(args)...);
}

__device__ __forceinline__ void pdl_enter() {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
}

// ------------------------------------------------------------------ embed
template <typename T, bool kVec>
__global__ void __launch_bounds__(128)
embed_kernel(const T* __restrict__ table, int V, int d, const int32_t* __restrict__ tokens,
             T* __restrict__ out, int32_t* err) {
  pdl_enter();
  const int r = blockIdx.x;
  const int tok = tokens[r];
  const bool ok = tok >= 0 && tok < V;
  if (!ok && threadIdx.x == 0) set_err(err, ORTHRUS_EINVAL);
  const T* src = table + (int64_t)(ok ? tok : 0) * d;
  T* dst = out + (int64_t)r * d;
  for (int c = threadIdx.x; c < ceil_div(d, kW<T>); c += blockDim.x) {
    float v[kW<T>];
    load_chunk<T, kVec>(src, c, d, v);
    if (!ok) {
#pragma unroll
      for (int i = 0; i < kW<T>; ++i) v[i] = 0.f;
    }
    store_chunk<T, kVec>(dst, c, d, v);
  }
}

// ---------------------------------------------------------------- RMSNorm
// One CTA per row.  Chunk c of the row belongs to thread c % kNormThreads;
// each thread sums the squares of its chunks in order (chunk by chunk,
// element by element), then the threads' sums meet in a fixed xor butterfly
// within each warp and in warp order across warps.  The order depends on d
// alone, so a row's result does not depend on the other rows of the call.
// kChunks > 0: the thread's chunks stay in registers between the two
// passes; kChunks == 0: the row is read again for the output.
constexpr int kNormThreads = 256;

template <typename T, bool kVec, int kChunks>
__global__ void __launch_bounds__(kNormThreads)
rmsnorm_kernel(const T* x, const T* __restrict__ gain, int d, float eps, T* out) {
  pdl_enter();
  const T* xr = x + (int64_t)blockIdx.x * d;
  T* yr = out + (int64_t)blockIdx.x * d;
  const int nch = ceil_div(d, kW<T>);
  constexpr int kC = kChunks > 0 ? kChunks : 1;
  float v[kC][kW<T>];
  float ss = 0.f;
  if (kChunks > 0) {
#pragma unroll
    for (int k = 0; k < kC; ++k) {
      const int c = threadIdx.x + k * kNormThreads;
      if (c < nch) load_chunk<T, kVec>(xr, c, d, v[k]);
    }
#pragma unroll
    for (int k = 0; k < kC; ++k) {
      if (threadIdx.x + k * kNormThreads < nch) {
#pragma unroll
        for (int i = 0; i < kW<T>; ++i) ss = fmaf(v[k][i], v[k][i], ss);
      }
    }
  } else {
    for (int c = threadIdx.x; c < nch; c += kNormThreads) {
      load_chunk<T, kVec>(xr, c, d, v[0]);
#pragma unroll
      for (int i = 0; i < kW<T>; ++i) ss = fmaf(v[0][i], v[0][i], ss);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  __shared__ float warp_ss[kNormThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_ss[threadIdx.x >> 5] = ss;
  __syncthreads();  // also: every thread has read its x before any writes (out may alias x)
  ss = 0.f;
#pragma unroll
  for (int w = 0; w < kNormThreads / 32; ++w) ss += warp_ss[w];
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  auto emit = [&](int c, float (&xv)[kW<T>]) {
    float g[kW<T>];
    load_chunk<T, kVec>(gain, c, d, g);
#pragma unroll
    for (int i = 0; i < kW<T>; ++i) xv[i] = rnd<T>(xv[i] * inv) * g[i];
    store_chunk<T, kVec>(yr, c, d, xv);
  };
  if (kChunks > 0) {
#pragma unroll
    for (int k = 0; k < kC; ++k) {
      const int c = threadIdx.x + k * kNormThreads;
      if (c < nch) emit(c, v[k]);
    }
  } else {
    for (int c = threadIdx.x; c < nch; c += kNormThreads) {
      load_chunk<T, kVec>(xr, c, d, v[0]);
      emit(c, v[0]);
    }
  }
}

// ----------------------------------------------------------------- linear
// 128 x 128 output tile per CTA, k in steps of 8 through double-buffered
// shared memory, 8 x 8 outputs per thread.  Whatever the tiling, output
// (r, o) is acc = fma(x[r,k], w[o,k], acc) for k = 0, 1, ..., K-1 (k past K
// contributes fma(0, 0, acc)), so a row's result never depends on M.
constexpr int kLinBM = 128, kLinBN = 128, kLinBK = 8, kLinThreads = 256;

template <typename T, bool kVec>
__device__ __forceinline__ void load_k4(const T* __restrict__ base, int K, int row, int nrows,
                                        int k, float (&v)[4]) {
  if (row < nrows) {
    const T* p = base + (int64_t)row * K + k;
    if (kVec && k + 4 <= K) {
      const float4 f = load4(p);
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
      return;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = k + u < K ? to_f32(p[u]) : 0.f;
  } else {
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = 0.f;
  }
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kLinThreads)
linear_kernel(const T* __restrict__ X, const T* __restrict__ W, const T* R, T* Y, int M,
              int K, int N) {
  __shared__ __align__(16) float As[2][kLinBK][kLinBM];
  __shared__ __align__(16) float Bs[2][kLinBK][kLinBN];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.y * kLinBM, n0 = blockIdx.x * kLinBN;
  const int lr = tid >> 1, lk = (tid & 1) * 4;  // loader: one row, 4 consecutive k
  const int ty = tid >> 4, tx = tid & 15;       // compute: rows ty*4 (+64), cols tx*4 (+64)
  float xa[4], wb[4];
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int nk = ceil_div(K, kLinBK);
  load_k4<T, kVec>(X, K, m0 + lr, M, lk, xa);
  load_k4<T, kVec>(W, K, n0 + lr, N, lk, wb);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    As[0][lk + u][lr] = xa[u];
    Bs[0][lk + u][lr] = wb[u];
  }
  __syncthreads();
  for (int t = 0; t < nk; ++t) {
    const int cur = t & 1;
    const bool more = t + 1 < nk;
    if (more) {
      load_k4<T, kVec>(X, K, m0 + lr, M, (t + 1) * kLinBK + lk, xa);
      load_k4<T, kVec>(W, K, n0 + lr, N, (t + 1) * kLinBK + lk, wb);
    }
#pragma unroll
    for (int kk = 0; kk < kLinBK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        As[cur ^ 1][lk + u][lr] = xa[u];
        Bs[cur ^ 1][lk + u][lr] = wb[u];
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int row = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (row >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (col >= N) continue;
      const int64_t o = (int64_t)row * N + col;
      const float p = rnd<T>(acc[i][j]);
      Y[o] = from_f32<T>(R ? to_f32(R[o]) + p : p);
    }
  }
}

// --------------------------------------------------------- q/k/v + RoPE
// One CTA per block row.  Rotation pairs (x[i], x[i + hd/2]) of a head at the
// row's absolute position: the angle pos * theta^(-2i/hd) and its cosine and
// sine in double, once per row into shared memory; the rotation itself in
// float.  Work units: a 16-byte chunk of x[i..] together with the matching
// chunk of x[i + hd/2] (q and k heads), and 16-byte chunks of v (copied).
// kVec: hd/2 is a whole number of chunks and every row is 16-byte aligned;
// otherwise a unit is a single pair or a single element.  Each thread reads
// all of its units before the table is built, so the loads of a row are in
// flight together.
constexpr int kRopeThreads = 256;
constexpr int kRopeUnits = 4;  // units per thread held in registers per batch

template <typename T, bool kVec>
__global__ void __launch_bounds__(kRopeThreads)
qkv_rope_kernel(const T* __restrict__ qkv, int blk, int Hq, int Hkv, int hd,
                const int32_t* __restrict__ ctx_lens, double theta, T* __restrict__ q,
                T* __restrict__ k, T* __restrict__ v) {
  extern __shared__ float cs[];  // [hd/2] cos, then [hd/2] sin
  pdl_enter();
  constexpr int W = kVec ? kW<T> : 1;
  const int r = blockIdx.x, b = r / blk, j = r % blk;
  const int half = hd / 2, hc = half / W;  // chunks per half head
  const int width = (Hq + 2 * Hkv) * hd;
  const T* src = qkv + (int64_t)r * width;
  const int rot_units = (Hq + Hkv) * hc, copy_units = Hkv * hd / W;
  const int units = rot_units + copy_units;
  const int64_t pos = (int64_t)ctx_lens[b] + j;
  bool table = false;
  for (int base = 0; base < units; base += kRopeThreads * kRopeUnits) {
    float a[kRopeUnits][W], c2[kRopeUnits][W];
#pragma unroll
    for (int u = 0; u < kRopeUnits; ++u) {
      const int id = base + u * kRopeThreads + threadIdx.x;
      if (id < rot_units) {
        const int h = id / hc, i0 = (id % hc) * W;
        if constexpr (kVec) {
          load_chunk<T, true>(src + h * hd, i0 / W, hd, a[u]);
          load_chunk<T, true>(src + h * hd + half, i0 / W, hd, c2[u]);
        } else {
          a[u][0] = to_f32(src[h * hd + i0]);
          c2[u][0] = to_f32(src[h * hd + half + i0]);
        }
      } else if (id < units) {
        const int e0 = (id - rot_units) * W;
        if constexpr (kVec) load_chunk<T, true>(src + (Hq + Hkv) * hd, e0 / W, Hkv * hd, a[u]);
        else a[u][0] = to_f32(src[(Hq + Hkv) * hd + e0]);
      }
    }
    if (!table) {
      for (int i = threadIdx.x; i < half; i += kRopeThreads) {
        const float2 t = rope_cos_sin(pos, i, hd, theta);
        cs[i] = t.x;
        cs[half + i] = t.y;
      }
      __syncthreads();
      table = true;
    }
#pragma unroll
    for (int u = 0; u < kRopeUnits; ++u) {
      const int id = base + u * kRopeThreads + threadIdx.x;
      if (id < rot_units) {
        const int h = id / hc, i0 = (id % hc) * W;
        float y1[W], y2[W];
#pragma unroll
        for (int e = 0; e < W; ++e) {
          const float2 t = make_float2(cs[i0 + e], cs[half + i0 + e]);
          y1[e] = rope_first(a[u][e], c2[u][e], t);
          y2[e] = rope_second(a[u][e], c2[u][e], t);
        }
        T* dst = h < Hq ? q + ((int64_t)r * Hq + h) * hd : k + ((int64_t)r * Hkv + h - Hq) * hd;
        if constexpr (kVec) {
          store_chunk<T, true>(dst, i0 / W, hd, y1);
          store_chunk<T, true>(dst + half, i0 / W, hd, y2);
        } else {
          dst[i0] = from_f32<T>(y1[0]);
          dst[half + i0] = from_f32<T>(y2[0]);
        }
      } else if (id < units) {
        const int e0 = (id - rot_units) * W;
        T* vd = v + (int64_t)r * Hkv * hd;
        if constexpr (kVec) store_chunk<T, true>(vd, e0 / W, Hkv * hd, a[u]);
        else vd[e0] = from_f32<T>(a[u][0]);
      }
    }
  }
}

// ----------------------------------------------------------------- SwiGLU
template <typename T>
__global__ void swiglu_kernel(const T* __restrict__ gu, int64_t n, int F, T* __restrict__ out) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / F;
    const int i = (int)(e - r * F);
    const float g = to_f32(gu[r * 2 * F + i]), u = to_f32(gu[r * 2 * F + F + i]);
    const float s = rnd<T>(g / (1.0f + expf(-g)));
    out[e] = from_f32<T>(s * u);
  }
}

// ------------------------------------------------------------ block tokens
__global__ void __launch_bounds__(32)
block_tokens_kernel(const int32_t* __restrict__ anchor, const int32_t* __restrict__ draft,
                    int blk, int mask_id, int32_t* __restrict__ out) {
  const int b = blockIdx.x, j = threadIdx.x;
  if (j >= blk) return;
  out[(int64_t)b * blk + j] =
      j == 0 ? anchor[b] : (draft ? draft[(int64_t)b * blk + j - 1] : mask_id);
}

template <typename T, bool kVec>
cudaError_t launch_rmsnorm(const T* x, const T* gain, int rows, int d, float eps, T* out,
                           cudaStream_t st) {
  const int per_thread = ceil_div(ceil_div(d, kW<T>), kNormThreads);
  auto go = [&](auto kernel) {
    return launch_pdl(kernel, rows, kNormThreads, 0, st, x, gain, d, eps, out);
  };
  if (per_thread <= 1) return go(rmsnorm_kernel<T, kVec, 1>);
  if (per_thread <= 2) return go(rmsnorm_kernel<T, kVec, 2>);
  if (per_thread <= 4) return go(rmsnorm_kernel<T, kVec, 4>);
  return go(rmsnorm_kernel<T, kVec, 0>);
}

}  // namespace
}  // namespace orthrus

using namespace orthrus;

extern "C" {

int orthrus_embed(int32_t dtype, const void* table, int32_t V, int32_t d,
                  const int32_t* tokens, int32_t rows, void* out, int32_t* err,
                  orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || V <= 0 || d <= 0 || rows < 0) return ORTHRUS_EINVAL;
  if (rows == 0) return ORTHRUS_OK;
  if (!table || !tokens || !out) return ORTHRUS_EINVAL;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const bool vec = (d * esize(dtype)) % 16 == 0 && aligned_to(table, 16) && aligned_to(out, 16);
  cudaError_t e;
  if (dtype == ORTHRUS_F32) {
    auto t = static_cast<const float*>(table);
    auto o = static_cast<float*>(out);
    e = vec ? launch_pdl(embed_kernel<float, true>, rows, 128, 0, st, t, V, d, tokens, o, err)
            : launch_pdl(embed_kernel<float, false>, rows, 128, 0, st, t, V, d, tokens, o, err);
  } else {
    auto t = static_cast<const __nv_bfloat16*>(table);
    auto o = static_cast<__nv_bfloat16*>(out);
    e = vec ? launch_pdl(embed_kernel<__nv_bfloat16, true>, rows, 128, 0, st, t, V, d, tokens,
                         o, err)
            : launch_pdl(embed_kernel<__nv_bfloat16, false>, rows, 128, 0, st, t, V, d, tokens,
                         o, err);
  }
  return status(e);
}

int orthrus_rmsnorm(int32_t dtype, const void* x, const void* gain, int32_t rows, int32_t d,
                    float eps, void* out, orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || rows < 0 || d <= 0 || !(eps >= 0.f)) return ORTHRUS_EINVAL;
  if (rows == 0) return ORTHRUS_OK;
  if (!x || !gain || !out) return ORTHRUS_EINVAL;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const bool vec = (d * esize(dtype)) % 16 == 0 && aligned_to(x, 16) && aligned_to(gain, 16) &&
                   aligned_to(out, 16);
  cudaError_t e;
  if (dtype == ORTHRUS_F32) {
    auto X = static_cast<const float*>(x), G = static_cast<const float*>(gain);
    auto Y = static_cast<float*>(out);
    e = vec ? launch_rmsnorm<float, true>(X, G, rows, d, eps, Y, st)
            : launch_rmsnorm<float, false>(X, G, rows, d, eps, Y, st);
  } else {
    auto X = static_cast<const __nv_bfloat16*>(x), G = static_cast<const __nv_bfloat16*>(gain);
    auto Y = static_cast<__nv_bfloat16*>(out);
    e = vec ? launch_rmsnorm<__nv_bfloat16, true>(X, G, rows, d, eps, Y, st)
            : launch_rmsnorm<__nv_bfloat16, false>(X, G, rows, d, eps, Y, st);
  }
  return status(e);
}

int orthrus_linear(int32_t dtype, const void* x, const void* w, const void* residual,
                   int32_t rows, int32_t K, int32_t N, void* out, orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || rows < 0 || K <= 0 || N <= 0) return ORTHRUS_EINVAL;
  if (rows == 0) return ORTHRUS_OK;
  if (!x || !w || !out) return ORTHRUS_EINVAL;
  if (out == x || out == w) return ORTHRUS_EINVAL;
  if (ceil_div(rows, kLinBM) > 65535) return ORTHRUS_EUNSUPPORTED;
  const size_t es = esize(dtype);
  // 4-element vector loads need K % 4 == 0 and 4-element-aligned x and w
  const bool vec = K % 4 == 0 && aligned_to(x, 4 * es) && aligned_to(w, 4 * es);
  auto st = reinterpret_cast<cudaStream_t>(stream);
  dim3 grid(ceil_div(N, kLinBN), ceil_div(rows, kLinBM));
  if (dtype == ORTHRUS_F32) {
    auto X = static_cast<const float*>(x), Wt = static_cast<const float*>(w),
         R = static_cast<const float*>(residual);
    auto Y = static_cast<float*>(out);
    if (vec) linear_kernel<float, true><<<grid, kLinThreads, 0, st>>>(X, Wt, R, Y, rows, K, N);
    else linear_kernel<float, false><<<grid, kLinThreads, 0, st>>>(X, Wt, R, Y, rows, K, N);
  } else {
    auto X = static_cast<const __nv_bfloat16*>(x), Wt = static_cast<const __nv_bfloat16*>(w),
         R = static_cast<const __nv_bfloat16*>(residual);
    auto Y = static_cast<__nv_bfloat16*>(out);
    if (vec)
      linear_kernel<__nv_bfloat16, true><<<grid, kLinThreads, 0, st>>>(X, Wt, R, Y, rows, K, N);
    else
      linear_kernel<__nv_bfloat16, false><<<grid, kLinThreads, 0, st>>>(X, Wt, R, Y, rows, K, N);
  }
  return status(cudaGetLastError());
}

int orthrus_qkv_rope(int32_t dtype, const void* qkv, int32_t B, int32_t blk, int32_t Hq,
                     int32_t Hkv, int32_t hd, const int32_t* ctx_lens, double theta, void* q,
                     void* k, void* v, orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || B < 0 || blk <= 0 || Hq <= 0 || Hkv <= 0 || hd <= 0 || hd % 2 ||
      !(theta > 0.0))
    return ORTHRUS_EINVAL;
  if (B == 0) return ORTHRUS_OK;
  if (!qkv || !ctx_lens || !q || !k || !v) return ORTHRUS_EINVAL;
  const int64_t rows = (int64_t)B * blk;
  if (rows > 2147483647LL) return ORTHRUS_EUNSUPPORTED;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const size_t smem = sizeof(float) * hd;
  const size_t es = esize(dtype);
  const bool vec = (hd / 2) % (16 / es) == 0 && aligned_to(qkv, 16) && aligned_to(q, 16) &&
                   aligned_to(k, 16) && aligned_to(v, 16);
  cudaError_t e;
  const unsigned g = (unsigned)rows;
  if (dtype == ORTHRUS_F32) {
    auto src = static_cast<const float*>(qkv);
    auto Q = static_cast<float*>(q), K = static_cast<float*>(k), Vv = static_cast<float*>(v);
    e = vec ? launch_pdl(qkv_rope_kernel<float, true>, g, kRopeThreads, smem, st, src, blk, Hq,
                         Hkv, hd, ctx_lens, theta, Q, K, Vv)
            : launch_pdl(qkv_rope_kernel<float, false>, g, kRopeThreads, smem, st, src, blk,
                         Hq, Hkv, hd, ctx_lens, theta, Q, K, Vv);
  } else {
    auto src = static_cast<const __nv_bfloat16*>(qkv);
    auto Q = static_cast<__nv_bfloat16*>(q), K = static_cast<__nv_bfloat16*>(k),
         Vv = static_cast<__nv_bfloat16*>(v);
    e = vec ? launch_pdl(qkv_rope_kernel<__nv_bfloat16, true>, g, kRopeThreads, smem, st, src,
                         blk, Hq, Hkv, hd, ctx_lens, theta, Q, K, Vv)
            : launch_pdl(qkv_rope_kernel<__nv_bfloat16, false>, g, kRopeThreads, smem, st, src,
                         blk, Hq, Hkv, hd, ctx_lens, theta, Q, K, Vv);
  }
  return status(e);
}

int orthrus_swiglu(int32_t dtype, const void* gu, int32_t rows, int32_t F, void* out,
                   orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || rows < 0 || F <= 0) return ORTHRUS_EINVAL;
  if (rows == 0) return ORTHRUS_OK;
  if (!gu || !out) return ORTHRUS_EINVAL;
  const int64_t n = (int64_t)rows * F;
  const int threads = 256;
  const int grid = (int)std::min<int64_t>((n + threads - 1) / threads, 148 * 16);
  auto st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == ORTHRUS_F32)
    swiglu_kernel<float><<<grid, threads, 0, st>>>(static_cast<const float*>(gu), n, F,
                                                   static_cast<float*>(out));
  else
    swiglu_kernel<__nv_bfloat16><<<grid, threads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(gu), n, F, static_cast<__nv_bfloat16*>(out));
  return status(cudaGetLastError());
}

int orthrus_block_tokens(const int32_t* anchor, const int32_t* draft, int32_t B, int32_t blk,
                         int32_t mask_id, int32_t* out, orthrus_stream_t stream) {
  if (B < 0 || blk < 1 || blk > 32) return ORTHRUS_EINVAL;
  if (B == 0) return ORTHRUS_OK;
  if (!anchor || !out) return ORTHRUS_EINVAL;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  block_tokens_kernel<<<B, 32, 0, st>>>(anchor, draft, blk, mask_id, out);
  return status(cudaGetLastError());
}

}  // extern "C"
