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

// ------------------------------------------------------------------ embed
template <typename T>
__global__ void __launch_bounds__(128)
embed_kernel(const T* __restrict__ table, int V, int d, const int32_t* __restrict__ tokens,
             T* __restrict__ out, int32_t* err) {
  const int r = blockIdx.x;
  const int tok = tokens[r];
  const bool ok = tok >= 0 && tok < V;
  if (!ok && threadIdx.x == 0) set_err(err, ORTHRUS_EINVAL);
  const T* src = table + (int64_t)(ok ? tok : 0) * d;
  T* dst = out + (int64_t)r * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) dst[i] = ok ? src[i] : from_f32<T>(0.f);
}

// ---------------------------------------------------------------- RMSNorm
// One warp per row.  Lane l sums x[i]^2 for i = l, l+32, ... in order, then
// the 32 partial sums meet in a fixed xor butterfly.
constexpr int kNormRowsPerCta = 4;

template <typename T>
__global__ void __launch_bounds__(32 * kNormRowsPerCta)
rmsnorm_kernel(const T* x, const T* __restrict__ gain, int rows, int d, float eps, T* out) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kNormRowsPerCta + (threadIdx.x >> 5);
  if (r >= rows) return;
  const T* xr = x + (int64_t)r * d;
  T* yr = out + (int64_t)r * d;
  float ss = 0.f;
  for (int i = lane; i < d; i += 32) {
    const float v = to_f32(xr[i]);
    ss = fmaf(v, v, ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  __syncwarp();  // every lane has read its x before any lane writes (out may alias x)
  for (int i = lane; i < d; i += 32) {
    const float y = rnd<T>(to_f32(xr[i]) * inv);
    yr[i] = from_f32<T>(y * to_f32(gain[i]));
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
template <typename T>
__global__ void __launch_bounds__(128)
qkv_rope_kernel(const T* __restrict__ qkv, int blk, int Hq, int Hkv, int hd,
                const int32_t* __restrict__ ctx_lens, double theta, T* __restrict__ q,
                T* __restrict__ k, T* __restrict__ v) {
  extern __shared__ float cs[];  // [hd/2] cos, then [hd/2] sin
  const int r = blockIdx.x, b = r / blk, j = r % blk;
  const int half = hd / 2;
  const int64_t pos = (int64_t)ctx_lens[b] + j;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double ang = (double)pos * pow(theta, -2.0 * i / hd);
    double s, c;
    sincos(ang, &s, &c);
    cs[i] = (float)c;
    cs[half + i] = (float)s;
  }
  __syncthreads();
  const int width = (Hq + 2 * Hkv) * hd;
  const T* src = qkv + (int64_t)r * width;
  const int pairs = (Hq + Hkv) * half;
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    const int h = p / half, i = p % half;
    const float c = cs[i], s = cs[half + i];
    const float x1 = to_f32(src[h * hd + i]), x2 = to_f32(src[h * hd + i + half]);
    const float y1 = x1 * c - x2 * s, y2 = x2 * c + x1 * s;
    T* dst = h < Hq ? q + ((int64_t)r * Hq + h) * hd : k + ((int64_t)r * Hkv + h - Hq) * hd;
    dst[i] = from_f32<T>(y1);
    dst[i + half] = from_f32<T>(y2);
  }
  const T* vs = src + (Hq + Hkv) * hd;
  T* vd = v + (int64_t)r * Hkv * hd;
  for (int e = threadIdx.x; e < Hkv * hd; e += blockDim.x) vd[e] = vs[e];
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
  if (dtype == ORTHRUS_F32)
    embed_kernel<float><<<rows, 128, 0, st>>>(static_cast<const float*>(table), V, d, tokens,
                                              static_cast<float*>(out), err);
  else
    embed_kernel<__nv_bfloat16><<<rows, 128, 0, st>>>(
        static_cast<const __nv_bfloat16*>(table), V, d, tokens,
        static_cast<__nv_bfloat16*>(out), err);
  return status(cudaGetLastError());
}

int orthrus_rmsnorm(int32_t dtype, const void* x, const void* gain, int32_t rows, int32_t d,
                    float eps, void* out, orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || rows < 0 || d <= 0 || !(eps >= 0.f)) return ORTHRUS_EINVAL;
  if (rows == 0) return ORTHRUS_OK;
  if (!x || !gain || !out) return ORTHRUS_EINVAL;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const int grid = ceil_div(rows, kNormRowsPerCta);
  if (dtype == ORTHRUS_F32)
    rmsnorm_kernel<float><<<grid, 32 * kNormRowsPerCta, 0, st>>>(
        static_cast<const float*>(x), static_cast<const float*>(gain), rows, d, eps,
        static_cast<float*>(out));
  else
    rmsnorm_kernel<__nv_bfloat16><<<grid, 32 * kNormRowsPerCta, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(gain), rows,
        d, eps, static_cast<__nv_bfloat16*>(out));
  return status(cudaGetLastError());
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
  if (dtype == ORTHRUS_F32)
    qkv_rope_kernel<float><<<(unsigned)rows, 128, smem, st>>>(
        static_cast<const float*>(qkv), blk, Hq, Hkv, hd, ctx_lens, theta,
        static_cast<float*>(q), static_cast<float*>(k), static_cast<float*>(v));
  else
    qkv_rope_kernel<__nv_bfloat16><<<(unsigned)rows, 128, smem, st>>>(
        static_cast<const __nv_bfloat16*>(qkv), blk, Hq, Hkv, hd, ctx_lens, theta,
        static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
        static_cast<__nv_bfloat16*>(v));
  return status(cudaGetLastError());
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
