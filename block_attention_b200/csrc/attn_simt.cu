// attn_simt.cu -- FP32 (and bf16-input) block attention on CUDA cores.
//
// Computes the Orthrus round's attention for both views (explainer on
// arXiv:2605.12825, §二: the block's queries attend to the AR KV cache
// concatenated with the block's own K/V; §三: the diffusion view sees its
// whole block, the AR view is causal).
//
// Split-KV by ABSOLUTE key position: split s covers key positions
// [s*kChunk, (s+1)*kChunk) of the concatenated sequence cache[0,n) ++ block,
// and inside a split keys are consumed in 16-key tiles aligned to absolute
// positions.  A row's visible keys are always a prefix of each tile, masked
// keys are never touched, and the combine runs over splits in index order.
// So the arithmetic a row sees depends only on the positions it can see:
// causal row i over (cache n, block) is bit-identical to a one-row decode at
// n + i over (cache n + i, block of 1) -- the property that makes FP32
// consensus decoding reproduce greedy decoding exactly.
//
// Thread layout: four lanes per query row (row r = block row i * G + local
// head), each lane holding D/4 of q and of the output accumulator; dims are
// interleaved in groups of four so a tile row read by a quad is one
// contiguous segment.  K/V tiles come into shared memory by cp.async, two
// tiles deep: the next tile's copies are in flight while the current one is
// used (tiles past the keys are zero-filled, as before).
#include "attn_simt.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace orthrus {

template <typename T, int D>
__global__ void __launch_bounds__(512)
attn_simt_split_kernel(const SimtParams p) {
  constexpr int kG = D / 16;  // float4 groups per lane
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv;
  const int rows = G * p.blk;
  const int tid = threadIdx.x;
  const int r = tid >> 2, lane4 = tid & 3;
  const bool row_ok = r < rows;
  const int i = row_ok ? r / G : 0;
  const int h = g * G + (row_ok ? r % G : 0);

  __shared__ __align__(16) T Ks[2][kSimtTile][D];
  __shared__ __align__(16) T Vs[2][kSimtTile][D];

  const int n = p.ctx_lens[b];
  const bool bad = n < 0 || n > p.max_ctx;
  if (bad && s == 0 && g == 0 && tid == 0) set_err(p.err, ORTHRUS_ECAPACITY);

  const int total = bad ? 0 : n + p.blk;
  const int lo = s * kSimtChunk;
  const int hi = min(lo + kSimtChunk, total);
  const int lim = p.mask_mode == ORTHRUS_BIDIR_BLOCK ? total : n + i + 1;
  const int row_end = min(lim, hi);

  const T* qrow = static_cast<const T*>(p.q) + ((int64_t)(b * p.blk + i) * p.Hq + h) * D;
  float q[4 * kG], o[4 * kG];
#pragma unroll
  for (int t = 0; t < kG; ++t) {
    float4 v = load4(qrow + 16 * t + 4 * lane4);
    q[4 * t] = v.x; q[4 * t + 1] = v.y; q[4 * t + 2] = v.z; q[4 * t + 3] = v.w;
    o[4 * t] = o[4 * t + 1] = o[4 * t + 2] = o[4 * t + 3] = 0.f;
  }
  float m = -INFINITY, l = 0.f;

  const T* kc = static_cast<const T*>(p.k_cache) + ((int64_t)b * p.Hkv + g) * p.cap * D;
  const T* vc = static_cast<const T*>(p.v_cache) + ((int64_t)b * p.Hkv + g) * p.cap * D;
  const T* kb = static_cast<const T*>(p.k_blk) + ((int64_t)b * p.blk * p.Hkv + g) * D;
  const T* vb = static_cast<const T*>(p.v_blk) + ((int64_t)b * p.blk * p.Hkv + g) * D;
  const int64_t blk_stride = (int64_t)p.Hkv * D;

  // issue the 16-byte copies of the tile at t0 into buffer `buf`, as one group
  constexpr int kVec = 16 / (int)sizeof(T);
  auto issue = [&](int t0, int buf) {
    for (int e = tid; e < kSimtTile * D / kVec; e += blockDim.x) {
      const int j = e / (D / kVec), c = (e % (D / kVec)) * kVec;
      const int pos = t0 + j;
      const T* ks = kc;
      const T* vs = vc;
      uint32_t bytes = 0;  // past the keys: zero-fill, nothing read
      if (pos < n) {
        ks = kc + (int64_t)pos * D + c;
        vs = vc + (int64_t)pos * D + c;
        bytes = 16;
      } else if (pos < total) {
        ks = kb + (pos - n) * blk_stride + c;
        vs = vb + (pos - n) * blk_stride + c;
        bytes = 16;
      }
      ptx::cp_async16_zfill(ptx::smem_u32(&Ks[buf][j][c]), ks, bytes);
      ptx::cp_async16_zfill(ptx::smem_u32(&Vs[buf][j][c]), vs, bytes);
    }
    ptx::cp_async_commit();
  };
  if (lo < hi) issue(lo, 0);
  int buf = 0;
  for (int t0 = lo; t0 < hi; t0 += kSimtTile, buf ^= 1) {
    if (t0 + kSimtTile < hi) {
      issue(t0 + kSimtTile, buf ^ 1);  // its buffer was released by the last barrier
      ptx::cp_async_wait<1>();
    } else {
      ptx::cp_async_wait<0>();
    }
    __syncthreads();  // every thread's copies of this tile have landed

    // Scores for every key of the tile (the quad shuffles need every lane); a row then
    // uses only its visible prefix [t0, row_end).
    const int cnt = row_ok ? max(0, min(row_end - t0, kSimtTile)) : 0;
    float sc[kSimtTile];
#pragma unroll
    for (int j = 0; j < kSimtTile; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < kG; ++t) {
        const float4 k4 = load4(&Ks[buf][j][16 * t + 4 * lane4]);
        acc = fmaf(q[4 * t], k4.x, acc);
        acc = fmaf(q[4 * t + 1], k4.y, acc);
        acc = fmaf(q[4 * t + 2], k4.z, acc);
        acc = fmaf(q[4 * t + 3], k4.w, acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      sc[j] = acc * p.scale_log2;
    }
    if (cnt > 0) {
      float mt = sc[0];
#pragma unroll
      for (int j = 1; j < kSimtTile; ++j)
        if (j < cnt) mt = fmaxf(mt, sc[j]);
      const float mn = fmaxf(m, mt);
      const float alpha = exp2f(m - mn);
      l *= alpha;
#pragma unroll
      for (int d = 0; d < 4 * kG; ++d) o[d] *= alpha;
#pragma unroll
      for (int j = 0; j < kSimtTile; ++j) {
        if (j < cnt) {
          const float pj = exp2f(sc[j] - mn);
          l += pj;
#pragma unroll
          for (int t = 0; t < kG; ++t) {
            const float4 v4 = load4(&Vs[buf][j][16 * t + 4 * lane4]);
            o[4 * t] = fmaf(pj, v4.x, o[4 * t]);
            o[4 * t + 1] = fmaf(pj, v4.y, o[4 * t + 1]);
            o[4 * t + 2] = fmaf(pj, v4.z, o[4 * t + 2]);
            o[4 * t + 3] = fmaf(pj, v4.w, o[4 * t + 3]);
          }
        }
      }
      m = mn;
    }
    __syncthreads();  // the buffer is free for the copies issued next iteration
  }

  if (!row_ok) return;
  // Partial for (b, h, i, split s); an empty split leaves m = -inf, l = 0, o = 0.
  const int64_t pi = (((int64_t)b * p.Hq + h) * p.blk + i) * p.nsplit + s;
  float* po = p.ws_o + pi * D;
#pragma unroll
  for (int t = 0; t < kG; ++t)
    *reinterpret_cast<float4*>(po + 16 * t + 4 * lane4) =
        make_float4(o[4 * t], o[4 * t + 1], o[4 * t + 2], o[4 * t + 3]);
  if (lane4 == 0) {
    p.ws_m[pi] = m;
    p.ws_l[pi] = l;
  }
}

// out = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s, splits in index order.
template <typename T, int D>
__global__ void __launch_bounds__(D) attn_simt_combine_kernel(const SimtParams p) {
  const int row = blockIdx.x;  // ((b * blk) + i) * Hq + h
  const int h = row % p.Hq;
  const int bi = row / p.Hq;
  const int i = bi % p.blk, b = bi / p.blk;
  const int n = p.ctx_lens[b];
  if (n < 0 || n > p.max_ctx) return;
  const int64_t pi0 = (((int64_t)b * p.Hq + h) * p.blk + i) * p.nsplit;
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, p.ws_m[pi0 + s]);
  float L = 0.f, O = 0.f;
  const int d = threadIdx.x;
  for (int s = 0; s < p.nsplit; ++s) {
    const float w = exp2f(p.ws_m[pi0 + s] - M);
    L = fmaf(w, p.ws_l[pi0 + s], L);
    O = fmaf(w, p.ws_o[(pi0 + s) * D + d], O);
  }
  static_cast<T*>(p.out)[(int64_t)row * D + d] = from_f32<T>(O / L);
}

// The first kSimtSkipBytes bytes of the caller's buffer are left alone: the
// tensor-core path keeps its merge counters there, and one buffer may serve
// both paths.
constexpr int64_t kSimtSkipBytes = 2048;

size_t simt_workspace_bytes(int B, int Hq, int D, int blk, int max_ctx) {
  const int64_t nsplit = ceil_div(max_ctx + blk, kSimtChunk);
  const int64_t parts = (int64_t)B * Hq * blk * nsplit;
  auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
  return (size_t)(kSimtSkipBytes + up(parts * D * 4) + 2 * up(parts * 4));
}

template <typename T, int D>
static cudaError_t launch_typed(SimtParams p, cudaStream_t st) {
  const int rows = (p.Hq / p.Hkv) * p.blk;
  const int threads = ceil_div(4 * rows, 32) * 32;
  dim3 grid(p.nsplit, p.Hkv, p.B);
  attn_simt_split_kernel<T, D><<<grid, threads, 0, st>>>(p);
  attn_simt_combine_kernel<T, D><<<p.B * p.blk * p.Hq, D, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_attn_simt(const orthrus_attn_args& a, cudaStream_t st) {
  SimtParams p;
  p.q = a.q; p.k_blk = a.k_blk; p.v_blk = a.v_blk;
  p.k_cache = a.k_cache; p.v_cache = a.v_cache;
  p.ctx_lens = a.ctx_lens; p.out = a.out; p.err = a.err;
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.blk = a.blk; p.cap = a.cap;
  p.max_ctx = a.max_ctx; p.mask_mode = a.mask_mode;
  p.scale_log2 = (float)((double)a.scale * 1.4426950408889634);
  p.nsplit = ceil_div(a.max_ctx + a.blk, kSimtChunk);
  const int64_t parts = (int64_t)a.B * a.Hq * a.blk * p.nsplit;
  auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
  char* ws = static_cast<char*>(a.workspace) + kSimtSkipBytes;
  p.ws_o = reinterpret_cast<float*>(ws);
  p.ws_m = reinterpret_cast<float*>(ws + up(parts * a.D * 4));
  p.ws_l = reinterpret_cast<float*>(ws + up(parts * a.D * 4) + up(parts * 4));
  const bool bf = a.dtype == ORTHRUS_BF16;
  if (a.D == 64)
    return bf ? launch_typed<__nv_bfloat16, 64>(p, st) : launch_typed<float, 64>(p, st);
  return bf ? launch_typed<__nv_bfloat16, 128>(p, st) : launch_typed<float, 128>(p, st);
}

}  // namespace orthrus
