// sampling.cu -- the stochastic variant of the Orthrus consensus (cjcn.com.cn
// explainer of "Orthrus", §四: for sampling with a temperature the framework
// aligns the two views' distributions by strict rejection sampling).
// Declared in orthrus.h:
//   orthrus_vocab_sample      draft tokens d_j ~ softmax(z_diff[j] / T) by Gumbel-max,
//                             with log q(d_j) and the rows' log-sum-exp from the same pass
//   orthrus_consensus_sample  log p(d_j), accept while u_j < p/q, then the correction
//                             ~ normalize(max(0, p - q))
//   orthrus_token_logprob     log-probability of given tokens at T (the precision
//                             study; drafts that do not come from the sampler)
// Random numbers: Philox4x32-10 (philox.cuh), counter layout in orthrus.h.
#include "common.cuh"
#include "philox.cuh"
#include "tc_ptx.cuh"

namespace orthrus {
namespace {

bool dtype_ok(int32_t t) { return t == ORTHRUS_F32 || t == ORTHRUS_BF16; }
int status(cudaError_t e) { return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA; }

// Every kernel here is launched with programmatic stream serialization: it
// may start while the preceding kernel finishes, lets its own dependents
// start at once, and waits for its predecessor before reading anything.
template <typename... KA, typename... A>
cudaError_t launch_pdl(void (*kernel)(KA...), dim3 grid, cudaStream_t st, A... args) {
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KA>(args)...);
}

__device__ __forceinline__ void pdl_enter() {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
}

// Keys ordering (value, lowest index first) as one unsigned 64-bit number.
__device__ __forceinline__ unsigned long long order_key(float v, int j) {
  if (v != v) return 0ull;  // NaN never wins
  if (v == 0.f) v = 0.f;    // -0 == +0
  unsigned u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (unsigned)j);
}
__device__ __forceinline__ int key_index(unsigned long long k) {
  return (int)(0xFFFFFFFFu - (unsigned)(k & 0xFFFFFFFFull));
}
__device__ __forceinline__ unsigned long long umax64(unsigned long long a,
                                                     unsigned long long b) {
  return a > b ? a : b;
}
__device__ __forceinline__ uint32_t word(const uint4& v, int e) {
  return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
}

// ------------------------------------------------------------ shared pieces
// Every kernel here cuts rows into chunks of kChunk elements, one CTA per
// (chunk, row), kPer elements per thread held in registers.
// 24 elements per thread (six Philox groups of four): a 151936-entry row is
// 25 chunks, so 32 rows are 800 CTAs -- one wave at six CTAs per SM.
constexpr int kThreads = 256;
constexpr int kPer = 24;
constexpr int kChunk = kThreads * kPer;
constexpr int kWarps = kThreads / 32;
static_assert(kThreads == 256, "launch_pdl launches 256-thread CTAs");
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float qnan() { return __int_as_float(0x7fc00000); }

// The hardware base-2 logarithm and exponential (MUFU; absolute error of
// lg2 about 2^-22, relative error of ex2 about 2^-22), flushing subnormals:
// lg2 only ever sees normal arguments here (uniforms >= 2^-24, exponential
// variates >= 8e-8), and an ex2 result below 2^-126 adds nothing to a sum
// that holds at least exp(0) = 1.
__device__ __forceinline__ float hw_lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float hw_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Gumbel noise in base 2: log2(e) times -ln(E) of the exponential variate
// E = -ln u, u = philox_uniform(w) = ((w >> 9) + 1/2) 2^-23, less the
// constant log2(log2 e) (which no comparison of keys sees):
//   gumbel2(w) = -log2(E2),  E2 = E / ln 2 = -log2 u,
// to a few parts in 10^6:
//   E2: for u <= 15/16 from lg2 (|log2 u| >= 0.093, so lg2's absolute error
//       of about 2^-22 is under 3e-6 relative); above, from the series
//       -ln(1 - v) = v (1 + v/2 + v^2/3 + v^3/4 + ...) times log2 e, with
//       v = 1 - u exact (Sterbenz) and the truncation below v^4/5 < 4e-6
//       relative for v <= 1/16;
//   -log2 E2 from lg2: absolute error a few 10^-7 over E2's whole range.
// Keys x log2(e) / T + gumbel2 then order as x / T + Gumbel does, and their
// argmax agrees with exact arithmetic wherever the two best keys are more
// than ~1e-5 apart.
constexpr float kS1 = kLog2e, kS2 = kLog2e / 2, kS3 = kLog2e / 3, kS4 = kLog2e / 4;
__device__ __forceinline__ float gumbel2(uint32_t w) {
  const float u = philox_uniform(w);
  const float v = 1.f - u;
  const float series = v * fmaf(v, fmaf(v, fmaf(v, kS4, kS3), kS2), kS1);
  const float e2 = v <= 0.0625f ? series : -hw_lg2(u);
  return -hw_lg2(e2);
}

// Block-wide max or sum in a fixed tree; every thread gets the result.
__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, v, off);
    v = is_max ? fmaxf(v, o) : v + o;
  }
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = v;
  __syncthreads();
  if (w == 0) {
    v = lane < kWarps ? red[lane] : (is_max ? -INFINITY : 0.f);
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) {
      const float o = __shfl_xor_sync(0xffffffffu, v, off);
      v = is_max ? fmaxf(v, o) : v + o;
    }
    if (lane == 0) red[kWarps] = v;
  }
  __syncthreads();
  const float res = red[kWarps];
  __syncthreads();
  return res;
}

// (max, sum of exp(x - max)) over the CTA's chunk.
__device__ __forceinline__ float2 chunk_pair(const float (&x)[kPer], float m, float* red) {
  m = block_reduce(m, true, red);
  // the difference first (exact near the maximum), then the base change:
  // at a low temperature x and m are large and x log2(e) - m log2(e) would
  // lose the difference to rounding
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < kPer; ++e) s += hw_ex2((x[e] - m) * kLog2e);  // 0 past the row
  return make_float2(m, block_reduce(s, false, red));
}

// The same from per-thread running pairs (m, s): s = sum exp(x - m) over the
// thread's elements.
__device__ __forceinline__ float2 merge_thread_pairs(float m, float s, float* red) {
  const float M = block_reduce(m, true, red);
  s = m == -INFINITY ? 0.f : s * hw_ex2((m - M) * kLog2e);
  return make_float2(M, block_reduce(s, false, red));
}

// One warp merges a row's chunk pairs -- lane i takes chunks i, i + 32, ...,
// then a fixed shuffle tree -- and zeroes them (where pairs sit depends on
// the call's shapes: a later call may read these bytes as counters).
// Returns log sum_k exp(x_k) in every lane.
__device__ __forceinline__ float merge_pairs(float2* pr, int nchunks, int lane) {
  float M = -INFINITY;
  for (int i = lane; i < nchunks; i += 32) M = fmaxf(M, __ldcg(&pr[i].x));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float S = 0.f;
  for (int i = lane; i < nchunks; i += 32) {
    const float2 q = __ldcg(&pr[i]);
    S += q.y * expf(q.x - M);
    pr[i] = make_float2(0.f, 0.f);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) S += __shfl_xor_sync(0xffffffffu, S, off);
  return M + logf(S);
}

__device__ __forceinline__ unsigned long long warp_max64(unsigned long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = umax64(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// ------------------------------------------------------------ draft sample
// Thread t of chunk c takes the groups g = c * kChunk/4 + i * kThreads + t
// (i < kPer/4), each the 4 consecutive elements one Philox call covers (one
// 16-byte load when the row allows).  A thread visits its elements in
// increasing index, so it keeps its best as a (value, index) pair replaced
// only by a strictly larger value (NaN never wins; equal values keep the
// lower index) and forms the 64-bit order key once; with kLse it also keeps
// a running (max, sum of exp(x - max)) pair.  The best key of the CTA goes
// to the row's slot by atomicMax; with kLse the CTA also stores its chunk
// pair.  The row's last CTA (ticket) writes idx, lse and logprob and returns
// slot and ticket to zero.
template <typename T, bool kLse, bool kVec>
__global__ void __launch_bounds__(kThreads, 6)  // 6 CTAs per SM: 800 fill one wave
vocab_sample_kernel(const T* __restrict__ logits, int vocab, int64_t stride, float inv_t,
                    uint32_t k0, uint32_t k1, uint32_t step, int nchunks,
                    unsigned long long* keys, unsigned* tickets, float2* pairs,
                    int32_t* __restrict__ idx, float* __restrict__ logprob,
                    float* __restrict__ lse) {
  __shared__ float red[kWarps + 1];
  __shared__ unsigned long long wbest[kWarps];
  __shared__ bool last;
  const int c = blockIdx.x, r = blockIdx.y, t = threadIdx.x, lane = t & 31;
  // two batches of three groups: a batch's loads first, then its arithmetic
  constexpr int kB = kPer / 8;
  // the first batch's noise depends only on (row, index, step): drawn before
  // the wait, while the preceding kernel (the one writing the logits) ends
  ptx::griddep_launch_dependents();
  float gn0[4 * kB];
#pragma unroll
  for (int ii = 0; ii < kB; ++ii) {
    const int g = c * (kChunk / 4) + ii * kThreads + t;
    const uint4 w = philox4x32_10(make_uint4((uint32_t)g, (uint32_t)r, kPurposeDraft, step),
                                  k0, k1);
#pragma unroll
    for (int e = 0; e < 4; ++e) gn0[4 * ii + e] = gumbel2(word(w, e));
  }
  ptx::griddep_wait();
  const T* row = logits + (int64_t)r * stride;
  // keys in base 2 (x log2(e) / T + gumbel2); the running (max, sum of
  // exp(x / T - max)) in natural units, each difference taken before the
  // base change (see chunk_pair)
  float bv = -INFINITY, m = -INFINITY, sum = 0.f;
  int bi = -1;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float xs[4 * kB];  // past the row: -inf (never wins, adds exp(-inf) = 0)
#pragma unroll
    for (int ii = 0; ii < kB; ++ii) {
      const int j0 = 4 * (c * (kChunk / 4) + (half * kB + ii) * kThreads + t);
      if (kVec && j0 + 3 < vocab) {
        if constexpr (sizeof(T) == 4) {
          const float4 f = __ldcs(reinterpret_cast<const float4*>(row + j0));
          xs[4 * ii] = f.x; xs[4 * ii + 1] = f.y; xs[4 * ii + 2] = f.z; xs[4 * ii + 3] = f.w;
        } else {
          const uint2 u = __ldcs(reinterpret_cast<const uint2*>(row + j0));
          xs[4 * ii] = __uint_as_float(u.x << 16);
          xs[4 * ii + 1] = __uint_as_float(u.x & 0xffff0000u);
          xs[4 * ii + 2] = __uint_as_float(u.y << 16);
          xs[4 * ii + 3] = __uint_as_float(u.y & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          xs[4 * ii + e] = j0 + e < vocab ? to_f32(row[j0 + e]) : -INFINITY;
      }
    }
#pragma unroll
    for (int ii = 0; ii < kB; ++ii) {
      const int g = c * (kChunk / 4) + (half * kB + ii) * kThreads + t;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (half == 1)
        w = philox4x32_10(make_uint4((uint32_t)g, (uint32_t)r, kPurposeDraft, step), k0, k1);
      float x[4];
      float gm = -INFINITY;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[e] = xs[4 * ii + e] * inv_t;
        gm = fmaxf(gm, x[e]);
        // strictly larger: equal keys keep the lower index, NaN never wins
        const float key = fmaf(x[e], kLog2e, half == 0 ? gn0[4 * ii + e] : gumbel2(word(w, e)));
        if (key > bv) { bv = key; bi = 4 * g + e; }
      }
      if constexpr (kLse) {
        if (gm > m) {
          sum = m == -INFINITY ? 0.f : sum * hw_ex2((m - gm) * kLog2e);
          m = gm;
        }
        if (m != -INFINITY) {
#pragma unroll
          for (int e = 0; e < 4; ++e) sum += hw_ex2((x[e] - m) * kLog2e);
        }
      }
    }
  }
  unsigned long long best = bi < 0 ? 0ull : order_key(bv, bi);
  best = warp_max64(best);
  if (lane == 0) wbest[t >> 5] = best;
  float2 pr = make_float2(0.f, 0.f);
  if constexpr (kLse) pr = merge_thread_pairs(m, sum, red);  // its barriers publish wbest
  else __syncthreads();
  if (t == 0) {
    for (int w = 1; w < kWarps; ++w) best = umax64(best, wbest[w]);
    atomicMax(&keys[r], best);
    if constexpr (kLse) pairs[(int64_t)r * nchunks + c] = pr;
    __threadfence();
    last = atomicAdd(&tickets[r], 1u) == (unsigned)nchunks - 1u;
  }
  __syncthreads();
  if (!last || t >= 32) return;
  __threadfence();
  int j = 0;
  if (lane == 0) {
    const unsigned long long k = atomicExch(&keys[r], 0ull);
    tickets[r] = 0u;
    j = k ? key_index(k) : 0;
    idx[r] = j;
  }
  if constexpr (kLse) {
    const float l = merge_pairs(pairs + (int64_t)r * nchunks, nchunks, lane);
    if (lane == 0) {
      if (lse) lse[r] = l;
      if (logprob) logprob[r] = to_f32(row[j]) * inv_t - l;
    }
  }
}

// ------------------------------------------------------------ log-prob at T
// Grid (chunks, rows); chunk c holds elements [c kChunk, (c + 1) kChunk) of
// the row.  With kVec thread t reads groups of four, elements c kChunk +
// 4 (g kThreads + t) + 0..3 for g < kPer / 4 (one 16- or 8-byte load each);
// otherwise element e is c kChunk + e kThreads + t.  Both coalesce.  The
// row's last CTA merges the chunk pairs.  Workspace: tickets [rows] then the
// pairs [rows][chunks].
template <typename T, bool kVec>
__device__ __forceinline__ float load_chunk(const T* row, int c, int vocab, float inv_t,
                                            float (&x)[kPer]) {
  float m = -INFINITY;
  if constexpr (kVec) {
    // groups of four consecutive logits, one 16-byte (f32) or 8-byte (bf16)
    // load each, as the sampler reads them; every load in flight first
#pragma unroll
    for (int e4 = 0; e4 < kPer / 4; ++e4) {
      const int k = c * kChunk + (e4 * kThreads + threadIdx.x) * 4;
      if (k + 3 < vocab) {
        if constexpr (sizeof(T) == 4) {
          const float4 f = __ldcs(reinterpret_cast<const float4*>(row + k));
          x[4 * e4] = f.x; x[4 * e4 + 1] = f.y; x[4 * e4 + 2] = f.z; x[4 * e4 + 3] = f.w;
        } else {
          const uint2 u = __ldcs(reinterpret_cast<const uint2*>(row + k));
          x[4 * e4] = __uint_as_float(u.x << 16);
          x[4 * e4 + 1] = __uint_as_float(u.x & 0xffff0000u);
          x[4 * e4 + 2] = __uint_as_float(u.y << 16);
          x[4 * e4 + 3] = __uint_as_float(u.y & 0xffff0000u);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[4 * e4 + e] = k + e < vocab ? to_f32(row[k + e]) : -INFINITY;
      }
    }
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      x[e] *= inv_t;
      m = fmaxf(m, x[e]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int k = c * kChunk + e * kThreads + threadIdx.x;
      x[e] = k < vocab ? to_f32(row[k]) * inv_t : -INFINITY;
      m = fmaxf(m, x[e]);
    }
  }
  return m;
}

template <typename T, bool kVec>
__global__ void __launch_bounds__(kThreads)
token_logprob_kernel(const T* __restrict__ logits, int vocab, int64_t stride,
                     const int32_t* __restrict__ idx, float inv_t, int nchunks,
                     unsigned* tickets, float2* pairs, float* __restrict__ logprob,
                     float* __restrict__ lse) {
  __shared__ float red[kWarps + 1];
  __shared__ bool last;
  pdl_enter();
  const int c = blockIdx.x, r = blockIdx.y, t = threadIdx.x;
  const T* row = logits + (int64_t)r * stride;
  float x[kPer];
  const float2 pr = chunk_pair(x, load_chunk<T, kVec>(row, c, vocab, inv_t, x), red);
  if (t == 0) {
    pairs[(int64_t)r * nchunks + c] = pr;
    __threadfence();
    last = atomicAdd(&tickets[r], 1u) == (unsigned)nchunks - 1u;
  }
  __syncthreads();
  if (!last || t >= 32) return;
  __threadfence();
  const float l = merge_pairs(pairs + (int64_t)r * nchunks, nchunks, t);
  if (t == 0) {
    tickets[r] = 0u;
    if (lse) lse[r] = l;
    const int k = idx[r];
    logprob[r] = (k >= 0 && k < vocab) ? to_f32(row[k]) * inv_t - l : qnan();
  }
}

// ------------------------------------------------------ stochastic consensus
// Launch 1, grid (chunks, B*blk) over the AR logits: log p_j(d_j) and the
// row's log-sum-exp as in token_logprob_kernel, and the row's acceptance
// test log u_j < log p_j(d_j) - log q_j(d_j); the CTA that merges a
// sequence's last row (per-sequence count) takes the first rejection, left
// to right, and writes every output except the correction.
// Launch 2, grid (kResChunk-element chunks, B): one group of four per thread,
// so the two rows' work spreads over about one wave; Gumbel-max over the
// rejected row's residual max(0, p - q) (the AR row's argmax as the
// fallback), folded per sequence with atomicMax; the last CTA writes the
// correction.
// Workspace: SeqSlot [B], row tickets [B*blk], chunk pairs [B*blk][chunks].
constexpr int kResChunk = kThreads * 4;

struct SeqSlot {
  // rows verified (high word) and the rejected positions (low word, bit j
  // for row j: rows are distinct, so adding a row's bit is or-ing it)
  unsigned long long verified;
  unsigned long long key_res, key_max;
  uint32_t ticket, pad;
};

template <typename T, bool kVec>
__global__ void __launch_bounds__(kThreads, 6)
consensus_verify_kernel(const orthrus_sample_args p, uint32_t k0, uint32_t k1, float inv_t,
                        int nchunks, SeqSlot* seq, unsigned* row_tickets, float2* pairs) {
  __shared__ float red[kWarps + 1];
  __shared__ bool last;
  pdl_enter();
  const int c = blockIdx.x, r = blockIdx.y, t = threadIdx.x, blk = p.blk, b = r / blk;
  const T* row = static_cast<const T*>(p.logits_ar) + (int64_t)r * p.row_stride;
  float x[kPer];
  const float2 pr = chunk_pair(x, load_chunk<T, kVec>(row, c, p.vocab, inv_t, x), red);
  if (t == 0) {
    pairs[(int64_t)r * nchunks + c] = pr;
    __threadfence();
    last = atomicAdd(&row_tickets[r], 1u) == (unsigned)nchunks - 1u;
  }
  __syncthreads();
  if (!last || t >= 32) return;
  __threadfence();
  const int lane = t;
  const float l = merge_pairs(pairs + (int64_t)r * nchunks, nchunks, lane);
  // the row's own acceptance test, folded with the row count into one
  // atomic: the warp whose row completes the sequence reads the first
  // rejection from the folded bits (no other row's values are read back)
  unsigned long long st = 0ull;
  if (lane == 0) {
    row_tickets[r] = 0u;
    const int d = p.draft[r], j = r - b * blk;
    const float lp = (d >= 0 && d < p.vocab) ? to_f32(row[d]) * inv_t - l : qnan();
    p.lse_ar[r] = l;
    p.logp[r] = lp;
    const uint4 w = philox4x32_10(make_uint4((uint32_t)j, (uint32_t)b, kPurposeAccept, p.step),
                                  k0, k1);
    const bool acc = logf(philox_uniform(w.x)) < lp - p.logq[r];  // NaN: reject
    const unsigned long long add = (1ull << 32) | (acc ? 0ull : 1ull << j);
    st = atomicAdd(&seq[b].verified, add) + add;
  }
  st = __shfl_sync(0xffffffffu, st, 0);
  if ((unsigned)(st >> 32) != (unsigned)blk) return;
  const unsigned miss = (unsigned)st;
  const int L = miss ? __ffs(miss) - 1 : blk;
  if (lane < blk) {
    const int d = p.draft[(int64_t)b * blk + lane];
    if (p.emitted && lane != L) p.emitted[(int64_t)b * blk + lane] = lane < L ? d : -1;
    if (L == blk && lane == blk - 1 && p.next_anchor) p.next_anchor[b] = d;
  }
  if (lane == 0) {
    seq[b].verified = 0ull;
    p.accept_len[b] = L;
    p.n_emit[b] = min(L + 1, blk);
  }
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
consensus_residual_kernel(const orthrus_sample_args p, uint32_t k0, uint32_t k1, float inv_t,
                          int nchunks, SeqSlot* seq) {
  __shared__ unsigned long long wres[kWarps], wmax[kWarps];
  const int c = blockIdx.x, b = blockIdx.y, t = threadIdx.x, blk = p.blk;
  // the noise depends on the vocabulary index, not on which row is
  // corrected: drawn while the log p pass finishes, before the wait
  ptx::griddep_launch_dependents();
  const int g = c * (kResChunk / 4) + t;
  const uint4 w = philox4x32_10(make_uint4((uint32_t)g, (uint32_t)b, kPurposeResidual, p.step),
                                k0, k1);
  float gn[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) gn[e] = gumbel2(word(w, e));
  ptx::griddep_wait();
  const int L = p.accept_len[b];
  if (L >= blk) return;  // every draft accepted: no correction
  const int r = b * blk + L;
  const T* za = static_cast<const T*>(p.logits_ar) + (int64_t)r * p.row_stride;
  const T* zd = static_cast<const T*>(p.logits_diff) + (int64_t)r * p.row_stride;
  const float la = p.lse_ar[r], ld = p.lse_diff[r];
  unsigned long long best = 0ull, bmax = 0ull;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int k = 4 * g + e;
    if (k < p.vocab) {
      const float xa = to_f32(za[k]);
      const float d = expf(xa * inv_t - la) - expf(to_f32(zd[k]) * inv_t - ld);
      if (d > 0.f) best = umax64(best, order_key(log2f(d) + gn[e], k));
      bmax = umax64(bmax, order_key(xa, k));
    }
  }
  best = warp_max64(best);
  bmax = warp_max64(bmax);
  if ((t & 31) == 0) { wres[t >> 5] = best; wmax[t >> 5] = bmax; }
  __syncthreads();
  if (t != 0) return;
  for (int i = 1; i < kWarps; ++i) {
    best = umax64(best, wres[i]);
    bmax = umax64(bmax, wmax[i]);
  }
  SeqSlot* sc = &seq[b];
  atomicMax(&sc->key_res, best);
  atomicMax(&sc->key_max, bmax);
  __threadfence();
  if (atomicAdd(&sc->ticket, 1u) == (unsigned)nchunks - 1u) {
    const unsigned long long kr = atomicExch(&sc->key_res, 0ull);
    const unsigned long long km = atomicExch(&sc->key_max, 0ull);
    sc->ticket = 0u;
    const int corr = kr ? key_index(kr) : key_index(km);
    if (p.emitted) p.emitted[(int64_t)b * blk + L] = corr;
    if (p.next_anchor) p.next_anchor[b] = corr;
  }
}

size_t round256(int64_t n) { return (size_t)((n + 255) / 256 * 256); }

// One 16-byte (f32) or 8-byte (bf16) load per group of four logits: the
// base aligned to a group and every row starting on a group boundary.
bool vec_rows(const void* logits, int64_t row_stride, int32_t dtype) {
  const size_t gbytes = dtype == ORTHRUS_F32 ? 16 : 8;
  return reinterpret_cast<uintptr_t>(logits) % gbytes == 0 && row_stride % 4 == 0;
}
constexpr int32_t kMaxVocab = 1 << 30;

}  // namespace
}  // namespace orthrus

using namespace orthrus;

extern "C" {

size_t orthrus_vocab_sample_workspace(int32_t rows, int32_t vocab) {
  if (rows < 0 || vocab <= 0 || vocab > kMaxVocab) return 0;
  const int64_t nchunks = ceil_div(vocab, kChunk);
  return round256((int64_t)rows * 8) + round256((int64_t)rows * 4) +
         (size_t)((int64_t)rows * nchunks * 8);
}

int orthrus_vocab_sample(int32_t dtype, const void* logits, int32_t rows, int32_t vocab,
                         int64_t row_stride, float temperature, uint64_t seed, uint32_t step,
                         int32_t* idx, float* logprob, float* lse, void* workspace,
                         size_t workspace_bytes, orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || rows < 0 || vocab <= 0 || row_stride < vocab ||
      !(temperature > 0.f) || !isfinite(temperature))
    return ORTHRUS_EINVAL;
  if (vocab > kMaxVocab) return ORTHRUS_EUNSUPPORTED;
  if (rows == 0) return ORTHRUS_OK;
  if (!logits || !idx) return ORTHRUS_EINVAL;
  if (!workspace || workspace_bytes < orthrus_vocab_sample_workspace(rows, vocab) ||
      reinterpret_cast<uintptr_t>(workspace) % 16)
    return ORTHRUS_EWORKSPACE;
  if (rows > 65535) return ORTHRUS_EUNSUPPORTED;
  char* ws = static_cast<char*>(workspace);
  auto keys = reinterpret_cast<unsigned long long*>(ws);
  auto tickets = reinterpret_cast<unsigned*>(ws + round256((int64_t)rows * 8));
  auto pairs = reinterpret_cast<float2*>(ws + round256((int64_t)rows * 8) +
                                         round256((int64_t)rows * 4));
  const int nchunks = ceil_div(vocab, kChunk);
  const uint32_t k0 = (uint32_t)seed, k1 = (uint32_t)(seed >> 32);
  const float inv_t = 1.f / temperature;
  const bool want = logprob || lse;
  // one 16-byte (f32) or 8-byte (bf16) load per group of four: the base
  // aligned to a group and every row starting on a group boundary
  const size_t gbytes = dtype == ORTHRUS_F32 ? 16 : 8;
  const bool vec = reinterpret_cast<uintptr_t>(logits) % gbytes == 0 && row_stride % 4 == 0;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  dim3 grid(nchunks, rows);
  cudaError_t e;
#define ORTHRUS_SAMPLE(T, L, V)                                                              \
  e = launch_pdl(vocab_sample_kernel<T, L, V>, grid, st, static_cast<const T*>(logits), vocab, \
                 row_stride, inv_t, k0, k1, step, nchunks, keys, tickets, pairs, idx, logprob, \
                 lse)
  if (dtype == ORTHRUS_F32) {
    if (vec) {
      if (want) ORTHRUS_SAMPLE(float, true, true); else ORTHRUS_SAMPLE(float, false, true);
    } else {
      if (want) ORTHRUS_SAMPLE(float, true, false); else ORTHRUS_SAMPLE(float, false, false);
    }
  } else {
    if (vec) {
      if (want) ORTHRUS_SAMPLE(__nv_bfloat16, true, true);
      else ORTHRUS_SAMPLE(__nv_bfloat16, false, true);
    } else {
      if (want) ORTHRUS_SAMPLE(__nv_bfloat16, true, false);
      else ORTHRUS_SAMPLE(__nv_bfloat16, false, false);
    }
  }
#undef ORTHRUS_SAMPLE
  return status(e);
}

size_t orthrus_token_logprob_workspace(int32_t rows, int32_t vocab) {
  if (rows < 0 || vocab <= 0 || vocab > kMaxVocab) return 0;
  const int64_t nchunks = ceil_div(vocab, kChunk);
  return round256((int64_t)rows * 4) + (size_t)((int64_t)rows * nchunks * 8);
}

int orthrus_token_logprob(int32_t dtype, const void* logits, int32_t rows, int32_t vocab,
                          int64_t row_stride, const int32_t* idx, float temperature,
                          float* logprob, float* lse, void* workspace, size_t workspace_bytes,
                          orthrus_stream_t stream) {
  if (!dtype_ok(dtype) || rows < 0 || vocab <= 0 || row_stride < vocab ||
      !(temperature > 0.f) || !isfinite(temperature))
    return ORTHRUS_EINVAL;
  if (vocab > kMaxVocab) return ORTHRUS_EUNSUPPORTED;
  if (rows == 0) return ORTHRUS_OK;
  if (!logits || !idx || !logprob) return ORTHRUS_EINVAL;
  if (!workspace || workspace_bytes < orthrus_token_logprob_workspace(rows, vocab) ||
      reinterpret_cast<uintptr_t>(workspace) % 16)
    return ORTHRUS_EWORKSPACE;
  if (rows > 65535) return ORTHRUS_EUNSUPPORTED;
  const int nchunks = ceil_div(vocab, kChunk);
  auto tickets = static_cast<unsigned*>(workspace);
  auto pairs = reinterpret_cast<float2*>(static_cast<char*>(workspace) +
                                         round256((int64_t)rows * 4));
  const float inv_t = 1.f / temperature;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  dim3 grid(nchunks, rows);
  const bool vec = vec_rows(logits, row_stride, dtype);
#define ORTHRUS_LOGPROB(T, V)                                                                  \
  return status(launch_pdl(token_logprob_kernel<T, V>, grid, st, static_cast<const T*>(logits), \
                           vocab, row_stride, idx, inv_t, nchunks, tickets, pairs, logprob, lse))
  if (dtype == ORTHRUS_F32) {
    if (vec) ORTHRUS_LOGPROB(float, true);
    ORTHRUS_LOGPROB(float, false);
  }
  if (vec) ORTHRUS_LOGPROB(__nv_bfloat16, true);
  ORTHRUS_LOGPROB(__nv_bfloat16, false);
#undef ORTHRUS_LOGPROB
}

size_t orthrus_consensus_sample_workspace(int32_t B, int32_t blk, int32_t vocab) {
  if (B < 0 || blk < 1 || vocab <= 0 || vocab > kMaxVocab) return 0;
  const int64_t rows = (int64_t)B * blk, nchunks = ceil_div(vocab, kChunk);
  return round256((int64_t)B * sizeof(SeqSlot)) + round256(rows * 4) +
         (size_t)(rows * nchunks * 8);
}

int orthrus_consensus_sample(const orthrus_sample_args* a, orthrus_stream_t stream) {
  if (!a || !dtype_ok(a->dtype) || a->B < 0 || a->blk < 1 || a->vocab <= 0 ||
      a->row_stride < a->vocab || !(a->temperature > 0.f) || !isfinite(a->temperature))
    return ORTHRUS_EINVAL;
  if (a->blk > 32 || a->vocab > kMaxVocab) return ORTHRUS_EUNSUPPORTED;
  if (a->B == 0) return ORTHRUS_OK;
  if (!a->draft || !a->logq || !a->lse_diff || !a->logits_ar || !a->logits_diff ||
      !a->logp || !a->lse_ar || !a->accept_len || !a->n_emit)
    return ORTHRUS_EINVAL;
  if (!a->workspace ||
      a->workspace_bytes < orthrus_consensus_sample_workspace(a->B, a->blk, a->vocab) ||
      reinterpret_cast<uintptr_t>(a->workspace) % 16)
    return ORTHRUS_EWORKSPACE;
  const int64_t rows = (int64_t)a->B * a->blk;
  if (rows > 65535) return ORTHRUS_EUNSUPPORTED;
  const uint32_t k0 = (uint32_t)a->seed, k1 = (uint32_t)(a->seed >> 32);
  char* ws = static_cast<char*>(a->workspace);
  auto seq = reinterpret_cast<SeqSlot*>(ws);
  auto row_tickets = reinterpret_cast<unsigned*>(ws + round256((int64_t)a->B * sizeof(SeqSlot)));
  auto pairs = reinterpret_cast<float2*>(ws + round256((int64_t)a->B * sizeof(SeqSlot)) +
                                         round256(rows * 4));
  const int nchunks = ceil_div(a->vocab, kChunk);
  const float inv_t = 1.f / a->temperature;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const int nres = ceil_div(a->vocab, kResChunk);
  const dim3 g1(nchunks, (unsigned)rows), g2(nres, a->B);
  const orthrus_sample_args args = *a;
  const bool vec = vec_rows(a->logits_ar, a->row_stride, a->dtype);
  cudaError_t e;
  if (a->dtype == ORTHRUS_F32) {
    e = vec ? launch_pdl(consensus_verify_kernel<float, true>, g1, st, args, k0, k1, inv_t,
                         nchunks, seq, row_tickets, pairs)
            : launch_pdl(consensus_verify_kernel<float, false>, g1, st, args, k0, k1, inv_t,
                         nchunks, seq, row_tickets, pairs);
    if (e == cudaSuccess)
      e = launch_pdl(consensus_residual_kernel<float>, g2, st, args, k0, k1, inv_t, nres, seq);
  } else {
    e = vec ? launch_pdl(consensus_verify_kernel<__nv_bfloat16, true>, g1, st, args, k0, k1,
                         inv_t, nchunks, seq, row_tickets, pairs)
            : launch_pdl(consensus_verify_kernel<__nv_bfloat16, false>, g1, st, args, k0, k1,
                         inv_t, nchunks, seq, row_tickets, pairs);
    if (e == cudaSuccess)
      e = launch_pdl(consensus_residual_kernel<__nv_bfloat16>, g2, st, args, k0, k1, inv_t,
                     nres, seq);
  }
  return status(e);
}

}  // extern "C"
