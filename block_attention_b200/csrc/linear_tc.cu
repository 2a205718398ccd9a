// linear_tc.cu -- the attention block's projections on the tensor cores:
//   y[r, n] = bf16( sum_k x[r, k] w[n, k] )              (residual == NULL)
//   y[r, n] = bf16( residual[r, n] + bf16(sum_k ...) )    (otherwise)
// for a handful of rows (the 32 rows of a decoding block) against a large
// weight matrix w [N, K] (the QKV and output projections around the round's
// attention -- cjcn.com.cn explainer of "Orthrus", §二: the diffusion view
// has its own copy of these projections, everything else is shared).
//
// With 32 rows the product is weight-streaming: every weight byte is used
// 32 times, so the bound is HBM.  tcgen05 GEMM with the weights as the A
// operand (M = 128 output features per tile, from shared memory) and the
// rows as the B operand (N = rows rounded up to 16), so one MMA of K = 16
// consumes 4 KB of weights.  A tile's K range is split over `ksplit` CTAs so
// the 32-48 tiles of a projection fill the SMs; each writes its fp32 partial
// to the workspace and the tile's last CTA (ticket) sums the partials in
// split order -- the result does not depend on timing -- and writes y.  Per
// CTA:
//   warp 0     TMA producer: per 64-wide K step one box of 128 weight rows
//              (16 KB, 128-byte swizzle) and one box of the x rows, through
//              a ring of stages.  The weights never depend on the preceding
//              kernel, so the first stages' weight boxes are requested before
//              the programmatic-dependency wait; x only after it.
//   warp 1     MMA issuer (one thread): 4 MMAs per K step into one TMEM
//              accumulator (128 lanes = output features, rows in columns).
//   warps 2-5  epilogue: each thread owns one output feature (TMEM lane) and
//              reads its row of results 32 columns at a time.
// QKV mode (orthrus_linear_tc_qkv_rope): the tile of 128 features is one head
// of the fused QKV output; instead of y the epilogue writes q and k rotated by
// RoPE (the pair (i, i + 64) of a head lies in one tile: the threads of
// features n and n ^ 64 swap their bf16 values through shared memory) and v
// as is, with the cos/sin table of orthrus_rope_table -- the same bits as
// orthrus_linear_tc followed by orthrus_qkv_rope.
// Every mbarrier wait is bounded: on a timeout the kernel records
// ORTHRUS_ETIMEOUT, stops issuing, drains what it issued and still takes its
// ticket, so it always terminates.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "orthrus.h"
#include "tc_ptx.cuh"

namespace orthrus {
namespace {

constexpr int kThreads = 192;
constexpr int kTileN = 128;                // output features per tile (UMMA M)
constexpr int kStepK = 64;                 // K per box: one 128-byte swizzle row
constexpr int kMaxRows = 128;              // x rows per call (UMMA N)
constexpr int kMaxStages = 16;
constexpr int kRingBudget = 208 * 1024;
constexpr int kWBox = kTileN * 128;        // bytes of one weight box
constexpr int kNumBars = 2 * kMaxStages + 2;
constexpr int kXchgBytes = kTileN * 33 * 4;  // QKV mode: [128][33] floats

struct __align__(64) LinParams {
  CUtensorMap tm_w;  // 2D (K, N), box (64, 128)
  CUtensorMap tm_x;  // 2D (K, R), row pitch ldx, box (64, Rp); rows past R read as zero
  const __nv_bfloat16* residual;  // [R] rows of pitch ldy, or null
  __nv_bfloat16* y;               // [R] rows of pitch ldy
  float* part;                    // [tiles][ksplit][128][Rp + 4] fp32 split-K partials
  unsigned* tickets;              // [tiles], zero between calls
  int32_t* err;
  int R, Rp, N, ldy, tiles, ksplit, ksteps, stages, stage_bytes, tmem_cols;
  int kb;  // 64-wide K steps (weight box + x box each) per stage
  // QKV mode (rope != null): q [R, Hq, 128], k / v [R, Hkv, 128] instead of y
  const float2* rope;  // [R][64] (cos, sin)
  __nv_bfloat16 *q, *k, *v;
  int Hq, Hkv;
  // L2 warm-up hint: after its own loads each CTA prefetches its share
  const uint8_t* l2_next;
  int64_t l2_next_bytes;
};

struct Bars {
  uint32_t base;
  __device__ uint32_t at(int i) const { return base + 8 * i; }
  __device__ uint32_t full(int s) const { return at(s); }
  __device__ uint32_t empty(int s) const { return at(kMaxStages + s); }
  __device__ uint32_t acc_full() const { return at(2 * kMaxStages); }
  __device__ uint32_t red_full() const { return at(2 * kMaxStages + 1); }  // partials staged
};

__device__ __forceinline__ void record_timeout(int32_t* err, volatile int* abort_flag) {
  *abort_flag = 1;
  set_err(err, ORTHRUS_ETIMEOUT);
}

__device__ __forceinline__ float bf16_round(float v) {
  return __uint_as_float(ptx::pack_bf16x2(v, 0.f) << 16);
}

// The scalars of LinParams, read from the parameter space once at the start
// of the kernel (while the first loads are in flight) and kept in registers:
// left to the compiler, the epilogue's first reads of them are constant-cache
// misses on the critical path after the last MMA.
struct Scalars {
  const __nv_bfloat16* residual;
  __nv_bfloat16* y;
  float* part;
  unsigned* tickets;
  int32_t* err;
  int R, Rp, N, ldy, ksplit, ksteps, stages, stage_bytes, tmem_cols, kb;
  const float2* rope;
  __nv_bfloat16 *q, *k, *v;
  int Hq, Hkv;
};

template <typename T> __device__ __forceinline__ T* keep(T* v) {
  uint64_t u = reinterpret_cast<uint64_t>(v);
  asm volatile("" : "+l"(u));
  return reinterpret_cast<T*>(u);
}
__device__ __forceinline__ int keep(int v) {
  asm volatile("" : "+r"(v));
  return v;
}

__device__ __forceinline__ Scalars load_scalars(const LinParams& p) {
  Scalars c;
  c.residual = keep(p.residual); c.y = keep(p.y); c.part = keep(p.part);
  c.tickets = keep(p.tickets); c.err = keep(p.err);
  c.R = keep(p.R); c.Rp = keep(p.Rp); c.N = keep(p.N); c.ldy = keep(p.ldy);
  c.ksplit = keep(p.ksplit); c.ksteps = keep(p.ksteps); c.stages = keep(p.stages);
  c.stage_bytes = keep(p.stage_bytes); c.tmem_cols = keep(p.tmem_cols); c.kb = keep(p.kb);
  c.rope = keep(p.rope); c.q = keep(p.q); c.k = keep(p.k); c.v = keep(p.v);
  c.Hq = keep(p.Hq); c.Hkv = keep(p.Hkv);
  return c;
}

// The residual of rows cb .. cb + 31 of feature ng (zero past the rows, or
// without a residual), all loads in flight together.
__device__ __forceinline__ void load_residual(const Scalars& c, int cb, int ng,
                                              float (&res)[32]) {
  const int nr = min(32, c.R - cb);
#pragma unroll
  for (int j = 0; j < 32; ++j)
    res[j] = c.residual && j < nr
                 ? __bfloat162float(c.residual[(int64_t)(cb + j) * c.ldy + ng]) : 0.f;
}

// y[cb + j, ng] = bf16(bf16(v[j]) + res[j]) for the rows j < 32 of this chunk
// that exist (bf16(v[j]) without a residual).  The caller reads the residual
// before any y is written: the residual may be y itself.
__device__ __forceinline__ void store_rows(const Scalars& c, int cb, int ng, const float (&v)[32],
                                           const float (&res)[32]) {
  const int nr = min(32, c.R - cb);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (j < nr) {
      float o = bf16_round(v[j]);
      if (c.residual) o += res[j];
      c.y[(int64_t)(cb + j) * c.ldy + ng] = __float2bfloat16_rn(o);
    }
  }
}

// What a chunk of rows (cb .. cb + 31) of feature n needs besides its sums:
// the residual (plain mode) or the cos/sin of its rotation pair (QKV mode),
// all loads in flight together.
struct ChunkIn {
  float res[32];
  float2 cs[32];
};
__device__ __forceinline__ void load_chunk_in(const Scalars& c, int cb, int n, int ng,
                                              ChunkIn& in) {
  if (c.rope) {
    const int nr = min(32, c.R - cb);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      in.cs[j] = j < nr ? c.rope[(int64_t)(cb + j) * (kTileN / 2) + (n & (kTileN / 2 - 1))]
                        : make_float2(0.f, 0.f);
  } else {
    load_residual(c, cb, ng, in.res);
  }
}

// The chunk's outputs from its fp32 sums v[j].  Plain mode: y (store_rows).
// QKV mode: the 128 threads of the tile (named barrier 1; every one of them
// calls this, `live` says whether its values count) swap bf16 values with
// the feature n ^ 64 through `xchg` ([128][33] floats), rotate, and store
// to q / k (v: as is).
__device__ __forceinline__ void finish_chunk(const Scalars& c, int tile, int cb, int n, bool live,
                                             const float (&v)[32], const ChunkIn& in,
                                             float* xchg) {
  const int ng = tile * kTileN + n;
  if (!c.rope) {
    if (live && ng < c.N) store_rows(c, cb, ng, v, in.res);
    return;
  }
  float y[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    y[j] = bf16_round(v[j]);  // the projection's bf16 value
    xchg[n * 33 + j] = y[j];
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  const int nr = min(32, c.R - cb);
  const int pn = n ^ (kTileN / 2);
  const bool rot = tile < c.Hq + c.Hkv;
  __nv_bfloat16* dst;
  int pitch;  // elements between rows
  if (tile < c.Hq) {
    dst = c.q + (int64_t)tile * kTileN + n;
    pitch = c.Hq * kTileN;
  } else if (rot) {
    dst = c.k + (int64_t)(tile - c.Hq) * kTileN + n;
    pitch = c.Hkv * kTileN;
  } else {
    dst = c.v + (int64_t)(tile - c.Hq - c.Hkv) * kTileN + n;
    pitch = c.Hkv * kTileN;
  }
  float o[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float yp = xchg[pn * 33 + j];
    o[j] = !rot ? y[j]
           : n < kTileN / 2 ? rope_first(y[j], yp, in.cs[j]) : rope_second(yp, y[j], in.cs[j]);
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");  // xchg free for the next chunk
  if (live) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < nr) dst[(int64_t)(cb + j) * pitch] = __float2bfloat16_rn(o[j]);
  }
}

template <bool kQkv>
__global__ void __launch_bounds__(kThreads, 1) linear_tc_kernel(const __grid_constant__ LinParams p) {
  Scalars c = load_scalars(p);
  if (!kQkv) c.rope = nullptr;  // plain mode: the compiler drops the QKV paths
  extern __shared__ uint8_t smem_raw[];
  // 1 KB aligned for the 128-byte swizzle; offset from smem_raw itself so
  // the compiler keeps the shared address space
  uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned full_mask = 0xffffffffu;
  const int ST = c.stages, SB = c.stage_bytes;
  const Bars bars{sbase + (uint32_t)(ST * SB)};
  uint8_t* misc = smem + ST * SB + kNumBars * 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(misc + 8);
  // QKV mode's swap area: the end of the ring, idle by the time it is used
  float* xchg = reinterpret_cast<float*>(smem + ST * SB - kXchgBytes);

  const int tile = blockIdx.x / c.ksplit, ks = blockIdx.x % c.ksplit;
  const int k_beg = (int)((int64_t)ks * c.ksteps / c.ksplit);
  const int nsteps = (int)((int64_t)(ks + 1) * c.ksteps / c.ksplit) - k_beg;
  const int KB = c.kb;
  const int nk = ceil_div(nsteps, KB);  // stages this CTA streams (the last may be short)
  const int n0 = tile * kTileN;
  const uint32_t x_bytes = (uint32_t)(c.Rp * 128);
  const uint32_t x_off = (uint32_t)(KB * kWBox);  // the x boxes follow the stage's weight boxes
  // K steps of stage i: [k_beg + i KB, k_beg + min(nsteps, (i + 1) KB))
  auto steps_of = [&](int i) { return min(KB, nsteps - i * KB); };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *last_flag = 0;
    for (int s = 0; s < ST; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.empty(s), 1);
    }
    ptx::mbar_init(bars.acc_full(), 1);
    ptx::mbar_init(bars.red_full(), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&p.tm_w);
    ptx::tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), (uint32_t)c.tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  ptx::griddep_launch_dependents();

  // the weights are constant: their first boxes stream before the wait for
  // the preceding kernel (which may be writing x or the residual)
  const int early = min(nk, ST);
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < early; ++i) {
      const int ns = steps_of(i);
      ptx::mbar_expect_tx(bars.full(i), (uint32_t)ns * ((uint32_t)kWBox + x_bytes));
      for (int j = 0; j < ns; ++j)
        ptx::tma_load_2d(sbase + (uint32_t)(i * SB + j * kWBox), &p.tm_w, bars.full(i),
                         (k_beg + i * KB + j) * kStepK, n0);
    }
  }
  ptx::griddep_wait();

  if (warp == 0) {
    // ================================================== TMA producer
    if (lane == 0) {
      // the x boxes of the early stages first: with them every stage whose
      // weights are in flight can complete
      for (int i = 0; i < early; ++i)
        for (int j = 0; j < steps_of(i); ++j)
          ptx::tma_load_2d(sbase + (uint32_t)(i * SB) + x_off + (uint32_t)(j * x_bytes), &p.tm_x,
                           bars.full(i), (k_beg + i * KB + j) * kStepK, 0);
      int issued = early;
      for (int i = early; i < nk; ++i) {
        if (*abort_flag) break;
        const int s = i % ST, ns = steps_of(i);
        const uint32_t dst = sbase + (uint32_t)(s * SB);
        if (!ptx::mbar_wait(bars.empty(s), ((i / ST) & 1) ^ 1)) {
          record_timeout(c.err, abort_flag);
          break;
        }
        ptx::mbar_expect_tx(bars.full(s), (uint32_t)ns * ((uint32_t)kWBox + x_bytes));
        for (int j = 0; j < ns; ++j) {
          ptx::tma_load_2d(dst + (uint32_t)(j * kWBox), &p.tm_w, bars.full(s),
                           (k_beg + i * KB + j) * kStepK, n0);
          ptx::tma_load_2d(dst + x_off + (uint32_t)(j * x_bytes), &p.tm_x, bars.full(s),
                           (k_beg + i * KB + j) * kStepK, 0);
        }
        issued = i + 1;
      }
      // every issued load lands before the CTA can exit
      for (int u = max(0, issued - ST); u < issued; ++u)
        if (!ptx::mbar_wait(bars.full(u % ST), (u / ST) & 1)) record_timeout(c.err, abort_flag);
      // this CTA's share of the next call's weights into L2 (a hint: the
      // loads are not waited for and change no result)
      if (p.l2_next && p.l2_next_bytes > 0) {
        const int64_t units = p.l2_next_bytes / 16, per = (units + gridDim.x - 1) / gridDim.x;
        const int64_t beg = (int64_t)blockIdx.x * per, end = min(units, beg + per);
        for (int64_t u0 = beg; u0 < end; u0 += 2048)  // 32 KB a request
          ptx::bulk_prefetch_l2(p.l2_next + u0 * 16, (uint32_t)(min(end - u0, (int64_t)2048) * 16));
      }
    }
  } else if (warp == 1) {
    // ================================================== MMA issuer
    if (lane == 0) {
      const uint32_t id = ptx::idesc_bf16(kTileN, c.Rp, false, false);
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int s = i % ST;
        if (*abort_flag || !ptx::mbar_wait(bars.full(s), (i / ST) & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t wa = sbase + (uint32_t)(s * SB);
        for (int j = 0; j < steps_of(i); ++j) {
#pragma unroll
          for (int kk = 0; kk < kStepK / 16; ++kk)
            ptx::mma_ss(tmem, ptx::sdesc_sw128(wa + j * kWBox + kk * 32, 16, 1024),
                        ptx::sdesc_sw128(wa + x_off + j * x_bytes + kk * 32, 16, 1024), id,
                        (i > 0 || j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::tc_commit(bars.empty(s));
      }
      if (!ok) record_timeout(c.err, abort_flag);
      ptx::tc_commit(bars.acc_full());  // also: every MMA has finished
      if (!ptx::mbar_wait(bars.acc_full(), 0)) record_timeout(c.err, abort_flag);
    }
  } else {
    // ================================================== epilogue
    const int quad = warp & 3;
    const int n = quad * 32 + lane;  // output feature within the tile (TMEM lane)
    const int ng = n0 + n;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    bool ok = nk > 0 && __all_sync(full_mask, ptx::mbar_wait(bars.acc_full(), 0));
    if (nk > 0 && !ok) record_timeout(c.err, abort_flag);
    ok = ok && !__any_sync(full_mask, *abort_flag != 0);
    if (ok) ptx::tc_fence_after();
    const int RP4 = c.Rp + 4;  // padded column of the partials: conflict-free reads
    float* part = c.part + (((int64_t)tile * c.ksplit + ks) * kTileN + n) * RP4;
    for (int cb = 0; cb < c.Rp; cb += 32) {
      const int nc = min(32, c.Rp - cb);  // 32, or the last 16 (Rp is a multiple of 16)
      uint32_t d[32];
      if (ok) {
        if (nc == 32) {
          ptx::tmem_ld32_sync(lane_addr + (uint32_t)cb, d);
        } else {
          uint32_t d16[16];
          ptx::tmem_ld16_sync(lane_addr + (uint32_t)cb, d16);
#pragma unroll
          for (int j = 0; j < 16; ++j) d[j] = d16[j];
#pragma unroll
          for (int j = 16; j < 32; ++j) d[j] = 0u;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) d[j] = 0u;
      }
      if (c.ksplit == 1) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(d[j]);
        ChunkIn in;
        if (ok && ng < c.N) load_chunk_in(c, cb, n, ng, in);
        finish_chunk(c, tile, cb, n, ok, v, in, xchg);
      } else {
        // this feature's partial sums of rows cb .. cb + nc - 1, contiguous
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          if (j < nc)
            __stcg(reinterpret_cast<float4*>(part + cb + j),
                   make_float4(__uint_as_float(d[j]), __uint_as_float(d[j + 1]),
                               __uint_as_float(d[j + 2]), __uint_as_float(d[j + 3])));
      }
    }
  }

  // ---- teardown; with split K, the tile's last CTA sums the partials
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, (uint32_t)c.tmem_cols);
  }
  if (c.ksplit == 1) return;
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's partial is visible before its ticket
    *last_flag = atomicAdd(c.tickets + tile, 1u) == (unsigned)c.ksplit - 1u;
  }
  __syncthreads();
  if (!*last_flag) return;
  // the tile's partials (one contiguous 128 x (Rp + 4) block per split) come
  // into the idle ring by bulk copies, all in flight at once; thread n then
  // sums feature n's rows in split order
  const int RP4 = c.Rp + 4;
  const float* base = c.part + (int64_t)tile * c.ksplit * kTileN * RP4;
  const uint32_t blk_bytes = (uint32_t)(kTileN * RP4 * 4);
  if (threadIdx.x == 0) {
    __threadfence();
    ptx::fence_proxy_async_global();  // the partials were written by generic stores
    ptx::mbar_expect_tx(bars.red_full(), blk_bytes * (uint32_t)c.ksplit);
    for (int s = 0; s < c.ksplit; ++s)
      ptx::bulk_g2s(sbase + (uint32_t)s * blk_bytes, base + (int64_t)s * kTileN * RP4, blk_bytes,
                    bars.red_full());
  }
  // the first rows' residual (or cos/sin) comes in while the partials do
  const int n = threadIdx.x, ng = n0 + n;
  ChunkIn in;
  if (n < kTileN && ng < c.N) load_chunk_in(c, 0, n, ng, in);
  const bool got = ptx::mbar_wait(bars.red_full(), 0);
  if (!got) set_err(c.err, ORTHRUS_ETIMEOUT);
  if (n < kTileN) {  // every thread of the tile: QKV mode's barriers
    const float* st = reinterpret_cast<const float*>(smem) + n * RP4;
    {
      for (int cb = 0; cb < c.Rp; cb += 32) {
        if (cb > 0 && ng < c.N) load_chunk_in(c, cb, n, ng, in);
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
        for (int sp = 0; sp < c.ksplit; ++sp) {
          const float* src = st + (int64_t)sp * kTileN * RP4 + cb;
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            if (got && cb + j < c.Rp) {
              const float4 f = *reinterpret_cast<const float4*>(src + j);
              v[j] += f.x; v[j + 1] += f.y; v[j + 2] += f.z; v[j + 3] += f.w;
            }
          }
        }
        finish_chunk(c, tile, cb, n, got, v, in, xchg);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) c.tickets[tile] = 0u;
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

bool encode_2d(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t pitch_bytes,
               int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)pitch_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)kStepK, (cuuint32_t)box_rows};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

struct Plan {
  int Rp, tiles, ksplit, ksteps, stages, stage_bytes, smem, tmem_cols, kb;
};

// Launch shape for rows x K x N on `sms` SMs: 128-feature tiles, the K range
// of each split over enough CTAs to fill the SMs (at most one 64-wide K step
// less than an even share each), a ring of as many stages as fit.
Plan plan(int rows, int K, int N, int sms, int kb, bool qkv = false) {
  Plan q;
  q.Rp = (rows + 15) / 16 * 16;
  q.ksteps = K / kStepK;
  q.tiles = ceil_div(N, kTileN);
  // kb K steps per stage: their weight boxes, then their x boxes (each x box
  // Rp rows of 128 bytes; kb * Rp * 128 rounded up to 1 KB keeps every box
  // of the next stage 1 KB aligned for the 128-byte swizzle)
  q.kb = kb;
  q.stage_bytes = kb * kWBox + (kb * q.Rp * 128 + 1023) / 1024 * 1024;
  q.stages = min(kMaxStages, kRingBudget / q.stage_bytes);
  // splits: enough to fill the SMs, at most one per K step, at most 16, and
  // no more than the ring can stage for the last CTA's sum
  q.ksplit = q.tiles >= sms ? 1 : sms / q.tiles;
  q.ksplit = min(q.ksplit, min(q.ksteps, 16));
  // (QKV mode keeps the ring's last kXchgBytes for its swap area)
  q.ksplit = max(1, min(q.ksplit, (q.stages * q.stage_bytes - (qkv ? kXchgBytes : 0)) /
                                      ((q.Rp + 4) * kTileN * 4)));
  q.smem = q.stages * q.stage_bytes + kNumBars * 8 + 16 + 1024;
  q.tmem_cols = 32;
  while (q.tmem_cols < q.Rp) q.tmem_cols *= 2;
  return q;
}

// The most K steps per stage (up to kMaxKb) that still leave two stages.
constexpr int kMaxKb = 4;
int choose_kb(int rows) {
  const int Rp = (rows + 15) / 16 * 16;
  for (int kb = kMaxKb; kb > 1; kb /= 2)
    if (kRingBudget / (kb * kWBox + (kb * Rp * 128 + 1023) / 1024 * 1024) >= 2) return kb;
  return 1;
}

Plan plan(int rows, int K, int N, int sms, bool qkv = false) {
  return plan(rows, K, N, sms, choose_kb(rows), qkv);
}

size_t round256(int64_t n) { return (size_t)((n + 255) / 256 * 256); }

size_t workspace_bytes(int rows, int K, int N) {
  // sized for any SM count up to 256
  const Plan q = plan(rows, K, N, 256);
  const int64_t parts = q.ksplit > 1 ? (int64_t)q.tiles * 16 * (q.Rp + 4) * kTileN * 4 : 0;
  return round256((int64_t)q.tiles * 4) + (size_t)parts;
}

// cos/sin table of RoPE for the rows of the blocks: row r = b * blk + j at
// position ctx_lens[b] + j, frequencies i < hd / 2 (the values the
// stand-alone RoPE kernel computes).
__global__ void rope_table_kernel(const int32_t* __restrict__ ctx_lens, int blk, int hd,
                                  double theta, float2* __restrict__ table) {
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int r = blockIdx.x, half = hd / 2;
  const int64_t pos = (int64_t)ctx_lens[r / blk] + r % blk;
  for (int i = threadIdx.x; i < half; i += blockDim.x)
    table[(int64_t)r * half + i] = rope_cos_sin(pos, i, hd, theta);
}

bool prepare() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < 64 && done[dev]) return true;
  if (cudaFuncSetAttribute(linear_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           227 * 1024) != cudaSuccess ||
      cudaFuncSetAttribute(linear_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           227 * 1024) != cudaSuccess)
    return false;
  if (dev >= 0 && dev < 64) done[dev] = true;
  return true;
}

// Common tail of the entry points: plan, tensor maps, workspace, launch.
int launch_linear(LinParams& p, const void* x, int rows, int K, int64_t ldx, const void* w,
                  int N, bool qkv, const void* l2_next, int64_t l2_next_bytes, int32_t* err,
                  void* workspace, size_t workspace_bytes_given, orthrus_stream_t stream) {
  if (l2_next_bytes < 0 || (l2_next && (reinterpret_cast<uintptr_t>(l2_next) % 16 ||
                                        l2_next_bytes % 16)))
    return ORTHRUS_EINVAL;
  p.l2_next = l2_next_bytes > 0 ? static_cast<const uint8_t*>(l2_next) : nullptr;
  p.l2_next_bytes = p.l2_next ? l2_next_bytes : 0;
  if (!workspace || workspace_bytes_given < workspace_bytes(rows, K, N) ||
      reinterpret_cast<uintptr_t>(workspace) % 256)
    return ORTHRUS_EWORKSPACE;
  const int sms = sm_count();
  if (sms <= 0) return ORTHRUS_ECUDA;
  if (!prepare()) return ORTHRUS_ECUDA;
  const Plan q = plan(rows, K, N, sms, qkv);
  if (!encode_2d(&p.tm_w, w, K, N, (int64_t)K * 2, kTileN) ||
      !encode_2d(&p.tm_x, x, K, rows, ldx * 2, q.Rp))
    return ORTHRUS_ECUDA;
  char* ws = static_cast<char*>(workspace);
  p.tickets = reinterpret_cast<unsigned*>(ws);
  p.part = reinterpret_cast<float*>(ws + round256((int64_t)q.tiles * 4));
  p.err = err;
  p.R = rows; p.Rp = q.Rp; p.N = N;
  p.tiles = q.tiles; p.ksplit = q.ksplit; p.ksteps = q.ksteps; p.stages = q.stages;
  p.stage_bytes = q.stage_bytes; p.tmem_cols = q.tmem_cols; p.kb = q.kb;

  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(q.tiles * q.ksplit);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = q.smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = qkv ? cudaLaunchKernelEx(&cfg, linear_tc_kernel<true>, p)
                            : cudaLaunchKernelEx(&cfg, linear_tc_kernel<false>, p);
  return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA;
}

}  // namespace
}  // namespace orthrus

using namespace orthrus;

extern "C" {

int orthrus_linear_tc_plan(int32_t rows, int32_t K, int32_t N, int32_t sms, int32_t* out) {
  if (!out || rows < 1 || rows > kMaxRows || K < kStepK || K % kStepK || N < 1 || sms < 1)
    return ORTHRUS_EINVAL;
  const Plan q = plan(rows, K, N, sms);
  out[0] = q.tiles;
  out[1] = q.ksplit;
  out[2] = q.stages;
  out[3] = q.stage_bytes;
  out[4] = q.smem;
  out[5] = q.tiles * q.ksplit;  // grid
  out[6] = q.tmem_cols;
  out[7] = q.Rp;
  return ORTHRUS_OK;
}

size_t orthrus_linear_tc_workspace(int32_t rows, int32_t K, int32_t N) {
  if (rows < 1 || rows > kMaxRows || K < kStepK || K % kStepK || N < 1) return 0;
  return workspace_bytes(rows, K, N);
}

int orthrus_linear_tc(int32_t dtype, const void* x, int32_t rows, int32_t K, int64_t ldx,
                      const void* w, int32_t N, const void* residual, void* y, int64_t ldy,
                      const void* l2_next, int64_t l2_next_bytes, int32_t* err,
                      void* workspace, size_t workspace_bytes_given, orthrus_stream_t stream) {
  if (dtype != ORTHRUS_F32 && dtype != ORTHRUS_BF16) return ORTHRUS_EINVAL;
  if (rows < 0 || K <= 0 || N <= 0 || ldx < K || ldy < N) return ORTHRUS_EINVAL;
  if (dtype != ORTHRUS_BF16) return ORTHRUS_EUNSUPPORTED;
  if (rows == 0) return ORTHRUS_OK;
  if (rows > kMaxRows || K % kStepK || ldx % 8) return ORTHRUS_EUNSUPPORTED;
  if (!x || !w || !y) return ORTHRUS_EINVAL;
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(w) % 16 ||
      reinterpret_cast<uintptr_t>(y) % 2 || reinterpret_cast<uintptr_t>(residual) % 2)
    return ORTHRUS_EINVAL;
  LinParams p = {};
  p.residual = static_cast<const __nv_bfloat16*>(residual);
  p.y = static_cast<__nv_bfloat16*>(y);
  p.ldy = (int)ldy;
  return launch_linear(p, x, rows, K, ldx, w, N, false, l2_next, l2_next_bytes, err, workspace,
                       workspace_bytes_given, stream);
}

int orthrus_rope_table(const int32_t* ctx_lens, int32_t B, int32_t blk, int32_t hd, double theta,
                       float* cos_sin, orthrus_stream_t stream) {
  if (B < 0 || blk <= 0 || hd <= 0 || hd % 2 || !(theta > 0.0)) return ORTHRUS_EINVAL;
  if (B == 0) return ORTHRUS_OK;
  if (!ctx_lens || !cos_sin || reinterpret_cast<uintptr_t>(cos_sin) % 8) return ORTHRUS_EINVAL;
  const int64_t rows = (int64_t)B * blk;
  if (rows > 2147483647LL) return ORTHRUS_EUNSUPPORTED;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3((unsigned)std::min(hd / 2, 256));
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, rope_table_kernel, ctx_lens, (int)blk, (int)hd, theta,
                            reinterpret_cast<float2*>(cos_sin)) == cudaSuccess
             ? ORTHRUS_OK
             : ORTHRUS_ECUDA;
}

int orthrus_linear_tc_qkv_rope(int32_t dtype, const void* x, int32_t rows, int32_t K,
                               int64_t ldx, const void* w, int32_t Hq, int32_t Hkv, int32_t hd,
                               const float* cos_sin, void* q, void* k, void* v,
                               const void* l2_next, int64_t l2_next_bytes, int32_t* err,
                               void* workspace, size_t workspace_bytes_given,
                               orthrus_stream_t stream) {
  if (dtype != ORTHRUS_F32 && dtype != ORTHRUS_BF16) return ORTHRUS_EINVAL;
  if (rows < 0 || K <= 0 || ldx < K || Hq <= 0 || Hkv <= 0 || hd <= 0 || hd % 2)
    return ORTHRUS_EINVAL;
  if (dtype != ORTHRUS_BF16 || hd != kTileN) return ORTHRUS_EUNSUPPORTED;
  if (rows == 0) return ORTHRUS_OK;
  if (rows > kMaxRows || K % kStepK || ldx % 8) return ORTHRUS_EUNSUPPORTED;
  if (!x || !w || !cos_sin || !q || !k || !v) return ORTHRUS_EINVAL;
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(w) % 16 ||
      reinterpret_cast<uintptr_t>(cos_sin) % 8 || reinterpret_cast<uintptr_t>(q) % 2 ||
      reinterpret_cast<uintptr_t>(k) % 2 || reinterpret_cast<uintptr_t>(v) % 2)
    return ORTHRUS_EINVAL;
  const int64_t N = (int64_t)(Hq + 2 * Hkv) * hd;
  if (N > 2147483647LL) return ORTHRUS_EUNSUPPORTED;
  LinParams p = {};
  p.rope = reinterpret_cast<const float2*>(cos_sin);
  p.q = static_cast<__nv_bfloat16*>(q);
  p.k = static_cast<__nv_bfloat16*>(k);
  p.v = static_cast<__nv_bfloat16*>(v);
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.ldy = (int)N;
  return launch_linear(p, x, rows, K, ldx, w, (int)N, true, l2_next, l2_next_bytes, err,
                       workspace, workspace_bytes_given, stream);
}

}  // extern "C"
