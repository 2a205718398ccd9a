// lm_head.cu -- the LM head with the row argmax in its epilogue: for each
// row r of the final hidden states h [R, d] (bf16),
//   idx[r] = argmax_v sum_k h[r, k] w[v, k]      (lowest index on ties)
// over the output embedding w [V, d] (bf16), without the R x V logits ever
// leaving the SM.  Every Orthrus view ends in this product (cjcn.com.cn
// explainer of "Orthrus", §二: the LM head is shared by both views) and the
// round takes the argmax of its rows twice (§四: drafts from the diffusion
// rows, the AR tokens from the verify rows).
//
// tcgen05 GEMM, D[hidden row, vocab row] = h w^T, one CTA per SM over a
// contiguous range of vocabulary tiles of nv rows (nv chosen on the host so
// the tiles spread evenly over the SMs: at vocabulary 151936, 176 rows when
// four boxes per stage fit, else 208):
//   warp 0     TMA producers: lane 0 streams per stage kb consecutive
//              64-column boxes of the w slice (nv rows each, K-major, 128-byte
//              swizzle) -- the HBM stream -- into the w ring; lane 1 the
//              matching columns of h (L2-resident) into a separate, short h
//              ring, whose slots are free again as soon as the copying warps
//              have moved them into TMEM, so h takes little of the shared
//              memory the w stream needs for its bytes in flight.  w never
//              depends on the preceding kernel: its first stages are requested
//              before the programmatic-dependency wait, h only after it
//   warp 1     MMA issuer (one thread): per stage 4 kb MMAs of K = 16 with
//              A = the stage's 64 kb columns of h from TMEM (128 lanes = hidden
//              rows, zero past R) and B = the w slice from shared memory,
//              N = nv, into one TMEM accumulator (the rest of TMEM holds the
//              h ring)
//   warps 2-5  per warp quadrant holding hidden rows: copy each stage's h
//              columns from the h ring into a small TMEM ring ahead of the
//              MMAs, then for each finished tile scan the thread's row of D
//              for its best (value, index), kept across the CTA's tiles; a
//              w stage is free once its MMAs are done, an h slot once it is
//              copied
// Operand A from TMEM leaves shared memory to the w stream: with A in shared
// memory as well, the MMA issue rate, not HBM, bounded the kernel.
// At the end each hidden row's CTA best goes to a 64-bit slot (value order,
// lowest index) by atomicMax, and the last CTA (ticket) writes idx / maxval
// and returns the workspace to zero.
//
// Every mbarrier wait is bounded: on a timeout the kernel records
// ORTHRUS_ETIMEOUT in the error word, stops issuing work, drains what it
// issued and still reaches the final ticket, so it always terminates.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <climits>
#include <mutex>

#include "common.cuh"
#include "orthrus.h"
#include "tc_ptx.cuh"

namespace orthrus {
namespace {

constexpr int kThreads = 192;
constexpr int kRowsMax = 128;           // hidden rows per call (UMMA M, TMEM lanes)
constexpr int kStepK = 64;              // d elements per box (one 128-byte swizzle row)
constexpr int kMaxStages = 12;
constexpr int kRingBudget = 220 * 1024; // shared memory for the w and h rings
constexpr int kTmemCols = 512;
constexpr int kMaxASlots = 8;
constexpr int kMaxHSlots = 4;           // h ring slots (kb boxes each)
constexpr int kHBoxesAhead = 4;         // h boxes the h ring holds at least
constexpr int kNumBars = 2 * kMaxStages + 2 * kMaxASlots + 2 * kMaxHSlots + 3;

struct __align__(64) LmParams {
  CUtensorMap tm_w;                 // 2D (d, V), box (64, nv)
  CUtensorMap tm_h;                 // 2D (d, R), row pitch ldh, box (64, 32 * writers)
  unsigned long long* slots;        // [R] 64-bit (value, index) keys, zero between calls
  unsigned* ticket;
  int32_t* idx;
  float* maxval;
  int32_t* err;
  int R, V, nv, nvp, ksteps, tiles, stages, stage_bytes, w_bytes, aslots, a_col, writers, kb,
      kst, hb;  // kb boxes per stage, kst stages per tile, hb bytes of one h box
  // w ring: stages x stage_bytes (= w_bytes, kb w boxes); h ring: hslots x
  // h_bytes (kb h boxes)
  int h_bytes, hslots;
};

struct Layout {
  int bars, misc, total;
};
__host__ __device__ inline Layout layout(int stages, int stage_bytes, int h_bytes, int hslots) {
  Layout l;
  l.bars = stages * stage_bytes + hslots * h_bytes;
  l.misc = l.bars + kNumBars * 8;
  l.total = l.misc + 16;
  return l;
}

struct Bars {
  uint32_t base;
  __device__ uint32_t at(int i) const { return base + 8 * i; }
  __device__ uint32_t full(int s) const { return at(s); }
  __device__ uint32_t empty(int s) const { return at(kMaxStages + s); }
  __device__ uint32_t a_full(int j) const { return at(2 * kMaxStages + j); }
  __device__ uint32_t a_empty(int j) const { return at(2 * kMaxStages + kMaxASlots + j); }
  __device__ uint32_t acc_full() const { return at(2 * kMaxStages + 2 * kMaxASlots); }
  __device__ uint32_t acc_empty() const { return at(2 * kMaxStages + 2 * kMaxASlots + 1); }
  __device__ uint32_t mma_done() const { return at(2 * kMaxStages + 2 * kMaxASlots + 2); }
  __device__ uint32_t h_full(int j) const { return at(2 * kMaxStages + 2 * kMaxASlots + 3 + j); }
  __device__ uint32_t h_empty(int j) const {
    return at(2 * kMaxStages + 2 * kMaxASlots + 3 + kMaxHSlots + j);
  }
};

__device__ __forceinline__ void record_timeout(int32_t* err, volatile int* abort_flag) {
  *abort_flag = 1;
  set_err(err, ORTHRUS_ETIMEOUT);
}

// 64-bit key ordering (value, lowest index first); -0 == +0.
__device__ __forceinline__ unsigned long long pack_key(float v, int i) {
  if (v == 0.f) v = 0.f;
  unsigned u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (unsigned)i);
}
__device__ __forceinline__ int key_index(unsigned long long k) {
  return (int)(0xFFFFFFFFu - (unsigned)(k & 0xFFFFFFFFull));
}
__device__ __forceinline__ float key_value(unsigned long long k) {
  unsigned u = (unsigned)(k >> 32);
  u = (u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u;
  return __uint_as_float(u);
}

__global__ void __launch_bounds__(kThreads, 1)
lm_head_argmax_kernel(const __grid_constant__ LmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned full_mask = 0xffffffffu;
  const int ST = p.stages, SB = p.stage_bytes, AS = p.aslots;
  const int HS = p.hslots;
  const Layout L = layout(ST, SB, p.h_bytes, HS);
  const uint32_t hbase = (uint32_t)(ST * SB);  // the h ring follows the w ring
  const Bars bars{sbase + (uint32_t)L.bars};
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L.misc + 8);

  const int t_beg = (int)((int64_t)blockIdx.x * p.tiles / gridDim.x);
  const int t_end = (int)((int64_t)(blockIdx.x + 1) * p.tiles / gridDim.x);
  const int ntiles = t_end - t_beg;
  const int total = ntiles * p.kst;  // stages of this CTA
  const int KB = p.kb;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *last_flag = 0;
    for (int s = 0; s < kMaxStages; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.empty(s), 1);  // the stage's MMA commit
    }
    for (int j = 0; j < kMaxHSlots; ++j) {
      ptx::mbar_init(bars.h_full(j), 1);
      ptx::mbar_init(bars.h_empty(j), (uint32_t)p.writers);  // every copying warp
    }
    for (int j = 0; j < kMaxASlots; ++j) {
      ptx::mbar_init(bars.a_full(j), (uint32_t)p.writers);
      ptx::mbar_init(bars.a_empty(j), 1);
    }
    ptx::mbar_init(bars.acc_full(), 1);
    ptx::mbar_init(bars.acc_empty(), (uint32_t)p.writers);
    ptx::mbar_init(bars.mma_done(), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&p.tm_w);
    ptx::tma_prefetch_desc(&p.tm_h);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int quad = warp & 3;  // TMEM lane quadrant of warps 2-5
  const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
  if (warp >= 2) {  // the A ring starts zero on every lane (rows past R stay zero)
    uint32_t z[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) z[j] = 0u;
    for (int j = 0; j < AS; ++j) ptx::tmem_st32(lane_addr + (uint32_t)(p.a_col + 32 * j), z);
    ptx::tmem_wait_st();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  ptx::griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    // ================================================== w producer
    // the output embedding is never written by the preceding kernel: the
    // first stages stream before the wait for it
    auto issue_w = [&](int it) {
      const int s = it % ST, t = t_beg + it / p.kst, k0 = (it % p.kst) * KB;
      const uint32_t dst = sbase + (uint32_t)(s * SB);
      ptx::mbar_expect_tx(bars.full(s), (uint32_t)SB);
      for (int j = 0; j < KB; ++j)
        ptx::tma_load_2d(dst + (uint32_t)(j * p.nv * 128), &p.tm_w, bars.full(s),
                         (k0 + j) * kStepK, t * p.nv);
    };
    const int early = min(total, ST);
    for (int it = 0; it < early; ++it) issue_w(it);
    ptx::griddep_wait();
    int it = early;
    for (; it < total; ++it) {
      if (*abort_flag) break;
      if (!ptx::mbar_wait(bars.empty(it % ST), ((it / ST) & 1) ^ 1)) {
        record_timeout(p.err, abort_flag);
        break;
      }
      issue_w(it);
    }
    // every issued load lands before the CTA can exit
    for (int u = max(0, it - ST); u < it; ++u)
      if (!ptx::mbar_wait(bars.full(u % ST), (u / ST) & 1)) record_timeout(p.err, abort_flag);
  } else if (warp == 0) {
    ptx::griddep_wait();
    if (lane == 1) {
      // ================================================== h producer
      int it = 0;
      for (; it < total; ++it) {
        if (*abort_flag) break;
        const int j = it % HS, k0 = (it % p.kst) * KB;
        if (!ptx::mbar_wait(bars.h_empty(j), ((it / HS) & 1) ^ 1)) {
          record_timeout(p.err, abort_flag);
          break;
        }
        const uint32_t dst = sbase + hbase + (uint32_t)(j * p.h_bytes);
        ptx::mbar_expect_tx(bars.h_full(j), (uint32_t)p.h_bytes);
        for (int b = 0; b < KB; ++b)
          ptx::tma_load_2d(dst + (uint32_t)(b * p.hb), &p.tm_h, bars.h_full(j),
                           (k0 + b) * kStepK, 0);
      }
      for (int u = max(0, it - HS); u < it; ++u)
        if (!ptx::mbar_wait(bars.h_full(u % HS), (u / HS) & 1))
          record_timeout(p.err, abort_flag);
    }
  } else if (warp == 1) {
    // ================================================== MMA issuer
    ptx::griddep_wait();
    if (lane == 0) {
      const uint32_t id = ptx::idesc_bf16(kRowsMax, p.nv, false, false);
      bool ok = true;
      int it = 0;
      for (int i = 0; ok && i < ntiles; ++i) {
        if (i >= 1 && !ptx::mbar_wait(bars.acc_empty(), (i - 1) & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        for (int k = 0; k < p.kst; ++k, ++it) {
          const int s = it % ST, a = it % AS;
          if (*abort_flag || !ptx::mbar_wait(bars.full(s), (it / ST) & 1) ||
              !ptx::mbar_wait(bars.a_full(a), (it / AS) & 1)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t b0 = sbase + (uint32_t)(s * SB);
          const uint32_t a0 = tmem + (uint32_t)(p.a_col + 32 * KB * a);
          for (int j = 0; j < KB; ++j) {
#pragma unroll
            for (int kk = 0; kk < kStepK / 16; ++kk) {
              ptx::mma_ts(tmem, a0 + 32 * j + 8 * kk,
                          ptx::sdesc_sw128(b0 + j * p.nv * 128 + kk * 32, 16, 1024), id,
                          (k > 0 || j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          ptx::tc_commit(bars.empty(s));
          ptx::tc_commit(bars.a_empty(a));
        }
        if (!ok) break;
        ptx::tc_commit(bars.acc_full());
      }
      if (!ok) record_timeout(p.err, abort_flag);
      // every MMA issued has finished before TMEM is released
      ptx::tc_commit(bars.mma_done());
      if (!ptx::mbar_wait(bars.mma_done(), 0)) record_timeout(p.err, abort_flag);
    }
  } else if (quad >= p.writers) {
    ptx::griddep_wait();  // idle warp: it still takes part in the ticket's write-out
  } else {
    // ================================================== h writer + epilogue
    ptx::griddep_wait();
    const int r = quad * 32 + lane;  // hidden row of this thread
    const bool valid = r < p.R;
    float best_v = -INFINITY;
    int best_i = INT_MAX;
    bool ok = true;
    int it_w = 0;  // next h slice to copy (global stage index)
    for (int i = 0; ok && i < ntiles; ++i) {
      // this tile's slices, then the next tile's first ones: at most as many
      // as the TMEM slice ring holds, so that the slot of each is freed by an
      // MMA of this tile, which does not wait on this tile's scan (one more
      // would wait on an MMA of the next tile, which waits on that scan).  An
      // h slot depends on nothing but this loop: it is free once copied.
      const int limit = min(min((i + 1) * p.kst + AS, (i + 2) * p.kst), total);
      for (; it_w < limit; ++it_w) {
        const int a = it_w % AS, j = it_w % HS;
        if (__any_sync(full_mask, *abort_flag != 0) ||
            !__all_sync(full_mask, ptx::mbar_wait(bars.h_full(j), (it_w / HS) & 1)) ||
            !__all_sync(full_mask, ptx::mbar_wait(bars.a_empty(a), ((it_w / AS) & 1) ^ 1))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        for (int b = 0; b < KB; ++b) {
          // row r of box b: 128 bytes, 16-byte chunk j at (j ^ (r & 7)) (128-byte swizzle)
          const uint8_t* hs = smem + hbase + j * p.h_bytes + b * p.hb + r * 128;
          uint32_t x[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint4 q = *reinterpret_cast<const uint4*>(hs + ((j ^ (r & 7)) << 4));
            x[4 * j] = q.x; x[4 * j + 1] = q.y; x[4 * j + 2] = q.z; x[4 * j + 3] = q.w;
          }
          ptx::tmem_st32(lane_addr + (uint32_t)(p.a_col + 32 * (KB * a + b)), x);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(bars.a_full(a));
          ptx::mbar_arrive(bars.h_empty(j));  // this warp is done with the slot's h rows
        }
      }
      if (!ok) break;
      // scan this thread's row of tile i
      if (__any_sync(full_mask, *abort_flag != 0) ||
          !__all_sync(full_mask, ptx::mbar_wait(bars.acc_full(), i & 1))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const int v0 = (t_beg + i) * p.nv;
      for (int cb = 0; cb < p.nv; cb += 32) {
        float val[32];
        if (p.nv - cb >= 32) {
          uint32_t raw[32];
          ptx::tmem_ld32_sync(lane_addr + (uint32_t)cb, raw);
#pragma unroll
          for (int j = 0; j < 32; ++j) val[j] = __uint_as_float(raw[j]);
        } else {  // the last 16 columns (nv is a multiple of 16)
          uint32_t raw[16];
          ptx::tmem_ld16_sync(lane_addr + (uint32_t)cb, raw);
#pragma unroll
          for (int j = 0; j < 16; ++j) val[j] = __uint_as_float(raw[j]);
#pragma unroll
          for (int j = 16; j < 32; ++j) val[j] = -INFINITY;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {  // ascending index: strict > keeps the lowest
          const int v = v0 + cb + j;
          if (val[j] > best_v && v < p.V) {
            best_v = val[j];
            best_i = v;
          } else if (best_i == INT_MAX && v < p.V && j < p.nv - cb) {
            best_i = v;  // all values so far -inf or NaN: the lowest index stands in
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bars.acc_empty());
    }
    if (!ok) record_timeout(p.err, abort_flag);
    if (valid && best_i != INT_MAX) atomicMax(&p.slots[r], pack_key(best_v, best_i));
    __threadfence();
  }

  // ---- teardown and the last CTA's write-out
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    *last_flag = atomicAdd(p.ticket, 1u) == gridDim.x - 1u;
  }
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  for (int col = threadIdx.x; col < p.R; col += kThreads) {
    const unsigned long long k = atomicExch(&p.slots[col], 0ull);
    p.idx[col] = k ? key_index(k) : 0;
    if (p.maxval) p.maxval[col] = k ? key_value(k) : __int_as_float(0x7fc00000);
  }
  if (threadIdx.x == 0) *p.ticket = 0u;
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

// 2D bf16 map (inner extent d, outer extent rows, row pitch in bytes), box
// (64, box_rows), 128-byte swizzle; out-of-range rows read as zero.
bool encode_2d(CUtensorMap* m, const void* base, int64_t d, int64_t rows, int64_t pitch_bytes,
               int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
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

bool prepare() {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev >= 0 && dev < 64 && done[dev]) return true;
  if (cudaFuncSetAttribute(lm_head_argmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           227 * 1024) != cudaSuccess)
    return false;
  if (dev >= 0 && dev < 64) done[dev] = true;
  return true;
}

size_t round256(int64_t n) { return (size_t)((n + 255) / 256 * 256); }


// Vocabulary rows per tile (a multiple of 16 in [128, 256], the UMMA N
// range used): the one that minimises the rows of the busiest CTA, ties
// going to the larger tile (fewer MMAs).
int choose_nv(int vocab, int sms, int max_nv) {
  int best = max_nv;
  int64_t best_cost = INT64_MAX;
  for (int nv = max_nv; nv >= 128; nv -= 16) {
    const int tiles = ceil_div(vocab, nv);
    const int grid = tiles < sms ? tiles : sms;
    const int64_t cost = (int64_t)ceil_div(tiles, grid) * nv;
    if (cost < best_cost) {
      best_cost = cost;
      best = nv;
    }
  }
  return best;
}

// The launch's shape for rows x d x vocab on `sms` SMs (host only): tile rows,
// boxes per stage, the w ring, the h ring, the TMEM slice ring.  The h ring
// holds at least kHBoxesAhead boxes in at least two slots (each slot's
// refill is a round trip to L2, so fewer would pace the MMAs).  Boxes per
// stage: the most w bytes in flight (stages x boxes) with at least two
// stages beside the h ring, fewer boxes per stage only for more than 5% more
// bytes in flight (a stage is one handshake); four boxes use tiles of at
// most 176 rows so that two such stages fit.  One box per stage only where
// the K steps leave no choice: measured at 128 rows, one box per stage with
// 5 stages took 318 us against 234 us for two boxes with 2 stages.
void plan(LmParams& p, int rows, int d, int vocab, int sms) {
  p.R = rows;
  p.V = vocab;
  p.ksteps = d / kStepK;
  p.writers = ceil_div(rows, 32);
  p.hb = p.writers * 32 * 128;
  p.kb = 1;
  p.nv = choose_nv(vocab, sms, 256);
  p.stages = 0;
  int64_t best = 0;
  for (int cand = 4; cand >= 1; cand /= 2) {
    if (p.ksteps % cand || (cand == 1 && p.ksteps % 2 == 0)) continue;
    const int nv = choose_nv(vocab, sms, cand == 4 ? 176 : 256);
    const int hs = ceil_div(kHBoxesAhead, cand) > 2 ? ceil_div(kHBoxesAhead, cand) : 2;
    const int ring = kRingBudget - hs * cand * p.hb;
    int st = ring / (cand * nv * 128);
    st = st < kMaxStages ? st : kMaxStages;
    if (st < 2) continue;
    const int64_t bytes = (int64_t)st * cand * nv * 128;
    if (best == 0 || bytes * 20 > best * 21) {
      best = bytes;
      p.kb = cand;
      p.nv = nv;
      p.stages = st;
      p.hslots = hs;
    }
  }
  p.nvp = (p.nv + 31) / 32 * 32;
  p.tiles = ceil_div(vocab, p.nv);
  p.kst = p.ksteps / p.kb;
  p.w_bytes = p.kb * p.nv * 128;
  p.stage_bytes = p.w_bytes;
  p.h_bytes = p.kb * p.hb;
  // TMEM: the accumulator (nv columns, 32-aligned), then the ring of h slices
  // (32 columns per box)
  p.a_col = p.nvp;
  p.aslots = (kTmemCols - p.a_col) / (32 * p.kb) < kMaxASlots
                 ? (kTmemCols - p.a_col) / (32 * p.kb) : kMaxASlots;
}

}  // namespace
}  // namespace orthrus

using namespace orthrus;

extern "C" {

int orthrus_lm_head_argmax_plan(int32_t rows, int32_t d, int32_t vocab, int32_t sms,
                                int32_t* out) {
  if (!out || rows < 1 || rows > kRowsMax || d <= 0 || d % kStepK != 0 || vocab <= 0 ||
      vocab > (1 << 30) || sms <= 0)
    return ORTHRUS_EINVAL;
  LmParams p;
  plan(p, rows, d, vocab, sms);
  out[0] = p.nv;
  out[1] = p.kb;
  out[2] = p.stages;
  out[3] = p.aslots;
  out[4] = layout(p.stages, p.stage_bytes, p.h_bytes, p.hslots).total + 1024;
  out[5] = p.tiles < sms ? p.tiles : sms;
  out[6] = p.tiles;
  out[7] = kTmemCols;
  return ORTHRUS_OK;
}

size_t orthrus_lm_head_argmax_workspace(int32_t rows) {
  if (rows < 0) return 0;
  return round256((int64_t)rows * 8) + 256;
}

int orthrus_lm_head_argmax(int32_t dtype, const void* h, int32_t rows, int32_t d,
                           int64_t h_row_stride, const void* w, int32_t vocab, int32_t* idx,
                           float* maxval, int32_t* err, void* workspace, size_t workspace_bytes,
                           orthrus_stream_t stream) {
  if (dtype != ORTHRUS_F32 && dtype != ORTHRUS_BF16) return ORTHRUS_EINVAL;
  if (rows < 0 || d <= 0 || vocab <= 0 || h_row_stride < d) return ORTHRUS_EINVAL;
  if (dtype != ORTHRUS_BF16) return ORTHRUS_EUNSUPPORTED;
  if (rows == 0) return ORTHRUS_OK;
  if (rows > kRowsMax || d % kStepK != 0 || h_row_stride % 8 != 0 || vocab > (1 << 30))
    return ORTHRUS_EUNSUPPORTED;
  if (!h || !w || !idx) return ORTHRUS_EINVAL;
  if (reinterpret_cast<uintptr_t>(h) % 16 || reinterpret_cast<uintptr_t>(w) % 16)
    return ORTHRUS_EINVAL;
  if (!workspace || workspace_bytes < orthrus_lm_head_argmax_workspace(rows) ||
      reinterpret_cast<uintptr_t>(workspace) % 16)
    return ORTHRUS_EWORKSPACE;
  const int sms = sm_count();
  if (sms <= 0) return ORTHRUS_ECUDA;

  LmParams p;
  plan(p, rows, d, vocab, sms);
  char* ws = static_cast<char*>(workspace);
  p.slots = reinterpret_cast<unsigned long long*>(ws);
  p.ticket = reinterpret_cast<unsigned*>(ws + round256((int64_t)rows * 8));
  p.idx = idx;
  p.maxval = maxval;
  p.err = err;
  if (!encode_2d(&p.tm_w, w, d, vocab, (int64_t)d * 2, p.nv) ||
      !encode_2d(&p.tm_h, h, d, rows, h_row_stride * 2, 32 * p.writers))
    return ORTHRUS_ECUDA;
  const int smem = layout(p.stages, p.stage_bytes, p.h_bytes, p.hslots).total + 1024;
  if (!prepare()) return ORTHRUS_ECUDA;
  const int grid = p.tiles < sms ? p.tiles : sms;
  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lm_head_argmax_kernel, p) == cudaSuccess ? ORTHRUS_OK
                                                                           : ORTHRUS_ECUDA;
}

}  // extern "C"
