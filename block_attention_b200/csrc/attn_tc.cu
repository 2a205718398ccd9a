// attn_tc.cu -- bf16 block attention on the 5th-generation tensor cores.
//
// What it computes is the Orthrus round's attention (explainer on
// arXiv:2605.12825, §二: the block's queries attend to the frozen AR model's
// KV cache concatenated with the block's own K/V; §三: bidirectional inside
// the block for the diffusion view, causal for the AR verify view).
//
// Shape of the work.  Decoding reads every cached K/V row once per layer and
// view, so the path is bound by HBM bandwidth; the G = Hq/Hkv query heads
// that share a kv-head and the blk block rows form one M = G*blk <= 128 row
// tile, so each K/V tile fetched from HBM feeds a full 128-row tcgen05 MMA
// (128 FLOP per KV byte at the Qwen3-8B shape -- beyond CUDA cores, so the
// QK^T and PV products run on the tensor pipe).
//
// Two kernels per call, chained by programmatic dependent launch:
//
// attn_tc_partial, grid (S splits, Hkv, B), one CTA per SM.  The keys
// cache[0, n) of a (sequence, kv-head) are cut into 128-key tiles, followed by
// one tile holding the blk block rows; the tiles are dealt out contiguously
// over the S splits.  Per CTA:
//   warp 0      TMA producers: lane 0 streams K tiles, lane 1 V tiles, through
//               a 3-stage ring (32 KB of K + 32 KB of V per stage); a K slot
//               is refilled as soon as its S = Q K^T product has read it, a V
//               slot once its P V product has
//   warp 1      MMA issuer (one thread): S = Q K^T (M=128, N=128 per
//               instruction, Q read from TMEM) into a double-buffered TMEM
//               tile, and O += P V with P read from TMEM.  Once P(u) is ready
//               the 8 instructions of P(u) V(u) go out, then the 8 of S(u+2):
//               each product is a chain of dependent accumulations, and the
//               second chain overlaps the tail of the first in the tensor pipe
//   warps 2..5  softmax, one query row per thread: first they copy Q from
//               shared memory into TMEM; per tile, online softmax with lazy
//               rescaling (O in TMEM is rescaled only when a row's running
//               maximum grows by more than 2^8), P written to its own TMEM
//               buffer as bf16; finally the split's unnormalised O, row max
//               and row sum go to an L2-resident workspace.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O [256,256+D) Q (bf16 pairs,
// D/2 columns) and P (64 columns) after it.  Operands read from TMEM leave
// shared-memory bandwidth to the TMA stream: per tile the tensor pipe reads
// only the K and V tiles from shared memory.
// 128-key S tiles: a tcgen05.mma with N = 64 costs the issuing thread as much
// as one with N = 128, so the wider tile halves the MMA issue time per key.
//
// attn_tc_combine, grid (8-row groups, Hkv, B): merges the S partials of each
// query row (deterministic order) and writes bf16 output.  Its CTAs are small,
// so they start while the partial kernel drains, and the next kernel in the
// stream can take the SMs the partial kernel frees.  Partial O is stored as
// bf16 (one extra rounding, relative 2^-9), halving the epilogue's stores.
//
// With ORTHRUS_ATTN_EARLY_KV the partial kernel reads ctx_lens and starts
// streaming its first K/V tiles before waiting on the preceding kernel; Q and
// the block K/V are read only after that wait.
//
// Every mbarrier wait is bounded: on a timeout the kernel records
// ORTHRUS_ETIMEOUT in the error word, stops issuing work and drains what it
// issued, so it always terminates.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "attn_tc.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace orthrus {
namespace {

constexpr int kRows = 128;          // UMMA M
constexpr int kTile = 128;          // keys per tile (UMMA N of S = Q K^T)
constexpr int kStages = 3;          // K/V ring depth
// Cache tiles requested before the dependency wait under EARLY_KV.  They
// stream while the preceding kernel drains; requesting the whole ring makes
// the burst collide with that kernel's own memory traffic (measured on B200:
// 2 tiles ahead beat both 1 and 3 by 3% per call at the Qwen3-8B shape).
constexpr int kEarlyTiles = 2;
constexpr int kThreads = 192;       // 6 warps
constexpr int kTmemCols = 512;      // S0 [0,128) S1 [128,256) O [256,256+D) Q, P after it
constexpr int kOCol = 256;
static_assert(kOCol + 128 + 64 + kTile / 2 <= kTmemCols, "TMEM columns at D = 128");
constexpr float kLazyThresh = 8.f;  // log2 units
constexpr int kMaxSplits = 24;     // the combine keeps every split's loads in registers
constexpr int kGroupRows = 8;       // rows per combine CTA
constexpr int kCombineThreads = 256;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kHalfTile = kTile * 128;      // one 64-dim half of a K or V tile (16 KB)
constexpr int kQBytes = 2 * kRows * 128;    // two 64-dim halves, 128 B rows
constexpr int kStageBytes = 4 * kHalfTile;  // K (2 halves) + V (2 halves)
constexpr int kRingOff = kQBytes;
constexpr int kBarOff = kRingOff + kStages * kStageBytes;
constexpr int kNumBars = 9 + 4 * kStages;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack

// One split's partial, in 4-byte words: O as bf16 [16 row groups][D/4][8 rows]
// x 4 values (8 bytes each), then m[128], l[128] as fp32.
template <int kD>
__host__ __device__ constexpr int part_floats() { return kRows * kD / 2 + 2 * kRows; }
template <int kD>
__host__ __device__ constexpr int part_ml() { return kRows * kD / 2; }

struct __align__(64) TcParams {
  CUtensorMap tm_q;   // 3D (D, Hq, B*blk), box (64, G, blk)
  CUtensorMap tm_kc;  // 2D (D, B*Hkv*cap), box (64, 128)
  CUtensorMap tm_vc;
  CUtensorMap tm_kb;  // 3D (D, Hkv, B*blk), box (64, 1, blk)
  CUtensorMap tm_vb;
  const int32_t* ctx_lens;
  __nv_bfloat16* out;
  int32_t* err;
  float* part;  // [B][Hkv][S] partials
  int B, Hq, Hkv, blk, cap, max_ctx, mask_mode, G, S, early;
  float scale_log2;
};

// mbarrier addresses, laid out consecutively from `base` (8 bytes each)
struct Bars {
  uint32_t base;
  __device__ uint32_t at(int i) const { return base + 8 * i; }
  __device__ uint32_t q_full() const { return at(0); }   // Q landed in shared memory
  __device__ uint32_t q_tmem() const { return at(1); }   // Q copied into TMEM
  __device__ uint32_t k_full(int s) const { return at(2 + s); }
  __device__ uint32_t v_full(int s) const { return at(2 + kStages + s); }
  __device__ uint32_t k_empty(int s) const { return at(2 + 2 * kStages + s); }
  __device__ uint32_t v_empty(int s) const { return at(2 + 3 * kStages + s); }
  __device__ uint32_t s_full(int b) const { return at(2 + 4 * kStages + b); }
  __device__ uint32_t p_full(int b) const { return at(4 + 4 * kStages + b); }
  __device__ uint32_t pv_done(int b) const { return at(6 + 4 * kStages + b); }
  __device__ uint32_t mma_done() const { return at(8 + 4 * kStages); }
};

__device__ __forceinline__ void record_timeout(int32_t* err, volatile int* abort_flag) {
  *abort_flag = 1;
  set_err(err, ORTHRUS_ETIMEOUT);
}

template <int kD>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_partial(const __grid_constant__ TcParams p) {
  constexpr int halves = kD / 64;
  constexpr uint32_t kQCol = kOCol + kD;           // Q as bf16 pairs, D/2 columns
  constexpr uint32_t kPCol = kOCol + kD + kD / 2;  // P as bf16 pairs, 64 columns
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int S = p.S;
  const unsigned full_mask = 0xffffffffu;

  const Bars bars{sbase + kBarOff};
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff + 8);
  const int rows = p.G * p.blk;

  // ---- setup that reads nothing a preceding kernel writes
  if (threadIdx.x == 0) {
    *abort_flag = 0;
    ptx::mbar_init(bars.q_full(), 1);
    ptx::mbar_init(bars.q_tmem(), 128);
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bars.k_full(s), 1);
      ptx::mbar_init(bars.v_full(s), 1);
      ptx::mbar_init(bars.k_empty(s), 1);
      ptx::mbar_init(bars.v_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bars.s_full(s), 1);
      ptx::mbar_init(bars.p_full(s), 128);
      ptx::mbar_init(bars.pv_done(s), 1);
    }
    ptx::mbar_init(bars.mma_done(), 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::tma_prefetch_desc(&p.tm_q);
    ptx::tma_prefetch_desc(&p.tm_kc);
    ptx::tma_prefetch_desc(&p.tm_vc);
    ptx::tma_prefetch_desc(&p.tm_kb);
    ptx::tma_prefetch_desc(&p.tm_vb);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), kTmemCols);
    ptx::tmem_relinquish();
  }
  for (int e = threadIdx.x; e < (kRows - rows) * 8 * halves; e += kThreads) {
    const int h = e / ((kRows - rows) * 8), rem = e % ((kRows - rows) * 8);
    const int r = rows + rem / 8, c = rem % 8;
    *reinterpret_cast<uint4*>(smem + h * (kRows * 128) + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
  }
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  ptx::griddep_launch_dependents();

  const uint32_t q_s = sbase;
  auto k_s = [&](int stage) { return sbase + kRingOff + stage * kStageBytes; };
  auto v_s = [&](int stage) { return sbase + kRingOff + stage * kStageBytes + 2 * kHalfTile; };
  const int slab = (b * p.Hkv + g) * p.cap;
  // tiles of this split: cache tiles [0, Tc) then the block tile Tc
  auto geometry = [&](int n, int& Tc, int& t0, int& U) {
    const bool bad = n < 0 || n > p.max_ctx;
    Tc = bad ? 0 : ceil_div(n, kTile);
    const int T = bad ? 0 : Tc + 1;
    t0 = (int)(((int64_t)split * T) / S);
    U = (int)(((int64_t)(split + 1) * T) / S) - t0;
  };
  // K (is_v false) or V half of tile t into ring slot u % kStages
  auto issue = [&](bool is_v, int u, int t, int Tc) {
    const int st = u % kStages;
    const bool blk_tile = t == Tc;
    const int rows_ld = blk_tile ? p.blk : kTile;
    const uint32_t bar = is_v ? bars.v_full(st) : bars.k_full(st);
    const uint32_t dst = is_v ? v_s(st) : k_s(st);
    ptx::mbar_expect_tx(bar, (uint32_t)(halves * rows_ld * 128));
    for (int h = 0; h < halves; ++h) {
      if (blk_tile)
        ptx::tma_load_3d(dst + h * kHalfTile, is_v ? &p.tm_vb : &p.tm_kb, bar, 64 * h, g,
                         b * p.blk);
      else
        ptx::tma_load_2d(dst + h * kHalfTile, is_v ? &p.tm_vc : &p.tm_kc, bar, 64 * h,
                         slab + t * kTile);
    }
  };

  // Early cache streaming: the first kEarlyTiles cache tiles (never the
  // block tile, which the preceding kernel may still be writing).
  int early_issued = 0;
  int early_n = 0;
  if (warp == 0 && lane == 0) {
    for (int h = 0; h < halves; ++h) {
      ptx::tma_prefetch_l2_3d(&p.tm_q, 64 * h, g * p.G, b * p.blk);
      ptx::tma_prefetch_l2_3d(&p.tm_kb, 64 * h, g, b * p.blk);
      ptx::tma_prefetch_l2_3d(&p.tm_vb, 64 * h, g, b * p.blk);
    }
  }
  if (p.early && warp == 0 && lane == 0) {
    early_n = p.ctx_lens[b];
    int Tc, t0, U;
    geometry(early_n, Tc, t0, U);
    while (early_issued < min(U, kEarlyTiles) && t0 + early_issued < Tc) {
      issue(false, early_issued, t0 + early_issued, Tc);
      issue(true, early_issued, t0 + early_issued, Tc);
      ++early_issued;
    }
  }
  ptx::griddep_wait();
  if (warp == 0 && lane == 0) {
    // Q does not depend on the length: start it before reading ctx_lens
    ptx::mbar_expect_tx(bars.q_full(), (uint32_t)(halves * rows * 128));
    for (int h = 0; h < halves; ++h)
      ptx::tma_load_3d(q_s + h * (kRows * 128), &p.tm_q, bars.q_full(), 64 * h, g * p.G,
                       b * p.blk);
  }

  const int n = p.ctx_lens[b];
  const bool bad = n < 0 || n > p.max_ctx;
  if (bad && split == 0 && g == 0 && threadIdx.x == 0) set_err(p.err, ORTHRUS_ECAPACITY);
  int Tc, t0, U;
  geometry(n, Tc, t0, U);
  if (warp == 0 && lane == 0 && early_issued > 0 && early_n != n) {
    // the EARLY_KV contract was broken (the length changed under us): drain
    // the early loads and produce nothing for this split
    for (int u = 0; u < early_issued; ++u)
      if (!ptx::mbar_wait(bars.k_full(u % kStages), (u / kStages) & 1) ||
          !ptx::mbar_wait(bars.v_full(u % kStages), (u / kStages) & 1))
        record_timeout(p.err, abort_flag);
    set_err(p.err, ORTHRUS_EINVAL);
    *abort_flag = 1;
    early_issued = 0;
  }
  // lane 0 issued the early tiles: both producer lanes start after them
  if (warp == 0) early_issued = __shfl_sync(full_mask, early_issued, 0);
  __syncthreads();
  if (*abort_flag) U = 0;
  float* part = p.part + ((int64_t)(b * p.Hkv + g) * S + split) * part_floats<kD>();

  if (warp == 0) {
    // ================================================== TMA producers
    if (lane < 2 && U > 0) {
      const bool is_v = lane == 1;
      int issued = early_issued;
      for (int u = early_issued; u < U && !*abort_flag; ++u) {
        const int st = u % kStages;
        const uint32_t empty = is_v ? bars.v_empty(st) : bars.k_empty(st);
        if (!ptx::mbar_wait(empty, ((u / kStages) & 1) ^ 1)) {
          record_timeout(p.err, abort_flag);
          break;
        }
        issue(is_v, u, t0 + u, Tc);
        issued = u + 1;
      }
      // drain: every issued load must have landed before the CTA exits
      for (int u = max(0, issued - kStages); u < issued; ++u) {
        const uint32_t full = is_v ? bars.v_full(u % kStages) : bars.k_full(u % kStages);
        if (!ptx::mbar_wait(full, (u / kStages) & 1)) record_timeout(p.err, abort_flag);
      }
    }
    if (lane == 0 && !ptx::mbar_wait(bars.q_full(), 0)) record_timeout(p.err, abort_flag);
  } else if (warp == 1) {
    // ================================================== MMA issuer
    if (lane == 0 && U > 0) {
      const uint32_t id_s = ptx::idesc_bf16(kRows, kTile, false, false);
      const uint32_t id_pv = ptx::idesc_bf16(kRows, kD, false, true);
      // S(u) = Q K(u)^T into S buffer u & 1 (dims in 16-wide steps k), and
      // O += P(u) V(u) (keys in 16-wide steps k); S(u + 2) reuses the buffer
      // of S(u), which the softmax has read before it published P(u)
      auto s_step = [&](int u, int k) {
        const int st = u % kStages;
        const uint32_t h = k >> 2, kk = k & 3;  // 64-dim half, 16-dim step in it
        const uint64_t bd = ptx::sdesc_sw128(k_s(st) + h * kHalfTile + kk * 32, 16, 1024);
        ptx::mma_ts(tmem + (u & 1) * kTile, tmem + kQCol + k * 8, bd, id_s, k > 0 ? 1u : 0u);
      };
      auto pv_step = [&](int u, int k) {
        // V tile as the MN-major B operand: 8-key groups 1024 B apart,
        // 64-dim halves kHalfTile apart
        const uint64_t bd = ptx::sdesc_sw128(v_s(u % kStages) + k * 2048, kHalfTile, 1024);
        ptx::mma_ts(tmem + kOCol, tmem + kPCol + k * 8, bd, id_pv, (u > 0 || k > 0) ? 1u : 0u);
      };
      auto s_done = [&](int u) {
        ptx::tc_commit(bars.s_full(u & 1));
        ptx::tc_commit(bars.k_empty(u % kStages));
      };
      bool ok = ptx::mbar_wait(bars.q_tmem(), 0);
      // S(0) and S(1): two independent chains, back to back
      for (int u = 0; ok && u < min(U, 2); ++u) {
        if (!ptx::mbar_wait(bars.k_full(u % kStages), (u / kStages) & 1)) { ok = false; break; }
        ptx::tc_fence_after();
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) s_step(u, k);
        s_done(u);
      }
      for (int u = 0; ok && u < U && !*abort_flag; ++u) {
        const int st = u % kStages, nx = u + 2;
        const bool with_s = nx < U;
        if (!ptx::mbar_wait(bars.v_full(st), (u / kStages) & 1) ||
            !ptx::mbar_wait(bars.p_full(u & 1), (u >> 1) & 1) ||
            (with_s && !ptx::mbar_wait(bars.k_full(nx % kStages), (nx / kStages) & 1))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        // P(u) V(u) first and committed on its own: the softmax waits on it
        // before writing P(u + 1); S(u + 2) is needed only a tile later
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) pv_step(u, k);
        ptx::tc_commit(bars.pv_done(u & 1));
        ptx::tc_commit(bars.v_empty(st));
        if (with_s) {
#pragma unroll
          for (int k = 0; k < kD / 16; ++k) s_step(nx, k);
          s_done(nx);
        }
      }
      if (!ok) record_timeout(p.err, abort_flag);
      // every MMA issued so far has finished before TMEM is released
      ptx::tc_commit(bars.mma_done());
      if (!ptx::mbar_wait(bars.mma_done(), 0)) record_timeout(p.err, abort_flag);
    }
  } else {
    // ================================================== softmax
    const int quad = warp & 3;            // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;       // query row of this thread
    const int i_blk = r < rows ? r / p.G : p.blk;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int sm_tid = threadIdx.x - 64;  // 0..127
    const float c = p.scale_log2;         // > 0 (checked on the host)
    float m_ref = -INFINITY, l = 0.f;
    bool alive = U > 0;
    // Q row r -> TMEM columns [kQCol, kQCol + D/2) as bf16 pairs; in shared
    // memory the row's 16-byte chunks sit 128-byte swizzled (chunk j at j ^ (r & 7))
    if (alive) {
      if (!__all_sync(full_mask, ptx::mbar_wait(bars.q_full(), 0))) {
        record_timeout(p.err, abort_flag);
        alive = false;
      }
#pragma unroll
      for (int h = 0; h < halves; ++h) {
        uint32_t qv[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(smem + h * (kRows * 128) + r * 128 +
                                                           ((j ^ (r & 7)) << 4));
          qv[4 * j] = q4.x; qv[4 * j + 1] = q4.y; qv[4 * j + 2] = q4.z; qv[4 * j + 3] = q4.w;
        }
        ptx::tmem_st32(lane_addr + kQCol + h * 32, qv);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bars.q_tmem());
    }
    for (int u = 0; alive && u < U; ++u) {
      if (__any_sync(full_mask, *abort_flag != 0)) { alive = false; break; }
      const int t = t0 + u, buf = u & 1, st = u % kStages;
      if (!__all_sync(full_mask, ptx::mbar_wait(bars.s_full(buf), (u >> 1) & 1))) {
        record_timeout(p.err, abort_flag); alive = false; break;
      }
      ptx::tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) ptx::tmem_ld32(lane_addr + buf * kTile + cb * 32, sv[cb]);
      ptx::tmem_wait_ld();
      const bool blk_tile = t == Tc;
      const int nv_tile = blk_tile ? p.blk : min(kTile, n - t * kTile);
      int nv = nv_tile;
      if (blk_tile && p.mask_mode == ORTHRUS_CAUSAL_VERIFY) nv = min(i_blk + 1, p.blk);
      // masked keys -> -inf before the max and the exponent (exactly 0 in P)
      if (nv < kTile) {
#pragma unroll
        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (cb * 32 + j >= nv) sv[cb][j] = __float_as_uint(-INFINITY);
      }
      float mt[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int cb = 0; cb < 4; ++cb)
#pragma unroll
        for (int j = 0; j < 32; ++j) mt[cb] = fmaxf(mt[cb], __uint_as_float(sv[cb][j]));
      const float ms = fmaxf(fmaxf(mt[0], mt[1]), fmaxf(mt[2], mt[3])) * c;
      const bool need = ms > m_ref + kLazyThresh;
      const bool rescale = __any_sync(full_mask, need);
      float f = 1.f;
      if (rescale) {
        const float m_new = need ? ms : m_ref;
        f = ptx::ex2(m_ref - m_new);  // 0 for the first tile, 1 if unchanged
        m_ref = m_new;
      }
      // P = 2^(s*c - m_ref) as bf16 pairs; ex2(-inf) = 0 for masked keys
      const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[2][32];
#pragma unroll
      for (int half = 0; half < 2; ++half)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float p0 = ptx::ex2(fmaf(__uint_as_float(sv[2 * half][2 * j]), c, nm));
          const float p1 = ptx::ex2(fmaf(__uint_as_float(sv[2 * half][2 * j + 1]), c, nm));
          const float p2 = ptx::ex2(fmaf(__uint_as_float(sv[2 * half + 1][2 * j]), c, nm));
          const float p3 = ptx::ex2(fmaf(__uint_as_float(sv[2 * half + 1][2 * j + 1]), c, nm));
          ls[0] += p0; ls[1] += p1; ls[2] += p2; ls[3] += p3;
          pk[half][j] = ptx::pack_bf16x2(p0, p1);
          pk[half][16 + j] = ptx::pack_bf16x2(p2, p3);
        }
      l = l * f + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
      // P(u - 1) V(u - 1) must be done: it reads the P buffer and adds into O
      if (u > 0) {
        if (!__all_sync(full_mask, ptx::mbar_wait(bars.pv_done((u - 1) & 1), ((u - 1) >> 1) & 1))) {
          record_timeout(p.err, abort_flag); alive = false; break;
        }
        ptx::tc_fence_after();
        if (rescale) {
#pragma unroll
          for (int cb = 0; cb < kD / 32; ++cb) {
            uint32_t o[32];
            ptx::tmem_ld32_sync(lane_addr + kOCol + cb * 32, o);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
            ptx::tmem_st32(lane_addr + kOCol + cb * 32, o);
          }
        }
      }
      ptx::tmem_st32(lane_addr + kPCol, pk[0]);
      ptx::tmem_st32(lane_addr + kPCol + 32, pk[1]);
      ptx::tmem_wait_st();
      if (nv_tile < kTile) {
        // rows past the valid keys hold stale or foreign data: zero them in V
        // so 0 * garbage cannot reach O
        if (!__all_sync(full_mask, ptx::mbar_wait(bars.v_full(st), (u / kStages) & 1))) {
          record_timeout(p.err, abort_flag); alive = false; break;
        }
        const int nz = (kTile - nv_tile) * 8 * halves;  // 16-byte chunks
        for (int e = sm_tid; e < nz; e += 128) {
          const int h = e / ((kTile - nv_tile) * 8), rem = e % ((kTile - nv_tile) * 8);
          const int row = nv_tile + rem / 8, cc = rem % 8;
          *reinterpret_cast<uint4*>(smem + kRingOff + st * kStageBytes + 2 * kHalfTile +
                                    h * kHalfTile + row * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(bars.p_full(buf));
    }
    // ---- this split's unnormalised O, row max and row sum -> workspace
    bool have = alive && U > 0 && !__any_sync(full_mask, *abort_flag != 0);
    if (have && !__all_sync(full_mask, ptx::mbar_wait(bars.pv_done((U - 1) & 1), ((U - 1) >> 1) & 1))) {
      record_timeout(p.err, abort_flag);
      have = false;
    }
    if (have) ptx::tc_fence_after();
    const int rg = r / kGroupRows, ri = r % kGroupRows;
    uint2* po = reinterpret_cast<uint2*>(part) + (int64_t)rg * (kD / 4) * kGroupRows + ri;
#pragma unroll
    for (int cb = 0; cb < kD / 32; ++cb) {
      uint32_t o[32];
      if (have) ptx::tmem_ld32_sync(lane_addr + kOCol + cb * 32, o);
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        uint2 v = make_uint2(0u, 0u);
        if (have) {
          v.x = ptx::pack_bf16x2(__uint_as_float(o[j]), __uint_as_float(o[j + 1]));
          v.y = ptx::pack_bf16x2(__uint_as_float(o[j + 2]), __uint_as_float(o[j + 3]));
        }
        __stcg(po + (cb * 8 + j / 4) * kGroupRows, v);
      }
    }
    __stcg(part + part_ml<kD>() + r, have ? m_ref : -INFINITY);
    __stcg(part + part_ml<kD>() + kRows + r, have ? l : 0.f);
  }
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the S split partials of one 8-row group and write bf16.  One thread
// per output item (4 dims of one row); consecutive lanes take consecutive
// rows, so each split's slice is read as contiguous 256-byte runs, and every
// split's loads are issued before any is used (one L2 round trip).  Splits
// are merged in index order, so the result does not depend on timing.
template <int kD>
__global__ void __launch_bounds__(kCombineThreads, 2)
attn_tc_combine(const __grid_constant__ TcParams p) {
  constexpr int kItemsPerRow = kD / 4;
  const int rg = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int it = threadIdx.x;
  const int d4 = it / kGroupRows, ri = it % kGroupRows;
  const int r = rg * kGroupRows + ri;
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int n = p.ctx_lens[b];
  if (n < 0 || n > p.max_ctx) return;  // reported by the partial kernel
  if (d4 >= kItemsPerRow || r >= p.G * p.blk) return;
  const int S = p.S;
  const float* base = p.part + (int64_t)(b * p.Hkv + g) * S * part_floats<kD>();
  const int64_t o_off = ((int64_t)rg * kItemsPerRow + d4) * kGroupRows + ri;  // uint2 index
  float ms[kMaxSplits], ls[kMaxSplits];
  uint2 os[kMaxSplits];
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    if (s < S) {
      const float* ps = base + (int64_t)s * part_floats<kD>();
      ms[s] = __ldcg(ps + part_ml<kD>() + r);
      ls[s] = __ldcg(ps + part_ml<kD>() + kRows + r);
      os[s] = __ldcg(reinterpret_cast<const uint2*>(ps) + o_off);
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s)
    if (s < S) M = fmaxf(M, ms[s]);
  float L = 0.f, O0 = 0.f, O1 = 0.f, O2 = 0.f, O3 = 0.f;
#pragma unroll
  for (int s = 0; s < kMaxSplits; ++s) {
    if (s < S) {
      const float w = M == -INFINITY ? 0.f : ptx::ex2(ms[s] - M);
      L = fmaf(w, ls[s], L);
      O0 = fmaf(w, __uint_as_float(os[s].x << 16), O0);
      O1 = fmaf(w, __uint_as_float(os[s].x & 0xffff0000u), O1);
      O2 = fmaf(w, __uint_as_float(os[s].y << 16), O2);
      O3 = fmaf(w, __uint_as_float(os[s].y & 0xffff0000u), O3);
    }
  }
  const float inv = 1.f / L;
  const int i = r / p.G, h = g * p.G + r % p.G;
  uint2 pkd;
  pkd.x = ptx::pack_bf16x2(O0 * inv, O1 * inv);
  pkd.y = ptx::pack_bf16x2(O2 * inv, O3 * inv);
  *reinterpret_cast<uint2*>(p.out + ((int64_t)(b * p.blk + i) * p.Hq + h) * kD + 4 * d4) = pkd;
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

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
            const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
            strides_bytes, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int kD>
bool prepare(int device) {
  static bool done[64] = {false};
  if (device >= 0 && device < 64 && done[device]) return true;
  if (cudaFuncSetAttribute(attn_tc_partial<kD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes) != cudaSuccess)
    return false;
  if (device >= 0 && device < 64) done[device] = true;
  return true;
}

// Splits per (sequence, kv-head): enough to fill one wave of CTAs (one per
// SM) when the batch is small, and at least enough that no split of the
// longest possible sequence exceeds 64 tiles, so long or ragged batches spread
// over several waves instead of leaving their longest sequences to a few CTAs;
// never more splits than the longest sequence has tiles.
int choose_splits(const orthrus_attn_args& a) {
  const int heads = a.B * a.Hkv;
  const int tiles = ceil_div(a.max_ctx, kTile) + 1;
  int S = heads >= 148 ? 1 : 148 / heads;
  S = max(S, ceil_div(tiles, 64));
  S = min(S, tiles);
  return max(1, min(S, kMaxSplits));
}

}  // namespace

bool tc_supported(const orthrus_attn_args& a) {
  return a.dtype == ORTHRUS_BF16 && (a.D == 64 || a.D == 128) &&
         (a.Hq / a.Hkv) * a.blk <= kRows && a.blk <= 32 && a.Hq / a.Hkv <= 256 &&
         a.B <= 65535 && a.Hkv <= 65535;
}

size_t tc_workspace_bytes(const orthrus_attn_args& a) {
  const int64_t per = a.D == 64 ? part_floats<64>() : part_floats<128>();
  return (size_t)((int64_t)a.B * a.Hkv * choose_splits(a) * per * 4);
}

int tc_launches(const orthrus_attn_args&) { return 2; }

int tc_launch(const orthrus_attn_args& a, cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ORTHRUS_ECUDA;
  if (!(a.D == 64 ? prepare<64>(dev) : prepare<128>(dev))) return ORTHRUS_ECUDA;
  const int S = choose_splits(a);
  TcParams p;
  const int G = a.Hq / a.Hkv;
  const cuuint64_t es = 2;
  {
    cuuint64_t dims[3] = {(cuuint64_t)a.D, (cuuint64_t)a.Hq, (cuuint64_t)a.B * a.blk};
    cuuint64_t str[2] = {a.D * es, (cuuint64_t)a.Hq * a.D * es};
    cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)a.blk};
    if (!encode(&p.tm_q, a.q, 3, dims, str, box)) return ORTHRUS_ECUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.D, (cuuint64_t)a.B * a.Hkv * a.cap};
    cuuint64_t str[1] = {a.D * es};
    cuuint32_t box[2] = {64, (cuuint32_t)kTile};
    if (!encode(&p.tm_kc, a.k_cache, 2, dims, str, box)) return ORTHRUS_ECUDA;
    if (!encode(&p.tm_vc, a.v_cache, 2, dims, str, box)) return ORTHRUS_ECUDA;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)a.D, (cuuint64_t)a.Hkv, (cuuint64_t)a.B * a.blk};
    cuuint64_t str[2] = {a.D * es, (cuuint64_t)a.Hkv * a.D * es};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)a.blk};
    if (!encode(&p.tm_kb, a.k_blk, 3, dims, str, box)) return ORTHRUS_ECUDA;
    if (!encode(&p.tm_vb, a.v_blk, 3, dims, str, box)) return ORTHRUS_ECUDA;
  }
  p.ctx_lens = a.ctx_lens;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.err = a.err;
  p.part = static_cast<float*>(a.workspace);
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.blk = a.blk; p.cap = a.cap;
  p.max_ctx = a.max_ctx; p.mask_mode = a.mask_mode; p.G = G; p.S = S;
  p.early = (a.flags & ORTHRUS_ATTN_EARLY_KV) ? 1 : 0;
  p.scale_log2 = (float)((double)a.scale * 1.4426950408889634);

  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, a.Hkv, a.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  cudaError_t e = a.D == 64 ? cudaLaunchKernelEx(&cfg, attn_tc_partial<64>, p)
                            : cudaLaunchKernelEx(&cfg, attn_tc_partial<128>, p);
  if (e != cudaSuccess) return ORTHRUS_ECUDA;
  cfg.gridDim = dim3(ceil_div(G * a.blk, kGroupRows), a.Hkv, a.B);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = 0;
  e = a.D == 64 ? cudaLaunchKernelEx(&cfg, attn_tc_combine<64>, p)
                : cudaLaunchKernelEx(&cfg, attn_tc_combine<128>, p);
  return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA;
}

}  // namespace orthrus
