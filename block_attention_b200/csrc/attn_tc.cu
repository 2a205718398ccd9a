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
// attn_tc_kernel, grid (Hkv, B, S splits), one CTA per SM.  The keys
// cache[0, n) of a (sequence, kv-head) are cut into 128-key tiles, followed by
// one tile holding the blk block rows; the T tiles are dealt out contiguously
// over the S splits, the first T mod S splits taking one tile more.  The
// splits vary slowest in the grid, so the CTAs launched last -- on the SMs the
// preceding kernel frees last -- are the high splits, the ones with fewer
// tiles.  Per CTA (10 warps):
//   warp 0      TMA producers: lane 0 streams K tiles, lane 1 V tiles, through
//               a 2-stage ring (32 KB of K + 32 KB of V per stage); a K slot
//               is refilled as soon as its S = Q K^T product has read it, a V
//               slot once its P V product has
//   warp 1      MMA issuer (one thread): S(u) = Q K(u)^T (M=128, N=128 per
//               instruction, Q and K from shared memory) into TMEM buffer
//               u & 1; S(u + 2) goes out as soon as softmax(u) has read S(u),
//               ahead of O_(u & 1) += P(u) V(u) (P(u) from shared memory)
//   warps 2..9  softmax, two warpgroups taking turns: warps 2-5 the even
//               tiles, warps 6-9 the odd ones, one query row per thread, so
//               that one warpgroup's exponentials overlap the other's.  Each
//               keeps its own running max and sum and its own O accumulator
//               with lazy rescaling (O is rescaled only when a row's running
//               maximum grows by more than 2^8).  S is read from TMEM 64
//               columns at a time (three loads per tile: both halves for the
//               maximum, the second kept into the exponentials); P goes to the
//               warpgroup's shared-memory buffer as bf16, in the MMA's K-major
//               128-byte-swizzled layout.  At the end the two swap (max, sum)
//               and each writes half of the combined unnormalised O, with the
//               row max and sum, to the workspace.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O_0 [256,256+D) O_1 [256+D,
// 256+2D).
// 128-key S tiles: a tcgen05.mma with N = 64 costs the issuing thread as much
// as one with N = 128, so the wider tile halves the MMA issue time per key.
//
// Split merge.  Each split writes its unnormalised O (bf16), row max and row
// sum (fp32) to an L2-resident workspace, grouped by the query rows one
// merging CTA owns, so that the owner fetches a split's share with one bulk
// copy.  When the grid fits one wave (every CTA resident at once, the batch-1
// decoding case) the merge runs inside the same launch: a barrier per
// (sequence, kv-head) on one (generation, count) word -- each CTA adds its
// arrival without waiting for the atomic, the merging CTAs wait (bounded)
// for the count of their generation to reach S, and split 0 then starts the
// next generation -- then every merging CTA stages its row group of all S
// partials by bulk copies and merges them in split order (the result does
// not depend on timing) into bf16 output.
// Larger grids, whose CTAs cannot all be resident, end instead and a second
// kernel (attn_tc_combine, PDL-chained) merges the same way.  In such a grid
// over 2..32 sequences the CTAs take their (sequence, split, kv-head) in
// order of decreasing context length rather than by grid position: the
// hardware starts CTAs in launch order as SMs come free, so the longest
// splits start first and the short ones fill the tail (longest processing
// time first list scheduling).
//
// With ORTHRUS_ATTN_EARLY_KV the kernel reads ctx_lens and starts
// streaming its first K/V tiles before waiting on the preceding kernel; Q and
// the block K/V are read only after that wait.
//
// Every mbarrier wait is bounded: on a timeout the kernel records
// ORTHRUS_ETIMEOUT in the error word, stops issuing work and drains what it
// issued; the merge's wait for the other splits is bounded too, so the kernel
// always terminates.
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
constexpr int kStages = 2;          // K/V ring depth
// Cache tiles requested before the dependency wait under EARLY_KV.  They
// stream while the preceding kernel drains; requesting the whole ring makes
// the burst collide with that kernel's own memory traffic (measured on B200:
// 2 tiles ahead beat both 1 and 3 by 3% per call at the Qwen3-8B shape).
constexpr int kEarlyTiles = 2;
constexpr int kThreads = 320;       // 10 warps: producers, MMA issuer, two softmax warpgroups
constexpr int kTmemCols = 512;      // S0 [0,128) S1 [128,256) O_0 [256,256+D) O_1 after it
constexpr int kOCol = 256;
static_assert(kOCol + 2 * 128 <= kTmemCols, "TMEM columns at D = 128");
constexpr float kLazyThresh = 8.f;  // log2 units
constexpr int kMaxSplits = 24;      // bounds the partials (kPartRows) and the merge's staging
constexpr int kCounterBytes = 2048;  // workspace head: merge counters, never partials
constexpr int kMaxFusedHeads = kCounterBytes / 8;  // one 64-bit (generation, count) word each
constexpr int kGroupRows = 8;        // rows per CTA of the separate combine kernel
constexpr int kCombineThreads = 256;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kHalfTile = kTile * 128;      // one 64-dim half of a K or V tile (16 KB)
constexpr int kQBytes = 2 * kRows * 128;    // two 64-dim halves, 128 B rows
constexpr int kStageBytes = 4 * kHalfTile;  // K (2 halves) + V (2 halves)
constexpr int kRingOff = kQBytes;
constexpr int kPBytes = 2 * kRows * 128;    // P of one tile: two 64-key halves, 128 B rows
constexpr int kPOff = kRingOff + kStages * kStageBytes;  // one P buffer per softmax warpgroup
constexpr int kBarOff = kPOff + 2 * kPBytes;
constexpr int kNumBars = 11 + 4 * kStages;
constexpr int kMiscOff = kBarOff + kNumBars * 8;
constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + alignment slack

// One split's partial in the workspace: its query rows in groups of R (the
// rows one merging CTA owns), each group one contiguous block of D/8 + 1
// 16-byte columns x R rows -- O as bf16, 8 dims per 16-byte chunk, then
// (max, sum, 0, 0) in fp32 -- so a merging CTA fetches its rows of a split
// with one bulk copy.  Groups cover at most kRows + kMaxSplits rows
// (R = ceil(rows / S) rounds up).  bf16 halves the partials' round trip
// through L2 at one more rounding of O (relative 2^-9).
constexpr int kPartRows = kRows + kMaxSplits;
template <int kD>
__host__ __device__ constexpr int part_floats() { return kPartRows * (kD / 2 + 4); }
template <int kD>
__host__ __device__ constexpr int group_f4(int R) { return (kD / 8 + 1) * R; }  // 16-byte units
// the in-launch merge stages every split's group of its rows in the idle ring
static_assert(kPartRows * (128 / 8 + 1) * 16 <= kStages * kStageBytes,
              "merge staging fits the ring");

struct __align__(64) TcParams {
  CUtensorMap tm_q;   // 3D (D, Hq, B*blk), box (64, G, blk)
  CUtensorMap tm_kc;  // 2D (D, B*Hkv*cap), box (64, 128)
  CUtensorMap tm_vc;
  CUtensorMap tm_kb;  // 3D (D, Hkv, B*blk), box (64, 1, blk)
  CUtensorMap tm_vb;
  const int32_t* ctx_lens;
  __nv_bfloat16* out;
  int32_t* err;
  const __nv_bfloat16* next_k;  // caches of the next call, warmed into L2 (nullable)
  const __nv_bfloat16* next_v;
  float* part;         // [B][Hkv] x S split partials (workspace after the counters)
  int R;               // query rows per partial group = rows one merging CTA owns
  int order;           // launch order sorted by context length (B in [2, 32], unfused)
  unsigned long long* counters;  // [B * Hkv] in-kernel merge: generation << 32 | arrivals
  int B, Hq, Hkv, blk, cap, max_ctx, mask_mode, G, S, early;
  float scale_log2;
};

// mbarrier addresses, laid out consecutively from `base` (8 bytes each)
struct Bars {
  uint32_t base;
  __device__ uint32_t at(int i) const { return base + 8 * i; }
  __device__ uint32_t q_full() const { return at(0); }   // Q landed in shared memory
  __device__ uint32_t k_full(int s) const { return at(1 + s); }
  __device__ uint32_t v_full(int s) const { return at(1 + kStages + s); }
  __device__ uint32_t k_empty(int s) const { return at(1 + 2 * kStages + s); }
  __device__ uint32_t v_empty(int s) const { return at(1 + 3 * kStages + s); }
  __device__ uint32_t s_full(int b) const { return at(1 + 4 * kStages + b); }  // S in buffer b
  __device__ uint32_t s_free(int b) const { return at(3 + 4 * kStages + b); }  // S(b) read
  __device__ uint32_t p_full(int b) const { return at(5 + 4 * kStages + b); }  // P buffer b
  __device__ uint32_t pv_done(int b) const { return at(7 + 4 * kStages + b); } // P(b) V done
  __device__ uint32_t mma_done() const { return at(9 + 4 * kStages); }
  __device__ uint32_t merge_full() const { return at(10 + 4 * kStages); }  // rows staged
};

__device__ __forceinline__ void record_timeout(int32_t* err, volatile int* abort_flag) {
  *abort_flag = 1;
  set_err(err, ORTHRUS_ETIMEOUT);
}

// 64 S values of keys [k0, k0 + 64) of a tile: those at or past nv -> -inf
__device__ __forceinline__ void mask_keys(uint32_t (&sv)[2][32], int k0, int nv) {
#pragma unroll
  for (int cb = 0; cb < 2; ++cb)
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (k0 + 32 * cb + j >= nv) sv[cb][j] = __float_as_uint(-INFINITY);
}

template <int kD>
__device__ __forceinline__ void merge_rows(const TcParams& p, int b, int g, int q, int tid,
                                           int nthreads, uint8_t* stage, uint32_t bar);

template <int kD, bool kFused>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ TcParams p) {
  constexpr int halves = kD / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int g = blockIdx.x, b = blockIdx.y, split = blockIdx.z;
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
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bars.k_full(s), 1);
      ptx::mbar_init(bars.v_full(s), 1);
      ptx::mbar_init(bars.k_empty(s), 1);
      ptx::mbar_init(bars.v_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(bars.s_full(s), 1);
      ptx::mbar_init(bars.s_free(s), 128);  // one softmax warpgroup
      ptx::mbar_init(bars.p_full(s), 128);
      ptx::mbar_init(bars.pv_done(s), 1);
    }
    ptx::mbar_init(bars.mma_done(), 1);
    ptx::mbar_init(bars.merge_full(), 1);
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

  // Longest sequences first, for grids of more than one wave: CTAs start in
  // launch order, so launch position `lin` takes entry `lin` of the list of
  // (sequence, split, kv-head) sorted by decreasing context length (kv-head
  // fastest, ties by sequence index).  The long splits start first and the
  // short ones fill the tail.  Warp 0 keeps the lengths it ranked (`seen`):
  // under ORTHRUS_ATTN_EARLY_KV they were read before the dependency wait,
  // and a change under the kernel is caught after it.
  int seen = 0;
  if (!kFused && p.order) {
    if (!p.early) ptx::griddep_wait();  // the lengths may come from the preceding kernel
    int* map = reinterpret_cast<int*>(smem + kPOff);  // P is written only after the MMAs
    if (warp == 0) {
      seen = lane < p.B ? p.ctx_lens[lane] : 0;
      const int key = lane >= p.B ? -2 : (seen < 0 || seen > p.max_ctx ? -1 : seen);
      int rank = 0;
      for (int i = 0; i < p.B; ++i) {
        const int ki = __shfl_sync(full_mask, key, i);
        rank += (ki > key || (ki == key && i < lane)) ? 1 : 0;
      }
      const int lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
      const unsigned hit = __ballot_sync(full_mask, lane < p.B && rank == lin / (p.Hkv * S));
      if (lane == 0) {
        map[0] = __ffs(hit) - 1;
        map[1] = (lin / p.Hkv) % S;
        map[2] = lin % p.Hkv;
      }
    }
    __syncthreads();
    b = map[0];
    split = map[1];
    g = map[2];
    __syncthreads();
  }

  const uint32_t q_s = sbase;
  auto k_s = [&](int stage) { return sbase + kRingOff + stage * kStageBytes; };
  auto v_s = [&](int stage) { return sbase + kRingOff + stage * kStageBytes + 2 * kHalfTile; };
  auto p_s = [&](int x) { return sbase + kPOff + x * kPBytes; };
  const int slab = (b * p.Hkv + g) * p.cap;
  // tiles of this split: cache tiles [0, Tc) then the block tile Tc
  auto geometry = [&](int n, int& Tc, int& t0, int& U) {
    const bool bad = n < 0 || n > p.max_ctx;
    Tc = bad ? 0 : ceil_div(n, kTile);
    const int T = bad ? 0 : Tc + 1;
    const int base = T / S, extra = T % S;  // the first `extra` splits take base + 1
    t0 = split * base + min(split, extra);
    U = base + (split < extra ? 1 : 0);
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
  // the merge barrier's generation, read off the critical path: it cannot
  // change before this CTA has arrived, and the previous call has completed
  unsigned gen0 = 0;
  if (kFused && threadIdx.x == 0)
    gen0 = (unsigned)(ptx::ld_acquire_gpu_u64(p.counters + (b * p.Hkv + g)) >> 32);
  if (bad && split == 0 && g == 0 && threadIdx.x == 0) set_err(p.err, ORTHRUS_ECAPACITY);
  int Tc, t0, U;
  geometry(n, Tc, t0, U);
  // with the sorted launch order, any length read early must hold
  const bool moved = !kFused && p.order && p.early && warp == 0 &&
                     __any_sync(full_mask, lane < p.B && p.ctx_lens[lane] != seen);
  if (warp == 0 && lane == 0 && ((early_issued > 0 && early_n != n) || moved)) {
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
      // with every load of this call's tiles issued, warm L2 with the same
      // tiles of the next call's cache (a hint: no data reaches this CTA)
      const __nv_bfloat16* nxt = is_v ? p.next_v : p.next_k;
      if (nxt && !*abort_flag) {
        const __nv_bfloat16* nb = nxt + (int64_t)slab * kD;
        for (int u = 0; u < U && t0 + u < Tc; ++u) {
          const int t = t0 + u;
          const int nrows = min(kTile, n - t * kTile);
          ptx::bulk_prefetch_l2(nb + (int64_t)t * kTile * kD, (uint32_t)(nrows * kD * 2));
        }
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
      // S(u) = Q K(u)^T into TMEM buffer u & 1, Q and K from shared memory
      // (dims in 16-wide steps k); O_(u & 1) += P(u) V(u) with P(u) from its
      // warpgroup's shared-memory buffer (keys in 16-wide steps k).  S(u + 2)
      // needs only that softmax(u) has read S(u), so it is issued ahead of
      // P(u) V(u) and computes while softmax(u) takes its exponentials.
      auto s_tile = [&](int u) {
        const int st = u % kStages;
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {
          const uint32_t h = k >> 2, kk = k & 3;  // 64-dim half, 16-dim step in it
          const uint64_t ad = ptx::sdesc_sw128(q_s + h * (kRows * 128) + kk * 32, 16, 1024);
          const uint64_t bd = ptx::sdesc_sw128(k_s(st) + h * kHalfTile + kk * 32, 16, 1024);
          ptx::mma_ss(tmem + (u & 1) * kTile, ad, bd, id_s, k > 0 ? 1u : 0u);
        }
        ptx::tc_commit(bars.s_full(u & 1));
        ptx::tc_commit(bars.k_empty(st));
      };
      auto pv_tile = [&](int u) {
        const int st = u % kStages;
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          const uint32_t h = k >> 2, kk = k & 3;  // 64-key half of P, 16-key step in it
          const uint64_t ad =
              ptx::sdesc_sw128(p_s(u & 1) + h * (kRows * 128) + kk * 32, 16, 1024);
          // V tile as the MN-major B operand: 8-key groups 1024 B apart,
          // 64-dim halves kHalfTile apart
          const uint64_t bd = ptx::sdesc_sw128(v_s(st) + k * 2048, kHalfTile, 1024);
          ptx::mma_ss(tmem + kOCol + (u & 1) * kD, ad, bd, id_pv, (u > 1 || k > 0) ? 1u : 0u);
        }
        ptx::tc_commit(bars.pv_done(u & 1));
        ptx::tc_commit(bars.v_empty(st));
      };
      bool ok = ptx::mbar_wait(bars.q_full(), 0);
      // S(0) and S(1): one for each softmax warpgroup
      for (int u = 0; ok && u < min(U, 2); ++u) {
        if (!ptx::mbar_wait(bars.k_full(u % kStages), (u / kStages) & 1)) { ok = false; break; }
        ptx::tc_fence_after();
        s_tile(u);
      }
      for (int u = 0; ok && u < U && !*abort_flag; ++u) {
        const int nx = u + 2;
        if (nx < U) {
          if (!ptx::mbar_wait(bars.s_free(u & 1), (u >> 1) & 1) ||
              !ptx::mbar_wait(bars.k_full(nx % kStages), (nx / kStages) & 1)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          s_tile(nx);
        }
        if (!ptx::mbar_wait(bars.p_full(u & 1), (u >> 1) & 1) ||
            !ptx::mbar_wait(bars.v_full(u % kStages), (u / kStages) & 1)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        pv_tile(u);
      }
      if (!ok) record_timeout(p.err, abort_flag);
      // every MMA issued so far has finished before O is read and TMEM freed
      ptx::tc_commit(bars.mma_done());
      if (!ptx::mbar_wait(bars.mma_done(), 0)) record_timeout(p.err, abort_flag);
    }
  } else {
    // ================================================== softmax
    // Two warpgroups take turns: X = 0 (warps 2-5) the even tiles, X = 1
    // (warps 6-9) the odd ones, each with its own running max and sum and
    // its own O accumulator, so one warpgroup's exponentials overlap the
    // other's.  Every thread owns one query row of its warpgroup's tiles.
    const int X = (warp - 2) >> 2;
    const int quad = warp & 3;            // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;       // query row of this thread
    const int i_blk = r < rows ? r / p.G : p.blk;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int wg_tid = threadIdx.x - 64 - 128 * X;  // 0..127 within the warpgroup
    const float c = p.scale_log2;         // > 0 (checked on the host)
    float m_ref = -INFINITY, l = 0.f;
    bool alive = U > 0;
    for (int u = X; alive && u < U; u += 2) {
      if (__any_sync(full_mask, *abort_flag != 0)) { alive = false; break; }
      const int t = t0 + u, st = u % kStages;
      if (!__all_sync(full_mask, ptx::mbar_wait(bars.s_full(X), (u >> 1) & 1))) {
        record_timeout(p.err, abort_flag); alive = false; break;
      }
      ptx::tc_fence_after();
      const bool blk_tile = t == Tc;
      const int nv_tile = blk_tile ? p.blk : min(kTile, n - t * kTile);
      int nv = nv_tile;
      if (blk_tile && p.mask_mode == ORTHRUS_CAUSAL_VERIFY) nv = min(i_blk + 1, p.blk);
      const uint32_t s_addr = lane_addr + X * kTile;
      // S(u) is read from TMEM 64 columns at a time, so that no more than 64
      // of its values are live in registers: both halves for the row
      // maximum, then the exponentials of the second half, still in
      // registers, and of the first half, read again (three loads, not
      // four); masked keys -> -inf (exactly 0 in P)
      float mt[2] = {-INFINITY, -INFINITY};
      uint32_t sv[2][32];  // after the maximum: the second half, masked
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        ptx::tmem_ld32(s_addr + 64 * half, sv[0]);
        ptx::tmem_ld32(s_addr + 64 * half + 32, sv[1]);
        ptx::tmem_wait_ld();
        if (nv < kTile) mask_keys(sv, 64 * half, nv);
#pragma unroll
        for (int cb = 0; cb < 2; ++cb)
#pragma unroll
          for (int j = 0; j < 32; ++j) mt[cb] = fmaxf(mt[cb], __uint_as_float(sv[cb][j]));
      }
      const float ms = fmaxf(mt[0], mt[1]) * c;
      const bool need = ms > m_ref + kLazyThresh;
      const bool rescale = __any_sync(full_mask, need);
      float f = 1.f;
      if (rescale) {
        const float m_new = need ? ms : m_ref;
        f = ptx::ex2(m_ref - m_new);  // 0 for the first tile, 1 if unchanged
        m_ref = m_new;
      }
      // P(u - 2) V(u - 2), this warpgroup's previous tile, must be done: it
      // reads the P buffer and adds into the O this tile may rescale
      if (u > 1) {
        if (!__all_sync(full_mask, ptx::mbar_wait(bars.pv_done(X), ((u >> 1) - 1) & 1))) {
          record_timeout(p.err, abort_flag); alive = false; break;
        }
        ptx::tc_fence_after();
      }
      // P = 2^(s*c - m_ref) as bf16 (ex2(-inf) = 0 for masked keys), row r
      // of this warpgroup's P buffer: the MMA's K-major layout, two 64-key
      // halves of 128-byte rows, 16-byte chunk j of row r at j ^ (r & 7)
      const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      uint8_t* prow = smem + kPOff + X * kPBytes + r * 128;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int half = 1 - hh;
        if (hh == 1) {
          ptx::tmem_ld32(s_addr, sv[0]);
          ptx::tmem_ld32(s_addr + 32, sv[1]);
          ptx::tmem_wait_ld();
          // S(u) is read: its TMEM buffer may take S(u + 2)
          ptx::tc_fence_before();
          ptx::mbar_arrive(bars.s_free(X));
          if (nv < kTile) mask_keys(sv, 0, nv);
        }
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {  // 8 keys: 64 half + 8 ch .. + 7
          uint32_t w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int k0 = 8 * ch + 2 * e;  // key of the pair's low half within the half
            const float p0 = ptx::ex2(fmaf(__uint_as_float(sv[k0 >> 5][k0 & 31]), c, nm));
            const float p1 = ptx::ex2(fmaf(__uint_as_float(sv[k0 >> 5][(k0 & 31) + 1]), c, nm));
            ls[e] += p0 + p1;
            w4[e] = ptx::pack_bf16x2(p0, p1);
          }
          *reinterpret_cast<uint4*>(prow + half * (kRows * 128) + ((ch ^ (r & 7)) << 4)) =
              make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      l = l * f + ((ls[0] + ls[1]) + (ls[2] + ls[3]));
      if (rescale && u > 1) {  // O holds this warpgroup's earlier tiles
#pragma unroll
        for (int cb = 0; cb < kD / 32; ++cb) {
          uint32_t o[32];
          ptx::tmem_ld32_sync(lane_addr + kOCol + X * kD + cb * 32, o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          ptx::tmem_st32(lane_addr + kOCol + X * kD + cb * 32, o);
        }
        ptx::tmem_wait_st();
      }
      if (nv_tile < kTile) {
        // rows past the valid keys hold stale or foreign data: zero them in V
        // so 0 * garbage cannot reach O
        if (!__all_sync(full_mask, ptx::mbar_wait(bars.v_full(st), (u / kStages) & 1))) {
          record_timeout(p.err, abort_flag); alive = false; break;
        }
        const int nz = (kTile - nv_tile) * 8 * halves;  // 16-byte chunks
        for (int e = wg_tid; e < nz; e += 128) {
          const int h = e / ((kTile - nv_tile) * 8), rem = e % ((kTile - nv_tile) * 8);
          const int row = nv_tile + rem / 8, cc = rem % 8;
          *reinterpret_cast<uint4*>(smem + kRingOff + st * kStageBytes + 2 * kHalfTile +
                                    h * kHalfTile + row * 128 + cc * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      // the tensor core reads P (and the zeroed V rows) through the async proxy
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bars.p_full(X));
    }
    // ---- this split's unnormalised O, row max and row sum -> workspace (L2).
    // The two warpgroups swap (max, sum) through shared memory; each then
    // writes half of the row's columns of O_0 2^(m_0 - m) + O_1 2^(m_1 - m).
    // (the exchange reuses Q's shared memory: every MMA has finished with it)
    const bool mine = alive && U > X && !__any_sync(full_mask, *abort_flag != 0);
    bool have = U > 0;
    if (have && !__all_sync(full_mask, ptx::mbar_wait(bars.mma_done(), 0))) {
      record_timeout(p.err, abort_flag);
      have = false;
    }
    float2* xch = reinterpret_cast<float2*>(smem);  // [2][128]
    ptx::named_bar_sync(1, 256);  // both warpgroups are past every read of Q
    xch[X * kRows + r] = mine ? make_float2(m_ref, l) : make_float2(-INFINITY, 0.f);
    ptx::named_bar_sync(1, 256);
    have = have && !__any_sync(full_mask, *abort_flag != 0);
    if (have) ptx::tc_fence_after();
    const float2 a0 = xch[r], a1 = xch[kRows + r];
    const float m = fmaxf(a0.x, a1.x);
    const float f0 = a0.x == -INFINITY ? 0.f : ptx::ex2(a0.x - m);
    const float f1 = a1.x == -INFINITY ? 0.f : ptx::ex2(a1.x - m);
    // row r's place in its group: chunk c at c * R + r % R, then (max, sum)
    const int R = p.R;
    float4* po = reinterpret_cast<float4*>(part) + (r / R) * group_f4<kD>(R) + r % R;
    const bool keep = r < rows;  // rows past G * blk are padding
#pragma unroll
    for (int cb = 0; cb < kD / 64; ++cb) {
      const int col = X * (kD / 2) + cb * 32;
      uint32_t o0[32], o1[32];
      if (have) {  // warp-uniform: the TMEM loads are warp-wide; one wait for both
        ptx::tmem_ld32(lane_addr + kOCol + col, o0);
        ptx::tmem_ld32(lane_addr + kOCol + kD + col, o1);
        ptx::tmem_wait_ld();
      }
#pragma unroll
      for (int j8 = 0; j8 < 4; ++j8) {
        uint32_t w4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int k = 8 * j8 + 2 * e + h;
            // selects, not products: an O that no tile wrote may hold anything
            const float x0 = have && f0 != 0.f ? f0 * __uint_as_float(o0[k]) : 0.f;
            v[h] = have && f1 != 0.f ? fmaf(f1, __uint_as_float(o1[k]), x0) : x0;
          }
          w4[e] = ptx::pack_bf16x2(v[0], v[1]);
        }
        if (keep)
          __stcg(reinterpret_cast<uint4*>(po) + (col / 8 + j8) * R,
                 make_uint4(w4[0], w4[1], w4[2], w4[3]));
      }
    }
    if (X == 0 && keep)
      __stcg(po + (kD / 8) * R,
             have && m != -INFINITY ? make_float4(m, f0 * a0.y + f1 * a1.y, 0.f, 0.f)
                                    : make_float4(-INFINITY, 0.f, 0.f, 0.f));
  }
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
  if (!kFused) return;  // the combine kernel merges the splits

  // ---- split merge inside the launch (every CTA of the grid is resident at
  // once: the host takes this path only when the grid fits one wave).  One
  // 64-bit word per (sequence, kv-head): generation << 32 | arrivals.  Each
  // CTA publishes its partial and adds one arrival (fire and forget, after a
  // fence); the CTAs that merge wait until the count reaches S within their
  // generation.  Split 0, having seen it, moves to the next generation and
  // returns the count to zero in one atomic -- a CTA that looks after that
  // sees the new generation and goes on too.  Then CTA `split` merges query
  // rows [split * R, split * R + R) in split order and writes them; the
  // splits that own no rows leave once counted.
  const bool merger = split * p.R < rows;
  volatile int* go = abort_flag + 1;
  if (threadIdx.x == 0) {
    unsigned long long* word = p.counters + (b * p.Hkv + g);
    __threadfence();  // this CTA's partial is visible before it is counted
    atomicAdd(word, 1ull);
    int ok = 1;
    if (merger) {
      const uint64_t t0 = ptx::globaltimer();
      for (;;) {
        const unsigned long long w = ptx::ld_acquire_gpu_u64(word);
        if ((unsigned)(w >> 32) != gen0 || (unsigned)w == (unsigned)S) break;
        if (ptx::globaltimer() - t0 > 1000000000ull) {
          set_err(p.err, ORTHRUS_ETIMEOUT);
          ok = 0;
          break;
        }
      }
      if (ok && split == 0) atomicAdd(word, (1ull << 32) - (unsigned long long)S);
    }
    *go = ok;
  }
  if (!merger) return;
  __syncthreads();
  if (*go && !bad)
    merge_rows<kD>(p, b, g, split, threadIdx.x, kThreads, smem + kRingOff, bars.merge_full());
}

// Merge the S split partials of query-row group q (rows [q R, q R + R)) of
// (sequence b, kv-head g) and write bf16 output.  The first warp stages
// every split's block of the group into shared memory with bulk copies (lane
// s the split s, all in flight at once, completing on `bar`); then one item
// per (row, 16-byte chunk) merges the splits in index order, so the result
// does not depend on timing.  `stage` holds S * (D/4 + 1) * R float4s.  Every thread
// of the CTA calls this with the same q (the barrier inside is CTA-wide).
template <int kD>
__device__ __forceinline__ void merge_rows(const TcParams& p, int b, int g, int q, int tid,
                                           int nthreads, uint8_t* stage, uint32_t bar) {
  constexpr int kChunks = kD / 8;  // 16-byte chunks of 8 bf16 dims
  const int R = p.R, S = p.S;
  const int r0 = q * R;
  const int nr = min(R, p.G * p.blk - r0);
  if (nr <= 0) return;
  const int gf4 = group_f4<kD>(R);
  float4* st4 = reinterpret_cast<float4*>(stage);
  const float4* base = reinterpret_cast<const float4*>(
      p.part + (int64_t)(b * p.Hkv + g) * S * part_floats<kD>());
  if (tid < 32) {
    // lane s copies split s's block (the copies go out together); the
    // partials were written by other CTAs' generic stores, acquired through
    // the CTA's barrier after thread 0's acquire, and the bulk copies read
    // them through the async proxy
    if (tid == 0) ptx::mbar_expect_tx(bar, (uint32_t)(S * gf4 * 16));
    __syncwarp();
    for (int s2 = tid; s2 < S; s2 += 32) {
      ptx::fence_proxy_async_global();
      ptx::bulk_g2s(ptx::smem_u32(st4 + s2 * gf4),
                    base + (int64_t)s2 * (part_floats<kD>() / 4) + (int64_t)q * gf4,
                    (uint32_t)(gf4 * 16), bar);
    }
  }
  if (!ptx::mbar_wait(bar, 0)) {
    set_err(p.err, ORTHRUS_ETIMEOUT);
    return;
  }
  // One item per (row, 16-byte chunk).  With threads to spare and enough
  // splits to share, two threads take an item, one the even splits and one
  // the odd (lanes 2k and 2k + 1: nthreads is even), and the even one adds
  // the odd one's sums to its own.
  const int items = nr * kChunks;
  const bool pair = 2 * items <= nthreads && S >= 8;
  const int per = pair ? 2 : 1;
  for (int it2 = tid; it2 < items * per; it2 += nthreads) {
    const int it = it2 / per, half = it2 % per;
    const int c8 = it / nr, rl = it % nr, r = r0 + rl;
    float M = -INFINITY;
    for (int s2 = 0; s2 < S; ++s2) M = fmaxf(M, st4[s2 * gf4 + kChunks * R + rl].x);
    if (M == -INFINITY) continue;  // no split has keys: an error was recorded
    float L = 0.f, acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int s2 = half; s2 < S; s2 += per) {
      const float4 ml = st4[s2 * gf4 + kChunks * R + rl];
      const uint4 o = reinterpret_cast<const uint4*>(st4)[s2 * gf4 + c8 * R + rl];
      const float w = ptx::ex2(ml.x - M);  // 0 for an empty split
      L = fmaf(w, ml.y, L);
      const uint32_t ow[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] = fmaf(w, __uint_as_float(ow[e] << 16), acc[2 * e]);
        acc[2 * e + 1] = fmaf(w, __uint_as_float(ow[e] & 0xffff0000u), acc[2 * e + 1]);
      }
    }
    if (pair) {
      // both lanes of the pair are here: same item, same M
      const unsigned pm = 3u << ((threadIdx.x & 31) & ~1);
      L += __shfl_xor_sync(pm, L, 1);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(pm, acc[e], 1);
      if (half) continue;
    }
    const float inv = 1.f / L;
    const int i = r / p.G, h = g * p.G + r % p.G;
    uint4 pkd;
    pkd.x = ptx::pack_bf16x2(acc[0] * inv, acc[1] * inv);
    pkd.y = ptx::pack_bf16x2(acc[2] * inv, acc[3] * inv);
    pkd.z = ptx::pack_bf16x2(acc[4] * inv, acc[5] * inv);
    pkd.w = ptx::pack_bf16x2(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4*>(p.out + ((int64_t)(b * p.blk + i) * p.Hq + h) * kD + 8 * c8) = pkd;
  }
}

// Separate merge for grids larger than one wave: grid (8-row groups, Hkv, B),
// after the partial kernel has completed.
template <int kD>
__global__ void __launch_bounds__(kCombineThreads)
attn_tc_combine(const __grid_constant__ TcParams p) {
  extern __shared__ __align__(128) uint8_t stage[];
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_u32(&bar), 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  ptx::griddep_launch_dependents();
  ptx::griddep_wait();
  const int n = p.ctx_lens[blockIdx.z];
  if (n < 0 || n > p.max_ctx) return;  // reported by the partial kernel
  merge_rows<kD>(p, blockIdx.z, blockIdx.y, blockIdx.x, threadIdx.x, kCombineThreads, stage,
                 ptx::smem_u32(&bar));
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

// Shared memory a combine CTA stages its 8 rows of every split in.
int combine_smem_bytes(int D, int S) { return S * (D / 8 + 1) * kGroupRows * 16; }

template <int kD>
bool prepare(int device) {
  static bool done[64] = {false};
  if (device >= 0 && device < 64 && done[device]) return true;
  if (cudaFuncSetAttribute(attn_tc_combine<kD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           combine_smem_bytes(kD, kMaxSplits)) != cudaSuccess ||
      cudaFuncSetAttribute(attn_tc_kernel<kD, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(attn_tc_kernel<kD, false>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return false;
  if (device >= 0 && device < 64) done[device] = true;
  return true;
}

int sm_count(int device) {
  static int cache[64] = {0};
  if (device < 0 || device >= 64) return 0;
  if (!cache[device]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return 0;
    cache[device] = n;
  }
  return cache[device];
}

// The SM count the workspace is sized for: the splits grow with the SM count
// only (through sms / heads), so a buffer sized for this many serves any GPU
// with at most as many SMs; the launch checks it.
constexpr int kSizingSms = 256;

}  // namespace

// Splits per (sequence, kv-head) on a GPU with `sms` SMs: enough to fill one
// wave of CTAs (one per SM) when the batch is small, and at least enough that
// no split of the longest possible sequence exceeds 64 tiles, so long or
// ragged batches spread over several waves instead of leaving their longest
// sequences to a few CTAs; never more splits than the longest sequence has
// tiles, nor more than the merge holds.
int tc_plan_splits(const orthrus_attn_args& a, int sms) {
  const int heads = a.B * a.Hkv;
  const int tiles = ceil_div(a.max_ctx, kTile) + 1;
  int S = heads >= sms ? 1 : sms / max(heads, 1);
  S = max(S, ceil_div(tiles, 64));
  // at least two tiles a split: a CTA's start-up and its partial cost more
  // than a second tile (Qwen3-1.7B layer, 17 tiles: 17 splits 11.1 us, 8
  // splits 10.3 us per call)
  S = min(S, max(1, tiles / 2));
  return max(1, min(S, kMaxSplits));
}

// The merge runs inside the one launch when every CTA of the grid is
// resident at once (one per SM) and the counters fit the workspace head.
bool tc_plan_fused(const orthrus_attn_args& a, int sms, int S) {
  return (int64_t)a.B * a.Hkv * S <= sms && a.B * a.Hkv <= kMaxFusedHeads;
}

int tc_smem_bytes() { return kSmemBytes; }
int tc_threads() { return kThreads; }

bool tc_supported(const orthrus_attn_args& a) {
  return a.dtype == ORTHRUS_BF16 && (a.D == 64 || a.D == 128) &&
         (a.Hq / a.Hkv) * a.blk <= kRows && a.blk <= 32 && a.Hq / a.Hkv <= 256 &&
         a.B <= 65535 && a.Hkv <= 65535;
}

size_t tc_workspace_bytes(const orthrus_attn_args& a) {
  const int64_t per = a.D == 64 ? part_floats<64>() : part_floats<128>();
  return (size_t)(kCounterBytes +
                  (int64_t)a.B * a.Hkv * tc_plan_splits(a, kSizingSms) * per * 4);
}

int tc_launches(const orthrus_attn_args& a) {
  int sms = 148, dev = 0;  // the current device's count when there is one
  if (cudaGetDevice(&dev) == cudaSuccess && sm_count(dev) > 0) sms = sm_count(dev);
  else cudaGetLastError();
  return tc_plan_fused(a, sms, tc_plan_splits(a, sms)) ? 1 : 2;
}

int tc_launch(const orthrus_attn_args& a, cudaStream_t st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ORTHRUS_ECUDA;
  if (!(a.D == 64 ? prepare<64>(dev) : prepare<128>(dev))) return ORTHRUS_ECUDA;
  const int sms = sm_count(dev);
  if (sms <= 0) return ORTHRUS_ECUDA;
  const int S = tc_plan_splits(a, sms);
  const bool fused = tc_plan_fused(a, sms, S);
  const int64_t per = a.D == 64 ? part_floats<64>() : part_floats<128>();
  if ((int64_t)a.workspace_bytes < kCounterBytes + (int64_t)a.B * a.Hkv * S * per * 4)
    return ORTHRUS_EWORKSPACE;
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
  p.next_k = static_cast<const __nv_bfloat16*>(a.next_k_cache);
  p.next_v = static_cast<const __nv_bfloat16*>(a.next_v_cache);
  if (!p.next_k || !p.next_v) p.next_k = p.next_v = nullptr;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.err = a.err;
  p.counters = static_cast<unsigned long long*>(a.workspace);
  p.part = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + kCounterBytes);
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.blk = a.blk; p.cap = a.cap;
  p.max_ctx = a.max_ctx; p.mask_mode = a.mask_mode; p.G = G; p.S = S;
  p.R = fused ? ceil_div(G * a.blk, S) : kGroupRows;
  p.early = (a.flags & ORTHRUS_ATTN_EARLY_KV) ? 1 : 0;
  p.order = !fused && a.B >= 2 && a.B <= 32;
  p.scale_log2 = (float)((double)a.scale * 1.4426950408889634);

  cudaLaunchAttribute pdl;
  pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.Hkv, a.B, S);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cfg.attrs = &pdl;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (fused)
    e = a.D == 64 ? cudaLaunchKernelEx(&cfg, attn_tc_kernel<64, true>, p)
                  : cudaLaunchKernelEx(&cfg, attn_tc_kernel<128, true>, p);
  else
    e = a.D == 64 ? cudaLaunchKernelEx(&cfg, attn_tc_kernel<64, false>, p)
                  : cudaLaunchKernelEx(&cfg, attn_tc_kernel<128, false>, p);
  if (e != cudaSuccess || fused) return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA;
  cfg.gridDim = dim3(ceil_div(G * a.blk, kGroupRows), a.Hkv, a.B);
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = combine_smem_bytes(a.D, S);
  e = a.D == 64 ? cudaLaunchKernelEx(&cfg, attn_tc_combine<64>, p)
                : cudaLaunchKernelEx(&cfg, attn_tc_combine<128>, p);
  return e == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA;
}

}  // namespace orthrus
