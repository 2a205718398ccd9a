// selftest.cu -- exercises the bounded waits every kernel of this library
// relies on, without any fault: a wait on something that never happens
// gives up after its limit, records ORTHRUS_ETIMEOUT in the caller's error
// word and returns, and the context stays usable.  Two forms, the ones the
// kernels use:
//   0  an mbarrier phase that never completes (the TMA / MMA handshakes)
//   1  a generation word in global memory that nothing advances (the split
//      merge barrier of the attention kernel)
#include "common.cuh"
#include "orthrus.h"
#include "tc_ptx.cuh"

namespace orthrus {
namespace {

__global__ void bounded_wait_kernel(int which, uint64_t timeout_ns, const unsigned* never,
                                    int32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  bool ok = true;
  if (which == 0) {
    const uint32_t b = ptx::smem_u32(&bar);
    ptx::mbar_init(b, 1);
    ptx::fence_mbar_init();
    ok = ptx::mbar_wait(b, 0, timeout_ns);  // no arrival ever comes
  } else {
    const unsigned gen0 = ptx::ld_acquire_gpu(never);
    const uint64_t t0 = ptx::globaltimer();
    while (ptx::ld_acquire_gpu(never) == gen0) {
      if (ptx::globaltimer() - t0 > timeout_ns) {
        ok = false;
        break;
      }
    }
  }
  if (!ok) set_err(err, ORTHRUS_ETIMEOUT);
}

}  // namespace
}  // namespace orthrus

extern "C" int orthrus_selftest_bounded_wait(int32_t which, uint32_t timeout_us,
                                             const uint32_t* never, int32_t* err,
                                             orthrus_stream_t stream) {
  using namespace orthrus;
  if ((which != 0 && which != 1) || timeout_us == 0 || timeout_us > 10000000u || !err)
    return ORTHRUS_EINVAL;
  if (which == 1 && (!never || reinterpret_cast<uintptr_t>(never) % 4)) return ORTHRUS_EINVAL;
  bounded_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      which, (uint64_t)timeout_us * 1000ull, never, err);
  return cudaGetLastError() == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA;
}
