// Self-test of the bounded waits every kernel of the library relies on (gdn_ptx.cuh): a wait
// on an mbarrier that nothing arrives on, or on a ready flag that nothing sets, must give up
// after kWaitLimitCycles, OR error bit 1 into the error word and return, so that the kernel
// unwinds and the context stays usable; and once one waiter has given up, the block's other
// waiters must leave at their next poll instead of running out their own limits.  No fault,
// no trap: each launch ends after about one wait limit (~2^31 cycles).  Built into the test
// library (libgdn_selftest.so); the mixer library does not contain it.
#include "gdn_ptx.cuh"

using namespace gdn;

namespace {

// mode 0: warp 0 waits on an mbarrier nothing arrives on; warp 1 starts waiting on a second
//         such barrier 2^30 cycles later and must leave when warp 0 raises the abort.
// mode 1: warp 0 waits on a ready flag nothing sets (warp 1 idles).
// out[2w] = 1 if warp w's wait succeeded, out[2w + 1] = the cycles it waited.
__global__ void __launch_bounds__(64) wait_selftest_kernel(int mode, int* err, const int* flag, long long* out) {
  __shared__ uint64_t bar[2];
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_s = 0;
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  Abort ab{err, &abort_s};
  bool ok = false;
  long long waited = 0;
  if (mode == 0) {
    if (warp == 1) {  // a bounded delay before this warp starts to wait
      const long long d0 = clock64();
      while (clock64() - d0 < (1ll << 30)) __nanosleep(1000);
    }
    const long long t0 = clock64();
    ok = mbar_wait_warp(&bar[warp], 0, ab);
    waited = clock64() - t0;
  } else if (warp == 0) {
    const long long t0 = clock64();
    ok = flag_wait(flag, ab, 256);
    waited = clock64() - t0;
  }
  if (lane == 0) {
    out[2 * warp] = ok ? 1 : 0;
    out[2 * warp + 1] = waited;
  }
}

}  // namespace

// Launches one self-test block on the legacy default stream (asynchronous).  All pointers are
// device pointers: err (the error word), flag (an int that stays 0), out (4 long long).
// Returns 0 if the launch was accepted.
extern "C" int gdn_selftest_wait(int mode, int* err, const int* flag, long long* out) {
  if (mode < 0 || mode > 1 || !err || !flag || !out) return 1;
  wait_selftest_kernel<<<1, 64>>>(mode, err, flag, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 1;
}

// The limit after which a bounded wait gives up, in SM cycles.
extern "C" long long gdn_selftest_wait_limit_cycles() { return kWaitLimitCycles; }
