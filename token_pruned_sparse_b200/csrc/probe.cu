// tps_wait_probe: self-test of the failure-detection path. One CTA waits on a
// shared-memory barrier that nothing completes, through the bounded wait all
// TMA/MMA kernels of the library use, with a short limit; the wait gives up,
// records the timeout in the device status word, and the CTA exits normally.
#include "tc_ptx.cuh"

namespace tps {
namespace {

__global__ void wait_probe_kernel(long long limit, unsigned int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);               // one arrival completes phase 0; none comes
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  tc::mbar_wait_for(b, 0, &abort_flag, status, limit);
}

}  // namespace
}  // namespace tps

extern "C" int tps_wait_probe(int64_t limit_cycles, tps_stream stream) {
  using namespace tps;
  long long lim = limit_cycles < 1000 ? 1000 : limit_cycles;
  if (lim > tc::kWaitLimitCycles) lim = tc::kWaitLimitCycles;
  int err;
  unsigned int* st = device_status(&err);
  if (!st) return err;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(lim, st);
  if (int e = launch_status("tps_wait_probe")) return e;
  return ok();
}
