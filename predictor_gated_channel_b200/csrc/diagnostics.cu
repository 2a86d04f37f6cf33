// diagnostics.cu -- a self-test of the bounded pipeline wait (no counterpart
// in the paper).
//
// Every kernel of this library waits on its shared-memory mbarriers through
// mbar_wait_limit (async_util.cuh): after a limit of SM clock cycles the wait
// gives up, sets kDevErrWaitTimeout in the library's device error word and
// returns false, and the kernel winds down instead of hanging the GPU.  No
// correct pipeline ever reaches that branch, so k_wait_timeout_probe reaches
// it on purpose: one warp waits on an mbarrier that nothing arrives on (no
// copy or MMA is in flight), with a caller-chosen short limit, and the CTA
// returns.  The device stays usable; the host reads the error bit through
// sfn_device_errors.
#include "async_util.cuh"
#include "sfn_internal.cuh"

namespace sfn {
namespace {

constexpr long long kProbeMaxCycles = 1000000000LL;  // about half a second

__global__ void __launch_bounds__(32) k_wait_timeout_probe(long long limit, unsigned *err,
                                                           int *gave_up) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival, which never comes
    fence_barrier_init();
  }
  __syncwarp();
  // every lane waits on phase 0 of the barrier, as the pipelines' consumer
  // warps do; each gives up after `limit` cycles
  const bool ok = mbar_wait_limit(&bar, 0u, err, limit);
  const unsigned all_gave_up = __ballot_sync(kFull, !ok);
  if (threadIdx.x == 0 && gave_up != nullptr) *gave_up = (all_gave_up == kFull) ? 1 : 0;
}

}  // namespace
}  // namespace sfn

using namespace sfn;

extern "C" sfn_status sfn_debug_wait_timeout(long long limit_cycles, int *gave_up,
                                             sfn_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > kProbeMaxCycles) return SFN_ERR_INVALID_VALUE;
  if (gave_up != nullptr && ((uintptr_t)gave_up % 4) != 0) return SFN_ERR_MISALIGNED;
  DeviceInfo dev;
  if (!device_info(&dev)) return SFN_ERR_CUDA;
  k_wait_timeout_probe<<<1, 32, 0, (cudaStream_t)stream>>>(limit_cycles, dev.err, gave_up);
  count_launches(1);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SFN_OK : SFN_ERR_CUDA;
}
