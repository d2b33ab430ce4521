// Self-test of the bounded waits every kernel's pipeline relies on (no wait can hang a GPU):
// an mbarrier phase that nothing completes is awaited with a short poll limit, the wait
// gives up, and the give-up is reported in the status word exactly as a kernel reports a
// page copy that never lands; a phase that does complete is observed as completed.
#include "isoq_check.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"

namespace isoq {
namespace {

__global__ void bounded_wait_selftest_kernel(uint32_t* status, unsigned polls, uint32_t* result) {
  __shared__ __align__(8) uint64_t bars[2];
  if (threadIdx.x != 0) return;
  ptx::mbar_init(bars, 1);      // never arrived at
  ptx::mbar_init(bars + 1, 1);  // arrived at once below
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  const bool gave_up = !ptx::mbar_wait_n(bars, 0, polls);  // false: the phase never completes
  ptx::mbar_arrive(bars + 1);
  const bool done = ptx::mbar_wait_n(bars + 1, 0, polls);
  if (gave_up) set_status(status, ISOQ_ST_TIMEOUT);  // as a kernel reports a lost page copy
  result[0] = gave_up ? 1u : 0u;
  result[1] = done ? 1u : 0u;
}

// An index check on an index outside its extent (index 8 of an 8-element buffer): nothing
// is accessed; the checked build reports it.
__global__ void bounds_selftest_kernel(uint32_t* status, int index, int extent) {
  if (threadIdx.x != 0) return;
  if (in_bounds(index < extent, status)) {
    // an access at index would go here
  }
}

}  // namespace
}  // namespace isoq

extern "C" int isoq_selftest_bounded_wait(uint32_t* status, unsigned polls, uint32_t* result,
                                          void* stream) {
  if (!status || !result || polls == 0) return ISOQ_E_ARG;
  isoq::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      status, polls, result);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ISOQ_OK : isoq::record_cuda_error(e);
}

extern "C" int isoq_selftest_bounds(uint32_t* status, void* stream) {
  if (!status) return ISOQ_E_ARG;
  isoq::bounds_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, 8, 8);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ISOQ_OK : isoq::record_cuda_error(e);
}
