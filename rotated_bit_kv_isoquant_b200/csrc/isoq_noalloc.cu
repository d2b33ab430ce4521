// isoq_decode_attention_noalloc: decode attention for callers that cannot allocate device
// memory.  Same kernels as isoq_decode_attention; the split-K partial results live in a
// fixed array inside this library instead of a caller-provided workspace.
//
// Who needs it: a caller that has no device allocator of its own to draw a workspace from
// -- e.g. a plug-in handed only its input and output buffers by a host application that
// owns all device memory, or a thread that must not call cudaMalloc because that call can
// synchronise the device and stall other work.  Such a caller still passes Q, seq_lens
// and out; it just does not pass (or size) a workspace.
//
// Costs and rules (also stated in include/isoq.h):
//   * every GPU that loads the library holds the array (ISOQ_NOALLOC_SCRATCH_BYTES) until
//     the process exits;
//   * calls share the array, so two calls that overlap on the GPU (on different streams,
//     or from different threads without ordering) race and corrupt each other's results;
//   * the array keeps the previous call's contents; nothing needs clearing, because every
//     partial result the combine kernel reads is written by the split kernel of the same
//     call;
//   * the first call on a device looks up the array's device address there
//     (cudaGetSymbolAddress), so make that first call before any stream capture.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/isoq.h"
#include "isoq_internal.h"

namespace {

// The scratch array.  In host code `g_noalloc_scratch` names a host-side stand-in, not a
// device address: a kernel must be given the address obtained with cudaGetSymbolAddress.
constexpr size_t kScratchFloats = ISOQ_NOALLOC_SCRATCH_BYTES / sizeof(float);
static __device__ __align__(256) float g_noalloc_scratch[kScratchFloats];

// Device address of g_noalloc_scratch, per device, looked up once with that device current.
float* scratch_address(int device, cudaError_t* err) {
  static std::mutex mu;
  static float* addr[64] = {nullptr};
  *err = cudaSuccess;
  if (device < 0 || device >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      *err = e;
      return nullptr;
    }
    addr[device] = static_cast<float*>(p);
  }
  return addr[device];
}

}  // namespace

extern "C" int isoq_decode_attention_noalloc(const isoq_params* params, const isoq_cache* cache,
                                             const void* Q, int q_dtype, int n_seqs,
                                             int n_q_heads, const int32_t* seq_lens,
                                             int max_seq_len, float* out, float scale,
                                             void* stream) {
  if (!params) return ISOQ_E_ARG;
  // The array's address is looked up with the parameters' device current (the address is
  // per device); the decode then runs exactly as isoq_decode_attention does -- same checks,
  // same split plan, same kernels -- with the array as its workspace, and refuses a plan
  // whose partials do not fit the array (ISOQ_E_WORKSPACE, nothing launched).
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    isoq::record_cuda_error(e);
    cudaGetLastError();
    return ISOQ_E_DEVICE;
  }
  if (dev != isoq::params_device(params)) return ISOQ_E_DEVICE;
  float* scratch = scratch_address(dev, &e);
  if (!scratch) return isoq::record_cuda_error(e);
  return isoq::decode_run(params, cache, Q, q_dtype, n_seqs, 1, n_q_heads, seq_lens, max_seq_len,
                          out, nullptr, scale, scratch, (size_t)ISOQ_NOALLOC_SCRATCH_BYTES,
                          stream);
}
