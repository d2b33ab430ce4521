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
#include <math.h>

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

bool valid_dtype(int t) { return t == ISOQ_F32 || t == ISOQ_BF16 || t == ISOQ_F16; }

}  // namespace

extern "C" int isoq_decode_attention_noalloc(const isoq_params* params, const isoq_cache* cache,
                                             const void* Q, int q_dtype, int n_seqs,
                                             int n_q_heads, const int32_t* seq_lens,
                                             int max_seq_len, float* out, float scale,
                                             void* stream) {
  if (!params || !cache || !cache->blocks || !cache->page_table) return ISOQ_E_ARG;
  int pd = 0, ph = 0;
  isoq_params_shape(params, &pd, &ph);
  if (cache->page_size != ISOQ_PAGE_SIZE || (cache->d != 128 && cache->d != 256))
    return ISOQ_E_DIM;
  if (cache->d != pd || cache->n_kv_heads != ph) return ISOQ_E_DIM;
  if ((cache->bits == 0 ? 3 : cache->bits) != isoq::params_bits(params)) return ISOQ_E_DIM;
  if (cache->n_pages < 0 || cache->max_pages_per_seq < 1 || cache->n_seqs < 1 ||
      cache->n_kv_heads < 1)
    return ISOQ_E_ARG;
  if (n_seqs < 0 || n_q_heads < 0 || max_seq_len < 0 || !valid_dtype(q_dtype)) return ISOQ_E_ARG;
  if (!(scale == scale) || isinf(scale)) return ISOQ_E_ARG;
  if (n_q_heads % cache->n_kv_heads || n_q_heads / cache->n_kv_heads > 16) return ISOQ_E_GQA;
  if (n_seqs > cache->n_seqs) return ISOQ_E_ARG;
  if (n_seqs == 0 || n_q_heads == 0) return ISOQ_OK;
  if (!Q || !seq_lens || !out) return ISOQ_E_ARG;

  // Same context chunking as isoq_decode_attention; reject what does not fit the array.
  const size_t need = isoq_decode_workspace_bytes(n_seqs, n_q_heads, cache->n_kv_heads,
                                                  cache->d, max_seq_len);
  if (need == 0 || need > (size_t)ISOQ_NOALLOC_SCRATCH_BYTES) return ISOQ_E_WORKSPACE;
  const int n_splits =
      isoq_decode_num_splits(n_seqs, n_q_heads, cache->n_kv_heads, cache->d, max_seq_len);
  if (n_splits < 1) return n_splits < 0 ? n_splits : ISOQ_E_ARG;
  const int max_pages = max_seq_len > 0 ? (max_seq_len + ISOQ_PAGE_SIZE - 1) / ISOQ_PAGE_SIZE : 1;
  const int pages_per_split = (max_pages + n_splits - 1) / n_splits;

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

  isoq::DecodeArgs a{};
  a.params = isoq::params_device_mats(params);
  a.bits = isoq::params_bits(params);
  a.blocks = cache->blocks;
  a.page_table = cache->page_table;
  a.n_pages = cache->n_pages;
  a.max_pages = cache->max_pages_per_seq;
  a.n_kv_heads = cache->n_kv_heads;
  a.d = cache->d;
  a.Q = Q;
  a.q_dtype = q_dtype;
  a.n_seqs = n_seqs;
  a.n_q_heads = n_q_heads;
  a.n_q = 1;
  a.seq_lens = seq_lens;
  a.scale = scale;
  a.n_splits = n_splits;
  a.pages_per_split = pages_per_split;
  a.partials = scratch;
  a.out = out;
  a.status = cache->status;
  e = isoq::launch_decode(a, (cudaStream_t)stream);
  return e == cudaSuccess ? ISOQ_OK : isoq::record_cuda_error(e);
}
