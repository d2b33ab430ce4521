// Internal launch interface between the C-ABI layer (isoq_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

struct isoq_params;
struct isoq_cache;

namespace isoq {

// One layer's cache and inputs for a quantize-append launch.
struct QuantLayer {
  const float* mats;    // device [H][d/4][4][4]: block rotations as matrices
  uint8_t* blocks;
  const int32_t* page_table;
  const void* K;
  const void* V;
  uint32_t* status;
  int n_pages, max_pages, n_seqs;
};

// Layers quantised by one launch (blockIdx.y = layer), passed by value as a kernel
// parameter (32 * 64 bytes).
constexpr int kMaxLayers = 32;
struct QuantLayers {
  QuantLayer l[kMaxLayers];
  int n;
};

struct QuantizeArgs {
  QuantLayers layers;
  int bits;             // bits per code (2, 3, 4), the same for every layer
  int n_kv_heads, d;
  int dtype;
  int n_tokens;
  const int32_t* seq_ids;
  const int32_t* positions;
  const float* rope;    // optional device [rope_max_pos][d/2][2] (cos, sin): RoPE applied to K
  int rope_max_pos;
};

struct DecodeArgs {
  const float* params;  // the heads' 4x4 block matrices [n_kv_heads][d/4][16]
  int bits;             // bits per code (2, 3, 4)
  const uint8_t* blocks;
  const int32_t* page_table;
  int n_pages, max_pages, n_kv_heads, d;
  const void* Q;
  int q_dtype;
  int n_seqs, n_q_heads;
  int n_q;              // query tokens per sequence (1 = decode)
  const int32_t* seq_lens;
  float scale;
  int n_splits;         // context chunks per (sequence, KV head)
  int pages_per_split;  // pages in each chunk
  float* partials;      // [n_seqs][n_q][n_q_heads][n_splits][d + 4]
  float* out;           // [n_seqs][n_q][n_q_heads][d] (when state is null)
  float* state;         // if set: merged state [n_seqs][n_q][n_q_heads][d + 4] instead of out
  uint32_t* status;
};

cudaError_t launch_quantize_append(const QuantizeArgs& a, cudaStream_t stream, int n_sm);
// d = 128, bf16 / f16 inputs without RoPE: the WHT as a tensor-core product.
bool use_quantize_tc(const QuantizeArgs& a);
cudaError_t launch_quantize_tc(const QuantizeArgs& a, cudaStream_t stream, int n_sm);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
// Merge of context-slice states [n_states][n_seqs][n_q_heads][d + 4] into the output.
cudaError_t launch_merge_states(const float* params, int n_kv_heads, int d, int n_seqs,
                                int n_q_heads, int n_states, const float* states, float* out,
                                cudaStream_t stream);
// Tensor-core split kernel (partials only); the combine runs separately.  The 2- and
// 4-bit formats (f16 operands).
cudaError_t launch_decode_split_mma(const DecodeArgs& a, cudaStream_t stream);
// Resident CTAs per SM of that kernel for head dimension d on the current device.
int decode_resident_ctas(int d);
// The 3-bit split kernel on 8-bit integer tensor-core products.  With `combined` non-null,
// a decode with a single context chunk writes its output directly (no combine needed:
// *combined is set); otherwise partials only.
cudaError_t launch_decode_split_i8(const DecodeArgs& a, cudaStream_t stream,
                                   bool* combined = nullptr);
int decode_i8_resident_ctas(int d);
// Rows ((query token, head) pairs of one KV head) per CTA of the 3-bit split kernel: 4
// when a KV head has at most 4 rows (the query digits of all of them then fit the 16 rows
// of one mma) or d = 256 (register budget), else 8.
inline int decode_rows_per_block(int d, int n_q, int group) {
  return (d == 256 || (long long)n_q * group <= 4) ? 4 : 8;
}
// Pages per context chunk at most: a warp of the 3-bit kernel then sums at most 32768
// tokens into its s32 value accumulators (|per-token term| < 2^16, far from overflow).
constexpr int kMaxPagesPerSplit = 2048;
// Multi-token chunks with many rows per KV head (d = 128): the page dequantised once per
// CTA into shared memory and shared by 64 (query token, head) rows (partials only).
bool use_shared_mq(const DecodeArgs& a);
cudaError_t launch_decode_split_mq(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_split_mqtc(const DecodeArgs& a, cudaStream_t stream);

// Rows ((query token, head) pairs of one KV head) per CTA of the attention kernels for a
// chunk of n_q query tokens and `group` query heads per KV head: the tensor-memory
// multi-token kernel takes 128 rows, the shared-page mma.sync kernel 64, the per-row
// kernel 8.  Both multi-token kernels keep 2 CTAs per SM.
#ifndef ISOQ_MQTC_MIN_ROWS
#define ISOQ_MQTC_MIN_ROWS 128
#endif
inline int attention_rows_per_cta(int d, int n_q, int group) {
  const long long rows = (long long)n_q * group;
  if (d != 128 || n_q <= 1 || rows < 16) return 8;
  return rows >= ISOQ_MQTC_MIN_ROWS ? 128 : 64;
}

// Accessors of the opaque parameter handle (defined in isoq_api.cu).
const float* params_device_mats(const struct ::isoq_params* p);  // [H][d/4][4][4]
int params_bits(const struct ::isoq_params* p);
int params_device(const struct ::isoq_params* p);
// Records e as the thread's last CUDA error and returns ISOQ_E_CUDA.
int record_cuda_error(cudaError_t e);
// The decode entry points' shared body (defined in isoq_api.cu): argument checks, the
// split plan, the split kernel and the combine, with the split partials in `workspace`.
int decode_run(const struct ::isoq_params* params, const ::isoq_cache* cache, const void* Q,
               int q_dtype, int n_seqs, int n_q, int n_q_heads, const int32_t* seq_lens,
               int max_seq_len, float* out, float* state, float scale, void* workspace,
               size_t workspace_bytes, void* stream);

// Partial-result stride (floats) of one (sequence, head, split): acc[d], m, l, 2 pad.
inline int partial_stride(int d) { return d + 4; }

}  // namespace isoq
