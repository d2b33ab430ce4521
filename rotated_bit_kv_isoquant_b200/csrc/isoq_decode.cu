// Decode attention on the packed 3-bit cache: split-K partials + combine with the
// inverse rotation.
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: attention is computed on the packed 3-bit codes
// and full-precision K/V are never reconstructed.  Because the rotation R is
// orthogonal, q.k_hat = (R q).(R k_hat): the query is rotated once, every score and the
// value accumulation run on codebook levels in the rotated space, and only the final
// output is rotated back.  The context is split into chunks that run in parallel and are
// merged by log-sum-exp ("FreeToken releases", v0.2.0, Kernels: split decode attention by
// context length and SM count); an empty chunk reports m = -inf and is skipped by the
// merge rather than exponentiated (the same release notes a NaN from a softmax chunk that
// starts at -inf).
#include <math_constants.h>

#include "isoq_check.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"

namespace isoq {

// a9: merge the partial softmax states of one (sequence, query head) by log-sum-exp.
// FINAL: normalise, inverse SO(4) blocks and inverse (orthonormal, self-inverse) WHT, write
// the output row; otherwise write the merged state (acc, m, l) in the partial layout, for
// a later merge with the states of other context slices.  Part j of (s, h) sits at
// parts + (s * n_q_heads + h) * sh_stride + j * part_stride floats.  One CTA of 128
// threads per (sequence, head): the parts are spread over 4 groups of 32 lanes (each lane
// 4 or 8 dims, 16-byte loads, several parts in flight), each group merging its parts in
// one pass with a running maximum; the groups then merge in shared memory and warp 0
// finishes.  Launched as a programmatic dependent of the split kernel: the rotation
// parameters are read before griddepcontrol.wait, the partials after it.
template <int D, bool FINAL>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(const float* __restrict__ params, int H, int n_q_heads,
                          int rows_per_seq, int n_splits, const float* __restrict__ partials,
                          size_t sh_stride, size_t part_stride, float* __restrict__ out,
                          size_t parts_len, uint32_t* status) {
  constexpr int E = D / 32;   // dims per lane
  constexpr int NB = E / 4;
  constexpr int PS = D + 4;
  constexpr int UNROLL = 8;  // one round of loads covers 32 chunks
  __shared__ float red_m[4];
  __shared__ float red_acc[4][D];
  __shared__ float red_l[4];
  const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
  const int s = blockIdx.y, h = blockIdx.x;
  const int G = n_q_heads / H;
  const float* base = partials + ((size_t)s * rows_per_seq + h) * sh_stride;

  // the inverse rotation's block matrices (independent of the split kernel)
  float Mb[NB][16];
  if (FINAL && grp == 0) {
    const float* hp = params + (size_t)((h % n_q_heads) / G) * D * 4;
#pragma unroll
    for (int k = 0; k < NB; ++k) load_block_mat(hp, lane * NB + k, Mb[k]);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials are complete

  // this group's parts j = grp, grp + 4, ...: running maximum Mg, acc and L relative to it
  float acc[E], L = 0.f, Mg = -CUDART_INF_F;
#pragma unroll
  for (int i = 0; i < E; ++i) acc[i] = 0.f;
  auto take = [&](float mj, float lj, const float4 (&v)[NB]) {
    if (mj == -CUDART_INF_F) return;  // an empty chunk
    if (mj > Mg) {                    // group-uniform
      const float r = __expf(Mg - mj);  // 0 when Mg was -inf
      L *= r;
#pragma unroll
      for (int i = 0; i < E; ++i) acc[i] *= r;
      Mg = mj;
    }
    const float w = __expf(mj - Mg);
    L = fmaf(w, lj, L);
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      acc[4 * k + 0] = fmaf(w, v[k].x, acc[4 * k + 0]);
      acc[4 * k + 1] = fmaf(w, v[k].y, acc[4 * k + 1]);
      acc[4 * k + 2] = fmaf(w, v[k].z, acc[4 * k + 2]);
      acc[4 * k + 3] = fmaf(w, v[k].w, acc[4 * k + 3]);
    }
  };
  // checked build: every part read lies inside the partials (parts_len floats)
  [[maybe_unused]] const size_t base_off = base - partials;
  if (!in_bounds(base_off + (size_t)(n_splits > 0 ? n_splits - 1 : 0) * part_stride + PS <= parts_len,
                 status))
    n_splits = 0;
  int j = grp;
  for (; j + 4 * (UNROLL - 1) < n_splits; j += 4 * UNROLL) {
    float mj[UNROLL], lj[UNROLL];
    float4 v[UNROLL][NB];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const float* p = base + (size_t)(j + 4 * u) * part_stride;
      mj[u] = __ldg(p + D);
      lj[u] = __ldg(p + D + 1);
#pragma unroll
      for (int k = 0; k < NB; ++k) v[u][k] = __ldg(reinterpret_cast<const float4*>(p + lane * E) + k);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) take(mj[u], lj[u], v[u]);
  }
  for (; j < n_splits; j += 4) {
    const float* p = base + (size_t)j * part_stride;
    float4 v[NB];
#pragma unroll
    for (int k = 0; k < NB; ++k) v[k] = __ldg(reinterpret_cast<const float4*>(p + lane * E) + k);
    take(__ldg(p + D), __ldg(p + D + 1), v);
  }
  if (lane == 0) red_m[grp] = Mg;
  __syncthreads();
  const float M = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
  const float r = Mg == -CUDART_INF_F ? 0.f : __expf(Mg - M);  // this group's share
#pragma unroll
  for (int i = 0; i < E; ++i) red_acc[grp][lane * E + i] = acc[i] * r;
  if (lane == 0) red_l[grp] = L * r;
  __syncthreads();
  if (grp != 0) return;

  const float Ls = red_l[0] + red_l[1] + red_l[2] + red_l[3];
  if constexpr (!FINAL) {
    float* dst = out + ((size_t)s * rows_per_seq + h) * PS;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int dd = lane * E + i;
      dst[dd] = red_acc[0][dd] + red_acc[1][dd] + red_acc[2][dd] + red_acc[3][dd];
    }
    if (lane < 4) dst[D + lane] = lane == 0 ? M : (lane == 1 ? Ls : 0.f);
    return;
  }
  const float inv = Ls > 0.f ? 1.f / (Ls * sqrtf((float)D)) : 0.f;
  float o[E];
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int dd = lane * E + i;
    o[i] = (red_acc[0][dd] + red_acc[1][dd] + red_acc[2][dd] + red_acc[3][dd]) * inv;
  }
  float y[E];
#pragma unroll
  for (int k = 0; k < NB; ++k) mat_inv(Mb[k], o + 4 * k, y + 4 * k);
  wht_warp<E>(y, lane);
  const float rs = rsqrtf((float)D);
  float* dst = out + ((size_t)s * rows_per_seq + h) * D + lane * E;
#pragma unroll
  for (int i = 0; i < E; ++i) dst[i] = y[i] * rs;
}

// The combine on `stream` as a programmatic dependent launch of the kernel before it (it
// may start while that kernel drains; it waits in-kernel for its results).
template <int D, bool FINAL>
static cudaError_t launch_combine(dim3 grid, cudaStream_t stream, bool dependent,
                                  const float* params, int H, int n_q_heads, int rows_per_seq,
                                  int n_splits, const float* partials, size_t sh_stride,
                                  size_t part_stride, float* out, size_t parts_len,
                                  uint32_t* status) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, decode_combine_kernel<D, FINAL>, params, H, n_q_heads,
                            rows_per_seq, n_splits, partials, sh_stride, part_stride, out,
                            parts_len, status);
}

template <int D>
static cudaError_t launch_dq(const DecodeArgs& a, cudaStream_t stream) {
  bool combined = false;  // a single-chunk 3-bit decode writes the output itself
  cudaError_t e = use_shared_mq(a) ? launch_decode_split_mq(a, stream)
                  : a.bits == 3    ? launch_decode_split_i8(a, stream, &combined)
                                   : launch_decode_split_mma(a, stream);
  if (e != cudaSuccess) return e;
  if (combined) return cudaSuccess;
  const int rows = a.n_q * a.n_q_heads;
  dim3 grid(rows, a.n_seqs);
  const size_t PS = partial_stride(D);
  const size_t parts_len = (size_t)a.n_seqs * rows * a.n_splits * PS;
  if (a.state)
    e = launch_combine<D, false>(grid, stream, true, a.params, a.n_kv_heads, a.n_q_heads, rows,
                                 a.n_splits, a.partials, a.n_splits * PS, PS, a.state, parts_len,
                                 a.status);
  else
    e = launch_combine<D, true>(grid, stream, true, a.params, a.n_kv_heads, a.n_q_heads, rows,
                                a.n_splits, a.partials, a.n_splits * PS, PS, a.out, parts_len,
                                a.status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.n_seqs == 0 || a.n_q_heads == 0) return cudaSuccess;
  if (a.d == 128) return launch_dq<128>(a, stream);
  if (a.d == 256) return launch_dq<256>(a, stream);
  return cudaErrorInvalidValue;
}

// Merge of n_states context-slice states laid out [n_states][n_seqs][n_q_heads][d + 4].
cudaError_t launch_merge_states(const float* params, int n_kv_heads, int d, int n_seqs,
                                int n_q_heads, int n_states, const float* states, float* out,
                                cudaStream_t stream) {
  if (n_seqs == 0 || n_q_heads == 0) return cudaSuccess;
  dim3 grid(n_q_heads, n_seqs);
  const size_t PS = partial_stride(d);
  const size_t slice = (size_t)n_seqs * n_q_heads * PS;
  cudaError_t e;
  if (d == 128)
    e = launch_combine<128, true>(grid, stream, false, params, n_kv_heads, n_q_heads, n_q_heads,
                                  n_states, states, PS, slice, out, slice * n_states, nullptr);
  else if (d == 256)
    e = launch_combine<256, true>(grid, stream, false, params, n_kv_heads, n_q_heads, n_q_heads,
                                  n_states, states, PS, slice, out, slice * n_states, nullptr);
  else
    return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace isoq
