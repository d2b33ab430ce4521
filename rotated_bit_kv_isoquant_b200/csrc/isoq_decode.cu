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

#include "isoq_common.cuh"
#include "isoq_internal.h"

namespace isoq {

// a9: merge the partial softmax states of one (sequence, query head) by log-sum-exp.
// FINAL: normalise, inverse SO(4) blocks and inverse (orthonormal, self-inverse) WHT, write
// the output row; otherwise write the merged state (acc, m, l) in the partial layout, for
// a later merge with the states of other context slices.  Part j of (s, h) sits at
// parts + (s * n_q_heads + h) * sh_stride + j * part_stride floats.  One CTA of 128
// threads per (sequence, head): the parts are spread over 4 groups of 32 lanes (each lane
// 4 or 8 dims, 16-byte loads, several parts in flight), so the merge costs a few memory
// round trips however many parts there are; warp 0 then finishes.
template <int D, bool FINAL>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(const float* __restrict__ params, int H, int n_q_heads,
                          int rows_per_seq, int n_splits, const float* __restrict__ partials,
                          size_t sh_stride, size_t part_stride, float* __restrict__ out) {
  constexpr int E = D / 32;   // dims per lane
  constexpr int NB = E / 4;
  constexpr int PS = D + 4;
  constexpr int UNROLL = 4;
  __shared__ float red_m[4];
  __shared__ float red_acc[4][D];
  __shared__ float red_l[4];
  const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
  const int s = blockIdx.y, h = blockIdx.x;
  const int G = n_q_heads / H;
  const float* base = partials + ((size_t)s * rows_per_seq + h) * sh_stride;

  // global max of the splits' running maxima (empty splits report -inf)
  float M = -CUDART_INF_F;
  for (int j = tid; j < n_splits; j += 128) M = fmaxf(M, __ldg(base + (size_t)j * part_stride + D));
  M = warp_max(M);
  if (lane == 0) red_m[grp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));

  float acc[E], L = 0.f;
#pragma unroll
  for (int i = 0; i < E; ++i) acc[i] = 0.f;
  if (M != -CUDART_INF_F) {
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
      for (int u = 0; u < UNROLL; ++u) {
        const float w = mj[u] == -CUDART_INF_F ? 0.f : __expf(mj[u] - M);
        L = fmaf(w, lj[u], L);
#pragma unroll
        for (int k = 0; k < NB; ++k) {
          acc[4 * k + 0] = fmaf(w, v[u][k].x, acc[4 * k + 0]);
          acc[4 * k + 1] = fmaf(w, v[u][k].y, acc[4 * k + 1]);
          acc[4 * k + 2] = fmaf(w, v[u][k].z, acc[4 * k + 2]);
          acc[4 * k + 3] = fmaf(w, v[u][k].w, acc[4 * k + 3]);
        }
      }
    }
    for (; j < n_splits; j += 4) {
      const float* p = base + (size_t)j * part_stride;
      const float mj = __ldg(p + D);
      const float w = mj == -CUDART_INF_F ? 0.f : __expf(mj - M);
      L = fmaf(w, __ldg(p + D + 1), L);
#pragma unroll
      for (int k = 0; k < NB; ++k) {
        const float4 x = __ldg(reinterpret_cast<const float4*>(p + lane * E) + k);
        acc[4 * k + 0] = fmaf(w, x.x, acc[4 * k + 0]);
        acc[4 * k + 1] = fmaf(w, x.y, acc[4 * k + 1]);
        acc[4 * k + 2] = fmaf(w, x.z, acc[4 * k + 2]);
        acc[4 * k + 3] = fmaf(w, x.w, acc[4 * k + 3]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < E; ++i) red_acc[grp][lane * E + i] = acc[i];
  if (lane == 0) red_l[grp] = L;
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
  const float* hp = params + (size_t)((h % n_q_heads) / G) * D * 4;  // block matrices
  float y[E];
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    float M[16];
    load_block_mat(hp, lane * NB + k, M);
    mat_inv(M, o + 4 * k, y + 4 * k);
  }
  wht_warp<E>(y, lane);
  const float r = rsqrtf((float)D);
  float* dst = out + ((size_t)s * rows_per_seq + h) * D + lane * E;
#pragma unroll
  for (int i = 0; i < E; ++i) dst[i] = y[i] * r;
}

template <int D>
static cudaError_t launch_dq(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e = use_shared_mq(a) ? launch_decode_split_mq(a, stream)
                  : a.bits == 3    ? launch_decode_split_i8(a, stream)
                                   : launch_decode_split_mma(a, stream);
  if (e != cudaSuccess) return e;
  const int rows = a.n_q * a.n_q_heads;
  dim3 grid(rows, a.n_seqs);
  const size_t PS = partial_stride(D);
  if (a.state)
    decode_combine_kernel<D, false><<<grid, 128, 0, stream>>>(
        a.params, a.n_kv_heads, a.n_q_heads, rows, a.n_splits, a.partials, a.n_splits * PS, PS,
        a.state);
  else
    decode_combine_kernel<D, true><<<grid, 128, 0, stream>>>(
        a.params, a.n_kv_heads, a.n_q_heads, rows, a.n_splits, a.partials, a.n_splits * PS, PS,
        a.out);
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
  if (d == 128)
    decode_combine_kernel<128, true><<<grid, 128, 0, stream>>>(
        params, n_kv_heads, n_q_heads, n_q_heads, n_states, states, PS, slice, out);
  else if (d == 256)
    decode_combine_kernel<256, true><<<grid, 128, 0, stream>>>(
        params, n_kv_heads, n_q_heads, n_q_heads, n_states, states, PS, slice, out);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace isoq
