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

// Codes of the E dims E*lane .. E*lane+E-1 of one packed vector (the dims a lane owns in
// the warp layout of the WHT).
template <int E>
__device__ __forceinline__ void lane_codes(const uint8_t* __restrict__ rec, int lane,
                                           int (&c)[E]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(rec);
  if constexpr (E == 4) {
    const int g = lane >> 3, r = lane & 7;
    const uint32_t w0 = __ldg(w + 3 * g), w1 = __ldg(w + 3 * g + 1), w2 = __ldg(w + 3 * g + 2);
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = group_code(w0, w1, w2, 4 * r + i);
  } else {
    const int g = lane >> 2, r = lane & 3;
    const uint32_t w0 = __ldg(w + 3 * g), w1 = __ldg(w + 3 * g + 1), w2 = __ldg(w + 3 * g + 2);
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = group_code(w0, w1, w2, 8 * r + i);
  }
}

// One warp per (split, KV head, sequence).  GM = the largest group size the instance
// handles (G <= GM; heads >= G are idle).
template <int D, int GM, typename TQ>
__global__ void __launch_bounds__(32)
    decode_split_kernel(const float* __restrict__ params, const uint8_t* __restrict__ blocks,
                        const int32_t* __restrict__ page_table, int n_pages, int max_pages,
                        int H, const TQ* __restrict__ Q, int n_q_heads,
                        const int32_t* __restrict__ seq_lens, float scale, int pages_per_split,
                        int n_splits, float* __restrict__ partials, uint32_t* status) {
  constexpr int E = D / 32;
  constexpr int NB = E / 4;
  constexpr int CB = code_bytes(D);
  constexpr int BB = block_bytes(D);
  constexpr int PS = D + 4;
  __shared__ float qs[GM][D];     // rotated queries, unnormalised: sqrt(d) * R q
  __shared__ float pw[GM][32];    // chunk weights p_t * n^V_t
  __shared__ float lev[8];

  const int lane = threadIdx.x;
  const int split = blockIdx.x, hk = blockIdx.y, s = blockIdx.z;
  const int G = n_q_heads / H;
  if (lane < 8) lev[lane] = level_f32(lane);

  int len = __ldg(seq_lens + s);
  if (len > max_pages * kPage) {
    if (lane == 0 && split == 0 && hk == 0) set_status(status, ISOQ_ST_LEN_RANGE);
    len = max_pages * kPage;
  }
  const int t0 = split * pages_per_split * kPage;
  const int t1 = min(len, t0 + pages_per_split * kPage);

  float m[GM], l[GM], acc[GM][E];
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    m[h] = -CUDART_INF_F;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) acc[h][i] = 0.f;
  }

  if (t0 < t1) {
    // a6: rotate the group's queries once (unnormalised WHT, then the SO(4) blocks)
    const float* hp = params + (size_t)hk * D * 2;
    float pq[NB][8];
#pragma unroll
    for (int k = 0; k < NB; ++k) load_block_params(hp, lane * NB + k, pq[k]);
    for (int h = 0; h < G; ++h) {
      float v[E];
      const TQ* qp = Q + ((size_t)s * n_q_heads + hk * G + h) * D + lane * E;
#pragma unroll
      for (int i = 0; i < E; ++i) v[i] = to_f32<TQ>(qp[i]);
      wht_warp<E>(v, lane);
      float z[E];
#pragma unroll
      for (int k = 0; k < NB; ++k) so4_fwd(pq[k], v + 4 * k, z + 4 * k);
#pragma unroll
      for (int i = 0; i < E; ++i) qs[h][lane * E + i] = z[i];
    }
    __syncwarp();

    const float sscale = scale / (float)D;  // s = scale * (n/sqrt d) * (qs/sqrt d) . L
    for (int c0 = t0; c0 < t1; c0 += 32) {
      // a7: scores, lane <-> token
      const int tok = c0 + lane;
      const bool valid_t = tok < t1;
      int phys = 0;
      bool ok = false;
      if (valid_t) {
        phys = __ldg(page_table + (size_t)s * max_pages + (tok >> 6));
        ok = phys >= 0 && phys < n_pages;
        if (!ok) set_status(status, ISOQ_ST_PAGE_RANGE);
      }
      float sc[GM];
      float nv = 0.f;
      if (ok) {
        const uint8_t* blk = blocks + ((size_t)phys * H + hk) * BB;
        const int slot = tok & (kPage - 1);
        const uint32_t* rec = reinterpret_cast<const uint32_t*>(blk + slot * CB);
        const float nk = __half2float(
            __ushort_as_half(*reinterpret_cast<const uint16_t*>(blk + k_norm_off(D) + 2 * slot)));
        nv = __half2float(
            __ushort_as_half(*reinterpret_cast<const uint16_t*>(blk + v_norm_off(D) + 2 * slot)));
        float dot[GM];
#pragma unroll
        for (int h = 0; h < GM; ++h) dot[h] = 0.f;
        for (int g = 0; g < D / 32; ++g) {
          const uint32_t w0 = __ldg(rec + 3 * g), w1 = __ldg(rec + 3 * g + 1),
                         w2 = __ldg(rec + 3 * g + 2);
#pragma unroll 8
          for (int e = 0; e < 32; ++e) {
            const float L = lev[group_code(w0, w1, w2, e)];
#pragma unroll
            for (int h = 0; h < GM; ++h)
              if (h < G) dot[h] = fmaf(qs[h][32 * g + e], L, dot[h]);
          }
        }
#pragma unroll
        for (int h = 0; h < GM; ++h) sc[h] = dot[h] * sscale * nk;
      } else {
#pragma unroll
        for (int h = 0; h < GM; ++h) sc[h] = -CUDART_INF_F;
      }

      // a8: online softmax over the chunk; weights p * n^V to shared memory
#pragma unroll
      for (int h = 0; h < GM; ++h) {
        if (h >= G) break;
        const float cm = warp_max(sc[h]);
        const float mn = fmaxf(m[h], cm);
        if (mn == -CUDART_INF_F) {  // nothing valid yet
          pw[h][lane] = 0.f;
          continue;
        }
        const float alpha = __expf(m[h] - mn);
        const float p = ok ? __expf(sc[h] - mn) : 0.f;
        l[h] = l[h] * alpha + warp_sum(p);
#pragma unroll
        for (int i = 0; i < E; ++i) acc[h][i] *= alpha;
        m[h] = mn;
        pw[h][lane] = p * nv;
      }
      __syncwarp();

      // a8: value accumulation, lane <-> E dims, over the chunk's tokens
      const unsigned okmask = __ballot_sync(kFull, ok);
      for (int j = 0; j < 32; ++j) {
        if (!((okmask >> j) & 1u)) continue;
        const int tj = c0 + j;
        const int pj = __shfl_sync(kFull, phys, j);
        const uint8_t* blk = blocks + ((size_t)pj * H + hk) * BB;
        int cv[E];
        lane_codes<E>(blk + v_codes_off(D) + (tj & (kPage - 1)) * CB, lane, cv);
        float Lv[E];
#pragma unroll
        for (int i = 0; i < E; ++i) Lv[i] = lev[cv[i]];
#pragma unroll
        for (int h = 0; h < GM; ++h) {
          if (h < G) {
            const float wgt = pw[h][j];
#pragma unroll
            for (int i = 0; i < E; ++i) acc[h][i] = fmaf(wgt, Lv[i], acc[h][i]);
          }
        }
      }
      __syncwarp();
    }
  }

  // partial for each head of the group: acc[d] (rotated, times sqrt d), m, l
#pragma unroll
  for (int h = 0; h < GM; ++h) {
    if (h >= G) break;
    float* o = partials + (((size_t)s * n_q_heads + hk * G + h) * n_splits + split) * PS;
#pragma unroll
    for (int i = 0; i < E; ++i) o[lane * E + i] = acc[h][i];
    if (lane == 0) {
      o[D] = m[h];
      o[D + 1] = l[h];
    }
  }
}

// a9: merge the splits of one (sequence, query head), normalise, inverse SO(4) blocks and
// inverse (orthonormal, self-inverse) WHT.  One CTA of 128 threads per (sequence, head):
// the splits are spread over 4 groups of 32 lanes (each lane 4 or 8 dims, 16-byte loads,
// several splits in flight), so the merge costs a few memory round trips however many
// splits there are; warp 0 then applies the inverse rotation.
template <int D>
__global__ void __launch_bounds__(128)
    decode_combine_kernel(const float* __restrict__ params, int H, int n_q_heads, int n_splits,
                          const float* __restrict__ partials, float* __restrict__ out) {
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
  const float* base = partials + ((size_t)s * n_q_heads + h) * n_splits * PS;

  // global max of the splits' running maxima (empty splits report -inf)
  float M = -CUDART_INF_F;
  for (int j = tid; j < n_splits; j += 128) M = fmaxf(M, __ldg(base + (size_t)j * PS + D));
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
        const float* p = base + (size_t)(j + 4 * u) * PS;
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
      const float* p = base + (size_t)j * PS;
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
  const float inv = Ls > 0.f ? 1.f / (Ls * sqrtf((float)D)) : 0.f;
  float o[E];
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const int dd = lane * E + i;
    o[i] = (red_acc[0][dd] + red_acc[1][dd] + red_acc[2][dd] + red_acc[3][dd]) * inv;
  }
  const float* hp = params + (size_t)(h / G) * D * 2;
  float y[E];
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    float pq[8];
    load_block_params(hp, lane * NB + k, pq);
    so4_inv(pq, o + 4 * k, y + 4 * k);
  }
  wht_warp<E>(y, lane);
  const float r = rsqrtf((float)D);
  float* dst = out + ((size_t)s * n_q_heads + h) * D + lane * E;
#pragma unroll
  for (int i = 0; i < E; ++i) dst[i] = y[i] * r;
}

template <int D, int GM, typename TQ>
static cudaError_t launch_split(const DecodeArgs& a, cudaStream_t stream) {
  dim3 grid(a.n_splits, a.n_kv_heads, a.n_seqs);
  decode_split_kernel<D, GM, TQ><<<grid, 32, 0, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_kv_heads,
      static_cast<const TQ*>(a.Q), a.n_q_heads, a.seq_lens, a.scale, a.pages_per_split,
      a.n_splits, a.partials, a.status);
  return cudaGetLastError();
}

template <int D, typename TQ>
static cudaError_t launch_g(const DecodeArgs& a, cudaStream_t stream) {
  const int G = a.n_q_heads / a.n_kv_heads;
  if (G <= 1) return launch_split<D, 1, TQ>(a, stream);
  if (G <= 2) return launch_split<D, 2, TQ>(a, stream);
  if (G <= 4) return launch_split<D, 4, TQ>(a, stream);
  if (G <= 8) return launch_split<D, 8, TQ>(a, stream);
  return launch_split<D, 16, TQ>(a, stream);
}

template <int D>
static cudaError_t launch_dq(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e = (kUseTc128 && D == 128) ? launch_decode_split_tc(a, stream)
                                           : launch_decode_split_mma(a, stream);
  if (e != cudaSuccess) return e;
  dim3 grid(a.n_q_heads, a.n_seqs);
  decode_combine_kernel<D><<<grid, 128, 0, stream>>>(a.params, a.n_kv_heads, a.n_q_heads,
                                                    a.n_splits, a.partials, a.out);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  if (a.n_seqs == 0 || a.n_q_heads == 0) return cudaSuccess;
  if (a.d == 128) return launch_dq<128>(a, stream);
  if (a.d == 256) return launch_dq<256>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace isoq
