// Quantize-append kernel: WHT -> SO(4) blocks -> 3-bit codes -> packed paged cache.
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: each K/V vector goes through a Walsh-Hadamard
// transform, then block-diagonal SO(4) rotations, then a 3-bit scalar quantiser, at
// O(d log d) cost per vector.
//
// One warp per (token, KV head); it quantises the K vector and then the V vector, which
// share the head's rotation parameters.  Lane l holds elements E*l .. E*l+E-1 (E = d/32),
// which makes the WHT's first log2(E) butterfly stages lane-local and the remaining five
// __shfl_xor_sync stages; the lane's E elements are exactly its E/4 quaternion blocks, so
// the SO(4) step is lane-local too.  The norm is a warp sum of squares.  Codes are counted
// against the 7 thresholds scaled by the norm (no division), packed with shuffles into the
// 12-byte group layout of isoq.h and written as 16-byte stores.
#include "isoq_common.cuh"
#include "isoq_internal.h"

namespace isoq {

template <int D, typename T>
__global__ void __launch_bounds__(256)
    quantize_append_kernel(const float* __restrict__ params, uint8_t* __restrict__ blocks,
                           const int32_t* __restrict__ page_table, int n_pages, int max_pages,
                           int n_seqs, int H, const T* __restrict__ K, const T* __restrict__ V,
                           int n_tokens, const int32_t* __restrict__ seq_ids,
                           const int32_t* __restrict__ positions, uint32_t* status) {
  constexpr int E = D / 32;       // elements per lane
  constexpr int NB = E / 4;       // quaternion blocks per lane
  constexpr int CB = code_bytes(D);
  constexpr int BB = block_bytes(D);
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const long long total = (long long)n_tokens * H;
  const long long stride = (long long)gridDim.x * wpb;

  for (long long w = (long long)blockIdx.x * wpb + (threadIdx.x >> 5); w < total; w += stride) {
    const int t = (int)(w / H);
    const int h = (int)(w - (long long)t * H);
    const int sid = __ldg(seq_ids + t);
    const int pos = __ldg(positions + t);
    uint32_t bad = 0;
    int phys = -1;
    if (sid < 0 || sid >= n_seqs) {
      bad = ISOQ_ST_SEQ_RANGE;
    } else if (pos < 0 || (pos >> 6) >= max_pages) {
      bad = ISOQ_ST_POS_RANGE;
    } else {
      phys = __ldg(page_table + (size_t)sid * max_pages + (pos >> 6));
      if (phys < 0 || phys >= n_pages) bad = ISOQ_ST_PAGE_RANGE;
    }
    if (bad) {
      if (lane == 0) set_status(status, bad);
      continue;
    }
    uint8_t* blk = blocks + ((size_t)phys * H + h) * BB;
    const int slot = pos & (kPage - 1);

    float pq[NB][8];
#pragma unroll
    for (int k = 0; k < NB; ++k) load_block_params(params + (size_t)h * D * 2, lane * NB + k, pq[k]);

#pragma unroll
    for (int kind = 0; kind < 2; ++kind) {
      const T* src = (kind == 0 ? K : V) + ((size_t)t * H + h) * D + lane * E;
      float v[E];
      load_vec<T, E>(src, v);

      float ss = 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) ss = fmaf(v[i], v[i], ss);
      const float n = sqrtf(warp_sum(ss));

      // y = H x (unnormalised), z = blocks(y) = sqrt(d) * (rotated unit-scale vector)
      wht_warp<E>(v, lane);
      float z[E];
#pragma unroll
      for (int k = 0; k < NB; ++k) so4_fwd(pq[k], v + 4 * k, z + 4 * k);

      // code = #{j : sqrt(d) z_i >= n t_j}; zero vector -> 4
      float nt[7];
#pragma unroll
      for (int j = 0; j < 7; ++j) nt[j] = n * threshold_f32(j);
      uint32_t nib = 0;  // this lane's codes, one per nibble
#pragma unroll
      for (int i = 0; i < E; ++i) {
        uint32_t c = 0;
#pragma unroll
        for (int j = 0; j < 7; ++j) c += (z[i] >= nt[j]) ? 1u : 0u;
        if (n == 0.f) c = 4;
        nib |= c << (4 * i);
      }

      // Assemble the 12-byte groups.  val = direct part of word j of the lane's group for
      // lanes that own one, N = the nibble word of the group's 8 trailing codes.
      uint32_t val;
      uint32_t word;
      if constexpr (E == 4) {
        const int r = lane & 7;
        uint32_t half = nib << (16 * (r & 1));
        val = half | __shfl_xor_sync(kFull, half, 1);         // lanes 2j,2j+1: w_j; 6,7: N
        const uint32_t N = __shfl_sync(kFull, val, (lane & ~7) | 6);
        const int j = r >> 1;                                   // valid for r in {0,2,4}
        word = val | (((N >> (2 - (j < 3 ? j : 0))) & 0x11111111u) << 3);
      } else {
        const int r = lane & 3;
        val = nib;                                              // lanes r<3: w_r; r=3: N
        const uint32_t N = __shfl_sync(kFull, val, (lane & ~3) | 3);
        const int j = r;
        word = val | (((N >> (2 - (j < 3 ? j : 0))) & 0x11111111u) << 3);
      }
      // record word m lives on lane src(m); gather 4 words per storing lane
      uint32_t q4[4];
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4) {
        const int m = (4 * lane + r4) % (CB / 4);
        const int src_lane = (E == 4) ? (8 * (m / 3) + 2 * (m % 3)) : (4 * (m / 3) + (m % 3));
        q4[r4] = __shfl_sync(kFull, word, src_lane);
      }
      uint8_t* dst = blk + (kind == 0 ? 0 : v_codes_off(D)) + slot * CB;
      if (lane < CB / 16)
        *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(q4[0], q4[1], q4[2], q4[3]);

      if (lane == 0) {
        __half hn = __float2half_rn(n);
        uint16_t nb = __half_as_ushort(hn);
        if ((nb & 0x7fffu) == 0x7c00u) {  // overflowed binary16
          nb = 0x7bffu;
          set_status(status, ISOQ_ST_NORM_SAT);
        }
        *reinterpret_cast<uint16_t*>(blk + (kind == 0 ? k_norm_off(D) : v_norm_off(D)) +
                                     2 * slot) = nb;
      }
    }
  }
}

template <int D, typename T>
static cudaError_t launch_t(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  const long long warps = (long long)a.n_tokens * a.n_kv_heads;
  const int wpb = 8;
  long long grid = (warps + wpb - 1) / wpb;
  const long long cap = (long long)n_sm * 32;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  quantize_append_kernel<D, T><<<(unsigned)grid, wpb * 32, 0, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_seqs, a.n_kv_heads,
      static_cast<const T*>(a.K), static_cast<const T*>(a.V), a.n_tokens, a.seq_ids, a.positions,
      a.status);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_d(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  switch (a.dtype) {
    case ISOQ_F32: return launch_t<D, float>(a, stream, n_sm);
    case ISOQ_BF16: return launch_t<D, __nv_bfloat16>(a, stream, n_sm);
    case ISOQ_F16: return launch_t<D, __half>(a, stream, n_sm);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_append(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  if (a.n_tokens == 0) return cudaSuccess;
  if (a.d == 128) return launch_d<128>(a, stream, n_sm);
  if (a.d == 256) return launch_d<256>(a, stream, n_sm);
  return cudaErrorInvalidValue;
}

}  // namespace isoq
