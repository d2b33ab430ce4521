// Device helpers shared by the IsoQuant kernels (quantize-append, decode, combine).
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract -- Walsh-Hadamard transform, block-diagonal SO(4)
// rotations (quaternion pairs), 3-bit scalar quantisation, attention on packed codes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/isoq.h"

namespace isoq {

constexpr int kPage = ISOQ_PAGE_SIZE;
constexpr unsigned kFull = 0xffffffffu;

// Lloyd-Max 8-level quantiser for N(0,1) (J. Max, 1960), ascending; binary32.
__host__ __device__ constexpr float level_f32(int c) {
  return c == 0   ? -2.1520f
         : c == 1 ? -1.3440f
         : c == 2 ? -0.7560f
         : c == 3 ? -0.2451f
         : c == 4 ? 0.2451f
         : c == 5 ? 0.7560f
         : c == 6 ? 1.3440f
                  : 2.1520f;
}

// Decision thresholds: midpoints of adjacent levels (binary32 of the decimal values).
__host__ __device__ constexpr float threshold_f32(int j) {
  return j == 0   ? -1.748f
         : j == 1 ? -1.05f
         : j == 2 ? -0.50055f
         : j == 3 ? 0.0f
         : j == 4 ? 0.50055f
         : j == 5 ? 1.05f
                  : 1.748f;
}

// Bytes of packed codes per vector and per (page, head) block.
__host__ __device__ constexpr int code_bytes(int D) { return 3 * D / 8; }
__host__ __device__ constexpr int block_bytes(int D) { return 2 * kPage * (code_bytes(D) + 2); }
// Offsets inside a block.
__host__ __device__ constexpr int k_norm_off(int D) { return kPage * code_bytes(D); }
__host__ __device__ constexpr int v_codes_off(int D) { return kPage * (code_bytes(D) + 2); }
__host__ __device__ constexpr int v_norm_off(int D) {
  return kPage * (code_bytes(D) + 2) + kPage * code_bytes(D);
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

// Loads E contiguous elements (E = 4 or 8) starting at p into fp32 registers.
template <typename T, int E>
__device__ __forceinline__ void load_vec(const T* __restrict__ p, float (&v)[E]) {
  static_assert(E == 4 || E == 8, "E");
  if constexpr (sizeof(T) == 4) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < E / 4; ++i) {
      float4 f = __ldg(q + i);
      v[4 * i + 0] = f.x;
      v[4 * i + 1] = f.y;
      v[4 * i + 2] = f.z;
      v[4 * i + 3] = f.w;
    }
  } else {
    // 2-byte types: E=4 -> one 8-byte load, E=8 -> one 16-byte load
    if constexpr (E == 4) {
      uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
      const T* e = reinterpret_cast<const T*>(&r);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = to_f32<T>(e[i]);
    } else {
      uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
      const T* e = reinterpret_cast<const T*>(&r);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = to_f32<T>(e[i]);
    }
  }
}

// Unnormalised Walsh-Hadamard transform (natural / Sylvester order) of a d = 32*E vector
// spread over a warp, lane l holding elements E*l .. E*l+E-1.  Butterfly stages of stride
// 1..E/2 run inside the lane; stride E*2^s pairs lane l with lane l ^ 2^s, the lower lane
// keeping a+b and the upper a-b.
template <int E>
__device__ __forceinline__ void wht_warp(float (&v)[E], int lane) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int i = 0; i < E; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const bool upper = (lane >> s) & 1;
#pragma unroll
    for (int j = 0; j < E; ++j) {
      float p = __shfl_xor_sync(kFull, v[j], 1 << s);
      v[j] = upper ? (p - v[j]) : (v[j] + p);
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Hamilton product of quaternions (w, x, y, z).
__device__ __forceinline__ void qmul(const float* a, const float* b, float* o) {
  float w = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
  float x = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
  float y = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
  float z = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
  o[0] = w;
  o[1] = x;
  o[2] = y;
  o[3] = z;
}

// z = p * y * conj(q)  (one SO(4) block).  pq: 8 floats, p then q.
__device__ __forceinline__ void so4_fwd(const float* pq, const float* y, float* z) {
  float t[4];
  qmul(pq, y, t);
  const float qc[4] = {pq[4], -pq[5], -pq[6], -pq[7]};
  qmul(t, qc, z);
}

// y = conj(p) * z * q  (inverse block).
__device__ __forceinline__ void so4_inv(const float* pq, const float* z, float* y) {
  const float pc[4] = {pq[0], -pq[1], -pq[2], -pq[3]};
  float t[4];
  qmul(pc, z, t);
  qmul(t, pq + 4, y);
}

// Loads the 8 parameters (p, q) of block b of one head into registers.
__device__ __forceinline__ void load_block_params(const float* __restrict__ head_params, int b,
                                                  float (&pq)[8]) {
  const float4* s = reinterpret_cast<const float4*>(head_params + 8 * b);
  float4 a = __ldg(s), c = __ldg(s + 1);
  pq[0] = a.x;
  pq[1] = a.y;
  pq[2] = a.z;
  pq[3] = a.w;
  pq[4] = c.x;
  pq[5] = c.y;
  pq[6] = c.z;
  pq[7] = c.w;
}

// Code of one packed element: element e (0..31) of a 12-byte group (w0, w1, w2).
__device__ __forceinline__ int group_code(uint32_t w0, uint32_t w1, uint32_t w2, int e) {
  if (e < 24) {
    uint32_t w = e < 8 ? w0 : (e < 16 ? w1 : w2);
    return (w >> (4 * (e & 7))) & 7;
  }
  int k = e - 24;
  return (((w0 >> (4 * k + 3)) & 1) << 2) | (((w1 >> (4 * k + 3)) & 1) << 1) |
         ((w2 >> (4 * k + 3)) & 1);
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace isoq
