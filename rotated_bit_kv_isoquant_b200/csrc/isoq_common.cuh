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

// Variants of the same family (Max 1960, Table I): 4 levels (2 bits) and 16 levels
// (4 bits), ascending; only the non-negative halves are stored (the codebooks are
// symmetric).  mag_f32(bits, k) = level 2^(bits-1) + k.
__host__ __device__ constexpr float mag_f32(int bits, int k) {
  return bits == 2 ? (k == 0 ? 0.4528f : 1.5104f)
         : bits == 4
             ? (k == 0   ? 0.1284f
                : k == 1 ? 0.3881f
                : k == 2 ? 0.6568f
                : k == 3 ? 0.9424f
                : k == 4 ? 1.2562f
                : k == 5 ? 1.6180f
                : k == 6 ? 2.0690f
                         : 2.7326f)
             : level_f32(4 + k);
}
__host__ __device__ constexpr float level_f32(int bits, int c) {
  return c >= (1 << (bits - 1)) ? mag_f32(bits, c - (1 << (bits - 1)))
                                : -mag_f32(bits, (1 << (bits - 1)) - 1 - c);
}
// Positive decision thresholds: midpoint of magnitudes k and k+1 (k = 0 .. 2^(bits-1)-2),
// computed in double and rounded once to binary32 (3 bits: the decimal 0.50055, 1.05,
// 1.748 of threshold_f32).
__host__ __device__ constexpr float pos_threshold_f32(int bits, int k) {
  return bits == 3 ? threshold_f32(4 + k)
                   : (float)(0.5 * ((double)mag_f32(bits, k) + (double)mag_f32(bits, k + 1)));
}

// Bytes of packed codes per vector and per (page, head) block; offsets inside a block.
__host__ __device__ constexpr int code_bytes(int D, int bits = 3) { return bits * D / 8; }
__host__ __device__ constexpr int block_bytes(int D, int bits = 3) {
  return 2 * kPage * (code_bytes(D, bits) + 2);
}
__host__ __device__ constexpr int k_norm_off(int D, int bits = 3) {
  return kPage * code_bytes(D, bits);
}
__host__ __device__ constexpr int v_codes_off(int D, int bits = 3) {
  return kPage * (code_bytes(D, bits) + 2);
}
__host__ __device__ constexpr int v_norm_off(int D, int bits = 3) {
  return kPage * (code_bytes(D, bits) + 2) + kPage * code_bytes(D, bits);
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

// The rotation blocks of a head as 4x4 row-major matrices (one per 4 dims: an SO(4)
// block p y conj(q), or two SO(2) blocks on the diagonal), derived from the parameters in
// binary64 when the parameter handle is made.  head_mats = mats + head * (d / 4) * 16.
__device__ __forceinline__ void load_block_mat(const float* __restrict__ head_mats, int b,
                                               float (&M)[16]) {
  const float4* s = reinterpret_cast<const float4*>(head_mats + 16 * b);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float4 v = __ldg(s + r);
    M[4 * r + 0] = v.x;
    M[4 * r + 1] = v.y;
    M[4 * r + 2] = v.z;
    M[4 * r + 3] = v.w;
  }
}

// z = M y (forward block rotation).
__device__ __forceinline__ void mat_fwd(const float (&M)[16], const float* y, float* z) {
#pragma unroll
  for (int r = 0; r < 4; ++r)
    z[r] = fmaf(M[4 * r + 3], y[3], fmaf(M[4 * r + 2], y[2], fmaf(M[4 * r + 1], y[1], M[4 * r] * y[0])));
}

// y = M^T z (inverse block rotation: the blocks are orthogonal).
__device__ __forceinline__ void mat_inv(const float (&M)[16], const float* z, float* y) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    y[c] = fmaf(M[12 + c], z[3], fmaf(M[8 + c], z[2], fmaf(M[4 + c], z[1], M[c] * z[0])));
}

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

}  // namespace isoq
