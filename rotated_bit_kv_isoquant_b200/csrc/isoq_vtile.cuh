// The 3-bit V tile layout of a page's V codes (include/isoq.h, "3-bit V tile layout").
//
// The V region of a (page, KV head) block holds 4 blocks of 16 token slots, 6 d bytes
// each.  In block B, quad t (0..3) is the slots 16B + 2t + {0, 1, 8, 9} (member j = slot
// bits 3 and 0), and unit u is dims 8u .. 8u+7.  The 12-byte group of (quad t, unit u)
// sits at byte ((u >> 1) * 8 + 2t + (u & 1)) * 12 of the block; in its word b (0..2),
// nibble n (bits 4n .. 4n+2) is the code of member n & 3 at dim 8u + 2b + (n >> 2), and
// bit 4n+3 is bit 2-b of the code of member n & 3 at dim 8u + 6 + (n >> 2).  So the low
// and the high 16 bits of a word are each four tokens' codes of one dim: one byte-permute
// selector for a tensor-core operand register of four tokens.
//
// The quantisers produce, per vector, the "unit words" U of its units: nibble e of U_u
// is the code of dim 8u + e (bit 3 of every nibble clear).
#pragma once

#include <stdint.h>

#include "isoq_check.cuh"
#include "isoq_common.cuh"

namespace isoq {

// Byte offset of group (quad t, unit u) of block B inside a V region, head dimension D.
__host__ __device__ constexpr int vt_group_off(int D, int B, int t, int u) {
  return B * 6 * D + ((u >> 1) * 8 + 2 * t + (u & 1)) * 12;
}

// Slot (0..63) -> block B, quad t and member j.
__device__ __forceinline__ void vt_slot(int slot, int& B, int& t, int& j) {
  B = slot >> 4;
  t = (slot >> 1) & 3;
  j = (slot & 1) | ((slot >> 2) & 2);
}

// Slot of member j of quad t in block B.
__host__ __device__ constexpr int vt_member_slot(int B, int t, int j) {
  return 16 * B + 2 * t + (j & 1) + 8 * (j >> 1);
}

__device__ __forceinline__ uint32_t vt_prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Nibbles (L0 H0 L1 H1 L2 H2 L3 H3) -> (L0 L1 L2 L3 H0 H1 H2 H3) (nibble 0 lowest).
__device__ __forceinline__ uint32_t vt_unshuffle(uint32_t x) {
  const uint32_t t = (x ^ (x >> 4)) & 0x00F000F0u;  // swap nibbles 1 <-> 2 and 5 <-> 6
  x = x ^ t ^ (t << 4);
  return vt_prmt(x, 0u, 0x3120u);                   // swap bytes 1 and 2
}

// The three words of the group of one unit from the four members' unit words U0..U3.
__device__ __forceinline__ void vt_group_words(uint32_t U0, uint32_t U1, uint32_t U2, uint32_t U3,
                                               uint32_t (&W)[3]) {
  // byte transpose: T_k byte j = byte k of U_j (dims 2k, 2k+1 of member j)
  const uint32_t A01 = vt_prmt(U0, U1, 0x5140u), A23 = vt_prmt(U2, U3, 0x5140u);
  const uint32_t B01 = vt_prmt(U0, U1, 0x7362u), B23 = vt_prmt(U2, U3, 0x7362u);
  const uint32_t T0 = vt_prmt(A01, A23, 0x5410u), T1 = vt_prmt(A01, A23, 0x7632u);
  const uint32_t T2 = vt_prmt(B01, B23, 0x5410u), T3 = vt_prmt(B01, B23, 0x7632u);
  // words 0..2 (dims 0..5) and the spare unit (dims 6, 7) as clean nibble words
  const uint32_t N = vt_unshuffle(T3);
  W[0] = vt_unshuffle(T0) | ((N << 1) & 0x88888888u);
  W[1] = vt_unshuffle(T1) | ((N << 2) & 0x88888888u);
  W[2] = vt_unshuffle(T2) | ((N << 3) & 0x88888888u);
}

// The bits of member j alone in the three words of its group (the other members' bits
// zero) and the mask of member j's bits (the same in each word).
__device__ __forceinline__ void vt_member_words(uint32_t U, int j, uint32_t (&W)[3],
                                                uint32_t& mask) {
  vt_group_words(j == 0 ? U : 0u, j == 1 ? U : 0u, j == 2 ? U : 0u, j == 3 ? U : 0u, W);
  mask = 0x000F000Fu << (4 * j);
}

// Writes the 3-bit V codes of a warp's vectors into the V tile layout.  Lane L holds a
// vector of KV head h (token: sequence sid, position pos, physical page phys; phys < 0 =
// nothing to write) whose D/8 unit words are in warp_stage + L * SW.  A half-warp whose 16
// lanes hold slots 16B .. 16B+15 of one page in lane order (the prefill case) assembles
// that block's groups and stores them whole; any other valid vector clears and sets its
// own bits with atomics (a decode step's appends, unaligned ranges).  All 32 lanes call
// this, after their unit words are in shared memory and a __syncwarp.
template <int D, int SW>
__device__ __forceinline__ void vt_store_warp(const uint32_t* warp_stage, int lane, int sid,
                                              int pos, int phys, uint8_t* blocks, int H, int h,
                                              uint32_t* status = nullptr) {
  constexpr int BB = block_bytes(D, 3);
  constexpr int NU = D / 8;  // units
  const int hb = lane & 16, hl = lane & 15;  // half-warp base lane, position in it
  const int s0 = __shfl_sync(kFull, sid, hb), p0 = __shfl_sync(kFull, pos, hb);
  const int ph0 = __shfl_sync(kFull, phys, hb);
  const bool in_order = phys >= 0 && sid == s0 && pos == p0 + hl && (p0 & 15) == 0 && phys == ph0;
  const unsigned hmask = 0xFFFFu << hb;
  const bool whole = (__ballot_sync(kFull, in_order) & hmask) == hmask;
  if (whole) {
    // lane hl builds quad t = hl & 3, units 4m .. 4m+3 for m = hl >> 2 (+ 4 per D/128)
    const int t = hl & 3;
    const uint32_t* st = warp_stage + hb * SW;
    uint8_t* vb = blocks + ((size_t)phys * H + h) * BB + v_codes_off(D, 3) +
                  vt_group_off(D, (p0 & (kPage - 1)) >> 4, 0, 0);
#pragma unroll
    for (int m = hl >> 2; m < NU / 4; m += 4) {
      if (!in_bounds(4 * m + 4 <= SW && h < H && vt_group_off(D, 0, t, 4 * m + 3) + 12 <= 6 * D,
                     status))
        continue;
      uint4 U[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        U[j] = *reinterpret_cast<const uint4*>(st + vt_member_slot(0, t, j) * SW + 4 * m);
      uint32_t W[4][3];
      vt_group_words(U[0].x, U[1].x, U[2].x, U[3].x, W[0]);
      vt_group_words(U[0].y, U[1].y, U[2].y, U[3].y, W[1]);
      vt_group_words(U[0].z, U[1].z, U[2].z, U[3].z, W[2]);
      vt_group_words(U[0].w, U[1].w, U[2].w, U[3].w, W[3]);
      // units (4m, 4m+1) and (4m+2, 4m+3) are two 24-byte runs, 8-byte aligned
      uint2* a = reinterpret_cast<uint2*>(vb + vt_group_off(D, 0, t, 4 * m));
      uint2* b = reinterpret_cast<uint2*>(vb + vt_group_off(D, 0, t, 4 * m + 2));
      a[0] = make_uint2(W[0][0], W[0][1]);
      a[1] = make_uint2(W[0][2], W[1][0]);
      a[2] = make_uint2(W[1][1], W[1][2]);
      b[0] = make_uint2(W[2][0], W[2][1]);
      b[1] = make_uint2(W[2][2], W[3][0]);
      b[2] = make_uint2(W[3][1], W[3][2]);
    }
  } else if (phys >= 0) {
    int B, t, j;
    vt_slot(pos & (kPage - 1), B, t, j);
    uint8_t* vb = blocks + ((size_t)phys * H + h) * BB + v_codes_off(D, 3);
    const uint32_t* mine = warp_stage + lane * SW;
#pragma unroll 4
    for (int u = 0; u < NU; ++u) {
      uint32_t W[3], mask;
      vt_member_words(mine[u], j, W, mask);
      uint32_t* g = reinterpret_cast<uint32_t*>(vb + vt_group_off(D, B, t, u));
      if (!in_bounds(u < SW && h < H && vt_group_off(D, B, t, u) + 12 <= kPage * code_bytes(D, 3),
                     status))
        continue;
#pragma unroll
      for (int w = 0; w < 3; ++w) {
        atomicAnd(g + w, ~mask);
        atomicOr(g + w, W[w]);
      }
    }
  }
}

}  // namespace isoq
