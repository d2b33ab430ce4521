// PTX helpers shared by the decode kernels: mma.sync / movmatrix, mbarriers and bulk
// copies, byte-permute dequantisation of packed codes into f16 operands.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "isoq_common.cuh"

namespace isoq {
namespace ptx {


constexpr float kAlpha = 3618.98939633f;  // level scale with near-exact binary16 levels
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;          // rescale the running max only when it grows by 2^8
constexpr float kSigmaSlack = 16.0f;   // ... and the V-norm reference when it grows 16x
constexpr int kWarps = 4;
constexpr unsigned kWaitLimit = 1u << 24;  // bounded mbarrier polls (~seconds)

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// 2^x with the hardware approximation (relative error ~2^-22; -inf -> 0).
__device__ __forceinline__ float ex2(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Packed pairs of binary32 operations (one instruction each, the same per-lane rounding
// as the scalar forms): a * b + c, a * b, a + b.
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) {
  float2 o;
  asm("{\n .reg .b64 pa, pb, pc, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
      " mov.b64 pc, {%6, %7};\n fma.rn.f32x2 pd, pa, pb, pc;\n mov.b64 {%0, %1}, pd;\n}"
      : "=f"(o.x), "=f"(o.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return o;
}
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) {
  float2 o;
  asm("{\n .reg .b64 pa, pb, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
      " mul.rn.f32x2 pd, pa, pb;\n mov.b64 {%0, %1}, pd;\n}"
      : "=f"(o.x), "=f"(o.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return o;
}
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) {
  float2 o;
  asm("{\n .reg .b64 pa, pb, pd;\n mov.b64 pa, {%2, %3};\n mov.b64 pb, {%4, %5};\n"
      " add.rn.f32x2 pd, pa, pb;\n mov.b64 {%0, %1}, pd;\n}"
      : "=f"(o.x), "=f"(o.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return o;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Polls the phase with the given parity; false if it did not complete within `limit` polls
// (the kernels use kWaitLimit; a self-test uses a short limit to exercise the give-up path).
__device__ __forceinline__ bool mbar_wait_n(uint64_t* bar, unsigned parity, unsigned limit) {
  const uint32_t a = smem_u32(bar);
  for (unsigned i = 0; i < limit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity) {
  return mbar_wait_n(bar, parity, kWaitLimit);
}

__device__ __forceinline__ void bulk_copy(void* dst, const void* src, unsigned bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Spare codes of a group: bit (2-b) of code 24+k is bit 4k+3 of w_b -> nibble k.
__device__ __forceinline__ uint32_t spare_codes(uint32_t w0, uint32_t w1, uint32_t w2) {
  return ((w2 & 0x88888888u) >> 3) | ((w1 & 0x88888888u) >> 2) | ((w0 & 0x88888888u) >> 1);
}

// The three words of group q of a packed vector -> four 8-nibble selector words:
// S[j] nibble n = code of dim 32q + 8j + n (bit 3 of every nibble clear).
__device__ __forceinline__ void selectors(uint32_t w0, uint32_t w1, uint32_t w2,
                                          uint32_t (&S)[4]) {
  S[0] = w0 & 0x77777777u;
  S[1] = w1 & 0x77777777u;
  S[2] = w2 & 0x77777777u;
  S[3] = spare_codes(w0, w1, w2);
}

// Eight f16 values of the nibbles of S: o[i] = (level(nibble 2i), level(nibble 2i+1)).
__device__ __forceinline__ void deq8(uint32_t S, uint32_t tl0, uint32_t tl1, uint32_t th0,
                                     uint32_t th1, uint32_t (&o)[4]) {
  uint32_t lo = prmt(tl0, tl1, S);
  uint32_t hi = prmt(th0, th1, S);
  o[0] = prmt(lo, hi, 0x5140);
  o[1] = prmt(lo, hi, 0x7362);
  const uint32_t S2 = S >> 16;
  lo = prmt(tl0, tl1, S2);
  hi = prmt(th0, th1, S2);
  o[2] = prmt(lo, hi, 0x5140);
  o[3] = prmt(lo, hi, 0x7362);
}

// Token pair (a, b), selector words Sa, Sb of the same dims: o[i] = (level a, level b) of
// nibble 4 part + i (i = 0..3), i.e. an f16x2 of two tokens for one dim.
__device__ __forceinline__ void deq4_pair(uint32_t Sa, uint32_t Sb, int part, uint32_t tl0,
                                          uint32_t tl1, uint32_t th0, uint32_t th1,
                                          uint32_t (&o)[4]) {
  // nibbles (a n, a n+1, b n, b n+1, a n+2, a n+3, b n+2, b n+3) with n = 4 part
  const uint32_t X = prmt(Sa, Sb, part == 0 ? 0x5140u : 0x7362u);
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const uint32_t sel = hh == 0 ? X : X >> 16;
    const uint32_t lo = prmt(tl0, tl1, sel);
    const uint32_t hi = prmt(th0, th1, sel);
    o[2 * hh + 0] = prmt(lo, hi, 0x6240);
    o[2 * hh + 1] = prmt(lo, hi, 0x7351);
  }
}

// ---- per-format dequantisation ---------------------------------------------------------
// A 32-dim group of a packed vector is BITS little-endian words; it splits into four
// "units" of 8 dims (dims 8u..8u+7).  kdeq<BITS> turns unit u of a token into four f16x2
// (dims 8u+2i, 8u+2i+1) -- a K fragment; vdeq<BITS> turns the same unit of two tokens a, b
// into four f16x2 (a, b) of dims 8u + 4 part + i -- a V fragment.  Values are ALPHA(BITS)
// times the level.  ALPHA is chosen so that every level magnitude is (nearly) exact in
// binary16: relative error < 2e-5 (3 bits), exact (2 bits), < 6e-5 (4 bits).
template <int BITS>
constexpr float alpha_of() { return BITS == 3 ? kAlpha : (BITS == 2 ? 7500.0f : 5992.94213044f); }

// Level-byte tables.  3 bits: lo/hi bytes of the 8 levels (tl0,tl1 | th0,th1); 4 bits:
// of the 8 magnitudes; 2 bits: tl0 = low bytes of the 4 levels, th0 = high bytes.
template <int BITS>
__device__ __forceinline__ void level_tables(uint32_t& tl0, uint32_t& tl1, uint32_t& th0,
                                             uint32_t& th1) {
  tl0 = tl1 = th0 = th1 = 0;
  constexpr int N = BITS == 2 ? 4 : 8;
#pragma unroll
  for (int c = 0; c < N; ++c) {
    const float v = BITS == 4 ? mag_f32(4, c) : level_f32(BITS, c);
    const uint32_t hbits = __half_as_ushort(__float2half_rn(alpha_of<BITS>() * v));
    const uint32_t lo = hbits & 0xffu, hi = hbits >> 8;
    if (c < 4) {
      tl0 |= lo << (8 * c);
      th0 |= hi << (8 * c);
    } else {
      tl1 |= lo << (8 * (c - 4));
      th1 |= hi << (8 * (c - 4));
    }
  }
}

// 4 bits: flip the f16 sign of o (values of nibbles n, n') where the selected sign bits
// (bit 3 of the nibbles, replicated by prmt's sign mode from S / S << 4) are set.
__device__ __forceinline__ uint32_t apply_sign(uint32_t o, uint32_t S, uint32_t S4, uint32_t sel) {
  return o ^ (prmt(S, S4, sel) & 0x80008000u);
}

// 2 bits: f16x2 of the codes in bits 0-1 and 8-9 of x (the rest of the low 16 bits zero):
// selector nibbles (c0, 4 + c0, c1, 4 + c1) on the pool (low bytes | high bytes).
__device__ __forceinline__ uint32_t deq2(uint32_t x, uint32_t tl0, uint32_t th0) {
  return prmt(tl0, th0, x * 0x11u + 0x4040u);
}

template <int BITS>
__device__ __forceinline__ void kdeq(const uint32_t* w, int u, uint32_t tl0, uint32_t tl1,
                                     uint32_t th0, uint32_t th1, uint32_t (&o)[4]) {
  if constexpr (BITS == 3) {
    const uint32_t S = u < 3 ? (w[u] & 0x77777777u) : spare_codes(w[0], w[1], w[2]);
    deq8(S, tl0, tl1, th0, th1, o);
  } else if constexpr (BITS == 4) {
    const uint32_t S = w[u], S4 = S << 4;
    deq8(S & 0x77777777u, tl0, tl1, th0, th1, o);
    o[0] = apply_sign(o[0], S, S4, 0x80C0u);
    o[1] = apply_sign(o[1], S, S4, 0x90D0u);
    o[2] = apply_sign(o[2], S, S4, 0xA0E0u);
    o[3] = apply_sign(o[3], S, S4, 0xB0F0u);
  } else {
    const uint32_t U = w[u >> 1] >> (16 * (u & 1));  // slots 0..7 of the unit
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = deq2((U >> (2 * i)) & 0x0303u, tl0, th0);
  }
}

template <int BITS>
__device__ __forceinline__ void vdeq(uint32_t Sa, uint32_t Sb, int part, uint32_t tl0,
                                     uint32_t tl1, uint32_t th0, uint32_t th1,
                                     uint32_t (&o)[4]) {
  if constexpr (BITS == 3) {
    deq4_pair(Sa, Sb, part, tl0, tl1, th0, th1, o);
  } else if constexpr (BITS == 4) {
    const uint32_t X = prmt(Sa, Sb, part == 0 ? 0x5140u : 0x7362u), X4 = X << 4;
    deq4_pair(Sa & 0x77777777u, Sb & 0x77777777u, part, tl0, tl1, th0, th1, o);
    o[0] = apply_sign(o[0], X, X4, 0xD0C0u);
    o[1] = apply_sign(o[1], X, X4, 0x9080u);
    o[2] = apply_sign(o[2], X, X4, 0xF0E0u);
    o[3] = apply_sign(o[3], X, X4, 0xB0A0u);
  } else {
    // units = slots 0..7 in the low 16 bits; M bytes: a slots 0-3, b 0-3, a 4-7, b 4-7
    const uint32_t M = prmt(Sa, Sb, 0x5140u);
    // dims 4 part + i -> slots (2 part, 2 part + 4, 2 part + 1, 2 part + 5)
    o[0] = deq2((M >> (4 * part)) & 0x0303u, tl0, th0);
    o[1] = deq2((M >> (16 + 4 * part)) & 0x0303u, tl0, th0);
    o[2] = deq2((M >> (4 * part + 2)) & 0x0303u, tl0, th0);
    o[3] = deq2((M >> (16 + 4 * part + 2)) & 0x0303u, tl0, th0);
  }
}

// 3-bit V tile layout: the group (W0, W1, W2) of one unit (8 dims) of four member tokens
// -> o[j][i] = f16x2 (dims 2i, 2i+1 of the unit) of member j, the values ALPHA * level.
// The low / high 16 bits of a word are one dim of the four members: one lookup of the
// level's low bytes and one of its high bytes give that dim of all four, then permutes
// regroup them per token.
__device__ __forceinline__ void vdeq_group(uint32_t W0, uint32_t W1, uint32_t W2, uint32_t tl0,
                                           uint32_t tl1, uint32_t th0, uint32_t th1,
                                           uint32_t (&o)[4][4]) {
  const uint32_t Sp = spare_codes(W0, W1, W2);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t S = i == 0 ? (W0 & 0x77777777u)
                     : i == 1 ? (W1 & 0x77777777u)
                     : i == 2 ? (W2 & 0x77777777u)
                              : Sp;
    const uint32_t Sh = S >> 16;
    const uint32_t le = prmt(tl0, tl1, S), he = prmt(th0, th1, S);    // dim 2i, members 0-3
    const uint32_t lo = prmt(tl0, tl1, Sh), ho = prmt(th0, th1, Sh);  // dim 2i + 1
    const uint32_t A01 = prmt(le, he, 0x5140u), A23 = prmt(le, he, 0x7362u);
    const uint32_t B01 = prmt(lo, ho, 0x5140u), B23 = prmt(lo, ho, 0x7362u);
    o[0][i] = prmt(A01, B01, 0x5410u);
    o[1][i] = prmt(A01, B01, 0x7632u);
    o[2][i] = prmt(A23, B23, 0x5410u);
    o[3][i] = prmt(A23, B23, 0x7632u);
  }
}

__device__ __forceinline__ float half_at(const uint8_t* p) {
  return __half2float(__ushort_as_half(*reinterpret_cast<const uint16_t*>(p)));
}


}  // namespace ptx
}  // namespace isoq
