// Quantize-append kernel: WHT -> SO(4) blocks -> 3-bit codes -> packed paged cache.
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: each K/V vector goes through a Walsh-Hadamard
// transform, then block-diagonal SO(4) rotations, then a 3-bit scalar quantiser, at
// O(d log d) cost per vector.
//
// One warp per token: for each KV head it quantises the K and the V vector together (they
// share the head's rotation).  Lane l holds elements E*l .. E*l+E-1 (E = d/32), which makes
// the WHT's first log2(E) butterfly stages lane-local and the remaining five
// __shfl_xor_sync stages (one FFMA each); the lane's E elements are exactly its E/4 SO(4)
// blocks, so the rotation is lane-local too (applied as the block's 4x4 matrix, derived
// from the quaternion pair when the parameters are made).  The norm is a warp sum of
// squares.  Codes are decided against the thresholds scaled by the norm (no division),
// packed with shuffles into the 12-byte group layout of isoq.h and written as 16-byte
// stores.
#include <math_constants.h>

#include "isoq_check.cuh"
#include "isoq_codes.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_vtile.cuh"

namespace isoq {

// One warp per token; it walks the KV heads and, per head, quantises K and V together
// (two independent chains for the scheduler).  Each head's loads and shuffle stages are
// latency chains, so the register budget is set for 4 CTAs (32 warps) per SM: 64
// registers with a few spilled words, 20% faster at d = 256 than 80 registers and 3 CTAs.
template <int D, typename T>
__global__ void __launch_bounds__(256, 4)
    quantize_append_kernel(const __grid_constant__ QuantLayers layers, int H, int n_tokens,
                           const int32_t* __restrict__ seq_ids,
                           const int32_t* __restrict__ positions,
                           const float* __restrict__ rope, int rope_max_pos) {
  const QuantLayer& L = layers.l[blockIdx.y];  // this launch row's layer
  const float* __restrict__ mats = L.mats;
  uint8_t* __restrict__ blocks = L.blocks;
  const int32_t* __restrict__ page_table = L.page_table;
  const int n_pages = L.n_pages, max_pages = L.max_pages, n_seqs = L.n_seqs;
  const T* __restrict__ K = static_cast<const T*>(L.K);
  const T* __restrict__ V = static_cast<const T*>(L.V);
  uint32_t* status = L.status;
  constexpr int E = D / 32;       // elements per lane
  constexpr int NB = E / 4;       // quaternion blocks per lane
  constexpr int CB = code_bytes(D);
  constexpr int BB = block_bytes(D);
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  // butterfly sign of this lane in cross-lane stage s: the lower lane keeps a+b, the upper
  // a-b, i.e. fma(sign, own, partner)
  float bsign[5];
#pragma unroll
  for (int st = 0; st < 5; ++st) bsign[st] = ((lane >> st) & 1) ? -1.f : 1.f;

  for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < n_tokens; t += gridDim.x * wpb) {
    const int sid = __ldg(seq_ids + t);
    const int pos = __ldg(positions + t);
    uint32_t bad = 0;
    int phys = -1;
    if (sid < 0 || sid >= n_seqs) {
      bad = ISOQ_ST_SEQ_RANGE;
    } else if (pos < 0 || (pos >> 6) >= max_pages || (rope && pos >= rope_max_pos)) {
      bad = ISOQ_ST_POS_RANGE;
    } else {
      phys = __ldg(page_table + (size_t)sid * max_pages + (pos >> 6));
      if (phys < 0 || phys >= n_pages) bad = ISOQ_ST_PAGE_RANGE;
    }
    if (bad) {
      if (lane == 0) set_status(status, bad);
      continue;
    }
    const int slot = pos & (kPage - 1);

    if (!in_bounds(phys < n_pages && slot < kPage, status)) continue;
    for (int h = 0; h < H; ++h) {
      uint8_t* blk = blocks + ((size_t)phys * H + h) * BB;
      const size_t row = ((size_t)t * H + h) * D + lane * E;
      float x[2][E];
      load_vec<T, E>(K + row, x[0]);
      load_vec<T, E>(V + row, x[1]);
      if (rope) {  // RoPE of K at its position: dims (i, i + D/2) live on lanes l, l ^ 16
        float pv[E];
#pragma unroll
        for (int j = 0; j < E; ++j) pv[j] = __shfl_xor_sync(kFull, x[0][j], 16);
        const float4* tab = reinterpret_cast<const float4*>(rope + (size_t)pos * D) +
                            (E * (lane & 15)) / 2;
#pragma unroll
        for (int jj = 0; jj < E / 2; ++jj) {
          const float4 cs = __ldg(tab + jj);
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 2 * jj + e;
            const float c = e ? cs.z : cs.x, sn = e ? cs.w : cs.y;
            x[0][j] = lane < 16 ? fmaf(x[0][j], c, -pv[j] * sn) : fmaf(pv[j], sn, x[0][j] * c);
          }
        }
      }

      // a1: norms (both vectors' reductions interleaved)
      float ss[2] = {0.f, 0.f};
#pragma unroll
      for (int i = 0; i < E; ++i) {
        ss[0] = fmaf(x[0][i], x[0][i], ss[0]);
        ss[1] = fmaf(x[1][i], x[1][i], ss[1]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ss[0] += __shfl_xor_sync(kFull, ss[0], o);
        ss[1] += __shfl_xor_sync(kFull, ss[1], o);
      }
      const float n[2] = {sqrtf(ss[0]), sqrtf(ss[1])};

      // a2: unnormalised WHT, natural order; lane-local stages then 5 shuffle stages
#pragma unroll
      for (int hs = 1; hs < E; hs <<= 1) {
#pragma unroll
        for (int i = 0; i < E; i += 2 * hs) {
#pragma unroll
          for (int j = i; j < i + hs; ++j) {
#pragma unroll
            for (int kv = 0; kv < 2; ++kv) {
              const float a = x[kv][j], b = x[kv][j + hs];
              x[kv][j] = a + b;
              x[kv][j + hs] = a - b;
            }
          }
        }
      }
#pragma unroll
      for (int st = 0; st < 5; ++st) {
#pragma unroll
        for (int j = 0; j < E; ++j) {
#pragma unroll
          for (int kv = 0; kv < 2; ++kv) {
            const float pv = __shfl_xor_sync(kFull, x[kv][j], 1 << st);
            x[kv][j] = fmaf(bsign[st], x[kv][j], pv);
          }
        }
      }

      // a3: SO(4) blocks as 4x4 matrices (z = M y), this lane's blocks of head h
      float z[2][E];
#pragma unroll
      for (int k = 0; k < NB; ++k) {
        const float4* mp = reinterpret_cast<const float4*>(mats + ((size_t)h * (D / 4) + lane * NB + k) * 16);
        float M[16];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 v = __ldg(mp + r);
          M[4 * r + 0] = v.x;
          M[4 * r + 1] = v.y;
          M[4 * r + 2] = v.z;
          M[4 * r + 3] = v.w;
        }
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          const float* y = x[kv] + 4 * k;
#pragma unroll
          for (int r = 0; r < 4; ++r)
            z[kv][4 * k + r] =
                fmaf(M[4 * r + 3], y[3], fmaf(M[4 * r + 2], y[2], fmaf(M[4 * r + 1], y[1], M[4 * r] * y[0])));
        }
      }

#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        // a4: codes against n * tau (a zero vector codes 4 everywhere)
        float TB[3];
#pragma unroll
        for (int k = 0; k < 3; ++k)
          TB[k] = n[kv] == 0.f ? CUDART_INF_F : n[kv] * threshold_f32(4 + k) * 0x1p64f;
        uint32_t nib = 0;  // this lane's codes, one per nibble
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const uint32_t c = code_sat<3>(z[kv][i], TB);
          nib |= c << (4 * i);
        }

        // a5: assemble the 12-byte groups.  val = direct part of word j of the lane's group
        // for lanes that own one, N = the nibble word of the group's 8 trailing codes.
        uint32_t val, word;
        if constexpr (E == 4) {
          const int r = lane & 7;
          const uint32_t half = nib << (16 * (r & 1));
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
        if (kv == 0) {
          uint8_t* dst = blk + slot * CB;
          if (lane < CB / 16 && in_bounds(slot * CB + 16 * lane + 16 <= kPage * CB, status))
            *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(q4[0], q4[1], q4[2], q4[3]);
        } else {
          // V in the tile layout: the unit word of unit u (dims 8u..8u+7) is lane u's
          // nibble word (8 dims per lane), or lanes 2u, 2u+1 joined (4 dims per lane); the
          // token's bits of that unit's group are set in place
          const uint32_t pair = E == 4 ? __shfl_xor_sync(kFull, nib, 1) : 0u;
          const bool owner = E == 8 || (lane & 1) == 0;
          const int u = E == 8 ? lane : lane >> 1;
          if (owner) {
            const uint32_t U = E == 8 ? nib : (nib | (pair << 16));
            int B, t, j;
            vt_slot(slot, B, t, j);
            uint32_t W[3], mask;
            vt_member_words(U, j, W, mask);
            uint32_t* g = reinterpret_cast<uint32_t*>(blk + v_codes_off(D) + vt_group_off(D, B, t, u));
            if (in_bounds(vt_group_off(D, B, t, u) + 12 <= kPage * CB, status)) {
#pragma unroll
              for (int w = 0; w < 3; ++w) {
                atomicAnd(g + w, ~mask);
                atomicOr(g + w, W[w]);
              }
            }
          }
        }

        if (lane == 0) {
          uint16_t nb = __half_as_ushort(__float2half_rn(n[kv]));
          if ((nb & 0x7fffu) == 0x7c00u) {  // overflowed binary16
            nb = 0x7bffu;
            set_status(status, ISOQ_ST_NORM_SAT);
          }
          *reinterpret_cast<uint16_t*>(blk + (kv == 0 ? k_norm_off(D) : v_norm_off(D)) +
                                       2 * slot) = nb;
        }
      }
    }
  }
}

// Thread-per-vector variant for d = 128: thread i of a warp quantises token t0+i of one
// (KV head, K|V) pair.  The whole vector lives in the thread's registers, so the WHT needs
// no shuffles and every per-vector cost (addressing, validation, norm, packing) is paid
// once per 128 elements instead of once per 4.  A warp's 32 vectors share the head, so the
// 4x4 block matrices are read as warp-uniform (broadcast) 16-byte loads from shared memory;
// they hold B H4, which takes over the WHT's two innermost stages.  Codes are summed into
// exact float half-words (add_code) instead of being converted and shifted one by one.
// The next task's vector, sequence and position are fetched while the current one is
// processed; the page-table entry is loaded before the arithmetic and used after it.
constexpr int kTpvThreads = 128;
constexpr int kTpvStage = 20;  // words per thread of the 3-bit V unit-word stage (16 + pad)
#ifndef ISOQ_TPV_MINB
#define ISOQ_TPV_MINB 3
#endif
#ifndef ISOQ_TPV_WAVES  // grid cap in waves of resident CTAs
#define ISOQ_TPV_WAVES 3
#endif

template <typename T, int BITS, bool ROPE>
__global__ void __launch_bounds__(kTpvThreads, ISOQ_TPV_MINB)
    quantize_tpv_kernel(const __grid_constant__ QuantLayers layers, int H, int n_tokens,
                        const int32_t* __restrict__ seq_ids,
                        const int32_t* __restrict__ positions, const float* __restrict__ rope,
                        int rope_max_pos) {
  const QuantLayer& L = layers.l[blockIdx.y];  // this launch row's layer
  const float* __restrict__ mats = L.mats;
  uint8_t* __restrict__ blocks = L.blocks;
  const int32_t* __restrict__ page_table = L.page_table;
  const int n_pages = L.n_pages, max_pages = L.max_pages, n_seqs = L.n_seqs;
  const T* __restrict__ K = static_cast<const T*>(L.K);
  const T* __restrict__ V = static_cast<const T*>(L.V);
  uint32_t* status = L.status;
  constexpr int D = 128, CB = code_bytes(D, BITS), BB = block_bytes(D, BITS);
  constexpr int NT = (1 << (BITS - 1)) - 1;  // positive thresholds
  // shared memory: the heads' block matrices [H][32 blocks][16], then one vector slot per
  // thread (padded so that a warp's 16-byte reads of its 32 slots hit distinct banks) into
  // which the next task's vector is copied (cp.async) while the current one is processed
  constexpr int VB = D * (int)sizeof(T), VS = VB + 16;
  extern __shared__ __align__(16) float smats[];
  uint8_t* slot_mem = reinterpret_cast<uint8_t*>(smats + H * (D / 4) * 16) + threadIdx.x * VS;
  // 3-bit V: the unit words of this thread's vector, for the warp's V tile store
  uint32_t* stage = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(smats + H * (D / 4) * 16) +
                                                kTpvThreads * VS) +
                    threadIdx.x * kTpvStage;

  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;
  const int chunks = (n_tokens + 31) >> 5;
  const int n_tasks = H * 2 * chunks;  // task = (32-token chunk, head, kind), chunk-major
  const int stride = gridDim.x * wpb;
  // copy this lane's vector of task tk into its slot (nothing for a missing token); the
  // source address needs only the task, not the token's validity.  The copy is issued
  // after this thread's reads of the slot's previous contents (program order, and the
  // "memory" clobber keeps the compiler from moving them); its shared-memory write lands
  // only once the global read has returned.
  int nsid = -1, npos = -1;  // token of the prefetched task, read with its vector
  auto prefetch = [&](int tk) {
    nsid = npos = -1;
    if (tk < n_tasks) {
      const int ck = tk / (2 * H), rr = tk - ck * 2 * H;
      const int tt = ck * 32 + lane;
      if (tt < n_tokens) {
        const uint8_t* src = reinterpret_cast<const uint8_t*>(((rr & 1) == 0 ? K : V) +
                                                              ((size_t)tt * H + (rr >> 1)) * D);
#pragma unroll
        for (int q = 0; q < VB / 16; ++q)
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                           static_cast<uint32_t>(__cvta_generic_to_shared(slot_mem + 16 * q))),
                       "l"(src + 16 * q)
                       : "memory");
        nsid = __ldg(seq_ids + tt);
        npos = __ldg(positions + tt);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // the first task's copy is in flight while the block matrices are staged
  int task = blockIdx.x * wpb + (threadIdx.x >> 5);
  prefetch(task);
  // The WHT's two innermost butterfly stages act inside each 4-element block as the 4x4
  // Sylvester matrix H4[k][c] = (-1)^popc(k & c); the stages commute, so they are applied
  // last and folded into the block matrix: smats holds B H4 for every block.
  for (int i = threadIdx.x; i < H * (D / 4); i += blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(mats) + 4 * i;
    float4* dst = reinterpret_cast<float4*>(smats) + 4 * i;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 v = __ldg(src + r);  // row r of B
      dst[r] = make_float4((v.x + v.y) + (v.z + v.w), (v.x - v.y) + (v.z - v.w),
                           (v.x + v.y) - (v.z + v.w), (v.x - v.y) - (v.z - v.w));
    }
  }
  __syncthreads();
  for (; task < n_tasks; task += stride) {
    const int chunk = task / (2 * H);
    const int r = task - chunk * 2 * H;
    const int h = r >> 1, kind = r & 1;
    const int t = chunk * 32 + lane;
    // this task's vector: wait for the copy, read the slot, then start the next task's copy
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    float x[D];
#pragma unroll
    for (int i = 0; i < D; i += 8) {
      const uint4 raw = *reinterpret_cast<const uint4*>(slot_mem + i * sizeof(T));
      if constexpr (sizeof(T) == 4) {
        const uint4 raw2 = *reinterpret_cast<const uint4*>(slot_mem + (i + 4) * sizeof(T));
        const uint32_t w[8] = {raw.x, raw.y, raw.z, raw.w, raw2.x, raw2.y, raw2.z, raw2.w};
#pragma unroll
        for (int k = 0; k < 8; ++k) x[i + k] = __uint_as_float(w[k]);
      } else {
        const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
        for (int k = 0; k < 8; ++k) x[i + k] = to_f32<T>(e[k]);
      }
    }
    const int sid = nsid, pos = npos;
    prefetch(task + stride);
    // a lane without a valid token still runs the arithmetic (on whatever its slot holds)
    // and stores nothing: every lane takes part in the warp's 3-bit V store
    bool valid = t < n_tokens;
    // the page-table entry is loaded here and first used by the stores at the end
    int phys = -1;
    if (valid) {
      uint32_t bad = 0;
      if (sid < 0 || sid >= n_seqs) {
        bad = ISOQ_ST_SEQ_RANGE;
      } else if (pos < 0 || (pos >> 6) >= max_pages || (ROPE && pos >= rope_max_pos)) {
        bad = ISOQ_ST_POS_RANGE;
      } else {
        phys = __ldg(page_table + (size_t)sid * max_pages + (pos >> 6));
      }
      if (bad) {
        set_status(status, bad);
        valid = false;
      }
    }

    if (ROPE && kind == 0 && valid) {  // RoPE of K at its position: dims (i, i + D/2)
      const float4* tab = reinterpret_cast<const float4*>(rope + (size_t)pos * D);
#pragma unroll
      for (int i = 0; i < D / 4; ++i) {
        const float4 cs = __ldg(tab + i);
        const float a0 = x[2 * i], b0 = x[2 * i + D / 2], a1 = x[2 * i + 1], b1 = x[2 * i + 1 + D / 2];
        x[2 * i] = fmaf(a0, cs.x, -b0 * cs.y);
        x[2 * i + D / 2] = fmaf(a0, cs.y, b0 * cs.x);
        x[2 * i + 1] = fmaf(a1, cs.z, -b1 * cs.w);
        x[2 * i + 1 + D / 2] = fmaf(a1, cs.w, b1 * cs.z);
      }
    }

    // a1: norm (four partial sums)
    float ss0 = 0.f, ss1 = 0.f, ss2 = 0.f, ss3 = 0.f;
#pragma unroll
    for (int i = 0; i < D; i += 4) {
      ss0 = fmaf(x[i], x[i], ss0);
      ss1 = fmaf(x[i + 1], x[i + 1], ss1);
      ss2 = fmaf(x[i + 2], x[i + 2], ss2);
      ss3 = fmaf(x[i + 3], x[i + 3], ss3);
    }
    const float n = sqrtf((ss0 + ss1) + (ss2 + ss3));

    // a2: unnormalised WHT, natural order: the five outer butterfly stages here, the two
    // innermost ones inside the block matrices
#pragma unroll
    for (int hs = 4; hs < D; hs <<= 1) {
#pragma unroll
      for (int i = 0; i < D; i += 2 * hs) {
#pragma unroll
        for (int j = i; j < i + hs; ++j) {
          const float a = x[j], b = x[j + hs];
          x[j] = a + b;
          x[j + hs] = a - b;
        }
      }
    }

    // a3 + a4: rotation (B H4 of each block, from shared memory) and codes.  The codes of a
    // 16-bit half of a packed word (4 dims at 3 and 4 bits, 8 at 2 bits) are summed as an
    // exact float W = sum coef * code, converted once per half-word.
    float TB[NT];
#pragma unroll
    for (int k = 0; k < NT; ++k)
      TB[k] = n == 0.f ? CUDART_INF_F : n * pos_threshold_f32(BITS, k) * 0x1p64f;
    const float4* mh = reinterpret_cast<const float4*>(smats) + (size_t)h * (D / 4) * 4;
    constexpr int HPB = BITS == 2 ? 2 : 1;  // blocks per 16-bit half-word
    uint32_t half[D / 4 / HPB];
#pragma unroll
    for (int hw = 0; hw < D / 4 / HPB; ++hw) {
      float W = code_base<BITS>() * (BITS == 2 ? 21845.0f : 4369.0f);  // sum coef * base
      float2 W2 = make_float2(W, 0.f);  // 3 bits: the half-word as two partial sums
#pragma unroll
      for (int hb = 0; hb < HPB; ++hb) {
        const int b = hw * HPB + hb;
        float zr[4];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const float4 m = mh[4 * b + rr];
          // the chain starts from +0, so z is never -0 (which would code as negative)
          zr[rr] = fmaf(m.w, x[4 * b + 3],
                        fmaf(m.z, x[4 * b + 2], fmaf(m.y, x[4 * b + 1], fmaf(m.x, x[4 * b], 0.0f))));
        }
        if constexpr (BITS == 3) {
          add_code3_pair(W2, zr[0], zr[1], 1.0f, 16.0f, TB);
          add_code3_pair(W2, zr[2], zr[3], 256.0f, 4096.0f, TB);
        } else {
#pragma unroll
          for (int rr = 0; rr < 4; ++rr) {
            const int e = 4 * hb + rr;  // dim inside the half-word's dims
            const float coef = BITS == 2 ? (float)(1 << (2 * (slot2(8 * (hw & 1) + e) & 7)))
                                         : (float)(1 << (4 * e));
            W = add_code<BITS>(W, zr[rr], coef, TB);
          }
        }
      }
      if constexpr (BITS == 3) W = W2.x + W2.y;
      half[hw] = __float_as_uint(W + 8388608.0f);  // 0x4B000000 | W (W in [0, 65535])
    }
    uint32_t rec[CB / 4];
    if constexpr (BITS == 3) {
      // a5: per 32-dim group, words 0..2 = nibble words of dims 8j..8j+7 with bit 3 taken
      // from the group's trailing 8 codes (bit 2 - j of each)
      uint32_t nib[D / 8];
#pragma unroll
      for (int j = 0; j < D / 8; ++j) nib[j] = join_halves(half[2 * j], half[2 * j + 1]);
#pragma unroll
      for (int g = 0; g < D / 32; ++g) {
        const uint32_t N3 = nib[4 * g + 3];
#pragma unroll
        for (int j = 0; j < 3; ++j) rec[3 * g + j] = nib[4 * g + j] | ((N3 << (j + 1)) & 0x88888888u);
      }
      if (kind == 1 && in_bounds(D / 8 <= kTpvStage, status)) {  // V: the unit words
#pragma unroll
        for (int q = 0; q < D / 32; ++q)
          *reinterpret_cast<uint4*>(stage + 4 * q) =
              make_uint4(nib[4 * q], nib[4 * q + 1], nib[4 * q + 2], nib[4 * q + 3]);
      }
    } else {
#pragma unroll
      for (int j = 0; j < CB / 4; ++j) rec[j] = join_halves(half[2 * j], half[2 * j + 1]);
    }
    if (valid && (phys < 0 || phys >= n_pages)) {
      set_status(status, ISOQ_ST_PAGE_RANGE);
      valid = false;
    }
    if (valid && !in_bounds(h < H && (pos & (kPage - 1)) < kPage, status)) valid = false;
    if (!valid) phys = -1;
    if (valid) {
      uint8_t* blk = blocks + ((size_t)phys * H + h) * BB;
      const int slot = pos & (kPage - 1);
      if (BITS != 3 || kind == 0) {
        uint4* dst =
            reinterpret_cast<uint4*>(blk + (kind == 0 ? 0 : v_codes_off(D, BITS)) + slot * CB);
#pragma unroll
        for (int q = 0; q < CB / 16; ++q)
          dst[q] = make_uint4(rec[4 * q], rec[4 * q + 1], rec[4 * q + 2], rec[4 * q + 3]);
      }
      uint16_t nb = __half_as_ushort(__float2half_rn(n));
      if ((nb & 0x7fffu) == 0x7c00u) {  // overflowed binary16
        nb = 0x7bffu;
        set_status(status, ISOQ_ST_NORM_SAT);
      }
      *reinterpret_cast<uint16_t*>(blk + (kind == 0 ? k_norm_off(D, BITS) : v_norm_off(D, BITS)) +
                                   2 * slot) = nb;
    }
    if constexpr (BITS == 3) {
      if (kind == 1) {  // warp-uniform: the task is the warp's
        __syncwarp();
        vt_store_warp<D, kTpvStage>(stage - lane * kTpvStage, lane, sid, pos, phys, blocks, H, h,
                                    status);
        __syncwarp();  // the stage is rewritten by the next task
      }
    }
  }
}

template <int D, typename T>
static cudaError_t launch_t(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  const long long warps = a.n_tokens;  // one warp per token
  const int wpb = 8;
  long long grid = (warps + wpb - 1) / wpb;
  const long long cap = (long long)n_sm * 16 / a.layers.n + 1;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  quantize_append_kernel<D, T><<<dim3((unsigned)grid, a.layers.n), wpb * 32, 0, stream>>>(
      a.layers, a.n_kv_heads, a.n_tokens, a.seq_ids, a.positions, a.rope, a.rope_max_pos);
  return cudaGetLastError();
}

template <typename T, int BITS, bool ROPE>
static cudaError_t launch_tpv(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  const size_t smem = (size_t)a.n_kv_heads * 32 * 16 * sizeof(float) +
                      (size_t)kTpvThreads * (128 * sizeof(T) + 16) +
                      (size_t)kTpvThreads * kTpvStage * 4;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(quantize_tpv_kernel<T, BITS, ROPE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const long long tasks = (long long)a.n_kv_heads * 2 * ((a.n_tokens + 31) / 32);
  const int wpb = kTpvThreads / 32;
  long long grid = (tasks + wpb - 1) / wpb;
  const long long cap = (long long)n_sm * ISOQ_TPV_MINB * ISOQ_TPV_WAVES / a.layers.n + 1;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  quantize_tpv_kernel<T, BITS, ROPE><<<dim3((unsigned)grid, a.layers.n), kTpvThreads, smem,
                                       stream>>>(
      a.layers, a.n_kv_heads, a.n_tokens, a.seq_ids, a.positions, a.rope, a.rope_max_pos);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t launch_tpv_b(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  const bool r = a.rope != nullptr;
  switch (a.bits) {
    case 2: return r ? launch_tpv<T, 2, true>(a, stream, n_sm) : launch_tpv<T, 2, false>(a, stream, n_sm);
    case 3: return r ? launch_tpv<T, 3, true>(a, stream, n_sm) : launch_tpv<T, 3, false>(a, stream, n_sm);
    case 4: return r ? launch_tpv<T, 4, true>(a, stream, n_sm) : launch_tpv<T, 4, false>(a, stream, n_sm);
  }
  return cudaErrorInvalidValue;
}

template <int D>
static cudaError_t launch_d(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  if constexpr (D == 128) {
#ifndef ISOQ_NO_QUANTIZE_TC
    if (use_quantize_tc(a)) return launch_quantize_tc(a, stream, n_sm);
#endif
    switch (a.dtype) {
      case ISOQ_F32: return launch_tpv_b<float>(a, stream, n_sm);
      case ISOQ_BF16: return launch_tpv_b<__nv_bfloat16>(a, stream, n_sm);
      case ISOQ_F16: return launch_tpv_b<__half>(a, stream, n_sm);
    }
    return cudaErrorInvalidValue;
  }
  if (a.bits != 3) return cudaErrorInvalidValue;  // the variants exist at d = 128
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
