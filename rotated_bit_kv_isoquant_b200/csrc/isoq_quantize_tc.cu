// Quantize-append for d = 128 (2-, 3- and 4-bit codes), bf16 / f16 inputs, with the
// Walsh-Hadamard transform on the 5th-generation tensor cores.
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: each K/V vector goes through a Walsh-Hadamard
// transform, then block-diagonal SO(4) rotations, then a 3-bit scalar quantiser.
//
// The unnormalised WHT in natural (Sylvester) order is the symmetric matrix
// H[k][n] = (-1)^popc(k & n).  Its entries are exact in bf16 and f16, and so are the
// inputs, so the transform of a tile of 128 vectors (128 consecutive tokens of one KV head,
// K or V) is one 128 x 128 x 128 UMMA (kind::f16, f32 accumulator in tensor memory) with
// exact products.  The rest runs on the CUDA cores over the accumulator rows: thread r
// owns vector r (tensor-memory lane r).  It sums the squares of its row for the norm
// (|H x|^2 = 128 |x|^2), then, one 64-dim half at a time, applies the head's 4x4 block
// matrices, decides the codes against the norm-scaled thresholds, packs them and stores
// that half of the record (24 bytes at 3 bits) into the paged cache.
//
// Pipeline of a CTA over its tiles j: the copies of tile j+2 (cp.async of the 128 rows
// into the operand layout, and the head's block matrices) and the UMMA of tile j+1 run
// while the threads work on tile j's accumulator; two accumulators alternate in tensor
// memory (256 columns) and two operand stages in shared memory.  Every mbarrier wait is
// bounded; a wait that gives up reports ISOQ_ST_TIMEOUT and the CTA stops after draining
// what it issued.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <type_traits>

#include "isoq_check.cuh"
#include "isoq_codes.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"
#include "isoq_tc.cuh"
#include "isoq_vtile.cuh"

namespace isoq {
namespace {
using namespace ptx;

constexpr int kQtD = 128;
constexpr int kQtRows = 128;                      // vectors per tile = UMMA M
constexpr int kQtThreads = 128;                   // one thread per vector (row)
constexpr int kQtTile = kQtRows * kQtD * 2;       // one 16-bit operand tile, 32 KiB
constexpr int kQtMat = 32 * 16 * 4;               // one head's block matrices, 2 KiB
constexpr int kOffX = 0;                          // [2] input tiles
constexpr int kOffH = 2 * kQtTile;                // the Hadamard operand
constexpr int kOffM = kOffH + kQtTile;            // [3] block-matrix stages
constexpr int kOffBar = kOffM + 3 * kQtMat;       // 2 mbarriers (UMMA completion)
constexpr int kOffSlot = kOffBar + 16;            // tensor-memory base address
constexpr int kStageWords = 20;                   // per thread: 16 unit words (+4 pad)
constexpr int kOffStage = kOffSlot + 16;          // [128 threads][20] 3-bit V unit words
constexpr int kQtSmem = kOffStage + kQtThreads * kStageWords * 4;
constexpr uint32_t kQtCols = 256;                 // two 128-column f32 accumulators

// Byte offset of element (row, k) of a K-major no-swizzle operand tile: core matrices of
// 8 rows x 16 bytes, 128 bytes apart along k (the descriptor's leading offset) and 2048
// bytes apart along the rows (its stride offset).
__host__ __device__ constexpr uint32_t qt_off(int row, int k) {
  return (uint32_t)((row >> 3) * 2048 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

// Packed pair of binary32 FMAs (one instruction, the same rounding per lane as fmaf).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("{\n .reg .b64 pa, pb, pc;\n mov.b64 pa, {%1, %2};\n mov.b64 pb, {%3, %4};\n"
      " mov.b64 pc, {%5, %6};\n fma.rn.f32x2 %0, pa, pb, pc;\n}"
      : "=l"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  float2 o;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(o.x), "=f"(o.y) : "l"(r));
  return o;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <typename T, int BITS>
__global__ void __launch_bounds__(kQtThreads, 2)
    quantize_tc_kernel(const __grid_constant__ QuantLayers layers, int H, int n_tokens,
                       const int32_t* __restrict__ seq_ids,
                       const int32_t* __restrict__ positions) {
  constexpr int D = kQtD, CB = code_bytes(D, BITS), BB = block_bytes(D, BITS);
  constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
  constexpr uint32_t kIdesc = tc::idesc_f16(128, 128, false, false, kBf16);
  const QuantLayer& L = layers.l[blockIdx.y];  // this launch row's layer
  const float* __restrict__ mats = L.mats;
  uint8_t* __restrict__ blocks = L.blocks;
  const int32_t* __restrict__ page_table = L.page_table;
  const int n_pages = L.n_pages, max_pages = L.max_pages, n_seqs = L.n_seqs;
  const uint8_t* __restrict__ Kb = static_cast<const uint8_t*>(L.K);
  const uint8_t* __restrict__ Vb = static_cast<const uint8_t*>(L.V);
  uint32_t* status = L.status;

  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t* stage = reinterpret_cast<uint32_t*>(smem + kOffStage) + tid * kStageWords;
  const int quad = warp;           // tensor-memory lane quarter
  const int r = quad * 32 + lane;  // this thread's vector (row) of the tile
  const int n_chunks = (n_tokens + kQtRows - 1) / kQtRows;
  const int n_kinds = 2 * H;             // (head, K|V) pairs: rr = 2 head + kind
  const int n_tiles = n_chunks * n_kinds;  // tile = (128-token chunk, head, K|V), chunk-major
  const int first = blockIdx.x, stride = gridDim.x;
  if (first >= n_tiles) return;
  // this CTA's tiles first, first + stride, ... as (chunk, rr), advanced without division
  struct Tile {
    int chunk, rr;
  };
  const int step_c = stride / n_kinds, step_r = stride - step_c * n_kinds;
  auto advance = [&](Tile t) {
    t.chunk += step_c;
    t.rr += step_r;
    if (t.rr >= n_kinds) {
      t.rr -= n_kinds;
      ++t.chunk;
    }
    return t;
  };
  Tile cur{first / n_kinds, first % n_kinds};  // tiles li, li + 1, li + 2
  Tile nxt = advance(cur), nn = advance(nxt);

  // copies of tile t (local index li) into input stage li & 1 and matrix stage li % 3; a
  // warp's copy covers 8 rows x 64 bytes, 512 contiguous bytes of the tile.  Rows past the
  // last token are not copied (their accumulator rows are never used).
  const int cp_row = tid & 7, cp_j = (tid >> 3) & 15;  // + 8 c
  const uint32_t cp_dst = qt_off(cp_row, 8 * cp_j);
  const size_t row_bytes = (size_t)H * D * sizeof(T);
  auto prefetch = [&](Tile t, int li) {
    if (t.chunk < n_chunks && in_bounds((t.rr >> 1) < H, status)) {
      const int h = t.rr >> 1;
      const int t0 = t.chunk * kQtRows;
      const uint8_t* src = ((t.rr & 1) ? Vb : Kb) + (size_t)(t0 + cp_row) * row_bytes +
                           (size_t)h * D * sizeof(T) + 16 * cp_j;
      const uint32_t xs = sbase + kOffX + (li & 1) * kQtTile + cp_dst;
      const int rows_left = n_tokens - t0 - cp_row;
#pragma unroll
      for (int c = 0; c < 16; ++c)
        if (8 * c < rows_left) cp_async16(xs + 2048 * c, src + 8 * c * row_bytes);
      if (tid < kQtMat / 16)
        cp_async16(sbase + kOffM + (li % 3) * kQtMat + 16 * tid,
                   reinterpret_cast<const uint8_t*>(mats) + (size_t)h * kQtMat + 16 * tid);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  prefetch(cur, 0);
  prefetch(nxt, 1);

  // the Hadamard operand (N x K, K-major; symmetric): thread -> row tid
  {
    const uint32_t one = kBf16 ? 0x3F80u : 0x3C00u;
    const int n = tid;
#pragma unroll 4
    for (int kc = 0; kc < 16; ++kc) {
      const int k0 = 8 * kc;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = one | ((__popc(n & (k0 + 2 * e)) & 1u) << 15);
        const uint32_t hi = one | ((__popc(n & (k0 + 2 * e + 1)) & 1u) << 15);
        w[e] = lo | (hi << 16);
      }
      *reinterpret_cast<uint4*>(smem + kOffH + qt_off(n, k0)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  if (tid == 0) {
    mbar_init(bars + 0, 1);
    mbar_init(bars + 1, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tc::alloc(tmem_slot, kQtCols);

  auto issue_mma = [&](int li) {  // thread 0: the tile's transform into accumulator li & 1
    const uint32_t xs = sbase + kOffX + (li & 1) * kQtTile, hs = sbase + kOffH;
    const uint32_t d = *tmem_slot + (uint32_t)(li & 1) * 128;
#pragma unroll
    for (int s = 0; s < D / 16; ++s)
      tc::mma_ss(d, tc::sdesc(xs + 256 * s, 128, 2048), tc::sdesc(hs + 256 * s, 128, 2048), kIdesc,
                 s > 0);
    tc::commit(bars + (li & 1));
  };

  // sequence, position and page entry of this thread's token, loaded one tile ahead of use
  int sid = -1, pos = -1, phys = -1;
  auto load_page = [&](int t) {  // validates (sid, pos) of token t; page entry or -1
    phys = -1;
    if (t >= n_tokens) return;
    if (sid < 0 || sid >= n_seqs) {
      set_status(status, ISOQ_ST_SEQ_RANGE);
    } else if (pos < 0 || (pos >> 6) >= max_pages) {
      set_status(status, ISOQ_ST_POS_RANGE);
    } else {
      phys = __ldg(page_table + (size_t)sid * max_pages + (pos >> 6));
      if (phys < 0 || phys >= n_pages) {
        set_status(status, ISOQ_ST_PAGE_RANGE);
        phys = -1;
      }
    }
  };
  {
    const int t = cur.chunk * kQtRows + r;
    if (t < n_tokens) {
      sid = __ldg(seq_ids + t);
      pos = __ldg(positions + t);
    }
    load_page(t);
  }

  // tile 0's copies, the Hadamard operand and the barriers are visible; first transform
  asm volatile("cp.async.wait_group 1;" ::: "memory");
  fence_proxy_async();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_row = tmem + ((uint32_t)(quad * 32) << 16);  // this thread's lane
  if (tid == 0) issue_mma(0);

  bool failed = false, ok = true;  // ok: the last wait for a transform completed
  int li = 0;
  for (;; ++li) {
    if (cur.chunk >= n_chunks) break;
    const bool has_next = nxt.chunk < n_chunks;
    // tile li+1's copies landed, tile li-1's accumulator reads are done: transform li+1
    // (unless a wait gave up anywhere in the CTA)
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    fence_proxy_async();
    tc::fence_before();
    if (__syncthreads_or(!ok)) {
      failed = true;
      break;
    }
    if (tid == 0 && has_next) {
      tc::fence_after();
      issue_mma(li + 1);
    }
    int nsid = -1, npos = -1;
    if (has_next) {
      const int tn = nxt.chunk * kQtRows + r;
      if (tn < n_tokens) {
        nsid = __ldg(seq_ids + tn);
        npos = __ldg(positions + tn);
      }
    }
    ok = mbar_wait(bars + (li & 1), (li >> 1) & 1);  // transform li done
    tc::fence_after();
    prefetch(nn, li + 2);  // input stage li & 1 is free again

    const int h = cur.rr >> 1, kind = cur.rr & 1;
    const uint32_t acc = t_row + (uint32_t)(li & 1) * 128;  // this thread's vector

    // a1: norm from the transform, |x|^2 = |H x|^2 / 128
    uint32_t y[64];
    float n;
    {
      float2 s01 = make_float2(0.f, 0.f), s23 = make_float2(0.f, 0.f);  // four partial sums
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (!in_bounds((li & 1) * 128 + 64 * hh + 64 <= (int)kQtCols, status)) break;
        tc::ld64(acc + 64 * hh, y);
#pragma unroll
        for (int e = 0; e < 64; e += 4) {
          const float2 ab = make_float2(__uint_as_float(y[e]), __uint_as_float(y[e + 1]));
          const float2 cd = make_float2(__uint_as_float(y[e + 2]), __uint_as_float(y[e + 3]));
          s01 = fma2(ab, ab, s01);
          s23 = fma2(cd, cd, s23);
        }
      }
      n = sqrtf(((s01.x + s01.y) + (s23.x + s23.y)) * (1.0f / 128.0f));
    }

    // a3 + a4 + a5: per 64-dim half hf of the vector, block matrices and codes of its 16
    // blocks, summed into 16-bit half-words (one block at 3 and 4 bits, two at 2 bits) and
    // packed into that half of the record: bytes [CB/2 hf, CB/2 (hf + 1))
    constexpr int NT = (1 << (BITS - 1)) - 1;  // positive thresholds
    constexpr int HPB = BITS == 2 ? 2 : 1;     // blocks per half-word
    constexpr int NHW = 16 / HPB;              // half-words of a half
    float TB[NT];
#pragma unroll
    for (int k = 0; k < NT; ++k)
      TB[k] = n == 0.f ? CUDART_INF_F : n * pos_threshold_f32(BITS, k) * 0x1p64f;
    // the second half first: the norm pass left its columns in y
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int hf = 1 - pass;
      if (pass) tc::ld64(acc, y);  // the first half's columns
      const float4* mh = reinterpret_cast<const float4*>(smem + kOffM + (li % 3) * kQtMat) + 64 * hf;
      uint32_t half[NHW];
#pragma unroll
      for (int hw = 0; hw < NHW; ++hw) {
        float W = code_base<BITS>() * (BITS == 2 ? 21845.0f : 4369.0f);  // sum coef * base
        float2 W2 = make_float2(W, 0.f);  // 3 bits: the half-word as two partial sums
#pragma unroll
        for (int hb = 0; hb < HPB; ++hb) {
          const int bl = hw * HPB + hb;  // block of the half
          float zr[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float4 m = mh[4 * bl + e];
            // row e of the block as two packed FMA chains (dims 0, 2 and 1, 3) from +0, so z
            // is never -0 (which would code as negative)
            const uint32_t* yb = y + 4 * bl;
            float2 p = fma2(make_float2(m.x, m.y),
                            make_float2(__uint_as_float(yb[0]), __uint_as_float(yb[1])),
                            make_float2(0.f, 0.f));
            p = fma2(make_float2(m.z, m.w),
                     make_float2(__uint_as_float(yb[2]), __uint_as_float(yb[3])), p);
            zr[e] = p.x + p.y;
          }
          if constexpr (BITS == 3) {
            add_code3_pair(W2, zr[0], zr[1], 1.0f, 16.0f, TB);
            add_code3_pair(W2, zr[2], zr[3], 256.0f, 4096.0f, TB);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float coef = BITS == 2 ? (float)(1 << (2 * (slot2(8 * (hw & 1) + 4 * hb + e) & 7)))
                                           : (float)(1 << (4 * e));
              W = add_code<BITS>(W, zr[e], coef, TB);
            }
          }
        }
        if constexpr (BITS == 3) W = W2.x + W2.y;
        half[hw] = __float_as_uint(W + 8388608.0f);  // 0x4B000000 | W
      }
      constexpr int NR = CB / 8;  // words of half the record
      uint32_t rec[NR];
      if constexpr (BITS == 3) {
        // per 32-dim group: nibble words of dims 8j..8j+7, bit 3 from the group's last 8 codes
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          uint32_t nib[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) nib[j] = join_halves(half[8 * gg + 2 * j], half[8 * gg + 2 * j + 1]);
#pragma unroll
          for (int j = 0; j < 3; ++j) rec[3 * gg + j] = nib[j] | ((nib[3] << (j + 1)) & 0x88888888u);
          if (kind == 1 && in_bounds(8 * hf + 4 * gg + 4 <= kStageWords, status))
            // V: the unit words 8 hf + 4 gg .. +3, for the V tile layout
            *reinterpret_cast<uint4*>(stage + 8 * hf + 4 * gg) =
                make_uint4(nib[0], nib[1], nib[2], nib[3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < NR; ++j) rec[j] = join_halves(half[2 * j], half[2 * j + 1]);
      }

      if (phys >= 0 && in_bounds(phys < n_pages && h < H && (CB / 2) * (hf + 1) <= CB, status)) {
        uint8_t* blk = blocks + ((size_t)phys * H + h) * BB;
        const int slot = pos & (kPage - 1);
        uint8_t* dst = blk + (kind == 0 ? 0 : v_codes_off(D, BITS)) + slot * CB + (CB / 2) * hf;
        if (BITS == 3 && kind == 1) {
          // V at 3 bits: written after both halves, in the V tile layout
        } else if constexpr (BITS == 3) {  // 24 bytes at 0 or 24: 16 + 8 or 8 + 16
          if (hf == 0) {
            *reinterpret_cast<uint4*>(dst) = make_uint4(rec[0], rec[1], rec[2], rec[3]);
            *reinterpret_cast<uint2*>(dst + 16) = make_uint2(rec[4], rec[5]);
          } else {
            *reinterpret_cast<uint2*>(dst) = make_uint2(rec[0], rec[1]);
            *reinterpret_cast<uint4*>(dst + 8) = make_uint4(rec[2], rec[3], rec[4], rec[5]);
          }
        } else {
#pragma unroll
          for (int q = 0; q < NR / 4; ++q)
            *reinterpret_cast<uint4*>(dst + 16 * q) =
                make_uint4(rec[4 * q], rec[4 * q + 1], rec[4 * q + 2], rec[4 * q + 3]);
        }
        if (hf == 0) {
          uint16_t nb = __half_as_ushort(__float2half_rn(n));
          if ((nb & 0x7fffu) == 0x7c00u) {  // overflowed binary16
            nb = 0x7bffu;
            set_status(status, ISOQ_ST_NORM_SAT);
          }
          *reinterpret_cast<uint16_t*>(blk + (kind == 0 ? k_norm_off(D, BITS) : v_norm_off(D, BITS)) +
                                       2 * slot) = nb;
        }
      }
    }
    if constexpr (BITS == 3) {
      if (kind == 1) {  // CTA-uniform
        __syncwarp();
        vt_store_warp<kQtD, kStageWords>(stage - lane * kStageWords, lane, sid, pos, phys, blocks, H, h,
                                         status);
      }
    }
    if (has_next) {
      sid = nsid;
      pos = npos;
      load_page(nxt.chunk * kQtRows + r);
    }
    cur = nxt;
    nxt = nn;
    nn = advance(nn);
  }

  // a wait that gave up (anywhere in the CTA; the loop's end has the last one): report it
  // and wait (bounded) for the last transform issued before the tensor memory is released
  if (failed || __syncthreads_or(!ok)) {
    if (tid == 0) set_status(status, ISOQ_ST_TIMEOUT);
    const int last = failed ? li : li - 1;
    if (last >= 0) mbar_wait(bars + (last & 1), (last >> 1) & 1);
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::dealloc(tmem, kQtCols);
  }
}

template <typename T, int BITS>
cudaError_t launch_qt(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(quantize_tc_kernel<T, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kQtSmem);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  const long long tiles = (long long)((a.n_tokens + kQtRows - 1) / kQtRows) * a.n_kv_heads * 2;
  long long grid = tiles;
  const long long cap = (long long)n_sm * 2 / a.layers.n;  // one wave of resident CTAs
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  quantize_tc_kernel<T, BITS><<<dim3((unsigned)grid, a.layers.n), kQtThreads, kQtSmem, stream>>>(
      a.layers, a.n_kv_heads, a.n_tokens, a.seq_ids, a.positions);
  return cudaGetLastError();
}

}  // namespace

bool use_quantize_tc(const QuantizeArgs& a) {
  return a.d == kQtD && a.bits >= 2 && a.bits <= 4 && a.rope == nullptr &&
         (a.dtype == ISOQ_BF16 || a.dtype == ISOQ_F16);
}

template <typename T>
cudaError_t launch_qt_b(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  switch (a.bits) {
    case 2: return launch_qt<T, 2>(a, stream, n_sm);
    case 3: return launch_qt<T, 3>(a, stream, n_sm);
    case 4: return launch_qt<T, 4>(a, stream, n_sm);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_tc(const QuantizeArgs& a, cudaStream_t stream, int n_sm) {
  switch (a.dtype) {
    case ISOQ_BF16: return launch_qt_b<__nv_bfloat16>(a, stream, n_sm);
    case ISOQ_F16: return launch_qt_b<__half>(a, stream, n_sm);
  }
  return cudaErrorInvalidValue;
}

}  // namespace isoq
