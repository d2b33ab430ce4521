// Decode attention on the packed 3-bit cache with 8-bit integer tensor-core products
// (split-K partials).
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: attention is computed directly on the packed
// 3-bit codes and full-precision K/V are never rebuilt.  With R orthogonal,
// q.k_hat = (R q).(R k_hat), so the rows' queries are rotated once per CTA and the scores
// and the value sum run on codebook levels in the rotated space.
//
// Scores in exact integer arithmetic.  The levels are 4-decimal numbers, so 10000 L[c] is
// an exact 16-bit integer, split into two signed bytes kh * 256 + kl.  Each thread turns a
// 16-bit half of a packed word (four 3-bit codes) into four such bytes with one byte
// permute against an 8-entry table of the levels' high bytes and one against their low
// bytes: two permutes per four keys, the operand of an int8 mma.sync as it is.  The
// rotated query of a row is scaled to a 24-bit integer (8e6 / max|q~|) and split into
// three balanced signed bytes d2 d1 d0, so a score is
//   2^24 d2.kh + 2^16 (d2.kl + d1.kh) + 2^8 (d1.kl + d0.kh)   (+ d0.kl, below 2^-23 of it)
// from s8 x s8 -> s32 products that are exact; the query's rounding (relative 1e-7) is
// the only error before the binary32 softmax.
// Values in f16.  The value weights P' = p nV / sigma (lazily rescaled running maximum and
// V-norm reference) span many binades, which a fixed-point operand would cut short, so the
// value product keeps f16 operands with f32 accumulators: V_hat^T from byte permutes of
// f16 level bytes (ALPHA times the levels, < 2e-5 relative error), P' as f16.
//
// Work: one CTA of 4 warps per (context chunk, KV head, block of RB rows, sequence); a
// row is a (query token, query head) pair.  Each warp streams its own pages of the chunk
// through a private ring of shared-memory stages filled by 1-D bulk copies (one page
// block per copy, completion on an mbarrier, every wait bounded).  Per 32-token tile:
//   scores  C[16 x 8 tokens] = A[16 x 32 dims] . K_hat^T, m16n8k32 s8, 4 tiles of 8 tokens:
//           RB = 8: A = [d2; d1] against kh and kl, [0; d0] against kh added to the kl
//           product (3 mma per k-step, two accumulators);
//           RB = 4: A = [d2; d1; d0; 0] against kh, [d2; d1; 0; 0] against kl (2 mma).
//           Lane t of a quad owns 32-dim group t of every token (the k order inside a
//           k-step is a permutation of the dims, the query digits follow it).
//   online softmax per row, rescaled only when a running maximum grows (lazy), so the
//           common tile needs no shuffles
//   values  O^T[16 dims x 8 rows] += V_hat^T[16 x 16 tokens] . P'^T, m16n8k16 f16 per
//           16-token block: the score tile's columns 2t, 2t+1 of two 8-token tiles are
//           exactly the k slots 2t, 2t+1, 2t+8, 2t+9 of the value product, and the V tile
//           layout stores those four tokens' codes of one dim as the four nibbles of a
//           16-bit half-word: two level-byte lookups and two interleaves give the A
//           registers of two k slots each, with no cross-token merging.
#include <math_constants.h>

#include <type_traits>

#include "isoq_check.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"
#include "isoq_vtile.cuh"

namespace isoq {
using namespace ptx;
int decode_i8_sms();
namespace {

constexpr float kQMax = 8.0e6f;       // |24-bit query integer| bound (digits stay in s8)
constexpr float kLevelScale = 1.0e4f; // integer levels: 10000 L[c]

__device__ __forceinline__ void mma_s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same with a zero accumulator (c = a . b): no zeroing of c beforehand.
__device__ __forceinline__ void mma_s8_first(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {0,0,0,0};"
      : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The decode is bound by the logic pipe (byte permutes, shifts, masks) and by the latency of
// its dependent chains.  A code word's selector (its nibbles with the top bit clear) is
// formed as w - top_bits(w) on the multiply-add pipe, which has room to spare; the -1 is a
// kernel argument so that the compiler keeps the multiply-add instead of folding it back
// into a logic operation.  (Right shifts as high words of products lengthen the chains more
// than they relieve the logic pipe, so the spare unit and the upper halves stay shifts.)
struct I8Mul {
  uint32_t neg1;
};
__device__ __forceinline__ uint32_t mad_lo_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
// Top bits of the nibbles of a code word (the spare unit's bits)
__device__ __forceinline__ uint32_t top_bits(uint32_t w) { return w & 0x88888888u; }
// Selector word of a code word: its nibbles with the top bit clear
__device__ __forceinline__ uint32_t sel_word(uint32_t w, uint32_t top, const I8Mul& mk) {
  return mad_lo_u32(top, mk.neg1, w);
}
// The spare unit's selector from the three top-bit words: nibble k = bits 4k+3 of w0, w1,
// w2 as bits 2, 1, 0
__device__ __forceinline__ uint32_t sel_spare(uint32_t t0, uint32_t t1, uint32_t t2) {
  return (t2 >> 3) | (t1 >> 2) | (t0 >> 1);
}

template <bool FIRST>
__device__ __forceinline__ void mma_s8_acc(int (&c)[4], uint4 a, uint32_t b0, uint32_t b1) {
  if constexpr (FIRST) mma_s8_first(c, a.x, a.y, a.z, a.w, b0, b1);
  else mma_s8(c, a.x, a.y, a.z, a.w, b0, b1);
}

// Integer level 10000 L[c] = kh * 256 + kl with kl in [-128, 127], kh = floor((v + 128) / 256).
__host__ __device__ constexpr int ilevel(int c) {
  return c == 0 ? -21520 : c == 1 ? -13440 : c == 2 ? -7560 : c == 3 ? -2451
       : c == 4 ? 2451 : c == 5 ? 7560 : c == 6 ? 13440 : 21520;
}
__host__ __device__ constexpr int ilevel_hi(int c) {
  return (ilevel(c) + 128 >= 0) ? (ilevel(c) + 128) / 256 : -((-(ilevel(c) + 128) + 255) / 256);
}
__host__ __device__ constexpr int ilevel_lo(int c) { return ilevel(c) - 256 * ilevel_hi(c); }
__host__ __device__ constexpr uint32_t level_bytes(bool hi, int c0) {
  uint32_t w = 0;
  for (int k = 0; k < 4; ++k)
    w |= (uint32_t)((hi ? ilevel_hi(c0 + k) : ilevel_lo(c0 + k)) & 0xff) << (8 * k);
  return w;
}
static_assert(ilevel_hi(2) * 256 + ilevel_lo(2) == -7560 && ilevel_lo(1) == -128 &&
                  ilevel_lo(6) == -128 && ilevel_hi(7) == 84 && ilevel_lo(7) == 16,
              "integer level split");
constexpr uint32_t kTH0 = level_bytes(true, 0), kTH1 = level_bytes(true, 4);
constexpr uint32_t kTL0 = level_bytes(false, 0), kTL1 = level_bytes(false, 4);

// Balanced base-256 digits of a 24-bit integer: q = d2 * 65536 + d1 * 256 + d0.
__device__ __forceinline__ void digits3(int q, int& d2, int& d1, int& d0) {
  d0 = ((q + 128) & 255) - 128;
  const int r = (q - d0) >> 8;
  d1 = ((r + 128) & 255) - 128;
  d2 = (r - d1) >> 8;
}

__device__ __forceinline__ uint32_t pack_s8x4(int a, int b, int c, int d) {
  return (uint32_t)(a & 255) | ((uint32_t)(b & 255) << 8) | ((uint32_t)(c & 255) << 16) |
         ((uint32_t)(d & 255) << 24);
}

// Shared memory: [NW warps][NST] page stages, the mbarriers, the score mma's A fragments
// (A1 and A2, 4 words per k-step and lane; A2 holds its zero rows explicitly, so each is
// one 16-byte load straight into the mma's register quad), per-row score factors, output
// row indices.  The stage area is reused for the final merge.
template <int D, int NST, int RB, int NW>
struct I8Smem {
  static constexpr int kStageBytes = block_bytes(D, 3);
  static constexpr int kRing = NW * NST * kStageBytes;
  static constexpr int kBarOff = kRing;
  static constexpr int kAOff = kBarOff + NW * NST * 8;                 // uint4 [D/32][32]
  static constexpr int kA2Off = kAOff + (D / 32) * 32 * 16;            // uint4 [D/32][32]
  static constexpr int kKfOff = kA2Off + (D / 32) * 32 * 16;           // float [8]
  static constexpr int kRowOff = kKfOff + 8 * 4;                      // int [8]
  static constexpr int kBytes = kRowOff + 8 * 4;
  // the warps' states [NW][8][D + 4] and, for a single chunk, the merged rows [8][D + 1]
  static constexpr int kMergeBytes = NW * 8 * (D + 4) * 4 + 8 * (D + 1) * 4;
  static_assert(kMergeBytes <= kRing, "merge buffer must fit in the ring");
  static_assert(kAOff % 16 == 0 && kA2Off % 16 == 0, "A fragments must be aligned");
};

#ifndef ISOQ_I8_MINB128
#define ISOQ_I8_MINB128 4
#endif
#ifndef ISOQ_I8_NT  // 8-token score tiles per load of the query fragments (1, 2 or 4)
#define ISOQ_I8_NT 2
#endif
constexpr int kI8NT = ISOQ_I8_NT;
static_assert(4 % kI8NT == 0, "score tiles per fragment load");

// CTAs per SM the register budget is set for: 4-warp CTAs as many as fit (d = 128: 4, d =
// 256: 2); the wide CTAs of small grids (one per SM) get the same per-thread budget.
#ifndef ISOQ_I8_MINB256
#define ISOQ_I8_MINB256 2
#endif
template <int D>
constexpr int i8_min_blocks(int nw) {
  return nw == 4 ? (D == 128 ? ISOQ_I8_MINB128 : ISOQ_I8_MINB256) : 1;
}


// MQ: chunks of several query tokens per sequence with causal limits; the decode (one
// query token, every row attending the whole context) is compiled without them.
// NW: warps per CTA.  4 normally (several CTAs per SM); a grid with fewer CTAs than the
// GPU holds gives each CTA more warps (16 at d = 128, 8 at d = 256), so that the pages of
// a chunk are in flight at once instead of one after another per warp, at the cost of one
// query rotation and one merge per CTA as before.
// out (decode with a single chunk only, else null): the CTA holds the whole context of its
// rows, so it finishes the combine itself -- normalise, inverse rotation -- and writes the
// output rows [n_seqs][n_q_heads][D] instead of partials.
template <int D, int NST, int RB, typename TQ, bool MQ, int NW>
__global__ void __launch_bounds__(NW * 32, i8_min_blocks<D>(NW))
    decode_i8_kernel(const float* __restrict__ params, const uint8_t* __restrict__ blocks,
                     const int32_t* __restrict__ page_table, int n_pages, int max_pages, int H,
                     const TQ* __restrict__ Q, int n_q_heads, int n_q,
                     const int32_t* __restrict__ seq_lens, float scale, int pages_per_split,
                     int n_splits, float* __restrict__ partials, uint32_t* status,
                     float* __restrict__ out, const I8Mul mk) {
  using SM = I8Smem<D, NST, RB, NW>;
  constexpr int E = D / 32;           // elements per lane in the warp WHT layout
  constexpr int NB = E / 4;
  constexpr int CB = code_bytes(D, 3);
  constexpr int BB = block_bytes(D, 3);
  constexpr int NG = D / 128;         // 32-dim groups per lane and token (groups t, t + 4)
  constexpr int NU = D / 128;         // unit pairs per lane in the V tile (g, g + 8)
  constexpr int MT = 8 * NU;          // m-tiles of the value product
  constexpr int PS = D + 4;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint32_t* afr = reinterpret_cast<uint32_t*>(smem + SM::kAOff);    // [D/32][32][4]
  uint32_t* afr2 = reinterpret_cast<uint32_t*>(smem + SM::kA2Off);  // [D/32][32][4]
  float* kf_row = reinterpret_cast<float*>(smem + SM::kKfOff);
  int* row_off = reinterpret_cast<int*>(smem + SM::kRowOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.x, s = blockIdx.z;
  // The CTA's RB rows are (query token i, query head) pairs of KV head hk: row r is pair
  // R = RB rb + r of the group's n_q * G pairs, i = R / G, head hk * G + R % G.  Query
  // token i of a sequence of len tokens sits at position len - n_q + i and attends the
  // tokens before and at it (n_q = 1: the decode, every row attends the whole context).
  if constexpr (!MQ) n_q = 1;
  const int G = n_q_heads / H;
  const int n_rows = n_q * G;
  const int nrb = (n_rows + RB - 1) / RB;
  const int hk = blockIdx.y / nrb, rb = blockIdx.y - hk * nrb;
  const int nh = min(RB, n_rows - rb * RB);      // rows handled here
  const int rg = RB == 8 ? g : (g & 3);           // this lane's score row
  auto row_token = [&](int r) { return (rb * RB + r) / G; };
  auto row_index = [&](int r) {                   // row of the sequence's output / partials
    const int R = rb * RB + r;
    return (R / G) * n_q_heads + hk * G + R % G;
  };

  int len = __ldg(seq_lens + s);
  if (len > max_pages * kPage) {
    if (tid == 0 && split == 0 && blockIdx.y == 0) set_status(status, ISOQ_ST_LEN_RANGE);
    len = max_pages * kPage;
  }
  // causal limits: lim(r) = len - n_q + 1 + i(r), clamped to [0, len]
  const int lim_lo = MQ ? max(0, min(len, len - n_q + 1 + row_token(0))) : len;
  const int lim_hi = MQ ? max(0, min(len, len - n_q + 1 + row_token(nh - 1))) : len;
  const int lim_g = MQ && rg < nh ? max(0, min(len, len - n_q + 1 + row_token(rg))) : lim_hi;
  const int p_begin = split * pages_per_split;
  const int p_end = min((lim_hi + kPage - 1) / kPage, p_begin + pages_per_split);

  float* out_base = partials + ((size_t)s * n_q * n_q_heads) * n_splits * PS + (size_t)split * PS;
  // extents of the checked build: partials / Q rows of the launch, the head's parameters
  [[maybe_unused]] const size_t parts_len = (size_t)gridDim.z * n_q * n_q_heads * n_splits * PS;
  [[maybe_unused]] const size_t q_rows = (size_t)gridDim.z * n_q * n_q_heads;
  [[maybe_unused]] const size_t out_off0 = out_base - partials;
  if (tid < RB) row_off[tid] = tid < nh ? row_index(tid) : 0;
  __syncthreads();
  // extent of the direct output (single chunk): [gridDim.z][n_q_heads][D]
  [[maybe_unused]] const size_t out_len = (size_t)gridDim.z * n_q_heads * D;
  if (p_begin >= p_end) {  // empty chunk: m = -inf, l = 0, acc = 0
    if (out != nullptr) {  // the whole context is empty: zero output rows
      for (int i = tid; i < nh * D; i += blockDim.x) {
        const int h = i / D, c = i - h * D;
        const size_t o = ((size_t)s * n_q_heads + row_off[h]) * D + c;
        if (in_bounds(o < out_len, status)) out[o] = 0.f;
      }
      return;
    }
    for (int i = tid; i < nh * PS; i += blockDim.x) {
      const int h = i / PS, c = i - h * PS;
      const size_t o = (size_t)row_off[h] * n_splits * PS + c;
      if (in_bounds(out_off0 + o < parts_len, status))
        out_base[o] = (c == D) ? -CUDART_INF_F : 0.f;
    }
    return;
  }

  // ---- barriers, then prefetch the first pages of every warp --------------------------
  uint64_t* mybar = bars + warp * NST;
  uint8_t* myring = smem + warp * NST * BB;
  if (lane == 0) {
    for (int i = 0; i < NST; ++i) mbar_init(mybar + i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const int* pt_row = page_table + (size_t)s * max_pages;
  // page k of this warp = p_begin + warp + NW * k
  const int n_my = (p_end - p_begin - warp + NW - 1) / NW;  // may be <= 0
  auto issue = [&](int k) {  // lane 0 only
    const int pg = p_begin + warp + NW * k;
    const int st = k % NST;
    const int phys = in_bounds(pg < max_pages && st < NST, status) ? __ldg(pt_row + pg) : -1;
    if (phys >= 0 && phys < n_pages && in_bounds(hk < H, status)) {
      mbar_expect_tx(mybar + st, BB);
      bulk_copy(myring + st * BB, blocks + ((size_t)phys * H + hk) * BB, BB, mybar + st);
    } else {
      set_status(status, ISOQ_ST_PAGE_RANGE);
      mbar_arrive(mybar + st);  // complete the phase without data; tokens are masked
    }
  };
  if (lane == 0)
    for (int k = 0; k < NST && k < n_my; ++k) issue(k);
  int issued = min(NST, max(n_my, 0));  // warp-uniform count of copies issued

  // ---- a6: rotate the CTA's queries (unnormalised WHT + SO(4)), scale each row to a
  // 24-bit integer and store its balanced digits as the score mma's A fragments.  k-step
  // kb, lane (g', t') covers dims base..base+7, base = 32 (t' + 4 (kb / 4)) + 8 (kb % 4):
  // bytes 0-3 of a0/a1 are dims base..base+3, of a2/a3 dims base+4..base+7.
  {
    const float* hp = params + (size_t)hk * D * 4;  // this head's block matrices
    float pq[NB][16];
#pragma unroll
    for (int k = 0; k < NB; ++k)
      if (in_bounds(hk < H && lane * NB + k < D / 4, status)) load_block_mat(hp, lane * NB + k, pq[k]);
    for (int r = warp; r < RB; r += NW) {
      float v[E];
      if (r < nh) {
        const TQ* qp = Q + ((size_t)s * n_q * n_q_heads + row_off[r]) * D + lane * E;
#pragma unroll
        for (int i = 0; i < E; ++i)
          v[i] = in_bounds((size_t)s * n_q * n_q_heads + row_off[r] < q_rows, status)
                     ? to_f32<TQ>(qp[i]) : 0.f;
      } else {
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] = 0.f;
      }
      wht_warp<E>(v, lane);
      float z[E];
#pragma unroll
      for (int k = 0; k < NB; ++k) mat_fwd(pq[k], v + 4 * k, z + 4 * k);
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < E; ++i) amax = fmaxf(amax, fabsf(z[i]));
      amax = warp_max(amax);
      const float S = amax > 0.f ? kQMax / amax : 0.f;
      // log2 score per (integer score / 2^16 * nK): the unnormalised WHT makes z = sqrt(d)
      // q~ and K_hat = (nK / sqrt(d)) L, so q~.K_hat = nK (score / (S 10000)) / d
      if (lane == 0 && in_bounds(r < 8, status))
        kf_row[r] = S > 0.f ? scale * kLog2e * 65536.0f / (kLevelScale * (float)D * S) : 0.f;
      // this lane's E dims: lane * E .. + E-1 = E/4 runs of 4 dims (one A register each)
#pragma unroll
      for (int k = 0; k < NB; ++k) {
        const int base = lane * E + 4 * k;  // dims base..base+3
        int d2[4], d1[4], d0[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) digits3(__float2int_rn(z[4 * k + e] * S), d2[e], d1[e], d0[e]);
        const uint32_t w2 = pack_s8x4(d2[0], d2[1], d2[2], d2[3]);
        const uint32_t w1 = pack_s8x4(d1[0], d1[1], d1[2], d1[3]);
        const uint32_t w0 = pack_s8x4(d0[0], d0[1], d0[2], d0[3]);
        // base = 32 q + 8 u + 4 hf: group q -> lane t' = q % 4, k-step 4 (q / 4) + u; hf
        // selects a0/a1 (dims +0..3) or a2/a3 (dims +4..7)
        const int q = base >> 5, u = (base >> 3) & 3, hf = (base >> 2) & 1;
        const int kb = 4 * (q >> 2) + u, tq = q & 3;
        if (!in_bounds(kb < D / 32 && r < RB && tq < 4, status)) continue;
        if constexpr (RB == 8) {
          // lane (g' = r, t' = tq): A1 = (d2, d1, d2+4, d1+4), A2 = (0, d0, 0, d0+4)
          uint32_t* f = afr + (kb * 32 + 4 * r + tq) * 4;
          f[2 * hf] = w2;
          f[2 * hf + 1] = w1;
          uint32_t* f2 = afr2 + (kb * 32 + 4 * r + tq) * 4;  // A2 = [0; d0]
          f2[2 * hf] = 0u;
          f2[2 * hf + 1] = w0;
        } else {
          // A1: rows 0-3: d2 of rows r, 4-7: d1, 8-11: d0 (12-15 zero); A2: the same
          // without d0.  Lanes g' = r and r + 4.
          uint32_t* fa = afr + (kb * 32 + 4 * r + tq) * 4;         // g' = r
          uint32_t* fb = afr + (kb * 32 + 4 * (r + 4) + tq) * 4;   // g' = r + 4
          uint32_t* ga = afr2 + (kb * 32 + 4 * r + tq) * 4;
          uint32_t* gb = afr2 + (kb * 32 + 4 * (r + 4) + tq) * 4;
          fa[2 * hf] = w2;      // row r
          fa[2 * hf + 1] = w0;  // row r + 8
          fb[2 * hf] = w1;      // row r + 4
          fb[2 * hf + 1] = 0u;  // row r + 12
          ga[2 * hf] = w2;
          ga[2 * hf + 1] = 0u;
          gb[2 * hf] = w1;
          gb[2 * hf + 1] = 0u;
        }
      }
    }
    if constexpr (RB == 4) {  // rows nh..3 of lanes g' >= 4 are written above (r < RB)
    }
  }
  __syncthreads();

  const float kf = kf_row[rg];
  // level byte tables: the scores' integer level bytes and the value product's f16 level
  // bytes (ALPHA times the levels).  They are constants, but opaque to the compiler here:
  // otherwise it rebuilds a table word with a move before every byte permute instead of
  // keeping the eight words in registers.
  uint32_t tl0, tl1, th0, th1;
  level_tables<3>(tl0, tl1, th0, th1);
  uint32_t kh0 = kTH0, kh1 = kTH1, kl0 = kTL0, kl1 = kTL1;
  asm volatile("" : "+r"(tl0), "+r"(tl1), "+r"(th0), "+r"(th1));
  asm volatile("" : "+r"(kh0), "+r"(kh1), "+r"(kl0), "+r"(kl1));
  constexpr float ALPHA = alpha_of<3>();

  // Softmax state of row rg (the score rows of this lane); the value accumulator columns
  // of this lane are rows 2t, 2t+1 (RB = 4: columns 4-7 unused), whose rescale factors come
  // from lanes 8t and 8t + 4.
  float m2 = -CUDART_INF_F;  // running max of the log2 scores of row rg
  float lsum = 0.f;          // this lane's share of sum p of row rg
  float sigma = 0.f;         // V-norm reference (warp-uniform)
  float inv_sigma = 0.f;
  float acc[MT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  bool timed_out = false;
  int k = 0;
  for (; k < n_my; ++k) {
    const int st = k % NST;
    if (!mbar_wait(mybar + st, (k / NST) & 1)) {
      timed_out = true;
      break;
    }
    const uint8_t* blk = myring + st * BB;
    const int pg = p_begin + warp + NW * k;
    const int phys = in_bounds(pg < max_pages && st < NST, status) ? __ldg(pt_row + pg) : -1;
    const bool page_ok = phys >= 0 && phys < n_pages;
    const int tok0 = pg * kPage;

    // a page whose 64 tokens are all valid takes the tile body without masking
    const bool full = page_ok && tok0 + kPage <= lim_lo;
    auto tile = [&](const int tb, auto full_c) {
      constexpr bool FULL = decltype(full_c)::value;
      // ---- a7: scores of 4 tiles of 8 tokens; B = K_hat^T of token tb + 8n + g ----------
      // NT tiles at a time share each load of the query fragments
      float sv[4][2];  // log2-domain scores of tokens tb + 8n + 2t + c (row rg)
#pragma unroll
      for (int n0 = 0; n0 < 4; n0 += kI8NT) {
        // RB = 8: C1 = [d2.kh; d1.kh], C2 = [d2.kl; d1.kl + d0.kh]
        int C1[kI8NT][4], C2[kI8NT][4];
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
          uint32_t w[kI8NT][3], wt[kI8NT][3];
#pragma unroll
          for (int nn = 0; nn < kI8NT; ++nn) {
            const int ko = (tb + 8 * (n0 + nn) + g) * CB + 12 * (t + 4 * gq);
            const uint32_t* p = reinterpret_cast<const uint32_t*>(blk + ko);
            const bool kin = in_bounds(ko + 12 <= kPage * CB, status);
#pragma unroll
            for (int j = 0; j < 3; ++j) {
              w[nn][j] = kin ? p[j] : 0u;
              wt[nn][j] = top_bits(w[nn][j]);
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int kb = 4 * gq + u;
            const bool ain = in_bounds(kb < D / 32, status);
            const uint4 A1 = ain ? *reinterpret_cast<const uint4*>(afr + (kb * 32 + lane) * 4)
                                 : make_uint4(0, 0, 0, 0);
            const uint4 A2 = ain ? *reinterpret_cast<const uint4*>(afr2 + (kb * 32 + lane) * 4)
                                 : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int nn = 0; nn < kI8NT; ++nn) {
              const uint32_t S = u < 3 ? sel_word(w[nn][u], wt[nn][u], mk)
                                       : sel_spare(wt[nn][0], wt[nn][1], wt[nn][2]);
              const uint32_t S2 = S >> 16;
              const uint32_t bh0 = prmt(kh0, kh1, S), bh1 = prmt(kh0, kh1, S2);
              const uint32_t bl0 = prmt(kl0, kl1, S), bl1 = prmt(kl0, kl1, S2);
              // the first k-step starts the accumulators from zero
              auto step = [&](auto first) {
                constexpr bool F = decltype(first)::value;
                mma_s8_acc<F>(C1[nn], A1, bh0, bh1);
                if constexpr (RB == 8) {
                  mma_s8_acc<F>(C2[nn], A1, bl0, bl1);
                  mma_s8_acc<false>(C2[nn], A2, bh0, bh1);
                } else {
                  mma_s8_acc<F>(C2[nn], A2, bl0, bl1);
                }
              };
              if (gq == 0 && u == 0) step(std::true_type{});
              else step(std::false_type{});
            }
          }
        }
        // tokens tb + 8n + 2t + c: raw = (integer score) / 2^16
#pragma unroll
        for (int nn = 0; nn < kI8NT; ++nn) {
          const int n = n0 + nn;
          const int tk = tb + 8 * n + 2 * t;
          const float2 nk2 = in_bounds(tk + 2 <= kPage, status)
              ? __half22float2(*reinterpret_cast<const __half2*>(blk + k_norm_off(D, 3) + 2 * tk))
              : make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float raw;
            if constexpr (RB == 8) {
              const int Z = C1[nn][c] * 256 + (C2[nn][c] + C1[nn][2 + c]);
              raw = fmaf((float)C2[nn][2 + c], 1.0f / 256.0f, (float)Z);
            } else {
              // lanes g < 4: d2.kh, d0.kh (row g + 8), d2.kl; lanes g >= 4: d1.kh, d1.kl
              const bool top = g < 4;
              const int hi = top ? C1[nn][c] * 256 + C2[nn][c] : C1[nn][c];
              const int lo = top ? C1[nn][2 + c] : C2[nn][c];
              const float part = fmaf((float)lo, 1.0f / 256.0f, (float)hi);
              raw = part + __shfl_xor_sync(kFull, part, 16);
            }
            sv[n][c] = raw * ((c ? nk2.y : nk2.x) * kf);
          }
        }
      }

      // norms of this lane's V tokens (the same 8 tokens) and the masks
      float nv[4][2];
      const float sthr = m2 + kLazy, vthr = sigma * kSigmaSlack;
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const int tk = tb + 8 * n + 2 * t;
        const float2 nv2 = in_bounds(tk + 2 <= kPage, status)
            ? __half22float2(*reinterpret_cast<const __half2*>(blk + v_norm_off(D, 3) + 2 * tk))
            : make_float2(0.f, 0.f);
        nv[n][0] = nv2.x;
        nv[n][1] = nv2.y;
        if constexpr (!FULL) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const bool vld = page_ok && (tok0 + tk + c) < lim_hi;
            sv[n][c] = vld && (!MQ || (tok0 + tk + c) < lim_g) ? sv[n][c] : -CUDART_INF_F;
            nv[n][c] = vld ? nv[n][c] : 0.f;
          }
        }
      }
      // this lane's largest score and V norm of the tile (three-input max instructions)
      float tmax = fmaxf(fmaxf(fmaxf(sv[0][0], sv[0][1]), fmaxf(sv[1][0], sv[1][1])),
                         fmaxf(fmaxf(sv[2][0], sv[2][1]), fmaxf(sv[3][0], sv[3][1])));
      float vmax = fmaxf(fmaxf(fmaxf(nv[0][0], nv[0][1]), fmaxf(nv[1][0], nv[1][1])),
                         fmaxf(fmaxf(nv[2][0], nv[2][1]), fmaxf(nv[3][0], nv[3][1])));
      const bool grow = (tmax > sthr) | (vmax > vthr);
      // ---- a8: online softmax.  The running max m2 of a row (shared by the 4 lanes t)
      // and the V-norm reference sigma move only when a score exceeds m2 + 8 or a norm
      // exceeds 16 sigma (first tile included), so the common tile needs no shuffles.
      if (__any_sync(kFull, grow)) {
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
          tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, o));
          vmax = fmaxf(vmax, __shfl_xor_sync(kFull, vmax, o));
        }
        float resc = 1.f;
        if (tmax > sthr) {
          resc = ex2(m2 - tmax);  // 0 when m2 was -inf
          lsum *= resc;
          m2 = tmax;
        }
        float vr = 1.f;
        if (vmax > vthr) {   // warp-uniform
          vr = sigma / vmax;  // 0 on the first valid tile
          sigma = vmax;
          inv_sigma = 1.f / vmax;
        }
        // columns 2t, 2t+1 are rows 2t, 2t+1 (RB = 4: rows 2t & 3, unused for t >= 2)
        const float r0 = __shfl_sync(kFull, resc, 4 * ((2 * t) % RB)) * vr;
        const float r1 = __shfl_sync(kFull, resc, 4 * ((2 * t + 1) % RB)) * vr;
#pragma unroll
        for (int i = 0; i < MT; ++i) {
          acc[i][0] *= r0;
          acc[i][1] *= r1;
          acc[i][2] *= r0;
          acc[i][3] *= r1;
        }
      }
      // P'^T B fragments of the value mma: 16-token block jb = score tiles 2jb, 2jb+1;
      // b0 = tile 2jb's tokens 2t, 2t+1, b1 = tile 2jb+1's, column = row g (RB = 4: rows
      // 4-7 are zero)
      uint32_t pb[2][2];
      const bool col_live = RB == 8 || g < 4;
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        float p0 = ex2(sv[n][0] - m2), p1 = ex2(sv[n][1] - m2);
        if constexpr (!FULL) {  // a masked token while m2 is still -inf: -inf - -inf
          p0 = sv[n][0] != -CUDART_INF_F ? p0 : 0.f;
          p1 = sv[n][1] != -CUDART_INF_F ? p1 : 0.f;
        }
        lsum += p0 + p1;
        const uint32_t w = pack_f16x2(p0 * (nv[n][0] * inv_sigma), p1 * (nv[n][1] * inv_sigma));
        pb[n >> 1][n & 1] = col_live ? w : 0u;
      }

      // ---- a8: V accumulation, A = V_hat^T (rows = dims, k = the block's tokens) --------
#pragma unroll
      for (int up = 0; up < NU; ++up) {
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
          // this lane's 24 bytes of the 16-token block: units 2 (g + 8 up), +1 of quad t
          uint32_t W[6];
          const int vo = ((tb >> 4) + jb) * 6 * D + vt_group_off(D, 0, t, 2 * (g + 8 * up));
          const uint2* src = reinterpret_cast<const uint2*>(blk + v_codes_off(D, 3) + vo);
          const bool vin = in_bounds(vo + 24 <= kPage * CB, status);
#pragma unroll
          for (int i = 0; i < 3; ++i) {
            const uint2 w = vin ? src[i] : make_uint2(0, 0);
            W[2 * i] = w.x;
            W[2 * i + 1] = w.y;
          }
#pragma unroll
          for (int p = 0; p < 2; ++p) {      // unit 2 (g + 8 up) + p
            const uint32_t* w = W + 3 * p;
            const uint32_t wt0 = top_bits(w[0]), wt1 = top_bits(w[1]), wt2 = top_bits(w[2]);
            const uint32_t Sp = sel_spare(wt0, wt1, wt2);
#pragma unroll
            for (int b = 0; b < 4; ++b) {    // words 0..2, then the spare unit
              const int mt = 8 * up + 4 * p + b;
              const uint32_t S = b == 0 ? sel_word(w[0], wt0, mk)
                               : b == 1 ? sel_word(w[1], wt1, mk)
                               : b == 2 ? sel_word(w[2], wt2, mk) : Sp;
              // low half: dim 8u + 2b of members 0-3 (row g); high half: dim + 1 (row g+8)
              const uint32_t Sh = S >> 16;
              const uint32_t le = prmt(tl0, tl1, S), he = prmt(th0, th1, S);
              const uint32_t lo = prmt(tl0, tl1, Sh), ho = prmt(th0, th1, Sh);
              mma16816(acc[mt], prmt(le, he, 0x5140u), prmt(lo, ho, 0x5140u),
                       prmt(le, he, 0x7362u), prmt(lo, ho, 0x7362u), pb[jb][0], pb[jb][1]);
            }
          }
        }
      }
    };
#pragma unroll
    for (int tb = 0; tb < kPage; tb += 32) {
      if (full) tile(tb, std::true_type{});
      else tile(tb, std::false_type{});
    }
    __syncwarp();
    // stage st is consumed: refill it with page k + NST
    if (k + NST < n_my) {
      if (lane == 0) {
        fence_proxy_async();
        issue(k + NST);
      }
      ++issued;
    }
  }

  if (timed_out) {
    if (lane == 0) set_status(status, ISOQ_ST_TIMEOUT);
    // copies k .. issued-1 may still be in flight: wait for them (bounded) before the
    // CTA's shared memory can be reused or released
    for (int kk = k; kk < issued; ++kk)
      if (!mbar_wait(mybar + (kk % NST), (kk / NST) & 1)) break;
  }

  // the combine (launched as a programmatic dependent) may be scheduled from here on; it
  // waits in-kernel until this grid has completed and its writes are visible
  asm volatile("griddepcontrol.launch_dependents;");

  // ---- merge the warps' states in shared memory, write the chunk's partials -----------
  // row rg's sum p over the lanes t (RB = 4: lanes g and g + 4 hold the same row)
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) lsum += __shfl_xor_sync(kFull, lsum, o);
  __syncthreads();  // all warps done with their rings
  float* mb = reinterpret_cast<float*>(smem);  // [NW][8 rows][D + 4]
  {
    // acc_true = acc * sigma / ALPHA (times 1 / exp2(m2) in the log2 frame).  Lane (g, t):
    // m-tile mt = 8 up + 4 p + b, rows g / g + 8 = dims 8u + 2b / + 1 with u = 2 (g + 8 up)
    // + p (b = 3: the spare unit, dims 8u + 6, 8u + 7); columns 2t, 2t+1 = rows
    const float f = sigma / ALPHA;
    if (2 * t < RB) {
#pragma unroll
      for (int up = 0; up < NU; ++up)
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const int mt = 8 * up + 4 * p + b;
            const int d0 = 8 * (2 * (g + 8 * up) + p) + 2 * b;
            if (!in_bounds(d0 + 1 < D && 2 * t + 1 < 8, status)) continue;
            float* r0 = mb + (warp * 8 + 2 * t) * PS;
            float* r1 = mb + (warp * 8 + 2 * t + 1) * PS;
            r0[d0] = acc[mt][0] * f;
            r1[d0] = acc[mt][1] * f;
            r0[d0 + 1] = acc[mt][2] * f;
            r1[d0 + 1] = acc[mt][3] * f;
          }
    }
    if (t == 0 && g < RB) {
      float* r = mb + (warp * 8 + g) * PS;
      r[D] = m2;
      r[D + 1] = lsum;
    }
  }
  __syncthreads();
  for (int i = tid; i < nh * (D + 1); i += blockDim.x) {
    const int h = i / (D + 1), c = i - h * (D + 1);
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mb[(w * 8 + h) * PS + D]);
    float v = 0.f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float mw = mb[(w * 8 + h) * PS + D];
        if (mw == -CUDART_INF_F) continue;
        const float sc = ex2(mw - M);
        v += sc * mb[(w * 8 + h) * PS + (c == D ? D + 1 : c)];
      }
    }
    if (out != nullptr) {  // single chunk: the merged row goes on to the rotation below
      if (in_bounds(NW * 8 * PS + h * (D + 1) + c < SM::kRing / 4, status))
        mb[NW * 8 * PS + h * (D + 1) + c] = v;
      continue;
    }
    float* o = out_base + (size_t)row_off[h] * n_splits * PS;
    if (!in_bounds(out_off0 + (size_t)row_off[h] * n_splits * PS + D + 1 < parts_len, status)) continue;
    if (c < D) o[c] = v;
    else {
      o[D] = M == -CUDART_INF_F ? -CUDART_INF_F : M / kLog2e;  // natural-log units
      o[D + 1] = v;
    }
  }
  if (out == nullptr) return;
  // ---- a9 for a single chunk: o = acc / l, inverse SO(4) blocks, inverse WHT, as the
  // combine computes it for one part (bitwise the same); a warp per row
  __syncthreads();
  const float* fin = mb + NW * 8 * PS;  // [nh][D + 1]: acc, l
  const float* hp = params + (size_t)hk * D * 4;
  float Mb[NB][16];
#pragma unroll
  for (int k = 0; k < NB; ++k)
    if (in_bounds(hk < H && lane * NB + k < D / 4, status)) load_block_mat(hp, lane * NB + k, Mb[k]);
  for (int h = warp; h < nh; h += NW) {
    const float Ls = fin[h * (D + 1) + D];
    const float inv = Ls > 0.f ? 1.f / (Ls * sqrtf((float)D)) : 0.f;
    float o[E];
#pragma unroll
    for (int i = 0; i < E; ++i) o[i] = fin[h * (D + 1) + lane * E + i] * inv;
    float y[E];
#pragma unroll
    for (int k = 0; k < NB; ++k) mat_inv(Mb[k], o + 4 * k, y + 4 * k);
    wht_warp<E>(y, lane);
    const float rs = rsqrtf((float)D);
    const size_t ob = ((size_t)s * n_q_heads + row_off[h]) * D + lane * E;
    if (!in_bounds(ob + E <= out_len, status)) continue;
#pragma unroll
    for (int i = 0; i < E; ++i) out[ob + i] = y[i] * rs;
  }
}

template <int D, int NST, int RB, typename TQ, bool MQ, int NW>
cudaError_t launch_i8_t(const DecodeArgs& a, cudaStream_t stream, float* direct_out) {
  using SM = I8Smem<D, NST, RB, NW>;
  // the dynamic shared-memory opt-in is per function and per device
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_i8_kernel<D, NST, RB, TQ, MQ, NW>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  const int G = a.n_q_heads / a.n_kv_heads;
  dim3 grid(a.n_splits, a.n_kv_heads * ((a.n_q * G + RB - 1) / RB), a.n_seqs);
  decode_i8_kernel<D, NST, RB, TQ, MQ, NW><<<grid, NW * 32, SM::kBytes, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_kv_heads,
      static_cast<const TQ*>(a.Q), a.n_q_heads, a.n_q, a.seq_lens, a.scale, a.pages_per_split,
      a.n_splits, a.partials, a.status, direct_out,
      I8Mul{0xFFFFFFFFu});
  return cudaGetLastError();
}

// Wide CTAs (more warps, one CTA per SM) when the whole grid fits in one CTA per SM: the
// GPU would otherwise run a small decode with a few warps per SM, each walking its pages
// one after another.
template <int D, int NST, int RB, typename TQ, bool MQ>
cudaError_t launch_i8_w(const DecodeArgs& a, cudaStream_t stream, float* direct_out) {
  constexpr int kWide = D == 128 ? 16 : 8;
  const int G = a.n_q_heads / a.n_kv_heads;
  const long long ctas =
      (long long)a.n_splits * a.n_kv_heads * ((a.n_q * G + RB - 1) / RB) * a.n_seqs;
  if (ctas <= (long long)decode_i8_sms())
    return launch_i8_t<D, NST, RB, TQ, MQ, kWide>(a, stream, direct_out);
  return launch_i8_t<D, NST, RB, TQ, MQ, 4>(a, stream, direct_out);
}

template <int D, int NST, int RB>
cudaError_t launch_i8_rb(const DecodeArgs& a, cudaStream_t stream, float* direct_out) {
  const bool mq = a.n_q > 1;
  switch (a.q_dtype) {
    case ISOQ_F32:
      return mq ? launch_i8_w<D, NST, RB, float, true>(a, stream, nullptr)
                : launch_i8_w<D, NST, RB, float, false>(a, stream, direct_out);
    case ISOQ_BF16:
      return mq ? launch_i8_w<D, NST, RB, __nv_bfloat16, true>(a, stream, nullptr)
                : launch_i8_w<D, NST, RB, __nv_bfloat16, false>(a, stream, direct_out);
    case ISOQ_F16:
      return mq ? launch_i8_w<D, NST, RB, __half, true>(a, stream, nullptr)
                : launch_i8_w<D, NST, RB, __half, false>(a, stream, direct_out);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

#ifndef ISOQ_I8_NST128
#define ISOQ_I8_NST128 2
#endif
#ifndef ISOQ_I8_NST256
#define ISOQ_I8_NST256 2
#endif

#ifndef ISOQ_I8_DIRECT  // single-chunk decodes write their output without the combine
#define ISOQ_I8_DIRECT 1
#endif

cudaError_t launch_decode_split_i8(const DecodeArgs& a, cudaStream_t stream, bool* combined) {
  if (combined) *combined = false;
  if (a.bits != 3) return cudaErrorInvalidValue;
  const bool direct = ISOQ_I8_DIRECT && combined && a.n_splits == 1 && a.n_q == 1 &&
                      a.state == nullptr && a.out != nullptr;
  float* out = direct ? a.out : nullptr;
  const int rb = decode_rows_per_block(a.d, a.n_q, a.n_q_heads / a.n_kv_heads);
  cudaError_t e = cudaErrorInvalidValue;
  if (a.d == 128)
    e = rb == 8 ? launch_i8_rb<128, ISOQ_I8_NST128, 8>(a, stream, out)
                : launch_i8_rb<128, ISOQ_I8_NST128, 4>(a, stream, out);
  else if (a.d == 256)
    e = launch_i8_rb<256, ISOQ_I8_NST256, 4>(a, stream, out);
  if (e == cudaSuccess && combined) *combined = direct;
  return e;
}

// Resident 4-warp CTAs per SM of the decode kernel for head dimension d on the current
// device (cached per device; 2 when it cannot be queried).
int decode_i8_resident_ctas(int d) {
  static int cache[64][2] = {{0}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 2;
  }
  const int di = d == 256 ? 1 : 0;
  if (!cache[dev][di]) {
    int n = 0;
    cudaError_t e;
    if (d == 256) {
      using SM = I8Smem<256, ISOQ_I8_NST256, 4, 4>;
      auto k = decode_i8_kernel<256, ISOQ_I8_NST256, 4, __nv_bfloat16, false, 4>;
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, 4 * 32, SM::kBytes);
    } else {
      using SM = I8Smem<128, ISOQ_I8_NST128, 8, 4>;
      auto k = decode_i8_kernel<128, ISOQ_I8_NST128, 8, __nv_bfloat16, false, 4>;
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, 4 * 32, SM::kBytes);
    }
    if (e != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 2;
    }
    cache[dev][di] = n;
  }
  return cache[dev][di];
}

// SM count of the current device (148 when it cannot be queried).
int decode_i8_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
    cudaGetLastError();
    sms = 148;
  }
  return sms;
}

}  // namespace isoq
