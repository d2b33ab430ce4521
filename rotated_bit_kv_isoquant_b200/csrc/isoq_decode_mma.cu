// Tensor-core decode attention on the packed 3-bit cache (split-K partials).
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: attention is computed on the packed 3-bit codes
// and full-precision K/V are never reconstructed.  With R orthogonal, q.k_hat =
// (R q).(R k_hat), so the group's queries are rotated once per CTA and everything else
// happens on codebook levels in the rotated space.
//
// Work: one CTA of 4 warps per (context chunk, KV head, block of <= 8 query heads,
// sequence).  Each warp streams its own pages of the chunk through a private ring of
// shared-memory stages filled by 1-D bulk copies (cp.async.bulk, one page block per copy,
// completion on an mbarrier; every wait is bounded).  Per 32-token tile:
//   scores  S[16 x 8 tok] = Q~2[16 x d] . K_hat^T[d x 8 tok]  (mma.sync m16n8k16, f16 ->
//           f32, 4 tiles of 8 tokens; rows 0-7 of Q~2 are the heads' f16 high parts,
//           rows 8-15 the low parts, so one mma carries both and their sum is the score)
//   online softmax per head, P' = p * nV / sigma, rescaled only when a running maximum
//           grows (lazy), so the common tile needs no shuffles
//   out^T[d x 8 heads] += V_hat^T[d x 16 tok] . P'^T  (mma.sync; the score accumulator of
//           two 8-token tiles is already the P'^T fragment, no transpose)
// K_hat / V_hat are never stored: each thread turns its codes into f16 mma fragments in
// registers with byte permutes (prmt) against 8-entry tables of the levels' low and high
// bytes.  The packed layout puts 24 of every 32 codes in nibbles (bit 3 clear), which is
// exactly a prmt byte selector; the other 8 come from the spare bit 3 of three words.
// Levels are scaled by ALPHA, a constant for which all four magnitudes round to binary16
// with relative error < 2e-5 (1/ALPHA is folded into the score and output scales).
// The 2- and 4-bit variants (d = 128) swap in their own unit dequantisers (isoq_ptx.cuh):
// 4 bits look up the magnitude nibble and flip the sign bit; 2 bits turn two codes into
// one selector with a multiply-add and look up an f16x2 in a single byte permute.
#include <math_constants.h>

#include <type_traits>

#include "isoq_check.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"

namespace isoq {
using namespace ptx;


// Dynamic shared memory: [kWarps][NST] page stages of block_bytes(D), then the mbarriers,
// then the score mma's A fragments of the rotated queries (one uint4 per k-step and lane,
// shared by the four warps).  The stage area is reused for the final merge.
template <int D, int NST, int BITS = 3>
struct MmaSmem {
  static constexpr int kStageBytes = block_bytes(D, BITS);
  static constexpr int kRing = kWarps * NST * kStageBytes;
  static constexpr int kBarOff = kRing;
  static constexpr int kAOff = kBarOff + kWarps * NST * 8;
  static constexpr int kRowOff = kAOff + (D / 16) * 32 * 16;  // int [8]: output row per CTA row
  static constexpr int kBytes = kRowOff + 8 * 4;
  static constexpr int kMergeBytes = kWarps * 8 * (D + 4) * 4;
  static_assert(kMergeBytes <= kRing, "merge buffer must fit in the ring");
  static_assert(kAOff % 16 == 0, "A fragments must be 16-byte aligned");
};

// d = 128: <= 128 registers, 4 CTAs (16 warps) per SM; d = 256: two CTAs fill the shared
// memory, so registers are not the limit
template <int D>
constexpr int dec_min_blocks() { return D == 128 ? 4 : 2; }

// MQ: chunks of several query tokens per sequence with causal limits; the decode (one
// query token, every row attending the whole context) is compiled without them.
template <int D, int NST, typename TQ, bool MQ, int BITS>
__global__ void __launch_bounds__(kWarps * 32, dec_min_blocks<D>())
    decode_mma_kernel(const float* __restrict__ params, const uint8_t* __restrict__ blocks,
                      const int32_t* __restrict__ page_table, int n_pages, int max_pages, int H,
                      const TQ* __restrict__ Q, int n_q_heads, int n_q,
                      const int32_t* __restrict__ seq_lens, float scale, int pages_per_split,
                      int n_splits, float* __restrict__ partials, uint32_t* status) {
  using SM = MmaSmem<D, NST, BITS>;
  constexpr int E = D / 32;           // elements per lane in the warp WHT layout
  constexpr int NB = E / 4;
  constexpr int CB = code_bytes(D, BITS);
  constexpr int BB = block_bytes(D, BITS);
  constexpr int W = BITS;             // words per 32-dim group of a packed vector
  constexpr float ALPHA = alpha_of<BITS>();
  constexpr int KS = D / 16;          // k-steps of the score mma = m-tiles of the PV mma
  constexpr int NG = D / 128;         // 32-dim groups per thread and token (score: t, t+4)
  constexpr int PS = D + 4;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  uint4* qa = reinterpret_cast<uint4*>(smem + SM::kAOff);
  int* row_off = reinterpret_cast<int*>(smem + SM::kRowOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.x, s = blockIdx.z;
  // The CTA's 8 rows are (query token i, query head) pairs of KV head hk: row r is pair
  // R = 8 rb + r of the group's n_q * G pairs, i = R / G, head hk * G + R % G.  Query token
  // i of a sequence of len tokens sits at position len - n_q + i and attends the tokens
  // before and at it (n_q = 1: the decode, every row attends the whole context).
  if constexpr (!MQ) n_q = 1;
  const int G = n_q_heads / H;
  const int n_rows = n_q * G;
  const int nrb = (n_rows + 7) >> 3;
  const int hk = blockIdx.y / nrb, rb = blockIdx.y - hk * nrb;
  const int nh = min(8, n_rows - rb * 8);        // rows handled here
  auto row_token = [&](int r) { return (rb * 8 + r) / G; };
  auto row_index = [&](int r) {                  // row of the sequence's output / partials
    const int R = rb * 8 + r;
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
  const int lim_g =
      MQ && g < nh ? max(0, min(len, len - n_q + 1 + row_token(g))) : lim_hi;
  const int p_begin = split * pages_per_split;
  const int p_end = min((lim_hi + kPage - 1) / kPage, p_begin + pages_per_split);

  float* out_base = partials + ((size_t)s * n_q * n_q_heads) * n_splits * PS + (size_t)split * PS;
  // extents of the checked build: partials / Q rows of the launch
  [[maybe_unused]] const size_t parts_len = (size_t)gridDim.z * n_q * n_q_heads * n_splits * PS;
  [[maybe_unused]] const size_t q_rows = (size_t)gridDim.z * n_q * n_q_heads;
  [[maybe_unused]] const size_t out_off0 = out_base - partials;
  if (tid < 8) row_off[tid] = tid < nh ? row_index(tid) : 0;
  __syncthreads();
  if (p_begin >= p_end) {  // empty chunk: m = -inf, l = 0, acc = 0
    for (int i = tid; i < nh * PS; i += blockDim.x) {
      const int h = i / PS, c = i - h * PS;
      const size_t o = (size_t)row_off[h] * n_splits * PS + c;
      if (in_bounds(out_off0 + o < parts_len, status)) out_base[o] = (c == D) ? -CUDART_INF_F : 0.f;
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
  // page k of this warp = p_begin + warp + kWarps * k
  const int n_my = (p_end - p_begin - warp + kWarps - 1) / kWarps;  // may be <= 0
  auto issue = [&](int k) {  // lane 0 only
    const int pg = p_begin + warp + kWarps * k;
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

  // ---- a6: rotate the CTA's queries (unnormalised WHT + SO(4)) into the A fragments ----
  // Rows 0-7 of the score mma's A are the f16 high parts of the 8 heads' rotated queries,
  // rows 8-15 the low parts (q = hi + lo to ~2^-22 relative; one f16 rounding of q alone
  // costs up to ~5e-3 relative error in the output when a few large scores dominate the
  // softmax), so one mma yields both products.  k-step kb of lane (g, t) covers dims
  // base..base+3, base = 32 (t + 4 (kb / 8)) + 4 (kb % 8):
  //   a0 = hi(g; base, base+1)  a1 = lo(g; base, base+1)
  //   a2 = hi(g; base+2, +3)    a3 = lo(g; base+2, +3)
  {
    const float* hp = params + (size_t)hk * D * 4;  // this head's block matrices
    float pq[NB][16];
#pragma unroll
    for (int k = 0; k < NB; ++k)
      if (in_bounds(hk < H && lane * NB + k < D / 4, status)) load_block_mat(hp, lane * NB + k, pq[k]);
    for (int h = warp; h < 8; h += kWarps) {
      float v[E];
      if (h < nh && in_bounds((size_t)s * n_q * n_q_heads + row_off[h] < q_rows, status)) {
        const TQ* qp = Q + ((size_t)s * n_q * n_q_heads + row_off[h]) * D + lane * E;
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] = to_f32<TQ>(qp[i]);
      } else {
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] = 0.f;
      }
      wht_warp<E>(v, lane);
      float z[E];
#pragma unroll
      for (int k = 0; k < NB; ++k) mat_fwd(pq[k], v + 4 * k, z + 4 * k);
#pragma unroll
      for (int k = 0; k < NB; ++k) {
        const int base = lane * E + 4 * k;  // dims base..base+3
        const int q = base >> 5;
        const int kb = 8 * (q >> 2) + ((base & 31) >> 2);
        float hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = __half2float(__float2half_rn(z[4 * k + e]));
          lo[e] = z[4 * k + e] - hi[e];
        }
        if (!in_bounds(kb < D / 16 && h < 8, status)) continue;
        qa[kb * 32 + h * 4 + (q & 3)] =
            make_uint4(pack_f16x2(hi[0], hi[1]), pack_f16x2(lo[0], lo[1]),
                       pack_f16x2(hi[2], hi[3]), pack_f16x2(lo[2], lo[3]));
      }
    }
  }
  __syncthreads();

  // level byte tables of the format (f16 of ALPHA times the levels or magnitudes)
  uint32_t tl0, tl1, th0, th1;
  level_tables<BITS>(tl0, tl1, th0, th1);

  // Softmax state of head g (the score rows of this lane); the PV accumulator columns of
  // this lane are heads 2t, 2t+1, whose rescale factors come from lanes 8t and 8t + 4.
  float m2 = -CUDART_INF_F;  // running max of the log2 scores of head g
  float lsum = 0.f;          // this lane's share of sum p of head g
  float sigma = 0.f;         // V-norm reference (warp-uniform)
  float inv_sigma = 0.f;
  float acc[KS][4];
#pragma unroll
  for (int i = 0; i < KS; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const float kf = scale * kLog2e / (ALPHA * (float)D);  // log2 score per (dot * nK)

  bool timed_out = false;
  int k = 0;
  for (; k < n_my; ++k) {
    const int st = k % NST;
    if (!mbar_wait(mybar + st, (k / NST) & 1)) {
      timed_out = true;
      break;
    }
    const uint8_t* blk = myring + st * BB;
    const int pg = p_begin + warp + kWarps * k;
    const int phys = in_bounds(pg < max_pages && st < NST, status) ? __ldg(pt_row + pg) : -1;
    const bool page_ok = phys >= 0 && phys < n_pages;
    const int tok0 = pg * kPage;

    // a page whose 64 tokens are all valid takes the tile body without masking
    const bool full = page_ok && tok0 + kPage <= lim_lo;
    auto tile = [&](const int tb, auto full_c) {
      constexpr bool FULL = decltype(full_c)::value;
      // ---- a7: scores of 4 tiles of 8 tokens; B = K_hat^T of token tb + 8n + g ------------
      float C[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n) C[n][0] = C[n][1] = C[n][2] = C[n][3] = 0.f;
#pragma unroll
      for (int gq = 0; gq < NG; ++gq) {
        uint32_t w[4][W];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          const int ko = (tb + 8 * n + g) * CB + 4 * W * (t + 4 * gq);
          const uint32_t* p = reinterpret_cast<const uint32_t*>(blk + ko);
          const bool kin = in_bounds(ko + 4 * W <= kPage * CB, status);
#pragma unroll
          for (int i = 0; i < W; ++i) w[n][i] = kin ? p[i] : 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool ain = in_bounds(8 * gq + 2 * j + 1 < D / 16, status);
          const uint4 A0 = ain ? qa[(8 * gq + 2 * j) * 32 + lane] : make_uint4(0, 0, 0, 0);
          const uint4 A1 = ain ? qa[(8 * gq + 2 * j + 1) * 32 + lane] : make_uint4(0, 0, 0, 0);
          uint32_t f[4][4];
#pragma unroll
          for (int n = 0; n < 4; ++n) kdeq<BITS>(w[n], j, tl0, tl1, th0, th1, f[n]);
#pragma unroll
          for (int n = 0; n < 4; ++n) mma16816(C[n], A0.x, A0.y, A0.z, A0.w, f[n][0], f[n][1]);
#pragma unroll
          for (int n = 0; n < 4; ++n) mma16816(C[n], A1.x, A1.y, A1.z, A1.w, f[n][2], f[n][3]);
        }
      }

      // tokens of this lane: tb + 8n + 2t + e (n = 0..3, e = 0, 1).  sv = log2-domain score
      // (-inf when masked), nv = V norm (0 when masked)
      float sv[4][2], nv[4][2];
      const float sthr = m2 + kLazy, vthr = sigma * kSigmaSlack;
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        const int tk = tb + 8 * n + 2 * t;
        const bool nin = in_bounds(tk + 2 <= kPage, status);
        const float2 nk2 = nin ? __half22float2(*reinterpret_cast<const __half2*>(
                                     blk + k_norm_off(D, BITS) + 2 * tk))
                               : make_float2(0.f, 0.f);
        const float2 nv2 = nin ? __half22float2(*reinterpret_cast<const __half2*>(
                                     blk + v_norm_off(D, BITS) + 2 * tk))
                               : make_float2(0.f, 0.f);
        sv[n][0] = (C[n][0] + C[n][2]) * (nk2.x * kf);
        sv[n][1] = (C[n][1] + C[n][3]) * (nk2.y * kf);
        nv[n][0] = nv2.x;
        nv[n][1] = nv2.y;
        if constexpr (!FULL) {
          const bool v0 = page_ok && (tok0 + tk) < lim_hi;
          const bool v1 = page_ok && (tok0 + tk + 1) < lim_hi;
          sv[n][0] = v0 && (!MQ || (tok0 + tk) < lim_g) ? sv[n][0] : -CUDART_INF_F;
          sv[n][1] = v1 && (!MQ || (tok0 + tk + 1) < lim_g) ? sv[n][1] : -CUDART_INF_F;
          nv[n][0] = v0 ? nv[n][0] : 0.f;
          nv[n][1] = v1 ? nv[n][1] : 0.f;
        }
      }
      // this lane's largest score and V norm of the tile (three-input max instructions)
      float tmax = fmaxf(fmaxf(fmaxf(sv[0][0], sv[0][1]), fmaxf(sv[1][0], sv[1][1])),
                         fmaxf(fmaxf(sv[2][0], sv[2][1]), fmaxf(sv[3][0], sv[3][1])));
      float vmax = fmaxf(fmaxf(fmaxf(nv[0][0], nv[0][1]), fmaxf(nv[1][0], nv[1][1])),
                         fmaxf(fmaxf(nv[2][0], nv[2][1]), fmaxf(nv[3][0], nv[3][1])));
      const bool grow = (tmax > sthr) | (vmax > vthr);
      // ---- a8: online softmax.  The running max m2 of head g (shared by the 4 lanes t)
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
        const float r0 = __shfl_sync(kFull, resc, 8 * t) * vr;
        const float r1 = __shfl_sync(kFull, resc, 8 * t + 4) * vr;
#pragma unroll
        for (int i = 0; i < KS; ++i) {
          acc[i][0] *= r0;
          acc[i][1] *= r1;
          acc[i][2] *= r0;
          acc[i][3] *= r1;
        }
      }
      // P'^T B fragments of the PV mma: k16 block jb = tiles 2jb, 2jb+1; b0 = tile 2jb's
      // tokens 2t, 2t+1, b1 = tile 2jb+1's, column = head g
      uint32_t pb[2][2];
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        float p0 = ex2(sv[n][0] - m2), p1 = ex2(sv[n][1] - m2);
        if constexpr (!FULL) {  // a masked token while m2 is still -inf: -inf - -inf
          p0 = sv[n][0] != -CUDART_INF_F ? p0 : 0.f;
          p1 = sv[n][1] != -CUDART_INF_F ? p1 : 0.f;
        }
        lsum += p0 + p1;
        pb[n >> 1][n & 1] = pack_f16x2(p0 * (nv[n][0] * inv_sigma), p1 * (nv[n][1] * inv_sigma));
      }

      // ---- a8: V accumulation, A = V_hat^T (rows = dims, k = tokens 2t,2t+1,2t+8,2t+9) --
#pragma unroll
      for (int jb = 0; jb < 2; ++jb) {
        const int r = tb + 16 * jb;
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
          const int q = (g >> 1) + 4 * gq;
          const uint8_t* vbase = blk + v_codes_off(D, BITS);
          const bool odd = (g & 1) != 0;  // odd g: units 2, 3 of the group, even g: 0, 1
          uint32_t S[4][2];  // [token 2t, 2t+1, 2t+8, 2t+9][unit j0, j0+1]
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int tk = r + 2 * t + (x & 1) + 8 * (x >> 1);
            const int vo = in_bounds(tk * CB + 4 * W * (q + 1) <= kPage * CB, status) ? tk * CB : 0;
            const uint32_t* w = reinterpret_cast<const uint32_t*>(vbase + vo) + W * q;
            if constexpr (BITS == 3) {  // unit 3 = the spare bits of the three words
              const uint32_t w0 = w[0], w1 = w[1], w2 = w[2];
              S[x][0] = (odd ? w2 : w0) & 0x77777777u;
              S[x][1] = odd ? spare_codes(w0, w1, w2) : (w1 & 0x77777777u);
            } else if constexpr (BITS == 4) {  // unit = word
              S[x][0] = w[odd ? 2 : 0];
              S[x][1] = w[odd ? 3 : 1];
            } else {  // two units per word, low half first
              const uint32_t w0 = w[odd ? 1 : 0];
              S[x][0] = w0;
              S[x][1] = w0 >> 16;
            }
          }
          // m-tile 4 ww + 2 part + hh: row g = nibble 4 part + 2 hh of word j0 + ww, row g+8
          // = the next nibble, so each A quad is two output pairs of two lookups
#pragma unroll
          for (int ww = 0; ww < 2; ++ww) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              uint32_t fa[4], fb[4];  // tokens (2t, 2t+1) and (2t+8, 2t+9)
              vdeq<BITS>(S[0][ww], S[1][ww], part, tl0, tl1, th0, th1, fa);
              vdeq<BITS>(S[2][ww], S[3][ww], part, tl0, tl1, th0, th1, fb);
#pragma unroll
              for (int hh = 0; hh < 2; ++hh)
                mma16816(acc[8 * gq + 4 * ww + 2 * part + hh], fa[2 * hh], fa[2 * hh + 1],
                         fb[2 * hh], fb[2 * hh + 1], pb[jb][0], pb[jb][1]);
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

  // ---- merge the 4 warps' states in shared memory, write the chunk's partials ---------
  // head g's sum p over the lanes t
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) lsum += __shfl_xor_sync(kFull, lsum, o);
  __syncthreads();  // all warps done with their rings
  float* mb = reinterpret_cast<float*>(smem);  // [kWarps][8 heads][D + 4]
  {
    // acc_true = acc * sigma / ALPHA (times 1 / exp2(m2) in the log2 frame)
    const float f = sigma / ALPHA;
#pragma unroll
    for (int gq = 0; gq < NG; ++gq) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int q = (g >> 1) + 4 * gq;
        const int j0 = 2 * (g & 1);
        const int d0 = 32 * q + 8 * j0 + 2 * mt;  // row g of m-tile; row g+8 is d0 + 1
        if (!in_bounds(d0 + 1 < D && 2 * t + 1 < 8, status)) continue;
        float* r0 = mb + (warp * 8 + 2 * t) * PS;
        float* r1 = mb + (warp * 8 + 2 * t + 1) * PS;
        r0[d0] = acc[8 * gq + mt][0] * f;
        r1[d0] = acc[8 * gq + mt][1] * f;
        r0[d0 + 1] = acc[8 * gq + mt][2] * f;
        r1[d0 + 1] = acc[8 * gq + mt][3] * f;
      }
    }
    if (t == 0) {
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
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mb[(w * 8 + h) * PS + D]);
    float v = 0.f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = mb[(w * 8 + h) * PS + D];
        if (mw == -CUDART_INF_F) continue;
        const float sc = ex2(mw - M);
        v += sc * mb[(w * 8 + h) * PS + (c == D ? D + 1 : c)];
      }
    }
    float* o = out_base + (size_t)row_off[h] * n_splits * PS;
    if (!in_bounds(out_off0 + (size_t)row_off[h] * n_splits * PS + D + 1 < parts_len, status)) continue;
    if (c < D) o[c] = v;
    else {
      o[D] = M == -CUDART_INF_F ? -CUDART_INF_F : M / kLog2e;  // natural-log units
      o[D + 1] = v;
    }
  }
}

template <int D, int NST, typename TQ, bool MQ, int BITS>
static cudaError_t launch_mma_t(const DecodeArgs& a, cudaStream_t stream) {
  using SM = MmaSmem<D, NST, BITS>;
  // the dynamic shared-memory opt-in is per function and per device
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_mma_kernel<D, NST, TQ, MQ, BITS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  const int G = a.n_q_heads / a.n_kv_heads;
  dim3 grid(a.n_splits, a.n_kv_heads * ((a.n_q * G + 7) / 8), a.n_seqs);
  decode_mma_kernel<D, NST, TQ, MQ, BITS><<<grid, kWarps * 32, SM::kBytes, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_kv_heads,
      static_cast<const TQ*>(a.Q), a.n_q_heads, a.n_q, a.seq_lens, a.scale, a.pages_per_split,
      a.n_splits, a.partials, a.status);
  return cudaGetLastError();
}

template <int D, int NST, int BITS>
cudaError_t launch_decode_mma_b(const DecodeArgs& a, cudaStream_t stream) {
  const bool mq = a.n_q > 1;
  switch (a.q_dtype) {
    case ISOQ_F32:
      return mq ? launch_mma_t<D, NST, float, true, BITS>(a, stream)
                : launch_mma_t<D, NST, float, false, BITS>(a, stream);
    case ISOQ_BF16:
      return mq ? launch_mma_t<D, NST, __nv_bfloat16, true, BITS>(a, stream)
                : launch_mma_t<D, NST, __nv_bfloat16, false, BITS>(a, stream);
    case ISOQ_F16:
      return mq ? launch_mma_t<D, NST, __half, true, BITS>(a, stream)
                : launch_mma_t<D, NST, __half, false, BITS>(a, stream);
  }
  return cudaErrorInvalidValue;
}

template <int D, int NST>
cudaError_t launch_decode_mma_d(const DecodeArgs& a, cudaStream_t stream) {
  // 3-bit caches use the V tile layout and the integer kernel (isoq_decode_i8.cu)
  if constexpr (D == 128) {  // the 2- and 4-bit variants exist at d = 128
    if (a.bits == 2) return launch_decode_mma_b<D, NST, 2>(a, stream);
    if (a.bits == 4) return launch_decode_mma_b<D, NST, 4>(a, stream);
  }
  return cudaErrorInvalidValue;
}

#ifndef ISOQ_DEC_NST128
#define ISOQ_DEC_NST128 2
#endif
#ifndef ISOQ_DEC_NST256
#define ISOQ_DEC_NST256 2
#endif

cudaError_t launch_decode_split_mma(const DecodeArgs& a, cudaStream_t stream) {
  if (a.d == 128) return launch_decode_mma_d<128, ISOQ_DEC_NST128>(a, stream);
  if (a.d == 256) return launch_decode_mma_d<256, ISOQ_DEC_NST256>(a, stream);
  return cudaErrorInvalidValue;
}

// Resident CTAs per SM of the decode kernel for head dimension d on the current device
// (cached per device; 2 when it cannot be queried).
int decode_resident_ctas(int d) {
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
      n = 2;  // the 2- and 4-bit formats exist at d = 128 only
      e = cudaSuccess;
    } else {
      using SM = MmaSmem<128, ISOQ_DEC_NST128, 4>;
      e = cudaFuncSetAttribute(decode_mma_kernel<128, ISOQ_DEC_NST128, __nv_bfloat16, false, 4>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, decode_mma_kernel<128, ISOQ_DEC_NST128, __nv_bfloat16, false, 4>, kWarps * 32, SM::kBytes);
    }
    if (e != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 2;
    }
    cache[dev][di] = n;
  }
  return cache[dev][di];
}

}  // namespace isoq
