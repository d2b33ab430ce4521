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
// shared-memory stages filled by 1-D bulk copies (cp.async.bulk, one 6400-byte page block
// per copy, completion on an mbarrier; every wait is bounded).  Per 16-token tile:
//   scores  S[16 tok x 8 heads] = K_hat[16 x d] . Q~^T   (mma.sync m16n8k16, f16 -> f32;
//                                                          Q~ as f16 hi + lo parts)
//   online softmax per head (max by 3 shuffles, lazily rescaled), P' = p * nV / sigma
//   out^T[d x 8 heads] += V_hat^T[d x 16 tok] . P'^T     (mma.sync, P' transposed in
//                                                          registers with movmatrix)
// K_hat / V_hat are never stored: each thread turns its codes into f16 mma fragments in
// registers with byte permutes (prmt) against 8-entry tables of the levels' low and high
// bytes.  The packed layout puts 24 of every 32 codes in nibbles (bit 3 clear), which is
// exactly a prmt byte selector; the other 8 come from the spare bit 3 of three words.
// Levels are scaled by ALPHA, a constant for which all four magnitudes round to binary16
// with relative error < 2e-5 (1/ALPHA is folded into the score and output scales).
#include <math_constants.h>

#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"

namespace isoq {
using namespace ptx;


// Dynamic shared memory: [kWarps][NST] page stages of block_bytes(D), then the mbarriers,
// then the rotated queries (fp32 [8][D]).  The stage area is reused for the final merge.
template <int D, int NST>
struct MmaSmem {
  static constexpr int kStageBytes = block_bytes(D);
  static constexpr int kRing = kWarps * NST * kStageBytes;
  static constexpr int kBarOff = kRing;
  static constexpr int kQOff = kBarOff + kWarps * NST * 8;
  // rotated queries, row stride kQS floats: dim d of head h at h*kQS + 40*(d/32) + d%32, so
  // the 16-byte fragment loads of a quarter warp hit distinct banks
  static constexpr int kQS = 40 * (D / 32) + 4;
  static constexpr int kBytes = kQOff + 8 * kQS * 4;
  static constexpr int kMergeBytes = kWarps * 8 * (D + 4) * 4;
  static_assert(kMergeBytes <= kRing, "merge buffer must fit in the ring");
};

#ifndef ISOQ_DEC_MINB
#define ISOQ_DEC_MINB 4  // <= 128 registers: 4 CTAs (16 warps) per SM
#endif

template <int D, int NST, typename TQ>
__global__ void __launch_bounds__(kWarps * 32, ISOQ_DEC_MINB)
    decode_mma_kernel(const float* __restrict__ params, const uint8_t* __restrict__ blocks,
                      const int32_t* __restrict__ page_table, int n_pages, int max_pages, int H,
                      const TQ* __restrict__ Q, int n_q_heads, const int32_t* __restrict__ seq_lens,
                      float scale, int pages_per_split, int n_splits, float* __restrict__ partials,
                      uint32_t* status, uint32_t mul16) {
  using SM = MmaSmem<D, NST>;
  constexpr int E = D / 32;           // elements per lane in the warp WHT layout
  constexpr int NB = E / 4;
  constexpr int CB = code_bytes(D);
  constexpr int BB = block_bytes(D);
  constexpr int KS = D / 16;          // k-steps of the score mma, m-tiles of the PV mma
  constexpr int NG = D / 128;         // groups per thread (score side: t, t+4; PV side)
  constexpr int PS = D + 4;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBarOff);
  float* qs = reinterpret_cast<float*>(smem + SM::kQOff);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.x, s = blockIdx.z;
  const int G = n_q_heads / H;
  const int nhb = (G + 7) >> 3;
  const int hk = blockIdx.y / nhb, hb = blockIdx.y - hk * nhb;
  const int h0 = hk * G + hb * 8;                // first query head of this CTA
  const int nh = min(8, G - hb * 8);             // query heads handled here

  int len = __ldg(seq_lens + s);
  if (len > max_pages * kPage) {
    if (tid == 0 && split == 0 && blockIdx.y == 0) set_status(status, ISOQ_ST_LEN_RANGE);
    len = max_pages * kPage;
  }
  const int p_begin = split * pages_per_split;
  const int p_end = min((len + kPage - 1) / kPage, p_begin + pages_per_split);

  float* out_base = partials + ((size_t)s * n_q_heads + h0) * n_splits * PS + (size_t)split * PS;
  if (p_begin >= p_end) {  // empty chunk: m = -inf, l = 0, acc = 0
    for (int i = tid; i < nh * PS; i += blockDim.x) {
      const int h = i / PS, c = i - h * PS;
      out_base[(size_t)h * n_splits * PS + c] = (c == D) ? -CUDART_INF_F : 0.f;
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
    const int phys = __ldg(pt_row + pg);
    if (phys >= 0 && phys < n_pages) {
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

  // ---- a6: rotate the CTA's queries (unnormalised WHT + SO(4)) into shared memory ------
  {
    const float* hp = params + (size_t)hk * D * 2;
    float pq[NB][8];
#pragma unroll
    for (int k = 0; k < NB; ++k) load_block_params(hp, lane * NB + k, pq[k]);
    for (int h = warp; h < 8; h += kWarps) {
      float v[E];
      if (h < nh) {
        const TQ* qp = Q + ((size_t)s * n_q_heads + h0 + h) * D + lane * E;
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] = to_f32<TQ>(qp[i]);
      } else {
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] = 0.f;
      }
      wht_warp<E>(v, lane);
      float z[E];
#pragma unroll
      for (int k = 0; k < NB; ++k) so4_fwd(pq[k], v + 4 * k, z + 4 * k);
#pragma unroll
      for (int i = 0; i < E; ++i) {
        const int dd = lane * E + i;
        qs[h * SM::kQS + 40 * (dd >> 5) + (dd & 31)] = z[i];
      }
    }
  }
  __syncthreads();

  // B fragments of Q~^T for the score mma: k-step kk covers dims base..base+3 of group
  // t + 4*(kk / 8), base = 32*(t + 4*(kk/8)) + 4*(kk%8); b0 = dims (0,1), b1 = (2,3).
  // The query is split into f16 high and low parts (q = hi + lo to ~2^-22 relative) and
  // both are multiplied: one f16 rounding of q alone costs up to ~5e-3 relative error
  // in the output when a few large scores dominate the softmax.
  uint32_t qb0[KS], qb1[KS], ql0[KS], ql1[KS];
#pragma unroll
  for (int kk = 0; kk < KS; ++kk) {
    const float* q = qs + g * SM::kQS + 40 * (t + 4 * (kk / 8)) + 4 * (kk % 8);
    float hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hi[i] = __half2float(__float2half_rn(q[i]));
      lo[i] = q[i] - hi[i];
    }
    qb0[kk] = pack_f16x2(hi[0], hi[1]);
    qb1[kk] = pack_f16x2(hi[2], hi[3]);
    ql0[kk] = pack_f16x2(lo[0], lo[1]);
    ql1[kk] = pack_f16x2(lo[2], lo[3]);
  }

  // level byte tables: tl = low bytes, th = high bytes of f16(ALPHA * L[c]), c = 0..7
  uint32_t tl0 = 0, tl1 = 0, th0 = 0, th1 = 0;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t hbits = __half_as_ushort(__float2half_rn(kAlpha * level_f32(c)));
    const uint32_t lo = hbits & 0xffu, hi = hbits >> 8;
    if (c < 4) {
      tl0 |= lo << (8 * c);
      th0 |= hi << (8 * c);
    } else {
      tl1 |= lo << (8 * (c - 4));
      th1 |= hi << (8 * (c - 4));
    }
  }

  // running state (heads 2t, 2t+1 of this thread's C columns)
  float m2[2] = {-CUDART_INF_F, -CUDART_INF_F};  // running max of the log2 scores
  float lsum[2] = {0.f, 0.f};                    // this thread's share of sum p
  float sigma = 0.f;                             // V-norm reference (warp-uniform)
  float acc[KS][4];
#pragma unroll
  for (int i = 0; i < KS; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const float kf = scale * kLog2e / (kAlpha * (float)D);  // log2 score per (dot * nK)

  const Shifter sh(mul16);
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
    const int phys = __ldg(pt_row + pg);
    const bool page_ok = phys >= 0 && phys < n_pages;
    const int tok0 = pg * kPage;

#pragma unroll
    for (int tb = 0; tb < kPage; tb += 32) {
      // ---- a7: scores for two 16-token sub-tiles; A = K_hat rows (tokens r+g, r+g+8) ----
      // four independent accumulator chains per sub-tile (k-step parity x hi/lo part of
      // the query) so consecutive mma instructions do not wait on each other's results
      float sc[2][4], part[2][4][4];
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        const int r = tb + 16 * sub;
#pragma unroll
        for (int c = 0; c < 4; ++c) part[sub][c][0] = part[sub][c][1] = part[sub][c][2] = part[sub][c][3] = 0.f;
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
          const int q = t + 4 * gq;
          const uint32_t* ra = reinterpret_cast<const uint32_t*>(blk + (r + g) * CB) + 3 * q;
          const uint32_t* rb = reinterpret_cast<const uint32_t*>(blk + (r + g + 8) * CB) + 3 * q;
          uint32_t Sa[4], Sb[4];
          selectors(ra[0], ra[1], ra[2], sh, Sa);
          selectors(rb[0], rb[1], rb[2], sh, Sb);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t fa[4], fb[4];
            deq8(Sa[j], tl0, tl1, th0, th1, sh, fa);
            deq8(Sb[j], tl0, tl1, th0, th1, sh, fb);
            const int kk0 = 8 * gq + 2 * j;
            mma16816(part[sub][0], fa[0], fb[0], fa[1], fb[1], qb0[kk0], qb1[kk0]);
            mma16816(part[sub][1], fa[2], fb[2], fa[3], fb[3], qb0[kk0 + 1], qb1[kk0 + 1]);
            mma16816(part[sub][2], fa[0], fb[0], fa[1], fb[1], ql0[kk0], ql1[kk0]);
            mma16816(part[sub][3], fa[2], fb[2], fa[3], fb[3], ql0[kk0 + 1], ql1[kk0 + 1]);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          sc[sub][i] = (part[sub][0][i] + part[sub][1][i]) + (part[sub][2][i] + part[sub][3][i]);
      }
      // token validity and norms of this thread's C rows: tokens tb+16sub+g (+8)
      float s2[2][4], nv[2][2];
      bool vd[2][2];
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int tk = tb + 16 * sub + g + 8 * rr;
          vd[sub][rr] = page_ok && (tok0 + tk) < len;
          const float nk = half_at(blk + k_norm_off(D) + 2 * tk);
          nv[sub][rr] = vd[sub][rr] ? half_at(blk + v_norm_off(D) + 2 * tk) : 0.f;
          s2[sub][2 * rr + 0] = vd[sub][rr] ? sc[sub][2 * rr + 0] * nk * kf : -CUDART_INF_F;
          s2[sub][2 * rr + 1] = vd[sub][rr] ? sc[sub][2 * rr + 1] * nk * kf : -CUDART_INF_F;
        }
      }

      // ---- a8: online softmax over the 32 tokens (per head: 4 values here, 3 shuffles) --
      float tmax[2] = {fmaxf(fmaxf(s2[0][0], s2[0][2]), fmaxf(s2[1][0], s2[1][2])),
                       fmaxf(fmaxf(s2[0][1], s2[0][3]), fmaxf(s2[1][1], s2[1][3]))};
      float vmax = fmaxf(fmaxf(nv[0][0], nv[0][1]), fmaxf(nv[1][0], nv[1][1]));
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        tmax[0] = fmaxf(tmax[0], __shfl_xor_sync(kFull, tmax[0], o));
        tmax[1] = fmaxf(tmax[1], __shfl_xor_sync(kFull, tmax[1], o));
        vmax = fmaxf(vmax, __shfl_xor_sync(kFull, vmax, o));
      }
      float resc[2] = {1.f, 1.f};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (tmax[e] > m2[e] + kLazy) {
          resc[e] = ex2(m2[e] - tmax[e]);  // 0 when m2 was -inf
          lsum[e] *= resc[e];
          m2[e] = tmax[e];
        }
      }
      if (vmax > sigma * kSigmaSlack) {
        const float rr = sigma / vmax;  // 0 on the first valid tile
        resc[0] *= rr;
        resc[1] *= rr;
        sigma = vmax;
      }
      if (resc[0] != 1.f || resc[1] != 1.f) {
#pragma unroll
        for (int i = 0; i < KS; ++i) {
          acc[i][0] *= resc[0];
          acc[i][1] *= resc[1];
          acc[i][2] *= resc[0];
          acc[i][3] *= resc[1];
        }
      }
      const float inv_sigma = sigma > 0.f ? 1.f / sigma : 0.f;
      uint32_t pb[2][2];
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        float pw[4];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const float p0 = vd[sub][rr] ? ex2(s2[sub][2 * rr] - m2[0]) : 0.f;
          const float p1 = vd[sub][rr] ? ex2(s2[sub][2 * rr + 1] - m2[1]) : 0.f;
          lsum[0] += p0;
          lsum[1] += p1;
          const float w = nv[sub][rr] * inv_sigma;
          pw[2 * rr] = p0 * w;
          pw[2 * rr + 1] = p1 * w;
        }
        // P'^T fragments: transpose the two 8x8 blocks (tokens 0-7, 8-15 of the sub-tile)
        pb[sub][0] = movmatrix_t(pack_f16x2(pw[0], pw[1]));
        pb[sub][1] = movmatrix_t(pack_f16x2(pw[2], pw[3]));
      }

      // ---- a8: V accumulation, A = V_hat^T (rows = dims, k = tokens 2t,2t+1,2t+8,2t+9) --
#pragma unroll
      for (int sub = 0; sub < 2; ++sub) {
        const int r = tb + 16 * sub;
#pragma unroll
        for (int gq = 0; gq < NG; ++gq) {
          const int q = (g >> 1) + 4 * gq;
          const uint8_t* vbase = blk + v_codes_off(D);
          const bool odd = (g & 1) != 0;  // odd g: words 2, 3 (w2 and the spare bits)
          uint32_t S[4][2];  // [token 2t, 2t+1, 2t+8, 2t+9][word j0, j0+1]
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const int tk = r + 2 * t + (x & 1) + 8 * (x >> 1);
            const uint32_t* w = reinterpret_cast<const uint32_t*>(vbase + tk * CB) + 3 * q;
            const uint32_t w0 = w[0], w1 = w[1], w2 = w[2];
            S[x][0] = (odd ? w2 : w0) & 0x77777777u;
            S[x][1] = odd ? sh.spare(w0, w1, w2) : (w1 & 0x77777777u);
          }
          uint32_t f[4][8];  // [pair/word combo][nibble = m-tile]
          deq8_pair(S[0][0], S[1][0], tl0, tl1, th0, th1, sh, f[0]);
          deq8_pair(S[0][1], S[1][1], tl0, tl1, th0, th1, sh, f[1]);
          deq8_pair(S[2][0], S[3][0], tl0, tl1, th0, th1, sh, f[2]);
          deq8_pair(S[2][1], S[3][1], tl0, tl1, th0, th1, sh, f[3]);
#pragma unroll
          for (int mt = 0; mt < 8; ++mt)
            mma16816(acc[8 * gq + mt], f[0][mt], f[1][mt], f[2][mt], f[3][mt], pb[sub][0],
                     pb[sub][1]);
        }
      }
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
  // reduce this thread's lsum over the 8 rows g (lanes with the same t)
#pragma unroll
  for (int e = 0; e < 2; ++e) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) lsum[e] += __shfl_xor_sync(kFull, lsum[e], o);
  }
  __syncthreads();  // all warps done with their rings
  float* mb = reinterpret_cast<float*>(smem);  // [kWarps][8 heads][D + 4]
  {
    // acc_true = acc * sigma / ALPHA (times 1 / exp2(m2) in the log2 frame)
    const float f = sigma / kAlpha;
#pragma unroll
    for (int gq = 0; gq < NG; ++gq) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int q = (g >> 1) + 4 * gq;
        const int j0 = 2 * (g & 1);
        const int d0 = 32 * q + 8 * j0 + mt;  // row g of m-tile; row g+8 is d0 + 8
        float* r0 = mb + (warp * 8 + 2 * t) * PS;
        float* r1 = mb + (warp * 8 + 2 * t + 1) * PS;
        r0[d0] = acc[8 * gq + mt][0] * f;
        r1[d0] = acc[8 * gq + mt][1] * f;
        r0[d0 + 8] = acc[8 * gq + mt][2] * f;
        r1[d0 + 8] = acc[8 * gq + mt][3] * f;
      }
    }
    if (g == 0) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float* r = mb + (warp * 8 + 2 * t + e) * PS;
        r[D] = m2[e];
        r[D + 1] = lsum[e];
      }
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
    float* o = out_base + (size_t)h * n_splits * PS;
    if (c < D) o[c] = v;
    else {
      o[D] = M == -CUDART_INF_F ? -CUDART_INF_F : M / kLog2e;  // natural-log units
      o[D + 1] = v;
    }
  }
}

template <int D, int NST, typename TQ>
static cudaError_t launch_mma_t(const DecodeArgs& a, cudaStream_t stream) {
  using SM = MmaSmem<D, NST>;
  // the dynamic shared-memory opt-in is per function and per device
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_mma_kernel<D, NST, TQ>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  const int G = a.n_q_heads / a.n_kv_heads;
  dim3 grid(a.n_splits, a.n_kv_heads * ((G + 7) / 8), a.n_seqs);
  decode_mma_kernel<D, NST, TQ><<<grid, kWarps * 32, SM::kBytes, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_kv_heads,
      static_cast<const TQ*>(a.Q), a.n_q_heads, a.seq_lens, a.scale, a.pages_per_split,
      a.n_splits, a.partials, a.status, 65536u);
  return cudaGetLastError();
}

template <int D, int NST>
cudaError_t launch_decode_mma_d(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.q_dtype) {
    case ISOQ_F32: return launch_mma_t<D, NST, float>(a, stream);
    case ISOQ_BF16: return launch_mma_t<D, NST, __nv_bfloat16>(a, stream);
    case ISOQ_F16: return launch_mma_t<D, NST, __half>(a, stream);
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
      using SM = MmaSmem<256, ISOQ_DEC_NST256>;
      e = cudaFuncSetAttribute(decode_mma_kernel<256, ISOQ_DEC_NST256, __nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, decode_mma_kernel<256, ISOQ_DEC_NST256, __nv_bfloat16>, kWarps * 32, SM::kBytes);
    } else {
      using SM = MmaSmem<128, ISOQ_DEC_NST128>;
      e = cudaFuncSetAttribute(decode_mma_kernel<128, ISOQ_DEC_NST128, __nv_bfloat16>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
      if (e == cudaSuccess)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &n, decode_mma_kernel<128, ISOQ_DEC_NST128, __nv_bfloat16>, kWarps * 32, SM::kBytes);
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
