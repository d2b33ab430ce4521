// Multi-token attention on the packed cache with the dequantised page shared by many rows.
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: attention on the packed codes, full-precision K/V
// never written to memory; the queries are rotated once and scores and the value sum run
// on codebook levels in the rotated space.
//
// When a chunk of query tokens (chunked prefill, speculative verification) gives a KV head
// many (query token, head) rows, the per-row kernel would dequantise every page once per 8
// rows.  Here one CTA of 4 warps owns 64 rows (8 row-blocks of 8) of one KV head and one
// context chunk:
//   - the chunk's pages stream through a 2-stage shared-memory ring (1-D bulk copies,
//     mbarrier completion, bounded waits);
//   - per page the 128 threads dequantise K_hat and V_hat once into f16 tiles
//     [64 tokens][128 dims] in shared memory (16-byte chunks XOR-swizzled by the row);
//   - each warp then runs its two row-blocks over the tiles: scores on mma.sync m16n8k16
//     (rows 0-7 of A the f16 high parts of a block's rotated queries, rows 8-15 the low
//     parts; K_hat B fragments by ldmatrix, shared by both blocks), the lazy online softmax
//     per row, and out[16 rows x 128 dims] += P'[16 x 16 tok] . V_hat (A = the two blocks'
//     weights stacked, straight from the score accumulators; V_hat B fragments by
//     ldmatrix.trans), so each row's rescale stays in its own lane.
// The partial results have the layout of the per-row kernel and go to the same combine.
#include <math_constants.h>

#include "isoq_check.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"
#include "isoq_vtile.cuh"

namespace isoq {
using namespace ptx;
namespace {

constexpr int kMqD = 128;
constexpr int kMqWarps = 4;
constexpr int kMqRowBlocks = 2 * kMqWarps;  // 8 rows each: 64 rows per CTA
constexpr int kMqKS = kMqD / 16;             // k-steps of the score mma

template <int BITS>
struct MqSmem {
  static constexpr int kBB = block_bytes(kMqD, BITS);
  static constexpr int kOffRing = 0;                              // [2][kBB]
  // two tile buffers (page k computes from one while page k+1 is dequantised into the
  // other), each K_hat then V_hat f16 [64][128], swizzled
  static constexpr int kOffTile = (2 * kBB + 1023) / 1024 * 1024;
  static constexpr int kTileBytes = 2 * 64 * kMqD * 2;
  static constexpr int kOffQ = kOffTile + 2 * kTileBytes;         // uint4 [8 rb][KS][32]
  static constexpr int kOffNorm = kOffQ + kMqRowBlocks * kMqKS * 32 * 16;  // float [2][2][64]
  static constexpr int kOffBar = kOffNorm + 2 * 2 * 64 * 4;       // 2 mbarriers
  static constexpr int kOffRow = kOffBar + 16;                    // int [64] output rows
  static constexpr int kBytes = kOffRow + 64 * 4;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// byte offset of 16-byte chunk c (8 dims) of token row tk in a swizzled f16 tile
__device__ __forceinline__ uint32_t tile_off(int tk, int c) {
  return (uint32_t)(tk * (kMqD * 2) + ((c ^ (tk & 7)) << 4));
}

template <typename TQ, int BITS>
__global__ void __launch_bounds__(kMqWarps * 32, 2)
    decode_mq_kernel(const float* __restrict__ params, const uint8_t* __restrict__ blocks,
                     const int32_t* __restrict__ page_table, int n_pages, int max_pages, int H,
                     const TQ* __restrict__ Q, int n_q_heads, int n_q,
                     const int32_t* __restrict__ seq_lens, float scale, int pages_per_split,
                     int n_splits, float* __restrict__ partials, uint32_t* status) {
  using SM = MqSmem<BITS>;
  constexpr int D = kMqD, E = D / 32, NB = E / 4, KS = kMqKS, PS = D + 4;
  constexpr int CB = code_bytes(D, BITS), BB = block_bytes(D, BITS), W = BITS;
  constexpr float ALPHA = alpha_of<BITS>();
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kOffBar);
  uint4* qa = reinterpret_cast<uint4*>(smem + SM::kOffQ);
  float* nrm_all = reinterpret_cast<float*>(smem + SM::kOffNorm);  // [buf][K|V][tok]
  int* row_off = reinterpret_cast<int*>(smem + SM::kOffRow);
  const uint32_t sTile = smem_u32(smem + SM::kOffTile);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int split = blockIdx.x, s = blockIdx.z;
  const int G = n_q_heads / H;
  const int n_rows = n_q * G;
  const int n_groups = (n_rows + 63) >> 6;
  const int hk = blockIdx.y / n_groups, rg = blockIdx.y - hk * n_groups;
  const int row0 = rg * 64;                       // first row (of this KV head's) here
  const int nh = min(64, n_rows - row0);          // rows handled here

  int len = __ldg(seq_lens + s);
  if (len > max_pages * kPage) {
    if (tid == 0 && split == 0 && blockIdx.y == 0) set_status(status, ISOQ_ST_LEN_RANGE);
    len = max_pages * kPage;
  }
  // row r (0..63) = pair R = row0 + r: query token R / G, head hk * G + R % G; causal
  // limit len - n_q + 1 + token
  if (tid < 64) {
    const int R = row0 + tid;
    row_off[tid] = tid < nh ? (R / G) * n_q_heads + hk * G + R % G : 0;
  }
  auto lim_of = [&](int r) { return max(0, min(len, len - n_q + 1 + (row0 + r) / G)); };
  const int lim_hi = lim_of(nh - 1), lim_lo = lim_of(0);
  const int p_begin = split * pages_per_split;
  const int p_end = min((lim_hi + kPage - 1) / kPage, p_begin + pages_per_split);
  float* out_base = partials + ((size_t)s * n_q * n_q_heads) * n_splits * PS + (size_t)split * PS;
  __syncthreads();
  if (p_begin >= p_end) {  // empty chunk: m = -inf, l = 0, acc = 0
    for (int i = tid; i < nh * PS; i += blockDim.x) {
      const int r = i / PS, c = i - r * PS;
      if (in_bounds(row_off[r] < n_q * n_q_heads, status))
        out_base[(size_t)row_off[r] * n_splits * PS + c] = (c == D) ? -CUDART_INF_F : 0.f;
    }
    return;
  }

  // ---- page ring ------------------------------------------------------------------------
  const int* pt_row = page_table + (size_t)s * max_pages;
  const int n_my = p_end - p_begin;
  auto issue = [&](int k) {  // thread 0
    const int st = k & 1;
    const int phys = in_bounds(p_begin + k < max_pages, status) ? __ldg(pt_row + p_begin + k) : -1;
    uint64_t* bar = bars + st;
    if (phys >= 0 && phys < n_pages) {
      mbar_expect_tx(bar, BB);
      bulk_copy(smem + SM::kOffRing + st * BB, blocks + ((size_t)phys * H + hk) * BB, BB, bar);
    } else {
      set_status(status, ISOQ_ST_PAGE_RANGE);
      mbar_arrive(bar);
    }
  };
  if (tid == 0) {
    mbar_init(bars, 1);
    mbar_init(bars + 1, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    issue(0);
    if (n_my > 1) issue(1);
  }
  __syncthreads();  // barriers initialised before any thread waits on them

  // ---- a6: rotate the 64 rows' queries into the A fragments (natural dim order) ---------
  // rows 0-7 of a block's A are the f16 high parts of its 8 rows' rotated queries, rows
  // 8-15 the low parts; k-step kb of lane (g, t): dims 16 kb + 2t (+1) and 16 kb + 2t + 8 (+9)
  {
    const float* hp = params + (size_t)hk * D * 4;
    float M[NB][16];
#pragma unroll
    for (int k = 0; k < NB; ++k) load_block_mat(hp, lane * NB + k, M[k]);
    for (int r = warp; r < 64; r += kMqWarps) {
      float v[E];
      if (r < nh) {
        const TQ* qp = Q + ((size_t)s * n_q * n_q_heads +
                            (in_bounds(row_off[r] < n_q * n_q_heads, status) ? row_off[r] : 0)) *
                               D +
                       lane * E;
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] = to_f32<TQ>(qp[i]);
      } else {
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] = 0.f;
      }
      wht_warp<E>(v, lane);
      float z[E];
#pragma unroll
      for (int k = 0; k < NB; ++k) mat_fwd(M[k], v + 4 * k, z + 4 * k);
      // lane holds dims 4 lane .. 4 lane + 3: a pair (dims d, d+1) sits in k-step d / 16
      // at k index d % 16; write hi/lo halves into the A-fragment words of the owner lanes
      const int rb = r >> 3, gr = r & 7;
#pragma unroll
      for (int e = 0; e < E; e += 2) {
        const int d0 = lane * E + e, kb = d0 >> 4, kk = d0 & 15;
        const float hi0 = __half2float(__float2half_rn(z[e])), hi1 = __half2float(__float2half_rn(z[e + 1]));
        const uint32_t whi = pack_f16x2(hi0, hi1), wlo = pack_f16x2(z[e] - hi0, z[e + 1] - hi1);
        // k index kk = 2 tt (+8 for the second half): a0/a1 (kk < 8) or a2/a3
        const int tt = (kk & 7) >> 1;
        uint32_t* frag = reinterpret_cast<uint32_t*>(qa + ((size_t)rb * KS + kb) * 32 + gr * 4 + tt);
        frag[(kk >= 8 ? 2 : 0)] = whi;
        frag[(kk >= 8 ? 3 : 1)] = wlo;
      }
    }
  }

  uint32_t tl0, tl1, th0, th1;
  level_tables<BITS>(tl0, tl1, th0, th1);
  const float kf = scale * kLog2e / (ALPHA * (float)D);  // log2 score per (dot * nK)

  // this warp's two row-blocks: b = 2 warp + {0, 1}; lane's rows g of each
  const int rbA = 2 * warp, rbB = rbA + 1;
  const int limA = lim_of(8 * rbA + g), limB = lim_of(8 * rbB + g);
  const bool warp_active = 8 * rbA < nh;
  float m2[2] = {-CUDART_INF_F, -CUDART_INF_F}, lsum[2] = {0.f, 0.f};
  float sigma = 0.f, inv_sigma = 0.f;
  float acc[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  // dequantise page kk (ring stage kk & 1) into tile buffer kk & 1, with its norms
  auto dequant = [&](int kk) {
    const uint8_t* blk = smem + SM::kOffRing + (kk & 1) * BB;
    const uint32_t sK = sTile + (kk & 1) * SM::kTileBytes, sV = sK + 64 * D * 2;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int u = tid + 128 * half;  // (token, 32-dim group) unit
      const int tk = u >> 2, q = u & 3;
#pragma unroll
      for (int kv = 0; kv < 2; ++kv) {
        const uint32_t base = (kv ? sV : sK);
        if (BITS == 3 && kv == 1) {
          // V tile layout: unit u = (block, quad, 8-dim unit) group of four tokens
          const int B = u >> 6, t4 = (u >> 4) & 3, un = u & 15;
          const uint32_t* wp = reinterpret_cast<const uint32_t*>(
              blk + v_codes_off(D, BITS) + vt_group_off(D, B, t4, un));
          if (!in_bounds(vt_group_off(D, B, t4, un) + 12 <= kPage * CB, status)) continue;
          uint32_t o[4][4];
          vdeq_group(wp[0], wp[1], wp[2], tl0, tl1, th0, th1, o);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (!in_bounds(tile_off(vt_member_slot(B, t4, j), un) + 16 <= 64 * D * 2, status))
              continue;
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             base + tile_off(vt_member_slot(B, t4, j), un)),
                         "r"(o[j][0]), "r"(o[j][1]), "r"(o[j][2]), "r"(o[j][3])
                         : "memory");
          }
          continue;
        }
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(blk + (kv ? v_codes_off(D, BITS) : 0) +
                                                             tk * CB) + W * q;
        if (!in_bounds(tk * CB + 4 * W * (q + 1) <= kPage * CB, status)) continue;
        uint32_t w[W];
#pragma unroll
        for (int i = 0; i < W; ++i) w[i] = wp[i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t o[4];
          kdeq<BITS>(w, j, tl0, tl1, th0, th1, o);
          if (!in_bounds(tile_off(tk, 4 * q + j) + 16 <= 64 * D * 2, status)) continue;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(base + tile_off(tk, 4 * q + j)),
                       "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                       : "memory");
        }
      }
    }
    if (tid < 64) {
      float* nb = nrm_all + (kk & 1) * 128;
      nb[tid] = half_at(blk + k_norm_off(D, BITS) + 2 * tid) * kf;
      nb[64 + tid] = half_at(blk + v_norm_off(D, BITS) + 2 * tid);
    }
  };

  bool timed_out = false;
  int issued = min(n_my, 2);  // pages whose copy has been started (thread 0's count)
  int drain_from = 0;         // first page whose copy may still be in flight after a timeout
  // page 0 into tile buffer 0, then its ring stage takes page 2
  if (!mbar_wait(bars, 0)) timed_out = true;
  if (__syncthreads_or(timed_out)) {
    timed_out = true;
  } else {
    dequant(0);
  }
  __syncthreads();
  if (!timed_out && tid == 0 && 2 < n_my) {
    fence_proxy_async();
    issue(2);
    issued = 3;
  }
  int k = 0;
  for (; !timed_out && k < n_my; ++k) {
    // page k + 1: wait for its copy and dequantise it into the other tile buffer while the
    // CTA's warps compute page k
    if (k + 1 < n_my) {
      const bool ok = mbar_wait(bars + ((k + 1) & 1), ((k + 1) >> 1) & 1);
      if (__syncthreads_or(!ok)) {
        timed_out = true;
        drain_from = k + 1;
        break;
      }
      dequant(k + 1);
    }
    const int pg = p_begin + k;
    const int phys = in_bounds(pg < max_pages, status) ? __ldg(pt_row + pg) : -1;
    const bool page_ok = phys >= 0 && phys < n_pages;
    const int tok0 = pg * kPage;
    const uint32_t sK = sTile + (k & 1) * SM::kTileBytes, sV = sK + 64 * D * 2;
    const float* nrm = nrm_all + (k & 1) * 128;

    if (warp_active) {
      // a page whose 64 tokens are valid for every row of the CTA needs no masking
      const bool full = page_ok && tok0 + kPage <= lim_lo;
#pragma unroll 1
      for (int hb = 0; hb < 64; hb += 32) {
        // ---- a7: scores of both row-blocks for tokens hb + 8n + (0..7), n = 0..3 --------
        float C[2][4][4];
#pragma unroll
        for (int b = 0; b < 2; ++b)
#pragma unroll
          for (int n = 0; n < 4; ++n) C[b][n][0] = C[b][n][1] = C[b][n][2] = C[b][n][3] = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // dims 32c .. 32c + 31 = k-steps 2c, 2c + 1
          const uint4 A0a = qa[((size_t)rbA * KS + 2 * c) * 32 + lane];
          const uint4 A1a = qa[((size_t)rbA * KS + 2 * c + 1) * 32 + lane];
          const uint4 A0b = qa[((size_t)rbB * KS + 2 * c) * 32 + lane];
          const uint4 A1b = qa[((size_t)rbB * KS + 2 * c + 1) * 32 + lane];
          uint32_t bf[4][4];
#pragma unroll
          for (int n = 0; n < 4; ++n)
            ldsm_x4(sK + tile_off(hb + 8 * n + (lane & 7), 4 * c + (lane >> 3)), bf[n]);
          // eight independent accumulators per k-step: no mma waits on the one before
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            mma16816(C[0][n], A0a.x, A0a.y, A0a.z, A0a.w, bf[n][0], bf[n][1]);
            mma16816(C[1][n], A0b.x, A0b.y, A0b.z, A0b.w, bf[n][0], bf[n][1]);
          }
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            mma16816(C[0][n], A1a.x, A1a.y, A1a.z, A1a.w, bf[n][2], bf[n][3]);
            mma16816(C[1][n], A1b.x, A1b.y, A1b.z, A1b.w, bf[n][2], bf[n][3]);
          }
        }

        // ---- a8: online softmax per row (this lane: row g of blocks A and B) -------------
        float sv[2][4][2], nvv[4][2];
        bool grow = false;
        const float sthr0 = m2[0] + kLazy, sthr1 = m2[1] + kLazy, vthr = sigma * kSigmaSlack;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tk = hb + 8 * n + 2 * t + e;
            const float nk = nrm[tk];  // K norm times the log2 score scale
            float nvx = nrm[64 + tk];
            float s0 = (C[0][n][e] + C[0][n][e + 2]) * nk, s1 = (C[1][n][e] + C[1][n][e + 2]) * nk;
            if (!full) {
              const bool ok = page_ok && tok0 + tk < lim_hi;
              nvx = ok ? nvx : 0.f;
              s0 = ok && tok0 + tk < limA ? s0 : -CUDART_INF_F;
              s1 = ok && tok0 + tk < limB ? s1 : -CUDART_INF_F;
            }
            nvv[n][e] = nvx;
            sv[0][n][e] = s0;
            sv[1][n][e] = s1;
            grow |= (s0 > sthr0) | (s1 > sthr1) | (nvx > vthr);
          }
        }
        if (__any_sync(kFull, grow)) {
          float tmax[2] = {-CUDART_INF_F, -CUDART_INF_F}, vmax = 0.f;
#pragma unroll
          for (int n = 0; n < 4; ++n)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              tmax[0] = fmaxf(tmax[0], sv[0][n][e]);
              tmax[1] = fmaxf(tmax[1], sv[1][n][e]);
              vmax = fmaxf(vmax, nvv[n][e]);
            }
#pragma unroll
          for (int o = 1; o < 4; o <<= 1) {
            tmax[0] = fmaxf(tmax[0], __shfl_xor_sync(kFull, tmax[0], o));
            tmax[1] = fmaxf(tmax[1], __shfl_xor_sync(kFull, tmax[1], o));
            vmax = fmaxf(vmax, __shfl_xor_sync(kFull, vmax, o));
          }
          float resc[2] = {1.f, 1.f};
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            if (tmax[b] > m2[b] + kLazy) {
              resc[b] = ex2(m2[b] - tmax[b]);  // 0 when m2 was -inf
              lsum[b] *= resc[b];
              m2[b] = tmax[b];
            }
          }
          float vr = 1.f;
          vmax = __shfl_sync(kFull, vmax, 0);  // the same in every lane group; make it uniform
          if (vmax > vthr) {
            vr = sigma / vmax;
            sigma = vmax;
            inv_sigma = 1.f / vmax;
          }
          const float r0 = resc[0] * vr, r1 = resc[1] * vr;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            acc[i][0] *= r0;
            acc[i][1] *= r0;
            acc[i][2] *= r1;
            acc[i][3] *= r1;
          }
        }
        // P' A fragments of the value mma (k16 block j = tiles 2j, 2j+1): rows g = block A,
        // rows g + 8 = block B
        uint32_t pa[2][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          float p[2][2];
#pragma unroll
          for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float x = sv[b][n][e];
              const float pe = x != -CUDART_INF_F ? ex2(x - m2[b]) : 0.f;
              lsum[b] += pe;
              p[b][e] = pe * (nvv[n][e] * inv_sigma);
            }
          // tile n: a0 (block A, tokens 2t, 2t+1) / a1 (block B) for even n, a2 / a3 for odd n
          pa[n >> 1][(n & 1) * 2 + 0] = pack_f16x2(p[0][0], p[0][1]);
          pa[n >> 1][(n & 1) * 2 + 1] = pack_f16x2(p[1][0], p[1][1]);
        }

        // ---- a8: out[16 rows x 128 dims] += P'[16 x 16 tok] . V_hat[16 tok x 128] ---------
#pragma unroll
        for (int j = 0; j < 2; ++j) {
#pragma unroll
          for (int dp = 0; dp < 8; ++dp) {  // dims 16 dp .. 16 dp + 15 = n-tiles 2dp, 2dp+1
            uint32_t bf[4];
            const int mtx = lane >> 3;
            const int rtk = hb + 16 * j + 8 * (mtx & 1) + (lane & 7);
            ldsm_x4_t(sV + tile_off(rtk, 2 * dp + (mtx >> 1)), bf);
            mma16816(acc[2 * dp], pa[j][0], pa[j][1], pa[j][2], pa[j][3], bf[0], bf[1]);
            mma16816(acc[2 * dp + 1], pa[j][0], pa[j][1], pa[j][2], pa[j][3], bf[2], bf[3]);
          }
        }
      }
    }
    // every warp is done with page k's tiles (free for page k + 2) and page k+1's ring stage
    // has been dequantised (free for page k + 3)
    __syncthreads();
    if (tid == 0 && k + 3 < n_my) {
      fence_proxy_async();
      issue(k + 3);
      issued = k + 4;
    }
  }

  if (timed_out) {
    if (tid == 0) {
      set_status(status, ISOQ_ST_TIMEOUT);
      // copies of pages k+1 .. issued-1 may still be in flight: wait for them (bounded)
      // before the CTA's shared memory is released
      for (int kk = drain_from; kk < issued; ++kk)
        if (!mbar_wait(bars + (kk & 1), (kk >> 1) & 1)) break;
    }
    __syncthreads();
  }

  // ---- the two row-blocks' partial results straight from registers ----------------------
#pragma unroll
  for (int b = 0; b < 2; ++b)
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) lsum[b] += __shfl_xor_sync(kFull, lsum[b], o);
  if (warp_active) {
    const float f = sigma / ALPHA;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int r = 8 * (b ? rbB : rbA) + g;
      if (r >= nh || !in_bounds(row_off[r] < n_q * n_q_heads, status)) continue;
      float* o = out_base + (size_t)row_off[r] * n_splits * PS;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        *reinterpret_cast<float2*>(o + 8 * n + 2 * t) =
            make_float2(acc[n][2 * b] * f, acc[n][2 * b + 1] * f);
      }
      if (t == 0) {
        o[D] = m2[b] == -CUDART_INF_F ? -CUDART_INF_F : m2[b] / kLog2e;  // natural-log units
        o[D + 1] = lsum[b];
      }
    }
  }
}

template <typename TQ, int BITS>
cudaError_t launch_mq_t(const DecodeArgs& a, cudaStream_t stream) {
  using SM = MqSmem<BITS>;
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_mq_kernel<TQ, BITS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SM::kBytes);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  const int G = a.n_q_heads / a.n_kv_heads;
  dim3 grid(a.n_splits, a.n_kv_heads * ((a.n_q * G + 63) / 64), a.n_seqs);
  decode_mq_kernel<TQ, BITS><<<grid, kMqWarps * 32, SM::kBytes, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_kv_heads,
      static_cast<const TQ*>(a.Q), a.n_q_heads, a.n_q, a.seq_lens, a.scale, a.pages_per_split,
      a.n_splits, a.partials, a.status);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_mq_b(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.q_dtype) {
    case ISOQ_F32: return launch_mq_t<float, BITS>(a, stream);
    case ISOQ_BF16: return launch_mq_t<__nv_bfloat16, BITS>(a, stream);
    case ISOQ_F16: return launch_mq_t<__half, BITS>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool use_shared_mq(const DecodeArgs& a) {
  return a.d == 128 && a.n_q > 1 && a.n_q * (a.n_q_heads / a.n_kv_heads) >= 16;
}

cudaError_t launch_decode_split_mq(const DecodeArgs& a, cudaStream_t stream) {
  if (attention_rows_per_cta(a.d, a.n_q, a.n_q_heads / a.n_kv_heads) == 128)
    return launch_decode_split_mqtc(a, stream);
  switch (a.bits) {
    case 2: return launch_mq_b<2>(a, stream);
    case 3: return launch_mq_b<3>(a, stream);
    case 4: return launch_mq_b<4>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace isoq
