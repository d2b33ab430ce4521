// Multi-token attention on the packed cache with the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory), head dimension 128.
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: attention on the packed codes, full-precision K/V
// never written to memory; the queries are rotated once, and the scores and the value sum
// run on codebook levels in the rotated space.
//
// One CTA of 128 threads owns 128 (query token, head) rows of one KV head (thread r owns
// row r) and one context chunk.  Per 64-token page:
//   - thread 0 streams the page blocks through a 2-stage ring (1-D bulk copies, mbarrier
//     completion, bounded waits);
//   - the 128 threads dequantise the page's K_hat and V_hat once into f16 tiles in shared
//     memory, written directly in the tensor core's no-swizzle operand layouts;
//   - thread 0 issues S[128 rows x 64 tok] = Q~ . K_hat^T: the rotated queries' f16 high
//     and low parts are two A operands in shared memory, both products go to one f32
//     accumulator in tensor memory;
//   - each thread reads its row's 64 scores from tensor memory and runs the lazy online
//     softmax of its row on its own (no cross-thread reduction), then writes the weights
//     P' = p |v| / sigma as f16 into tensor memory;
//   - thread 0 issues O[128 rows x 128 dims] += P' . V_hat with A = P' in tensor memory and
//     B = the V_hat tile; O stays in tensor memory for the whole chunk and is rescaled in
//     place, row by row, on the rare tiles that raise a row's running maximum.
// At the end each thread reads its row of O once and writes the chunk's partial result in
// the layout of the other decode kernels, which the same combine merges.
#include <math_constants.h>

#include <type_traits>

#include "isoq_check.cuh"
#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"
#include "isoq_vtile.cuh"
#include "isoq_tc.cuh"

namespace isoq {
using namespace ptx;
namespace {

constexpr int kXD = 128;    // head dimension
constexpr int kXRows = 128; // rows per CTA = threads per CTA
constexpr uint32_t kXCols = 256;  // tensor-memory columns: S 64 | O 128 | P' 32
constexpr uint32_t kColS = 0, kColO = 64, kColP = 192;
static_assert(kColS + 64 <= kColO && kColO + 128 <= kColP && kColP + 32 <= kXCols,
              "tensor-memory columns overlap or exceed the allocation");

// Shared memory (bytes).  Operand tiles, no swizzle, core matrix = 8 rows x 16 bytes:
//   Q~ hi / lo (A, K-major, 128 rows x 128 dims): (k/8) 2048 + (m/8) 128 + (m%8) 16 + (k%8) 2
//   K_hat (B of the scores, K-major, 64 tok x 128 dims): (k/8) 1024 + (n/8) 128 + ...
//   V_hat (B of the value product, MN-major: K = 64 tok, N = 128 dims):
//         (tok/8) 2048 + (dim/8) 128 + (tok%8) 16 + (dim%8) 2
template <int BITS>
struct MqtcSmem {
  static constexpr int kBB = block_bytes(kXD, BITS);
  static constexpr int kOffQh = 0;
  static constexpr int kOffQl = 32768;
  static constexpr int kOffK = 65536;
  static constexpr int kOffV = 81920;
  static constexpr int kOffRing = 98304;                               // [2][kBB]
  static constexpr int kOffNorm = kOffRing + (2 * kBB + 15) / 16 * 16;  // float [64 K | 64 V]
  static constexpr int kOffRed = kOffNorm + 128 * 4;                   // float [4]
  static constexpr int kOffBar = kOffRed + 16;                         // ring 0, 1, S, PV
  static constexpr int kOffTmem = kOffBar + 4 * 8;
  static constexpr int kOffRow = kOffTmem + 16;                        // int [128]
  static constexpr int kBytes = kOffRow + kXRows * 4;
};

__device__ __forceinline__ void st_v4(uint32_t addr, const uint32_t (&o)[4]) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(o[0]), "r"(o[1]),
               "r"(o[2]), "r"(o[3])
               : "memory");
}

template <typename TQ, int BITS>
__global__ void __launch_bounds__(kXRows, 2)
    decode_mqtc_kernel(const float* __restrict__ params, const uint8_t* __restrict__ blocks,
                       const int32_t* __restrict__ page_table, int n_pages, int max_pages,
                       int H, const TQ* __restrict__ Q, int n_q_heads, int n_q,
                       const int32_t* __restrict__ seq_lens, float scale, int pages_per_split,
                       int n_splits, float* __restrict__ partials, uint32_t* status) {
  using SM = MqtcSmem<BITS>;
  constexpr int D = kXD, E = D / 32, NB = E / 4, PS = D + 4;
  constexpr int CB = code_bytes(D, BITS), BB = block_bytes(D, BITS), W = BITS;
  constexpr float ALPHA = alpha_of<BITS>();
  constexpr uint32_t kIdS = tc::idesc_f16(128, 64, false, false);   // scores
  constexpr uint32_t kIdO = tc::idesc_f16(128, 128, false, true);   // value product
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kOffBar);
  uint64_t* bar_s = bars + 2;
  uint64_t* bar_pv = bars + 3;
  float* nrm = reinterpret_cast<float*>(smem + SM::kOffNorm);
  float* red = reinterpret_cast<float*>(smem + SM::kOffRed);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kOffTmem);
  int* row_off = reinterpret_cast<int*>(smem + SM::kOffRow);
  const uint32_t sQh = smem_u32(smem + SM::kOffQh), sQl = smem_u32(smem + SM::kOffQl);
  const uint32_t sK = smem_u32(smem + SM::kOffK), sV = smem_u32(smem + SM::kOffV);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, s = blockIdx.z;
  const int G = n_q_heads / H;
  const int n_rows = n_q * G;
  const int n_groups = (n_rows + kXRows - 1) / kXRows;
  const int hk = blockIdx.y / n_groups, rg = blockIdx.y - hk * n_groups;
  const int row0 = rg * kXRows;
  const int nh = min(kXRows, n_rows - row0);  // rows handled here

  int len = __ldg(seq_lens + s);
  if (len > max_pages * kPage) {
    if (tid == 0 && split == 0 && blockIdx.y == 0) set_status(status, ISOQ_ST_LEN_RANGE);
    len = max_pages * kPage;
  }
  // row r = pair R = row0 + r: query token R / G, head hk * G + R % G, which sits at
  // position len - n_q + R / G and attends the tokens before and at it
  {
    const int R = row0 + tid;
    row_off[tid] = tid < nh ? (R / G) * n_q_heads + hk * G + R % G : 0;
  }
  auto lim_of = [&](int r) { return max(0, min(len, len - n_q + 1 + (row0 + r) / G)); };
  const int lim_hi = lim_of(nh - 1), lim_lo = lim_of(0);
  const int my_lim = tid < nh ? lim_of(tid) : lim_hi;
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
  const int n_my = p_end - p_begin;
  const int* pt_row = page_table + (size_t)s * max_pages;

  // ---- tensor memory, barriers, the first two pages ------------------------------------
  if (warp == 0) tc::alloc(tmem_slot, kXCols);
  auto issue = [&](int k) {  // thread 0
    const int st = k & 1;
    const int phys = in_bounds(p_begin + k < max_pages, status) ? __ldg(pt_row + p_begin + k) : -1;
    if (phys >= 0 && phys < n_pages) {
      mbar_expect_tx(bars + st, BB);
      bulk_copy(smem + SM::kOffRing + st * BB, blocks + ((size_t)phys * H + hk) * BB, BB, bars + st);
    } else {
      set_status(status, ISOQ_ST_PAGE_RANGE);
      mbar_arrive(bars + st);  // complete the phase without data; the page is masked
    }
  };
  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    issue(0);
    if (n_my > 1) issue(1);
  }
  int issued = min(n_my, 2);  // pages whose copy has been started (CTA-uniform count)

  // ---- a6: rotate the 128 rows' queries into the A tiles (f16 high and low parts) -------
  {
    const float* hp = params + (size_t)hk * D * 4;
    float M[NB][16];
#pragma unroll
    for (int k = 0; k < NB; ++k) load_block_mat(hp, lane * NB + k, M[k]);
    for (int r = warp; r < kXRows; r += 4) {
      float v[E];
      if (r < nh && in_bounds(row_off[r] < n_q * n_q_heads, status)) {
        const TQ* qp = Q + ((size_t)s * n_q * n_q_heads + row_off[r]) * D + lane * E;
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
      // dims 4 lane .. 4 lane + 3: half of one 16-byte core-matrix row
      const int k0 = lane * E;
      const uint32_t off = (k0 >> 3) * 2048 + (r >> 3) * 128 + (r & 7) * 16 + (k0 & 7) * 2;
      if (!in_bounds(off + 8 <= SM::kOffQl - SM::kOffQh, status)) continue;
      float hi[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) hi[e] = __half2float(__float2half_rn(z[e]));
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sQh + off),
                   "r"(pack_f16x2(hi[0], hi[1])), "r"(pack_f16x2(hi[2], hi[3]))
                   : "memory");
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sQl + off),
                   "r"(pack_f16x2(z[0] - hi[0], z[1] - hi[1])),
                   "r"(pack_f16x2(z[2] - hi[2], z[3] - hi[3]))
                   : "memory");
    }
  }
  tc::fence_before();
  __syncthreads();  // barriers initialised, tensor memory allocated, query tiles written
  tc::fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_row = tmem + ((uint32_t)(warp * 32) << 16);  // this thread's lane

  uint32_t tl0, tl1, th0, th1;
  level_tables<BITS>(tl0, tl1, th0, th1);
  const float kf = scale * kLog2e / (ALPHA * (float)D);  // log2 score per (dot * nK)

  // this row's online-softmax state (log2 domain)
  float m2 = -CUDART_INF_F, lsum = 0.f;
  float sigma = 0.f;  // the CTA's V-norm reference (the same in every thread)
  bool fail = false;
  int n_s = 0, n_pv = 0;  // score / value-product commits so far (CTA-uniform)
  int k = 0;
  // dequantise K_hat (kv = 0) or V_hat (kv = 1) of the page in ring stage st into its tile
  auto dequant = [&](int st, int kv) {
    const uint8_t* blk = smem + SM::kOffRing + st * BB;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const int u = tid + 128 * hf;
      if (BITS == 3 && kv == 1) {
        // V tile layout: u = (block, quad, 8-dim unit) group of four tokens.  Lanes 4m ..
        // 4m+3 take quads 0-3 of one unit, so a warp's 12-byte group loads hit 32 distinct
        // banks.  A member's 16-byte tile row sits at chunk (2 quad + member bit 0) % 8 of
        // a 128-byte line, the same line for every member of a unit; lanes with an odd unit
        // store their members in the order 1 0 3 2 (nibbles swapped within each byte of
        // the words), so each quarter-warp's stores cover the 8 chunks once.
        const int t4 = u & 3, un = (u >> 2) & 15, B = u >> 6, jf = un & 1;
        const uint32_t* wp = reinterpret_cast<const uint32_t*>(
            blk + v_codes_off(D, BITS) + vt_group_off(D, B, t4, un));
        if (!in_bounds(vt_group_off(D, B, t4, un) + 12 <= kPage * CB, status)) continue;
        const int sh = 4 * jf;
        uint32_t w3[3];
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const uint32_t x = wp[i];
          w3[i] = ((x >> sh) & 0x0F0F0F0Fu) | ((x << sh) & 0xF0F0F0F0u);
        }
        uint32_t o[4][4];
        vdeq_group(w3[0], w3[1], w3[2], tl0, tl1, th0, th1, o);  // o[j]: member j ^ jf
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int tkj = vt_member_slot(B, t4, j ^ jf);
          const int vo = (tkj >> 3) * 2048 + un * 128 + (tkj & 7) * 16;
          if (!in_bounds(vo + 16 <= SM::kOffRing - SM::kOffV, status)) continue;
          st_v4(sV + vo, o[j]);
        }
        continue;
      }
      // token, 32-dim group: a warp takes 8 tokens x 4 groups, so its 32-bit code loads
      // (word 12 tk + 3 q + i) hit 32 distinct banks and each quarter-warp's 16-byte tile
      // stores 8 distinct bank groups (tk % 8)
      const int tk = 8 * (u >> 5) + (u & 7), q = (u >> 3) & 3;
      const uint32_t* wp = reinterpret_cast<const uint32_t*>(
                               blk + (kv ? v_codes_off(D, BITS) : 0) + tk * CB) + W * q;
      if (!in_bounds(tk * CB + 4 * W * (q + 1) <= kPage * CB, status)) continue;
      uint32_t w[W];
#pragma unroll
      for (int i = 0; i < W; ++i) w[i] = wp[i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t o[4];
        kdeq<BITS>(w, j, tl0, tl1, th0, th1, o);  // dims 32q + 8j .. +7 of token tk
        const int c = 4 * q + j;
        const uint32_t to = kv ? (tk >> 3) * 2048 + c * 128 + (tk & 7) * 16
                               : c * 1024 + (tk >> 3) * 128 + (tk & 7) * 16;
        if (!in_bounds(to + 16 <= (kv ? SM::kOffRing - SM::kOffV : SM::kOffV - SM::kOffK), status))
          continue;
        const uint32_t addr = (kv ? sV : sK) + to;
        st_v4(addr, o);
      }
    }
  };

  // Per page k: K_hat(k) -> tile; S(k) issued; V_hat(k) -> tile while S(k) runs; softmax;
  // O += P' V_hat issued, which runs while the next page's K_hat is dequantised.
  // page-table entry of the next page, loaded one page ahead (off the per-page chain)
  int phys_nx = n_my > 0 && in_bounds(p_begin < max_pages, status) ? __ldg(pt_row + p_begin) : -1;
  for (; k < n_my; ++k) {
    const int phys = phys_nx;
    if (k + 1 < n_my)
      phys_nx = in_bounds(p_begin + k + 1 < max_pages, status) ? __ldg(pt_row + p_begin + k + 1) : -1;
    // Three CTA barriers per page; every other hand-off is a thread's own mbarrier wait.
    // The K tile is free: S(k-1) completed before this thread's softmax read it.
    bool ok = mbar_wait(bars + (k & 1), (k >> 1) & 1);
    if (ok) dequant(k & 1, 0);
    fence_proxy_async();  // the generic-proxy tile writes, before the tensor core reads
    tc::fence_before();
    if (__syncthreads_or(!ok)) {
      fail = true;
      break;
    }
    if (tid == 0) {
      tc::fence_after();
      // ---- a7: S = Q~hi . K_hat^T + Q~lo . K_hat^T, 8 k-steps of 16 dims ---------------
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t bd = tc::sdesc(sK + kk * 2048, 1024, 128);
        tc::mma_ss(tmem + kColS, tc::sdesc(sQh + kk * 4096, 2048, 128), bd, kIdS, kk > 0);
        tc::mma_ss(tmem + kColS, tc::sdesc(sQl + kk * 4096, 2048, 128), bd, kIdS, 1);
      }
      tc::commit(bar_s);
    }
    ++n_s;
    // the V tile, P' and O are free once the previous value product has completed (this
    // thread's own wait); the norms of page k-1 were read before the last barrier
    ok = k == 0 || mbar_wait(bar_pv, (k - 1) & 1);
    if (ok) dequant(k & 1, 1);
    const int pg = p_begin + k;
    const bool page_ok = phys >= 0 && phys < n_pages;
    const int tok0 = pg * kPage;
    const bool full = page_ok && tok0 + kPage <= lim_lo;
    // norms: nrm[j] = |k_j| kf; nrm[64 + j] = |v_j| / sigma', where sigma' is the CTA's
    // V-norm reference (shared by all rows: it only scales the weights), raised when a
    // token valid for some row has |v| > kSigmaSlack sigma; computed by warps 2 and 3
    {
      const uint8_t* blk = smem + SM::kOffRing + (k & 1) * BB;
      if (tid < 64) {
        nrm[tid] = half_at(blk + k_norm_off(D, BITS) + 2 * tid) * kf;
      } else {
        const int j = tid - 64;
        float nv = half_at(blk + v_norm_off(D, BITS) + 2 * j);
        nv = page_ok && tok0 + j < lim_hi ? nv : 0.f;
        float pm = nv;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pm = fmaxf(pm, __shfl_xor_sync(kFull, pm, o));
        if (lane == 0) red[warp - 2] = pm;
        asm volatile("bar.sync 1, 64;" ::: "memory");  // warps 2 and 3 only
        pm = fmaxf(red[0], red[1]);
        const float sg = pm > sigma * kSigmaSlack ? pm : sigma;
        nrm[tid] = sg > 0.f ? nv * (1.f / sg) : 0.f;
        if (tid == 64) red[2] = sg;
      }
    }
    fence_proxy_async();
    if (__syncthreads_or(!ok)) {  // norms visible; the ring stage has been read in full
      fail = true;
      break;
    }
    if (tid == 0 && k + 2 < n_my) {  // the ring stage of page k takes page k + 2
      fence_proxy_async();
      issue(k + 2);
    }
    if (k + 2 < n_my) issued = k + 3;
    const float sigma_new = red[2];
    const float vr = sigma_new > sigma ? sigma / sigma_new : 1.f;  // 0 on the first valid page
    sigma = sigma_new;

    // ---- a8: this row's online softmax over the page's 64 tokens ----------------------
    ok = __all_sync(kFull, mbar_wait(bar_s, k & 1));  // warp-uniform: collectives below
    if (ok) {
    tc::fence_after();
    float x[64];
    {
      uint32_t sr[64];
      tc::ld64(t_row + kColS, sr);  // the row's 64 scores in one tensor-memory round trip
#pragma unroll
      for (int j = 0; j < 64; ++j) x[j] = __uint_as_float(sr[j]);
    }
    // FULL: every token of the page is valid for every row of the CTA (no masking).  The
    // exponents a_j = s_j - m2 come from one FMA each; the running maximum m2 moves only
    // when some a_j > kLazy (or on the row's first scores), and then O is rescaled in
    // place (it is idle: the last value product completed before this page's V tile was
    // written).
    auto softmax_page = [&](auto full_c) {
      constexpr bool FULL = decltype(full_c)::value;
      float resc = vr;
      bool moved = vr != 1.f;
      if (m2 == -CUDART_INF_F) {  // no finite score yet: exponents against this page's max
        float tm[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          float sc = x[j] * nrm[j];
          if constexpr (!FULL) sc = page_ok && tok0 + j < my_lim ? sc : -CUDART_INF_F;
          x[j] = sc;
          tm[j & 3] = fmaxf(tm[j & 3], sc);
        }
        const float tmax = fmaxf(fmaxf(tm[0], tm[1]), fmaxf(tm[2], tm[3]));
        if (tmax != -CUDART_INF_F) {
          m2 = tmax;
          resc = 0.f;  // nothing accumulated yet
          lsum = 0.f;
          moved = true;
        }
#pragma unroll
        for (int j = 0; j < 64; ++j) x[j] = x[j] - m2;  // -inf - -inf = NaN: masked below
      } else {
        float am[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
        const float2 nm2 = make_float2(-m2, -m2);
#pragma unroll
        for (int j4 = 0; j4 < 64; j4 += 4) {
          const float4 nk4 = *reinterpret_cast<const float4*>(nrm + j4);
          // a_j = s_j nK_j - m2, two tokens per packed FMA
          const float2 a01 = f2_fma(make_float2(x[j4], x[j4 + 1]), make_float2(nk4.x, nk4.y), nm2);
          const float2 a23 = f2_fma(make_float2(x[j4 + 2], x[j4 + 3]), make_float2(nk4.z, nk4.w), nm2);
          const float av[4] = {a01.x, a01.y, a23.x, a23.y};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = j4 + e;
            float a = av[e];
            if constexpr (!FULL) a = page_ok && tok0 + j < my_lim ? a : -CUDART_INF_F;
            x[j] = a;
            am[e] = fmaxf(am[e], a);
          }
        }
        const float amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
        if (amax > kLazy) {
          const float r = ex2(-amax);
          resc *= r;
          lsum *= r;
          m2 += amax;
#pragma unroll
          for (int j = 0; j < 64; ++j) x[j] -= amax;
          moved = true;
        }
      }
      // tensor-memory loads and stores are warp-collective: a warp rescales when any of its
      // rows moved (the others with factor 1)
      if (__any_sync(kFull, moved) && k > 0) {  // before the first product O holds nothing
        uint32_t ov[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tc::ld32(t_row + kColO + 32 * c, ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * resc);
          tc::st32(t_row + kColO + 32 * c, ov);
        }
      }
      uint32_t pw[32];
      float2 ls01 = make_float2(0.f, 0.f), ls23 = make_float2(0.f, 0.f);
#pragma unroll
      for (int j4 = 0; j4 < 64; j4 += 4) {
        const float4 nv4 = *reinterpret_cast<const float4*>(nrm + 64 + j4);
        float pe[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = x[j4 + e];
          pe[e] = ex2(a);  // a = -inf: 0
          if constexpr (!FULL) pe[e] = a == a ? pe[e] : 0.f;  // NaN from a row with no score yet
        }
        // row sums and weights p |v| / sigma' (masked tokens have p = 0), two per instruction
        const float2 p01 = make_float2(pe[0], pe[1]), p23 = make_float2(pe[2], pe[3]);
        ls01 = f2_add(ls01, p01);
        ls23 = f2_add(ls23, p23);
        const float2 w01 = f2_mul(p01, make_float2(nv4.x, nv4.y));
        const float2 w23 = f2_mul(p23, make_float2(nv4.z, nv4.w));
        pw[j4 / 2] = pack_f16x2(w01.x, w01.y);
        pw[j4 / 2 + 1] = pack_f16x2(w23.x, w23.y);
      }
      lsum += (ls01.x + ls01.y) + (ls23.x + ls23.y);
      tc::st32(t_row + kColP, pw);
    };
    if (full) softmax_page(std::true_type{});
    else softmax_page(std::false_type{});
    }
    tc::wait_st();
    tc::fence_before();
    if (__syncthreads_or(!ok)) {  // P' and any rescaled O rows are in TMEM; S has been read
      fail = true;
      break;
    }
    if (tid == 0) {
      tc::fence_after();
      // ---- a8: O += P' . V_hat, 4 k-steps of 16 tokens ---------------------------------
#pragma unroll
      for (int j = 0; j < 4; ++j)
        tc::mma_ts(tmem + kColO, tmem + kColP + 8 * j, tc::sdesc(sV + j * 4096, 2048, 128), kIdO,
                   (k > 0 || j > 0) ? 1u : 0u);
      tc::commit(bar_pv);
    }
    ++n_pv;
  }

  if (fail) {
    // a bounded wait gave up: wait (bounded) for this CTA's page copies and products still
    // in flight, so its shared and tensor memory are idle before they are released
    if (tid == 0) {
      set_status(status, ISOQ_ST_TIMEOUT);
      for (int kk = k; kk < issued; ++kk) mbar_wait(bars + (kk & 1), (kk >> 1) & 1);
    }
    if (n_s > 0) mbar_wait(bar_s, (n_s - 1) & 1);
    if (n_pv > 0) mbar_wait(bar_pv, (n_pv - 1) & 1);
  } else {
    // ---- the chunk's partial result of this row: O sigma / ALPHA, m, l ------------------
    const bool done = mbar_wait(bar_pv, (n_my - 1) & 1);
    if (__syncthreads_or(!done)) {
      if (tid == 0) set_status(status, ISOQ_ST_TIMEOUT);
    } else {
      tc::fence_after();
      float* o = out_base + (size_t)row_off[tid] * n_splits * PS;
      const bool w_ok = tid < nh && in_bounds(row_off[tid] < n_q * n_q_heads, status);
      const float f = sigma / ALPHA;  // O holds sum p |v| ALPHA L / sigma
      uint32_t ov[32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        tc::ld32(t_row + kColO + 32 * c, ov);  // warp-collective: every lane loads
        if (w_ok) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(o + 32 * c + j) =
                make_float4(__uint_as_float(ov[j]) * f, __uint_as_float(ov[j + 1]) * f,
                            __uint_as_float(ov[j + 2]) * f, __uint_as_float(ov[j + 3]) * f);
        }
      }
      if (w_ok) {
        o[D] = m2 == -CUDART_INF_F ? -CUDART_INF_F : m2 / kLog2e;  // natural-log units
        o[D + 1] = lsum;
      }
    }
  }
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::dealloc(tmem, kXCols);
  }
}

template <typename TQ, int BITS>
cudaError_t launch_mqtc_t(const DecodeArgs& a, cudaStream_t stream) {
  using SM = MqtcSmem<BITS>;
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_mqtc_kernel<TQ, BITS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, SM::kBytes);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  const int G = a.n_q_heads / a.n_kv_heads;
  dim3 grid(a.n_splits, a.n_kv_heads * ((a.n_q * G + kXRows - 1) / kXRows), a.n_seqs);
  decode_mqtc_kernel<TQ, BITS><<<grid, kXRows, SM::kBytes, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_kv_heads,
      static_cast<const TQ*>(a.Q), a.n_q_heads, a.n_q, a.seq_lens, a.scale, a.pages_per_split,
      a.n_splits, a.partials, a.status);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_mqtc_b(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.q_dtype) {
    case ISOQ_F32: return launch_mqtc_t<float, BITS>(a, stream);
    case ISOQ_BF16: return launch_mqtc_t<__nv_bfloat16, BITS>(a, stream);
    case ISOQ_F16: return launch_mqtc_t<__half, BITS>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_split_mqtc(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.bits) {
    case 2: return launch_mqtc_b<2>(a, stream);
    case 3: return launch_mqtc_b<3>(a, stream);
    case 4: return launch_mqtc_b<4>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace isoq
