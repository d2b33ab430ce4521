// Decode attention on the packed 3-bit cache with the 5th-generation tensor cores
// (tcgen05 / UMMA, accumulators in tensor memory), head dimension 128.
//
// Method: "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
// Compressed-Space Attention", Abstract: attention is computed on the packed 3-bit codes
// and full-precision K/V are never reconstructed in memory.  With R orthogonal,
// q.k_hat = (R q).(R k_hat): the queries are rotated once per CTA and scores and the value
// accumulation run on codebook levels in the rotated space.
//
// One CTA of 128 threads per (context chunk, KV head, block of <= 8 query heads,
// sequence); the chunk is processed in tiles of 128 tokens (two pages), thread i owning
// token i of the tile:
//   - thread 0 streams the tile's two page blocks into a 2-stage shared-memory ring with
//     1-D bulk copies (completion on mbarriers; every wait is bounded);
//   - every thread turns its token's K codes into 64 f16 pairs (byte-permute lookups of
//     the levels' low/high bytes) and stores them into its lane of tensor memory;
//   - thread 0 issues S[128 tok x 16] = K_hat . Q~^T (16 UMMAs, A from tensor memory, Q~
//     as f16 hi + lo parts in shared memory, accumulator in tensor memory);
//   - meanwhile every thread dequantises its token's V codes the same way into a
//     token-major shared tile (the MN-major A operand of the value product);
//   - each thread reads its token's 16 scores, runs the online softmax (running maxima
//     raised lazily, decided by one CTA-wide vote per tile) and writes its weights
//     P' = p * |v| / sigma for the 8 heads (the MN-major B operand);
//   - thread 0 issues O^T[128 dims x 16] += V_hat^T . P' (8 UMMAs, accumulator in tensor
//     memory for the whole chunk).
// At the end the accumulator is read back once and written as the chunk's partial result.
#include <math_constants.h>

#include "isoq_common.cuh"
#include "isoq_internal.h"
#include "isoq_ptx.cuh"

namespace isoq {
using namespace ptx;
namespace {

constexpr int kTcD = 128;
constexpr int kTcTile = 128;         // tokens per tile = threads per CTA
constexpr int kTcStages = 2;         // tiles in flight in the page ring
constexpr int kTmemCols = 128;       // A (64) | S (16) | O (16), rounded to a power of two
constexpr int kColA = 0, kColS = 64, kColO = 80;
// instruction descriptors (kind::f16, f16 inputs, f32 accumulate, M = 128, N = 16):
// scores with A and B K-major; the value product with A and B MN-major
constexpr uint32_t kIdescScores = (1u << 4) | (16u >> 3 << 17) | (128u >> 4 << 24);
constexpr uint32_t kIdescValues = kIdescScores | (1u << 15) | (1u << 16);

// shared-memory layout (bytes), every operand region 1024-byte aligned
constexpr int kBB = block_bytes(kTcD);                       // 6400
constexpr int kOffRing = 0;                                  // [stage][2 pages][6400]
constexpr int kOffV = 26624;                                 // V_hat tile, 32 KiB
constexpr int kOffP = kOffV + 32768;                         // P' tile, 4 KiB
constexpr int kOffQh = kOffP + 4096;                         // Q~ hi, 4 KiB
constexpr int kOffQl = kOffQh + 4096;                        // Q~ lo, 4 KiB
constexpr int kOffBar = kOffQl + 4096;                       // mbarriers
constexpr int kOffRed = kOffBar + 64;                        // reductions [4][12] floats
constexpr int kOffTmem = kOffRed + 4 * 12 * 4;               // tensor-memory base address
constexpr int kTcSmem = kOffTmem + 16;
static_assert(kTcStages * 2 * kBB <= kOffV, "ring overlaps the V tile");

// UMMA shared-memory matrix descriptor, no swizzle: start, leading-dimension byte offset
// (between the two 8-element K chunks of one instruction, or between K groups for
// MN-major), stride byte offset (between 8-row groups), version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&v)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, "
      "%47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64};" ::
          "r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
      "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31]),
      "r"(v[32]), "r"(v[33]), "r"(v[34]), "r"(v[35]), "r"(v[36]), "r"(v[37]), "r"(v[38]), "r"(v[39]),
      "r"(v[40]), "r"(v[41]), "r"(v[42]), "r"(v[43]), "r"(v[44]), "r"(v[45]), "r"(v[46]), "r"(v[47]),
      "r"(v[48]), "r"(v[49]), "r"(v[50]), "r"(v[51]), "r"(v[52]), "r"(v[53]), "r"(v[54]), "r"(v[55]),
      "r"(v[56]), "r"(v[57]), "r"(v[58]), "r"(v[59]), "r"(v[60]), "r"(v[61]), "r"(v[62]), "r"(v[63])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Load 16 columns of this thread's lane and wait for the load in the same statement, so no
// use of the registers can be scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];\n tcgen05.wait::ld.sync.aligned;"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

}  // namespace

template <typename TQ>
__global__ void __launch_bounds__(kTcTile)
    decode_tc_kernel(const float* __restrict__ params, const uint8_t* __restrict__ blocks,
                     const int32_t* __restrict__ page_table, int n_pages, int max_pages, int H,
                     const TQ* __restrict__ Q, int n_q_heads, const int32_t* __restrict__ seq_lens,
                     float scale, int pages_per_split, int n_splits, float* __restrict__ partials,
                     uint32_t* status) {
  constexpr int D = kTcD, E = D / 32, NB = E / 4, CB = code_bytes(D), PS = D + 4;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* ring_bar = reinterpret_cast<uint64_t*>(smem + kOffBar);   // [kTcStages]
  uint64_t* bar_s = ring_bar + kTcStages;                              // scores done
  uint64_t* bar_pv = bar_s + 1;                                        // value product done
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, s = blockIdx.z;
  const int G = n_q_heads / H;
  const int nhb = (G + 7) >> 3;
  const int hk = blockIdx.y / nhb, hb = blockIdx.y - hk * nhb;
  const int h0 = hk * G + hb * 8;
  const int nh = min(8, G - hb * 8);

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
  const int n_tiles = (p_end - p_begin + 1) / 2;
  const int* pt_row = page_table + (size_t)s * max_pages;

  // ---- tensor memory, barriers, first page copies ---------------------------------------
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int i = 0; i < kTcStages + 2; ++i) mbar_init(ring_bar + i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // tile t = pages p_begin + 2t, +1; a page beyond the chunk or with a bad id is not copied
  auto issue_tile = [&](int t) {  // thread 0 only
    const int st = t % kTcStages;
    int phys[2];
    unsigned bytes = 0;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int pg = p_begin + 2 * t + k;
      phys[k] = -1;
      if (pg < p_end) {
        const int ph = __ldg(pt_row + pg);
        if (ph >= 0 && ph < n_pages) {
          phys[k] = ph;
          bytes += kBB;
        } else {
          set_status(status, ISOQ_ST_PAGE_RANGE);
        }
      }
    }
    if (bytes) {
      mbar_expect_tx(ring_bar + st, bytes);
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (phys[k] >= 0)
          bulk_copy(smem + kOffRing + (st * 2 + k) * kBB, blocks + ((size_t)phys[k] * H + hk) * kBB,
                    kBB, ring_bar + st);
    } else {
      mbar_arrive(ring_bar + st);
    }
  };
  __syncthreads();
  if (tid == 0)
    for (int t = 0; t < kTcStages && t < n_tiles; ++t) issue_tile(t);
  int issued = min(kTcStages, n_tiles);  // tiles whose copies were issued (CTA-uniform)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_lane = (uint32_t)(warp * 32) << 16;  // this warp's lane quarter

  // ---- a6: rotate the CTA's queries (unnormalised WHT + SO(4)), staged fp32 in the V tile
  {
    float* qs = reinterpret_cast<float*>(smem + kOffV);  // [8][D], reused later
    const float* hp = params + (size_t)hk * D * 4;  // this head's block matrices
    float pq[NB][16];
#pragma unroll
    for (int k = 0; k < NB; ++k) load_block_mat(hp, lane * NB + k, pq[k]);
    for (int h = warp; h < 8; h += 4) {
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
      for (int k = 0; k < NB; ++k) mat_fwd(pq[k], v + 4 * k, z + 4 * k);
#pragma unroll
      for (int i = 0; i < E; ++i) qs[h * D + lane * E + i] = z[i];
    }
    __syncthreads();
    // B operand of the score product: N = 16 heads (8..15 zero) x K = 128 dims, K-major,
    // element (n, k) at (k/8)*256 + (n/8)*128 + (n%8)*16 + (k%8)*2; as f16 hi and lo parts.
    {
      const int n = tid >> 3;            // 0..15
      const int k0 = (tid & 7) * 16;     // 16 dims per thread
      uint32_t* qh = reinterpret_cast<uint32_t*>(smem + kOffQh);
      uint32_t* ql = reinterpret_cast<uint32_t*>(smem + kOffQl);
#pragma unroll
      for (int kp = 0; kp < 16; kp += 2) {
        const int k = k0 + kp;
        float a = 0.f, b = 0.f;
        if (n < 8) {
          a = qs[n * D + k];
          b = qs[n * D + k + 1];
        }
        const float ah = __half2float(__float2half_rn(a)), bh = __half2float(__float2half_rn(b));
        const int off = ((k >> 3) * 256 + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) >> 2;
        qh[off] = pack_f16x2(ah, bh);
        ql[off] = pack_f16x2(a - ah, b - bh);
      }
    }
    // P' tile: heads 8..15 stay zero for the whole chunk
    {
      uint32_t* pz = reinterpret_cast<uint32_t*>(smem + kOffP);
      for (int i = tid; i < 1024; i += kTcTile) pz[i] = 0u;
    }
    // zero the value accumulator (this thread's lane, 16 columns)
    {
      uint32_t z16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) z16[i] = 0u;
      tmem_st16(tmem + t_lane + kColO, z16);
      tmem_wait_st();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();  // qs (in the V tile) is dead from here on
    tc_fence_after();
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
  const float kf = scale * kLog2e / (kAlpha * (float)D);
  const uint32_t sQh = smem_u32(smem + kOffQh), sQl = smem_u32(smem + kOffQl);
  const uint32_t sV = smem_u32(smem + kOffV), sP = smem_u32(smem + kOffP);

  float m2[8], lsum[8];  // running max (log2 domain, CTA-uniform) and this token's share of l
#pragma unroll
  for (int h = 0; h < 8; ++h) {
    m2[h] = -CUDART_INF_F;
    lsum[h] = 0.f;
  }
  float sigma = 0.f;      // V-norm reference (CTA-uniform)
  bool fail = false;      // a bounded wait gave up (CTA-uniform after each vote)
  int t = 0;

  for (; t < n_tiles && !fail; ++t) {
    const int st = t % kTcStages;
    bool ok = mbar_wait(ring_bar + st, (t / kTcStages) & 1);
    const int pgi = tid >> 6, slot = tid & (kPage - 1);
    const int pg = p_begin + 2 * t + pgi;
    bool valid = false;
    if (pg < p_end) {
      const int ph = __ldg(pt_row + pg);
      valid = ph >= 0 && ph < n_pages && pg * kPage + slot < len;
    }
    const uint8_t* blk = smem + kOffRing + (st * 2 + pgi) * kBB;

    // ---- a7 (operand): this token's K_hat row -> tensor memory lane ------------------
    {
      const uint4* rec = reinterpret_cast<const uint4*>(blk + slot * CB);
      const uint4 r0 = rec[0], r1 = rec[1], r2 = rec[2];
      const uint32_t w[12] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w, r2.x, r2.y, r2.z, r2.w};
      uint32_t a[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t S[4];
        selectors(w[3 * q], w[3 * q + 1], w[3 * q + 2], S);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t o[4];
          deq8(S[j], tl0, tl1, th0, th1, o);
#pragma unroll
          for (int m = 0; m < 4; ++m) a[16 * q + 4 * j + m] = o[m];
        }
      }
      tmem_st64(tmem + t_lane + kColA, a);
      tmem_wait_st();
    }
    tc_fence_before();
    ok = !__syncthreads_or(!ok);  // every thread saw the pages (or the CTA gives up)
    if (!ok) {
      fail = true;
      break;
    }
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        mma_ts(tmem + kColS, tmem + kColA + 8 * kk, sdesc(sQh + 512 * kk, 256, 128), kIdescScores,
               kk > 0);
        mma_ts(tmem + kColS, tmem + kColA + 8 * kk, sdesc(sQl + 512 * kk, 256, 128), kIdescScores, 1);
      }
      mma_commit(bar_s);
    }

    // ---- a8 (operand): this token's V_hat row -> the token-major V tile -------------
    if (t > 0) ok = mbar_wait(bar_pv, (t - 1) & 1) && ok;  // previous value product done
    {
      const uint4* rec = reinterpret_cast<const uint4*>(blk + v_codes_off(D) + slot * CB);
      const uint4 r0 = rec[0], r1 = rec[1], r2 = rec[2];
      const uint32_t w[12] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w, r2.x, r2.y, r2.z, r2.w};
      // dims 8c..8c+7 of token i at c*128 + (i/8)*2048 + (i%8)*16
      const uint32_t vrow = sV + (tid >> 3) * 2048 + (tid & 7) * 16;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t S[4];
        selectors(w[3 * q], w[3 * q + 1], w[3 * q + 2], S);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t o[4];
          deq8(S[j], tl0, tl1, th0, th1, o);
          st_shared_v4(vrow + (4 * q + j) * 128, o[0], o[1], o[2], o[3]);
        }
      }
    }
    const float nk = half_at(blk + k_norm_off(D) + 2 * slot);
    const float nv = valid ? half_at(blk + v_norm_off(D) + 2 * slot) : 0.f;

    // ---- a7: this token's scores from tensor memory ---------------------------------
    ok = mbar_wait(bar_s, t & 1) && ok;
    tc_fence_after();
    uint32_t sr[16];
    tmem_ld16(tmem + t_lane + kColS, sr);
    float s2[8];
    const float f = nk * kf;
    bool grow = valid && nv > sigma * kSigmaSlack;
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      s2[h] = valid ? __uint_as_float(sr[h]) * f : -CUDART_INF_F;
      grow = grow || (s2[h] > m2[h] + kLazy);
    }

    // ---- a8: online softmax; the rare re-basing is decided by one CTA-wide vote -------
    const int vote = __syncthreads_or(grow ? 1 : 0);
    if (__syncthreads_or(!ok)) {
      fail = true;
      break;
    }
    if (vote) {
      float mx[9];
#pragma unroll
      for (int h = 0; h < 8; ++h) mx[h] = warp_max(s2[h]);
      mx[8] = warp_max(nv);
      if (lane == 0)
#pragma unroll
        for (int h = 0; h < 9; ++h) red[warp * 12 + h] = mx[h];
      __syncthreads();
      float resc[8];
      bool any = false;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float tm = fmaxf(fmaxf(red[h], red[12 + h]), fmaxf(red[24 + h], red[36 + h]));
        resc[h] = 1.f;
        if (tm > m2[h] + kLazy) {
          resc[h] = ex2(m2[h] - tm);  // 0 when m2 was -inf
          lsum[h] *= resc[h];
          m2[h] = tm;
          any = true;
        }
      }
      const float vm = fmaxf(fmaxf(red[8], red[20]), fmaxf(red[32], red[44]));
      if (vm > sigma * kSigmaSlack) {
        const float r = sigma / vm;  // 0 on the first valid tile
#pragma unroll
        for (int h = 0; h < 8; ++h) resc[h] *= r;
        sigma = vm;
        any = true;
      }
      if (any) {  // CTA-uniform; the previous value product has completed
        uint32_t o16[16];
        tmem_ld16(tmem + t_lane + kColO, o16);
#pragma unroll
        for (int h = 0; h < 8; ++h) o16[h] = __float_as_uint(__uint_as_float(o16[h]) * resc[h]);
        tmem_st16(tmem + t_lane + kColO, o16);
        tmem_wait_st();
      }
      __syncthreads();  // red[] is read by everyone before it can be reused
    }
    {
      const float w = sigma > 0.f ? nv / sigma : 0.f;
      float pw[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float p = valid ? ex2(s2[h] - m2[h]) : 0.f;
        lsum[h] += p;
        pw[h] = p * w;
      }
      // P' row of token i (heads 0..7) at (i/8)*256 + (i%8)*16
      st_shared_v4(sP + (tid >> 3) * 256 + (tid & 7) * 16, pack_f16x2(pw[0], pw[1]),
                   pack_f16x2(pw[2], pw[3]), pack_f16x2(pw[4], pw[5]), pack_f16x2(pw[6], pw[7]));
    }

    // ---- a8: O^T += V_hat^T . P' over the tile's 128 tokens -------------------------
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < 8; ++j)
        mma_ss(tmem + kColO, sdesc(sV + 2 * j * 2048, 2048, 128), sdesc(sP + 2 * j * 256, 256, 128),
               kIdescValues, 1);
      mma_commit(bar_pv);
      if (t + kTcStages < n_tiles) issue_tile(t + kTcStages);  // the stage has been consumed
    }
    if (t + kTcStages < n_tiles) ++issued;
  }
  if (fail) {
    // a wait gave up: wait (bounded) for this CTA's page copies and products still in
    // flight, so its shared and tensor memory are idle before they are released
    for (int k = t; k < issued; ++k) mbar_wait(ring_bar + k % kTcStages, (k / kTcStages) & 1);
    mbar_wait(bar_s, t & 1);
    if (t > 0) mbar_wait(bar_pv, (t - 1) & 1);
  }

  // ---- the chunk's partial: O (rows = dims), m, l ----------------------------------------
  bool done = !fail && mbar_wait(bar_pv, (n_tiles - 1) & 1);
  if (__syncthreads_or(!done)) {
    if (tid == 0) set_status(status, ISOQ_ST_TIMEOUT);
  } else {
    tc_fence_after();
    uint32_t o16[16];
    tmem_ld16(tmem + t_lane + kColO, o16);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float v = lsum[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
      if (lane == 0) red[warp * 12 + h] = v;
    }
    __syncthreads();
    const float fo = sigma / kAlpha;  // O holds sum p * |v| * ALPHA * L / sigma
    for (int h = 0; h < nh; ++h) {
      float* o = out_base + (size_t)h * n_splits * PS;
      o[tid] = __uint_as_float(o16[h]) * fo;
      if (tid == 0) {
        o[D] = m2[h] == -CUDART_INF_F ? -CUDART_INF_F : m2[h] / kLog2e;
        o[D + 1] = red[h] + red[12 + h] + red[24 + h] + red[36 + h];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

template <typename TQ>
static cudaError_t launch_tc_t(const DecodeArgs& a, cudaStream_t stream) {
  static unsigned long long attr_set = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && !((attr_set >> dev) & 1ull)) {
    e = cudaFuncSetAttribute(decode_tc_kernel<TQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kTcSmem);
    if (e != cudaSuccess) return e;
    attr_set |= 1ull << dev;
  }
  const int G = a.n_q_heads / a.n_kv_heads;
  dim3 grid(a.n_splits, a.n_kv_heads * ((G + 7) / 8), a.n_seqs);
  decode_tc_kernel<TQ><<<grid, kTcTile, kTcSmem, stream>>>(
      a.params, a.blocks, a.page_table, a.n_pages, a.max_pages, a.n_kv_heads,
      static_cast<const TQ*>(a.Q), a.n_q_heads, a.seq_lens, a.scale, a.pages_per_split,
      a.n_splits, a.partials, a.status);
  return cudaGetLastError();
}

cudaError_t launch_decode_split_tc(const DecodeArgs& a, cudaStream_t stream) {
  if (a.d != 128) return cudaErrorInvalidValue;
  switch (a.q_dtype) {
    case ISOQ_F32: return launch_tc_t<float>(a, stream);
    case ISOQ_BF16: return launch_tc_t<__nv_bfloat16>(a, stream);
    case ISOQ_F16: return launch_tc_t<__half>(a, stream);
  }
  return cudaErrorInvalidValue;
}

// Resident CTAs per SM: the smaller of what shared memory (per SM, minus the per-CTA
// reservation), registers and tensor-memory columns (512 per SM) allow.
int decode_tc_resident_ctas() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 3;
  }
  if (!cache[dev]) {
    int smem_sm = 0, reserved = 0, regs_sm = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, decode_tc_kernel<__nv_bfloat16>);
    int n = 3;
    if (e == cudaSuccess) {
      const int by_smem = smem_sm / (kTcSmem + reserved);
      const int regs_cta = ((fa.numRegs * 32 + 255) / 256 * 256) * (kTcTile / 32);
      const int by_regs = regs_cta > 0 ? regs_sm / regs_cta : by_smem;
      const int by_tmem = 512 / kTmemCols;
      n = by_smem < by_regs ? by_smem : by_regs;
      if (by_tmem < n) n = by_tmem;
      if (n < 1) n = 1;
    } else {
      cudaGetLastError();
    }
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace isoq
