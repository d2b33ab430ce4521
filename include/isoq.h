/*
 * isoq.h -- C ABI of libisoq: IsoQuant 3-bit KV-cache compression and decode attention
 * computed directly on the packed cache, for NVIDIA B200 (sm_100a).
 *
 * The method is the IsoQuant axis of "RotaryQuant: Fitting 120B MoE Models on Consumer
 * Hardware via Fused Compressed-Space Attention" (arXiv 2608.08081v1), Abstract: every
 * per-token, per-head K or V vector is passed through a Walsh-Hadamard transform, then
 * block-diagonal SO(4) rotations (quaternion rotations: "FreeToken issue #141, unified KV
 * cache backend", Proposed Solution, Quantization layer), then 3-bit scalar
 * quantisation; attention reads the packed 3-bit codes directly and never rebuilds
 * full-precision K/V.  The pages fix none of the numeric details below; this library's
 * choices are stated with each declaration.
 *
 * Conventions for every call:
 *   - Return value: ISOQ_OK (0) or a negative ISOQ_E_* code.  No exception, abort or
 *     device trap crosses this boundary.
 *   - Pointers documented as "device" must point to memory of the CUDA device that is
 *     current when the call is made; the caller owns all of them (the library keeps no
 *     reference after the call returns, except inside an isoq_params handle).
 *   - GPU work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = the legacy
 *     default stream) and the call returns without waiting for it.  Only
 *     isoq_make_params, isoq_params_copy and isoq_get_status synchronise.
 *   - Errors the device detects (an out-of-range sequence id, position or page id; a norm
 *     that overflows binary16) never fault: the offending write is skipped (or the value
 *     saturated) and a bit is OR-ed into the caller's status word, read with
 *     isoq_get_status.
 *   - The library allocates device memory only inside isoq_make_params.
 */
#ifndef ISOQ_H
#define ISOQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------------------ */
#define ISOQ_OK 0
#define ISOQ_E_ARG (-1)       /* null pointer, negative count, unknown dtype, bad scale */
#define ISOQ_E_DIM (-2)       /* head dimension or page size not supported */
#define ISOQ_E_GQA (-3)       /* n_q_heads not a multiple of n_kv_heads, or group > 16 */
#define ISOQ_E_WORKSPACE (-4) /* workspace smaller than isoq_decode_workspace_bytes() */
#define ISOQ_E_CUDA (-5)      /* a CUDA runtime call failed; see isoq_last_cuda_error() */
#define ISOQ_E_DEVICE (-6)    /* no CUDA device, or params made on another device */

/* ---- device status bits (sticky; OR-ed into isoq_cache.status) ------------------------ */
#define ISOQ_ST_SEQ_RANGE 0x1u  /* quantize: seq_id outside [0, n_seqs); token skipped */
#define ISOQ_ST_POS_RANGE 0x2u  /* quantize: position < 0 or beyond the page table; skipped */
#define ISOQ_ST_PAGE_RANGE 0x4u /* a page-table entry outside [0, n_pages); page skipped */
#define ISOQ_ST_NORM_SAT 0x8u   /* a norm >= 65520 was stored as 65504 (binary16 max) */
#define ISOQ_ST_LEN_RANGE 0x10u /* decode: seq_len beyond the page table; clamped */
#define ISOQ_ST_TIMEOUT 0x20u   /* decode: a bounded wait for a page copy gave up (no hang) */
#define ISOQ_ST_BOUNDS 0x40u    /* bounds-checked build only: a kernel index fell outside its
                                   extent; that access was skipped (see isoq_selftest_bounds) */

/* ---- element types of K, V and Q ---------------------------------------------------- */
#define ISOQ_F32 0
#define ISOQ_BF16 1
#define ISOQ_F16 2

/* ---- supported sizes ------------------------------------------------------------------ */
#define ISOQ_PAGE_SIZE 64 /* tokens per cache page (the only page size supported) */
/* Head dimensions d: 128 and 256.  The packed format needs d % 32 == 0. */

/* =======================================================================================
 * Rotation parameters.
 *
 * Per KV head, one unit-quaternion pair (p_b, q_b) per 4-element block b = 0..d/4-1,
 * rotating the block y_b (read as the quaternion w + x i + y j + z k, Hamilton
 * convention) to z_b = p_b * y_b * conj(q_b).  That is d/4 * 8 = 256 stored parameters
 * per head at d = 128 (the paper's count, versus d^2 = 16,384 for a dense rotation).
 * K and V of one KV head share the same parameters.
 *
 * Values are drawn from SplitMix64 (Steele, Lea & Flood, OOPSLA 2014) seeded with `seed`:
 * for head h, block b, then p before q, four standard normals, each from two successive
 * 64-bit draws k1, k2 as sqrt(-2 ln u1) cos(2 pi u2) with u1 = ((k1>>11)+1) 2^-53 and
 * u2 = (k2>>11) 2^-53 (Box-Muller), computed in binary64; the 4-vector is divided by its
 * Euclidean length (uniform on the 3-sphere, so the block rotation is Haar on SO(4)) and
 * rounded to binary32.  Layout of the float array: [n_kv_heads][d/4][2][4], component
 * order (w, x, y, z).
 * ===================================================================================== */
typedef struct isoq_params isoq_params; /* opaque: d, n_kv_heads, device copy, host copy */

/* Host only, needs no GPU: writes the n_kv_heads * d * 2 floats described above into
 * host_out.  Errors: ISOQ_E_ARG (null, n_kv_heads < 1), ISOQ_E_DIM (d not 128 or 256). */
int isoq_params_generate(uint64_t seed, int d, int n_kv_heads, float* host_out);

/* Generates the parameters and uploads them to the current device (cudaMalloc +
 * synchronous copy).  *out receives a handle to free with isoq_params_destroy.
 * Errors: as isoq_params_generate, plus ISOQ_E_DEVICE / ISOQ_E_CUDA. */
int isoq_make_params(uint64_t seed, int d, int n_kv_heads, isoq_params** out);

/* Copies the binary32 parameters ([n_kv_heads][d/4][2][4]; see the variants below for
 * SO(2) handles) to host_dst. */
int isoq_params_copy(const isoq_params* params, float* host_dst);

/* d and n_kv_heads of a handle (either pointer may be NULL). */
int isoq_params_shape(const isoq_params* params, int* d, int* n_kv_heads);

/* Frees the device copy and the handle.  NULL is ignored. */
void isoq_params_destroy(isoq_params* params);

/* =======================================================================================
 * Format variants of the same family.
 *
 * "RotaryQuant ...", Abstract, places IsoQuant in a family of 3-4 bit methods and names a
 * planar variant, PlanarQuant, without defining it.  This library offers:
 *   - bits: 3 (the method), or 2 / 4 bits per code with the 4- and 16-level Lloyd-Max
 *     quantisers for N(0,1) (J. Max 1960, Table I):
 *       2 bits: L = {-1.5104, -0.4528, 0.4528, 1.5104}
 *       4 bits: L = +-{0.1284, 0.3881, 0.6568, 0.9424, 1.2562, 1.6180, 2.0690, 2.7326};
 *     thresholds are midpoints, ties take the upper code, a zero vector codes 2^(bits-1);
 *     2 and 4 bits need d = 128 (ISOQ_E_DIM otherwise).
 *   - rotation: ISOQ_ROT_SO4 (the method: quaternion-pair blocks as above) or
 *     ISOQ_ROT_SO2 (PlanarQuant read as 2x2 blocks): after the same WHT, dims (2b, 2b+1)
 *     are rotated by [cos phi_b, -sin phi_b; sin phi_b, cos phi_b], phi_b = 2 pi u with u
 *     the top 53 bits of one SplitMix64 draw (seeded with `seed`, head-major) times 2^-53
 *     (Haar on SO(2)); parameters [n_kv_heads][d/2][2] = (cos, sin) rounded to binary32,
 *     d floats per head.
 * Packed codes (bits * d / 8 bytes per vector, little-endian 32-bit words):
 *   3 bits: the layout of the paged-cache section below;
 *   4 bits: word j holds dims 8j..8j+7, nibble k = dim 8j+k in sign-magnitude form: code
 *     c >= 8 -> c - 8, c < 8 -> 8 | (7 - c) (bit 3 = negative level, bits 0-2 the index of
 *     the level's magnitude);
 *   2 bits: word j holds dims 16j..16j+15, 2-bit slot s (bits 2s, 2s+1) holding dim
 *     16j + 2s (s < 4), 16j + 2(s-4) + 1 (s < 8), 16j + 8 + 2(s-8) (s < 12) or
 *     16j + 9 + 2(s-12), code = level index 0..3.
 * Every other call takes its format from the params handle; a cache (isoq_cache.bits
 * equal to the handle's bits) holds blocks of isoq_block_bytes_v(d, bits, 64) bytes.
 * ===================================================================================== */
#define ISOQ_ROT_SO4 0
#define ISOQ_ROT_SO2 1

/* Host only: the parameters of `rotation` (SO4: [H][d/4][2][4]; SO2: [H][d/2][2]). */
int isoq_params_generate_v(uint64_t seed, int d, int n_kv_heads, int rotation,
                           float* host_out);

/* As isoq_make_params with a format.  Errors: ISOQ_E_ARG (unknown rotation), ISOQ_E_DIM
 * (d, or bits not 2/3/4, or 2/4 bits with d != 128), ISOQ_E_DEVICE, ISOQ_E_CUDA.
 * isoq_make_params(seed, d, H, out) = isoq_make_params_v(seed, d, H, 3, ISOQ_ROT_SO4, out). */
int isoq_make_params_v(uint64_t seed, int d, int n_kv_heads, int bits, int rotation,
                       isoq_params** out);

/* bits and rotation of a handle (either pointer may be NULL).  isoq_params_copy writes
 * the rotation's parameter layout (d floats per head for SO2). */
int isoq_params_format(const isoq_params* params, int* bits, int* rotation);

/* Bytes of one (page, KV head) block: 2 * page_size * (bits * d / 8 + 2); 0 if unsupported. */
size_t isoq_block_bytes_v(int d, int bits, int page_size);

/* =======================================================================================
 * Paged cache.
 *
 * blocks: device uint8 [n_pages][n_kv_heads][isoq_block_bytes(d, 64)].  One block holds
 * one KV head of one 64-token page:
 *     K codes [64][3d/8] | K norms [64] binary16 | V codes (64 * 3d/8 bytes) | V norms [64]
 * (6400 bytes at d = 128, 12544 at d = 256; both multiples of 16).
 *
 * K codes of one slot (3 bits each, 3d/8 bytes): d/32 groups of 12 bytes; group g covers
 * dims 32g..32g+31 and is three little-endian 32-bit words w0, w1, w2:
 *     dim 32g + 8j + k (j = 0,1,2; k = 0..7): the code is bits 4k..4k+2 of w_j;
 *     dim 32g + 24 + k (k = 0..7): bit (2 - b) of the code is bit 4k+3 of w_b.
 * 3-bit V codes of a page ("V tile layout"): 4 blocks of 16 slots, 6d bytes each.  In
 * block B, quad t (0..3) is the slots 16B + 2t + {0, 1, 8, 9}, member j of the quad being
 * slot 16B + 2t + (j & 1) + 8 (j >> 1); unit u is dims 8u..8u+7.  The 12-byte group of
 * (quad t, unit u) starts at byte ((u >> 1) * 8 + 2t + (u & 1)) * 12 of the block and is
 * three little-endian words W0, W1, W2:
 *     bits 4n..4n+2 of W_b: the code of member n & 3 at dim 8u + 2b + (n >> 2);
 *     bit 4n+3 of W_b: bit (2 - b) of the code of member n & 3 at dim 8u + 6 + (n >> 2)
 * (n = 0..7).  Each 16-bit half of a word is thus four tokens' codes of one dim, the
 * operand shape of the decode's value product.  At 2 and 4 bits V codes are one record
 * per slot, like K.
 * A code c in 0..7 indexes the ascending levels
 *     L = {-2.1520, -1.3440, -0.7560, -0.2451, 0.2451, 0.7560, 1.3440, 2.1520}
 * (the 8-level Lloyd-Max quantiser for N(0,1), J. Max 1960), and stands for the rotated
 * coordinate (norm / sqrt(d)) * L[c].  The norm is the input vector's L2 norm rounded to
 * binary16 (round to nearest even; >= 65520 saturates to 65504 with ISOQ_ST_NORM_SAT).
 *
 * page_table: device int32 [n_seqs][max_pages_per_seq]: token position t of sequence s
 * lives in physical page page_table[s][t / 64], slot t % 64.  Pages may be in any order.
 * status: device uint32, one word; the caller zeroes it (isoq_reset_status) and the
 * kernels OR ISOQ_ST_* bits into it.  May be NULL (bits are then dropped).
 * ===================================================================================== */
typedef struct isoq_cache {
  int d;                     /* head dimension: 128 or 256 */
  int n_kv_heads;            /* KV heads held per page */
  int page_size;             /* must be ISOQ_PAGE_SIZE */
  int n_pages;               /* physical pages in `blocks` */
  int max_pages_per_seq;     /* row length of page_table */
  int n_seqs;                /* rows of page_table */
  uint8_t* blocks;           /* device */
  const int32_t* page_table; /* device */
  uint32_t* status;          /* device, optional */
  int bits;                  /* bits per code of the blocks (0 = 3, the method); must
                                equal the params' bits, else ISOQ_E_DIM */
} isoq_cache;

/* Bytes of one (page, KV head) block: 2 * page_size * (3d/8 + 2); 0 if unsupported. */
size_t isoq_block_bytes(int d, int page_size);

/* =======================================================================================
 * Quantize-append.
 *
 * For every token t < n_tokens and KV head h: x = K[t][h] (then V[t][h]), n = ||x||_2,
 * y = H x / sqrt(d) (orthonormal Walsh-Hadamard, natural order), z_b = p_b * y_b *
 * conj(q_b) with the KV head's parameters, u_i = sqrt(d) z_i / n, and
 * code_i = #{j : u_i >= t_j} over the 7 midpoint thresholds t_j = (L[j] + L[j+1]) / 2
 * (a zero vector gets code 4 everywhere).  The codes and the
 * binary16 norm are written to slot positions[t] % 64 of page
 * page_table[seq_ids[t]][positions[t] / 64].
 *
 * K, V: device [n_tokens][n_kv_heads][d] contiguous, 16-byte aligned (ISOQ_E_ARG
 * otherwise), element type `dtype` (ISOQ_F32, ISOQ_BF16 or ISOQ_F16).  seq_ids, positions: device int32 [n_tokens].
 * n_tokens == 0 is a no-op.  Arithmetic is binary32; the code decision compares
 * sqrt(d) z_i against n t_j with no division.
 * Errors: ISOQ_E_ARG (null pointers, n_tokens < 0, unknown dtype), ISOQ_E_DIM (cache d or
 * page size unsupported, or d / n_kv_heads differ from the params), ISOQ_E_CUDA (launch).
 * ===================================================================================== */
int isoq_quantize_append(const isoq_params* params, const isoq_cache* cache, const void* K,
                         const void* V, int dtype, int n_tokens, const int32_t* seq_ids,
                         const int32_t* positions, void* stream);

/* =======================================================================================
 * Fused epilogues of the K/V projection (no model weights involved).
 *
 * isoq_quantize_append_rope: as isoq_quantize_append, with the rotary position embedding
 *   applied to each K vector (given before RoPE) at its token's position, inside the same
 *   kernel and before the norm and the rotation: dims (i, i + d/2) are rotated by the
 *   angle with (cos, sin) = rope_table[position][i] (half-split pairing).  V is stored as
 *   given.  rope_table: device fp32 [rope_max_pos][d/2][2], e.g. from isoq_rope_table; a
 *   position >= rope_max_pos skips the token with ISOQ_ST_POS_RANGE.
 * isoq_rope_table: fills dst (device, isoq_rope_table_bytes(d, max_pos) bytes) with
 *   cos / sin (pos * base^(-2i/d)) for pos < max_pos, i < d/2, computed in binary64 on the
 *   device and rounded to binary32 (RoFormer frequencies).  Asynchronous on `stream`.
 *   Errors: ISOQ_E_ARG (null, max_pos < 1, base <= 1), ISOQ_E_DIM.
 * isoq_quantize_append_layers: the same tokens (seq_ids, positions, element type, count)
 *   appended to n_layers caches in one launch per 32 layers (a decode step's appends for
 *   a whole model): params[l], caches[l], K[l], V[l] are layer l's (host arrays of
 *   pointers).  All layers share d, n_kv_heads and bits (else ISOQ_E_DIM); rope_table may
 *   be NULL (no RoPE) or as for isoq_quantize_append_rope.  Per-layer errors as
 *   isoq_quantize_append.
 * ===================================================================================== */
int isoq_quantize_append_rope(const isoq_params* params, const isoq_cache* cache, const void* K,
                              const void* V, int dtype, int n_tokens, const int32_t* seq_ids,
                              const int32_t* positions, const float* rope_table,
                              int rope_max_pos, void* stream);

size_t isoq_rope_table_bytes(int d, int max_pos);

int isoq_rope_table(float* dst, int d, int max_pos, double base, void* stream);

int isoq_quantize_append_layers(const isoq_params* const* params,
                                const isoq_cache* const* caches, const void* const* K,
                                const void* const* V, int n_layers, int dtype, int n_tokens,
                                const int32_t* seq_ids, const int32_t* positions,
                                const float* rope_table, int rope_max_pos, void* stream);

/* =======================================================================================
 * Decode attention on the packed cache (one query token per sequence).
 *
 * For sequence s and query head h (KV head g = h / (n_q_heads / n_kv_heads)):
 *   q~ = R_g q            (the same WHT + SO(4) rotation as the cached vectors)
 *   s_t = scale * q~ . k~_t,   k~_t = (n_t / sqrt d) L[c_t]   for t = 0..seq_lens[s]-1
 *   o~  = sum_t softmax(s)_t v~_t                               (in the rotated space)
 *   out[s][h] = R_g^T o~                                        (inverse blocks, then WHT)
 * Full-precision K/V are never formed.  The context is split into chunks processed in
 * parallel (flash-decoding style, cf. "FreeToken releases", v0.2.0, Kernels: split
 * decode attention by context length and SM count); per-chunk partial results (running
 * max, sum, rotated accumulator) live in `workspace` and are merged, empty chunks
 * contributing nothing (the -inf start of an empty chunk is never exponentiated: cf. the
 * same release's note on a NaN from a softmax chunk that starts at -inf).
 *
 * Arithmetic (3 bits): the levels are given to four decimals, so each score is computed
 * exactly in integers -- the levels as 10000 L[c] split into two signed bytes, the rotated
 * query of a row scaled to 24 bits and split into three, products on the 8-bit tensor
 * cores with 32-bit sums -- and the only rounding before the binary32 softmax is that of
 * the query (relative ~1e-7).  The value sum uses binary16 operands (the levels times a
 * scale at which they round by < 2e-5, the weights p |v| / sigma) with binary32
 * accumulation.  Measured against a binary64 evaluation of the same codes: relative L2
 * error per (sequence, head) <= 5e-4 on the five test workloads.  2 and 4 bits: binary16
 * operands throughout, the query as a high and a low binary16 part.
 *
 * Q: device [n_seqs][n_q_heads][d], element type q_dtype.  seq_lens: device int32
 * [n_seqs], the number of cached tokens each query attends (0 gives an all-zero output;
 * beyond the page table it is clamped and ISOQ_ST_LEN_RANGE set).  max_seq_len: a host
 * upper bound of seq_lens used only to size the split; must equal the value passed to
 * isoq_decode_workspace_bytes.  out: device fp32 [n_seqs][n_q_heads][d].
 * workspace: device, at least isoq_decode_workspace_bytes(...) bytes, 16-byte aligned,
 * contents need not be initialised.  Calls that share a workspace must not overlap.
 * Errors: ISOQ_E_ARG, ISOQ_E_DIM, ISOQ_E_GQA, ISOQ_E_WORKSPACE, ISOQ_E_CUDA.
 * ===================================================================================== */
size_t isoq_decode_workspace_bytes(int n_seqs, int n_q_heads, int n_kv_heads, int d,
                                   int max_seq_len);

int isoq_decode_attention(const isoq_params* params, const isoq_cache* cache, const void* Q,
                          int q_dtype, int n_seqs, int n_q_heads, const int32_t* seq_lens,
                          int max_seq_len, float* out, float scale, void* workspace,
                          size_t workspace_bytes, void* stream);

/* =======================================================================================
 * Decode attention that allocates nothing and takes no workspace.
 *
 * The paper has no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory themselves -- for instance a plug-in that a host application
 * hands only its input and output buffers, or a thread that must not call cudaMalloc
 * because that call can synchronise the device.  It computes exactly what
 * isoq_decode_attention computes, with the same kernels and the same arguments minus
 * the workspace.  The split-K partial results go to a fixed device array inside the
 * library instead, of ISOQ_NOALLOC_SCRATCH_BYTES bytes, which every GPU that loads the
 * library keeps until the process exits.
 *
 * Limit: calls whose isoq_decode_workspace_bytes(n_seqs, n_q_heads, n_kv_heads, d,
 * max_seq_len) exceeds ISOQ_NOALLOC_SCRATCH_BYTES are rejected with ISOQ_E_WORKSPACE
 * (nothing is launched).  All calls share the one array: two calls that overlap on the
 * GPU (different streams, or threads without ordering between them) race and give wrong
 * results.  The array keeps the previous call's contents; nothing has to be cleared,
 * since each call writes every partial result it reads.  The first call on a device looks
 * up the array's device address there (cudaGetSymbolAddress), so make that first call
 * before any stream capture.  No cudaMalloc, cudaFree or allocating library routine is
 * called.
 * Errors: as isoq_decode_attention (ISOQ_E_WORKSPACE meaning "too large for the array").
 * ===================================================================================== */
#define ISOQ_NOALLOC_SCRATCH_BYTES (16u << 20) /* 16 MiB per device */

int isoq_decode_attention_noalloc(const isoq_params* params, const isoq_cache* cache,
                                  const void* Q, int q_dtype, int n_seqs, int n_q_heads,
                                  const int32_t* seq_lens, int max_seq_len, float* out,
                                  float scale, void* stream);

/* =======================================================================================
 * Multi-token attention on the packed cache (a chunk of n_q query tokens per sequence:
 * chunked prefill, speculative-decoding verification).
 *
 * The chunk's K/V must already be appended (isoq_quantize_append).  With L = seq_lens[s]
 * cached tokens, query token i (0 <= i < n_q) of sequence s sits at position L - n_q + i
 * and attends, causally, cache positions 0 .. L - n_q + i; for each (i, query head h) the
 * result is what isoq_decode_attention returns for one query attending the first
 * L - n_q + i + 1 tokens (the same rotation, codebook and merge), so the method is the
 * one of the decode above ("RotaryQuant ...", Abstract: attention on the packed codes).
 * A row whose position is negative (L < n_q - i) attends nothing and is all zeros.
 *
 * Q: device [n_seqs][n_q][n_q_heads][d], element type q_dtype.  out: device fp32
 * [n_seqs][n_q][n_q_heads][d].  workspace: device, 16-byte aligned, at least
 * isoq_multi_token_workspace_bytes(...) bytes for the same sizes.  Other arguments as
 * isoq_decode_attention; n_q = 1 is exactly the decode.  Requires
 * n_kv_heads * ceil(n_q * n_q_heads / n_kv_heads / 8) <= 65535, else ISOQ_E_ARG.
 * Errors: ISOQ_E_ARG, ISOQ_E_DIM, ISOQ_E_GQA, ISOQ_E_WORKSPACE, ISOQ_E_DEVICE, ISOQ_E_CUDA.
 * ===================================================================================== */
size_t isoq_multi_token_workspace_bytes(int n_seqs, int n_q, int n_q_heads, int n_kv_heads,
                                        int d, int max_seq_len);

int isoq_multi_token_attention(const isoq_params* params, const isoq_cache* cache,
                               const void* Q, int q_dtype, int n_seqs, int n_q, int n_q_heads,
                               const int32_t* seq_lens, int max_seq_len, float* out,
                               float scale, void* workspace, size_t workspace_bytes,
                               void* stream);

/* Number of context chunks (splits) the decode uses for these sizes on the current
 * device; >= 1, or a negative error code. */
int isoq_decode_num_splits(int n_seqs, int n_q_heads, int n_kv_heads, int d, int max_seq_len);

/* =======================================================================================
 * Context-parallel decode: one sequence's context spread over several ranks (GPUs).
 *
 * Softmax attention over a union of disjoint token sets is the log-sum-exp merge of the
 * per-set states, exactly as the split chunks above are merged (the same split-K rule,
 * "FreeToken releases", v0.2.0, Kernels), so a rank that holds a slice of every
 * sequence's context computes the state of its slice, the ranks exchange the states
 * (a few hundred bytes per (sequence, query head)), and each finishes the merge.  Which
 * tokens a rank holds is the caller's choice; positions only matter to RoPE, which is
 * part of the cached K, so each rank's cache stores its slice at local positions 0..n-1.
 *
 * State layout (fp32, per (sequence, query head), d + 4 floats): acc[d], m, l, 0, 0 with
 *   m = max over the slice of the score in natural-log units (-inf for an empty slice),
 *   l = sum_t exp(s_t - m),  acc = sqrt(d) * sum_t exp(s_t - m) v~_t  (rotated space).
 *
 * isoq_decode_partial_state: as isoq_decode_attention over this rank's cache (same
 *   arguments and errors), writing the state of each (sequence, query head) to `state`:
 *   device fp32 [n_seqs][n_q_heads][d + 4], 16-byte aligned, isoq_decode_state_bytes()
 *   bytes.
 * isoq_decode_merge_states: states = device fp32 [n_states][n_seqs][n_q_heads][d + 4]
 *   (what an all-gather of the ranks' `state` buffers produces, in any rank order),
 *   16-byte aligned; writes out = device fp32 [n_seqs][n_q_heads][d], the attention over
 *   the union of the slices (zeros where every slice is empty).  params gives d, the KV
 *   head count and the inverse rotation.  Errors: ISOQ_E_ARG, ISOQ_E_GQA, ISOQ_E_DEVICE,
 *   ISOQ_E_CUDA.
 * ===================================================================================== */
size_t isoq_decode_state_bytes(int n_seqs, int n_q_heads, int d);

int isoq_decode_partial_state(const isoq_params* params, const isoq_cache* cache, const void* Q,
                              int q_dtype, int n_seqs, int n_q_heads, const int32_t* seq_lens,
                              int max_seq_len, float* state, float scale, void* workspace,
                              size_t workspace_bytes, void* stream);

int isoq_decode_merge_states(const isoq_params* params, const float* states, int n_states,
                             int n_seqs, int n_q_heads, float* out, void* stream);

/* ---- status and errors ------------------------------------------------------------------ */
/* Synchronises the device and copies the status word to *host_bits (0 if status is NULL). */
int isoq_get_status(const isoq_cache* cache, uint32_t* host_bits);

/* Enqueues a zeroing of the status word on `stream`. */
int isoq_reset_status(const isoq_cache* cache, void* stream);

/* The cudaError_t of the last failing CUDA call in this thread (0 if none). */
int isoq_last_cuda_error(void);

/* ---- self-test of the bounded waits ------------------------------------------------------
 * Every wait in the kernels' copy and tensor-core pipelines (on an mbarrier phase) gives up
 * after a bounded number of polls, reports ISOQ_ST_TIMEOUT in the status word and lets the
 * kernel finish, so a copy that never lands cannot hang the GPU.  This call exercises that
 * path with the same wait helper: one kernel of one thread waits `polls` polls on a phase
 * that nothing completes, sets ISOQ_ST_TIMEOUT in *status (device word) when the wait gives
 * up, then waits on a phase it has completed itself.  result: device uint32[2] = (the stuck
 * wait gave up, the completed wait succeeded), 1 for yes.  Asynchronous on `stream`.
 * Errors: ISOQ_E_ARG (null pointer, polls = 0), ISOQ_E_CUDA. */
int isoq_selftest_bounded_wait(uint32_t* status, unsigned polls, uint32_t* result, void* stream);

/* Self-test of the bounds-checked build (this build step has no counterpart in the paper;
 * it stands in for a memory checker).  Every kernel of a library built with
 * -DISOQ_CHECK_BOUNDS compares each computed global, shared-memory and tensor-memory index
 * with its extent before the access; an index outside skips the access and ORs
 * ISOQ_ST_BOUNDS into the status word.  This call launches one kernel that performs such a
 * check on an index known to be outside (and accesses nothing), so a checked build sets
 * ISOQ_ST_BOUNDS in *status and a normal build leaves it clear.
 * status: device uint32.  Returns ISOQ_E_ARG for a null pointer, ISOQ_E_CUDA on a launch
 * error, else ISOQ_OK (asynchronous on stream). */
int isoq_selftest_bounds(uint32_t* status, void* stream);

/* A static string describing an ISOQ_* return code. */
const char* isoq_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* ISOQ_H */
