// C-ABI layer of libisoq: argument validation, rotation parameters, launch configuration.
// See include/isoq.h for the contract of every entry point.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "../../include/isoq.h"
#include "isoq_internal.h"

struct isoq_params {
  int d;
  int n_kv_heads;
  int bits;                 // 2, 3 or 4 bits per code
  int rotation;             // ISOQ_ROT_SO4 or ISOQ_ROT_SO2
  int device;
  float* dev;               // the parameters as generated (SO(4): [H][d/4][2][4] quaternions,
                            // the 256 parameters/head; SO(2): [H][d/2][2] cos, sin)
  float* dev_mat;           // [n_kv_heads][d/4][4][4] derived: each 4-dim block's matrix
  std::vector<float> host;  // same values as dev
};

namespace {

thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return ISOQ_E_CUDA;
}

bool supported_d(int d) { return d == 128 || d == 256; }
// 3 bits at d = 128 and 256; the 2- and 4-bit variants at d = 128.
bool supported_format(int d, int bits) { return bits == 3 || ((bits == 2 || bits == 4) && d == 128); }

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014).
uint64_t splitmix64(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

// Box-Muller (cosine branch) from two 53-bit uniforms, binary64.
double std_normal(uint64_t& state) {
  const double two_m53 = 1.0 / 9007199254740992.0;
  const uint64_t k1 = splitmix64(state) >> 11;
  const uint64_t k2 = splitmix64(state) >> 11;
  const double u1 = ((double)k1 + 1.0) * two_m53;
  const double u2 = (double)k2 * two_m53;
  const double two_pi = 2.0 * 3.14159265358979323846;
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

// Hamilton product of quaternions (w, x, y, z), binary64.
void hamilton(const double* a, const double* b, double* o) {
  o[0] = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
  o[1] = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
  o[2] = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
  o[3] = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
}

// SM count of the current device (148 on B200 when no device can be queried, which keeps
// the split arithmetic callable on a host without a GPU).
int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 148;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

struct SplitPlan {
  int n_splits;
  int pages_per_split;
};

#ifndef ISOQ_DEC_WAVES
#define ISOQ_DEC_WAVES 4
#endif
#ifndef ISOQ_DEC_MIN_PAGES  // pages per decode CTA worth a launch
#define ISOQ_DEC_MIN_PAGES 16
#endif
#ifndef ISOQ_DEC_MAX_CHUNK_PAGES  // longest decode chunk: a ragged batch sized by its
#define ISOQ_DEC_MAX_CHUNK_PAGES 64  // longest sequence still gets chunks this short
#endif
#ifndef ISOQ_MQ_WAVES  // the same for the multi-token kernels
#define ISOQ_MQ_WAVES 8
#endif

// Context chunking for the decode kernel: about ISOQ_DEC_WAVES waves of (chunk, KV head,
// query-head block, sequence) CTAs at the kernel's resident CTAs per SM, each chunk a whole
// number of pages and at least min_pages pages when the context allows.
SplitPlan plan_splits(int n_seqs, int n_q_heads, int n_kv_heads, int d, int max_seq_len,
                      int n_q = 1) {
  const int group = n_kv_heads > 0 ? n_q_heads / n_kv_heads : 1;
  // the multi-token kernels (64 or 128 rows per CTA, 2 CTAs per SM) when a chunk gives a
  // KV head at least 16 rows; else the per-row kernel (8 rows per CTA)
  const bool shared_mq = d == 128 && n_q > 1 && (long long)n_q * group >= 16;
  const int n_sm = sm_count() * (shared_mq ? 2 : isoq::decode_i8_resident_ctas(d));
  const int rows_per_cta = shared_mq ? isoq::attention_rows_per_cta(d, n_q, group)
                                     : isoq::decode_rows_per_block(d, n_q, group);
  // pages per CTA worth a launch: the tensor-memory kernel rotates 128 queries per CTA
  const int min_pages = shared_mq ? (rows_per_cta == 128 ? 16 : 4) : ISOQ_DEC_MIN_PAGES;
  const int max_pages = max_seq_len > 0 ? (max_seq_len + ISOQ_PAGE_SIZE - 1) / ISOQ_PAGE_SIZE : 1;
  const long long units =
      (long long)n_seqs * n_kv_heads * (((long long)n_q * group + rows_per_cta - 1) / rows_per_cta);
  const long long target = (long long)n_sm * (shared_mq ? ISOQ_MQ_WAVES : ISOQ_DEC_WAVES);
  long long want = units > 0 ? (target + units - 1) / units : 1;
  const long long cap = (max_pages + min_pages - 1) / min_pages;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  int pps = (int)((max_pages + want - 1) / want);
  if (!shared_mq && pps > ISOQ_DEC_MAX_CHUNK_PAGES) pps = ISOQ_DEC_MAX_CHUNK_PAGES;
  if (pps < 1) pps = 1;
  if (pps > isoq::kMaxPagesPerSplit) pps = isoq::kMaxPagesPerSplit;
  int n_splits = (max_pages + pps - 1) / pps;
  return SplitPlan{n_splits, pps};
}

int check_cache(const isoq_cache* c, const isoq_params* p) {
  if (!c || !p) return ISOQ_E_ARG;
  if (!c->blocks || !c->page_table) return ISOQ_E_ARG;
  if (c->page_size != ISOQ_PAGE_SIZE || !supported_d(c->d)) return ISOQ_E_DIM;
  if (c->d != p->d || c->n_kv_heads != p->n_kv_heads) return ISOQ_E_DIM;
  if ((c->bits == 0 ? 3 : c->bits) != p->bits) return ISOQ_E_DIM;
  if (c->n_pages < 0 || c->max_pages_per_seq < 1 || c->n_seqs < 1 || c->n_kv_heads < 1)
    return ISOQ_E_ARG;
  return ISOQ_OK;
}

int check_device(const isoq_params* p) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    g_last_cuda_error = (int)e;
    cudaGetLastError();
    return ISOQ_E_DEVICE;
  }
  return dev == p->device ? ISOQ_OK : ISOQ_E_DEVICE;
}

bool valid_dtype(int t) { return t == ISOQ_F32 || t == ISOQ_BF16 || t == ISOQ_F16; }

}  // namespace

extern "C" {

int isoq_params_generate_v(uint64_t seed, int d, int n_kv_heads, int rotation,
                           float* host_out) {
  if (rotation != ISOQ_ROT_SO2) return isoq_params_generate(seed, d, n_kv_heads, host_out);
  if (!host_out || n_kv_heads < 1) return ISOQ_E_ARG;
  if (!supported_d(d)) return ISOQ_E_DIM;
  // Haar on SO(2): phi = 2 pi u, u from the top 53 bits of one SplitMix64 draw
  const double two_m53 = 1.0 / 9007199254740992.0;
  const double two_pi = 2.0 * 3.14159265358979323846;
  uint64_t state = seed;
  for (size_t b = 0; b < (size_t)n_kv_heads * (d / 2); ++b) {
    const double phi = two_pi * (double)(splitmix64(state) >> 11) * two_m53;
    host_out[2 * b] = (float)cos(phi);
    host_out[2 * b + 1] = (float)sin(phi);
  }
  return ISOQ_OK;
}

int isoq_params_generate(uint64_t seed, int d, int n_kv_heads, float* host_out) {
  if (!host_out || n_kv_heads < 1) return ISOQ_E_ARG;
  if (!supported_d(d)) return ISOQ_E_DIM;
  uint64_t state = seed;
  const int nblk = d / 4;
  for (int h = 0; h < n_kv_heads; ++h)
    for (int b = 0; b < nblk; ++b)
      for (int which = 0; which < 2; ++which) {
        double g[4], s = 0.0;
        for (int c = 0; c < 4; ++c) {
          g[c] = std_normal(state);
          s += g[c] * g[c];
        }
        const double len = sqrt(s);
        for (int c = 0; c < 4; ++c)
          host_out[(((size_t)h * nblk + b) * 2 + which) * 4 + c] = (float)(g[c] / len);
      }
  return ISOQ_OK;
}

int isoq_make_params_v(uint64_t seed, int d, int n_kv_heads, int bits, int rotation,
                       isoq_params** out) {
  if (!out) return ISOQ_E_ARG;
  *out = nullptr;
  if (n_kv_heads < 1) return ISOQ_E_ARG;
  if (rotation != ISOQ_ROT_SO4 && rotation != ISOQ_ROT_SO2) return ISOQ_E_ARG;
  if (!supported_d(d) || !supported_format(d, bits)) return ISOQ_E_DIM;
  isoq_params* p = new isoq_params();
  p->d = d;
  p->n_kv_heads = n_kv_heads;
  p->bits = bits;
  p->rotation = rotation;
  p->dev = nullptr;
  p->dev_mat = nullptr;
  p->host.resize((size_t)n_kv_heads * (rotation == ISOQ_ROT_SO2 ? d : 2 * d));
  isoq_params_generate_v(seed, d, n_kv_heads, rotation, p->host.data());
  cudaError_t e = cudaGetDevice(&p->device);
  if (e != cudaSuccess) {
    g_last_cuda_error = (int)e;
    cudaGetLastError();
    delete p;
    return ISOQ_E_DEVICE;
  }
  // Derived copy used by every kernel: each 4-dim block's rotation as a 4x4 row-major
  // matrix, computed in binary64 from the binary32 parameters.  SO(4): column j =
  // p * e_j * conj(q).  SO(2): two 2x2 blocks [c -s; s c] on the diagonal.
  const size_t nq = p->host.size();
  std::vector<float> mats((size_t)n_kv_heads * (d / 4) * 16, 0.f);
  for (size_t blk = 0; blk < (size_t)n_kv_heads * (d / 4); ++blk) {
    float* M = mats.data() + blk * 16;
    if (rotation == ISOQ_ROT_SO2) {
      for (int half = 0; half < 2; ++half) {
        const float* cs = p->host.data() + (2 * blk + half) * 2;
        const int o = 2 * half;
        M[o * 4 + o] = cs[0];
        M[o * 4 + o + 1] = -cs[1];
        M[(o + 1) * 4 + o] = cs[1];
        M[(o + 1) * 4 + o + 1] = cs[0];
      }
      continue;
    }
    const float* pq = p->host.data() + blk * 8;
    const double P[4] = {pq[0], pq[1], pq[2], pq[3]};
    const double Qc[4] = {pq[4], -(double)pq[5], -(double)pq[6], -(double)pq[7]};
    for (int j = 0; j < 4; ++j) {
      double ev[4] = {0, 0, 0, 0}, tq[4], z[4];
      ev[j] = 1.0;
      hamilton(P, ev, tq);
      hamilton(tq, Qc, z);
      for (int i = 0; i < 4; ++i) M[i * 4 + j] = (float)z[i];
    }
  }
  const size_t bytes = (nq + mats.size()) * sizeof(float);
  e = cudaMalloc(&p->dev, bytes);
  if (e == cudaSuccess) {
    p->dev_mat = p->dev + nq;
    e = cudaMemcpy(p->dev, p->host.data(), nq * sizeof(float), cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess)
    e = cudaMemcpy(p->dev_mat, mats.data(), mats.size() * sizeof(float), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    if (p->dev) cudaFree(p->dev);
    delete p;
    return cuda_fail(e);
  }
  *out = p;
  return ISOQ_OK;
}

int isoq_make_params(uint64_t seed, int d, int n_kv_heads, isoq_params** out) {
  return isoq_make_params_v(seed, d, n_kv_heads, 3, ISOQ_ROT_SO4, out);
}

int isoq_params_format(const isoq_params* p, int* bits, int* rotation) {
  if (!p) return ISOQ_E_ARG;
  if (bits) *bits = p->bits;
  if (rotation) *rotation = p->rotation;
  return ISOQ_OK;
}

int isoq_params_copy(const isoq_params* p, float* host_dst) {
  if (!p || !host_dst) return ISOQ_E_ARG;
  memcpy(host_dst, p->host.data(), p->host.size() * sizeof(float));
  return ISOQ_OK;
}

int isoq_params_shape(const isoq_params* p, int* d, int* n_kv_heads) {
  if (!p) return ISOQ_E_ARG;
  if (d) *d = p->d;
  if (n_kv_heads) *n_kv_heads = p->n_kv_heads;
  return ISOQ_OK;
}

void isoq_params_destroy(isoq_params* p) {
  if (!p) return;
  if (p->dev) cudaFree(p->dev);
  delete p;
}

size_t isoq_block_bytes_v(int d, int bits, int page_size) {
  if (!supported_d(d) || !supported_format(d, bits) || page_size != ISOQ_PAGE_SIZE) return 0;
  return (size_t)2 * page_size * (bits * d / 8 + 2);
}

size_t isoq_block_bytes(int d, int page_size) { return isoq_block_bytes_v(d, 3, page_size); }

}  // extern "C"

namespace {

// Shared by the quantize-append entry points: every layer's params and cache are checked
// (same d, heads and bits), then the layers go out in launches of up to kMaxLayers.
int quantize_common(const isoq_params* const* params, const isoq_cache* const* caches,
                    const void* const* K, const void* const* V, int n_layers, int dtype,
                    int n_tokens, const int32_t* seq_ids, const int32_t* positions,
                    const float* rope, int rope_max_pos, void* stream) {
  if (!params || !caches || !K || !V || n_layers < 1) return ISOQ_E_ARG;
  for (int i = 0; i < n_layers; ++i) {
    const int rc = check_cache(caches[i], params[i]);
    if (rc) return rc;
    if (params[i]->d != params[0]->d || params[i]->n_kv_heads != params[0]->n_kv_heads ||
        params[i]->bits != params[0]->bits)
      return ISOQ_E_DIM;
  }
  if (n_tokens < 0 || !valid_dtype(dtype)) return ISOQ_E_ARG;
  if (rope && rope_max_pos < 1) return ISOQ_E_ARG;
  if (n_tokens == 0) return ISOQ_OK;
  if (!seq_ids || !positions) return ISOQ_E_ARG;
  for (int i = 0; i < n_layers; ++i) {
    // the kernels copy whole vectors in 16-byte pieces
    if (!K[i] || !V[i] || ((uintptr_t)K[i] & 15u) != 0 || ((uintptr_t)V[i] & 15u) != 0)
      return ISOQ_E_ARG;
    const int rc = check_device(params[i]);
    if (rc) return rc;
  }
  isoq::QuantizeArgs a{};
  a.bits = params[0]->bits;
  a.n_kv_heads = params[0]->n_kv_heads;
  a.d = params[0]->d;
  a.dtype = dtype;
  a.n_tokens = n_tokens;
  a.seq_ids = seq_ids;
  a.positions = positions;
  a.rope = rope;
  a.rope_max_pos = rope ? rope_max_pos : 0;
  for (int l0 = 0; l0 < n_layers; l0 += isoq::kMaxLayers) {
    a.layers.n = n_layers - l0 < isoq::kMaxLayers ? n_layers - l0 : isoq::kMaxLayers;
    for (int i = 0; i < a.layers.n; ++i) {
      const isoq_params* p = params[l0 + i];
      const isoq_cache* c = caches[l0 + i];
      isoq::QuantLayer& L = a.layers.l[i];
      L.mats = p->dev_mat;
      L.blocks = c->blocks;
      L.page_table = c->page_table;
      L.K = K[l0 + i];
      L.V = V[l0 + i];
      L.status = c->status;
      L.n_pages = c->n_pages;
      L.max_pages = c->max_pages_per_seq;
      L.n_seqs = c->n_seqs;
    }
    cudaError_t e = isoq::launch_quantize_append(a, (cudaStream_t)stream, sm_count());
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return ISOQ_OK;
}

// Device fp64 cos/sin table of the rotary embedding.
__global__ void rope_table_kernel(float* dst, int d, int max_pos, double base) {
  const int h = d / 2;
  const long long n = (long long)max_pos * h;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int pos = (int)(i / h), k = (int)(i % h);
    const double theta = pow(base, -2.0 * k / d);
    double sn, cs;
    sincos((double)pos * theta, &sn, &cs);
    dst[2 * i] = (float)cs;
    dst[2 * i + 1] = (float)sn;
  }
}

}  // namespace

extern "C" {

int isoq_quantize_append(const isoq_params* params, const isoq_cache* cache, const void* K,
                         const void* V, int dtype, int n_tokens, const int32_t* seq_ids,
                         const int32_t* positions, void* stream) {
  return quantize_common(&params, &cache, &K, &V, 1, dtype, n_tokens, seq_ids, positions,
                         nullptr, 0, stream);
}

int isoq_quantize_append_rope(const isoq_params* params, const isoq_cache* cache, const void* K,
                              const void* V, int dtype, int n_tokens, const int32_t* seq_ids,
                              const int32_t* positions, const float* rope_table,
                              int rope_max_pos, void* stream) {
  if (!rope_table) return ISOQ_E_ARG;
  return quantize_common(&params, &cache, &K, &V, 1, dtype, n_tokens, seq_ids, positions,
                         rope_table, rope_max_pos, stream);
}

int isoq_quantize_append_layers(const isoq_params* const* params,
                                const isoq_cache* const* caches, const void* const* K,
                                const void* const* V, int n_layers, int dtype, int n_tokens,
                                const int32_t* seq_ids, const int32_t* positions,
                                const float* rope_table, int rope_max_pos, void* stream) {
  return quantize_common(params, caches, K, V, n_layers, dtype, n_tokens, seq_ids, positions,
                         rope_table, rope_max_pos, stream);
}

size_t isoq_rope_table_bytes(int d, int max_pos) {
  if (!supported_d(d) || max_pos < 1) return 0;
  return (size_t)max_pos * d * sizeof(float);
}

int isoq_rope_table(float* dst, int d, int max_pos, double base, void* stream) {
  if (!dst || max_pos < 1 || !(base > 1.0)) return ISOQ_E_ARG;
  if (!supported_d(d)) return ISOQ_E_DIM;
  const long long n = (long long)max_pos * (d / 2);
  long long grid = (n + 255) / 256;
  if (grid > 4096) grid = 4096;
  rope_table_kernel<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(dst, d, max_pos, base);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? ISOQ_OK : cuda_fail(e);
}

int isoq_decode_num_splits(int n_seqs, int n_q_heads, int n_kv_heads, int d, int max_seq_len) {
  if (n_seqs < 0 || n_q_heads < 0 || n_kv_heads < 1 || max_seq_len < 0) return ISOQ_E_ARG;
  if (!supported_d(d)) return ISOQ_E_DIM;
  if (n_q_heads % n_kv_heads) return ISOQ_E_GQA;
  return plan_splits(n_seqs, n_q_heads, n_kv_heads, d, max_seq_len).n_splits;
}

size_t isoq_decode_workspace_bytes(int n_seqs, int n_q_heads, int n_kv_heads, int d,
                                   int max_seq_len) {
  const int ns = isoq_decode_num_splits(n_seqs, n_q_heads, n_kv_heads, d, max_seq_len);
  if (ns < 1) return 0;
  return (size_t)n_seqs * n_q_heads * ns * isoq::partial_stride(d) * sizeof(float);
}

}  // extern "C"

namespace {

// The split kernel's grid.y = n_kv_heads * ceil(n_q * group / 8) must stay <= 65535.
bool rows_fit(int n_q, int n_q_heads, int n_kv_heads) {
  const long long group = n_kv_heads > 0 ? n_q_heads / n_kv_heads : 0;
  return (long long)n_kv_heads * (((long long)n_q * group + 7) / 8) <= 65535;
}

// Shared by the decode entry points: validation, the split plan, then the split kernel and
// the combine into either the output rows (out) or merged states (state).
int decode_common_impl(const isoq_params* params, const isoq_cache* cache, const void* Q,
                  int q_dtype, int n_seqs, int n_q, int n_q_heads, const int32_t* seq_lens,
                  int max_seq_len, float* out, float* state, float scale, void* workspace,
                  size_t workspace_bytes, void* stream) {
  int rc = check_cache(cache, params);
  if (rc) return rc;
  if (n_seqs < 0 || n_q_heads < 0 || max_seq_len < 0 || !valid_dtype(q_dtype)) return ISOQ_E_ARG;
  if (!(scale == scale) || isinf(scale)) return ISOQ_E_ARG;
  if (n_q_heads % cache->n_kv_heads || n_q_heads / cache->n_kv_heads > 16) return ISOQ_E_GQA;
  if (n_seqs > cache->n_seqs) return ISOQ_E_ARG;
  if (n_q < 1 || !rows_fit(n_q, n_q_heads, cache->n_kv_heads)) return ISOQ_E_ARG;
  if (n_seqs == 0 || n_q_heads == 0) return ISOQ_OK;
  if (!Q || !seq_lens || !(out || state) || !workspace) return ISOQ_E_ARG;
  if (state && ((uintptr_t)state & 15u) != 0) return ISOQ_E_ARG;
  if (((uintptr_t)workspace & 15u) != 0) return ISOQ_E_WORKSPACE;
  const size_t need = isoq_multi_token_workspace_bytes(n_seqs, n_q, n_q_heads, cache->n_kv_heads,
                                                       cache->d, max_seq_len);
  if (workspace_bytes < need) return ISOQ_E_WORKSPACE;
  if ((rc = check_device(params))) return rc;
  const SplitPlan plan =
      plan_splits(n_seqs, n_q_heads, cache->n_kv_heads, cache->d, max_seq_len, n_q);
  isoq::DecodeArgs a{};
  a.n_q = n_q;
  a.params = params->dev_mat;
  a.bits = params->bits;
  a.blocks = cache->blocks;
  a.page_table = cache->page_table;
  a.n_pages = cache->n_pages;
  a.max_pages = cache->max_pages_per_seq;
  a.n_kv_heads = cache->n_kv_heads;
  a.d = cache->d;
  a.Q = Q;
  a.q_dtype = q_dtype;
  a.n_seqs = n_seqs;
  a.n_q_heads = n_q_heads;
  a.seq_lens = seq_lens;
  a.scale = scale;
  a.n_splits = plan.n_splits;
  a.pages_per_split = plan.pages_per_split;
  a.partials = static_cast<float*>(workspace);
  a.out = out;
  a.state = state;
  a.status = cache->status;
  cudaError_t e = isoq::launch_decode(a, (cudaStream_t)stream);
  return e == cudaSuccess ? ISOQ_OK : cuda_fail(e);
}

}  // namespace

namespace isoq {
int decode_run(const isoq_params* params, const isoq_cache* cache, const void* Q, int q_dtype,
               int n_seqs, int n_q, int n_q_heads, const int32_t* seq_lens, int max_seq_len,
               float* out, float* state, float scale, void* workspace, size_t workspace_bytes,
               void* stream) {
  return decode_common_impl(params, cache, Q, q_dtype, n_seqs, n_q, n_q_heads, seq_lens,
                            max_seq_len, out, state, scale, workspace, workspace_bytes, stream);
}
}  // namespace isoq

namespace {
inline int decode_common(const isoq_params* params, const isoq_cache* cache, const void* Q,
                         int q_dtype, int n_seqs, int n_q, int n_q_heads, const int32_t* seq_lens,
                         int max_seq_len, float* out, float* state, float scale, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return decode_common_impl(params, cache, Q, q_dtype, n_seqs, n_q, n_q_heads, seq_lens,
                            max_seq_len, out, state, scale, workspace, workspace_bytes, stream);
}
}  // namespace

extern "C" {

int isoq_decode_attention(const isoq_params* params, const isoq_cache* cache, const void* Q,
                          int q_dtype, int n_seqs, int n_q_heads, const int32_t* seq_lens,
                          int max_seq_len, float* out, float scale, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return decode_common(params, cache, Q, q_dtype, n_seqs, 1, n_q_heads, seq_lens, max_seq_len,
                       out, nullptr, scale, workspace, workspace_bytes, stream);
}

size_t isoq_multi_token_workspace_bytes(int n_seqs, int n_q, int n_q_heads, int n_kv_heads,
                                        int d, int max_seq_len) {
  if (n_seqs < 0 || n_q < 1 || n_q_heads < 0 || n_kv_heads < 1 || max_seq_len < 0) return 0;
  if (!supported_d(d) || n_q_heads % n_kv_heads) return 0;
  const int ns = plan_splits(n_seqs, n_q_heads, n_kv_heads, d, max_seq_len, n_q).n_splits;
  return (size_t)n_seqs * n_q * n_q_heads * ns * isoq::partial_stride(d) * sizeof(float);
}

int isoq_multi_token_attention(const isoq_params* params, const isoq_cache* cache,
                               const void* Q, int q_dtype, int n_seqs, int n_q, int n_q_heads,
                               const int32_t* seq_lens, int max_seq_len, float* out,
                               float scale, void* workspace, size_t workspace_bytes,
                               void* stream) {
  return decode_common(params, cache, Q, q_dtype, n_seqs, n_q, n_q_heads, seq_lens, max_seq_len,
                       out, nullptr, scale, workspace, workspace_bytes, stream);
}

size_t isoq_decode_state_bytes(int n_seqs, int n_q_heads, int d) {
  if (n_seqs < 0 || n_q_heads < 0 || !supported_d(d)) return 0;
  return (size_t)n_seqs * n_q_heads * isoq::partial_stride(d) * sizeof(float);
}

int isoq_decode_partial_state(const isoq_params* params, const isoq_cache* cache, const void* Q,
                              int q_dtype, int n_seqs, int n_q_heads, const int32_t* seq_lens,
                              int max_seq_len, float* state, float scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  if (!state) return ISOQ_E_ARG;
  return decode_common(params, cache, Q, q_dtype, n_seqs, 1, n_q_heads, seq_lens, max_seq_len,
                       nullptr, state, scale, workspace, workspace_bytes, stream);
}

int isoq_decode_merge_states(const isoq_params* params, const float* states, int n_states,
                             int n_seqs, int n_q_heads, float* out, void* stream) {
  if (!params || n_states < 1 || n_seqs < 0 || n_q_heads < 0) return ISOQ_E_ARG;
  if (n_q_heads % params->n_kv_heads || n_q_heads / params->n_kv_heads > 16) return ISOQ_E_GQA;
  if (n_seqs == 0 || n_q_heads == 0) return ISOQ_OK;
  if (!states || !out || ((uintptr_t)states & 15u) != 0) return ISOQ_E_ARG;
  int rc = check_device(params);
  if (rc) return rc;
  cudaError_t e = isoq::launch_merge_states(params->dev_mat, params->n_kv_heads, params->d, n_seqs,
                                            n_q_heads, n_states, states, out,
                                            (cudaStream_t)stream);
  return e == cudaSuccess ? ISOQ_OK : cuda_fail(e);
}

int isoq_get_status(const isoq_cache* cache, uint32_t* host_bits) {
  if (!cache || !host_bits) return ISOQ_E_ARG;
  *host_bits = 0;
  if (!cache->status) return ISOQ_OK;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(host_bits, cache->status, 4, cudaMemcpyDeviceToHost);
  return e == cudaSuccess ? ISOQ_OK : cuda_fail(e);
}

int isoq_reset_status(const isoq_cache* cache, void* stream) {
  if (!cache) return ISOQ_E_ARG;
  if (!cache->status) return ISOQ_OK;
  cudaError_t e = cudaMemsetAsync(cache->status, 0, 4, (cudaStream_t)stream);
  return e == cudaSuccess ? ISOQ_OK : cuda_fail(e);
}

int isoq_last_cuda_error(void) { return g_last_cuda_error; }

const char* isoq_error_string(int code) {
  switch (code) {
    case ISOQ_OK: return "ok";
    case ISOQ_E_ARG: return "invalid argument";
    case ISOQ_E_DIM: return "unsupported head dimension or page size";
    case ISOQ_E_GQA: return "n_q_heads is not a multiple (<= 16x) of n_kv_heads";
    case ISOQ_E_WORKSPACE: return "workspace too small or misaligned";
    case ISOQ_E_CUDA: return "CUDA runtime error";
    case ISOQ_E_DEVICE: return "no CUDA device or parameters on another device";
  }
  return "unknown";
}

}  // extern "C"

// Internal accessors for other translation units of the library (not part of the C ABI).
namespace isoq {
const float* params_device_mats(const isoq_params* p) { return p ? p->dev_mat : nullptr; }
int params_bits(const isoq_params* p) { return p ? p->bits : 3; }
int params_device(const isoq_params* p) { return p ? p->device : -1; }
}  // namespace isoq
namespace isoq {
int record_cuda_error(cudaError_t e) { return cuda_fail(e); }
}  // namespace isoq
