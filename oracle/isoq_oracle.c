/*
 * IsoQuant fp64 CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the package smoke check and the benchmark's CPU-baseline /
 * reference arm may load this library.  The product path (the CUDA library and its
 * Python binding) never calls it, and the two share no code, header, table or helper.
 *
 * What it computes follows the method page
 *   "RotaryQuant: Fitting 120B MoE Models on Consumer Hardware via Fused
 *    Compressed-Space Attention" (arXiv 2608.08081v1), Abstract:
 * each per-token, per-head K/V vector is (1) normalised by a Walsh-Hadamard transform,
 * (2) rotated by block-diagonal SO(4) rotations, (3) scalar-quantised to 3 bits; and
 * attention runs directly on the packed 3-bit tensors, never materialising full
 * precision K/V.  Page 1 ("FreeToken issue #141, unified KV cache backend", Proposed
 * Solution, Quantization layer) says the rotations are quaternion rotations.
 *
 * The pages leave these steps open; this oracle takes the plainest reading of each:
 *   - rotation parameters: one unit-quaternion pair (p, q) per 4-element block,
 *     z = p * y * conj(q) (Hamilton product, components ordered w, x, y, z), drawn
 *     Haar-uniformly from a SplitMix64 stream via Box-Muller; one set per KV head,
 *     shared by K and V (the only reading that keeps 256 parameters per head at d=128);
 *   - WHT: Sylvester (natural) order, scaled by 1/sqrt(d), no random sign diagonal;
 *   - codebook: the 8-level Lloyd-Max quantiser for N(0,1) (J. Max, "Quantizing for
 *     minimum distortion", IRE Trans. Inf. Theory IT-6, 1960) applied to
 *     u = sqrt(d) * z / ||x||; thresholds are midpoints of adjacent levels; a value
 *     exactly on a threshold takes the upper code; a zero vector has u = 0 (code 4);
 *   - norm: the L2 norm of the input vector, stored as IEEE binary16 (round to
 *     nearest even), saturating at 65504;
 *   - dequantised coordinate: (stored fp16 norm / sqrt(d)) * level, no renormalisation;
 *   - decode: softmax(scale * q.k) over positions 0..len-1 of each sequence, query head
 *     h reading KV head h / G.
 *
 * Format variants (functions with a _v suffix take bits and rot; the plain names are the
 * method's 3 bits and SO(4)): 2- and 4-bit Lloyd-Max codebooks of the same family (Max
 * 1960, N = 4 and 16), and the PlanarQuant variant the same abstract names, read as the
 * WHT followed by 2x2 (SO(2)) rotation blocks with Haar-uniform angles.
 *
 * Everything is plain fp64 scalar code in the order the method states it.  The only
 * parallelism is an OpenMP loop over independent vectors / (sequence, head) pairs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------------ */
/* Codebooks: Lloyd-Max quantisers for N(0,1) (Max, 1960, Table I), ascending:      */
/* 8 levels for the method's 3 bits; 4 and 16 levels for the 2- and 4-bit variants  */
/* of the same family.                                                               */
/* ------------------------------------------------------------------------------ */
static const double REF_LEVELS[8] = {-2.1520, -1.3440, -0.7560, -0.2451,
                                     0.2451,  0.7560,  1.3440,  2.1520};
static const double REF_LEVELS2[4] = {-1.5104, -0.4528, 0.4528, 1.5104};
static const double REF_LEVELS4[16] = {-2.7326, -2.0690, -1.6180, -1.2562, -0.9424, -0.6568,
                                       -0.3881, -0.1284, 0.1284,  0.3881,  0.6568,  0.9424,
                                       1.2562,  1.6180,  2.0690,  2.7326};

static const double *levels_of(int bits) {
  return bits == 2 ? REF_LEVELS2 : (bits == 4 ? REF_LEVELS4 : REF_LEVELS);
}

double ref_level_v(int bits, int code) { return levels_of(bits)[code]; }

/* Threshold j (0 .. 2^bits - 2) is the midpoint between levels j and j+1. */
double ref_threshold_v(int bits, int j) {
  const double *L = levels_of(bits);
  return 0.5 * (L[j] + L[j + 1]);
}

double ref_level(int code) { return REF_LEVELS[code]; }
double ref_threshold(int j) { return ref_threshold_v(3, j); }

int ref_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Thread count of the parallel loops that follow (timing only: every loop's iterations
 * are independent, so the results do not depend on it). */
void ref_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ------------------------------------------------------------------------------ */
/* Random rotation parameters.                                                      */
/* SplitMix64: G. Steele, D. Lea, C. Flood, "Fast splittable pseudorandom number   */
/* generators", OOPSLA 2014.  Box-Muller: G. Box, M. Muller, Ann. Math. Stat. 1958.  */
/* ------------------------------------------------------------------------------ */
uint64_t ref_splitmix64_next(uint64_t *state) {
  *state += 0x9E3779B97F4A7C15ULL;
  uint64_t z = *state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* One standard normal from two successive 64-bit draws: the top 53 bits of each give
 * u1 in (0, 1] and u2 in [0, 1); the cosine branch of Box-Muller is used. */
double ref_normal(uint64_t *state) {
  const double two_m53 = 1.0 / 9007199254740992.0; /* 2^-53 */
  uint64_t k1 = ref_splitmix64_next(state) >> 11;
  uint64_t k2 = ref_splitmix64_next(state) >> 11;
  double u1 = ((double)k1 + 1.0) * two_m53;
  double u2 = (double)k2 * two_m53;
  return sqrt(-2.0 * log(u1)) * cos(2.0 * M_PI * u2);
}

/* params: [n_kv_heads][d/4][2][4] = per block the unit quaternion p then q, each
 * (w, x, y, z).  Each quaternion is four normals divided by their Euclidean length,
 * which is uniform on the unit 3-sphere, so (p, q) -> (x -> p x conj(q)) is Haar on
 * SO(4).  params32 (optional) receives the same values rounded to binary32. */
void ref_make_params(uint64_t seed, int d, int n_kv_heads, double *params, float *params32) {
  uint64_t state = seed;
  int nblk = d / 4;
  for (int h = 0; h < n_kv_heads; h++)
    for (int b = 0; b < nblk; b++)
      for (int which = 0; which < 2; which++) {
        double g[4], s = 0.0;
        for (int c = 0; c < 4; c++) {
          g[c] = ref_normal(&state);
          s += g[c] * g[c];
        }
        double len = sqrt(s);
        for (int c = 0; c < 4; c++) {
          size_t idx = (((size_t)h * nblk + b) * 2 + which) * 4 + c;
          params[idx] = g[c] / len;
          if (params32) params32[idx] = (float)(g[c] / len);
        }
      }
}

/* PlanarQuant variant (a rotation by 2x2 blocks, SO(2)): params [n_kv_heads][d/2][2] =
 * per block (cos phi, sin phi) with phi = 2 pi u, u uniform in [0, 1) from the top 53 bits
 * of a SplitMix64 draw -- Haar on SO(2).  params32 (optional) receives binary32 copies. */
void ref_make_params_so2(uint64_t seed, int d, int n_kv_heads, double *params,
                         float *params32) {
  const double two_m53 = 1.0 / 9007199254740992.0;
  uint64_t state = seed;
  for (int h = 0; h < n_kv_heads; h++)
    for (int b = 0; b < d / 2; b++) {
      double u = (double)(ref_splitmix64_next(&state) >> 11) * two_m53;
      double phi = 2.0 * M_PI * u;
      size_t idx = ((size_t)h * (d / 2) + b) * 2;
      params[idx] = cos(phi);
      params[idx + 1] = sin(phi);
      if (params32) {
        params32[idx] = (float)cos(phi);
        params32[idx + 1] = (float)sin(phi);
      }
    }
}

/* Floats of rotation parameters per KV head: 2d for SO(4) quaternion pairs, d for SO(2). */
int ref_params_per_head(int rot, int d) { return rot == 1 ? d : 2 * d; }

/* ------------------------------------------------------------------------------ */
/* Walsh-Hadamard transform, natural (Sylvester) order, orthonormal (1/sqrt(d)).    */
/* The O(d log d) butterfly: at stride h, pairs (j, j+h) become (a+b, a-b).         */
/* ------------------------------------------------------------------------------ */
void ref_wht(double *x, int d) {
  for (int h = 1; h < d; h *= 2)
    for (int i = 0; i < d; i += 2 * h)
      for (int j = i; j < i + h; j++) {
        double a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
  double s = 1.0 / sqrt((double)d);
  for (int i = 0; i < d; i++) x[i] *= s;
}

/* ------------------------------------------------------------------------------ */
/* Quaternions (w, x, y, z), Hamilton convention i^2 = j^2 = k^2 = ijk = -1.        */
/* ------------------------------------------------------------------------------ */
void ref_quat_mul(const double *a, const double *b, double *out) {
  double w = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
  double x = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
  double y = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
  double z = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
  out[0] = w;
  out[1] = x;
  out[2] = y;
  out[3] = z;
}

static void quat_conj(const double *a, double *out) {
  out[0] = a[0];
  out[1] = -a[1];
  out[2] = -a[2];
  out[3] = -a[3];
}

/* z = p * y * conj(q): the SO(4) rotation of one 4-element block. */
void ref_so4_forward(const double *p, const double *q, const double *y, double *z) {
  double qc[4], t[4];
  quat_conj(q, qc);
  ref_quat_mul(p, y, t);
  ref_quat_mul(t, qc, z);
}

/* y = conj(p) * z * q: the inverse (transpose) of ref_so4_forward. */
void ref_so4_inverse(const double *p, const double *q, const double *z, double *y) {
  double pc[4], t[4];
  quat_conj(p, pc);
  ref_quat_mul(pc, z, t);
  ref_quat_mul(t, q, y);
}

/* 2x2 block (dims 2b, 2b+1): z = [c -s; s c] y, and its inverse (transpose). */
void ref_so2_forward(const double *cs, const double *y, double *z) {
  z[0] = cs[0] * y[0] - cs[1] * y[1];
  z[1] = cs[1] * y[0] + cs[0] * y[1];
}

void ref_so2_inverse(const double *cs, const double *z, double *y) {
  y[0] = cs[0] * z[0] + cs[1] * z[1];
  y[1] = -cs[1] * z[0] + cs[0] * z[1];
}

/* Forward rotation of one d-vector with one head's params: WHT, then the blocks
 * (rot 0: d/4 SO(4) quaternion blocks; rot 1: d/2 SO(2) blocks). */
void ref_rotate_v(int rot, const double *params_head, const double *x, double *z, int d) {
  double *y = (double *)malloc(sizeof(double) * d);
  memcpy(y, x, sizeof(double) * d);
  ref_wht(y, d);
  if (rot == 1) {
    for (int b = 0; b < d / 2; b++) ref_so2_forward(params_head + 2 * b, y + 2 * b, z + 2 * b);
  } else {
    for (int b = 0; b < d / 4; b++)
      ref_so4_forward(params_head + b * 8, params_head + b * 8 + 4, y + 4 * b, z + 4 * b);
  }
  free(y);
}

/* Inverse rotation: inverse blocks, then the WHT (orthonormal and symmetric, so it is
 * its own inverse). */
void ref_unrotate_v(int rot, const double *params_head, const double *z, double *x, int d) {
  if (rot == 1) {
    for (int b = 0; b < d / 2; b++) ref_so2_inverse(params_head + 2 * b, z + 2 * b, x + 2 * b);
  } else {
    for (int b = 0; b < d / 4; b++)
      ref_so4_inverse(params_head + b * 8, params_head + b * 8 + 4, z + 4 * b, x + 4 * b);
  }
  ref_wht(x, d);
}

void ref_rotate(const double *params_head, const double *x, double *z, int d) {
  ref_rotate_v(0, params_head, x, z, d);
}

void ref_unrotate(const double *params_head, const double *z, double *x, int d) {
  ref_unrotate_v(0, params_head, z, x, d);
}

/* ------------------------------------------------------------------------------ */
/* Rotary position embedding of a key before quantisation (the fused RoPE epilogue): */
/* half-split pairing, dims (i, i + d/2) rotated by pos * theta_i,                   */
/* theta_i = base^(-2i/d) (RoFormer's frequencies; NeoX pairing).                    */
/* ------------------------------------------------------------------------------ */
void ref_rope(const double *x, int d, int pos, double base, double *out) {
  int h = d / 2;
  for (int i = 0; i < h; i++) {
    double theta = pow(base, -2.0 * i / d);
    double c = cos(pos * theta), s = sin(pos * theta);
    double a = x[i], b = x[i + h];
    out[i] = a * c - b * s;
    out[i + h] = a * s + b * c;
  }
}

/* ------------------------------------------------------------------------------ */
/* IEEE 754 binary16, round to nearest, ties to even (from the format definition).   */
/* ------------------------------------------------------------------------------ */
uint16_t ref_fp16_bits(double v) {
  uint16_t sign = signbit(v) ? 0x8000 : 0;
  double a = fabs(v);
  if (isnan(v)) return 0x7e00;
  if (a >= 65520.0) return sign | 0x7c00; /* rounds past the largest finite, 65504 */
  int e;
  frexp(a, &e); /* a = f * 2^e, f in [0.5, 1): the leading bit has weight 2^(e-1) */
  if (a == 0.0 || e - 1 < -14) {
    /* subnormal range: quantum 2^-24; nearbyint rounds ties to even */
    double m = nearbyint(ldexp(a, 24));
    return sign | (uint16_t)m; /* m == 1024 is the smallest normal, same bits */
  }
  double m = nearbyint(ldexp(a, 10 - (e - 1))); /* in [1024, 2048] */
  int ex = e - 1;
  if (m == 2048.0) {
    m = 1024.0;
    ex += 1;
  }
  if (ex > 15) return sign | 0x7c00;
  return sign | (uint16_t)((ex + 15) << 10) | (uint16_t)((int)m - 1024);
}

double ref_fp16_value(uint16_t h) {
  int ex = (h >> 10) & 31, man = h & 1023;
  double s = (h & 0x8000) ? -1.0 : 1.0;
  if (ex == 0) return s * ldexp((double)man, -24);
  if (ex == 31) return man ? NAN : s * INFINITY;
  return s * ldexp(1024.0 + man, ex - 25);
}

/* ------------------------------------------------------------------------------ */
/* Quantise one vector: norm, WHT, rotation blocks, scalar quantisation.            */
/* ------------------------------------------------------------------------------ */
/* codes[i] in 0 .. 2^bits - 1 (ascending level index); *norm16 = binary16 bits of the
 * norm.  Returns 1 if the norm overflowed binary16 (stored as 65504), else 0.
 * z_out (optional) receives the rotated coordinates z. */
int ref_quantize_vector_v(int bits, int rot, const double *params_head, const double *x, int d,
                          uint8_t *codes, uint16_t *norm16, double *z_out) {
  double ss = 0.0;
  for (int i = 0; i < d; i++) ss += x[i] * x[i];
  double n = sqrt(ss);

  double *z = (double *)malloc(sizeof(double) * d);
  ref_rotate_v(rot, params_head, x, z, d);

  /* code_i = #{j : u_i >= t_j} with u_i = sqrt(d) z_i / n, compared as
   * sqrt(d) z_i >= n t_j.  A zero vector has no direction: u is taken as 0, which the
   * tie rule sends to the level just above 0 (code 2^(bits-1)). */
  double sqd = sqrt((double)d);
  int nl = 1 << bits;
  for (int i = 0; i < d; i++) {
    int c = 0;
    if (n == 0.0) {
      c = nl / 2;
    } else {
      for (int j = 0; j < nl - 1; j++)
        if (sqd * z[i] >= n * ref_threshold_v(bits, j)) c++;
    }
    codes[i] = (uint8_t)c;
  }
  if (z_out) memcpy(z_out, z, sizeof(double) * d);
  free(z);

  uint16_t h = ref_fp16_bits(n);
  int overflow = 0;
  if (h == 0x7c00) {
    h = 0x7bff;
    overflow = 1;
  }
  *norm16 = h;
  return overflow;
}

int ref_quantize_vector(const double *params_head, const double *x, int d, uint8_t *codes,
                        uint16_t *norm16, double *z_out) {
  return ref_quantize_vector_v(3, 0, params_head, x, d, codes, norm16, z_out);
}

/* ------------------------------------------------------------------------------ */
/* Packed code layouts (bits * d / 8 bytes per vector, little-endian 32-bit words).  */
/* 3 bits: d/32 groups of three words w0..w2; group g covers dims 32g..32g+31:       */
/*   dim 32g + 8j + k  (j = 0,1,2; k = 0..7): the code is bits 4k..4k+2 of w_j;       */
/*   dim 32g + 24 + k  (k = 0..7): code bit (2 - b) is bit 4k+3 of w_b.              */
/* 4 bits: word j holds dims 8j..8j+7, nibble k = dim 8j+k in sign-magnitude form:   */
/*   code c >= 8 -> c - 8;  c < 8 -> 8 | (7 - c)  (bit 3 = negative level, bits 0-2 =  */
/*   index of the level's magnitude, ascending).                                     */
/* 2 bits: word j holds dims 16j..16j+15; 2-bit slot s (bits 2s, 2s+1) holds dim     */
/*   16j + 2s (s < 4), 16j + 2(s-4) + 1 (4 <= s < 8), 16j + 8 + 2(s-8) (8 <= s < 12), */
/*   16j + 9 + 2(s-12) (s >= 12); the code is the level index 0..3.                 */
/* ------------------------------------------------------------------------------ */
static int slot2_dim(int s) {
  return s < 4 ? 2 * s : (s < 8 ? 2 * (s - 4) + 1 : (s < 12 ? 8 + 2 * (s - 8) : 9 + 2 * (s - 12)));
}

static void put_words(const uint32_t *w, int n, uint8_t *out) {
  for (int j = 0; j < n; j++)
    for (int byte = 0; byte < 4; byte++) out[4 * j + byte] = (uint8_t)(w[j] >> (8 * byte));
}

static uint32_t get_word(const uint8_t *in, int j) {
  uint32_t w = 0;
  for (int byte = 0; byte < 4; byte++) w |= (uint32_t)in[4 * j + byte] << (8 * byte);
  return w;
}

void ref_pack_codes_v(int bits, const uint8_t *codes, int d, uint8_t *out) {
  if (bits == 4) {
    for (int j = 0; j < d / 8; j++) {
      uint32_t w = 0;
      for (int k = 0; k < 8; k++) {
        uint32_t c = codes[8 * j + k] & 15u;
        uint32_t nib = c >= 8 ? c - 8 : (8u | (7u - c));
        w |= nib << (4 * k);
      }
      put_words(&w, 1, out + 4 * j);
    }
    return;
  }
  if (bits == 2) {
    for (int j = 0; j < d / 16; j++) {
      uint32_t w = 0;
      for (int sl = 0; sl < 16; sl++) w |= (uint32_t)(codes[16 * j + slot2_dim(sl)] & 3u) << (2 * sl);
      put_words(&w, 1, out + 4 * j);
    }
    return;
  }
  for (int g = 0; g < d / 32; g++) {
    uint32_t w[3] = {0, 0, 0};
    for (int e = 0; e < 32; e++) {
      uint32_t c = codes[32 * g + e] & 7u;
      if (e < 24) {
        int j = e / 8, k = e % 8;
        w[j] |= c << (4 * k);
      } else {
        int k = e - 24;
        for (int b = 0; b < 3; b++) w[b] |= ((c >> (2 - b)) & 1u) << (4 * k + 3);
      }
    }
    put_words(w, 3, out + 12 * g);
  }
}

void ref_unpack_codes_v(int bits, const uint8_t *in, int d, uint8_t *codes) {
  if (bits == 4) {
    for (int j = 0; j < d / 8; j++) {
      uint32_t w = get_word(in, j);
      for (int k = 0; k < 8; k++) {
        uint32_t nib = (w >> (4 * k)) & 15u;
        codes[8 * j + k] = (uint8_t)((nib & 8u) ? 7u - (nib & 7u) : 8u + nib);
      }
    }
    return;
  }
  if (bits == 2) {
    for (int j = 0; j < d / 16; j++) {
      uint32_t w = get_word(in, j);
      for (int sl = 0; sl < 16; sl++) codes[16 * j + slot2_dim(sl)] = (uint8_t)((w >> (2 * sl)) & 3u);
    }
    return;
  }
  for (int g = 0; g < d / 32; g++) {
    uint32_t w[3];
    for (int j = 0; j < 3; j++) w[j] = get_word(in + 12 * g, j);
    for (int e = 0; e < 32; e++) {
      uint32_t c = 0;
      if (e < 24) {
        c = (w[e / 8] >> (4 * (e % 8))) & 7u;
      } else {
        int k = e - 24;
        for (int b = 0; b < 3; b++) c |= ((w[b] >> (4 * k + 3)) & 1u) << (2 - b);
      }
      codes[32 * g + e] = (uint8_t)c;
    }
  }
}

void ref_pack_codes(const uint8_t *codes, int d, uint8_t *out) { ref_pack_codes_v(3, codes, d, out); }
void ref_unpack_codes(const uint8_t *in, int d, uint8_t *codes) { ref_unpack_codes_v(3, in, d, codes); }

/* ------------------------------------------------------------------------------ */
/* Paged cache: blocks[page][kv_head] of block_bytes; a block holds, for 64 (page)  */
/* token slots: K codes [P][cb] | K norms [P] binary16 | V codes | V norms, with     */
/* cb = bits * d / 8 code bytes per vector.  K codes are one record per slot (the    */
/* packing above).  V codes: one record per slot at 2 and 4 bits; at 3 bits the V    */
/* tile layout below.                                                                */
/* ------------------------------------------------------------------------------ */
static size_t cbytes(int bits, int d) { return (size_t)bits * d / 8; }

size_t ref_block_bytes_v(int bits, int d, int page) { return (size_t)2 * page * (cbytes(bits, d) + 2); }
size_t ref_block_bytes(int d, int page) { return ref_block_bytes_v(3, d, page); }

static size_t k_codes_off(size_t cb, int page, int slot) { (void)page; return (size_t)slot * cb; }
static size_t k_norm_off(size_t cb, int page, int slot) { return (size_t)page * cb + 2 * (size_t)slot; }
static size_t v_region_off(size_t cb, int page) { return (size_t)page * (cb + 2); }
static size_t v_norm_off(size_t cb, int page, int slot) {
  return (size_t)page * (cb + 2) + (size_t)page * cb + 2 * (size_t)slot;
}

/* ------------------------------------------------------------------------------ */
/* 3-bit V tile layout (this build's format; the pages fix none).  The V region of  */
/* a page is 4 blocks of 16 token slots, 6 d bytes each.  Inside block B the 16     */
/* slots form 4 quads: quad t (0..3) = slots 16B + 2t + {0, 1, 8, 9}, its member j   */
/* (0..3) being slot 16B + 2t + (j & 1) + 8 (j >> 1).  Dims form units of 8          */
/* (unit u = dims 8u .. 8u+7).  The 12-byte group of (quad t, unit u) sits at byte   */
/* ((u >> 1) * 8 + 2 t + (u & 1)) * 12 of the block and holds three little-endian   */
/* words W0, W1, W2:                                                                 */
/*   bits 4n .. 4n+2 of W_b hold the code of member (n & 3), dim 8u + 2b + (n >> 2)   */
/*   (nibbles 0-3: dim 8u+2b of the four members; nibbles 4-7: dim 8u+2b+1);        */
/*   bit 4n + 3 of W_b holds bit (2 - b) of the code of member (n & 3),               */
/*   dim 8u + 6 + (n >> 2).                                                          */
/* So each 16-bit half of a word is four members' codes of one dim: a decoder can    */
/* turn it into the values of four tokens of one dimension with byte permutes.       */
/* ------------------------------------------------------------------------------ */
static void v3_locate(int d, int slot, int dim, size_t *group, int *nib, int *spare) {
  int B = slot >> 4, r = slot & 15;
  int t = (r >> 1) & 3, j = (r & 1) | ((r >> 3) << 1);
  int u = dim >> 3, e = dim & 7;
  *group = (size_t)B * 6 * d + (size_t)(((u >> 1) * 8 + 2 * t + (u & 1)) * 12);
  *spare = e >= 6;
  *nib = *spare ? j + 4 * (e - 6) : j + 4 * (e & 1);
  if (!*spare) *group += 4 * (size_t)(e >> 1); /* word b = e / 2 */
}

static void put_bit(uint8_t *base, size_t byte, int bit, int v) {
  if (v) base[byte] |= (uint8_t)(1u << bit);
  else base[byte] &= (uint8_t)~(1u << bit);
}

static int get_bit(const uint8_t *base, size_t byte, int bit) { return (base[byte] >> bit) & 1; }

/* The codes of one slot into / out of a V region (3 bits: the tile layout; 2 and 4 bits:
 * the slot's record). */
void ref_v_put_codes(int bits, int d, int page, uint8_t *region, int slot, const uint8_t *codes) {
  if (bits != 3) {
    ref_pack_codes_v(bits, codes, d, region + (size_t)slot * cbytes(bits, d));
    return;
  }
  (void)page;
  for (int i = 0; i < d; i++) {
    size_t g;
    int n, sp;
    v3_locate(d, slot, i, &g, &n, &sp);
    unsigned c = codes[i] & 7u;
    if (!sp) {
      for (int k = 0; k < 3; k++) {
        size_t bit = 4 * (size_t)n + k;
        put_bit(region, g + bit / 8, (int)(bit % 8), (c >> k) & 1);
      }
    } else {
      for (int b = 0; b < 3; b++) {
        size_t bit = 4 * (size_t)n + 3;
        put_bit(region, g + 4 * (size_t)b + bit / 8, (int)(bit % 8), (c >> (2 - b)) & 1);
      }
    }
  }
}

void ref_v_get_codes(int bits, int d, int page, const uint8_t *region, int slot, uint8_t *codes) {
  if (bits != 3) {
    ref_unpack_codes_v(bits, region + (size_t)slot * cbytes(bits, d), d, codes);
    return;
  }
  (void)page;
  for (int i = 0; i < d; i++) {
    size_t g;
    int n, sp;
    v3_locate(d, slot, i, &g, &n, &sp);
    unsigned c = 0;
    if (!sp) {
      for (int k = 0; k < 3; k++) {
        size_t bit = 4 * (size_t)n + k;
        c |= (unsigned)get_bit(region, g + bit / 8, (int)(bit % 8)) << k;
      }
    } else {
      for (int b = 0; b < 3; b++) {
        size_t bit = 4 * (size_t)n + 3;
        c |= (unsigned)get_bit(region, g + 4 * (size_t)b + bit / 8, (int)(bit % 8)) << (2 - b);
      }
    }
    codes[i] = (uint8_t)c;
  }
}

/* A page's V region as per-slot records in the K record packing (tests compare GPU and
 * oracle codes record by record): records [page][cb]. */
void ref_v_region_records(int bits, int d, int page, const uint8_t *region, uint8_t *records) {
  uint8_t codes[1024];
  for (int s = 0; s < page; s++) {
    ref_v_get_codes(bits, d, page, region, s, codes);
    ref_pack_codes_v(bits, codes, d, records + (size_t)s * cbytes(bits, d));
  }
}

/* Quantise n_tokens tokens of K and V ([n_tokens][n_kv_heads][d], fp64) into the paged
 * cache at (seq_ids[t], positions[t]).  params: fp64, ref_params_per_head(rot, d) per
 * head.  Returns the number of norms that saturated. */
int ref_quantize_append_v(int bits, int rot, const double *params, int d, int n_kv_heads,
                          int page, uint8_t *blocks, const int32_t *page_table,
                          int max_pages_per_seq, const double *K, const double *V, int n_tokens,
                          const int32_t *seq_ids, const int32_t *positions) {
  size_t bb = ref_block_bytes_v(bits, d, page), cb = cbytes(bits, d);
  int pph = ref_params_per_head(rot, d);
  int overflow = 0;
#pragma omp parallel for schedule(static) reduction(+ : overflow)
  for (int t = 0; t < n_tokens; t++) {
    uint8_t codes[1024];
    for (int h = 0; h < n_kv_heads; h++) {
      int pos = positions[t];
      int phys = page_table[(size_t)seq_ids[t] * max_pages_per_seq + pos / page];
      int slot = pos % page;
      uint8_t *blk = blocks + ((size_t)phys * n_kv_heads + h) * bb;
      const double *ph = params + (size_t)h * pph;
      for (int kv = 0; kv < 2; kv++) {
        const double *x = (kv == 0 ? K : V) + ((size_t)t * n_kv_heads + h) * d;
        uint16_t n16;
        overflow += ref_quantize_vector_v(bits, rot, ph, x, d, codes, &n16, NULL);
        if (kv == 0)
          ref_pack_codes_v(bits, codes, d, blk + k_codes_off(cb, page, slot));
        else
          ref_v_put_codes(bits, d, page, blk + v_region_off(cb, page), slot, codes);
        uint8_t *nd = blk + (kv == 0 ? k_norm_off(cb, page, slot) : v_norm_off(cb, page, slot));
        nd[0] = (uint8_t)(n16 & 0xff);
        nd[1] = (uint8_t)(n16 >> 8);
      }
    }
  }
  return overflow;
}

int ref_quantize_append(const double *params, int d, int n_kv_heads, int page,
                        uint8_t *blocks, const int32_t *page_table, int max_pages_per_seq,
                        const double *K, const double *V, int n_tokens,
                        const int32_t *seq_ids, const int32_t *positions) {
  return ref_quantize_append_v(3, 0, params, d, n_kv_heads, page, blocks, page_table,
                               max_pages_per_seq, K, V, n_tokens, seq_ids, positions);
}

/* Dequantised vector in the rotated space: (stored norm / sqrt(d)) * level[code]. */
static void dequant_codes(int bits, const uint8_t *codes, const uint8_t *norm_bytes, int d,
                          double *out) {
  uint16_t n16 = (uint16_t)(norm_bytes[0] | (norm_bytes[1] << 8));
  double s = ref_fp16_value(n16) / sqrt((double)d);
  const double *L = levels_of(bits);
  for (int i = 0; i < d; i++) out[i] = s * L[codes[i]];
}

/* Slot `slot` of a block: K (kind 0) or V (kind 1) dequantised in the rotated space. */
static void dequant_slot(int bits, int d, int page, const uint8_t *blk, int slot, int kind,
                         double *out) {
  size_t cb = cbytes(bits, d);
  uint8_t codes[1024];
  if (kind == 0) {
    ref_unpack_codes_v(bits, blk + k_codes_off(cb, page, slot), d, codes);
    dequant_codes(bits, codes, blk + k_norm_off(cb, page, slot), d, out);
  } else {
    ref_v_get_codes(bits, d, page, blk + v_region_off(cb, page), slot, codes);
    dequant_codes(bits, codes, blk + v_norm_off(cb, page, slot), d, out);
  }
}

/* Materialise one cached vector back in the input space (K-hat or V-hat): inverse
 * rotation of the dequantised rotated vector.  kind 0 = K, 1 = V.  Used by tests to
 * check that attention in the rotated space equals attention over K-hat, V-hat. */
void ref_dequantize_slot_v(int bits, int rot, const double *params, int d, int n_kv_heads,
                           int page, const uint8_t *blocks, int phys_page, int kv_head, int slot,
                           int kind, double *out) {
  size_t bb = ref_block_bytes_v(bits, d, page);
  const uint8_t *blk = blocks + ((size_t)phys_page * n_kv_heads + kv_head) * bb;
  double zr[1024];
  dequant_slot(bits, d, page, blk, slot, kind, zr);
  ref_unrotate_v(rot, params + (size_t)kv_head * ref_params_per_head(rot, d), zr, out, d);
}

void ref_dequantize_slot(const double *params, int d, int n_kv_heads, int page,
                         const uint8_t *blocks, int phys_page, int kv_head, int slot, int kind,
                         double *out) {
  ref_dequantize_slot_v(3, 0, params, d, n_kv_heads, page, blocks, phys_page, kv_head, slot,
                        kind, out);
}

/* ------------------------------------------------------------------------------ */
/* Decode attention on the packed cache, all in the rotated space.                  */
/*   a6: q~ = R q (same WHT + blocks as the KV head's keys);                         */
/*   a7: s_t = scale * q~ . k~_t,  k~_t = (n_t / sqrt d) L[c_t];                      */
/*   a8: softmax over t = 0..len-1 and o~ = sum_t p_t v~_t;                          */
/*   a9: out = R^T o~.                                                               */
/* Q: [n_seqs][n_q_heads][d] fp64; out likewise.  A sequence of length 0 gives 0.    */
/* The (sequence, head) pairs listed in sel (pairs of ints; n_sel of them; NULL =    */
/* all) are the ones computed; others in out are left untouched.                     */
/* ------------------------------------------------------------------------------ */
void ref_decode_attention_v(int bits, int rot, const double *params, int d, int n_kv_heads,
                            int page, const uint8_t *blocks, const int32_t *page_table,
                            int max_pages_per_seq, int n_seqs, int n_q_heads,
                            const int32_t *seq_lens, const double *Q, double scale, double *out,
                            const int32_t *sel, int n_sel) {
  int G = n_q_heads / n_kv_heads;
  size_t bb = ref_block_bytes_v(bits, d, page);
  int pph = ref_params_per_head(rot, d);
  int total = sel ? n_sel : n_seqs * n_q_heads;
#pragma omp parallel for schedule(dynamic, 1)
  for (int w = 0; w < total; w++) {
    int s = sel ? sel[2 * w] : w / n_q_heads;
    int h = sel ? sel[2 * w + 1] : w % n_q_heads;
    int kvh = h / G;
    int len = seq_lens[s];
    const double *ph = params + (size_t)kvh * pph;
    double *o = out + ((size_t)s * n_q_heads + h) * d;
    if (len <= 0) {
      for (int i = 0; i < d; i++) o[i] = 0.0;
      continue;
    }
    double qt[1024], kt[1024], vt[1024], ot[1024];
    ref_rotate_v(rot, ph, Q + ((size_t)s * n_q_heads + h) * d, qt, d);

    double *sc = (double *)malloc(sizeof(double) * len);
    for (int t = 0; t < len; t++) {
      int phys = page_table[(size_t)s * max_pages_per_seq + t / page];
      const uint8_t *blk = blocks + ((size_t)phys * n_kv_heads + kvh) * bb;
      dequant_slot(bits, d, page, blk, t % page, 0, kt);
      double dot = 0.0;
      for (int i = 0; i < d; i++) dot += qt[i] * kt[i];
      sc[t] = scale * dot;
    }
    double m = -INFINITY;
    for (int t = 0; t < len; t++)
      if (sc[t] > m) m = sc[t];
    double l = 0.0;
    for (int i = 0; i < d; i++) ot[i] = 0.0;
    for (int t = 0; t < len; t++) {
      double p = exp(sc[t] - m);
      l += p;
      int phys = page_table[(size_t)s * max_pages_per_seq + t / page];
      const uint8_t *blk = blocks + ((size_t)phys * n_kv_heads + kvh) * bb;
      dequant_slot(bits, d, page, blk, t % page, 1, vt);
      for (int i = 0; i < d; i++) ot[i] += p * vt[i];
    }
    for (int i = 0; i < d; i++) ot[i] /= l;
    free(sc);
    ref_unrotate_v(rot, ph, ot, o, d);
  }
}

void ref_decode_attention(const double *params, int d, int n_kv_heads, int page,
                          const uint8_t *blocks, const int32_t *page_table,
                          int max_pages_per_seq, int n_seqs, int n_q_heads,
                          const int32_t *seq_lens, const double *Q, double scale, double *out,
                          const int32_t *sel, int n_sel) {
  ref_decode_attention_v(3, 0, params, d, n_kv_heads, page, blocks, page_table,
                         max_pages_per_seq, n_seqs, n_q_heads, seq_lens, Q, scale, out, sel,
                         n_sel);
}

/* Full-precision attention (no quantisation, no rotation) for the error-bound tests:
 * K, V [n_tokens][n_kv_heads][d], one sequence of n_tokens, Q [n_q_heads][d]. */
void ref_attention_full(int d, int n_kv_heads, int n_q_heads, int n_tokens, const double *K,
                        const double *V, const double *Q, double scale, double *out) {
  int G = n_q_heads / n_kv_heads;
  for (int h = 0; h < n_q_heads; h++) {
    int kvh = h / G;
    const double *q = Q + (size_t)h * d;
    double *sc = (double *)malloc(sizeof(double) * (n_tokens > 0 ? n_tokens : 1));
    double m = -INFINITY;
    for (int t = 0; t < n_tokens; t++) {
      const double *k = K + ((size_t)t * n_kv_heads + kvh) * d;
      double dot = 0.0;
      for (int i = 0; i < d; i++) dot += q[i] * k[i];
      sc[t] = scale * dot;
      if (sc[t] > m) m = sc[t];
    }
    double *o = out + (size_t)h * d;
    for (int i = 0; i < d; i++) o[i] = 0.0;
    double l = 0.0;
    for (int t = 0; t < n_tokens; t++) {
      double p = exp(sc[t] - m);
      l += p;
      const double *v = V + ((size_t)t * n_kv_heads + kvh) * d;
      for (int i = 0; i < d; i++) o[i] += p * v[i];
    }
    if (n_tokens > 0)
      for (int i = 0; i < d; i++) o[i] /= l;
    free(sc);
  }
}

/* ------------------------------------------------------------------------------ */
/* Batch helpers for parity checks.                                                 */
/* ------------------------------------------------------------------------------ */
/* Quantise n_rows rows of X ([n_rows][n_kv_heads][d]; row r, head h uses head h's
 * params) and report, per element, the distance of u = sqrt(d) z / n to the nearest
 * threshold (N(0,1) units; +inf for a zero vector).  codes [n_rows][H][d],
 * norms [n_rows][H] (binary16 bits), dist [n_rows][H][d] (may be NULL). */
void ref_quantize_rows_v(int bits, int rot, const double *params, int d, int n_kv_heads,
                         const double *X, int n_rows, uint8_t *codes, uint16_t *norms,
                         double *dist) {
  int pph = ref_params_per_head(rot, d);
  int nt = (1 << bits) - 1;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < n_rows; r++) {
    double z[1024];
    for (int h = 0; h < n_kv_heads; h++) {
      size_t v = (size_t)r * n_kv_heads + h;
      const double *x = X + v * d;
      ref_quantize_vector_v(bits, rot, params + (size_t)h * pph, x, d, codes + v * d, norms + v, z);
      if (!dist) continue;
      double ss = 0.0;
      for (int i = 0; i < d; i++) ss += x[i] * x[i];
      double n = sqrt(ss);
      for (int i = 0; i < d; i++) {
        double best = INFINITY;
        if (n > 0.0) {
          double u = sqrt((double)d) * z[i] / n;
          for (int j = 0; j < nt; j++) {
            double e = fabs(u - ref_threshold_v(bits, j));
            if (e < best) best = e;
          }
        }
        dist[v * d + i] = best;
      }
    }
  }
}

void ref_quantize_rows(const double *params, int d, int n_kv_heads, const double *X, int n_rows,
                       uint8_t *codes, uint16_t *norms, double *dist) {
  ref_quantize_rows_v(3, 0, params, d, n_kv_heads, X, n_rows, codes, norms, dist);
}

/* Unpack n records of packed codes (bits * d / 8 bytes each, contiguous) into codes [n][d]. */
void ref_unpack_codes_batch_v(int bits, const uint8_t *in, int d, long n, uint8_t *codes) {
#pragma omp parallel for schedule(static)
  for (long i = 0; i < n; i++) ref_unpack_codes_v(bits, in + i * cbytes(bits, d), d, codes + i * d);
}

void ref_unpack_codes_batch(const uint8_t *in, int d, long n, uint8_t *codes) {
  ref_unpack_codes_batch_v(3, in, d, n, codes);
}
