/*
 * Reference oracle for split-KV paged attention (decode and speculative
 * verification) over a fragment-addressed K/V cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with the
 * CUDA library; it reads the same arena bytes and page tables and does its
 * own address arithmetic and its own decoding of the stored formats.
 *
 * Plain, single-threaded, float64.  Every stored K/V element is widened to
 * double exactly; every sum runs in double, in logical key order.
 *
 * What it computes (passages followed):
 *  - K/V storage formats fp32, fp16, bf16, fp8 and bf8 with FP32-or-wider
 *    accumulation: LSE README (Geramy/LSE), "KV cache formats" paragraph and
 *    its bytes-per-token table.  "fp8" is read as OCP E4M3 (finite-only,
 *    max 448) and "bf8" as OCP E5M2 (IEEE-style inf/NaN).
 *  - Fixed-size fragments of shared arenas, one set of fragments per K or V
 *    tensor, reached through a per-sequence page table: LSE releases,
 *    v0.4.20 "K/V memory management and automatic split attention".
 *    Layout inside a fragment is token-major [token][kv_head][dim].
 *  - Query rows of a decode step or of a draft chain/tree sharing each K/V
 *    read: LSE releases, v0.4.21 "joint decode attention"; v0.4.19
 *    "Long-context split attention".  The R query rows are the last R
 *    positions of the sequence; every row sees the whole cached context and,
 *    among the draft positions, the ones set in its ancestor mask (the chain
 *    default is "itself and all earlier drafts").  Without masks the rows
 *    may be any number (a prefill block: row r sees positions up to its
 *    own, the causal rule of the long-query paged attention of LSE
 *    releases, v0.4.14 "Improvements", whose kernel skips 256-key windows
 *    that no row of a block sees); masks (tree rows) are 64 bits, so R <= 64.
 *  - Split attention with one partial family and one merge family, the
 *    partition count taken from page-table capacity, empty partitions
 *    skipped: LSE releases, v0.4.19 and v0.4.20.  The merge is the
 *    log-sum-exp combination, which reproduces unsplit softmax exactly.
 *
 * Definition, for sequence s with L keys of which the last R are query rows
 * (context C = L - R), query row r, query head h, kv head g = h / (Hq/Hkv):
 *    x_j  = scale * sum_d q[d] * K[j][g][d]          over visible j
 *    m    = max_j x_j
 *    out  = sum_j exp(x_j - m) V[j][g] / sum_j exp(x_j - m)
 *    lse  = m + ln sum_j exp(x_j - m)
 * GQA grouping (query head h reads kv head h / G, contiguous groups) is the
 * plain reading where the pages are silent.
 *
 * Per-vector scales (LSE README, "KV cache formats": fp8 and bf8 "with
 * scales", 33,280 bytes per token where the 8-bit elements take 32,768, so
 * one FP32 scale per (token, kv head) of K and one of V): the stored vector
 * times its scale is the key or value,
 *    K[j][g][d] = decode(stored K) * sK[j][g],  V likewise with sV.
 * The pages do not place the scales; the reading here is that they are paged
 * like the vectors: every fragment owns a block of T * Hkv FP32 scales,
 * kv-head-major [kv_head][token], at index fragment_id * Hkv * T of one scale
 * array, so K scales sit in the blocks of K fragments and V scales in those
 * of V fragments.  Without a scale array every scale is 1.
 *
 * K/V append (the write of a verify step's new tokens into their fragments,
 * FP32 cast to the storage format: LSE releases, v0.4.20, K/V memory
 * management): each new token's K and V vectors go to position
 * L_before + i of their sequence through its page tables.  The cast is the
 * nearest value of the format, ties to even, from the format's bit layout;
 * FP16/BF16 overflow to infinity as IEEE formats do; the FP8 formats
 * saturate to their largest finite value (E4M3 has no infinity; the pages
 * fix no overflow rule for E5M2, and saturating keeps a cache finite).
 * With per-vector scales (8-bit formats) the append also picks each new
 * vector's scale: the pages say only that scales exist, so the reading is
 * the usual per-vector one, scale = (largest magnitude in the vector) /
 * (largest finite value of the format), 1 for an all-zero vector, every
 * element stored as the FP32 quotient element / scale rounded to the
 * format.  Both divisions are FP32 operations (correctly rounded), so the
 * stored code is fixed to the bit.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

/* Status codes returned by the oracle (its own, not the library's). */
#define ORC_OK 0
#define ORC_BAD_SHAPE 1     /* a size or count is out of range            */
#define ORC_BAD_PAGE 2      /* a page-table entry names no fragment        */
#define ORC_BAD_MASK 3      /* an ancestor mask violates the tree rules    */
#define ORC_BAD_DTYPE 4     /* unknown storage format                      */

/* Storage formats, numbered for this file only. */
#define ORC_F32 0
#define ORC_F16 1
#define ORC_BF16 2
#define ORC_E4M3 3
#define ORC_E5M2 4

typedef struct {
  const uint8_t *const *chunks; /* host copies of each arena chunk          */
  int n_chunks;
  int64_t chunk_bytes;
  int64_t fragment_bytes;
  int dtype;
  int n_kv_heads;
  int head_dim;
  int n_q_heads;
  int n_seqs;
  int max_pages;            /* page-table row length (capacity in pages)   */
  const int32_t *k_pages;   /* [n_seqs][max_pages]                         */
  const int32_t *v_pages;   /* [n_seqs][max_pages]                         */
  const int32_t *seq_lens;  /* [n_seqs]  L_s, query rows included          */
  const int32_t *row_offsets; /* [n_seqs + 1]                              */
  const uint64_t *row_masks;  /* [total_rows] or NULL for the chain        */
  const float *q;           /* [total_rows][n_q_heads][head_dim]           */
  double scale;
  const float *scales;      /* per-vector scales by fragment, or NULL      */
  int64_t n_scales;         /* floats in scales                            */
} orc_problem;

/* ---- decoding of one stored element to double, from each format's bit
 * layout (sign, biased exponent, fraction) ------------------------------ */

static double pow2(int e) { return ldexp(1.0, e); }

static double decode_f32(const uint8_t *p) {
  float f;
  memcpy(&f, p, 4);
  return (double)f;
}

/* Generic sign/exponent/fraction decoder.  ebits/mbits: field widths.
 * ieee_special: exponent all-ones encodes inf (fraction 0) or NaN.
 * e4m3_special: only exponent all-ones with fraction all-ones is NaN. */
static double decode_minifloat(uint32_t bits, int ebits, int mbits, int ieee_special,
                               int e4m3_special) {
  uint32_t sign = (bits >> (ebits + mbits)) & 1u;
  uint32_t e = (bits >> mbits) & ((1u << ebits) - 1u);
  uint32_t m = bits & ((1u << mbits) - 1u);
  int bias = (1 << (ebits - 1)) - 1;
  double v;
  if (ieee_special && e == (1u << ebits) - 1u) {
    v = (m == 0) ? INFINITY : NAN;
  } else if (e4m3_special && e == (1u << ebits) - 1u && m == (1u << mbits) - 1u) {
    v = NAN;
  } else if (e == 0) {
    v = (double)m * pow2(1 - bias - mbits); /* subnormal */
  } else {
    v = (1.0 + (double)m * pow2(-mbits)) * pow2((int)e - bias);
  }
  return sign ? -v : v;
}

static double decode_elem(int dtype, const uint8_t *p) {
  switch (dtype) {
    case ORC_F32: return decode_f32(p);
    case ORC_F16: return decode_minifloat((uint32_t)p[0] | ((uint32_t)p[1] << 8), 5, 10, 1, 0);
    case ORC_BF16: return decode_minifloat((uint32_t)p[0] | ((uint32_t)p[1] << 8), 8, 7, 1, 0);
    case ORC_E4M3: return decode_minifloat(p[0], 4, 3, 0, 1);
    case ORC_E5M2: return decode_minifloat(p[0], 5, 2, 1, 0);
  }
  return NAN;
}

static int elem_size(int dtype) {
  switch (dtype) {
    case ORC_F32: return 4;
    case ORC_F16: case ORC_BF16: return 2;
    case ORC_E4M3: case ORC_E5M2: return 1;
  }
  return 0;
}

/* Exported so tests can compare the decoder with a library conversion. */
double orc_decode(int dtype, uint32_t bits) {
  uint8_t b[4];
  b[0] = (uint8_t)(bits & 0xff);
  b[1] = (uint8_t)((bits >> 8) & 0xff);
  b[2] = (uint8_t)((bits >> 16) & 0xff);
  b[3] = (uint8_t)((bits >> 24) & 0xff);
  return decode_elem(dtype, b);
}

/* ---- encoding of one double to a format's bits (nearest, ties to even) --- */

/* Generic sign/exponent/fraction encoder: ebits/mbits field widths; max_e /
 * max_m the fields of the largest finite value; sat: overflow saturates to
 * it (else it becomes infinity, exponent all ones and fraction 0); nan_bits:
 * the encoding used for NaN input. */
static uint32_t encode_minifloat(double x, int ebits, int mbits, uint32_t max_e, uint32_t max_m,
                                 int sat, uint32_t nan_bits) {
  if (isnan(x)) return nan_bits;
  const uint32_t sign = signbit(x) ? 1u << (ebits + mbits) : 0u;
  double a = fabs(x);
  const int bias = (1 << (ebits - 1)) - 1;
  const int emin = 1 - bias;  /* exponent of the smallest normal */
  const double maxv = (1.0 + (double)max_m * pow2(-mbits)) * pow2((int)max_e - bias);
  const double half_ulp_max = pow2((int)max_e - bias - mbits - 1);
  if (a >= maxv + half_ulp_max) {  /* rounds past the largest finite value */
    if (sat) return sign | (max_e << mbits) | max_m;
    return sign | (((1u << ebits) - 1u) << mbits);
  }
  if (a == 0.0) return sign;
  /* quantum of the binade of a (subnormals share the smallest normal's) */
  int e;
  frexp(a, &e);  /* a = f 2^e, f in [0.5, 1): binade exponent e - 1 */
  int be = e - 1 < emin ? emin : e - 1;
  const double q = pow2(be - mbits);
  const double n = a / q;  /* exact: a carries 24 significant bits at most */
  double r = floor(n);
  const double frac = n - r;
  if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
  const double v = r * q;  /* the rounded magnitude, exactly */
  if (v == 0.0) return sign;
  frexp(v, &e);
  be = e - 1;
  if (be < emin) /* subnormal: exponent field 0 */
    return sign | (uint32_t)(v / pow2(emin - mbits));
  const uint32_t ef = (uint32_t)(be + bias);
  const uint32_t mf = (uint32_t)((v / pow2(be) - 1.0) * pow2(mbits));
  return sign | (ef << mbits) | mf;
}

static uint32_t encode_elem(int dtype, double x) {
  switch (dtype) {
    case ORC_F16: return encode_minifloat(x, 5, 10, 30, 1023, 0, 0x7E00u);
    case ORC_BF16: return encode_minifloat(x, 8, 7, 254, 127, 0, 0x7FC0u);
    case ORC_E4M3: return encode_minifloat(x, 4, 3, 15, 6, 1, 0x7Fu);
    case ORC_E5M2: return encode_minifloat(x, 5, 2, 30, 3, 1, 0x7Fu);
  }
  return 0;
}

/* Exported so tests can compare the encoder with library conversions. */
uint32_t orc_encode(int dtype, double x) {
  if (dtype == ORC_F32) {
    float f = (float)x;
    uint32_t b;
    memcpy(&b, &f, 4);
    return b;
  }
  return encode_elem(dtype, x);
}

/* ---- fragment addressing ---------------------------------------------- */

static int64_t tokens_per_fragment(const orc_problem *pb) {
  return pb->fragment_bytes /
         ((int64_t)pb->n_kv_heads * pb->head_dim * elem_size(pb->dtype));
}

/* Address of element 0 of key j, kv head g, through a page table. */
static const uint8_t *kv_row(const orc_problem *pb, const int32_t *table, int s, int64_t j,
                             int g, int *status) {
  int64_t T = tokens_per_fragment(pb);
  int64_t page = j / T;
  int64_t off = j % T;
  int32_t frag = table[(int64_t)s * pb->max_pages + page];
  int64_t frags_per_chunk = pb->chunk_bytes / pb->fragment_bytes;
  if (frag < 0 || frag >= frags_per_chunk * pb->n_chunks) {
    *status = ORC_BAD_PAGE;
    return NULL;
  }
  int64_t chunk = frag / frags_per_chunk;
  int64_t byte = (frag % frags_per_chunk) * pb->fragment_bytes +
                 (off * pb->n_kv_heads + g) * (int64_t)pb->head_dim * elem_size(pb->dtype);
  return pb->chunks[chunk] + byte;
}

/* Per-vector scale of key j, kv head g, through a page table: entry
 * (g, j % T) of the block of the fragment holding key j (1 without scales). */
static double vec_scale(const orc_problem *pb, const int32_t *table, int s, int64_t j, int g,
                        int *status) {
  if (!pb->scales) return 1.0;
  int64_t T = tokens_per_fragment(pb);
  int32_t frag = table[(int64_t)s * pb->max_pages + j / T];
  int64_t at = ((int64_t)frag * pb->n_kv_heads + g) * T + j % T;
  if (frag < 0 || at >= pb->n_scales) {
    *status = ORC_BAD_PAGE;
    return 0.0;
  }
  return (double)pb->scales[at];
}

/* ---- visibility --------------------------------------------------------- */

static uint64_t row_mask(const orc_problem *pb, int s, int r) {
  if (pb->row_masks) return pb->row_masks[pb->row_offsets[s] + r];
  /* chain: row r sees drafts 0..r */
  return (r >= 63) ? ~(uint64_t)0 : (((uint64_t)1 << (r + 1)) - 1);
}

/* Key j visible to row r (C context keys): the context always; among the
 * drafts, the bits of the row's mask, or without masks the chain (drafts up
 * to the row itself, for any number of rows). */
static int visible(const orc_problem *pb, int64_t j, int64_t C, int r, uint64_t mask) {
  if (j < C) return 1;
  if (!pb->row_masks) return j - C <= r;
  return (int)((mask >> (j - C)) & 1u);
}

/* ---- checks --------------------------------------------------------------- */

static int check_problem(const orc_problem *pb) {
  if (pb->n_seqs < 0 || pb->n_kv_heads <= 0 || pb->head_dim <= 0 || pb->n_q_heads <= 0)
    return ORC_BAD_SHAPE;
  if (pb->n_q_heads % pb->n_kv_heads) return ORC_BAD_SHAPE;
  if (elem_size(pb->dtype) == 0) return ORC_BAD_DTYPE;
  if (pb->fragment_bytes <= 0 || pb->chunk_bytes % pb->fragment_bytes) return ORC_BAD_SHAPE;
  if (pb->fragment_bytes % ((int64_t)pb->n_kv_heads * pb->head_dim * elem_size(pb->dtype)))
    return ORC_BAD_SHAPE;
  int64_t T = tokens_per_fragment(pb);
  if (pb->scales && pb->n_scales < pb->n_chunks * (pb->chunk_bytes / pb->fragment_bytes) *
                                       pb->n_kv_heads * T)
    return ORC_BAD_SHAPE;  /* a block for every fragment of the arena */
  for (int s = 0; s < pb->n_seqs; ++s) {
    int64_t L = pb->seq_lens[s];
    int R = pb->row_offsets[s + 1] - pb->row_offsets[s];
    if (R < 0 || (pb->row_masks && R > 64) || L < R || L > (int64_t)pb->max_pages * T)
      return ORC_BAD_SHAPE;
    if (R > 0 && L < 1) return ORC_BAD_SHAPE;
    for (int r = 0; pb->row_masks && r < R; ++r) {
      uint64_t m = row_mask(pb, s, r);
      if (!((m >> r) & 1u)) return ORC_BAD_MASK;                 /* sees itself */
      if (r < 63 && (m >> (r + 1)) != 0) return ORC_BAD_MASK;    /* no later draft */
    }
  }
  return ORC_OK;
}

/* ---- one output row ------------------------------------------------------ */

/* Attention of query (seq s, row r, head h) over the visible keys in
 * [key_begin, key_end).  Writes out[head_dim] and *lse.  With no visible
 * key in the range: out = 0, lse = -inf (an empty partial). */
static int attend_range(const orc_problem *pb, int s, int r, int h, int64_t key_begin,
                        int64_t key_end, double *out, double *lse) {
  int status = ORC_OK;
  const int D = pb->head_dim;
  const int G = pb->n_q_heads / pb->n_kv_heads;
  const int g = h / G;
  const int64_t L = pb->seq_lens[s];
  const int R = pb->row_offsets[s + 1] - pb->row_offsets[s];
  const int64_t C = L - R;
  const uint64_t mask = pb->row_masks ? row_mask(pb, s, r) : 0;
  const float *q = pb->q + ((int64_t)(pb->row_offsets[s] + r) * pb->n_q_heads + h) * D;
  const int es = elem_size(pb->dtype);

  /* pass 1: the maximum score */
  double m = -INFINITY;
  for (int64_t j = key_begin; j < key_end; ++j) {
    if (!visible(pb, j, C, r, mask)) continue;
    const uint8_t *k = kv_row(pb, pb->k_pages, s, j, g, &status);
    const double sk = vec_scale(pb, pb->k_pages, s, j, g, &status);
    if (status) return status;
    double x = 0.0;
    for (int d = 0; d < D; ++d) x += (double)q[d] * (decode_elem(pb->dtype, k + d * es) * sk);
    x *= pb->scale;
    if (x > m) m = x;
  }
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return ORC_OK;
  }
  /* pass 2: weights, their sum and the weighted sum of V */
  double l = 0.0;
  for (int64_t j = key_begin; j < key_end; ++j) {
    if (!visible(pb, j, C, r, mask)) continue;
    const uint8_t *k = kv_row(pb, pb->k_pages, s, j, g, &status);
    const uint8_t *v = kv_row(pb, pb->v_pages, s, j, g, &status);
    const double sk = vec_scale(pb, pb->k_pages, s, j, g, &status);
    const double sv = vec_scale(pb, pb->v_pages, s, j, g, &status);
    if (status) return status;
    double x = 0.0;
    for (int d = 0; d < D; ++d) x += (double)q[d] * (decode_elem(pb->dtype, k + d * es) * sk);
    x *= pb->scale;
    double p = exp(x - m);
    l += p;
    for (int d = 0; d < D; ++d) out[d] += p * (decode_elem(pb->dtype, v + d * es) * sv);
  }
  for (int d = 0; d < D; ++d) out[d] /= l;
  *lse = m + log(l);
  return ORC_OK;
}

/* ---- exported entry points ---------------------------------------------- */

/* One output: (seq s, row r, head h) over the whole sequence. */
int orc_attention_one(const orc_problem *pb, int s, int r, int h, double *out, double *lse) {
  int st = check_problem(pb);
  if (st) return st;
  if (s < 0 || s >= pb->n_seqs || h < 0 || h >= pb->n_q_heads) return ORC_BAD_SHAPE;
  if (r < 0 || r >= pb->row_offsets[s + 1] - pb->row_offsets[s]) return ORC_BAD_SHAPE;
  return attend_range(pb, s, r, h, 0, pb->seq_lens[s], out, lse);
}

/* Every output: out [total_rows][n_q_heads][head_dim], lse [total_rows][n_q_heads]. */
int orc_attention(const orc_problem *pb, double *out, double *lse) {
  int st = check_problem(pb);
  if (st) return st;
  const int D = pb->head_dim;
  for (int s = 0; s < pb->n_seqs; ++s) {
    int R = pb->row_offsets[s + 1] - pb->row_offsets[s];
    for (int r = 0; r < R; ++r) {
      for (int h = 0; h < pb->n_q_heads; ++h) {
        int64_t o = (int64_t)(pb->row_offsets[s] + r) * pb->n_q_heads + h;
        st = attend_range(pb, s, r, h, 0, pb->seq_lens[s], out + o * D, lse + o);
        if (st) return st;
      }
    }
  }
  return ORC_OK;
}

/* Split mode: the keys of each sequence are cut into partitions of
 * keys_per_part keys; each partition yields a normalised partial output and
 * its log-sum-exp (an empty partition yields lse = -inf and is skipped);
 * the partials are then merged:
 *     M = max_p lse_p,  w_p = exp(lse_p - M),
 *     out = sum_p w_p o_p / sum_p w_p,  lse = M + ln sum_p w_p.
 * scratch must hold head_dim doubles. */
int orc_attention_split(const orc_problem *pb, int64_t keys_per_part, double *out,
                        double *lse, double *scratch) {
  int st = check_problem(pb);
  if (st) return st;
  if (keys_per_part <= 0) return ORC_BAD_SHAPE;
  const int D = pb->head_dim;
  for (int s = 0; s < pb->n_seqs; ++s) {
    int R = pb->row_offsets[s + 1] - pb->row_offsets[s];
    int64_t L = pb->seq_lens[s];
    int64_t n_parts = (L + keys_per_part - 1) / keys_per_part;
    for (int r = 0; r < R; ++r) {
      for (int h = 0; h < pb->n_q_heads; ++h) {
        int64_t o = (int64_t)(pb->row_offsets[s] + r) * pb->n_q_heads + h;
        double *acc = out + o * D;
        /* the maximum partial lse */
        double M = -INFINITY;
        for (int64_t p = 0; p < n_parts; ++p) {
          double lp;
          int64_t b = p * keys_per_part, e = b + keys_per_part < L ? b + keys_per_part : L;
          st = attend_range(pb, s, r, h, b, e, scratch, &lp);
          if (st) return st;
          if (lp > M) M = lp;
        }
        for (int d = 0; d < D; ++d) acc[d] = 0.0;
        double wsum = 0.0;
        for (int64_t p = 0; p < n_parts; ++p) {
          double lp;
          int64_t b = p * keys_per_part, e = b + keys_per_part < L ? b + keys_per_part : L;
          st = attend_range(pb, s, r, h, b, e, scratch, &lp);
          if (st) return st;
          if (lp == -INFINITY) continue; /* empty partition: skipped */
          double w = exp(lp - M);
          wsum += w;
          for (int d = 0; d < D; ++d) acc[d] += w * scratch[d];
        }
        for (int d = 0; d < D; ++d) acc[d] /= wsum;
        lse[o] = M + log(wsum);
      }
    }
  }
  return ORC_OK;
}

/* Bytes of K and V per token for a model with n_layers KV layers: the
 * accounting of the LSE README bytes-per-token table, where the 8-bit
 * formats carry one FP32 scale per (token, kv head) vector. */
int64_t orc_kv_bytes_per_token(int dtype, int n_layers, int n_kv_heads, int head_dim,
                               int with_scales) {
  int64_t per = (int64_t)n_layers * 2 * n_kv_heads * head_dim * elem_size(dtype);
  if (with_scales) per += (int64_t)n_layers * 2 * n_kv_heads * 4;
  return per;
}

/* K/V append: new tokens i in [new_offsets[s], new_offsets[s+1]) of
 * sequence s go to key position seq_lens_before[s] + (i - new_offsets[s]);
 * k_new / v_new are [total_new][n_kv_heads][head_dim] FP32.  Writes the
 * encoded elements into the (writable) host copies of the arena chunks.
 * A position past the page table or a page naming no fragment is skipped
 * and reported (ORC_BAD_PAGE); everything else is still written. */
int orc_kv_append(uint8_t *const *chunks, int n_chunks, int64_t chunk_bytes,
                  int64_t fragment_bytes, int dtype, int n_kv_heads, int head_dim, int n_seqs,
                  int max_pages, const int32_t *k_pages, const int32_t *v_pages,
                  const int32_t *seq_lens_before, const int32_t *new_offsets,
                  const float *k_new, const float *v_new, float *scales, int64_t n_scales) {
  const int es = elem_size(dtype);
  if (es == 0) return ORC_BAD_DTYPE;
  if (n_kv_heads < 1 || head_dim < 1 || fragment_bytes < (int64_t)n_kv_heads * head_dim * es)
    return ORC_BAD_SHAPE;
  const int64_t T = fragment_bytes / ((int64_t)n_kv_heads * head_dim * es);
  const int64_t per_chunk = chunk_bytes / fragment_bytes;
  if (scales && (es != 1 || n_scales < per_chunk * n_chunks * n_kv_heads * T))
    return ORC_BAD_SHAPE;  /* 8-bit formats, a block for every fragment */
  const float fmt_max = dtype == ORC_E4M3 ? 448.0f : 57344.0f;
  int status = ORC_OK;
  for (int s = 0; s < n_seqs; ++s) {
    for (int32_t i = new_offsets[s]; i < new_offsets[s + 1]; ++i) {
      const int64_t pos = (int64_t)seq_lens_before[s] + (i - new_offsets[s]);
      const int64_t page = pos / T, off = pos % T;
      for (int kv = 0; kv < 2; ++kv) {
        const int32_t *table = kv ? v_pages : k_pages;
        const float *src = kv ? v_new : k_new;
        if (pos < 0 || page >= max_pages) {
          status = ORC_BAD_PAGE;
          continue;
        }
        const int32_t frag = table[(int64_t)s * max_pages + page];
        if (frag < 0 || frag >= per_chunk * n_chunks) {
          status = ORC_BAD_PAGE;
          continue;
        }
        uint8_t *dst = chunks[frag / per_chunk] + (frag % per_chunk) * fragment_bytes +
                       off * (int64_t)n_kv_heads * head_dim * es;
        for (int g = 0; g < n_kv_heads; ++g) {
          const float *x = src + ((int64_t)i * n_kv_heads + g) * head_dim;
          float sc = 1.0f;
          if (scales) {
            float amax = 0.0f;
            for (int d = 0; d < head_dim; ++d)
              if (fabsf(x[d]) > amax) amax = fabsf(x[d]);
            if (amax > 0.0f) sc = amax / fmt_max;
            scales[((int64_t)frag * n_kv_heads + g) * T + off] = sc;
          }
          for (int d = 0; d < head_dim; ++d) {
            const float q = scales ? x[d] / sc : x[d];
            const uint32_t bits = orc_encode(dtype, (double)q);
            uint8_t *o = dst + ((int64_t)g * head_dim + d) * es;
            for (int b = 0; b < es; ++b) o[b] = (uint8_t)((bits >> (8 * b)) & 0xffu);
          }
        }
      }
    }
  }
  return status;
}
