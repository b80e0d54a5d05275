/*
 * dao.c -- the CPU oracle for split-KV decode attention over a paged,
 * variable-length KV cache ("Dynamic Attention").
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
 * baseline leg may load this library.  The product path (the CUDA library in
 * variable_length_paged_b200/) never calls it, and the two share no code,
 * header, table or helper.
 *
 * Source.  The method is described in "Tencent HPC lands in SGLang,
 * challenging default inference kernels":
 *   - section "Why Tencent HPC matters for online model serving": decode work
 *     over the key-value cache is uneven across requests (a 16,000-token
 *     context next to a 1,000-token one); the cache work is cut into smaller,
 *     uniform tiles that a scheduler hands to CTAs according to the current
 *     workload, and the mapping is rebuilt as request lengths change; a
 *     longer history means more cached data to read;
 *   - the same section, on the baseline: a static split policy either idles
 *     GPU units or launches empty chunks for the shorter requests.
 * The article gives no formula.  What is computed is therefore written out
 * from its plain definition:
 *   attention  softmax(scale * q . K^T) . V over the cached tokens of one
 *              request, with grouped KV heads (query head h reads KV head
 *              h / (Hq/Hkv)), returned with its natural-log log-sum-exp;
 *   plan       tiles of T tokens per request, balanced contiguous ranges of
 *              tiles per CTA, cut at request boundaries into segments;
 *   static     a fixed number of equal splits per request (the comparator).
 * Splitting the token range and merging the pieces by log-sum-exp is an exact
 * re-association of the softmax, so the oracle does not split at all: it is
 * the unsplit definition, in fp64, over the bf16-decoded inputs.
 *
 * Readings where the article is silent (each also listed in the design notes):
 *   - GQA grouping is consecutive: KV head g serves query heads
 *     [g*G, (g+1)*G), G = Hq / Hkv.
 *   - lse is the natural log of sum_t exp(s_t), s_t the SCALED score.
 *   - A request of length 0 has out = 0 and lse = -inf; it is not an error.
 *   - A length below 0 or above max_pages_per_req * page_size is a data error:
 *     it is reported (lowest such request index) and the request counts as
 *     length 0.
 *   - KV layout [num_pages][Hkv][page_size][head_dim]; token t of request b
 *     lives in page block_table[b][t / page_size], slot t % page_size.
 *   - Unit u belongs to CTA c exactly when floor(c*U/C) <= u < floor((c+1)*U/C)
 *     (balanced, contiguous; empty ranges allowed when U < C).
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC dao.c -o libdao.so
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define DAO_OK 0
#define DAO_ERR_ARG (-1)
#define DAO_ERR_BAD_SEQLEN (-2)
#define DAO_ERR_BAD_PAGE (-3)
#define DAO_ERR_CAPACITY (-4)

/* A bf16 value is the upper 16 bits of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * An FP8 E4M3 code (OCP 8-bit floating point, "E4M3FN"): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6); the
 * code S.1111.111 is NaN; there are no infinities.  Every code is exact in fp64.
 */
static double e4m3_to_double(uint8_t x) {
  const int sign = x >> 7, e = (x >> 3) & 15, m = x & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m, -9);
  else mag = ldexp((double)(8 + m), e - 10);
  return sign ? -mag : mag;
}

double dao_e4m3_value(uint8_t x) { return e4m3_to_double(x); }

/* Length of request b as the method sees it: out-of-range lengths count as 0. */
static int64_t effective_length(int32_t len, int64_t capacity) {
  if (len < 0 || (int64_t)len > capacity) return 0;
  return len;
}

int dao_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/*
 * K/V element access for the two cache formats: bf16 codes, or FP8 E4M3 codes
 * times a per-KV-head scale (the value stored for head g is x / scale[g]).
 */
typedef struct {
  int fp8;
  const void* k;
  const void* v;
  const double* k_scale;
  const double* v_scale;
} kv_view;

static double kv_elem(const kv_view* kv, int is_v, int64_t index, int32_t g) {
  if (!kv->fp8) return bf16_bits_to_double(((const uint16_t*)(is_v ? kv->v : kv->k))[index]);
  const double sc = is_v ? kv->v_scale[g] : kv->k_scale[g];
  return sc * e4m3_to_double(((const uint8_t*)(is_v ? kv->v : kv->k))[index]);
}

/*
 * Attention for a list of (request, query head) pairs.
 *
 * q       bf16 bits [batch][num_q_heads][head_dim]
 * kv      the cache, [num_pages][num_kv_heads][page_size][head_dim] elements
 * out     fp64 [n_pairs][head_dim];  lse fp64 [n_pairs]
 * pair_b, pair_h: the pairs; when pair_b is NULL every (b, h) pair is taken
 * in row-major order (n_pairs must then be batch * num_q_heads).
 *
 * Returns DAO_OK, or the first error found (bad argument, bad length, page id
 * out of range).  On a bad length or page the pair's outputs are still
 * written (length treated as 0 / the pair set to NaN respectively).
 */
static int attention_impl(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t page_size, int32_t max_pages_per_req, int64_t num_pages, double scale,
                          const uint16_t* q, const kv_view* kv, const int32_t* block_table,
                          const int32_t* seq_lens, int64_t n_pairs, const int32_t* pair_b, const int32_t* pair_h,
                          double* out, double* lse, int32_t num_threads) {
  if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || page_size <= 0 ||
      max_pages_per_req < 0 || num_pages < 0 || num_q_heads % num_kv_heads != 0)
    return DAO_ERR_ARG;
  if (!pair_b && n_pairs != (int64_t)batch * num_q_heads) return DAO_ERR_ARG;
  const int32_t group = num_q_heads / num_kv_heads;
  const int64_t capacity = (int64_t)max_pages_per_req * page_size;
  int status = DAO_OK;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#else
  (void)num_threads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < n_pairs; ++i) {
    const int32_t b = pair_b ? pair_b[i] : (int32_t)(i / num_q_heads);
    const int32_t h = pair_b ? pair_h[i] : (int32_t)(i % num_q_heads);
    double* o = out + i * head_dim;
    for (int32_t j = 0; j < head_dim; ++j) o[j] = 0.0;
    if (b < 0 || b >= batch || h < 0 || h >= num_q_heads) {
      lse[i] = NAN;
#pragma omp critical
      if (status == DAO_OK) status = DAO_ERR_ARG;
      continue;
    }
    const int32_t g = h / group; /* consecutive GQA grouping */
    const int64_t len = effective_length(seq_lens[b], capacity);
    if (len != seq_lens[b]) {
#pragma omp critical
      if (status == DAO_OK) status = DAO_ERR_BAD_SEQLEN;
    }
    if (len == 0) {
      lse[i] = -INFINITY;
      continue;
    }
    const uint16_t* qh = q + ((int64_t)b * num_q_heads + h) * head_dim;
    double* s = (double*)malloc((size_t)len * sizeof(double));
    int bad_page = 0;
    /* Pass 1: scaled scores s_t = scale * sum_j q_j k_tj. */
    for (int64_t t = 0; t < len; ++t) {
      const int32_t page = block_table[(int64_t)b * max_pages_per_req + t / page_size];
      if (page < 0 || (int64_t)page >= num_pages) { bad_page = 1; break; }
      const int64_t kt = (((int64_t)page * num_kv_heads + g) * page_size + t % page_size) * head_dim;
      double dot = 0.0;
      for (int32_t j = 0; j < head_dim; ++j) dot += bf16_bits_to_double(qh[j]) * kv_elem(kv, 0, kt + j, g);
      s[t] = scale * dot;
    }
    if (bad_page) {
      free(s);
      for (int32_t j = 0; j < head_dim; ++j) o[j] = NAN;
      lse[i] = NAN;
#pragma omp critical
      if (status == DAO_OK) status = DAO_ERR_BAD_PAGE;
      continue;
    }
    /* Pass 2: max, then the normaliser l = sum_t exp(s_t - M). */
    double m = -INFINITY;
    for (int64_t t = 0; t < len; ++t) if (s[t] > m) m = s[t];
    double l = 0.0;
    for (int64_t t = 0; t < len; ++t) l += exp(s[t] - m);
    /* Pass 3: out = sum_t exp(s_t - M) v_t / l. */
    for (int64_t t = 0; t < len; ++t) {
      const int32_t page = block_table[(int64_t)b * max_pages_per_req + t / page_size];
      const int64_t vt = (((int64_t)page * num_kv_heads + g) * page_size + t % page_size) * head_dim;
      const double w = exp(s[t] - m) / l;
      for (int32_t j = 0; j < head_dim; ++j) o[j] += w * kv_elem(kv, 1, vt + j, g);
    }
    lse[i] = m + log(l);
    free(s);
  }
  return status;
}

/*
 * Multi-query decode: q_len new tokens per request, the last q_len positions of
 * its cache.  Query i (0 <= i < q_len) sits at position L_b - q_len + i and
 * attends causally to tokens [0, L_b - q_len + i]; it is therefore plain
 * attention over the first L_b - q_len + i + 1 tokens (empty when that is <= 0).
 *   q    bf16 [batch][q_len][num_q_heads][head_dim]
 *   out  fp64 [batch][q_len][num_q_heads][head_dim];  lse fp64 [batch][q_len][num_q_heads]
 * Lengths out of range are reported as for dao_attention and count as 0.
 */
int dao_attention_mq(int32_t batch, int32_t q_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t page_size, int32_t max_pages_per_req, int64_t num_pages, double scale,
                     const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* block_table,
                     const int32_t* seq_lens, double* out, double* lse, int32_t num_threads) {
  if (batch < 0 || q_len <= 0 || max_pages_per_req < 0 || page_size <= 0) return DAO_ERR_ARG;
  const int64_t capacity = (int64_t)max_pages_per_req * page_size;
  const int64_t rows = (int64_t)batch * q_len;
  /* Every (request, query) becomes one single-query request with its own length. */
  int32_t* lens = (int32_t*)malloc((size_t)(rows > 0 ? rows : 1) * sizeof(int32_t));
  int32_t* bt = (int32_t*)malloc((size_t)(rows > 0 ? rows : 1) * (size_t)(max_pages_per_req > 0 ? max_pages_per_req : 1) *
                                 sizeof(int32_t));
  int status = DAO_OK;
  for (int32_t b = 0; b < batch; ++b) {
    int64_t L = seq_lens[b];
    if (L < 0 || L > capacity) {
      status = DAO_ERR_BAD_SEQLEN;
      L = 0;
    }
    for (int32_t i = 0; i < q_len; ++i) {
      const int64_t li = L - q_len + i + 1;
      lens[(int64_t)b * q_len + i] = (int32_t)(li > 0 ? li : 0);
      memcpy(bt + ((int64_t)b * q_len + i) * max_pages_per_req, block_table + (int64_t)b * max_pages_per_req,
             (size_t)max_pages_per_req * sizeof(int32_t));
    }
  }
  const kv_view kv = {0, k, v, NULL, NULL};
  const int st = attention_impl((int32_t)rows, num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_req,
                                num_pages, scale, q, &kv, bt, lens, rows * num_q_heads, NULL, NULL, out, lse,
                                num_threads);
  free(lens);
  free(bt);
  return st != DAO_OK ? st : status;
}

int dao_attention(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                  int32_t page_size, int32_t max_pages_per_req, int64_t num_pages, double scale,
                  const uint16_t* q, const uint16_t* k, const uint16_t* v,
                  const int32_t* block_table, const int32_t* seq_lens, int64_t n_pairs,
                  const int32_t* pair_b, const int32_t* pair_h, double* out, double* lse,
                  int32_t num_threads) {
  const kv_view kv = {0, k, v, NULL, NULL};
  return attention_impl(batch, num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_req, num_pages,
                        scale, q, &kv, block_table, seq_lens, n_pairs, pair_b, pair_h, out, lse, num_threads);
}

/*
 * Same, for an FP8 E4M3 cache: k_code, v_code [num_pages][Hkv][P][d] one byte
 * each, dequantised as k = k_scale[g] * e4m3(k_code) (per KV head g).
 */
int dao_attention_fp8(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                      int32_t page_size, int32_t max_pages_per_req, int64_t num_pages, double scale,
                      const uint16_t* q, const uint8_t* k_code, const uint8_t* v_code, const double* k_scale,
                      const double* v_scale, const int32_t* block_table, const int32_t* seq_lens,
                      int64_t n_pairs, const int32_t* pair_b, const int32_t* pair_h, double* out, double* lse,
                      int32_t num_threads) {
  const kv_view kv = {1, k_code, v_code, k_scale, v_scale};
  return attention_impl(batch, num_q_heads, num_kv_heads, head_dim, page_size, max_pages_per_req, num_pages,
                        scale, q, &kv, block_table, seq_lens, n_pairs, pair_b, pair_h, out, lse, num_threads);
}

/*
 * Log-sum-exp merge of n partial results of one (request, head):
 *   LSE = M + ln sum_i exp(lse_i - M),  M = max_i lse_i
 *   out = sum_i exp(lse_i - LSE) o_i
 * Partials with lse = -inf carry no weight; if all are -inf the result is
 * out = 0, lse = -inf.
 */
int dao_combine(int32_t n, int32_t head_dim, const double* o_parts, const double* lse_parts,
                double* out, double* lse) {
  if (n < 0 || head_dim <= 0) return DAO_ERR_ARG;
  double m = -INFINITY;
  for (int32_t i = 0; i < n; ++i) if (lse_parts[i] > m) m = lse_parts[i];
  for (int32_t j = 0; j < head_dim; ++j) out[j] = 0.0;
  if (m == -INFINITY) { *lse = -INFINITY; return DAO_OK; }
  double sum = 0.0;
  for (int32_t i = 0; i < n; ++i) sum += exp(lse_parts[i] - m);
  const double total = m + log(sum);
  for (int32_t i = 0; i < n; ++i) {
    const double w = exp(lse_parts[i] - total);
    for (int32_t j = 0; j < head_dim; ++j) out[j] += w * o_parts[(int64_t)i * head_dim + j];
  }
  *lse = total;
  return DAO_OK;
}

/* Tile count of one request: ceil(L / T) tiles of T tokens; bad lengths -> 0. */
static int64_t tiles_of(int32_t len, int32_t tile_tokens, int64_t capacity) {
  const int64_t l = effective_length(len, capacity);
  return (l + tile_tokens - 1) / tile_tokens;
}

/* Lowest request index with an out-of-range length, or -1. */
static int32_t first_bad_length(int32_t batch, const int32_t* seq_lens, int64_t capacity) {
  for (int32_t b = 0; b < batch; ++b)
    if (effective_length(seq_lens[b], capacity) != seq_lens[b]) return b;
  return -1;
}

/*
 * Dynamic (load-balanced) plan, written from its definition by walking the
 * global units in order.
 *
 *   n_b  = ceil(L_b / T) tiles;  w_b = n_b + sigma when n_b > 0, else 0
 *   prefix[b] = sum_{r<b} w_r,  U = prefix[B]
 *   The units of request r are [prefix[r], prefix[r+1]): the first sigma of
 *   them stand for the fixed cost of starting the request and carry no tokens
 *   ("start units"), the rest are its tiles 0 .. n_r - 1 in order.  With
 *   sigma = start_cost = 0 every unit is a tile.
 *   unit u belongs to the CTA c(u) = floor(((u+1)*C - 1) / U), the unique c with
 *   floor(c*U/C) <= u < floor((c+1)*U/C).
 *   A segment is a maximal run of consecutive tile units with the same
 *   (request, CTA); segments are numbered in unit order.
 *
 * The tiles are the article's uniform units of KV-cache work, spread over the
 * CTAs by the current lengths ("Tencent HPC lands in SGLang, challenging default
 * inference kernels", section "Why Tencent HPC matters for online model
 * serving").  The article gives no planner; the start units are this
 * implementation's addition: a CTA pays a fixed cost for every request it
 * starts (loading its query, merging and writing its result), so a CTA whose
 * range starts many short requests is given correspondingly fewer tiles.
 *
 * Outputs (caller-allocated):
 *   req_tile_prefix[B+1] (= prefix[], start units included), req_seg_begin[B+1]
 *   (segments of request b are [req_seg_begin[b], req_seg_begin[b+1])),
 *   cta_seg_begin[C+1] (segments of CTA c are [cta_seg_begin[c],
 *   cta_seg_begin[c+1])), seg_req, seg_cta, seg_tile_begin, seg_tile_end
 *   [max_segments] (tile indices relative to the request), *num_units (= U),
 *   *num_segments, *bad_index (-1 if none).
 * Returns DAO_OK, DAO_ERR_BAD_SEQLEN (outputs still valid, bad requests have
 * 0 tiles) or DAO_ERR_ARG / DAO_ERR_CAPACITY.
 *
 * Weighted ranges (dao_plan_weighted, cta_weights != NULL): CTA c's range is
 *   [first(c), first(c+1)),  first(c) = c + floor((U - C) * W_c / W)  when U >= C,
 * W_c = sum_{k<c} w_k, W = sum_k w_k: one unit each, and the other U - C units
 * in proportion to the weights (each w_k in [1, 65536]), so a CTA that will run on a
 * slower SM can be given less.  Equal weights give floor(c*U/C), the even split
 * above.  With U < C the weights are not used (every CTA holds at most one unit).
 * The weighting is this implementation's addition (the article spreads tiles
 * evenly over CTAs); it changes only who computes which tiles.
 */
int dao_plan_weighted(int32_t batch, const int32_t* seq_lens, int32_t tile_tokens, int32_t num_ctas,
                      int64_t capacity_tokens, int32_t max_segments, int32_t* num_units,
                      int32_t* num_segments, int32_t* req_tile_prefix, int32_t* req_seg_begin,
                      int32_t* cta_seg_begin, int32_t* seg_req, int32_t* seg_cta,
                      int32_t* seg_tile_begin, int32_t* seg_tile_end, int32_t* bad_index,
                      int32_t start_cost, const int32_t* cta_weights) {
  if (batch < 0 || tile_tokens <= 0 || num_ctas <= 0 || capacity_tokens < 0 || start_cost < 0) return DAO_ERR_ARG;
  if (cta_weights)
    for (int32_t c = 0; c < num_ctas; ++c)
      if (cta_weights[c] < 1 || cta_weights[c] > 65536) return DAO_ERR_ARG;
  req_tile_prefix[0] = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = tiles_of(seq_lens[b], tile_tokens, capacity_tokens);
    req_tile_prefix[b + 1] = req_tile_prefix[b] + (int32_t)(n > 0 ? n + start_cost : 0);
  }
  const int64_t U = req_tile_prefix[batch];
  const int64_t C = num_ctas;
  *num_units = (int32_t)U;
  *bad_index = first_bad_length(batch, seq_lens, capacity_tokens);

  /* weighted ranges: first[c] for c = 0..C, walked with the units */
  int64_t* first = NULL;
  const int weighted = cta_weights != NULL && U >= C;
  if (weighted) {
    first = (int64_t*)malloc((size_t)(C + 1) * sizeof(int64_t));
    if (!first) return DAO_ERR_ARG;
    int64_t W = 0;
    for (int64_t c = 0; c < C; ++c) W += cta_weights[c];
    int64_t Wc = 0;
    for (int64_t c = 0; c <= C; ++c) {
      first[c] = c + (U - C) * Wc / W;
      if (c < C) Wc += cta_weights[c];
    }
  }

  int32_t S = 0;
  int32_t r = 0;
  int32_t cw = 0; /* weighted: the CTA whose range holds unit u */
  int32_t prev_r = -1, prev_c = -1;
  for (int64_t u = 0; u < U; ++u) {
    while (req_tile_prefix[r + 1] <= u) ++r; /* request owning unit u */
    if (weighted)
      while (first[cw + 1] <= u) ++cw;
    const int64_t t = u - req_tile_prefix[r] - start_cost; /* its tile, or < 0 for a start unit */
    if (t < 0) continue;
    const int32_t c = weighted ? cw : (int32_t)(((u + 1) * C - 1) / U);
    if (r != prev_r || c != prev_c) {
      if (S >= max_segments) {
        free(first);
        return DAO_ERR_CAPACITY;
      }
      seg_req[S] = r;
      seg_cta[S] = c;
      seg_tile_begin[S] = (int32_t)t;
      ++S;
      prev_r = r;
      prev_c = c;
    }
    seg_tile_end[S - 1] = (int32_t)(t + 1);
  }
  free(first);
  *num_segments = S;
  /* req_seg_begin[b] = #segments of requests < b;  cta_seg_begin[c] = #segments of CTAs < c. */
  for (int32_t b = 0; b <= batch; ++b) {
    int32_t count = 0;
    for (int32_t s = 0; s < S; ++s) count += (seg_req[s] < b);
    req_seg_begin[b] = count;
  }
  for (int32_t c = 0; c <= num_ctas; ++c) {
    int32_t count = 0;
    for (int32_t s = 0; s < S; ++s) count += (seg_cta[s] < c);
    cta_seg_begin[c] = count;
  }
  return *bad_index >= 0 ? DAO_ERR_BAD_SEQLEN : DAO_OK;
}

/* The even split (no weights). */
int dao_plan_start_cost(int32_t batch, const int32_t* seq_lens, int32_t tile_tokens, int32_t num_ctas,
                        int64_t capacity_tokens, int32_t max_segments, int32_t* num_units,
                        int32_t* num_segments, int32_t* req_tile_prefix, int32_t* req_seg_begin,
                        int32_t* cta_seg_begin, int32_t* seg_req, int32_t* seg_cta,
                        int32_t* seg_tile_begin, int32_t* seg_tile_end, int32_t* bad_index,
                        int32_t start_cost) {
  return dao_plan_weighted(batch, seq_lens, tile_tokens, num_ctas, capacity_tokens, max_segments, num_units,
                           num_segments, req_tile_prefix, req_seg_begin, cta_seg_begin, seg_req, seg_cta,
                           seg_tile_begin, seg_tile_end, bad_index, start_cost, NULL);
}

/* The plan without start units (sigma = 0): every unit is a tile. */
int dao_plan(int32_t batch, const int32_t* seq_lens, int32_t tile_tokens, int32_t num_ctas,
             int64_t capacity_tokens, int32_t max_segments, int32_t* num_units,
             int32_t* num_segments, int32_t* req_tile_prefix, int32_t* req_seg_begin,
             int32_t* cta_seg_begin, int32_t* seg_req, int32_t* seg_cta,
             int32_t* seg_tile_begin, int32_t* seg_tile_end, int32_t* bad_index) {
  return dao_plan_start_cost(batch, seq_lens, tile_tokens, num_ctas, capacity_tokens, max_segments, num_units,
                             num_segments, req_tile_prefix, req_seg_begin, cta_seg_begin, seg_req, seg_cta,
                             seg_tile_begin, seg_tile_end, bad_index, 0);
}

/*
 * Static split-k plan (the comparator): every request gets the same number S
 * of equal splits, sized by the longest request.
 *   maxT  = ceil(max_b L_b / T)   (bad lengths count as 0)
 *   chunk = ceil(maxT / S)        tiles per split
 *   segment b*S + s: request b, CTA b*S + s,
 *     tiles [min(s*chunk, n_b), min((s+1)*chunk, n_b))  -- empty when s*chunk >= n_b
 * Same output arrays as dao_plan; num_ctas = B*S, max_segments >= B*S.
 */
int dao_static_plan(int32_t batch, const int32_t* seq_lens, int32_t tile_tokens, int32_t splits,
                    int64_t capacity_tokens, int32_t max_segments, int32_t* num_units,
                    int32_t* num_segments, int32_t* req_tile_prefix, int32_t* req_seg_begin,
                    int32_t* cta_seg_begin, int32_t* seg_req, int32_t* seg_cta,
                    int32_t* seg_tile_begin, int32_t* seg_tile_end, int32_t* bad_index) {
  if (batch < 0 || tile_tokens <= 0 || splits <= 0 || capacity_tokens < 0) return DAO_ERR_ARG;
  if ((int64_t)batch * splits > max_segments) return DAO_ERR_CAPACITY;
  int64_t max_tiles = 0;
  req_tile_prefix[0] = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = tiles_of(seq_lens[b], tile_tokens, capacity_tokens);
    req_tile_prefix[b + 1] = req_tile_prefix[b] + (int32_t)n;
    if (n > max_tiles) max_tiles = n;
  }
  *num_units = req_tile_prefix[batch];
  *bad_index = first_bad_length(batch, seq_lens, capacity_tokens);
  const int64_t chunk = (max_tiles + splits - 1) / splits;
  for (int32_t b = 0; b < batch; ++b) {
    const int64_t n = req_tile_prefix[b + 1] - req_tile_prefix[b];
    for (int32_t s = 0; s < splits; ++s) {
      const int64_t i = (int64_t)b * splits + s;
      const int64_t lo = s * chunk, hi = (s + 1) * chunk;
      seg_req[i] = b;
      seg_cta[i] = (int32_t)i;
      seg_tile_begin[i] = (int32_t)(lo < n ? lo : n);
      seg_tile_end[i] = (int32_t)(hi < n ? hi : n);
    }
  }
  *num_segments = batch * splits;
  for (int32_t b = 0; b <= batch; ++b) req_seg_begin[b] = b * splits;
  for (int32_t c = 0; c <= batch * splits; ++c) cta_seg_begin[c] = c;
  return *bad_index >= 0 ? DAO_ERR_BAD_SEQLEN : DAO_OK;
}
