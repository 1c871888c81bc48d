/*
 * CPU oracle for the CSA2 decode step, in plain C -- TEST INFRASTRUCTURE ONLY.
 *
 * A second, independent restatement of what the CSA2 decode path computes
 * (the first is the numpy package beside this directory; the two share no
 * code).  Only the tests and the benchmark's CPU baseline call it; it never
 * touches the CUDA library.  Every rounding below is written as its plain
 * definition -- the nearest point of a finite grid, found by scanning the
 * whole grid -- and every loop runs in the order the definitions state; no
 * blocking, no fusion, no reordering.  Compile with -ffp-contract=off so that
 * no multiply-add is fused.
 *
 * Sources (the pages' statements; the readings where they are silent are the
 * ones the numpy oracle's docstrings list):
 *  * FP4 main KV: E2M1 codes with one E4M3 scale per 16 channels, NVFP4
 *    without the global scale (agentnet.co.il, "DeepSeek V4.1-Flash" launch
 *    article, section on FP4 quantisation and layout; ai-wave.ru, "DeepSeek
 *    V4.1-Flash: 1M context, FP4 KV cache", fourth paragraph).  The element
 *    values are the OCP microscaling format definitions.  Readings: scale =
 *    the E4M3 value nearest to amax / 6, code = the E2M1 magnitude nearest to
 *    |x| / scale, both ties to the even code and saturating; a zero scale
 *    stores code 0; a negative value keeps its sign bit; channel 2j in the low
 *    nibble of byte j; 256 code bytes then 32 scale bytes = 288 B per token.
 *  * Indexer (agentnet.co.il, same article, section "CSA2: compression along
 *    the layer axis"): Full selects 512 fresh indices; Reindex ranks the Full
 *    layer's keys with its own query; the decoder's hierarchical indexer builds
 *    a pool of up to 16,384 positions = 2,048 blocks of 8.  Readings: score =
 *    sum_h w_h max(0, q_h . k) in fp32 (dims ascending, then heads ascending);
 *    block key = bf16 of the fp32 mean of the block's present keys; ranking
 *    by score descending, then position ascending; sets listed ascending,
 *    padded with -1; the pool only when the context has more than 2,048
 *    blocks.
 *  * Attention (ai-wave.ru, second paragraph; agentnet.co.il, section on the
 *    halved prefill): 512 selected positions joined with the 128-token
 *    sliding window, each position once; K = V = the decoded rows; exact
 *    softmax of sm_scale q . k in fp64.
 *  * Layer modes (same section): Full runs the indexer; Reindex ranks the
 *    Full layer's pool with its own query; Reuse keeps the latest set.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define D_LAT 512
#define GROUP 16
#define N_GROUPS (D_LAT / GROUP)
#define CODE_BYTES (D_LAT / 2)
#define ROW_BYTES (CODE_BYTES + N_GROUPS)
#define IDX_HEADS 4
#define IDX_DIM 64
#define BLOCK 8
#define POOL_BLOCKS 2048
#define TOP_K 512
#define WINDOW 128
#define REPLAY 128

/* ---------------- number formats ---------------- */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa; no inf/NaN. */
double csa2o_e2m1_value(int code) {
  const int e = (code >> 1) & 3, m = code & 1;
  const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return (code & 8) ? -mag : mag;
}

/* E4M3 (FN): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa;
 * S.1111.111 is NaN, no inf. */
double csa2o_e4m3_value(int byte) {
  const int e = (byte >> 3) & 15, m = byte & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return (byte & 0x80) ? -mag : mag;
}

static float bf16_to_float(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* float -> bf16 bits, round to nearest, ties to even (NaN stays NaN). */
static uint16_t float_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
  const uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7FFFu + lsb) >> 16);
}

/* ---------------- FP4 codec ---------------- */

/* Index of the grid value nearest to t (grid ascending, n points); on a tie
 * the even index.  Past either end the nearest end point.  The caller passes
 * values whose differences are exact in double. */
static int nearest_even(double t, const double* grid, int n) {
  int best = 0;
  double bd = fabs(t - grid[0]);
  for (int i = 1; i < n; ++i) {
    const double d = fabs(t - grid[i]);
    if (d < bd || (d == bd && (i & 1) == 0)) {
      best = i;
      bd = d;
    }
  }
  return best;
}

/* Encode one row of 512 exact float values into a 288-byte cache row. */
static void encode_row(const float* x, uint8_t* row) {
  double scale6[127], mag[8];
  for (int c = 0; c < 127; ++c) scale6[c] = 6.0 * csa2o_e4m3_value(c);   /* amax vs 6 x scale: exact */
  for (int c = 0; c < 8; ++c) mag[c] = csa2o_e2m1_value(c);
  uint8_t code[D_LAT];
  for (int g = 0; g < N_GROUPS; ++g) {
    double amax = 0.0;
    for (int j = 0; j < GROUP; ++j) {
      const double v = fabs((double)x[g * GROUP + j]);
      if (v > amax) amax = v;
    }
    const int sc = nearest_even(amax, scale6, 127);
    const double s = csa2o_e4m3_value(sc);
    row[CODE_BYTES + g] = (uint8_t)sc;
    double grid[8];
    for (int c = 0; c < 8; ++c) grid[c] = s * mag[c];   /* fp32 |x| vs scale x magnitude: exact in double */
    for (int j = 0; j < GROUP; ++j) {
      const float v = x[g * GROUP + j];
      int cd = 0;
      if (s != 0.0) cd = nearest_even(fabs((double)v), grid, 8) | (signbit(v) ? 8 : 0);
      code[g * GROUP + j] = (uint8_t)cd;
    }
  }
  for (int j = 0; j < CODE_BYTES; ++j) row[j] = (uint8_t)(code[2 * j] | (code[2 * j + 1] << 4));
}

/* Encode rows of 512 bf16 channels into 288-byte cache rows. */
void csa2o_encode_rows(const uint16_t* kv, int64_t n, uint8_t* out) {
  float x[D_LAT];
  for (int64_t r = 0; r < n; ++r) {
    for (int c = 0; c < D_LAT; ++c) x[c] = bf16_to_float(kv[r * D_LAT + c]);
    encode_row(x, out + r * ROW_BYTES);
  }
}

/* Entries at compression ratio 1 or 2: entry e is made of raw bf16 rows
 * [compress e, compress e + compress); at ratio 2 its value per channel is
 * fl32(fl32(a + b) x 0.5) (mean of the pair, the reading for the encoder's
 * compressed layers), encoded like a row. */
static void entry_values(const uint16_t* raw, int64_t e, int compress, int width, float* x) {
  for (int c = 0; c < width; ++c) {
    if (compress == 1) {
      x[c] = bf16_to_float(raw[e * width + c]);
    } else {
      const float a = bf16_to_float(raw[(2 * e) * width + c]), b = bf16_to_float(raw[(2 * e + 1) * width + c]);
      const float sum = a + b;
      x[c] = sum * 0.5f;
    }
  }
}

void csa2o_encode_entries(const uint16_t* raw, int64_t n, int compress, uint8_t* out) {
  float x[D_LAT];
  for (int64_t e = 0; e < n; ++e) {
    entry_values(raw, e, compress, D_LAT, x);
    encode_row(x, out + e * ROW_BYTES);
  }
}

/* Stored indexer keys of entries: the raw key at ratio 1, bf16 of the pair
 * mean at ratio 2. */
void csa2o_key_entries(const uint16_t* raw, int64_t n, int compress, uint16_t* out) {
  float x[IDX_DIM];
  for (int64_t e = 0; e < n; ++e) {
    entry_values(raw, e, compress, IDX_DIM, x);
    for (int d = 0; d < IDX_DIM; ++d) out[e * IDX_DIM + d] = float_to_bf16(x[d]);
  }
}

/* Decode 288-byte rows into fp64 values [n][512] (exact products). */
void csa2o_decode_rows(const uint8_t* rows, int64_t n, double* out) {
  for (int64_t r = 0; r < n; ++r) {
    const uint8_t* row = rows + r * ROW_BYTES;
    for (int c = 0; c < D_LAT; ++c) {
      const int byte = row[c / 2];
      const int cd = (c & 1) ? byte >> 4 : byte & 15;
      out[r * D_LAT + c] = csa2o_e2m1_value(cd) * csa2o_e4m3_value(row[CODE_BYTES + c / GROUP]);
    }
  }
}

/* ---------------- indexer ---------------- */

/* Block keys (bf16 bits [ceil(L/8)][64]) of the first L stored keys. */
void csa2o_block_keys(const uint16_t* keys, int64_t L, uint16_t* out) {
  const int64_t nb = (L + BLOCK - 1) / BLOCK;
  for (int64_t b = 0; b < nb; ++b) {
    const int64_t t0 = b * BLOCK, t1 = t0 + BLOCK < L ? t0 + BLOCK : L;
    for (int d = 0; d < IDX_DIM; ++d) {
      float acc = 0.0f, cnt = 0.0f;
      for (int64_t t = t0; t < t1; ++t) {
        acc = acc + bf16_to_float(keys[t * IDX_DIM + d]);
        cnt = cnt + 1.0f;
      }
      out[b * IDX_DIM + d] = float_to_bf16(acc / cnt);
    }
  }
}

/* score of one key: sum over heads of w_h max(0, q_h . k), fp32 in order. */
static float score_one(const uint16_t* q, const float* w, const uint16_t* k) {
  float total = 0.0f;
  for (int h = 0; h < IDX_HEADS; ++h) {
    float dot = 0.0f;
    for (int d = 0; d < IDX_DIM; ++d) {
      const float p = bf16_to_float(q[h * IDX_DIM + d]) * bf16_to_float(k[d]);
      dot = dot + p;
    }
    const float relu = dot > 0.0f ? dot : 0.0f;
    const float wh = w ? w[h] : 1.0f;
    const float t = wh * relu;
    total = total + t;
  }
  return total;
}

/* Scores [n] of query q [4][64] against keys [n][64] (w: 4 head weights or NULL). */
void csa2o_scores(const uint16_t* q, const float* w, const uint16_t* keys, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = score_one(q, w, keys + i * IDX_DIM);
}

typedef struct {
  float s;
  int64_t i;
} scored;

static int by_rank(const void* a, const void* b) {   /* score descending, then index ascending */
  const scored* x = (const scored*)a;
  const scored* y = (const scored*)b;
  if (x->s > y->s) return -1;
  if (x->s < y->s) return 1;
  return x->i < y->i ? -1 : (x->i > y->i ? 1 : 0);
}

static int by_value(const void* a, const void* b) {
  const int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
  return x < y ? -1 : (x > y ? 1 : 0);
}

/* The k best of n entries by (score desc, index asc), listed ascending,
 * padded with -1.  Returns the count selected. */
int64_t csa2o_topk(const float* scores, int64_t n, int64_t k, int64_t* out) {
  scored* v = (scored*)malloc((size_t)(n > 0 ? n : 1) * sizeof(scored));
  for (int64_t i = 0; i < n; ++i) {
    v[i].s = scores[i];
    v[i].i = i;
  }
  qsort(v, (size_t)n, sizeof(scored), by_rank);
  const int64_t m = n < k ? n : k;
  for (int64_t j = 0; j < m; ++j) out[j] = v[j].i;
  qsort(out, (size_t)m, sizeof(int64_t), by_value);
  for (int64_t j = m; j < k; ++j) out[j] = -1;
  free(v);
  return m;
}

/* Top-k positions among the candidate positions cand [ncand] (ascending). */
static void select_tokens(const uint16_t* q, const float* w, const uint16_t* keys, const int64_t* cand,
                          int64_t ncand, int64_t* idx) {
  float* s = (float*)malloc((size_t)(ncand > 0 ? ncand : 1) * sizeof(float));
  int64_t* sel = (int64_t*)malloc(TOP_K * sizeof(int64_t));
  for (int64_t i = 0; i < ncand; ++i) s[i] = score_one(q, w, keys + cand[i] * IDX_DIM);
  csa2o_topk(s, ncand, TOP_K, sel);
  for (int j = 0; j < TOP_K; ++j) idx[j] = sel[j] >= 0 ? cand[sel[j]] : -1;
  free(sel);
  free(s);
}

/* Token positions of the pool's blocks below L, ascending (pool ascending). */
static int64_t pool_tokens(const int64_t* pool, int64_t npool, int64_t L, int64_t* cand) {
  int64_t n = 0;
  for (int64_t j = 0; j < npool; ++j) {
    if (pool[j] < 0) continue;
    for (int t = 0; t < BLOCK; ++t) {
      const int64_t p = pool[j] * BLOCK + t;
      if (p < L) cand[n++] = p;
    }
  }
  return n;
}

/* Full layer over the first L keys: the pool [2048] (ascending block ids, -1
 * padded) and the selected positions [512].  Hierarchical: the pool is the
 * top 2,048 blocks by block-key score when there are more than 2,048 blocks,
 * else every block. */
void csa2o_full_indexer(const uint16_t* q, const float* w, const uint16_t* keys, int64_t L, int64_t* pool,
                        int64_t* idx) {
  const int64_t nb = (L + BLOCK - 1) / BLOCK;
  if (nb > POOL_BLOCKS) {
    uint16_t* kb = (uint16_t*)malloc((size_t)nb * IDX_DIM * sizeof(uint16_t));
    float* bs = (float*)malloc((size_t)nb * sizeof(float));
    csa2o_block_keys(keys, L, kb);
    csa2o_scores(q, w, kb, nb, bs);
    csa2o_topk(bs, nb, POOL_BLOCKS, pool);
    free(bs);
    free(kb);
  } else {
    for (int64_t j = 0; j < POOL_BLOCKS; ++j) pool[j] = j < nb ? j : -1;
  }
  int64_t* cand = (int64_t*)malloc((size_t)POOL_BLOCKS * BLOCK * sizeof(int64_t));
  const int64_t ncand = pool_tokens(pool, POOL_BLOCKS, L, cand);
  select_tokens(q, w, keys, cand, ncand, idx);
  free(cand);
}

/* Reindex layer: this layer's query ranks the tokens of the Full layer's pool. */
void csa2o_reindex_indexer(const uint16_t* q, const float* w, const uint16_t* keys, int64_t L,
                           const int64_t* pool, int64_t* idx) {
  int64_t* cand = (int64_t*)malloc((size_t)POOL_BLOCKS * BLOCK * sizeof(int64_t));
  const int64_t ncand = pool_tokens(pool, POOL_BLOCKS, L, cand);
  select_tokens(q, w, keys, cand, ncand, idx);
  free(cand);
}

/* Flat indexer (encoder Full layer): the top 512 of positions [0, visible). */
void csa2o_flat_indexer(const uint16_t* q, const float* w, const uint16_t* keys, int64_t visible, int64_t* idx) {
  int64_t* cand = (int64_t*)malloc((size_t)(visible > 0 ? visible : 1) * sizeof(int64_t));
  for (int64_t p = 0; p < visible; ++p) cand[p] = p;
  select_tokens(q, w, keys, cand, visible, idx);
  free(cand);
}

/* ---------------- attention ---------------- */

/* Selected positions (>= 0) joined with the window [max(0, L-128), L),
 * ascending, each once.  pos must hold TOP_K + WINDOW entries.  Returns the
 * count, or -1 if a selected position is not below L. */
int64_t csa2o_attended_positions(const int64_t* idx, int64_t L, int64_t* pos) {
  int64_t n = 0;
  for (int j = 0; j < TOP_K; ++j) {
    if (idx[j] < 0) continue;
    if (idx[j] >= L) return -1;
    pos[n++] = idx[j];
  }
  for (int64_t p = L > WINDOW ? L - WINDOW : 0; p < L; ++p) pos[n++] = p;
  qsort(pos, (size_t)n, sizeof(int64_t), by_value);
  int64_t u = 0;
  for (int64_t j = 0; j < n; ++j)
    if (u == 0 || pos[j] != pos[u - 1]) pos[u++] = pos[j];
  return u;
}

/* Exact softmax attention of q [H][512] (bf16 bits) over rows [T][512]
 * (fp64): out[h] = sum_t p_ht row_t, p_h = softmax_t(sm_scale q_h . row_t).
 * T = 0 gives zeros. */
void csa2o_attend(const uint16_t* q, int heads, const double* rows, int64_t T, double sm_scale, double* out) {
  double* s = (double*)malloc((size_t)(T > 0 ? T : 1) * sizeof(double));
  for (int h = 0; h < heads; ++h) {
    double* o = out + (int64_t)h * D_LAT;
    for (int c = 0; c < D_LAT; ++c) o[c] = 0.0;
    if (T == 0) continue;
    double m = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      double dot = 0.0;
      for (int c = 0; c < D_LAT; ++c) dot += (double)bf16_to_float(q[h * D_LAT + c]) * rows[t * D_LAT + c];
      s[t] = sm_scale * dot;
      if (s[t] > m) m = s[t];
    }
    double z = 0.0;
    for (int64_t t = 0; t < T; ++t) {
      s[t] = exp(s[t] - m);
      z += s[t];
    }
    for (int64_t t = 0; t < T; ++t) {
      const double p = s[t] / z;
      for (int c = 0; c < D_LAT; ++c) o[c] += p * rows[t * D_LAT + c];
    }
  }
  free(s);
}

/* ---------------- decode steps over host threads ---------------- */

/* The seeded input generator (the shared input module's host library) draws
 * a sequence's bf16 KV rows: this is its fill function's signature. */
typedef void (*csa2o_gen_fn)(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, float scale,
                             const float* col_scale, uint32_t ncols, uint16_t* out, int nthreads);

typedef struct {
  int nlayers;
  const char* modes;          /* per layer: 'F' Full, 'I' Reindex, 'R' Reuse */
  int heads;
  double sm_scale;
  uint64_t seed;              /* generator seed and the KV rows' column scales */
  const float* kv_col_scale;  /* [512] */
  csa2o_gen_fn gen;
} csa2o_schedule;

typedef struct {
  int64_t L;                  /* context length; the appended token is position L - 1 */
  const uint16_t* keys;       /* [L][64] stored indexer keys */
  const uint16_t* idxq;       /* [nlayers][4][64] indexer queries (Full / Reindex layers) */
  const uint16_t* q;          /* [nlayers][heads][512] attention queries */
  const uint16_t* new_row;    /* [512] the appended token's KV */
  uint64_t kv_stream;         /* generator stream of this sequence's KV rows */
  uint16_t* row_cache;        /* [L][512] KV rows drawn so far (caller memory) */
  uint8_t* drawn;             /* [L] 1 once row_cache holds the row */
  int64_t* idx;               /* [nlayers][512] out: each layer's index set */
  double* out;                /* [nlayers][heads][512] out: each layer's attention */
  int status;                 /* out: 0, or -1 for a bad schedule or position */
} csa2o_sequence;

/* One decode step of one sequence: encode the appended token, then the layer
 * schedule; each layer attends over its set's decoded rows (decoded once per
 * set: Reuse layers attend over the rows their set's layer decoded). */
static int decode_step(const csa2o_schedule* sc, csa2o_sequence* sq) {
  uint8_t enc[ROW_BYTES];
  csa2o_encode_rows(sq->new_row, 1, enc);
  int64_t pool[POOL_BLOCKS], latest[TOP_K], pos[TOP_K + WINDOW];
  int have_pool = 0, have_set = 0, fresh = 0;
  int64_t T = 0;
  uint8_t* rows8 = (uint8_t*)malloc((TOP_K + WINDOW) * ROW_BYTES);
  double* rows = (double*)malloc((size_t)(TOP_K + WINDOW) * D_LAT * sizeof(double));
  int st = 0;
  for (int l = 0; l < sc->nlayers && st == 0; ++l) {
    const char m = sc->modes[l];
    const uint16_t* iq = sq->idxq + (int64_t)l * IDX_HEADS * IDX_DIM;
    if (m == 'F') {
      csa2o_full_indexer(iq, NULL, sq->keys, sq->L, pool, latest);
      have_pool = have_set = fresh = 1;
    } else if (m == 'I') {
      if (!have_pool) {
        st = -1;
        break;
      }
      csa2o_reindex_indexer(iq, NULL, sq->keys, sq->L, pool, latest);
      have_set = fresh = 1;
    } else if (m != 'R' || !have_set) {
      st = -1;
      break;
    }
    if (fresh) {
      T = csa2o_attended_positions(latest, sq->L, pos);
      if (T < 0) {
        st = -1;
        break;
      }
      for (int64_t t = 0; t < T; ++t) {   /* the cache rows of the set: drawn once, encoded, decoded */
        const int64_t p = pos[t];
        if (!sq->drawn[p]) {
          sc->gen(sc->seed, sq->kv_stream, (uint64_t)p * D_LAT, D_LAT, 1.0f, sc->kv_col_scale, D_LAT,
                  sq->row_cache + p * D_LAT, 1);
          sq->drawn[p] = 1;
        }
        csa2o_encode_rows(sq->row_cache + p * D_LAT, 1, rows8 + t * ROW_BYTES);
      }
      csa2o_decode_rows(rows8, T, rows);
      fresh = 0;
    }
    memcpy(sq->idx + (int64_t)l * TOP_K, latest, sizeof(latest));
    csa2o_attend(sq->q + (int64_t)l * sc->heads * D_LAT, sc->heads, rows, T, sc->sm_scale,
                 sq->out + (int64_t)l * sc->heads * D_LAT);
  }
  free(rows);
  free(rows8);
  return st;
}

typedef struct {
  const csa2o_schedule* sc;
  csa2o_sequence* seqs;
  int nseq, first, stride;
} worker_arg;

static void* worker(void* p) {
  worker_arg* a = (worker_arg*)p;
  for (int i = a->first; i < a->nseq; i += a->stride) a->seqs[i].status = decode_step(a->sc, &a->seqs[i]);
  return NULL;
}

/* One decode step of every sequence, sequences dealt round-robin to
 * `nthreads` host threads.  Returns 0, or -1 if any sequence failed. */
int csa2o_decode_steps(const csa2o_schedule* sc, csa2o_sequence* seqs, int nseq, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nseq) nthreads = nseq > 0 ? nseq : 1;
  pthread_t* th = (pthread_t*)malloc((size_t)nthreads * sizeof(pthread_t));
  worker_arg* args = (worker_arg*)malloc((size_t)nthreads * sizeof(worker_arg));
  for (int t = 0; t < nthreads; ++t) {
    args[t].sc = sc;
    args[t].seqs = seqs;
    args[t].nseq = nseq;
    args[t].first = t;
    args[t].stride = nthreads;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, worker, &args[t]);
  worker(&args[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  int st = 0;
  for (int i = 0; i < nseq; ++i)
    if (seqs[i].status) st = -1;
  free(args);
  free(th);
  return st;
}

/* ---------------- prefill queries and ragged steps over host threads ---------------- */

/* Encoder prefill at compression ratio `compress`: the stored keys and the raw
 * bf16 KV rows of the whole sequence are given. */
typedef struct {
  int nlayers;
  int heads;
  double sm_scale;
  int compress;
  int64_t n_entries;
  const uint16_t* keys;       /* [n_entries][64] stored keys */
  const uint16_t* raw_kv;     /* [compress x n_entries][512] raw bf16 rows */
} csa2o_prefill;

typedef struct {
  int64_t P;                  /* raw position of the query */
  const uint16_t* iq;         /* [4][64] indexer query */
  const uint16_t* q;          /* [nlayers][heads][512] attention queries */
  int64_t* idx;               /* [512] out */
  double* out;                /* [nlayers][heads][512] out */
} csa2o_prefill_query;

/* One prefill query: it sees entries [0, (P + 1) / compress); the flat indexer
 * selects over them; every layer of the group (Full, then Reuse) attends over
 * the same set, its rows encoded from the raw rows and decoded. */
static void prefill_query(const csa2o_prefill* pf, csa2o_prefill_query* pq) {
  const int64_t v = (pq->P + 1) / pf->compress;
  int64_t pos[TOP_K + WINDOW];
  csa2o_flat_indexer(pq->iq, NULL, pf->keys, v, pq->idx);
  const int64_t T = csa2o_attended_positions(pq->idx, v, pos);
  uint8_t* rows8 = (uint8_t*)malloc((TOP_K + WINDOW) * ROW_BYTES);
  double* rows = (double*)malloc((size_t)(TOP_K + WINDOW) * D_LAT * sizeof(double));
  float x[D_LAT];
  for (int64_t t = 0; t < T; ++t) {
    entry_values(pf->raw_kv, pos[t], pf->compress, D_LAT, x);
    encode_row(x, rows8 + t * ROW_BYTES);
  }
  csa2o_decode_rows(rows8, T, rows);
  for (int l = 0; l < pf->nlayers; ++l)
    csa2o_attend(pq->q + (int64_t)l * pf->heads * D_LAT, pf->heads, rows, T, pf->sm_scale,
                 pq->out + (int64_t)l * pf->heads * D_LAT);
  free(rows);
  free(rows8);
}

typedef struct {
  const csa2o_prefill* pf;
  csa2o_prefill_query* qs;
  int n, first, stride;
  /* append ranges */
  const uint16_t* raw_k;
  uint8_t* rows_out;
  uint16_t* keys_out;
  int64_t e0, e1;
} prefill_arg;

static void* prefill_worker(void* p) {
  prefill_arg* a = (prefill_arg*)p;
  for (int i = a->first; i < a->n; i += a->stride) prefill_query(a->pf, &a->qs[i]);
  return NULL;
}

static void* append_worker(void* p) {
  prefill_arg* a = (prefill_arg*)p;
  const int c = a->pf->compress;
  if (a->e1 > a->e0) {
    csa2o_encode_entries(a->pf->raw_kv + a->e0 * c * D_LAT, a->e1 - a->e0, c, a->rows_out + a->e0 * ROW_BYTES);
    csa2o_key_entries(a->raw_k + a->e0 * c * IDX_DIM, a->e1 - a->e0, c, a->keys_out + a->e0 * IDX_DIM);
  }
  return NULL;
}

static void run_threads(void* (*fn)(void*), prefill_arg* args, int nthreads) {
  pthread_t* th = (pthread_t*)malloc((size_t)nthreads * sizeof(pthread_t));
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, fn, &args[t]);
  fn(&args[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(th);
}

/* The sampled prefill queries, dealt round-robin to host threads. */
void csa2o_prefill_queries(const csa2o_prefill* pf, csa2o_prefill_query* qs, int nq, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nq) nthreads = nq > 0 ? nq : 1;
  prefill_arg* args = (prefill_arg*)calloc((size_t)nthreads, sizeof(prefill_arg));
  for (int t = 0; t < nthreads; ++t) {
    args[t].pf = pf;
    args[t].qs = qs;
    args[t].n = nq;
    args[t].first = t;
    args[t].stride = nthreads;
  }
  run_threads(prefill_worker, args, nthreads);
  free(args);
}

/* The whole append of a prefill: every entry encoded (rows_out [n_entries][288])
 * and its key stored (keys_out [n_entries][64]), entry ranges split over host
 * threads. */
void csa2o_prefill_append(const csa2o_prefill* pf, const uint16_t* raw_k, uint8_t* rows_out, uint16_t* keys_out,
                          int nthreads) {
  if (nthreads < 1) nthreads = 1;
  prefill_arg* args = (prefill_arg*)calloc((size_t)nthreads, sizeof(prefill_arg));
  for (int t = 0; t < nthreads; ++t) {
    args[t].pf = pf;
    args[t].raw_k = raw_k;
    args[t].rows_out = rows_out;
    args[t].keys_out = keys_out;
    args[t].e0 = pf->n_entries * t / nthreads;
    args[t].e1 = pf->n_entries * (t + 1) / nthreads;
  }
  run_threads(append_worker, args, nthreads);
  free(args);
}

/* Ragged decode with bounded replay (one layer per sequence): a sequence
 * flagged as a cache miss re-encodes its last min(128, L) entries from the
 * supplied raw rows, any other its newest entry (its stored keys at ratio 1 are
 * the raw keys); a Reindex sequence ranks the Full layer's pool with its own
 * query, a Reuse one keeps the Full layer's set; then it attends. */
typedef struct {
  int64_t L;
  int reindex;                /* 1: Reindex, 0: Reuse */
  int miss;
  const uint16_t* kv_last;    /* [128][512] raw rows behind the last 128 entries */
  const uint16_t* keys;       /* [L][64] */
  const int64_t* pool;        /* [2048] the Full layer's pool */
  const int64_t* set;         /* [512] the Full layer's set (Reuse) */
  const uint16_t* iq;         /* [4][64] (Reindex) */
  const uint16_t* q;          /* [heads][512] */
  uint64_t kv_stream;
  uint16_t* row_cache;        /* [L][512] */
  uint8_t* drawn;             /* [L] */
  int64_t* idx;               /* [512] out */
  double* out;                /* [heads][512] out */
  uint8_t* replayed;          /* [128][288] out: the re-encoded entries, oldest first */
  int64_t nreplayed;          /* out: how many */
} csa2o_ragged_sequence;

static void ragged_step(const csa2o_schedule* sc, csa2o_ragged_sequence* sq) {
  const int64_t n = sq->miss ? (sq->L < REPLAY ? sq->L : REPLAY) : (sq->L > 0 ? 1 : 0);
  uint8_t* rows8 = (uint8_t*)malloc((TOP_K + WINDOW) * ROW_BYTES);
  csa2o_encode_rows(sq->kv_last + (REPLAY - n) * D_LAT, n, sq->replayed);   /* the replayed entries */
  sq->nreplayed = n;
  if (sq->reindex)
    csa2o_reindex_indexer(sq->iq, NULL, sq->keys, sq->L, sq->pool, sq->idx);
  else
    memcpy(sq->idx, sq->set, TOP_K * sizeof(int64_t));
  int64_t pos[TOP_K + WINDOW];
  const int64_t T = csa2o_attended_positions(sq->idx, sq->L, pos);
  double* rows = (double*)malloc((size_t)(TOP_K + WINDOW) * D_LAT * sizeof(double));
  for (int64_t t = 0; t < T; ++t) {
    const int64_t p = pos[t];
    if (!sq->drawn[p]) {
      sc->gen(sc->seed, sq->kv_stream, (uint64_t)p * D_LAT, D_LAT, 1.0f, sc->kv_col_scale, D_LAT,
              sq->row_cache + p * D_LAT, 1);
      sq->drawn[p] = 1;
    }
    csa2o_encode_rows(sq->row_cache + p * D_LAT, 1, rows8 + t * ROW_BYTES);
  }
  csa2o_decode_rows(rows8, T > 0 ? T : 0, rows);
  csa2o_attend(sq->q, sc->heads, rows, T > 0 ? T : 0, sc->sm_scale, sq->out);
  free(rows);
  free(rows8);
}

typedef struct {
  const csa2o_schedule* sc;
  csa2o_ragged_sequence* seqs;
  int n, first, stride;
} ragged_arg;

static void* ragged_worker(void* p) {
  ragged_arg* a = (ragged_arg*)p;
  for (int i = a->first; i < a->n; i += a->stride) ragged_step(a->sc, &a->seqs[i]);
  return NULL;
}

/* One ragged step of every sequence on host threads (the schedule supplies
 * heads, sm_scale and the generator; its modes are not used). */
void csa2o_ragged_steps(const csa2o_schedule* sc, csa2o_ragged_sequence* seqs, int n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > n) nthreads = n > 0 ? n : 1;
  pthread_t* th = (pthread_t*)malloc((size_t)nthreads * sizeof(pthread_t));
  ragged_arg* args = (ragged_arg*)malloc((size_t)nthreads * sizeof(ragged_arg));
  for (int t = 0; t < nthreads; ++t) {
    args[t].sc = sc;
    args[t].seqs = seqs;
    args[t].n = n;
    args[t].first = t;
    args[t].stride = nthreads;
  }
  for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, ragged_worker, &args[t]);
  ragged_worker(&args[0]);
  for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
  free(args);
  free(th);
}
