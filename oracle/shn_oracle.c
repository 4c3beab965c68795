/*
 * shn_oracle.c — plain, slow, obviously correct CPU oracle of the Shannonic INT8 codec.
 *
 * TEST INFRASTRUCTURE ONLY: used by tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference arm; never by the product path. Shares no code with the CUDA implementation.
 *
 * Source of the method: "Shannonic: Efficient Entropy-Optimal Compression for ML Workloads"
 * (MLSys 2026 talk notes):
 *   §4.1  histogram h[x]; DP range selection C[i,k] = min_{j<i} C[j,k-1] + Cost(j,i-1) with
 *         backtracking from C[256,16]; per-range base/nb/start/bias, rangeId[256]; tANS table
 *         from the range probabilities p_k = N_k / N.
 *   §4.2  Algorithm 2: encode = rangeId, emit offset in nb[s] bits, emit normalisation bits,
 *         encTable transition; decode = decTable[X] gives the range and bit count, read offset,
 *         x = base[s] + o.
 * Every step the notes leave open is fixed by the SHN1 format specification; its section
 * is named beside each function.
 *
 * Plain C99 + pthreads (threads only split independent chunks / segments).
 */
#include "shn_oracle.h"

#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------------ */
/* small integer helpers                                                                       */

static int floor_log2_u64(uint64_t x) { /* x >= 1 */
  int e = 0;
  while ((x >> 1) != 0) {
    x >>= 1;
    e++;
  }
  return e;
}

static int ceil_log2_u32(uint32_t m) { /* smallest w with 2^w >= m, m >= 1 */
  int w = 0;
  while ((1u << w) < m) w++;
  return w;
}

static uint64_t round_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

/* ------------------------------------------------------------------------------------------ */
/* SHN1 format §2 — fixed-point log2 by repeated squaring of the normalised mantissa.            */

int64_t orc_lg(uint64_t n) {
  if (n == 0) return 0;
  int e = floor_log2_u64(n);
  uint64_t m = n << (31 - e); /* n < 2^32, so e <= 31 */
  int64_t frac = 0;
  for (int it = 0; it < 24; it++) {
    m = (m * m) >> 31;
    frac <<= 1;
    if (m >= (1ull << 32)) {
      frac |= 1;
      m >>= 1;
    }
  }
  return ((int64_t)e << 24) | frac;
}

/* ------------------------------------------------------------------------------------------ */
/* §4.1 histogram h[x] over the symbols u = byte ^ 0x80 (SHN1 format §1).                        */

void orc_histogram(const uint8_t* bytes, uint64_t n, uint64_t hist[256]) {
  for (int u = 0; u < 256; u++) hist[u] = 0;
  for (uint64_t i = 0; i < n; i++) hist[bytes[i] ^ 0x80]++;
}

/* ------------------------------------------------------------------------------------------ */
/* §4.1 DP range selection (SHN1 format §3). Generic alphabet size A <= 256 so that the tests can
 * compare it with a brute force over all partitions of small alphabets.                       */

int orc_partition(const uint64_t* hist, int A, int K, uint16_t* lo, int64_t* cost_out) {
  if (A < 1 || A > 256 || K < 1 || K > A) return ORC_ERR_ARG;
  uint64_t total = 0;
  for (int u = 0; u < A; u++) total += hist[u];
  if (total >= (1ull << 32)) return ORC_ERR_ARG;

  uint64_t pre[257];
  pre[0] = 0;
  for (int u = 0; u < A; u++) pre[u + 1] = pre[u] + hist[u];

  /* Cost(j, i) for the range [j, i): c*(w<<24) - c*LG(c), memoised per pair. */
  int64_t* cost = (int64_t*)malloc(sizeof(int64_t) * (size_t)(A + 1) * (size_t)(A + 1));
  int64_t* D = (int64_t*)malloc(sizeof(int64_t) * (size_t)(A + 1) * (size_t)(K + 1));
  int* arg = (int*)malloc(sizeof(int) * (size_t)(A + 1) * (size_t)(K + 1));
  if (!cost || !D || !arg) {
    free(cost);
    free(D);
    free(arg);
    return ORC_ERR_NOMEM;
  }
  for (int j = 0; j < A; j++) {
    for (int i = j + 1; i <= A; i++) {
      int64_t c = (int64_t)(pre[i] - pre[j]);
      int64_t w = ceil_log2_u32((uint32_t)(i - j));
      cost[(size_t)j * (A + 1) + i] = c * (w << 24) - c * orc_lg((uint64_t)c);
    }
  }

  const int64_t INF = INT64_MAX;
#define DD(i, k) D[(size_t)(i) * (K + 1) + (k)]
#define ARG(i, k) arg[(size_t)(i) * (K + 1) + (k)]
  for (int i = 0; i <= A; i++)
    for (int k = 0; k <= K; k++) {
      DD(i, k) = INF;
      ARG(i, k) = -1;
    }
  DD(0, 0) = 0;
  for (int k = 1; k <= K; k++) {
    for (int i = k; i <= A; i++) {
      int64_t best = INF;
      int bj = -1;
      for (int j = k - 1; j <= i - 1; j++) {
        if (DD(j, k - 1) == INF) continue;
        int64_t v = DD(j, k - 1) + cost[(size_t)j * (A + 1) + i];
        if (v < best) { /* strict: the smallest j wins ties */
          best = v;
          bj = j;
        }
      }
      DD(i, k) = best;
      ARG(i, k) = bj;
    }
  }
  if (cost_out) *cost_out = DD(A, K);
  int i = A;
  for (int k = K; k >= 1; k--) {
    int j = ARG(i, k);
    lo[k - 1] = (uint16_t)j;
    i = j;
  }
#undef DD
#undef ARG
  free(cost);
  free(D);
  free(arg);
  return ORC_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* §4.1 "tANS table from the range probabilities p_k = N_k/N": state counts (SHN1 format §4).
 * Greedy: every occupied range gets one state, then each remaining state goes to the largest
 * marginal gain N_k * (LG(f_k+1) - LG(f_k)); ties to the smallest k.                          */

int orc_normalize(const uint64_t* N, int K, int R, uint32_t* f) {
  if (K < 1 || K > 256 || R < 1 || R > 12) return ORC_ERR_ARG;
  const uint32_t L = 1u << R;
  uint64_t total = 0;
  int nonzero = 0;
  for (int k = 0; k < K; k++) {
    total += N[k];
    if (N[k] > 0) nonzero++;
  }
  if (total >= (1ull << 32)) return ORC_ERR_ARG;
  if (total == 0) {
    for (int k = 0; k < K; k++) f[k] = 0;
    f[0] = L;
    return ORC_OK;
  }
  if ((uint32_t)nonzero > L) return ORC_ERR_ARG;
  for (int k = 0; k < K; k++) f[k] = N[k] > 0 ? 1u : 0u;
  for (uint32_t step = 0; step < L - (uint32_t)nonzero; step++) {
    int best = -1;
    uint64_t best_gain = 0;
    for (int k = 0; k < K; k++) {
      if (N[k] == 0) continue;
      uint64_t gain = N[k] * (uint64_t)(orc_lg(f[k] + 1) - orc_lg(f[k]));
      if (best < 0 || gain > best_gain) {
        best = k;
        best_gain = gain;
      }
    }
    f[best]++;
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* §4.1 per-range parameters and tANS tables (SHN1 format §5).                                   */

int orc_tables_init(const uint16_t* lo, const uint32_t* f, int K, int R, orc_tables* t) {
  if (K < 1 || K > 256 || R < 4 || R > 12) return ORC_ERR_ARG;
  const int L = 1 << R;
  if (K > L) return ORC_ERR_ARG;
  memset(t, 0, sizeof(*t));
  t->K = K;
  t->R = R;
  t->L = L;
  if (lo[0] != 0) return ORC_ERR_ARG;
  for (int k = 0; k < K; k++) {
    t->lo[k] = lo[k];
    if (k > 0 && lo[k] <= lo[k - 1]) return ORC_ERR_ARG;
    if (lo[k] > 255) return ORC_ERR_ARG;
  }
  t->lo[K] = 256;
  uint32_t sum = 0;
  for (int k = 0; k < K; k++) {
    if (f[k] > (uint32_t)L) return ORC_ERR_ARG;
    t->f[k] = f[k];
    t->cumul[k] = sum;
    sum += f[k];
    t->width_bits[k] = (uint8_t)ceil_log2_u32((uint32_t)(t->lo[k + 1] - t->lo[k]));
    for (int u = t->lo[k]; u < t->lo[k + 1]; u++) t->range_of[u] = (uint8_t)k;
  }
  if (sum != (uint32_t)L) return ORC_ERR_ARG;

  /* spread: the (cumul_k + r)-th placement goes to slot ((cumul_k + r) * step) mod L */
  const uint32_t step = (uint32_t)(L / 2 + L / 8 + 3);
  for (int k = 0; k < K; k++)
    for (uint32_t r = 0; r < f[k]; r++) t->spread[((t->cumul[k] + r) * step) % (uint32_t)L] = (uint16_t)k;

  /* decode and encode tables, slots in ascending order */
  uint32_t rank[256];
  for (int k = 0; k < K; k++) rank[k] = 0;
  for (int i = 0; i < L; i++) {
    int s = t->spread[i];
    uint32_t j = rank[s]++;
    uint32_t x = f[s] + j;
    int nb = R - floor_log2_u64(x);
    t->dec_sym[i] = (uint16_t)s;
    t->dec_nb[i] = (uint8_t)nb;
    t->dec_next[i] = (uint16_t)((x << nb) - (uint32_t)L);
    t->enc[t->cumul[s] + j] = (uint16_t)(L + i);
  }
  return ORC_OK;
}

int orc_build_segment_tables(const uint64_t hist[256], int K, int R, orc_tables* t, int64_t* dp_cost) {
  uint16_t lo[256];
  uint32_t f[256];
  uint64_t N[256];
  if (K < 1 || K > 256 || R < 4 || R > 12 || K > (1 << R)) return ORC_ERR_ARG;
  int rc = orc_partition(hist, 256, K, lo, dp_cost);
  if (rc) return rc;
  for (int k = 0; k < K; k++) {
    int hi = (k + 1 < K) ? lo[k + 1] : 256;
    N[k] = 0;
    for (int u = lo[k]; u < hi; u++) N[k] += hist[u];
  }
  rc = orc_normalize(N, K, R, f);
  if (rc) return rc;
  return orc_tables_init(lo, f, K, R, t);
}

/* ------------------------------------------------------------------------------------------ */
/* Bit strings, LSB-first (SHN1 format §7).                                                       */

typedef struct {
  uint32_t* words;
  uint64_t cap_words; /* words available (one extra slack word is required for straddles) */
  uint64_t P;         /* bits appended so far */
  int overflow;
} bitwriter;

static void bw_append(bitwriter* bw, uint32_t v, int n) { /* 0 <= n <= 32, v < 2^n */
  if (n == 0) return;
  uint64_t k = bw->P >> 5;
  if (k + 1 >= bw->cap_words) {
    bw->overflow = 1;
    return;
  }
  uint64_t acc = (uint64_t)v << (bw->P & 31);
  bw->words[k] |= (uint32_t)acc;
  bw->words[k + 1] |= (uint32_t)(acc >> 32);
  bw->P += (uint64_t)n;
}

typedef struct {
  const uint32_t* words;
  uint64_t nwords;
  int64_t P; /* unread bits are positions [0, P) */
  int underflow;
} bitreader;

static uint32_t br_read(bitreader* br, int n) {
  if (n == 0) return 0;
  if ((int64_t)n > br->P) {
    br->underflow = 1;
    br->P -= n;
    return 0;
  }
  uint64_t p = (uint64_t)(br->P - n);
  uint64_t k = p >> 5;
  uint64_t acc = br->words[k];
  if (k + 1 < br->nwords) acc |= (uint64_t)br->words[k + 1] << 32;
  br->P -= n;
  return (uint32_t)((acc >> (p & 31)) & ((1ull << n) - 1));
}

/* ------------------------------------------------------------------------------------------ */
/* §4.2 Algorithm 2 for one chunk (SHN1 format §7).                                              */

static uint64_t chunk_max_words(int S, int R, uint64_t c) {
  return ((uint64_t)S * R + c * (uint64_t)(R + 8) + 1 + 31) / 32;
}

int64_t orc_encode_chunk(const orc_tables* t, int S, const uint8_t* bytes, uint32_t c, uint32_t* words,
                         uint64_t cap_words, uint64_t* payload_bits) {
  if (S < 1 || S > 16) return -ORC_ERR_ARG;
  const uint32_t L = (uint32_t)t->L;
  for (uint64_t k = 0; k < cap_words; k++) words[k] = 0;
  bitwriter bw = {words, cap_words, 0, 0};
  uint32_t X[16];
  for (int q = 0; q < S; q++) X[q] = L;
  uint64_t fields = 0;
  for (int64_t i = (int64_t)c - 1; i >= 0; i--) {
    int q = (int)(i % S);
    int u = bytes[i] ^ 0x80;
    int s = t->range_of[u];
    uint32_t fs = t->f[s];
    if (fs == 0) return -ORC_ERR_ARG; /* symbol absent from the table's statistics */
    uint32_t o = (uint32_t)(u - t->lo[s]);
    int w = t->width_bits[s];
    bw_append(&bw, o, w); /* step 2: offset in nb[s] bits */
    int nb = 0;           /* step 3: normalisation bits, (X >> nb) in [f_s, 2 f_s) */
    while ((X[q] >> nb) >= 2 * fs) nb++;
    bw_append(&bw, X[q] & ((1u << nb) - 1u), nb);
    X[q] = t->enc[t->cumul[s] + (X[q] >> nb) - fs]; /* step 4: encTable transition */
    fields += (uint64_t)(w + nb);
  }
  for (int q = 0; q < S; q++) bw_append(&bw, X[q] - L, t->R);
  bw_append(&bw, 1u, 1);
  if (bw.overflow) return -ORC_ERR_CAPACITY;
  if (payload_bits) *payload_bits = fields;
  return (int64_t)((bw.P + 31) / 32);
}

int orc_decode_chunk(const orc_tables* t, int S, const uint32_t* words, uint64_t nwords, uint32_t c,
                     uint8_t* bytes) {
  if (S < 1 || S > 16) return ORC_ERR_ARG;
  if (nwords == 0 || words[nwords - 1] == 0) return ORC_ERR_CORRUPT;
  const uint32_t L = (uint32_t)t->L;
  bitreader br = {words, nwords, (int64_t)(32 * (nwords - 1) + (uint64_t)floor_log2_u64(words[nwords - 1])), 0};
  uint32_t X[16];
  for (int q = S - 1; q >= 0; q--) X[q] = L + br_read(&br, t->R);
  for (uint32_t i = 0; i < c; i++) {
    int q = (int)(i % S);
    uint32_t slot = X[q] - L;
    int s = t->dec_sym[slot];
    uint32_t r = br_read(&br, t->dec_nb[slot]);
    uint32_t o = br_read(&br, t->width_bits[s]);
    X[q] = L + t->dec_next[slot] + r;
    bytes[i] = (uint8_t)(((t->lo[s] + o) & 0xFF) ^ 0x80);
  }
  if (br.underflow || br.P != 0) return ORC_ERR_CORRUPT;
  for (int q = 0; q < S; q++)
    if (X[q] != L) return ORC_ERR_CORRUPT;
  return ORC_OK;
}

/* ------------------------------------------------------------------------------------------ */
/* Little-endian field access for the stream header (SHN1 format §6).                            */

static void put16(uint8_t* p, uint16_t v) {
  p[0] = (uint8_t)v;
  p[1] = (uint8_t)(v >> 8);
}
static void put32(uint8_t* p, uint32_t v) {
  for (int b = 0; b < 4; b++) p[b] = (uint8_t)(v >> (8 * b));
}
static void put64(uint8_t* p, uint64_t v) {
  for (int b = 0; b < 8; b++) p[b] = (uint8_t)(v >> (8 * b));
}
static uint16_t get16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get32(const uint8_t* p) {
  uint32_t v = 0;
  for (int b = 3; b >= 0; b--) v = (v << 8) | p[b];
  return v;
}
static uint64_t get64(const uint8_t* p) {
  uint64_t v = 0;
  for (int b = 7; b >= 0; b--) v = (v << 8) | p[b];
  return v;
}

static int params_ok(const orc_params* p) {
  if (p->K < 1 || p->K > 256 || p->R < 4 || p->R > 12 || p->K > (1 << p->R)) return 0;
  if (!(p->S == 1 || p->S == 2 || p->S == 4 || p->S == 8 || p->S == 16)) return 0;
  if (p->C < 128 || p->C > 65536 || (p->C % 128) != 0) return 0;
  return 1;
}

static uint64_t seg_chunks(uint64_t n, int C) { return (n + (uint64_t)C - 1) / (uint64_t)C; }

/* SHN1 format §6 "which symbols a chunk holds": chunks come in groups of up to 32; a group's symbols
 * are cut into 16-symbol pieces dealt round-robin to its chunks. Writes the positions (relative to
 * the segment start) of chunk c's symbols, in chunk order, to pos (if not NULL); returns the count. */
static uint32_t chunk_positions(uint64_t n, int C, uint64_t c, uint64_t* pos) {
  const uint64_t nch = seg_chunks(n, C);
  const uint64_t grp = c / 32, j = c % 32;
  const uint64_t m = (nch - 32 * grp < 32) ? nch - 32 * grp : 32;
  const uint64_t base = 32 * grp * (uint64_t)C;
  const uint64_t end = (32 * (grp + 1) * (uint64_t)C < n) ? 32 * (grp + 1) * (uint64_t)C : n;
  const uint64_t ng = end - base;
  const uint64_t P = (ng + 15) / 16;
  uint32_t count = 0;
  for (uint64_t p = j; p < P; p += m)
    for (uint64_t t = 0; t < 16 && 16 * p + t < ng; t++) {
      if (pos) pos[count] = base + 16 * p + t;
      count++;
    }
  return count;
}

uint64_t orc_stream_bound(const orc_params* p, const orc_segment* segs, int n_segs) {
  if (!params_ok(p) || n_segs < 0) return 0;
  uint64_t tb = round_up(3ull * (uint64_t)p->K, 4);
  uint64_t chunks = 0;
  for (int s = 0; s < n_segs; s++) chunks += seg_chunks(segs[s].length, p->C);
  uint64_t words = chunks * chunk_max_words(p->S, p->R, (uint64_t)p->C); /* every chunk holds <= C symbols */
  uint64_t index_off = 64 + 32ull * (uint64_t)n_segs + tb * (uint64_t)n_segs;
  uint64_t payload_off = round_up(index_off + 4 * chunks, 16);
  return round_up(payload_off + 4 * words, 16);
}

/* ------------------------------------------------------------------------------------------ */
/* A tiny parallel-for over independent items (chunks or segments).                            */

typedef struct {
  void (*fn)(void* ctx, uint64_t item);
  void* ctx;
  uint64_t n_items;
  uint64_t next;
  pthread_mutex_t mu;
} pfor_state;

static void* pfor_worker(void* arg) {
  pfor_state* st = (pfor_state*)arg;
  for (;;) {
    pthread_mutex_lock(&st->mu);
    uint64_t item = st->next++;
    pthread_mutex_unlock(&st->mu);
    if (item >= st->n_items) break;
    st->fn(st->ctx, item);
  }
  return NULL;
}

static void parallel_for(int n_threads, uint64_t n_items, void (*fn)(void*, uint64_t), void* ctx) {
  if (n_threads <= 1 || n_items <= 1) {
    for (uint64_t i = 0; i < n_items; i++) fn(ctx, i);
    return;
  }
  pfor_state st;
  st.fn = fn;
  st.ctx = ctx;
  st.n_items = n_items;
  st.next = 0;
  pthread_mutex_init(&st.mu, NULL);
  if (n_threads > 256) n_threads = 256;
  pthread_t th[256];
  int started = 0;
  for (int i = 0; i < n_threads; i++)
    if (pthread_create(&th[i], NULL, pfor_worker, &st) == 0) started++;
    else break;
  if (started == 0) pfor_worker(&st);
  for (int i = 0; i < started; i++) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&st.mu);
}

/* ------------------------------------------------------------------------------------------ */
/* Stream encoder (SHN1 format §6–§7).                                                            */

typedef struct {
  const uint8_t* input;
  const orc_segment* segs;
  const orc_params* p;
  orc_tables* tables;       /* per segment */
  uint64_t* chunk_seg;      /* per global chunk: segment */
  uint64_t* chunk_local;    /* per global chunk: index within its segment */
  uint32_t** chunk_words;   /* per global chunk: encoded words (malloc) */
  int64_t* chunk_nwords;    /* per global chunk: word count or -(error) */
  uint64_t* chunk_bits;     /* per global chunk: payload bits */
  const uint16_t* given_lo; /* optional caller tables */
  const uint32_t* given_f;
  orc_segment_stats* stats;
  int* seg_rc;
} enc_ctx;

static void enc_segment_tables(void* vctx, uint64_t s) {
  enc_ctx* ctx = (enc_ctx*)vctx;
  const orc_segment* sg = &ctx->segs[s];
  uint64_t hist[256];
  orc_histogram(ctx->input + sg->offset, sg->length, hist);
  int64_t cost = 0;
  int rc;
  if (ctx->given_lo) {
    rc = orc_tables_init(ctx->given_lo + s * (uint64_t)ctx->p->K, ctx->given_f + s * (uint64_t)ctx->p->K,
                         ctx->p->K, ctx->p->R, &ctx->tables[s]);
  } else {
    rc = orc_build_segment_tables(hist, ctx->p->K, ctx->p->R, &ctx->tables[s], &cost);
  }
  ctx->seg_rc[s] = rc;
  if (ctx->stats) {
    orc_segment_stats* st = &ctx->stats[s];
    memset(st, 0, sizeof(*st));
    st->dp_cost = cost;
    memcpy(st->hist, hist, sizeof(hist));
    for (int k = 0; k < ctx->p->K; k++) {
      st->lo[k] = ctx->tables[s].lo[k];
      st->f[k] = ctx->tables[s].f[k];
    }
  }
}

static void enc_chunk(void* vctx, uint64_t g) {
  enc_ctx* ctx = (enc_ctx*)vctx;
  uint64_t s = ctx->chunk_seg[g], c = ctx->chunk_local[g];
  const orc_segment* sg = &ctx->segs[s];
  const int C = ctx->p->C;
  if (ctx->seg_rc[s] != ORC_OK) {
    ctx->chunk_nwords[g] = -ctx->seg_rc[s];
    return;
  }
  uint64_t* pos = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)C);
  uint8_t* sym = (uint8_t*)malloc((size_t)C);
  const uint32_t len = chunk_positions(sg->length, C, c, pos);
  uint64_t cap = chunk_max_words(ctx->p->S, ctx->p->R, len) + 1;
  uint32_t* w = (uint32_t*)malloc(sizeof(uint32_t) * cap);
  if (!w || !pos || !sym) {
    free(w);
    free(pos);
    free(sym);
    ctx->chunk_nwords[g] = -ORC_ERR_NOMEM;
    return;
  }
  for (uint32_t i = 0; i < len; i++) sym[i] = ctx->input[sg->offset + pos[i]];
  uint64_t bits = 0;
  ctx->chunk_nwords[g] = orc_encode_chunk(&ctx->tables[s], ctx->p->S, sym, len, w, cap, &bits);
  ctx->chunk_words[g] = w;
  ctx->chunk_bits[g] = bits;
  free(pos);
  free(sym);
}

static int encode_stream_impl(const uint8_t* input, const orc_segment* segs, int n_segs, const orc_params* p,
                              const uint16_t* given_lo, const uint32_t* given_f, int n_threads, uint8_t* out,
                              uint64_t cap, uint64_t* out_bytes, orc_segment_stats* stats) {
  if (!params_ok(p) || n_segs < 0) return ORC_ERR_ARG;
  uint64_t total_chunks = 0, total_symbols = 0;
  for (int s = 0; s < n_segs; s++) {
    if (segs[s].length >= (1ull << 32)) return ORC_ERR_ARG;
    total_chunks += seg_chunks(segs[s].length, p->C);
    total_symbols += segs[s].length;
  }
  if (total_chunks >= (1ull << 32)) return ORC_ERR_ARG;

  enc_ctx ctx;
  memset(&ctx, 0, sizeof(ctx));
  ctx.input = input;
  ctx.segs = segs;
  ctx.p = p;
  ctx.given_lo = given_lo;
  ctx.given_f = given_f;
  ctx.stats = stats;
  ctx.tables = (orc_tables*)calloc((size_t)(n_segs > 0 ? n_segs : 1), sizeof(orc_tables));
  ctx.seg_rc = (int*)calloc((size_t)(n_segs > 0 ? n_segs : 1), sizeof(int));
  size_t nch = (size_t)(total_chunks > 0 ? total_chunks : 1);
  ctx.chunk_seg = (uint64_t*)calloc(nch, sizeof(uint64_t));
  ctx.chunk_local = (uint64_t*)calloc(nch, sizeof(uint64_t));
  ctx.chunk_words = (uint32_t**)calloc(nch, sizeof(uint32_t*));
  ctx.chunk_nwords = (int64_t*)calloc(nch, sizeof(int64_t));
  ctx.chunk_bits = (uint64_t*)calloc(nch, sizeof(uint64_t));
  int rc = ORC_OK;
  if (!ctx.tables || !ctx.seg_rc || !ctx.chunk_seg || !ctx.chunk_local || !ctx.chunk_words || !ctx.chunk_nwords ||
      !ctx.chunk_bits) {
    rc = ORC_ERR_NOMEM;
    goto done;
  }
  {
    uint64_t g = 0;
    for (int s = 0; s < n_segs; s++) {
      uint64_t nc = seg_chunks(segs[s].length, p->C);
      for (uint64_t c = 0; c < nc; c++, g++) {
        ctx.chunk_seg[g] = (uint64_t)s;
        ctx.chunk_local[g] = c;
      }
    }
  }
  parallel_for(n_threads, (uint64_t)n_segs, enc_segment_tables, &ctx);
  for (int s = 0; s < n_segs; s++)
    if (ctx.seg_rc[s] != ORC_OK) {
      rc = ctx.seg_rc[s];
      goto done;
    }
  parallel_for(n_threads, total_chunks, enc_chunk, &ctx);
  for (uint64_t g = 0; g < total_chunks; g++)
    if (ctx.chunk_nwords[g] < 0) {
      rc = (int)(-ctx.chunk_nwords[g]);
      goto done;
    }

  {
    const uint64_t tb = round_up(3ull * (uint64_t)p->K, 4);
    const uint64_t index_off = 64 + 32ull * (uint64_t)n_segs + tb * (uint64_t)n_segs;
    const uint64_t payload_off = round_up(index_off + 4 * total_chunks, 16);
    uint64_t payload_words = 0;
    for (uint64_t g = 0; g < total_chunks; g++) payload_words += (uint64_t)ctx.chunk_nwords[g];
    const uint64_t stream_bytes = round_up(payload_off + 4 * payload_words, 16);
    if (out_bytes) *out_bytes = stream_bytes;
    if (stream_bytes > cap) {
      rc = ORC_ERR_CAPACITY;
      goto done;
    }
    memset(out, 0, stream_bytes);
    put32(out + 0, 0x314E4853u);
    put16(out + 4, 1);
    put16(out + 6, 64);
    put32(out + 8, (uint32_t)n_segs);
    put16(out + 12, (uint16_t)p->K);
    out[14] = (uint8_t)p->R;
    out[15] = (uint8_t)p->S;
    put32(out + 16, (uint32_t)p->C);
    put32(out + 20, (uint32_t)tb);
    put64(out + 24, total_symbols);
    put64(out + 32, total_chunks);
    put64(out + 40, index_off);
    put64(out + 48, payload_off);
    put64(out + 56, stream_bytes);

    uint64_t g = 0, out_off = 0, pay_start = 0;
    for (int s = 0; s < n_segs; s++) {
      uint8_t* d = out + 64 + 32ull * (uint64_t)s;
      uint64_t nc = seg_chunks(segs[s].length, p->C);
      uint64_t seg_words = 0, seg_bits = 0;
      uint8_t* idx = out + index_off + 4 * g;
      for (uint64_t c = 0; c < nc; c++) {
        put32(idx + 4 * c, (uint32_t)seg_words);
        uint8_t* dst = out + payload_off + pay_start + 4 * seg_words;
        for (int64_t k = 0; k < ctx.chunk_nwords[g + c]; k++) put32(dst + 4 * k, ctx.chunk_words[g + c][k]);
        seg_words += (uint64_t)ctx.chunk_nwords[g + c];
        seg_bits += ctx.chunk_bits[g + c];
      }
      if (seg_words >= (1ull << 32)) {
        rc = ORC_ERR_ARG;
        goto done;
      }
      put64(d + 0, segs[s].length);
      put64(d + 8, out_off);
      put64(d + 16, pay_start);
      put32(d + 24, (uint32_t)seg_words);
      put32(d + 28, (uint32_t)g);
      uint8_t* rec = out + 64 + 32ull * (uint64_t)n_segs + tb * (uint64_t)s;
      for (int k = 0; k < p->K; k++) {
        put16(rec + 2 * k, (uint16_t)ctx.tables[s].f[k]);
        rec[2 * p->K + k] = (uint8_t)ctx.tables[s].lo[k];
      }
      if (stats) {
        stats[s].payload_bits = seg_bits;
        stats[s].payload_words = seg_words;
      }
      out_off += segs[s].length;
      pay_start += 4 * seg_words;
      g += nc;
    }
  }
done:
  if (ctx.chunk_words)
    for (uint64_t g = 0; g < total_chunks; g++) free(ctx.chunk_words[g]);
  free(ctx.tables);
  free(ctx.seg_rc);
  free(ctx.chunk_seg);
  free(ctx.chunk_local);
  free(ctx.chunk_words);
  free(ctx.chunk_nwords);
  free(ctx.chunk_bits);
  return rc;
}

int orc_encode_stream(const uint8_t* input, const orc_segment* segs, int n_segs, const orc_params* p, int n_threads,
                      uint8_t* out, uint64_t cap, uint64_t* out_bytes, orc_segment_stats* stats) {
  return encode_stream_impl(input, segs, n_segs, p, NULL, NULL, n_threads, out, cap, out_bytes, stats);
}

int orc_encode_stream_with_tables(const uint8_t* input, const orc_segment* segs, int n_segs, const orc_params* p,
                                  const uint16_t* lo, const uint32_t* f, int n_threads, uint8_t* out, uint64_t cap,
                                  uint64_t* out_bytes, orc_segment_stats* stats) {
  if (!lo || !f) return ORC_ERR_ARG;
  return encode_stream_impl(input, segs, n_segs, p, lo, f, n_threads, out, cap, out_bytes, stats);
}

/* ------------------------------------------------------------------------------------------ */
/* Stream decoder (SHN1 format §6–§7).                                                            */

typedef struct {
  const uint8_t* stream;
  uint64_t payload_off, index_off;
  int S, C;
  uint8_t* out;
  orc_tables* tables;
  uint64_t* chunk_seg;
  uint64_t* seg_first_chunk;
  uint64_t* seg_nsym;
  uint64_t* seg_out_off;
  uint64_t* seg_pay_start;
  uint64_t* seg_pay_words;
  int* chunk_rc;
} dec_ctx;

static void dec_chunk(void* vctx, uint64_t g) {
  dec_ctx* ctx = (dec_ctx*)vctx;
  uint64_t s = ctx->chunk_seg[g];
  uint64_t c = g - ctx->seg_first_chunk[s];
  uint64_t nc = seg_chunks(ctx->seg_nsym[s], ctx->C);
  uint64_t w0 = get32(ctx->stream + ctx->index_off + 4 * g);
  uint64_t w1 = (c + 1 < nc) ? get32(ctx->stream + ctx->index_off + 4 * (g + 1)) : ctx->seg_pay_words[s];
  if (w1 <= w0 || w1 > ctx->seg_pay_words[s] || (c == 0 && w0 != 0)) {
    ctx->chunk_rc[g] = ORC_ERR_CORRUPT;
    return;
  }
  /* words are little-endian in the stream; copy them out so the reader works on host ints */
  uint64_t nw = w1 - w0;
  uint32_t* words = (uint32_t*)malloc(sizeof(uint32_t) * nw);
  uint64_t* pos = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)ctx->C);
  uint8_t* sym = (uint8_t*)malloc((size_t)ctx->C);
  if (!words || !pos || !sym) {
    free(words);
    free(pos);
    free(sym);
    ctx->chunk_rc[g] = ORC_ERR_NOMEM;
    return;
  }
  const uint32_t len = chunk_positions(ctx->seg_nsym[s], ctx->C, c, pos);
  const uint8_t* base = ctx->stream + ctx->payload_off + ctx->seg_pay_start[s] + 4 * w0;
  for (uint64_t k = 0; k < nw; k++) words[k] = get32(base + 4 * k);
  ctx->chunk_rc[g] = orc_decode_chunk(&ctx->tables[s], ctx->S, words, nw, len, sym);
  for (uint32_t i = 0; i < len; i++) ctx->out[ctx->seg_out_off[s] + pos[i]] = sym[i];
  free(words);
  free(pos);
  free(sym);
}

int orc_decode_stream(const uint8_t* stream, uint64_t bytes, int n_threads, uint8_t* out, uint64_t cap,
                      uint64_t* out_symbols) {
  if (bytes < 64) return ORC_ERR_CORRUPT;
  if (get32(stream) != 0x314E4853u || get16(stream + 4) != 1 || get16(stream + 6) != 64) return ORC_ERR_CORRUPT;
  orc_params p;
  uint32_t n_segs = get32(stream + 8);
  p.K = get16(stream + 12);
  p.R = stream[14];
  p.S = stream[15];
  p.C = (int32_t)get32(stream + 16);
  if (!params_ok(&p)) return ORC_ERR_CORRUPT;
  uint64_t tb = get32(stream + 20);
  uint64_t total_symbols = get64(stream + 24), total_chunks = get64(stream + 32);
  uint64_t index_off = get64(stream + 40), payload_off = get64(stream + 48), stream_bytes = get64(stream + 56);
  if (tb != round_up(3ull * (uint64_t)p.K, 4)) return ORC_ERR_CORRUPT;
  if (n_segs > (1u << 30) || total_chunks >= (1ull << 32)) return ORC_ERR_CORRUPT;
  if (index_off != 64 + 32ull * n_segs + tb * n_segs) return ORC_ERR_CORRUPT;
  if (payload_off != round_up(index_off + 4 * total_chunks, 16)) return ORC_ERR_CORRUPT;
  if (stream_bytes > bytes || payload_off > stream_bytes) return ORC_ERR_CORRUPT;
  if (out_symbols) *out_symbols = total_symbols;
  if (total_symbols > cap) return ORC_ERR_CAPACITY;

  dec_ctx ctx;
  memset(&ctx, 0, sizeof(ctx));
  size_t ns = n_segs > 0 ? n_segs : 1, nch = total_chunks > 0 ? (size_t)total_chunks : 1;
  ctx.stream = stream;
  ctx.payload_off = payload_off;
  ctx.index_off = index_off;
  ctx.S = p.S;
  ctx.C = p.C;
  ctx.out = out;
  ctx.tables = (orc_tables*)calloc(ns, sizeof(orc_tables));
  ctx.chunk_seg = (uint64_t*)calloc(nch, sizeof(uint64_t));
  ctx.seg_first_chunk = (uint64_t*)calloc(ns, sizeof(uint64_t));
  ctx.seg_nsym = (uint64_t*)calloc(ns, sizeof(uint64_t));
  ctx.seg_out_off = (uint64_t*)calloc(ns, sizeof(uint64_t));
  ctx.seg_pay_start = (uint64_t*)calloc(ns, sizeof(uint64_t));
  ctx.seg_pay_words = (uint64_t*)calloc(ns, sizeof(uint64_t));
  ctx.chunk_rc = (int*)calloc(nch, sizeof(int));
  int rc = ORC_OK;
  if (!ctx.tables || !ctx.chunk_seg || !ctx.seg_first_chunk || !ctx.seg_nsym || !ctx.seg_out_off ||
      !ctx.seg_pay_start || !ctx.seg_pay_words || !ctx.chunk_rc) {
    rc = ORC_ERR_NOMEM;
    goto done;
  }
  {
    uint64_t g = 0, out_off = 0, pay = 0;
    for (uint32_t s = 0; s < n_segs; s++) {
      const uint8_t* d = stream + 64 + 32ull * s;
      uint64_t nsym = get64(d + 0);
      uint64_t nc = seg_chunks(nsym, p.C);
      if (nsym >= (1ull << 32) || get64(d + 8) != out_off || get64(d + 16) != pay || get32(d + 28) != g) {
        rc = ORC_ERR_CORRUPT;
        goto done;
      }
      ctx.seg_nsym[s] = nsym;
      ctx.seg_out_off[s] = out_off;
      ctx.seg_pay_start[s] = pay;
      ctx.seg_pay_words[s] = get32(d + 24);
      ctx.seg_first_chunk[s] = g;
      if (g + nc > total_chunks) {
        rc = ORC_ERR_CORRUPT;
        goto done;
      }
      for (uint64_t c = 0; c < nc; c++) ctx.chunk_seg[g + c] = s;
      const uint8_t* rec = stream + 64 + 32ull * n_segs + tb * s;
      uint16_t lo[256];
      uint32_t f[256];
      for (int k = 0; k < p.K; k++) {
        f[k] = get16(rec + 2 * k);
        lo[k] = rec[2 * p.K + k];
      }
      if (orc_tables_init(lo, f, p.K, p.R, &ctx.tables[s]) != ORC_OK) {
        rc = ORC_ERR_CORRUPT;
        goto done;
      }
      out_off += nsym;
      pay += 4 * ctx.seg_pay_words[s];
      g += nc;
    }
    if (g != total_chunks || out_off != total_symbols || payload_off + pay > stream_bytes ||
        stream_bytes != round_up(payload_off + pay, 16)) {
      rc = ORC_ERR_CORRUPT;
      goto done;
    }
  }
  parallel_for(n_threads, total_chunks, dec_chunk, &ctx);
  for (uint64_t g = 0; g < total_chunks; g++)
    if (ctx.chunk_rc[g] != ORC_OK) {
      rc = ctx.chunk_rc[g];
      break;
    }
done:
  free(ctx.tables);
  free(ctx.chunk_seg);
  free(ctx.seg_first_chunk);
  free(ctx.seg_nsym);
  free(ctx.seg_out_off);
  free(ctx.seg_pay_start);
  free(ctx.seg_pay_words);
  free(ctx.chunk_rc);
  return rc;
}
