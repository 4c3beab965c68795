/*
 * shn_oracle.h — plain, slow CPU oracle for the Shannonic INT8 entropy codec.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may include, link or call this code:
 * only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference arm use it.
 * It shares no code, header, table or constant generator with the CUDA path.
 *
 * Method: "Shannonic: Efficient Entropy-Optimal Compression for ML Workloads"
 * (MLSys 2026 talk notes) — §4.1 histogram, DP range selection, per-range parameters and tANS
 * tables; §4.2 Algorithm 2 encode/decode; §4 Theorem 1 (checked by the tests, not here).
 * Every detail the notes leave open follows the SHN1 format specification.
 *
 * Parity pins: every function below is pinned by tests/test_oracle_*.py against brute force,
 * closed forms or the mathematics (see the header comment of each test file).
 */
#ifndef SHN_ORACLE_H
#define SHN_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ORC_OK = 0,
  ORC_ERR_ARG = 1,      /* invalid parameter or size */
  ORC_ERR_CAPACITY = 2, /* output buffer too small */
  ORC_ERR_CORRUPT = 3,  /* stream fails a structural or end-of-chunk check */
  ORC_ERR_NOMEM = 4
};

#define ORC_MAX_L 4096

typedef struct {
  uint64_t offset; /* byte offset of the segment in the input */
  uint64_t length; /* symbols (bytes) in the segment */
} orc_segment;

typedef struct {
  int32_t K; /* number of ranges */
  int32_t R; /* log2 of the tANS state count L */
  int32_t S; /* interleaved states per chunk */
  int32_t C; /* symbols per chunk */
} orc_params;

/* All tables of one segment (SHN1 format §3–§5). */
typedef struct {
  int32_t K, R, L;
  uint16_t lo[257];         /* range k = [lo[k], lo[k+1]), lo[K] = 256 */
  uint32_t f[256];          /* state count per range, sum = L */
  uint32_t cumul[256];      /* sum of f over earlier ranges */
  uint8_t width_bits[256];  /* w_k = ceil(log2(range width)) */
  uint8_t range_of[256];    /* rangeId[u] */
  uint16_t spread[ORC_MAX_L];
  uint16_t dec_sym[ORC_MAX_L];  /* range id decoded at slot i */
  uint8_t dec_nb[ORC_MAX_L];    /* renormalisation bits read at slot i */
  uint16_t dec_next[ORC_MAX_L]; /* next slot base: (x << nb) - L */
  uint16_t enc[ORC_MAX_L];      /* enc[cumul_s + j] = L + j-th slot of s */
} orc_tables;

/* Per-segment statistics returned by the stream encoder. */
typedef struct {
  int64_t dp_cost;        /* D[256][K] of the range-selection DP (units of 2^-24 bit) */
  uint64_t payload_bits;  /* sum of offset + renormalisation field widths */
  uint64_t payload_words; /* segment payload size in 32-bit words */
  uint64_t hist[256];
  uint16_t lo[256];
  uint32_t f[256];
} orc_segment_stats;

int64_t orc_lg(uint64_t n);
void orc_histogram(const uint8_t* bytes, uint64_t n, uint64_t hist[256]);
int orc_partition(const uint64_t* hist, int A, int K, uint16_t* lo, int64_t* cost);
int orc_normalize(const uint64_t* N, int K, int R, uint32_t* f);
int orc_tables_init(const uint16_t* lo, const uint32_t* f, int K, int R, orc_tables* t);
int orc_build_segment_tables(const uint64_t hist[256], int K, int R, orc_tables* t, int64_t* dp_cost);

/* One chunk, given its symbol sequence (SHN1 format §6 says which tensor positions a chunk holds).
 * Symbols are u = byte ^ 0x80. Returns words written, or -(error). */
int64_t orc_encode_chunk(const orc_tables* t, int S, const uint8_t* bytes, uint32_t c, uint32_t* words,
                         uint64_t cap_words, uint64_t* payload_bits);
int orc_decode_chunk(const orc_tables* t, int S, const uint32_t* words, uint64_t nwords, uint32_t c,
                     uint8_t* bytes);

/* Whole SHN1 streams (SHN1 format §6). */
uint64_t orc_stream_bound(const orc_params* p, const orc_segment* segs, int n_segs);
int orc_encode_stream(const uint8_t* input, const orc_segment* segs, int n_segs, const orc_params* p,
                      int n_threads, uint8_t* out, uint64_t cap, uint64_t* out_bytes, orc_segment_stats* stats);
/* Same, with the tables supplied by the caller (lo, f per segment: K entries each). */
int orc_encode_stream_with_tables(const uint8_t* input, const orc_segment* segs, int n_segs, const orc_params* p,
                                  const uint16_t* lo, const uint32_t* f, int n_threads, uint8_t* out, uint64_t cap,
                                  uint64_t* out_bytes, orc_segment_stats* stats);
int orc_decode_stream(const uint8_t* stream, uint64_t bytes, int n_threads, uint8_t* out, uint64_t cap,
                      uint64_t* out_symbols);

#ifdef __cplusplus
}
#endif
#endif
