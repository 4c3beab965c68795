/*
 * shn.h — C ABI of the B200 Shannonic INT8 entropy codec (libshn.so).
 *
 * The codec is the Shannonic scheme of "Shannonic: Efficient Entropy-Optimal Compression for ML
 * Workloads" (MLSys 2026 talk notes): a 256-bin histogram, a dynamic-programming split of the value
 * space into K contiguous ranges, and tANS over the range indices with raw fixed-width offsets
 * (§4, §4.1, §4.2 Algorithm 2). The bitstream ("SHN1") is fixed by its own format specification.
 *
 * Conventions for every entry point:
 *  - Pointers named d_* are CUDA device pointers, h_* are host pointers. All memory belongs to the
 *    caller; the library never allocates device memory and never synchronises the device, except in
 *    shn_get_device_status (documented below).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). Work is enqueued
 *    asynchronously on it and runs on the device that is current for the calling thread.
 *  - Return value: an shn_status. Errors a host check can see (bad parameters, sizes, alignment,
 *    too-small buffers computable on the host) are returned immediately and nothing is enqueued.
 *    Errors only the device can see (a corrupt stream, an output larger than its buffer) are
 *    written to the status word at the start of the caller's workspace (d_work); kernels then skip
 *    the rest of their work and return normally — no trap, no hang. Read it with
 *    shn_get_device_status or by copying the first 8 bytes of d_work.
 *  - Symbols: byte b of an INT8 tensor is coded as u = b XOR 0x80 (signed value + 128).
 */
#ifndef SHN_H
#define SHN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SHN_VERSION 0x00010000u /* 1.0.0; the stream format version is 1 */

/* Size of one shn_table record in bytes (a multiple of 256). */
#define SHN_TABLE_BYTES 11264u
#define SHN_TABLE_PUBLIC_BYTES 800u

typedef enum shn_status {
  SHN_OK = 0,
  SHN_ERR_INVALID_ARG = 1, /* bad parameter, pointer, size or alignment */
  SHN_ERR_CAPACITY = 2,    /* an output buffer is too small */
  SHN_ERR_CORRUPT = 3,     /* the compressed stream fails a structural or end-of-chunk check */
  SHN_ERR_CUDA = 4,        /* a CUDA launch or runtime call failed */
  SHN_ERR_TIMEOUT = 5,     /* a bounded device wait gave up (reserved; current kernels never wait) */
  SHN_ERR_UNSUPPORTED = 6, /* valid parameters that the library's kernels do not implement */
  SHN_ERR_WORKSPACE = 7    /* the workspace is smaller than the *_workspace_bytes query returned */
} shn_status;

/* A segment is a run of input bytes coded with its own table (one tensor, one KV layer, …). */
typedef struct shn_segment {
  uint64_t offset; /* byte offset of the segment within d_in */
  uint64_t length; /* number of INT8 values; must be < 2^32 */
} shn_segment;

/* Codec parameters (SHN1 format §6 constraints). */
typedef struct shn_params {
  uint32_t K;                /* number of ranges, 1 <= K <= min(256, L); K = 256 is plain tANS */
  uint32_t log2L;            /* R: tANS state count L = 2^R, 4 <= R <= 12 */
  uint32_t chunk_symbols;    /* C: symbols per chunk, multiple of 128, 128 <= C <= 65536 */
  uint32_t states_per_chunk; /* S: interleaved tANS states per chunk, one of 1, 2, 4, 8, 16 */
} shn_params;

/*
 * Per-table device record written by shn_build_tables (SHN_TABLE_BYTES each, 256-byte aligned
 * when d_tables is). The leading fields are public and stable; `opaque` holds the encoder's
 * lookup tables and must not be modified.
 */
typedef struct shn_table {
  uint32_t K;       /* ranges */
  uint32_t log2L;   /* R */
  uint32_t status;  /* SHN_OK, or SHN_ERR_INVALID_ARG when the histogram total is >= 2^32 */
  uint32_t w_max;   /* largest offset field width over the ranges */
  int64_t dp_cost;  /* D[256][K] of the range DP, units of 2^-24 bit (SHN1 format §3) */
  uint64_t n;       /* histogram total */
  uint16_t f[256];  /* tANS state count of each range (sum = L); entries >= K are 0 */
  uint8_t lo[256];  /* first symbol u of each range; range k = [lo[k], lo[k+1]) with lo[K] = 256 */
  uint8_t opaque[SHN_TABLE_BYTES - SHN_TABLE_PUBLIC_BYTES];
} shn_table;

/* --- queries (host only, no CUDA calls) --------------------------------------------------- */

uint32_t shn_version(void);
const char* shn_status_string(int status);

/* SHN_OK if p satisfies the SHN1 format §6 constraints, else SHN_ERR_INVALID_ARG. */
int shn_check_params(const shn_params* p);

/* Bytes of one table record in d_tables (constant, = sizeof(shn_table)). */
size_t shn_table_bytes(const shn_params* p);

/* Largest SHN1 stream shn_encode can produce for these segments (0 on bad arguments). */
size_t shn_encode_bound(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs);

/* Device workspace for shn_encode's single-pass mode: the status word, per-chunk sizes and scan
 * scratch, plus one worst-case slot per chunk (about shn_encode_bound bytes in all). With this much
 * workspace every chunk's state machine runs once and a copy pass moves the slots into place. */
size_t shn_encode_workspace_bytes(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs);

/* The smallest workspace shn_encode accepts (status word, per-chunk sizes and scan scratch, a few
 * bytes per chunk). Below shn_encode_workspace_bytes it runs in two passes: one to size every chunk,
 * one to write it at its final place (the state machine runs twice). No counterpart in the paper:
 * a memory/time trade of this GPU implementation. */
size_t shn_encode_workspace_bytes_min(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs);

/* Device workspace shn_decode needs (the status word only). */
size_t shn_decode_workspace_bytes(const shn_params* p);

/* --- the codec ---------------------------------------------------------------------------- */

/*
 * 256-bin histogram of each segment (Shannonic §4.1, the preprocessing step that counts every
 * value of the tensor). d_hist[s*256 + u] = number of bytes b in segment s with (b ^ 0x80) == u.
 *  d_in    device, the input bytes; any alignment.
 *  h_segs  host array of n_segs segments; every segment must lie inside d_in's allocation.
 *  d_hist  device, n_segs*256 uint64, 8-byte aligned; fully overwritten.
 * Errors: SHN_ERR_INVALID_ARG (NULL pointers with n_segs > 0, segment length >= 2^32),
 *         SHN_ERR_CUDA.
 */
int shn_histogram(const uint8_t* d_in, const shn_segment* h_segs, uint32_t n_segs, uint64_t* d_hist,
                  void* stream);

/*
 * Range selection and tANS tables for each histogram (Shannonic §4.1: DP range selection
 * C[i,k] = min_{j<i} C[j,k-1] + Cost(j,i-1) with backtracking from C[256,K]; per-range base,
 * offset width, encTable start and bias; rangeId[256]; an L-state tANS table from the range
 * probabilities). Exact rules: SHN1 format §2-§5. Each table is built by a cluster of 2, 4 or 8
 * blocks when the launch leaves SMs free for that, otherwise by one block (same records).
 *  d_hist    device, n_tables*256 uint64 (as written by shn_histogram).
 *  d_tables  device, n_tables*shn_table_bytes(p) bytes, 256-byte aligned; fully overwritten.
 * A histogram whose total is >= 2^32 gets status SHN_ERR_INVALID_ARG in its record (and makes
 * shn_encode report SHN_ERR_INVALID_ARG on the device).
 * Errors: SHN_ERR_INVALID_ARG, SHN_ERR_CUDA.
 */
int shn_build_tables(const uint64_t* d_hist, uint32_t n_tables, const shn_params* p, void* d_tables,
                     void* stream);

/*
 * Encode segments into one SHN1 stream (Shannonic §4.2, Algorithm 2: per value, s = rangeId[x],
 * emit the offset x - base[s] in nb[s] bits, emit the state-normalisation bits, move the state
 * through encTable). Chunks of C symbols are coded independently with S interleaved states.
 *  d_in          device input bytes, any alignment (chunks whose bytes start on a 16-byte
 *                boundary are read with 16-byte loads, the others byte by byte).
 *  h_segs        host, n_segs segments; segment s is coded with table s of d_tables.
 *  d_tables      device, n_segs records from shn_build_tables with the same params.
 *  d_work        device workspace of >= shn_encode_workspace_bytes_min(p, h_segs, n_segs) bytes,
 *                256-byte aligned; >= shn_encode_workspace_bytes(...) selects the single-pass
 *                mode (same output). Its first 8 bytes receive the device status.
 *  d_out         device, out_capacity bytes, 16-byte aligned; receives the stream. May be pinned
 *                host memory mapped into the device address space (offload): with the
 *                single-pass workspace the compressed bytes then cross the link exactly once.
 *  d_out_bytes   device uint64: the stream size in bytes (written even when it exceeds the
 *                capacity, in which case the device status is SHN_ERR_CAPACITY and d_out holds
 *                no complete stream).
 * Streams whose shn_encode_bound exceeds 16 GiB are rejected with SHN_ERR_INVALID_ARG.
 * Errors: SHN_ERR_INVALID_ARG, SHN_ERR_WORKSPACE, SHN_ERR_CUDA; device: SHN_ERR_CAPACITY,
 *         SHN_ERR_INVALID_ARG (a table with bad status or a symbol absent from its table).
 */
int shn_encode(const uint8_t* d_in, const shn_segment* h_segs, uint32_t n_segs, const void* d_tables,
               const shn_params* p, void* d_work, size_t work_bytes, uint8_t* d_out, size_t out_capacity,
               uint64_t* d_out_bytes, void* stream);

/*
 * Decode an SHN1 stream (Shannonic §4.2: decTable[X] gives the range s and the bit count; read the
 * offset o; x = base[s] + o). The stream is self-describing (segments, tables, chunk index);
 * `p` must equal the parameters it was encoded with (checked on the device) and selects the
 * kernel configuration. Output: segment after segment, total_symbols bytes.
 *  d_comp      device, comp_bytes of stream, 16-byte aligned.
 *  d_work      device workspace of >= shn_decode_workspace_bytes(p) bytes, 256-byte aligned.
 *  d_out       device, out_capacity bytes, any alignment.
 * Errors: SHN_ERR_INVALID_ARG, SHN_ERR_CUDA; device: SHN_ERR_CORRUPT (bad header/descriptor/index, missing sentinel,
 *         end-of-chunk state or position check failed), SHN_ERR_CAPACITY (out_capacity too small).
 * A chunk that fails its checks leaves its output bytes unspecified; every other chunk is decoded.
 */
int shn_decode(const uint8_t* d_comp, size_t comp_bytes, const shn_params* p, void* d_work, size_t work_bytes,
               uint8_t* d_out, size_t out_capacity, void* stream);

/*
 * Decode fused with the consumer's dequantisation: instead of the INT8 tensor, write
 *   d_out[i] = bf16_rn( float(int8 value i) * d_scales[i >> log2_group] )
 * (the product rounded once in fp32, then to bfloat16 round-to-nearest-even), e.g. a KV cache
 * quantised with one absmax scale per head_dim group. Saves the INT8 write-back and the separate
 * dequantisation pass (Shannonic §6.2: compression for KV/activation transfer; the paper decodes
 * to INT8 and has no fused form).
 *  d_scales    device float[n_scales], 4-byte aligned; n_scales >= ceil(total_symbols / 2^log2_group).
 *  log2_group  4 <= log2_group <= 31 (groups of >= 16 positions).
 *  d_out       device, out_elems bfloat16 values (as uint16), 16-byte aligned.
 * Every segment must start at an output position that is a multiple of 16 (device status
 * SHN_ERR_UNSUPPORTED otherwise). Other arguments, errors and status as in shn_decode; too few
 * scales gives device status SHN_ERR_CAPACITY.
 */
int shn_decode_bf16(const uint8_t* d_comp, size_t comp_bytes, const shn_params* p, const float* d_scales,
                    size_t n_scales, uint32_t log2_group, void* d_work, size_t work_bytes, uint16_t* d_out,
                    size_t out_elems, void* stream);

/*
 * Pipelined offload of a device tensor into host memory as n_batches SHN1 streams, one per batch of
 * segments (batch b = h_segs[batch_ends[b-1] .. batch_ends[b]), batch_ends[-1] = 0): for each batch
 * histogram, tables and encode run on `stream` into a device staging buffer; as soon as batch b is
 * encoded the host reads its size and the copy engine moves exactly that many bytes to
 * h_out + h_stream_offsets[b] on `copy_stream`, while batch b+1 encodes. Streams are placed back to
 * back at 16-byte boundaries. Shannonic §6.2 (compression for transfers); no counterpart in the
 * paper's code. The call blocks the host until the last batch is encoded; the copies complete in
 * `copy_stream` order.
 *  d_work   device workspace of >= shn_offload_workspace_bytes(...) bytes, 256-byte aligned.
 *  h_out    host, h_capacity bytes (pinned for asynchronous copies).
 *  h_stream_offsets, h_stream_bytes  host arrays of n_batches, filled by the call.
 * Errors: SHN_ERR_INVALID_ARG, SHN_ERR_WORKSPACE, SHN_ERR_CAPACITY (h_out too small), SHN_ERR_CUDA,
 *         or an encoder's device status (then the batches after it are not offloaded).
 */
size_t shn_offload_workspace_bytes(const shn_params* p, const shn_segment* h_segs, const uint32_t* batch_ends,
                                   uint32_t n_batches);
int shn_offload(const uint8_t* d_in, const shn_segment* h_segs, const uint32_t* batch_ends, uint32_t n_batches,
                const shn_params* p, void* d_work, size_t work_bytes, uint8_t* h_out, size_t h_capacity,
                size_t* h_stream_offsets, size_t* h_stream_bytes, void* stream, void* copy_stream);

/*
 * Pipelined reload of a tensor offloaded as n_streams SHN1 streams in host memory (e.g. written by
 * shn_encode into pinned host buffers, one stream per batch of segments): stream i is copied to a
 * device staging buffer on `copy_stream` (the copy engine) while stream i-1 decodes on `stream`,
 * into d_out + out_offsets[i]. Shannonic §6.2: a transfer carries r/8 instead of 1 byte per value,
 * which pays off when decoding keeps up with the link. No counterpart in the paper's code.
 *  h_streams[i]   host, stream_bytes[i] bytes (pinned for an asynchronous copy); read on the host
 *                 for its header (magic, symbol count) before anything is enqueued.
 *  d_staging      device, staging_bytes >= 2 * round_up(max stream_bytes[i], 16), 16-byte aligned.
 *  d_work         device workspace of >= 256 bytes (shared status word of all the decodes).
 *  d_out          device, out_capacity bytes; stream i's symbols go to [out_offsets[i], +its count).
 *  stream, copy_stream  the decode and copy streams (may be the same: then nothing overlaps).
 * Returns when everything is enqueued; the work completes in `stream` order.
 * Errors: SHN_ERR_INVALID_ARG, SHN_ERR_CORRUPT (a header that is not SHN1), SHN_ERR_CAPACITY (an
 *         output range outside d_out), SHN_ERR_WORKSPACE (staging too small), SHN_ERR_CUDA;
 *         device: as shn_decode (the first error of any stream).
 */
int shn_decode_from_host(const uint8_t* const* h_streams, const size_t* stream_bytes, uint32_t n_streams,
                         const shn_params* p, uint8_t* d_staging, size_t staging_bytes, void* d_work,
                         size_t work_bytes, uint8_t* d_out, const size_t* out_offsets, size_t out_capacity,
                         void* stream, void* copy_stream);

/*
 * shn_encode without a workspace, for callers that cannot allocate device memory. (This entry
 * point is an addition of this library; the paper has no counterpart.)
 *
 * Who needs it: code that must not call cudaMalloc — an allocator or out-of-memory handler, a
 * plugin whose host application owns all device memory, a path that cannot afford an allocation's
 * implicit synchronisation. shn_encode needs scratch beyond its inputs and outputs (per-chunk word
 * counts and their prefix sums); here that scratch is a fixed array inside libshn's own device
 * memory, sized for SHN_STATIC_MAX_CHUNKS chunks (about 6.3 MB). Every GPU that loads the library
 * holds this array until the process exits.
 *
 *  Arguments are those of shn_encode without d_work/work_bytes, plus
 *  d_status  device, 8 bytes, 8-byte aligned: receives the device status (as the first 8 bytes of
 *            shn_encode's workspace would); zeroed by this call.
 * The stream produced is byte-identical to shn_encode's.
 * Limits and caveats:
 *  - more than SHN_STATIC_MAX_CHUNKS chunks in total returns SHN_ERR_CAPACITY (nothing enqueued);
 *  - the first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *    that device current and keeps it for the life of the process; make that first call before any
 *    stream capture on that device. A device reset (cudaDeviceReset, or the primary context
 *    released and created again) may move the array: calls after one are not supported;
 *  - it runs shn_encode's two-pass mode (each chunk is coded twice: once to size it, once to write
 *    it in place), so it is slower than shn_encode with a single-pass workspace;
 *  - all calls share the one array: calls whose GPU work overlaps (different streams, or different
 *    host threads, without ordering between them) race and may produce corrupt streams. Order
 *    them on one stream or with events.
 * Never allocates: no cudaMalloc, cudaFree or allocating library routine is called.
 * Errors: as shn_encode, with the same host checks (including the 16 GiB stream limit, checked
 *         before the chunk count); SHN_ERR_WORKSPACE cannot occur.
 */
#define SHN_STATIC_MAX_CHUNKS 524288u
uint64_t shn_encode_static_max_chunks(void);
int shn_encode_static(const uint8_t* d_in, const shn_segment* h_segs, uint32_t n_segs, const void* d_tables,
                      const shn_params* p, uint8_t* d_out, size_t out_capacity, uint64_t* d_out_bytes,
                      uint32_t* d_status, void* stream);

/*
 * Copy the device status word of a workspace to the host. This call synchronises `stream`
 * (cudaStreamSynchronize) — it is the one synchronising entry point. h_detail (optional)
 * receives a hint: the global chunk index of the first failing chunk, or 0.
 */
int shn_get_device_status(const void* d_work, uint32_t* h_status, uint32_t* h_detail, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SHN_H */
