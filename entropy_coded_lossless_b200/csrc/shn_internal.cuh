// shn_internal.cuh — internal definitions shared by the libshn kernels and the C-ABI layer.
//
// The SHN1 stream layout and every table rule are those of the SHN1 format specification,
// which restates the Shannonic method ("Shannonic: Efficient Entropy-Optimal
// Compression for ML Workloads", MLSys 2026 notes, §4.1 preprocessing and §4.2 Algorithm 2).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/shn.h"

namespace shn {

// ---- stream layout (SHN1 format §6) -------------------------------------------------------------
constexpr uint32_t kMagic = 0x314E4853u;  // "SHN1"
constexpr uint32_t kHeaderBytes = 64;
constexpr uint32_t kSegDescBytes = 32;

__host__ __device__ inline uint64_t round_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }
__host__ __device__ inline uint32_t table_record_bytes(uint32_t K) { return (uint32_t)round_up(3ull * K, 4); }
__host__ __device__ inline uint64_t index_offset(uint32_t n_segs, uint32_t K) {
  return kHeaderBytes + (uint64_t)kSegDescBytes * n_segs + (uint64_t)table_record_bytes(K) * n_segs;
}
__host__ __device__ inline uint64_t payload_offset(uint32_t n_segs, uint32_t K, uint64_t total_chunks) {
  return round_up(index_offset(n_segs, K) + 4ull * total_chunks, 16);
}
__host__ __device__ inline uint64_t n_chunks(uint64_t n, uint32_t C) { return (n + C - 1) / C; }
// Words of a chunk of c symbols in the worst case: S states + c fields of <= R+8 bits + sentinel.
__host__ __device__ inline uint64_t chunk_max_words(uint32_t S, uint32_t R, uint64_t c) {
  return ((uint64_t)S * R + c * (uint64_t)(R + 8) + 1 + 31) / 32;
}

// ---- which symbols a chunk holds (SHN1 format §6) -----------------------------------------------
// Chunks come in groups of up to 32; a group's symbols are cut into 16-symbol pieces dealt round
// robin to its chunks. Chunk c of a segment of n symbols: group base symbol, index j in the group,
// stride m (chunks in the group), number of pieces, and the length of its last piece (1..16).
struct ChunkGeo {
  uint32_t base;      // first symbol of the group (relative to the segment)
  uint32_t j;         // chunk index within the group
  uint32_t m;         // chunks in the group: piece k of this chunk starts at base + 16*(j + k*m)
  uint32_t pieces;
  uint32_t last_len;  // symbols in the last piece
};

__host__ __device__ inline ChunkGeo chunk_geo(uint64_t n, uint32_t C, uint32_t c) {
  ChunkGeo g;
  const uint64_t nch = n_chunks(n, C);
  const uint32_t grp = c >> 5;
  g.j = c & 31u;
  g.m = (uint32_t)((nch - 32ull * grp) < 32 ? (nch - 32ull * grp) : 32);
  const uint64_t base = 32ull * grp * C;
  const uint64_t end = (32ull * (grp + 1) * C < n) ? 32ull * (grp + 1) * C : n;
  const uint32_t ng = (uint32_t)(end - base);
  const uint32_t P = (ng + 15) >> 4;
  g.base = (uint32_t)base;
  g.pieces = (P - g.j + g.m - 1) / g.m;
  g.last_len = (g.j + (g.pieces - 1) * g.m == P - 1) ? ng - 16 * (P - 1) : 16u;
  return g;
}

// ---- device table record (include/shn.h: shn_table) -----------------------------------------
// opaque part: uint2 sym[256] for every raw byte b (u = b ^ 0x80), range s, offset o = u - lo[s]:
//   .x = bias[s] + 2^22 + (o << (32 - w))   (w > 0; bias[s] alone in bits 0-19): (X + .x) >> 16
//        is nb + 64 with o's bits from bit 8 up, and the top w bits hold o,
//   .y = w | (start[s] + 4096) << 16   with start[s] = cumul_s - f_s; bit 7 marks a byte whose range
//        has no states (absent from the histogram the table was built from),
// then uint16 enc[L] holding the next state L + slot.
constexpr uint32_t kOpaqueSymOffset = 0;
constexpr uint32_t kOpaqueEncOffset = 2048;
static_assert(sizeof(shn_table) == SHN_TABLE_BYTES, "table record size");
static_assert(offsetof(shn_table, opaque) == SHN_TABLE_PUBLIC_BYTES, "table public size");

__device__ __forceinline__ const uint2* table_sym(const shn_table* t) {
  return reinterpret_cast<const uint2*>(t->opaque + kOpaqueSymOffset);
}
__device__ __forceinline__ const uint16_t* table_enc(const shn_table* t) {
  return reinterpret_cast<const uint16_t*>(t->opaque + kOpaqueEncOffset);
}

// SMs of the current device (grid sizing of the persistent kernels).
inline int sm_count_for_launch() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// Encoder block size: one thread per chunk, so also the chunks each encoder block codes. The host
// batching (block_start) and the encoder kernels both use it.
#ifndef ENC_THREADS
#define ENC_THREADS 256
#endif
constexpr int kEncBlockThreads = ENC_THREADS;
// Segments of at most kEncSmallMaxChunks chunks are coded by one-warp blocks with unreplicated
// tables (a few KB of shared memory), so that many small tensors share an SM.
constexpr int kEncSmallThreads = 32;
constexpr uint32_t kEncSmallMaxChunks = 64;

// ---- shared-memory accesses by 32-bit shared-window address ------------------------------------
// The per-symbol loops address their tables and rings with 32-bit shared addresses (no 64-bit
// generic-pointer arithmetic). The ring accessors are volatile with a memory clobber so they stay
// ordered after the cp.async waits and the __syncthreads that publish the data they read.
__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// ---- device status word (first 8 bytes of every workspace) -----------------------------------
struct DeviceStatus {
  uint32_t status;
  uint32_t detail;
};

__device__ __forceinline__ void report(DeviceStatus* st, uint32_t code, uint32_t detail) {
  if (atomicCAS(&st->status, 0u, code) == 0u) st->detail = detail;
}

// ---- SHN1 format §2 fixed-point log2: 24 fraction bits by repeated squaring -------------------
__device__ __forceinline__ uint32_t lg_fixed(uint32_t n) {
  if (n == 0) return 0;
  const int e = 31 - __clz(n);
  uint32_t m = n << (31 - e);  // mantissa in Q1.31: [2^31, 2^32)
  uint32_t frac = 0;
#pragma unroll
  for (int it = 0; it < 24; ++it) {
    // square, keep 31 fraction bits: p = m*m >> 31 (33 bits); the next bit is p >= 2, then halve
    const uint32_t hi = __umulhi(m, m), lo = m * m;
    const uint32_t bit = hi >> 31;
    m = bit ? hi : __funnelshift_l(lo, hi, 1);
    frac = (frac << 1) | bit;
  }
  return ((uint32_t)e << 24) | frac;
}

// ---- segment batches passed by value to kernels (no device allocation) ---------------------
constexpr int kSegBatch = 512;

struct HistBatch {
  uint32_t n;                      // segments in this batch
  uint32_t total_blocks;           // blocks of the launch
  uint64_t offset[kSegBatch];      // byte offset in d_in
  uint32_t length[kSegBatch];      // bytes
  uint32_t block_start[kSegBatch]; // first block of each segment
  uint32_t hist_index[kSegBatch];  // histogram row of each segment
  uint32_t bytes_per_block;        // input bytes per block (histogram_bytes_per_block)
};

struct EncBatch {
  uint32_t n;
  uint32_t total_blocks;
  uint32_t small;                  // 1: kEncSmallThreads-thread blocks, unreplicated tables
  uint64_t offset[kSegBatch];      // byte offset in d_in
  uint64_t out_offset[kSegBatch];  // sum of the lengths of all earlier segments
  uint32_t length[kSegBatch];
  uint32_t first_chunk[kSegBatch]; // global chunk index
  uint32_t block_start[kSegBatch];
  uint32_t seg_index[kSegBatch];   // segment / table index
};

// Host checks shared by shn_encode and shn_encode_static (capi.cu): parameters, segments (each
// shorter than 2^32 symbols, fewer than 2^32 chunks in all) and the worst-case stream size, which
// must stay within 16 GiB because chunk word offsets inside a payload are 32-bit. Returns SHN_OK or
// SHN_ERR_INVALID_ARG; on success the chunk and symbol totals. No CUDA call.
int check_encode_args(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs, uint64_t* total_chunks,
                      uint64_t* total_symbols);
// Fills b with the encoder batch that starts at segment s0: up to kSegBatch consecutive segments of
// one kind (segments of at most kEncSmallMaxChunks chunks are coded by one-warp blocks with
// unreplicated tables, the others by kEncBlockThreads-thread blocks). chunk and out_off are the
// global chunk index and output offset of segment s0, advanced past the batch. Returns the first
// segment after the batch. Both encoder entry points build their launches with it.
uint32_t fill_encode_batch(const shn_params& p, const shn_segment* h_segs, uint32_t n_segs, uint32_t s0,
                           uint64_t& chunk, uint64_t& out_off, EncBatch& b);

// Launch wrappers (defined in the .cu files; return a cudaError_t).
cudaError_t launch_histogram(const uint8_t* d_in, const HistBatch& b, uint64_t* d_hist, int threads,
                             cudaStream_t s);
uint32_t histogram_bytes_per_block(uint64_t batch_bytes, int sm_count);
uint32_t histogram_blocks_for(uint64_t length, uint32_t bytes_per_block);
cudaError_t launch_build_tables(const uint64_t* d_hist, uint32_t n_tables, const shn_params& p,
                                shn_table* d_tables, cudaStream_t s);

struct EncodeLayout {
  uint32_t n_segs;
  uint32_t K, R, S, C;
  uint64_t total_chunks;
  uint64_t total_symbols;
  uint64_t index_offset;
  uint64_t payload_offset;
  uint64_t out_capacity;
};

// Workspace layout of shn_encode: [status 256 B][chunk words u32 x total_chunks, padded]
// [global word offsets u64 x (total_chunks+1)][block partial sums u64 x n_blocks+1]
struct EncodeWork {
  DeviceStatus* status;
  uint32_t* chunk_words;
  unsigned long long* word_offset;  // exclusive prefix over all chunks, total at [total_chunks]
  unsigned long long* block_sums;
  uint32_t scan_blocks;
  uint32_t* slots;       // single-pass mode: chunk g's words at slots + g * slot_words (else null)
  uint32_t slot_words;   // worst-case words per chunk, a multiple of 4
};
constexpr uint32_t kScanBlock = 1024;  // chunks reduced per scan block

cudaError_t launch_encode_sizes(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                const EncodeLayout& lay, const EncodeWork& w, int threads, cudaStream_t s);
cudaError_t launch_scan(const EncodeWork& w, uint64_t total_chunks, cudaStream_t s);
cudaError_t launch_encode_header(const EncBatch& b, const shn_table* d_tables, const EncodeLayout& lay,
                                 const EncodeWork& w, uint8_t* d_out, uint64_t* d_out_bytes, bool first_batch,
                                 cudaStream_t s);
cudaError_t launch_encode_empty(const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, uint64_t* d_out_bytes,
                                cudaStream_t s);
cudaError_t launch_encode_write(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, bool slots,
                                cudaStream_t s);
cudaError_t launch_encode_compact(const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, int sm_count,
                                  cudaStream_t s);

cudaError_t launch_decode(const uint8_t* d_comp, uint64_t comp_bytes, const shn_params& p, DeviceStatus* st,
                          uint8_t* d_out, uint64_t out_capacity, int sm_count, cudaStream_t s);
cudaError_t launch_decode_bf16(const uint8_t* d_comp, uint64_t comp_bytes, const shn_params& p, DeviceStatus* st,
                               uint16_t* d_out, uint64_t out_elems, const float* d_scales, uint32_t log2_group,
                               uint64_t n_scales, int sm_count, cudaStream_t s);

}  // namespace shn
