// encode.cu — chunk-parallel Shannonic/tANS encoder (Shannonic §4.2, Algorithm 2).
//
// Per value x (symbol u = x ^ 0x80): s = rangeId[u]; emit the offset u - base[s] in nb[s] bits;
// emit the low state bits that renormalise X for s (count = (X + bias[s]) >> 16); move X through
// encTable[start[s] + (X >> nb)]. Only table lookups, shifts, masks and adds (§4.2: no multiply or
// divide on the critical path). Chunks of C symbols are independent (FORMAT.md §7): one thread
// encodes one chunk backwards with S interleaved states.
//
// The stream position of a chunk depends on the sizes of all chunks before it, so encoding runs
// in passes: (1) every thread runs its chunk's state machine and records the chunk's word count,
// (2) an exclusive scan turns counts into word offsets, (3) the header, segment descriptors, table
// records and chunk index are written, (4) every thread re-runs its chunk and writes the words to
// their final place. No device-wide spin waits; everything is ordered by the stream.
#include "shn_internal.cuh"

namespace shn {

constexpr int kEncThreads = 128;

struct EncSmem {
  uint2 sym[256];
  uint16_t enc[4096];
};

__device__ __forceinline__ void load_tables(EncSmem& sm, const shn_table* t, uint32_t L) {
  const uint2* sym = table_sym(t);
  const uint16_t* enc = table_enc(t);
  for (int i = threadIdx.x; i < 256; i += blockDim.x) sm.sym[i] = sym[i];
  for (uint32_t i = threadIdx.x; i < L; i += blockDim.x) sm.enc[i] = enc[i];
}

// Segment of this block: largest s with block_start[s] <= blockIdx.x.
__device__ __forceinline__ int block_segment(const EncBatch& b) {
  int lo = 0, hi = (int)b.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.block_start[mid] <= blockIdx.x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Bit sink of the write pass: LSB-first appends, 32-bit words stored as they fill.
struct WordWriter {
  uint32_t* out;
  uint32_t* end;  // first word past this chunk (the size pass counted exactly this many)
  unsigned long long acc;
  uint32_t cnt;
  __device__ __forceinline__ void put(uint32_t v, uint32_t n) {
    acc |= (unsigned long long)v << cnt;
    cnt += n;
    if (cnt >= 32) {
      if (out < end) *out = (uint32_t)acc;
      ++out;
      acc >>= 32;
      cnt -= 32;
    }
  }
};

// One encoder step for symbol byte b in state X. Returns the field (offset low, state bits high)
// and its width; updates X.
__device__ __forceinline__ uint32_t enc_step(const EncSmem& sm, uint32_t b, uint32_t& X, uint32_t& width,
                                             uint32_t& flags) {
  const uint2 e = sm.sym[b];
  const uint32_t nb = (X + e.x) >> 16;
  const uint32_t w = (e.y >> 24) & 15u;
  const uint32_t o = (e.y >> 16) & 0xFFu;
  const uint32_t r = X & ((1u << nb) - 1u);
  X = sm.enc[(e.y & 0xFFFFu) - 4096u + (X >> nb)];
  flags |= e.y;
  width = w + nb;
  return o | (r << w);
}

// Encode one chunk backwards (FORMAT.md §7). seg points at the segment's first byte; the chunk's
// symbols are its pieces in order (FORMAT.md §6), so the last piece is coded first. Full pieces are
// read as 16-byte loads, which a warp's 32 chunks of one group issue as 512 consecutive bytes.
template <int S, bool WRITE>
__device__ __forceinline__ void encode_chunk(const EncSmem& sm, const uint8_t* seg, const ChunkGeo& g, uint32_t L,
                                             uint32_t R, uint64_t& bits_out, uint32_t& flags, WordWriter* ww) {
  uint32_t X[S];
#pragma unroll
  for (int q = 0; q < S; ++q) X[q] = L;
  uint64_t bits = 0;
  int k = (int)g.pieces - 1;
  if (g.last_len < 16) {  // the group's short last piece, symbol by symbol
    const uint8_t* src = seg + g.base + 16u * (g.j + (uint32_t)k * g.m);
    for (int t = (int)g.last_len - 1; t >= 0; --t) {
      const int q = t & (S - 1);  // chunk index 16k + t, and S divides 16
      uint32_t Xq = X[0];
#pragma unroll
      for (int z = 1; z < S; ++z)
        if (z == q) Xq = X[z];
      uint32_t w;
      const uint32_t field = enc_step(sm, src[t], Xq, w, flags);
#pragma unroll
      for (int z = 0; z < S; ++z)
        if (z == q) X[z] = Xq;
      bits += w;
      if (WRITE) ww->put(field, w);
    }
    --k;
  }
  const bool aligned = ((reinterpret_cast<uintptr_t>(seg + g.base) & 15u) == 0);
  for (; k >= 0; --k) {
    const uint8_t* src = seg + g.base + 16u * (g.j + (uint32_t)k * g.m);
    uint32_t wv[4];
    if (aligned) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(src));
      wv[0] = v.x;
      wv[1] = v.y;
      wv[2] = v.z;
      wv[3] = v.w;
    } else {
#pragma unroll
      for (int z = 0; z < 4; ++z)
        wv[z] = (uint32_t)src[4 * z] | ((uint32_t)src[4 * z + 1] << 8) | ((uint32_t)src[4 * z + 2] << 16) |
                ((uint32_t)src[4 * z + 3] << 24);
    }
#pragma unroll
    for (int r = 15; r >= 0; --r) {
      const uint32_t b = (wv[r >> 2] >> (8 * (r & 3))) & 0xFFu;
      uint32_t w;
      const uint32_t field = enc_step(sm, b, X[r & (S - 1)], w, flags);
      bits += w;
      if (WRITE) ww->put(field, w);
    }
  }
#pragma unroll
  for (int q = 0; q < S; ++q) {
    if (WRITE) ww->put(X[q] - L, R);
  }
  bits_out = bits;
}

template <int S>
__global__ void __launch_bounds__(kEncThreads) encode_sizes_kernel(const uint8_t* __restrict__ in,
                                                                   const __grid_constant__ EncBatch b,
                                                                   const shn_table* __restrict__ tables,
                                                                   const EncodeLayout lay, EncodeWork w) {
  __shared__ EncSmem sm;
  const int seg = block_segment(b);
  const shn_table* t = tables + b.seg_index[seg];
  const uint32_t L = 1u << lay.R;
  load_tables(sm, t, L);
  __syncthreads();
  const uint32_t c = (blockIdx.x - b.block_start[seg]) * kEncThreads + threadIdx.x;
  const uint32_t len_seg = b.length[seg];
  const uint32_t nch = (uint32_t)n_chunks(len_seg, lay.C);
  if (c >= nch) return;
  const ChunkGeo geo = chunk_geo(len_seg, lay.C, c);
  uint64_t bits = 0;
  uint32_t flags = 0;
  encode_chunk<S, false>(sm, in + b.offset[seg], geo, L, lay.R, bits, flags, nullptr);
  const uint64_t total = bits + (uint64_t)S * lay.R + 1;
  w.chunk_words[b.first_chunk[seg] + c] = (uint32_t)((total + 31) >> 5);
  if ((flags & 0x80000000u) || t->status != 0) report(w.status, SHN_ERR_INVALID_ARG, b.first_chunk[seg] + c);
}

template <int S>
__global__ void __launch_bounds__(kEncThreads) encode_write_kernel(const uint8_t* __restrict__ in,
                                                                   const __grid_constant__ EncBatch b,
                                                                   const shn_table* __restrict__ tables,
                                                                   const EncodeLayout lay, EncodeWork w,
                                                                   uint8_t* __restrict__ out) {
  if (*(volatile uint32_t*)&w.status->status != 0) return;
  __shared__ EncSmem sm;
  const int seg = block_segment(b);
  const shn_table* t = tables + b.seg_index[seg];
  const uint32_t L = 1u << lay.R;
  load_tables(sm, t, L);
  __syncthreads();
  const uint32_t c = (blockIdx.x - b.block_start[seg]) * kEncThreads + threadIdx.x;
  const uint32_t len_seg = b.length[seg];
  const uint32_t nch = (uint32_t)n_chunks(len_seg, lay.C);
  if (c >= nch) return;
  const ChunkGeo geo = chunk_geo(len_seg, lay.C, c);
  const uint64_t g = (uint64_t)b.first_chunk[seg] + c;
  WordWriter ww;
  ww.out = reinterpret_cast<uint32_t*>(out + lay.payload_offset) + w.word_offset[g];
  ww.end = reinterpret_cast<uint32_t*>(out + lay.payload_offset) + w.word_offset[g + 1];
  ww.acc = 0;
  ww.cnt = 0;
  uint64_t bits = 0;
  uint32_t flags = 0;
  encode_chunk<S, true>(sm, in + b.offset[seg], geo, L, lay.R, bits, flags, &ww);
  ww.put(1u, 1u);  // sentinel
  if (ww.cnt > 0 && ww.out < ww.end) *ww.out = (uint32_t)ww.acc;
}

// ---- exclusive scan of the chunk word counts (3 small kernels, no inter-block waits) ----------
__global__ void scan_reduce_kernel(const uint32_t* __restrict__ v, uint64_t n, unsigned long long* __restrict__ sums) {
  __shared__ unsigned long long red[32];
  const uint64_t base = (uint64_t)blockIdx.x * kScanBlock;
  unsigned long long s = 0;
  for (uint32_t i = threadIdx.x; i < kScanBlock; i += blockDim.x)
    if (base + i < n) s += v[base + i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0ull;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) sums[blockIdx.x] = s;
  }
}

// Exclusive scan of `n` values in place by one block of 1024 threads, tile by tile.
__global__ void __launch_bounds__(1024) scan_sums_kernel(unsigned long long* __restrict__ sums, uint32_t n) {
  __shared__ unsigned long long warp_tot[32];
  __shared__ unsigned long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (uint32_t base = 0; base < n; base += 1024) {
    const uint32_t i = base + threadIdx.x;
    const unsigned long long v = (i < n) ? sums[i] : 0ull;
    unsigned long long x = v;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
      unsigned long long t = warp_tot[lane];
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    const unsigned long long before = carry + (wid > 0 ? warp_tot[wid - 1] : 0ull) + (x - v);
    if (i < n) sums[i] = before;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_tot[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) sums[n] = carry;
}

__global__ void __launch_bounds__(kScanBlock) scan_apply_kernel(const uint32_t* __restrict__ v, uint64_t n,
                                                                const unsigned long long* __restrict__ sums,
                                                                unsigned long long* __restrict__ out) {
  __shared__ unsigned long long warp_tot[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const uint64_t i = (uint64_t)blockIdx.x * kScanBlock + threadIdx.x;
  const unsigned long long val = (i < n) ? v[i] : 0ull;
  unsigned long long x = val;
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[wid] = x;
  __syncthreads();
  if (wid == 0) {
    unsigned long long t = warp_tot[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  const unsigned long long excl = sums[blockIdx.x] + (wid > 0 ? warp_tot[wid - 1] : 0ull) + (x - val);
  if (i < n) out[i] = excl;
  if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) out[n] = sums[gridDim.x];
}

// ---- header, descriptors, table records, chunk index (FORMAT.md §6) -------------------------
__device__ __forceinline__ void st16(uint8_t* p, uint32_t v) {
  p[0] = (uint8_t)v;
  p[1] = (uint8_t)(v >> 8);
}
__device__ __forceinline__ void st32(uint8_t* p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
__device__ __forceinline__ void st64(uint8_t* p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i));
}

__global__ void encode_header_kernel(const __grid_constant__ EncBatch b, const shn_table* __restrict__ tables,
                                     const EncodeLayout lay, EncodeWork w, uint8_t* __restrict__ out,
                                     unsigned long long* __restrict__ out_bytes, uint32_t is_first_batch) {
  const unsigned long long total_words = w.word_offset[lay.total_chunks];
  const uint64_t stream_bytes = round_up(lay.payload_offset + 4ull * total_words, 16);
  const bool fits = stream_bytes <= lay.out_capacity;
  if (blockIdx.x == 0) {
    if (is_first_batch && threadIdx.x == 0) {
      *out_bytes = stream_bytes;
      if (!fits) report(w.status, SHN_ERR_CAPACITY, 0);
    }
    if (is_first_batch && threadIdx.x == 0 && fits) {
      st32(out + 0, kMagic);
      st16(out + 4, 1);
      st16(out + 6, kHeaderBytes);
      st32(out + 8, lay.n_segs);
      st16(out + 12, lay.K);
      out[14] = (uint8_t)lay.R;
      out[15] = (uint8_t)lay.S;
      st32(out + 16, lay.C);
      st32(out + 20, table_record_bytes(lay.K));
      st64(out + 24, lay.total_symbols);
      st64(out + 32, lay.total_chunks);
      st64(out + 40, lay.index_offset);
      st64(out + 48, lay.payload_offset);
      st64(out + 56, stream_bytes);
      for (uint64_t q = lay.index_offset + 4 * lay.total_chunks; q < lay.payload_offset; ++q) out[q] = 0;
      for (uint64_t q = lay.payload_offset + 4ull * total_words; q < stream_bytes; ++q) out[q] = 0;
    }
    if (!fits) return;
    const uint32_t tb = table_record_bytes(lay.K);
    for (uint32_t s = threadIdx.x; s < b.n; s += blockDim.x) {
      const uint32_t si = b.seg_index[s];
      const uint64_t first = b.first_chunk[s];
      const uint64_t nch = n_chunks(b.length[s], lay.C);
      uint8_t* d = out + kHeaderBytes + (uint64_t)kSegDescBytes * si;
      st64(d + 0, b.length[s]);
      st64(d + 8, b.out_offset[s]);
      st64(d + 16, 4ull * w.word_offset[first]);
      st32(d + 24, (uint32_t)(w.word_offset[first + nch] - w.word_offset[first]));
      st32(d + 28, (uint32_t)first);
      const shn_table* t = tables + si;
      uint8_t* rec = out + kHeaderBytes + (uint64_t)kSegDescBytes * lay.n_segs + (uint64_t)tb * si;
      for (uint32_t k = 0; k < lay.K; ++k) {
        st16(rec + 2 * k, t->f[k]);
        rec[2 * lay.K + k] = t->lo[k];
      }
      for (uint32_t q = 3 * lay.K; q < tb; ++q) rec[q] = 0;
    }
    return;
  }
  if (!fits) return;
  // chunk index entries of this batch's chunks: one thread per chunk
  const uint64_t first0 = b.first_chunk[0];
  const uint64_t last = (uint64_t)b.first_chunk[b.n - 1] + n_chunks(b.length[b.n - 1], lay.C);
  const uint64_t g = first0 + (uint64_t)(blockIdx.x - 1) * blockDim.x + threadIdx.x;
  if (g >= last) return;
  int lo = 0, hi = (int)b.n - 1;  // segment of chunk g
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.first_chunk[mid] <= g) lo = mid;
    else hi = mid - 1;
  }
  st32(out + lay.index_offset + 4 * g, (uint32_t)(w.word_offset[g] - w.word_offset[b.first_chunk[lo]]));
}

template <int S>
static cudaError_t launch_sizes_t(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                  const EncodeLayout& lay, const EncodeWork& w, cudaStream_t s) {
  encode_sizes_kernel<S><<<b.total_blocks, kEncThreads, 0, s>>>(d_in, b, d_tables, lay, w);
  return cudaGetLastError();
}
template <int S>
static cudaError_t launch_write_t(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                  const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, cudaStream_t s) {
  encode_write_kernel<S><<<b.total_blocks, kEncThreads, 0, s>>>(d_in, b, d_tables, lay, w, d_out);
  return cudaGetLastError();
}

cudaError_t launch_encode_sizes(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                const EncodeLayout& lay, const EncodeWork& w, int, cudaStream_t s) {
  if (b.total_blocks == 0) return cudaSuccess;
  switch (lay.S) {
    case 1: return launch_sizes_t<1>(d_in, b, d_tables, lay, w, s);
    case 2: return launch_sizes_t<2>(d_in, b, d_tables, lay, w, s);
    case 4: return launch_sizes_t<4>(d_in, b, d_tables, lay, w, s);
    case 8: return launch_sizes_t<8>(d_in, b, d_tables, lay, w, s);
    case 16: return launch_sizes_t<16>(d_in, b, d_tables, lay, w, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_encode_write(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, int,
                                cudaStream_t s) {
  if (b.total_blocks == 0) return cudaSuccess;
  switch (lay.S) {
    case 1: return launch_write_t<1>(d_in, b, d_tables, lay, w, d_out, s);
    case 2: return launch_write_t<2>(d_in, b, d_tables, lay, w, d_out, s);
    case 4: return launch_write_t<4>(d_in, b, d_tables, lay, w, d_out, s);
    case 8: return launch_write_t<8>(d_in, b, d_tables, lay, w, d_out, s);
    case 16: return launch_write_t<16>(d_in, b, d_tables, lay, w, d_out, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_scan(const EncodeWork& w, uint64_t total_chunks, cudaStream_t s) {
  const uint32_t nb = (uint32_t)((total_chunks + kScanBlock - 1) / kScanBlock);
  if (nb == 0) {
    cudaError_t e = cudaMemsetAsync(w.word_offset, 0, sizeof(unsigned long long), s);
    return e;
  }
  scan_reduce_kernel<<<nb, 256, 0, s>>>(w.chunk_words, total_chunks, w.block_sums);
  scan_sums_kernel<<<1, 1024, 0, s>>>(w.block_sums, nb);
  scan_apply_kernel<<<nb, kScanBlock, 0, s>>>(w.chunk_words, total_chunks, w.block_sums, w.word_offset);
  return cudaGetLastError();
}

// A stream without segments is its 64-byte header alone.
__global__ void encode_empty_kernel(const EncodeLayout lay, EncodeWork w, uint8_t* __restrict__ out,
                                    unsigned long long* __restrict__ out_bytes) {
  if (threadIdx.x != 0) return;
  *out_bytes = kHeaderBytes;
  if (lay.out_capacity < kHeaderBytes) {
    report(w.status, SHN_ERR_CAPACITY, 0);
    return;
  }
  for (int q = 0; q < (int)kHeaderBytes; ++q) out[q] = 0;
  st32(out + 0, kMagic);
  st16(out + 4, 1);
  st16(out + 6, kHeaderBytes);
  st16(out + 12, lay.K);
  out[14] = (uint8_t)lay.R;
  out[15] = (uint8_t)lay.S;
  st32(out + 16, lay.C);
  st32(out + 20, table_record_bytes(lay.K));
  st64(out + 40, kHeaderBytes);
  st64(out + 48, kHeaderBytes);
  st64(out + 56, kHeaderBytes);
}

cudaError_t launch_encode_empty(const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, uint64_t* d_out_bytes,
                                cudaStream_t s) {
  encode_empty_kernel<<<1, 32, 0, s>>>(lay, w, d_out, reinterpret_cast<unsigned long long*>(d_out_bytes));
  return cudaGetLastError();
}

cudaError_t launch_encode_header(const EncBatch& b, const shn_table* d_tables, const EncodeLayout& lay,
                                 const EncodeWork& w, uint8_t* d_out, uint64_t* d_out_bytes, bool first_batch,
                                 cudaStream_t s) {
  if (b.n == 0) return cudaSuccess;
  const uint64_t first0 = b.first_chunk[0];
  const uint64_t last = (uint64_t)b.first_chunk[b.n - 1] + n_chunks(b.length[b.n - 1], lay.C);
  const uint32_t blocks = 1 + (uint32_t)((last - first0 + 255) / 256);
  encode_header_kernel<<<blocks, 256, 0, s>>>(b, d_tables, lay, w, d_out,
                                              reinterpret_cast<unsigned long long*>(d_out_bytes),
                                              first_batch ? 1u : 0u);
  return cudaGetLastError();
}

}  // namespace shn
