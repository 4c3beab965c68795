// encode.cu — chunk-parallel Shannonic/tANS encoder (Shannonic §4.2, Algorithm 2).
//
// Per value x (symbol u = x ^ 0x80): s = rangeId[u]; emit the offset u - base[s] in nb[s] bits;
// emit the low state bits that renormalise X for s; move X through encTable (§4.2: table lookups,
// shifts, masks and adds only). Chunks are independent (SHN1 format §7): one thread encodes one chunk
// backwards with S interleaved states.
//
// The stream position of a chunk depends on the sizes of all chunks before it. With a workspace
// large enough for one worst-case slot per chunk the state machine runs once: (1) every thread codes
// its chunk into its slot and records the word count, (2) an exclusive scan turns counts into word
// offsets, (3) the header, segment descriptors, table records and chunk index are written, (4) one
// warp per chunk moves the slot to its final place. With the minimal workspace it runs twice:
// (1) counts only, (2), (3), then (4) every thread re-runs its chunk and writes the words in place.
// No device-wide spin waits; everything is ordered by the stream.
//
// Shared-memory tables. Each block codes chunks of one segment and keeps Algorithm 2's per-range
// form in shared memory: sym[raw byte] = {bias + 2^22 with the offset in the top w bits,
// w | (start + 4096) << 16} (bit 7 of .y marks a byte absent from the table's histogram), and
// enc[L] (next state). The layout serves the ALU pipe, which bounds this loop: w sits where a shift
// reads its amount, and one funnel shift of the state bits into .x appends the offset below them,
// so a symbol's field costs one instruction instead of an extraction, a shift and an OR. A warp's 32
// lookups use 32 unrelated indices, so both tables are stored lane-interleaved: sym 16 times
// ([byte][16] x 8 bytes: an 8-byte load is served per half-warp, so the 16 lanes of a phase always
// hit 16 distinct bank pairs) and enc in up to 8 KB of copies ([index][copies] x 4-byte slots; 16
// copies at L = 128, so lanes l and l + 16 share one and may meet on a bank: measured 0.9 % faster
// than 32 conflict-free copies, the smaller table being quicker to stage into every block). Segments
// of at most 64 chunks use one-warp blocks and a single copy of each table instead (small tensors,
// many per SM).
#include "shn_internal.cuh"

namespace shn {

#ifndef ENC_AHEAD
#define ENC_AHEAD 2
#endif
constexpr int kEncThreads = kEncBlockThreads;
constexpr int kEncAhead = ENC_AHEAD;  // input pieces in flight while one is coded
constexpr uint32_t kSymCopies = 16;
constexpr uint32_t kEncCopyBudget = 8192;         // bytes for the replicated next-state table
constexpr uint32_t kRingWords = 16;               // per-thread output staging ring (write pass)
constexpr uint32_t kRingStride = kRingWords + 4;  // 80-byte rows: 16-byte reads of 8 rows hit distinct banks

#ifndef ENC_SLOT_BYTES
#define ENC_SLOT_BYTES 4
#endif
// Bytes per next-state entry copy: 4 gives every lane its own bank (2 would pack two lanes' copies
// into one bank word, where lanes 2j and 2j+1 can conflict; measured slower).
constexpr uint32_t kEncSlot = ENC_SLOT_BYTES;
__host__ __device__ inline uint32_t enc_copies(uint32_t R) {
  uint32_t c = 32;
  while (c > 1 && (kEncSlot << R) * c > kEncCopyBudget) c >>= 1;
  return c;
}
__host__ __device__ inline uint32_t enc_table_smem_bytes(uint32_t R, bool plain = false) {
  return plain ? 256 * 8 + (kEncSlot << R) : 256 * kSymCopies * 8 + (kEncSlot << R) * enc_copies(R);
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

// Algorithm 2 per symbol, on the lane-interleaved tables. State X in [L, 2L). Addresses are 32-bit
// shared-window addresses.
// PLAIN: one copy of each table (small segments; lanes may conflict on a bank).
template <bool PLAIN>
struct Coder {
  static constexpr uint32_t kSymRow = PLAIN ? 8u : kSymCopies * 8u;  // bytes per raw-byte row of sym
  uint32_t sym;      // this lane's column of sym: + raw byte * kSymRow
  uint32_t enc;      // this lane's column of enc, biased by -4096 rows (the +4096 in .y's start field)
  uint32_t enc_row;  // bytes per enc index (2 * copies)
  uint32_t L;
  uint32_t absent;   // bit 7 set if a byte this thread staged has no states in the table
  // Returns the symbol's fields (offset low, state bits above it); width = their total bit count in
  // bits 0-5 (bit 5 clear), with junk above bit 5 that the bit counters ignore.
  // CHECK: accumulate .y into flags (bit 7 set for a byte absent from the table's histogram).
  // Every variable shift is a funnel shift, which uses its amount modulo 32: nb and w come with
  // junk above bit 5 (see the entry layout), and no instruction is spent clearing it.
  template <bool CHECK>
  __device__ __forceinline__ uint32_t step(uint32_t b, uint32_t& X, uint32_t& width, uint32_t& flags) const {
    const uint2 e = lds64(sym + b * kSymRow);
    const uint32_t nb = (X + e.x) >> 16;                 // nb + 64, offset bits from bit 8
    const uint32_t q = __funnelshift_r(X, 0u, nb);       // X >> nb
    const uint32_t r = X - __funnelshift_l(0u, q, nb);   // the nb low state bits
    X = lds_u16(enc + ((e.y >> 16) + q) * enc_row);
    if (CHECK) flags |= e.y;
    width = e.y + nb;                                    // w + nb in bits 0-4
    return __funnelshift_l(e.x, r, e.y);                 // (r << w) | offset (the top w bits of .x)
  }
};

// Returns whether every offset field this thread copied fits beside R state bits in 16 bits (the
// block-wide AND of it decides whether two symbols' fields can share one 32-bit append).
template <bool PLAIN>
__device__ __forceinline__ bool load_coder(unsigned char* smem, const shn_table* t, uint32_t R, Coder<PLAIN>& cd) {
  const uint32_t L = 1u << R;
  const uint32_t copies = PLAIN ? 1u : enc_copies(R);
  const uint32_t sym_copies = PLAIN ? 1u : kSymCopies;
  const uint2* sym = table_sym(t);
  const uint16_t* enc = table_enc(t);
  uint2* s2 = reinterpret_cast<uint2*>(smem);
  unsigned char* e2 = smem + 256 * sym_copies * 8;
  bool narrow = true;
  cd.absent = 0;
  for (uint32_t i = threadIdx.x; i < 256 * sym_copies; i += blockDim.x) {
    const uint2 e = sym[i / sym_copies];
    s2[i] = e;
    narrow = narrow && R + (e.y & 31u) <= 16;
    cd.absent |= e.y & 0x80u;
  }
  for (uint32_t i = threadIdx.x; i < L * copies; i += blockDim.x)
    *reinterpret_cast<uint16_t*>(e2 + i * kEncSlot) = enc[i / copies];
  const uint32_t lane = threadIdx.x & 31;
  cd.sym = smem_addr(smem) + (lane & (sym_copies - 1)) * 8;
  cd.enc_row = kEncSlot * copies;
  // entry e of copy c is at e2 + (e * copies + c) * kEncSlot
  cd.enc = smem_addr(e2) + (lane & (copies - 1)) * kEncSlot - 4096u * cd.enc_row;
  cd.L = L;
  return narrow;
}

// Run one chunk backwards (SHN1 format §6-§7), calling sink(field, width) for every field. seg points
// at the segment's first byte; the chunk's symbols are its pieces in order, so the last piece is
// coded first. Full pieces are 16-byte loads, which a warp's 32 chunks of one group issue as 512
// consecutive bytes.
template <int S, bool PAIRS, bool CHECK, class CoderT, class Sink>
__device__ __forceinline__ void code_chunk(const CoderT& cd, const uint8_t* seg, const ChunkGeo& g, uint32_t* st,
                                           uint32_t& flags, Sink& sink) {
  int k = (int)g.pieces - 1;
  if (g.last_len < 16) {  // the group's short last piece, symbol by symbol
    const uint8_t* src = seg + g.base + 16u * (g.j + (uint32_t)k * g.m);
    for (int t = (int)g.last_len - 1; t >= 0; --t) {
      const int q = t & (S - 1);  // chunk index 16k + t, and S divides 16
      uint32_t x = st[0];
#pragma unroll
      for (int z = 1; z < S; ++z)
        if (z == q) x = st[z];
      uint32_t w;
      const uint32_t field = cd.template step<CHECK>(src[t], x, w, flags);
#pragma unroll
      for (int z = 0; z < S; ++z)
        if (z == q) st[z] = x;
      sink(field, w);
    }
    --k;
    sink.piece_done();
  }
  const bool aligned = ((reinterpret_cast<uintptr_t>(seg + g.base) & 15u) == 0);
  const uint8_t* piece0 = seg + g.base + 16u * g.j;
  const uint32_t stride = 16u * g.m;
  auto load_piece = [&](int kk) -> uint4 {
    const uint8_t* src = piece0 + (uint32_t)kk * stride;
    if (aligned) return __ldcs(reinterpret_cast<const uint4*>(src));
    uint32_t v[4];
#pragma unroll
    for (int z = 0; z < 4; ++z)
      v[z] = (uint32_t)src[4 * z] | ((uint32_t)src[4 * z + 1] << 8) | ((uint32_t)src[4 * z + 2] << 16) |
             ((uint32_t)src[4 * z + 3] << 24);
    return make_uint4(v[0], v[1], v[2], v[3]);
  };
  auto code_piece = [&](const uint4 cur) {
    const uint32_t wv[4] = {cur.x, cur.y, cur.z, cur.w};
    if (PAIRS) {  // symbols r and r-1: their fields (<= 16 bits each) as one append
#pragma unroll
      for (int r = 15; r >= 1; r -= 2) {
        const uint32_t b1 = __byte_perm(wv[r >> 2], 0u, 0x4440u + (uint32_t)(r & 3));
        const uint32_t b2 = __byte_perm(wv[(r - 1) >> 2], 0u, 0x4440u + (uint32_t)((r - 1) & 3));
        uint32_t w1, w2;
        const uint32_t f1 = cd.template step<CHECK>(b1, st[r & (S - 1)], w1, flags);
        const uint32_t f2 = cd.template step<CHECK>(b2, st[(r - 1) & (S - 1)], w2, flags);
        sink(f1 + __funnelshift_l(0u, f2, w1), w1 + w2);  // w1 modulo 32; the two fields do not overlap
      }
    } else {
#pragma unroll
      for (int r = 15; r >= 0; --r) {
        const uint32_t b = __byte_perm(wv[r >> 2], 0u, 0x4440u + (uint32_t)(r & 3));
        uint32_t w;
        const uint32_t field = cd.template step<CHECK>(b, st[r & (S - 1)], w, flags);
        sink(field, w);
      }
    }
    sink.piece_done();
  };
  // kEncAhead pieces are in flight while one is coded. The piece loop is unrolled by kEncAhead so
  // that every prefetch slot is a fixed set of registers: a slot is refilled right after it is
  // consumed, and no register copy ever waits on a load that was issued recently.
  uint4 pf[kEncAhead];
#pragma unroll
  for (int a = 0; a < kEncAhead; ++a) pf[a] = (k >= a) ? load_piece(k - a) : make_uint4(0, 0, 0, 0);
  while (k >= 0) {
#pragma unroll
    for (int a = 0; a < kEncAhead; ++a) {  // slot a holds piece k (the group's a-th)
      if (k >= 0) {
        const uint4 cur = pf[a];
        if (k >= kEncAhead) pf[a] = load_piece(k - kEncAhead);
        code_piece(cur);
        --k;
      }
    }
  }
}

struct BitCounter {
  uint32_t bits = 0;  // a chunk has at most 65536 fields of <= 20 bits
  // w: bit count in bits 0-5 (at most 32), junk above
  __device__ __forceinline__ void operator()(uint32_t, uint32_t w) { bits += w & 63u; }
  __device__ __forceinline__ void piece_done() {}
};

// Write-pass sink: LSB-first bit accumulator; complete words go to a per-thread ring in shared
// memory, and whole 16-byte-aligned groups of 4 words leave it as one 16-byte store.
struct RingWriter {
  uint32_t ring;         // shared address of this thread's row
  uint32_t* payload;     // stream payload, 16-byte aligned
  uint32_t wp, fp, end;  // next word to append, next word to store, end of this chunk (payload words)
  uint32_t a0;           // the bits not yet in the ring (cnt & 31 of them)
  uint32_t cnt;          // bits 0-5: bits pending in a0 (< 32 between appends); junk above bit 5
  __device__ __forceinline__ uint32_t slot(uint32_t word) const { return ring + (word & (kRingWords - 1)) * 4u; }
  // append the low (n & 63) <= 32 bits of v (junk in n above bit 5 is ignored); v < 2^(n & 63)
  __device__ __forceinline__ void operator()(uint32_t v, uint32_t n) {
    a0 += __funnelshift_l(0u, v, cnt);                  // v << (cnt & 31); a0 is zero from bit cnt & 31 up
    const uint32_t over = __funnelshift_l(v, 0u, cnt);  // bits of v beyond position 32 (0 when cnt & 31 == 0)
    cnt += n;                                            // bits 0-5: (cnt & 31) + (n & 63) <= 63, no carry out
    if (cnt & 32u) {
      sts32(slot(wp), a0);
      ++wp;
      a0 = over;
      cnt -= 32;
    }
  }
  __device__ __forceinline__ void piece_done() {
    while ((fp & 3u) != 0 && fp < wp) {  // unaligned head of the chunk
      if (fp < end) payload[fp] = lds32(slot(fp));
      ++fp;
    }
    while (fp + 4 <= wp) {
      if (fp + 4 <= end) *reinterpret_cast<uint4*>(payload + fp) = lds128(slot(fp));
      fp += 4;
    }
  }
  __device__ __forceinline__ void finish() {
    if (cnt & 31u) {
      sts32(slot(wp), a0);
      ++wp;
    }
    piece_done();
    for (; fp < wp; ++fp)
      if (fp < end) payload[fp] = lds32(slot(fp));
  }
};

// SMALL: kEncSmallThreads-thread blocks with unreplicated tables (segments of few chunks).
template <int S, bool PAIRS, bool SMALL>
__global__ void __launch_bounds__(SMALL ? kEncSmallThreads : kEncThreads) encode_sizes_kernel(
    const uint8_t* __restrict__ in, const __grid_constant__ EncBatch b, const shn_table* __restrict__ tables,
    const EncodeLayout lay, EncodeWork w) {
  constexpr int NT = SMALL ? kEncSmallThreads : kEncThreads;
  extern __shared__ __align__(16) unsigned char esm[];
  const int seg = block_segment(b);
  const shn_table* t = tables + b.seg_index[seg];
  Coder<SMALL> cd;
  const bool narrow = __syncthreads_and(load_coder(esm, t, lay.R, cd));
  const uint32_t c = (blockIdx.x - b.block_start[seg]) * NT + threadIdx.x;
  const uint32_t len_seg = b.length[seg];
  if (c >= (uint32_t)n_chunks(len_seg, lay.C)) return;
  const ChunkGeo geo = chunk_geo(len_seg, lay.C, c);
  uint32_t st[S];
#pragma unroll
  for (int q = 0; q < S; ++q) st[q] = cd.L;
  uint32_t flags = 0;
  BitCounter bc;
  if (PAIRS || narrow) code_chunk<S, true, true>(cd, in + b.offset[seg], geo, st, flags, bc);
  else code_chunk<S, false, true>(cd, in + b.offset[seg], geo, st, flags, bc);
  const uint64_t total = (uint64_t)bc.bits + (uint64_t)S * lay.R + 1;
  w.chunk_words[b.first_chunk[seg] + c] = (uint32_t)((total + 31) >> 5);
  if ((flags & 0x80u) || t->status != 0) report(w.status, SHN_ERR_INVALID_ARG, b.first_chunk[seg] + c);
}

// Writes every chunk's words. Two-pass mode (SLOTS = false): at the chunk's final place in the
// stream, from the word offsets of the scan. Single-pass mode (SLOTS = true): into the chunk's own
// worst-case-size slot in the workspace, recording the word count (and, as the size pass would,
// flagging symbols absent from the table); encode_compact_kernel then moves the slots into place.
template <int S, bool PAIRS, bool SLOTS, bool SMALL>
__global__ void __launch_bounds__(SMALL ? kEncSmallThreads : kEncThreads) encode_write_kernel(
    const uint8_t* __restrict__ in, const __grid_constant__ EncBatch b, const shn_table* __restrict__ tables,
    const EncodeLayout lay, EncodeWork w, uint8_t* __restrict__ out) {
  constexpr int NT = SMALL ? kEncSmallThreads : kEncThreads;
  // An error reported before this block started stops it. Another block of this launch may report
  // one at any time, so one thread reads the word and the barrier gives every thread its answer:
  // either all threads reach the barriers below or none does.
  if (__syncthreads_or(threadIdx.x == 0 && *(volatile uint32_t*)&w.status->status != 0)) return;
  extern __shared__ __align__(16) unsigned char esm[];
  const int seg = block_segment(b);
  const shn_table* t = tables + b.seg_index[seg];
  Coder<SMALL> cd;
  const bool narrow = __syncthreads_and(load_coder(esm, t, lay.R, cd));
  const bool any_absent = __syncthreads_or(cd.absent != 0);  // block-uniform
  const uint32_t c = (blockIdx.x - b.block_start[seg]) * NT + threadIdx.x;
  const uint32_t len_seg = b.length[seg];
  if (c >= (uint32_t)n_chunks(len_seg, lay.C)) return;
  const ChunkGeo geo = chunk_geo(len_seg, lay.C, c);
  const uint64_t g = (uint64_t)b.first_chunk[seg] + c;
  RingWriter rw;
  rw.ring = smem_addr(esm) + (uint32_t)round_up(enc_table_smem_bytes(lay.R, SMALL), 16) + threadIdx.x * (kRingStride * 4);
  if (SLOTS) {
    rw.payload = w.slots + g * w.slot_words;
    rw.wp = rw.fp = 0;
    rw.end = w.slot_words;
  } else {
    rw.payload = reinterpret_cast<uint32_t*>(out + lay.payload_offset);
    rw.wp = rw.fp = (uint32_t)w.word_offset[g];
    rw.end = (uint32_t)w.word_offset[g + 1];
  }
  rw.a0 = 0;
  rw.cnt = 0;
  uint32_t st[S];
#pragma unroll
  for (int q = 0; q < S; ++q) st[q] = cd.L;
  uint32_t flags = 0;
  if (SLOTS && any_absent) {  // the size pass is skipped: flag bytes absent from the table here
    if (PAIRS || narrow) code_chunk<S, true, true>(cd, in + b.offset[seg], geo, st, flags, rw);
    else code_chunk<S, false, true>(cd, in + b.offset[seg], geo, st, flags, rw);
  } else {
    if (PAIRS || narrow) code_chunk<S, true, false>(cd, in + b.offset[seg], geo, st, flags, rw);
    else code_chunk<S, false, false>(cd, in + b.offset[seg], geo, st, flags, rw);
  }
#pragma unroll
  for (int q = 0; q < S; ++q) rw(st[q] - cd.L, lay.R);
  rw(1u, 1u);  // sentinel
  rw.finish();
  if (SLOTS) {
    w.chunk_words[g] = rw.wp;
    if ((flags & 0x80u) || t->status != 0) report(w.status, SHN_ERR_INVALID_ARG, (uint32_t)g);
  }
}

// Single-pass mode: one warp per chunk moves its words from the slot (16-byte aligned) to the final
// place (4-byte aligned) in 16-byte pieces: lane l loads source quad j = j0 + l, takes quad j - 1
// from lane l - 1 (or from lane 31 of the previous round) and assembles destination quad j shifted
// by the destination's misalignment a; only the chunk's first and last destination quads, which it
// shares with its neighbours, are written word by word. The copy is bound by DRAM latency, so each
// lane issues kCompactLoads loads (32 * kCompactLoads quads per warp) before the first shuffle
// (measured on the 2 GiB KV cache: 6 in flight beat 1 by ~0.07 ms, 8 and 12 gave less).
constexpr int kCompactLoads = 6;
__global__ void __launch_bounds__(256) encode_compact_kernel(const EncodeLayout lay, EncodeWork w,
                                                             uint8_t* __restrict__ out) {
  if (*(volatile uint32_t*)&w.status->status != 0) return;
  uint32_t* payload = reinterpret_cast<uint32_t*>(out + lay.payload_offset);
  const uint32_t lane = threadIdx.x & 31;
  const uint64_t warps = (uint64_t)gridDim.x * (blockDim.x >> 5);
  for (uint64_t g = (uint64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); g < lay.total_chunks; g += warps) {
    const uint4* __restrict__ src = reinterpret_cast<const uint4*>(w.slots + g * w.slot_words);
    const uint64_t D = w.word_offset[g];
    const uint32_t n = w.chunk_words[g];  // >= 1 (the sentinel)
    const uint32_t a = (uint32_t)D & 3u;
    const uint64_t q0 = D >> 2;
    const uint32_t nq = (uint32_t)(((D + n - 1) >> 2) - q0 + 1);
    uint4 carry = make_uint4(0u, 0u, 0u, 0u);
    for (uint32_t j0 = 0; j0 < nq; j0 += 32 * kCompactLoads) {
      uint4 cur[kCompactLoads];
#pragma unroll
      for (int v = 0; v < kCompactLoads; ++v) {
        const uint32_t j = j0 + 32 * v + lane;
        cur[v] = (4 * j < n) ? __ldcs(src + j) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int v = 0; v < kCompactLoads; ++v) {
        const uint32_t j = j0 + 32 * v + lane;
        uint4 prv;
        prv.x = __shfl_up_sync(0xffffffffu, cur[v].x, 1);
        prv.y = __shfl_up_sync(0xffffffffu, cur[v].y, 1);
        prv.z = __shfl_up_sync(0xffffffffu, cur[v].z, 1);
        prv.w = __shfl_up_sync(0xffffffffu, cur[v].w, 1);
        if (lane == 0) prv = carry;
        carry.x = __shfl_sync(0xffffffffu, cur[v].x, 31);
        carry.y = __shfl_sync(0xffffffffu, cur[v].y, 31);
        carry.z = __shfl_sync(0xffffffffu, cur[v].z, 31);
        carry.w = __shfl_sync(0xffffffffu, cur[v].w, 31);
        if (j < nq) {
          uint4 o;
          switch (a) {  // warp-uniform
            case 0: o = cur[v]; break;
            case 1: o = make_uint4(prv.w, cur[v].x, cur[v].y, cur[v].z); break;
            case 2: o = make_uint4(prv.z, prv.w, cur[v].x, cur[v].y); break;
            default: o = make_uint4(prv.y, prv.z, prv.w, cur[v].x); break;
          }
          const uint64_t d0 = 4 * (q0 + j);  // first destination word of this quad
          if (d0 >= D && d0 + 4 <= D + n) {
            *reinterpret_cast<uint4*>(payload + d0) = o;
          } else {
            const uint32_t ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (d0 + t >= D && d0 + t < D + n) payload[d0 + t] = ov[t];
          }
        }
      }
    }
  }
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

// ---- header, descriptors, table records, chunk index (SHN1 format §6) -------------------------
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

template <int S, bool PAIRS, bool SMALL>
static cudaError_t launch_sizes_small_t(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                        const EncodeLayout& lay, const EncodeWork& w, cudaStream_t s) {
  const size_t smem = enc_table_smem_bytes(lay.R, SMALL);
  cudaError_t e = cudaFuncSetAttribute(encode_sizes_kernel<S, PAIRS, SMALL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  encode_sizes_kernel<S, PAIRS, SMALL><<<b.total_blocks, SMALL ? kEncSmallThreads : kEncThreads, smem, s>>>(
      d_in, b, d_tables, lay, w);
  return cudaGetLastError();
}
template <int S, bool PAIRS>
static cudaError_t launch_sizes_t(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                  const EncodeLayout& lay, const EncodeWork& w, cudaStream_t s) {
  return b.small ? launch_sizes_small_t<S, PAIRS, true>(d_in, b, d_tables, lay, w, s)
                 : launch_sizes_small_t<S, PAIRS, false>(d_in, b, d_tables, lay, w, s);
}
template <int S, bool PAIRS, bool SLOTS, bool SMALL>
static cudaError_t launch_write_small_t(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                        const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out,
                                        cudaStream_t s) {
  constexpr int NT = SMALL ? kEncSmallThreads : kEncThreads;
  const size_t smem = round_up(enc_table_smem_bytes(lay.R, SMALL), 16) + NT * kRingStride * 4;
  cudaError_t e = cudaFuncSetAttribute(encode_write_kernel<S, PAIRS, SLOTS, SMALL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  encode_write_kernel<S, PAIRS, SLOTS, SMALL><<<b.total_blocks, NT, smem, s>>>(d_in, b, d_tables, lay, w, d_out);
  return cudaGetLastError();
}
template <int S, bool PAIRS, bool SLOTS>
static cudaError_t launch_write_t(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                  const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, cudaStream_t s) {
  return b.small ? launch_write_small_t<S, PAIRS, SLOTS, true>(d_in, b, d_tables, lay, w, d_out, s)
                 : launch_write_small_t<S, PAIRS, SLOTS, false>(d_in, b, d_tables, lay, w, d_out, s);
}

// Two fields fit one 32-bit append when they are <= 16 bits each: always for L <= 256 (PAIRS); for
// larger tables each block decides from its table's widest offset field.
template <int S>
static cudaError_t sizes_dispatch(const uint8_t* d_in, const EncBatch& b, const shn_table* t, const EncodeLayout& lay,
                                  const EncodeWork& w, cudaStream_t s) {
  return lay.R <= 8 ? launch_sizes_t<S, true>(d_in, b, t, lay, w, s) : launch_sizes_t<S, false>(d_in, b, t, lay, w, s);
}
template <int S>
static cudaError_t write_dispatch(const uint8_t* d_in, const EncBatch& b, const shn_table* t, const EncodeLayout& lay,
                                  const EncodeWork& w, uint8_t* d_out, bool slots, cudaStream_t s) {
  if (slots)
    return lay.R <= 8 ? launch_write_t<S, true, true>(d_in, b, t, lay, w, d_out, s)
                      : launch_write_t<S, false, true>(d_in, b, t, lay, w, d_out, s);
  return lay.R <= 8 ? launch_write_t<S, true, false>(d_in, b, t, lay, w, d_out, s)
                    : launch_write_t<S, false, false>(d_in, b, t, lay, w, d_out, s);
}

cudaError_t launch_encode_sizes(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                const EncodeLayout& lay, const EncodeWork& w, int, cudaStream_t s) {
  if (b.total_blocks == 0) return cudaSuccess;
  switch (lay.S) {
    case 1: return sizes_dispatch<1>(d_in, b, d_tables, lay, w, s);
    case 2: return sizes_dispatch<2>(d_in, b, d_tables, lay, w, s);
    case 4: return sizes_dispatch<4>(d_in, b, d_tables, lay, w, s);
    case 8: return sizes_dispatch<8>(d_in, b, d_tables, lay, w, s);
    case 16: return sizes_dispatch<16>(d_in, b, d_tables, lay, w, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_encode_write(const uint8_t* d_in, const EncBatch& b, const shn_table* d_tables,
                                const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, bool slots,
                                cudaStream_t s) {
  if (b.total_blocks == 0) return cudaSuccess;
  switch (lay.S) {
    case 1: return write_dispatch<1>(d_in, b, d_tables, lay, w, d_out, slots, s);
    case 2: return write_dispatch<2>(d_in, b, d_tables, lay, w, d_out, slots, s);
    case 4: return write_dispatch<4>(d_in, b, d_tables, lay, w, d_out, slots, s);
    case 8: return write_dispatch<8>(d_in, b, d_tables, lay, w, d_out, slots, s);
    case 16: return write_dispatch<16>(d_in, b, d_tables, lay, w, d_out, slots, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_encode_compact(const EncodeLayout& lay, const EncodeWork& w, uint8_t* d_out, int sm_count,
                                  cudaStream_t s) {
  if (lay.total_chunks == 0) return cudaSuccess;
  const uint64_t want = (lay.total_chunks + 7) / 8;  // 8 warps per block, one chunk per warp
  const uint64_t cap = (uint64_t)sm_count * 16;      // two waves of 8 resident blocks (measured: 0.5 % faster than one)
  encode_compact_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(lay, w, d_out);
  return cudaGetLastError();
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
