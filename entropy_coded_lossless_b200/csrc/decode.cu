// decode.cu — chunk-parallel Shannonic/tANS decoder (Shannonic §4.2, decoding: the decode table
// entry of the state gives the range s and its bit count, the offset o follows, x = base[s] + o).
//
// Work layout. A persistent grid of 256-thread blocks, each taking a contiguous run of tiles of 256
// consecutive chunks; each thread decodes one chunk of C symbols with S interleaved states (SHN1
// format §7), reading the chunk backwards from its end sentinel.
//
// Tables. The decode table lives in shared memory as 8-byte entries
//   .x = shared-window address of the next state's row (row base, including this thread's replica)
//   .y = nb | w << 8 | base' << 16 | (-(nb + w) & 0xFF) << 24     (base' = range base ^ 0x80)
// so one lookup plus two funnel shifts and one multiply-add give the next state's address. Pipes:
// the loop is bound by the ALU pipe (funnel shifts, byte permutes, compares; half rate on sm_100),
// so work moves to the FMA pipe's integer multiply-add (also half rate, issued in parallel) where
// it can: the next-state address, and the output value y + o * 2^16 (base' + offset in bits 16-23,
// picked out by the byte permute that packs the output anyway). Multiply-highs are quarter rate
// there; only the bit-position update keeps one (a signed mulhi by 2^8 adds the negated field
// width from y's top byte). Per decoded value this is ~7.4 ALU and ~5.5 FMA-pipe instructions
// (ncu pipe counts on the KV cache). When a tile lies
// in one segment (the common case for large tensors) the table is stored interleaved
// ([slot][replica], replica = lane & (copies - 1)): 16 copies up to L = 512, where an 8-byte load
// is served per half-warp and the 16 lanes of a half-warp always hit 16 different bank pairs
// whatever their states (table lookups never conflict); 8, 4, 2 copies at L = 1024 ... 4096 (a 64 KB
// table). The bank conflicts ncu counts in this kernel (about a fifth of its shared wavefronts on the
// KV cache) come from the window refills: lanes whose rings are at the same word offset meet on one
// bank. They cost LSU cycles, not ALU ones, and the kernel is ALU-bound.
// Tiles that straddle segments (many small tensors) use plain per-segment copies, built up to 16 at
// a time. Tables are built in shared memory from the (f, lo) records of the stream.
//
// Bits. Each thread keeps a 64-bit window (two words) of its chunk in registers and refills it from
// a private 128-byte ring in shared memory, which cp.async (16-byte, L2-only) copies fill ahead of
// use. All shared-memory accesses of the per-symbol loop use 32-bit shared-window addresses. Two
// symbols are extracted per window position when every field fits 16 bits (R plus the widest
// offset of the tables in shared memory: always at L <= 256), one otherwise (fields <= 20 bits,
// L <= 4096). Decoded values go to an output sink: the INT8 tensor (16-byte
// stores of 16 values) or, fused with the consumer, bf16 values dequantised by a per-group scale.
//
// Robustness. Corrupt input never causes an out-of-bounds access: descriptors and the chunk index
// are validated against the stream and output sizes, the ring is filled only from the thread's own
// chunk, and a decoded next-state row is always inside the table by construction.
#include <cuda_bf16.h>

#include "shn_internal.cuh"

#ifndef DEC_WARPS
#define DEC_WARPS 8  // warps per block (tile = 32 * DEC_WARPS chunks)
#endif
#ifndef DEC_MIN_BLOCKS
#define DEC_MIN_BLOCKS (32 / DEC_WARPS)  // blocks per SM the register budget must allow (<= 64 regs)
#endif

namespace shn {

constexpr int kDecWarps = DEC_WARPS;
constexpr int kDecThreads = kDecWarps * 32;
constexpr uint32_t kRingQuads = 8;                // 16-byte quads per thread
constexpr uint32_t kRingBytes = kRingQuads * 16;  // per thread
// Copies of the decode table: 16 (a conflict-free half-warp phase) up to L = 256, then fewer so the
// replicated table stays at 32 KB: L = 512, 1024, 2048, 4096 keep 8, 4, 2, 1 copies (lanes that share
// a copy may then conflict on a bank).
// Interleaved copies of the decode table: 16 up to L = 512, then 8, 4, 2 for L = 1024 ... 4096 (a
// 64 KB table: bank conflicts cost more than the occupancy it takes; at L = 1024, 8 copies decode
// in 0.84 ms per GiB where 4 copies at one more block per SM took 0.97 ms).
__host__ __device__ inline uint32_t dec_replicas(uint32_t R) { return R <= 9 ? 16u : (16u >> (R - 9)); }
constexpr uint32_t kStageBytes = 8192;

struct DecHeader {
  uint32_t n_segs, K, R, S, C, tb;
  uint64_t total_symbols, total_chunks, index_off, payload_off, stream_bytes;
};

__device__ __forceinline__ uint32_t ld32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }
__device__ __forceinline__ uint64_t ld64(const uint8_t* p) {
  return (uint64_t)ld32(p) | ((uint64_t)ld32(p + 4) << 32);
}

__device__ __forceinline__ DecHeader read_header(const uint8_t* c) {
  DecHeader h;
  h.n_segs = ld32(c + 8);
  const uint32_t w12 = ld32(c + 12);
  h.K = w12 & 0xFFFFu;
  h.R = (w12 >> 16) & 0xFFu;
  h.S = w12 >> 24;
  h.C = ld32(c + 16);
  h.tb = ld32(c + 20);
  h.total_symbols = ld64(c + 24);
  h.total_chunks = ld64(c + 32);
  h.index_off = ld64(c + 40);
  h.payload_off = ld64(c + 48);
  h.stream_bytes = ld64(c + 56);
  return h;
}

__device__ __forceinline__ uint32_t width_bits(uint32_t m) { return m <= 1 ? 0u : 32u - __clz(m - 1u); }

// Validates the header, then every segment descriptor and table record in parallel (each against its
// successor), so later kernels may trust all offsets taken from them (SHN1 format §6).
__global__ void __launch_bounds__(256) decode_check_kernel(const uint8_t* __restrict__ comp, uint64_t comp_bytes,
                                                           shn_params p, DeviceStatus* st, uint64_t out_capacity) {
  __shared__ int s_ok;
  if (threadIdx.x == 0) {
    int ok = comp_bytes >= kHeaderBytes && ld32(comp) == kMagic && (ld32(comp + 4) & 0xFFFFu) == 1u &&
             (ld32(comp + 4) >> 16) == kHeaderBytes;
    if (ok) {
      const DecHeader h = read_header(comp);
      ok = h.K == p.K && h.R == p.log2L && h.S == p.states_per_chunk && h.C == p.chunk_symbols &&
           h.tb == table_record_bytes(h.K) && h.n_segs <= (1u << 30) && h.total_chunks < (1ull << 32) &&
           h.index_off == index_offset(h.n_segs, h.K) && h.payload_off == payload_offset(h.n_segs, h.K, h.total_chunks) &&
           h.stream_bytes <= comp_bytes && h.payload_off <= h.stream_bytes && (h.stream_bytes & 15) == 0 &&
           h.stream_bytes < (1ull << 35);
      if (ok && h.n_segs == 0) ok = h.total_chunks == 0 && h.total_symbols == 0 && h.stream_bytes == h.payload_off;
    }
    s_ok = ok;
    if (!ok) report(st, SHN_ERR_CORRUPT, 0);
  }
  __syncthreads();
  if (!s_ok) return;
  const DecHeader h = read_header(comp);
  const uint8_t* descs = comp + kHeaderBytes;
  const uint8_t* recs = descs + (uint64_t)kSegDescBytes * h.n_segs;
  const uint64_t payload_total = h.stream_bytes - h.payload_off;  // includes the final zero padding
  for (uint32_t s = threadIdx.x; s < h.n_segs; s += blockDim.x) {
    const uint8_t* d = descs + (uint64_t)kSegDescBytes * s;
    const uint64_t n = ld64(d), oo = ld64(d + 8), ps = ld64(d + 16);
    const uint32_t pw = ld32(d + 24), fc = ld32(d + 28);
    bool ok = n < (1ull << 32) && (ps & 3) == 0;
    if (s == 0) ok = ok && oo == 0 && ps == 0 && fc == 0;
    uint64_t n_oo, n_ps, n_fc;
    if (s + 1 < h.n_segs) {
      const uint8_t* dn = d + kSegDescBytes;
      n_oo = ld64(dn + 8);
      n_ps = ld64(dn + 16);
      n_fc = ld32(dn + 28);
      ok = ok && n_ps == ps + 4ull * pw;
    } else {
      n_oo = h.total_symbols;
      n_ps = ps + 4ull * pw;
      n_fc = h.total_chunks;
      ok = ok && round_up(h.payload_off + n_ps, 16) == h.stream_bytes;
    }
    ok = ok && n_oo == oo + n && n_fc == fc + n_chunks(n, h.C) && ps + 4ull * pw <= payload_total;
    const uint8_t* rec = recs + (uint64_t)h.tb * s;
    uint32_t fsum = 0, prev = 0;
    for (uint32_t k = 0; k < h.K; ++k) {
      fsum += (uint32_t)rec[2 * k] | ((uint32_t)rec[2 * k + 1] << 8);
      const uint32_t lo = rec[2 * h.K + k];
      if ((k == 0 && lo != 0) || (k > 0 && lo <= prev)) ok = false;
      prev = lo;
    }
    ok = ok && fsum == (1u << h.R);
    if (!ok) report(st, SHN_ERR_CORRUPT, 0);
  }
  if (threadIdx.x == 0 && h.total_symbols > out_capacity) report(st, SHN_ERR_CAPACITY, 0);
}

// ---- shared-memory decode tables -------------------------------------------------------------

struct SmemLayout {
  uint32_t table_bytes;  // replicated table (or several plain tables)
  uint32_t ring_off;
  uint32_t stage_off;
  uint32_t stage_per_table;
  uint32_t max_plain_tables;
  uint32_t total;
};

__host__ __device__ inline SmemLayout smem_layout(uint32_t R, uint32_t K) {
  SmemLayout l;
  const uint32_t L = 1u << R;
  l.table_bytes = L * dec_replicas(R) * 8;
  l.ring_off = l.table_bytes;
  // table builds happen only while no chunk is being decoded (rings idle, no copies in flight),
  // so the build staging area shares the rings' space
  l.stage_off = l.ring_off;
  l.stage_per_table = (uint32_t)round_up(2 * (K + 1) + 2 * K + 4 * K, 16);
  uint32_t by_table = l.table_bytes / (L * 8);
  uint32_t by_stage = kStageBytes / l.stage_per_table;
  l.max_plain_tables = by_table < by_stage ? by_table : by_stage;
  if (l.max_plain_tables < 1) l.max_plain_tables = 1;
  l.total = l.ring_off + (kDecThreads * kRingBytes > kStageBytes ? kDecThreads * kRingBytes : kStageBytes);
  return l;
}

// Build decode tables (SHN1 format §5) for segments seg0 .. seg0+nt-1. replicated: nt == 1, entry of
// slot i, replica c at byte (i*16 + c)*8; plain: table t at t*L*8, entry i at +i*8. All threads of
// the block take part; the caller synchronises before (readers of the old tables are done).
__device__ bool build_decode_tables(const uint8_t* recs, const DecHeader& h, const SmemLayout& lay, uint32_t seg0,
                                    uint32_t nt, bool replicated, unsigned char* dsm, uint32_t dsm_saddr) {
  const uint32_t K = h.K, R = h.R, L = 1u << R;
  const uint32_t tid = threadIdx.x;
  bool wide = false;  // a range of these tables whose offset field does not fit beside R state bits in 16
  for (uint32_t e = tid; e < nt * K; e += blockDim.x) {
    const uint32_t t = e / K, k = e - t * K;
    const uint8_t* rec = recs + (uint64_t)h.tb * (seg0 + t);
    unsigned char* sg = dsm + lay.stage_off + t * lay.stage_per_table;
    uint16_t* f = reinterpret_cast<uint16_t*>(sg + 2 * (K + 1));
    uint32_t* wb = reinterpret_cast<uint32_t*>(sg + 2 * (K + 1) + 2 * K + ((2 * (K + 1) + 2 * K) & 2));
    const uint32_t lo = rec[2 * K + k];
    const uint32_t hi = (k + 1 < K) ? rec[2 * K + k + 1] : 256u;
    const uint32_t w = width_bits(hi - lo);
    f[k] = (uint16_t)((uint32_t)rec[2 * k] | ((uint32_t)rec[2 * k + 1] << 8));
    wb[k] = w | (((lo ^ 0x80u) & 0xFFu) << 8);
    wide = wide || R + w > 16;
  }
  const bool narrow = !__syncthreads_or(wide);
  for (uint32_t t = tid; t < nt; t += blockDim.x) {
    unsigned char* sg = dsm + lay.stage_off + t * lay.stage_per_table;
    uint16_t* cumul = reinterpret_cast<uint16_t*>(sg);
    const uint16_t* f = reinterpret_cast<const uint16_t*>(sg + 2 * (K + 1));
    uint32_t acc = 0;
    for (uint32_t k = 0; k < K; ++k) {
      cumul[k] = (uint16_t)acc;
      acc += f[k];
    }
    cumul[K] = (uint16_t)acc;
  }
  __syncthreads();
  const uint32_t step = (L >> 1) + (L >> 3) + 3;
  uint32_t inv = step;  // inverse of the odd step modulo 2^32 (Newton), reduced mod L below
#pragma unroll
  for (int it = 0; it < 5; ++it) inv *= 2u - step * inv;
  for (uint32_t e = tid; e < nt * L; e += blockDim.x) {
    const uint32_t t = e >> R, i = e & (L - 1);
    const unsigned char* sg = dsm + lay.stage_off + t * lay.stage_per_table;
    const uint16_t* cumul = reinterpret_cast<const uint16_t*>(sg);
    const uint16_t* f = reinterpret_cast<const uint16_t*>(sg + 2 * (K + 1));
    const uint32_t* wb = reinterpret_cast<const uint32_t*>(sg + 2 * (K + 1) + 2 * K + ((2 * (K + 1) + 2 * K) & 2));
    const uint32_t tau = (i * inv) & (L - 1);  // placement index of slot i
    int a = 0, b = (int)K - 1;                // its range: largest k with cumul[k] <= tau
    while (a < b) {
      const int m = (a + b + 1) >> 1;
      if (cumul[m] <= tau) a = m;
      else b = m - 1;
    }
    const uint32_t s = (uint32_t)a, fs = f[s], c0 = cumul[s];
    uint32_t rank = 0;  // slots of range s below slot i
    for (uint32_t u = c0; u < c0 + fs; ++u) rank += (((u * step) & (L - 1)) < i) ? 1u : 0u;
    const uint32_t x = fs + rank;
    const uint32_t nb = R - (31u - __clz(x));
    const uint32_t next = (x << nb) - L;
    const uint32_t w = wb[s] & 0xFFu, base = wb[s] >> 8;
    const uint32_t y = nb | (w << 8) | (base << 16) | (((0u - (nb + w)) & 0xFFu) << 24);
    if (replicated) {
      const uint32_t reps = dec_replicas(R);
      uint2* row = reinterpret_cast<uint2*>(dsm + i * (reps * 8));
#pragma unroll
      for (uint32_t c = 0; c < reps; ++c) row[c] = make_uint2(dsm_saddr + next * (reps * 8) + c * 8, y);
    } else {
      reinterpret_cast<uint2*>(dsm + t * L * 8)[i] = make_uint2(dsm_saddr + t * L * 8 + next * 8, y);
    }
  }
  __syncthreads();
  return narrow;
}

// ---- per-thread chunk decoder -----------------------------------------------------------------

__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr), "l"(gptr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// y >> 8, y >> 16 and the signed top byte as multiply-highs by powers of two; the compiler picks the
// pipe (shift or integer multiply) for each.
__device__ __forceinline__ uint32_t shr8(uint32_t y) { return __umulhi(y, 1u << 24); }
__device__ __forceinline__ uint32_t add_shr16(uint32_t y, uint32_t a) {
  uint32_t d;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(y), "r"(1u << 16), "r"(a));
  return d;
}
__device__ __forceinline__ int32_t add_top_byte(uint32_t y, int32_t p) {  // p + (int8)(y >> 24)
  int32_t d;
  asm("mad.hi.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(y), "r"(256), "r"(p));
  return d;
}

struct ChunkCtx {
  const uint8_t* comp;
  uint32_t ring_saddr;  // this thread's ring (shared-window address, 128-byte aligned)
  uint64_t cb;          // chunk start, bytes from the stream start
  uint32_t nw;          // chunk words
  uint32_t tbase;       // shared-window address of slot 0's entry for this thread (replica / plain table)
  uint64_t pos0;        // output position (symbols) of the chunk's first piece (SHN1 format §6)
  uint32_t pos_stride;  // symbols between consecutive pieces of the chunk (16 * chunks in its group)
  uint32_t pieces;
  uint32_t last_len;    // symbols in the last piece (1..16)
};

// Output sinks: where a chunk's decoded symbols go. Pieces are 16 consecutive output positions
// (SHN1 format §6). Each sink forms a symbol's value from its table word y (base' in bits 16-23)
// and its offset o with val(y, o), and receives those values in put_pair/put.
struct ByteSink {  // the INT8 tensor itself
  // val = y + o * 2^16: the raw byte (base' + offset, mod 256) sits in bits 16-23, junk around it.
  // One integer multiply-add (the multiplier is a runtime value, so it stays on the FMA pipe, which
  // this ALU-bound loop has room on), where base' + o in the low byte would take ALU instructions.
  uint32_t m16;  // 65536
  __device__ __forceinline__ uint32_t val(uint32_t y, uint32_t o) const {
    uint32_t d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(o), "r"(m16), "r"(y));
    return d;
  }
  uint8_t* out;
  uint8_t* dst;
  uint32_t stride;
  bool aligned;
  uint32_t ov[4];
  __device__ __forceinline__ void start(const ChunkCtx& c) {
    dst = out + c.pos0;
    stride = c.pos_stride;
    aligned = (reinterpret_cast<uintptr_t>(dst) & 15u) == 0;
  }
  __device__ __forceinline__ void begin_piece() {}
  // pp and i are loop indices of fully unrolled loops, so they fold to constants
  __device__ __forceinline__ void put_pair(int pp, uint32_t ba, uint32_t bb) {
    const uint32_t pair = __byte_perm(ba, bb, 0x0062);  // bytes: ba.b2, bb.b2
    if ((pp & 1) == 0) ov[pp >> 1] = pair;
    else ov[pp >> 1] = __byte_perm(ov[pp >> 1], pair, 0x5410);
  }
  __device__ __forceinline__ void put(int i, uint32_t b) {  // b's byte 2 into byte i % 4 of word i / 4
    if ((i & 3) == 0) ov[i >> 2] = __byte_perm(b, 0u, 0x0002);
    else ov[i >> 2] = __byte_perm(ov[i >> 2], b, (i & 3) == 1 ? 0x3260u : (i & 3) == 2 ? 0x3610u : 0x6210u);
  }
  __device__ __forceinline__ void end_piece() {
    if (aligned) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
    } else {
#pragma unroll
      for (int r = 0; r < 16; ++r) dst[r] = (uint8_t)(ov[r >> 2] >> (8 * (r & 3)));
    }
    dst += stride;
  }
  __device__ __forceinline__ void put_tail(uint32_t i, uint32_t b) { dst[i] = (uint8_t)(b >> 16); }
};

// bf16 dequantisation fused into the decode: value = bf16_rn(float(int8) * scale[pos >> gshift]),
// the product rounded once in fp32 as a separate multiply would. A piece lies in one scale group
// (groups are >= 16 positions and pieces start at multiples of 16), so there is one scale load per
// piece, issued one piece ahead.
struct Bf16Sink {
  // val: the raw byte (base' + offset) in the low 8 bits, junk above
  __device__ __forceinline__ uint32_t val(uint32_t y, uint32_t o) const { return add_shr16(y, o); }
  uint16_t* out;
  const float* scales;
  uint32_t gshift;
  uint64_t gmax;  // last valid scale index
  uint64_t pos;
  uint32_t stride;
  float sc, sc_next;
  uint32_t ov[4];
  __device__ __forceinline__ void start(const ChunkCtx& c) {
    pos = c.pos0;
    stride = c.pos_stride;
    sc_next = __ldg(scales + min(pos >> gshift, gmax));
  }
  __device__ __forceinline__ void begin_piece() {
    sc = sc_next;
    sc_next = __ldg(scales + min((pos + stride) >> gshift, gmax));  // the next piece's (clamped past the end)
  }
  static __device__ __forceinline__ float value(uint32_t b) {
    // raw byte -> float(int8): 2^23 + (b ^ 0x80) as a float bit pattern, minus 2^23 + 128 (exact)
    return __int_as_float(int((b & 0xFFu) ^ 0x4B000080u)) - 8388736.0f;
  }
  __device__ __forceinline__ uint32_t pack(uint32_t ba, uint32_t bb) const {
    const __nv_bfloat162 h = __floats2bfloat162_rn(value(ba) * sc, value(bb) * sc);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  // pp and i are loop indices of fully unrolled loops, so they fold to constants
  __device__ __forceinline__ void put_pair(int pp, uint32_t ba, uint32_t bb) {
    ov[pp & 3] = pack(ba, bb);
    if ((pp & 3) == 3) *reinterpret_cast<uint4*>(out + pos + 8 * (pp >> 2)) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
  }
  uint32_t held;
  __device__ __forceinline__ void put(int i, uint32_t b) {
    if ((i & 1) == 0) held = b;
    else put_pair(i >> 1, held, b);
  }
  __device__ __forceinline__ void end_piece() { pos += stride; }
  __device__ __forceinline__ void put_tail(uint32_t i, uint32_t b) {
    const __nv_bfloat16 h = __float2bfloat16_rn(value(b) * sc_next);  // the tail piece's scale
    out[pos + i] = *reinterpret_cast<const uint16_t*>(&h);
  }
};

// Ring fetcher: quads of 16 bytes (absolute, stream-relative), fetched downwards from the chunk end.
// (Quad indices fit in 31 bits: streams are limited to 2^35 bytes by the header check.)
struct Fetcher {
  int32_t lo;      // lowest quad fetched so far
  int32_t bottom;  // lowest quad of the chunk
  __device__ __forceinline__ void fill_to(const ChunkCtx& c, int32_t limit) {
    const int32_t target = limit > bottom ? limit : bottom;
    while (lo > target) {
      --lo;
      cp_async16(c.ring_saddr + (((uint32_t)lo * 16u) & (kRingBytes - 1)), c.comp + (uint64_t)(uint32_t)lo * 16u);
    }
  }
  // Per 16-symbol piece at most N quads leave the ring (2 for fields of <= 16 bits; 3 for fields of
  // <= 20 bits), so topping it up with at most N fetches keeps it full: no loop, N
  // predicated copies.
  template <int N>
  __device__ __forceinline__ void top_up(const ChunkCtx& c, int32_t limit) {
    const int32_t target = limit > bottom ? limit : bottom;
#pragma unroll
    for (int i = 0; i < N; ++i) {
      if (lo > target) {
        --lo;
        cp_async16(c.ring_saddr + (((uint32_t)lo * 16u) & (kRingBytes - 1)), c.comp + (uint64_t)(uint32_t)lo * 16u);
      }
    }
  }
};

// One chunk. SH = log2 of the table row stride in bytes. PAIRS (every symbol's state bits plus offset
// bits fit in 16, i.e. R + widest offset <= 16: always for L <= 256, and for larger tables with
// narrow ranges such as plain tANS): two symbols per window position; otherwise one (fields <= 20
// bits).
template <int S, int SH, bool PAIRS, class Sink>
__device__ __forceinline__ bool decode_chunk(const ChunkCtx& c, uint32_t R, Sink& sk) {
  const uint32_t mask = kRingBytes - 1;
  const uint32_t cb_mod = (uint32_t)(c.cb & mask);
  Fetcher fe;
  const int32_t q_top = (int32_t)((c.cb + 4ull * c.nw - 1) >> 4);
  fe.bottom = (int32_t)(c.cb >> 4);
  fe.lo = q_top + 1;
  fe.fill_to(c, q_top - (int32_t)kRingQuads + 1);
  // quad of the window's low word: bottom + (chunk start word within its quad + window word) / 4,
  // kept in 32 bits for streams up to 32 GiB (the chunk's word offset alone would not be)
  const int32_t cb_wq = (int32_t)((c.cb >> 2) & 3u);
  cp_async_commit();
  cp_async_wait<0>();
  // ring address of chunk word k (k may be negative: a stale word, never used validly)
  auto waddr = [&](int32_t k) -> uint32_t { return c.ring_saddr | ((cb_mod + 4u * (uint32_t)k) & mask); };
  const uint32_t last = lds32(waddr((int32_t)c.nw - 1));
  if (last == 0u) return false;
  int32_t P = 32 * ((int32_t)c.nw - 1) + (31 - __clz(last));  // unread bits: [0, P)
  int32_t thr = P & ~31;                                        // window = words (thr/32 - 1, thr/32)
  uint32_t W1 = lds32(waddr((thr >> 5)));
  uint32_t W0 = lds32(waddr((thr >> 5) - 1));
  uint32_t ra_w = waddr((thr >> 5) - 1);  // ring address of W0
  auto advance = [&]() {  // keep P in [thr, thr + 32)
    if (P < thr) {
      W1 = W0;
      thr -= 32;
      ra_w = c.ring_saddr | ((ra_w - 4u) & mask);
      W0 = lds32(ra_w);
    }
  };
  uint32_t X[S];
#pragma unroll
  for (int q = S - 1; q >= 0; --q) {
    const uint32_t V = __funnelshift_r(W0, W1, (uint32_t)P);
    X[q] = c.tbase + ((V >> (32u - R)) << SH);
    P -= (int32_t)R;
    advance();
  }
  const uint32_t full = c.pieces - (c.last_len < 16 ? 1u : 0u);
  sk.start(c);
  for (uint32_t k = 0; k < full; ++k) {
    fe.top_up<PAIRS ? 2 : 3>(c, fe.bottom + ((cb_wq + (thr >> 5)) >> 2) - (int32_t)kRingQuads + 1);
    cp_async_commit();
    cp_async_wait<1>();
    sk.begin_piece();
    if (!PAIRS) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int q = i % S;
        const uint32_t V = __funnelshift_r(W0, W1, (uint32_t)P);
        const uint2 E = lds64(X[q]);
        const uint32_t r = __funnelshift_l(V, 0u, E.y);
        const uint32_t Vs = __funnelshift_l(0u, V, E.y);
        const uint32_t o = __funnelshift_l(Vs, 0u, shr8(E.y));
        X[q] = E.x + r * (1u << SH);
        P = add_top_byte(E.y, P);
        advance();
        sk.put(i, sk.val(E.y, o));
      }
    } else {
#pragma unroll
      for (int pp = 0; pp < 8; ++pp) {
        const int qa = (2 * pp) % S, qb = (2 * pp + 1) % S;
        const uint32_t V = __funnelshift_r(W0, W1, (uint32_t)P);  // next 32 bits, top-aligned
        const uint2 Ea = lds64(X[qa]);
        const uint32_t ra = __funnelshift_l(V, 0u, Ea.y);          // state bits: top nb of V
        const uint32_t Va = __funnelshift_l(0u, V, Ea.y);          // V << nb
        const uint32_t wa = shr8(Ea.y);                            // low 5 bits: w
        const uint32_t oa = __funnelshift_l(Va, 0u, wa);           // offset: next w bits
        const uint32_t V2 = __funnelshift_l(0u, Va, wa);           // V << (nb + w)
        const uint32_t ba = sk.val(Ea.y, oa);                      // base' + offset
        X[qa] = Ea.x + ra * (1u << SH);
        P = add_top_byte(Ea.y, P);                                 // P -= nb + w
        const uint2 Eb = lds64(X[qb]);
        const uint32_t rb = __funnelshift_l(V2, 0u, Eb.y);
        const uint32_t Vb = __funnelshift_l(0u, V2, Eb.y);
        const uint32_t wb = shr8(Eb.y);
        const uint32_t ob = __funnelshift_l(Vb, 0u, wb);
        const uint32_t bb = sk.val(Eb.y, ob);
        X[qb] = Eb.x + rb * (1u << SH);
        P = add_top_byte(Eb.y, P);
        advance();
        sk.put_pair(pp, ba, bb);
      }
    }
    sk.end_piece();
  }
  if (full < c.pieces) {  // the group's short last piece
    fe.fill_to(c, fe.bottom + ((cb_wq + (thr >> 5)) >> 2) - (int32_t)kRingQuads + 1);
    cp_async_commit();
    cp_async_wait<0>();
    for (uint32_t i = 0; i < c.last_len; ++i) {
      const int q = (int)(i % S);  // chunk index 16*full + i, and S divides 16
      uint32_t x = X[0];
#pragma unroll
      for (int k = 1; k < S; ++k)
        if (k == q) x = X[k];
      const uint32_t V = __funnelshift_r(W0, W1, (uint32_t)P);
      const uint2 E = lds64(x);
      const uint32_t r = __funnelshift_l(V, 0u, E.y);
      const uint32_t Vs = __funnelshift_l(0u, V, E.y);
      const uint32_t o = __funnelshift_l(Vs, 0u, shr8(E.y));
      x = E.x + r * (1u << SH);
      P = add_top_byte(E.y, P);
      advance();
      sk.put_tail(i, sk.val(E.y, o));
#pragma unroll
      for (int k = 0; k < S; ++k)
        if (k == q) X[k] = x;
    }
  }
  cp_async_wait<0>();
  bool ok = (P == 0);
#pragma unroll
  for (int q = 0; q < S; ++q) ok = ok && (X[q] == c.tbase);
  return ok;
}

// ---- the kernel --------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t segment_of(const uint8_t* descs, uint32_t n_segs, uint64_t g) {
  int a = 0, b = (int)n_segs - 1;  // largest s with first_chunk[s] <= g
  while (a < b) {
    const int m = (a + b + 1) >> 1;
    if (ld32(descs + (uint64_t)kSegDescBytes * m + 28) <= g) a = m;
    else b = m - 1;
  }
  return (uint32_t)a;
}

// Output of a decode launch: INT8 bytes, or bf16 values dequantised by a scale per 2^gshift positions.
struct DecOut {
  uint8_t* out;
  const float* scales;
  uint32_t gshift;
  uint64_t n_scales;
  uint32_t zero;  // 0, passed at run time so that multiplier operands stay opaque to the compiler
};

template <int S, bool BF16>
__global__ void __launch_bounds__(kDecThreads, DEC_MIN_BLOCKS) decode_kernel(const uint8_t* __restrict__ comp, DeviceStatus* st,
                                                                             const DecOut o) {
  extern __shared__ __align__(128) unsigned char dsm[];
  if (*(volatile uint32_t*)&st->status != 0) return;
  const DecHeader h = read_header(comp);
  const SmemLayout lay = smem_layout(h.R, h.K);
  const uint32_t L = 1u << h.R;
  const uint8_t* descs = comp + kHeaderBytes;
  const uint8_t* recs = descs + (uint64_t)kSegDescBytes * h.n_segs;
  const uint32_t* index = reinterpret_cast<const uint32_t*>(comp + h.index_off);
  const uint32_t tid = threadIdx.x, lane = tid & 31;
  const uint32_t dsm_saddr = smem_addr(dsm);
  const uint32_t ring_saddr = dsm_saddr + lay.ring_off + tid * kRingBytes;
  if ((dsm_saddr & 127u) != 0) {  // ring addressing below relies on 128-byte aligned rings
    if (tid == 0) report(st, SHN_ERR_CUDA, 0);
    return;
  }
  const uint64_t n_tiles = (h.total_chunks + kDecThreads - 1) / kDecThreads;
  uint32_t cur_seg = 0xFFFFFFFFu;  // segment whose replicated table is in shared memory (none: ~0 > n_segs - 1)
  bool cur_pairs = false;  // whether its fields fit two to a 32-bit window read
  const uint64_t gmax = h.total_symbols > 0 ? (h.total_symbols - 1) >> o.gshift : 0;
  if (BF16 && h.total_symbols > 0 && gmax >= o.n_scales) {
    if (blockIdx.x == 0 && tid == 0) report(st, SHN_ERR_CAPACITY, 0);
    return;
  }
  // decode one chunk into the launch's output
  auto run = [&](const ChunkCtx& cc, auto sh, auto pairs) -> bool {
    constexpr int SH = decltype(sh)::value;
    constexpr bool PAIRS = decltype(pairs)::value;
    if (BF16) {
      Bf16Sink sk;
      sk.out = reinterpret_cast<uint16_t*>(o.out);
      sk.scales = o.scales;
      sk.gshift = o.gshift;
      sk.gmax = gmax;
      return decode_chunk<S, SH, PAIRS>(cc, h.R, sk);
    }
    ByteSink sk;
    sk.m16 = 65536u | o.zero;
    sk.out = o.out;
    return decode_chunk<S, SH, PAIRS>(cc, h.R, sk);
  };

  // Each block takes a contiguous run of tiles: consecutive tiles usually lie in one segment, so the
  // replicated table is rebuilt only when the run crosses a segment boundary (a strided assignment
  // rebuilt it for nearly every tile of a many-segment stream).
  const uint64_t t_per = n_tiles / gridDim.x, t_rem = n_tiles % gridDim.x;
  const uint64_t t_begin = blockIdx.x * t_per + min((uint64_t)blockIdx.x, t_rem);
  const uint64_t t_end = t_begin + t_per + (blockIdx.x < t_rem ? 1u : 0u);
  for (uint64_t tile = t_begin; tile < t_end; ++tile) {
    const uint64_t g0 = tile * kDecThreads;
    const uint64_t g_last = min(g0 + kDecThreads, h.total_chunks) - 1;
    const uint32_t sa = segment_of(descs, h.n_segs, g0), sb = segment_of(descs, h.n_segs, g_last);
    // this thread's chunk
    const uint64_t g = g0 + tid;
    bool valid = g < h.total_chunks;
    ChunkCtx c;
    uint32_t seg = 0;
    if (valid) {
      seg = segment_of(descs, h.n_segs, g);
      const uint8_t* d = descs + (uint64_t)kSegDescBytes * seg;
      const uint64_t n = ld64(d), out_off = ld64(d + 8), pay_start = ld64(d + 16);
      const uint32_t pay_words = ld32(d + 24), first = ld32(d + 28);
      const uint32_t ci = (uint32_t)(g - first);
      const uint32_t nch = (uint32_t)n_chunks(n, h.C);
      const uint32_t w0 = index[g];
      const uint32_t w1 = (ci + 1 < nch) ? index[g + 1] : pay_words;
      if (ci >= nch || w1 <= w0 || w1 > pay_words || (ci == 0 && w0 != 0)) {
        report(st, SHN_ERR_CORRUPT, (uint32_t)g);
        valid = false;
      } else {
        c.comp = comp;
        c.ring_saddr = ring_saddr;
        c.cb = h.payload_off + pay_start + 4ull * w0;
        c.nw = w1 - w0;
        const ChunkGeo geo = chunk_geo(n, h.C, ci);
        c.pos0 = out_off + geo.base + 16u * geo.j;
        c.pos_stride = 16u * geo.m;
        c.pieces = geo.pieces;
        c.last_len = geo.last_len;
        if (BF16 && (out_off & 15) != 0) {  // pieces would straddle scale groups
          report(st, SHN_ERR_UNSUPPORTED, (uint32_t)g);
          valid = false;
        }
      }
    }
    if (sa == sb) {
      if (cur_seg != sa) {
        __syncthreads();
        cur_pairs = build_decode_tables(recs, h, lay, sa, 1, true, dsm, dsm_saddr);
        cur_seg = sa;
      }
      if (valid) {
        c.tbase = dsm_saddr + (lane & (dec_replicas(h.R) - 1)) * 8;
        auto run_sh = [&](auto sh) { return cur_pairs ? run(c, sh, std::true_type()) : run(c, sh, std::false_type()); };
        bool ok;
        switch (h.R) {  // row stride: 16 copies x 8 bytes up to L = 512, then 8, 4, 2 copies
          case 9: ok = run_sh(std::integral_constant<int, 7>()); break;
          case 10: ok = run_sh(std::integral_constant<int, 6>()); break;
          case 11: ok = run_sh(std::integral_constant<int, 5>()); break;
          case 12: ok = run_sh(std::integral_constant<int, 4>()); break;
          default: ok = run(c, std::integral_constant<int, 7>(), std::true_type()); break;
        }
        if (!ok) report(st, SHN_ERR_CORRUPT, (uint32_t)g);
      }
    } else {
      cur_seg = 0xFFFFFFFFu;
      for (uint32_t s0 = sa; s0 <= sb; s0 += lay.max_plain_tables) {
        const uint32_t nt = min(lay.max_plain_tables, sb - s0 + 1);
        __syncthreads();
        const bool pairs = build_decode_tables(recs, h, lay, s0, nt, false, dsm, dsm_saddr);
        if (valid && seg >= s0 && seg < s0 + nt) {
          c.tbase = dsm_saddr + (seg - s0) * L * 8;
          const bool ok = pairs ? run(c, std::integral_constant<int, 3>(), std::true_type())
                                : run(c, std::integral_constant<int, 3>(), std::false_type());
          if (!ok) report(st, SHN_ERR_CORRUPT, (uint32_t)g);
        }
      }
    }
  }
}

template <int S, bool BF16>
static cudaError_t launch_decode_t(const uint8_t* d_comp, DeviceStatus* st, const DecOut& o, const shn_params& p,
                                   int sm_count, cudaStream_t s) {
  const SmemLayout lay = smem_layout(p.log2L, p.K);
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<S, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)lay.total);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<S, BF16>, kDecThreads, lay.total);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  decode_kernel<S, BF16><<<sm_count * per_sm, kDecThreads, lay.total, s>>>(d_comp, st, o);
  return cudaGetLastError();
}

template <bool BF16>
static cudaError_t launch_decode_mode(const uint8_t* d_comp, uint64_t comp_bytes, const shn_params& p,
                                      DeviceStatus* st, const DecOut& o, uint64_t out_capacity, int sm_count,
                                      cudaStream_t s) {
  decode_check_kernel<<<1, 256, 0, s>>>(d_comp, comp_bytes, p, st, out_capacity);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  switch (p.states_per_chunk) {
    case 1: return launch_decode_t<1, BF16>(d_comp, st, o, p, sm_count, s);
    case 2: return launch_decode_t<2, BF16>(d_comp, st, o, p, sm_count, s);
    case 4: return launch_decode_t<4, BF16>(d_comp, st, o, p, sm_count, s);
    case 8: return launch_decode_t<8, BF16>(d_comp, st, o, p, sm_count, s);
    case 16: return launch_decode_t<16, BF16>(d_comp, st, o, p, sm_count, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const uint8_t* d_comp, uint64_t comp_bytes, const shn_params& p, DeviceStatus* st,
                          uint8_t* d_out, uint64_t out_capacity, int sm_count, cudaStream_t s) {
  const DecOut o{d_out, nullptr, 0u, 0ull, 0u};
  return launch_decode_mode<false>(d_comp, comp_bytes, p, st, o, out_capacity, sm_count, s);
}

cudaError_t launch_decode_bf16(const uint8_t* d_comp, uint64_t comp_bytes, const shn_params& p, DeviceStatus* st,
                               uint16_t* d_out, uint64_t out_elems, const float* d_scales, uint32_t log2_group,
                               uint64_t n_scales, int sm_count, cudaStream_t s) {
  const DecOut o{reinterpret_cast<uint8_t*>(d_out), d_scales, log2_group, n_scales, 0u};
  return launch_decode_mode<true>(d_comp, comp_bytes, p, st, o, out_elems, sm_count, s);
}

}  // namespace shn
