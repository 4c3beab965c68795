// decode.cu — chunk-parallel Shannonic/tANS decoder (Shannonic §4.2: "from state X, decTable[X]
// gives the symbol s and the bit count; read the offset o and restore x = base[s] + o").
//
// Layout of the work: a persistent grid of warps; each warp takes 32 consecutive chunks, one per
// lane. Every lane keeps the decode table of its own chunk's segment in its own shared-memory
// column ([slot][lane] u32), so all 32 lookups of a warp hit 32 different banks whatever the
// states are. A table entry packs everything a step needs:
//   bits 0..4 nb (state bits), 5..8 w (offset bits), 9..16 base' = base ^ 0x80 (output base),
//   17..28 next slot base.
// The lane reads its chunk backwards from the end sentinel (FORMAT.md §7) through a 64-bit window
// refilled one 32-bit word at a time; S interleaved states give independent lookups.
// Corrupt input never leads to an out-of-bounds access: every offset taken from the stream is
// checked against the stream and output sizes, the window only ever reads words of the lane's own
// chunk, and a decoded slot is always < L by construction.
#include "shn_internal.cuh"

namespace shn {

constexpr int kDecMaxR = 8;

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

// One thread validates the header and every segment descriptor / table record (FORMAT.md §6).
__global__ void decode_check_kernel(const uint8_t* __restrict__ comp, uint64_t comp_bytes, shn_params p,
                                    DeviceStatus* st, uint64_t out_capacity) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  if (comp_bytes < kHeaderBytes || ld32(comp) != kMagic || (ld32(comp + 4) & 0xFFFFu) != 1u ||
      (ld32(comp + 4) >> 16) != kHeaderBytes) {
    report(st, SHN_ERR_CORRUPT, 0);
    return;
  }
  const DecHeader h = read_header(comp);
  bool ok = h.K == p.K && h.R == p.log2L && h.S == p.states_per_chunk && h.C == p.chunk_symbols &&
            h.tb == table_record_bytes(h.K) && h.n_segs <= (1u << 30) && h.total_chunks < (1ull << 32);
  ok = ok && h.index_off == index_offset(h.n_segs, h.K) &&
       h.payload_off == payload_offset(h.n_segs, h.K, h.total_chunks) && h.stream_bytes <= comp_bytes &&
       h.payload_off <= h.stream_bytes;
  if (!ok) {
    report(st, SHN_ERR_CORRUPT, 0);
    return;
  }
  uint64_t out_off = 0, pay = 0, chunk = 0;
  for (uint32_t s = 0; s < h.n_segs; ++s) {
    const uint8_t* d = comp + kHeaderBytes + (uint64_t)kSegDescBytes * s;
    const uint64_t n = ld64(d);
    if (n >= (1ull << 32) || ld64(d + 8) != out_off || ld64(d + 16) != pay || ld32(d + 28) != chunk) {
      report(st, SHN_ERR_CORRUPT, 0);
      return;
    }
    const uint8_t* rec = comp + kHeaderBytes + (uint64_t)kSegDescBytes * h.n_segs + (uint64_t)h.tb * s;
    uint32_t fsum = 0, prev_lo = 0;
    for (uint32_t k = 0; k < h.K; ++k) {
      fsum += (uint32_t)rec[2 * k] | ((uint32_t)rec[2 * k + 1] << 8);
      const uint32_t lo = rec[2 * h.K + k];
      if ((k == 0 && lo != 0) || (k > 0 && lo <= prev_lo)) ok = false;
      prev_lo = lo;
    }
    if (!ok || fsum != (1u << h.R)) {
      report(st, SHN_ERR_CORRUPT, 0);
      return;
    }
    out_off += n;
    pay += 4ull * ld32(d + 24);
    chunk += n_chunks(n, h.C);
  }
  if (chunk != h.total_chunks || out_off != h.total_symbols || h.stream_bytes != round_up(h.payload_off + pay, 16)) {
    report(st, SHN_ERR_CORRUPT, 0);
    return;
  }
  if (h.total_symbols > out_capacity) report(st, SHN_ERR_CAPACITY, 0);
}

// Backward bit reader over the words of one chunk (FORMAT.md §7 "read n bits").
struct BackReader {
  const uint32_t* w;
  unsigned long long buf;  // words k (low) and k+1 (high)
  int k;
  int P;                   // unread bits are positions [0, P) of the chunk
  bool bad;
  __device__ __forceinline__ void init(const uint32_t* words, int nw) {
    w = words;
    const uint32_t last = words[nw - 1];
    bad = (last == 0u);
    P = 32 * (nw - 1) + (31 - __clz(last | (bad ? 1u : 0u)));
    k = P >= 32 ? (P >> 5) - 1 : 0;
    const uint32_t hi = (k + 1 < nw) ? words[k + 1] : 0u;
    buf = ((unsigned long long)hi << 32) | words[k];
  }
  // Read n <= 20 bits ending at P; refill afterwards so that 32 bits stay available.
  __device__ __forceinline__ uint32_t read(uint32_t n) {
    int sh = P - (int)n - 32 * k;
    if (sh < 0) {
      bad = true;
      sh = 0;
    }
    const uint32_t v = (uint32_t)(buf >> sh) & ((1u << n) - 1u);
    P -= (int)n;
    if (P - 32 * k < 32 && k > 0) {
      --k;
      buf = (buf << 32) | w[k];
    }
    return v;
  }
};

template <int S>
__global__ void __launch_bounds__(256) decode_kernel(const uint8_t* __restrict__ comp, DeviceStatus* st,
                                                     uint8_t* __restrict__ out, uint32_t col_words) {
  extern __shared__ __align__(16) uint32_t dsm[];
  if (*(volatile uint32_t*)&st->status != 0) return;
  const DecHeader h = read_header(comp);
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t L = 1u << h.R;
  // per-warp shared area: table [L][32] u32, spread [L][32] u8, counters [K][32] u8
  uint32_t* tab = dsm + (size_t)warp * col_words;
  uint8_t* spread = reinterpret_cast<uint8_t*>(tab + L * 32);
  uint8_t* cnt = spread + L * 32;
  const uint32_t step = (L >> 1) + (L >> 3) + 3;
  const uint8_t* descs = comp + kHeaderBytes;
  const uint8_t* recs = comp + kHeaderBytes + (uint64_t)kSegDescBytes * h.n_segs;
  const uint32_t* index = reinterpret_cast<const uint32_t*>(comp + h.index_off);
  int cur_seg = -1;
  bool seg_ok = false;

  const uint64_t n_groups = (h.total_chunks + 31) / 32;
  const uint64_t warps_total = (uint64_t)gridDim.x * (blockDim.x >> 5);
  for (uint64_t grp = (uint64_t)blockIdx.x * (blockDim.x >> 5) + warp; grp < n_groups; grp += warps_total) {
    const uint64_t g = grp * 32 + lane;
    if (g >= h.total_chunks) continue;
    // segment of chunk g: largest s with first_chunk[s] <= g
    int a = 0, b = (int)h.n_segs - 1;
    while (a < b) {
      const int m = (a + b + 1) >> 1;
      if (ld32(descs + (uint64_t)kSegDescBytes * m + 28) <= g) a = m;
      else b = m - 1;
    }
    const int seg = a;
    const uint8_t* d = descs + (uint64_t)kSegDescBytes * seg;
    const uint64_t n = ld64(d);
    const uint64_t out_off = ld64(d + 8);
    const uint64_t pay_start = ld64(d + 16);
    const uint32_t pay_words = ld32(d + 24);
    const uint32_t first = ld32(d + 28);
    const uint32_t c = (uint32_t)(g - first);
    const uint32_t nch = (uint32_t)n_chunks(n, h.C);
    if (c >= nch) continue;  // an empty segment shares its first_chunk with the next one
    const uint32_t len = (uint32_t)min((uint64_t)h.C, n - (uint64_t)c * h.C);

    if (seg != cur_seg) {
      cur_seg = seg;
      // build this lane's decode-table column (FORMAT.md §5)
      const uint8_t* rec = recs + (uint64_t)h.tb * seg;
      uint32_t t = 0;
      for (uint32_t k = 0; k < h.K; ++k) {
        const uint32_t fk = (uint32_t)rec[2 * k] | ((uint32_t)rec[2 * k + 1] << 8);
        for (uint32_t r = 0; r < fk && t < L; ++r, ++t) spread[((t * step) & (L - 1)) * 32 + lane] = (uint8_t)k;
        cnt[k * 32 + lane] = 0;
      }
      seg_ok = (t == L);
      for (uint32_t i = 0; i < L && seg_ok; ++i) {
        const uint32_t s = spread[i * 32 + lane];
        const uint32_t j = cnt[s * 32 + lane];
        cnt[s * 32 + lane] = (uint8_t)(j + 1);
        const uint32_t fs = (uint32_t)rec[2 * s] | ((uint32_t)rec[2 * s + 1] << 8);
        const uint32_t x = fs + j;
        const uint32_t nb = h.R - (31 - __clz(x));
        const uint32_t nxt = (x << nb) - L;
        const uint32_t lo = rec[2 * h.K + s];
        const uint32_t hi = (s + 1 < h.K) ? rec[2 * h.K + s + 1] : 256u;
        const uint32_t w = (hi - lo <= 1) ? 0u : 32u - __clz(hi - lo - 1);
        tab[i * 32 + lane] = nb | (w << 5) | ((lo ^ 0x80u) << 9) | (nxt << 17);
      }
    }
    const uint32_t w0 = index[g];
    const uint32_t w1 = (c + 1 < nch) ? index[g + 1] : pay_words;
    const uint64_t chunk_byte = h.payload_off + pay_start + 4ull * w0;
    if (!seg_ok || w1 <= w0 || w1 > pay_words || (c == 0 && w0 != 0) ||
        h.payload_off + pay_start + 4ull * w1 > h.stream_bytes) {
      report(st, SHN_ERR_CORRUPT, (uint32_t)g);
      continue;
    }
    BackReader br;
    br.init(reinterpret_cast<const uint32_t*>(comp + chunk_byte), (int)(w1 - w0));
    uint32_t X[S];
#pragma unroll
    for (int q = S - 1; q >= 0; --q) X[q] = br.read(h.R);
    const uint32_t* col = tab + lane;
    uint8_t* dst = out + out_off + (uint64_t)c * h.C;
    const bool aligned = ((reinterpret_cast<uintptr_t>(dst) & 15u) == 0);
    uint32_t i0 = 0;
    for (; i0 + 16 <= len; i0 += 16) {
      uint32_t ov[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        uint32_t& x = X[r & (S - 1)];
        const uint32_t e = col[x * 32];
        const uint32_t nb = e & 31u, w = (e >> 5) & 15u;
        const uint32_t F = br.read(nb + w);
        x = (e >> 17) + (F >> w);
        const uint32_t byte = ((e >> 9) + (F & ((1u << w) - 1u))) & 0xFFu;
        ov[r >> 2] |= byte << (8 * (r & 3));
      }
      if (aligned) {
        *reinterpret_cast<uint4*>(dst + i0) = make_uint4(ov[0], ov[1], ov[2], ov[3]);
      } else {
#pragma unroll
        for (int r = 0; r < 16; ++r) dst[i0 + r] = (uint8_t)(ov[r >> 2] >> (8 * (r & 3)));
      }
    }
    for (uint32_t i = i0; i < len; ++i) {
      const int q = (int)(i & (S - 1));
      uint32_t x = X[0];
#pragma unroll
      for (int k = 1; k < S; ++k)
        if (k == q) x = X[k];
      const uint32_t e = col[x * 32];
      const uint32_t nb = e & 31u, w = (e >> 5) & 15u;
      const uint32_t F = br.read(nb + w);
      x = (e >> 17) + (F >> w);
      dst[i] = (uint8_t)(((e >> 9) + (F & ((1u << w) - 1u))) & 0xFFu);
#pragma unroll
      for (int k = 0; k < S; ++k)
        if (k == q) X[k] = x;
    }
    bool ok = !br.bad && br.P == 0;
#pragma unroll
    for (int q = 0; q < S; ++q) ok = ok && (X[q] == 0u);
    if (!ok) report(st, SHN_ERR_CORRUPT, (uint32_t)g);
  }
}

template <int S>
static cudaError_t launch_decode_t(const uint8_t* d_comp, DeviceStatus* st, uint8_t* d_out, const shn_params& p,
                                   int sm_count, cudaStream_t s) {
  const uint32_t L = 1u << p.log2L;
  const uint32_t col_bytes = L * 32 * 4 + L * 32 + p.K * 32;
  const uint32_t col_words = (col_bytes + 15) / 16 * 4;
  int warps = (int)((96 * 1024) / (col_words * 4));
  warps = warps < 1 ? 1 : (warps > 8 ? 8 : warps);
  const size_t smem = (size_t)warps * col_words * 4;
  cudaError_t e = cudaFuncSetAttribute(decode_kernel<S>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<S>, warps * 32, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  decode_kernel<S><<<sm_count * per_sm, warps * 32, smem, s>>>(d_comp, st, d_out, col_words);
  return cudaGetLastError();
}

cudaError_t launch_decode(const uint8_t* d_comp, uint64_t comp_bytes, const shn_params& p, DeviceStatus* st,
                          uint8_t* d_out, uint64_t out_capacity, int sm_count, cudaStream_t s) {
  decode_check_kernel<<<1, 32, 0, s>>>(d_comp, comp_bytes, p, st, out_capacity);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  switch (p.states_per_chunk) {
    case 1: return launch_decode_t<1>(d_comp, st, d_out, p, sm_count, s);
    case 2: return launch_decode_t<2>(d_comp, st, d_out, p, sm_count, s);
    case 4: return launch_decode_t<4>(d_comp, st, d_out, p, sm_count, s);
    case 8: return launch_decode_t<8>(d_comp, st, d_out, p, sm_count, s);
    case 16: return launch_decode_t<16>(d_comp, st, d_out, p, sm_count, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace shn
