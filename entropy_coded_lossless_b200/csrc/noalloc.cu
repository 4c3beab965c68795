// noalloc.cu — shn_encode_static: the encoder for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside a custom allocator or an
// out-of-memory handler, a plugin whose host application owns every device allocation, or a
// latency-critical path that must not risk the implicit synchronisation of an allocation. shn_encode
// needs scratch memory beyond its inputs and outputs (per-chunk word counts and their prefix sums),
// which those callers cannot provide. This file gives them an entry point whose scratch is a
// fixed-size array in the library's own device memory, reserved when the library is loaded.
//
// The array lives at file scope as a `static __device__` variable. Host code cannot use its name as
// a device address (on the host the name denotes a host-side stand-in), so the device address is
// looked up once per device with cudaGetSymbolAddress while that device is current, and passed to
// the kernels like any other pointer.
#include <string.h>

#include <mutex>

#include "shn_internal.cuh"

using namespace shn;

namespace {

// chunk word counts (u32) + their exclusive prefix sums (u64, one extra) + scan block sums (u64).
constexpr uint64_t up256(uint64_t x) { return (x + 255) / 256 * 256; }
constexpr uint64_t kStaticMaxChunks = SHN_STATIC_MAX_CHUNKS;
constexpr uint64_t kWordsBytes = up256(4 * kStaticMaxChunks);
constexpr uint64_t kOffsetsBytes = up256(8 * (kStaticMaxChunks + 1));
constexpr uint64_t kSumsBytes = up256(8 * ((kStaticMaxChunks + kScanBlock - 1) / kScanBlock + 1));
constexpr uint64_t kScratchBytes = kWordsBytes + kOffsetsBytes + kSumsBytes;

static __device__ __align__(256) unsigned char g_encode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_encode_scratch on the current device (looked up on first use per device).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_encode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

bool params_ok(const shn_params* p) { return shn_check_params(p) == SHN_OK; }


}  // namespace

extern "C" {

uint64_t shn_encode_static_max_chunks(void) { return kStaticMaxChunks; }

int shn_encode_static(const uint8_t* d_in, const shn_segment* h_segs, uint32_t n_segs, const void* d_tables,
                      const shn_params* p, uint8_t* d_out, size_t out_capacity, uint64_t* d_out_bytes,
                      uint32_t* d_status, void* stream) {
  if (!params_ok(p)) return SHN_ERR_INVALID_ARG;
  if (n_segs > 0 && !h_segs) return SHN_ERR_INVALID_ARG;
  uint64_t tc = 0, ts = 0;
  for (uint32_t s = 0; s < n_segs; ++s) {
    if (h_segs[s].length >= (1ull << 32)) return SHN_ERR_INVALID_ARG;
    tc += n_chunks(h_segs[s].length, p->chunk_symbols);
    ts += h_segs[s].length;
  }
  if (tc > kStaticMaxChunks) return SHN_ERR_CAPACITY;
  if (!d_out || !d_out_bytes || !d_status || (n_segs > 0 && (!d_in || !d_tables))) return SHN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_out) & 15) || (reinterpret_cast<uintptr_t>(d_out_bytes) & 7) ||
      (reinterpret_cast<uintptr_t>(d_status) & 7) || (d_tables && (reinterpret_cast<uintptr_t>(d_tables) & 255)))
    return SHN_ERR_INVALID_ARG;
  EncodeLayout lay;
  lay.n_segs = n_segs;
  lay.K = p->K;
  lay.R = p->log2L;
  lay.S = p->states_per_chunk;
  lay.C = p->chunk_symbols;
  lay.total_chunks = tc;
  lay.total_symbols = ts;
  lay.index_offset = index_offset(n_segs, p->K);
  lay.payload_offset = payload_offset(n_segs, p->K, tc);
  lay.out_capacity = out_capacity;
  if (out_capacity < lay.payload_offset) return SHN_ERR_CAPACITY;

  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return SHN_ERR_CUDA;
  uint8_t* sb = static_cast<uint8_t*>(scratch);
  EncodeWork w;
  w.status = reinterpret_cast<DeviceStatus*>(d_status);
  w.chunk_words = reinterpret_cast<uint32_t*>(sb);
  w.word_offset = reinterpret_cast<unsigned long long*>(sb + kWordsBytes);
  w.block_sums = reinterpret_cast<unsigned long long*>(sb + kWordsBytes + kOffsetsBytes);
  w.scan_blocks = (uint32_t)((tc + kScanBlock - 1) / kScanBlock);
  w.slots = nullptr;  // the two-pass encoder: no per-chunk slots
  w.slot_words = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const shn_table* tables = static_cast<const shn_table*>(d_tables);
  // Only the status must start at zero: every scratch word the passes read is written first
  // (word counts by the size pass, offsets and block sums by the scan).
  if (cudaMemsetAsync(d_status, 0, sizeof(DeviceStatus), s) != cudaSuccess) return SHN_ERR_CUDA;

  EncBatch b;
  uint64_t chunk = 0, out_off = 0;
  // the same launch sequence as shn_encode: sizes, scan, header/index, write; the batch
  // parameters are rebuilt for each pass from h_segs
  for (int pass = 0; pass < 3; ++pass) {
    chunk = 0;
    out_off = 0;
    bool first = true;
    for (uint32_t s0 = 0; s0 < n_segs; s0 += kSegBatch) {
      memset(&b, 0, sizeof(b));
      b.n = (n_segs - s0 < (uint32_t)kSegBatch) ? n_segs - s0 : (uint32_t)kSegBatch;
      uint64_t blocks = 0;
      for (uint32_t i = 0; i < b.n; ++i) {
        const shn_segment& sg = h_segs[s0 + i];
        b.offset[i] = sg.offset;
        b.out_offset[i] = out_off;
        b.length[i] = (uint32_t)sg.length;
        b.first_chunk[i] = (uint32_t)chunk;
        b.block_start[i] = (uint32_t)blocks;
        b.seg_index[i] = s0 + i;
        const uint64_t nc = n_chunks(sg.length, p->chunk_symbols);
        blocks += (nc + kEncBlockThreads - 1) / kEncBlockThreads;
        chunk += nc;
        out_off += sg.length;
      }
      b.total_blocks = (uint32_t)blocks;
      cudaError_t e = cudaSuccess;
      if (pass == 0) e = launch_encode_sizes(d_in, b, tables, lay, w, 0, s);
      if (pass == 1) e = launch_encode_header(b, tables, lay, w, d_out, d_out_bytes, first, s);
      if (pass == 2) e = launch_encode_write(d_in, b, tables, lay, w, d_out, false, s);
      if (e != cudaSuccess) return SHN_ERR_CUDA;
      first = false;
    }
    if (pass == 0 && launch_scan(w, tc, s) != cudaSuccess) return SHN_ERR_CUDA;
    if (pass == 1 && n_segs == 0 && launch_encode_empty(lay, w, d_out, d_out_bytes, s) != cudaSuccess)
      return SHN_ERR_CUDA;
  }
  return SHN_OK;
}

}  // extern "C"
