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

}  // namespace

extern "C" {

uint64_t shn_encode_static_max_chunks(void) { return kStaticMaxChunks; }

int shn_encode_static(const uint8_t* d_in, const shn_segment* h_segs, uint32_t n_segs, const void* d_tables,
                      const shn_params* p, uint8_t* d_out, size_t out_capacity, uint64_t* d_out_bytes,
                      uint32_t* d_status, void* stream) {
  // the checks shn_encode makes (parameters, segments, the 16 GiB stream limit), then the chunk
  // count the static scratch holds
  uint64_t tc = 0, ts = 0;
  const int chk = check_encode_args(p, h_segs, n_segs, &tc, &ts);
  if (chk != SHN_OK) return chk;
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

  // shn_encode's two-pass launch sequence (sizes, scan, header and index, write in place) over the
  // same segment batches; a batch is rebuilt on the stack for each pass instead of being kept.
  EncBatch b;
  for (int pass = 0; pass < 3; ++pass) {
    uint64_t chunk = 0, out_off = 0;
    bool first = true;
    for (uint32_t s0 = 0; s0 < n_segs;) {
      s0 = fill_encode_batch(*p, h_segs, n_segs, s0, chunk, out_off, b);
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
