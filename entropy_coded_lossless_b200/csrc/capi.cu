// capi.cu — the extern "C" entry points of libshn (include/shn.h): argument checks, segment
// batching into kernel parameters, workspace layout, and the launch sequence of each call.
// No device allocation and no synchronisation happen here (shn_get_device_status excepted).
#include <stdint.h>
#include <string.h>

#include <vector>

#include "shn_internal.cuh"

using namespace shn;

namespace {

bool params_ok(const shn_params* p) {
  if (!p) return false;
  if (p->K < 1 || p->K > 256 || p->log2L < 4 || p->log2L > 12 || p->K > (1u << p->log2L)) return false;
  const uint32_t S = p->states_per_chunk;
  if (!(S == 1 || S == 2 || S == 4 || S == 8 || S == 16)) return false;
  if (p->chunk_symbols < 128 || p->chunk_symbols > 65536 || (p->chunk_symbols % 128) != 0) return false;
  return true;
}

bool segs_ok(const shn_segment* segs, uint32_t n, uint64_t* total_chunks, uint64_t* total_symbols, uint32_t C) {
  if (n > 0 && !segs) return false;
  uint64_t ch = 0, sy = 0;
  for (uint32_t s = 0; s < n; ++s) {
    if (segs[s].length >= (1ull << 32)) return false;
    if (C) ch += n_chunks(segs[s].length, C);
    sy += segs[s].length;
  }
  if (ch >= (1ull << 32)) return false;
  if (total_chunks) *total_chunks = ch;
  if (total_symbols) *total_symbols = sy;
  return true;
}

int sm_count() { return sm_count_for_launch(); }

// Encode workspace: status word, per-chunk word counts, their exclusive prefix, scan block sums
// (`total`, enough for the two-pass encoder); then, for the single-pass encoder, one worst-case
// slot per chunk (`total_slots`).
struct EncWorkLayout {
  size_t status_off, words_off, offsets_off, sums_off, total, slots_off, total_slots;
  uint32_t scan_blocks, slot_words;
};

EncWorkLayout enc_work_layout(uint64_t total_chunks, const shn_params* p) {
  EncWorkLayout l;
  l.scan_blocks = (uint32_t)((total_chunks + kScanBlock - 1) / kScanBlock);
  l.status_off = 0;
  l.words_off = 256;
  l.offsets_off = l.words_off + round_up(4ull * total_chunks, 256);
  l.sums_off = l.offsets_off + round_up(8ull * (total_chunks + 1), 256);
  l.total = l.sums_off + round_up(8ull * (l.scan_blocks + 1), 256);
  l.slot_words = (uint32_t)round_up(chunk_max_words(p->states_per_chunk, p->log2L, p->chunk_symbols), 4);
  l.slots_off = l.total;
  l.total_slots = l.slots_off + round_up(4ull * l.slot_words * total_chunks, 256);
  return l;
}


}  // namespace

namespace shn {

int check_encode_args(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs, uint64_t* total_chunks,
                      uint64_t* total_symbols) {
  if (!params_ok(p)) return SHN_ERR_INVALID_ARG;
  if (!segs_ok(h_segs, n_segs, total_chunks, total_symbols, p->chunk_symbols)) return SHN_ERR_INVALID_ARG;
  // word offsets inside the payload are 32-bit: streams are limited to 16 GiB
  if (shn_encode_bound(p, h_segs, n_segs) > (16ull << 30)) return SHN_ERR_INVALID_ARG;
  return SHN_OK;
}

uint32_t fill_encode_batch(const shn_params& p, const shn_segment* h_segs, uint32_t n_segs, uint32_t s0,
                           uint64_t& chunk, uint64_t& out_off, EncBatch& b) {
  memset(&b, 0, sizeof(EncBatch));
  uint64_t blocks = 0;
  uint32_t si = s0;
  for (; si < n_segs && b.n < (uint32_t)kSegBatch; ++si) {
    const shn_segment& sg = h_segs[si];
    const uint64_t nc = n_chunks(sg.length, p.chunk_symbols);
    const uint32_t small = (nc <= kEncSmallMaxChunks) ? 1u : 0u;
    if (b.n == 0) b.small = small;
    else if (b.small != small) break;
    const uint32_t i = b.n++;
    b.offset[i] = sg.offset;
    b.out_offset[i] = out_off;
    b.length[i] = (uint32_t)sg.length;
    b.first_chunk[i] = (uint32_t)chunk;
    b.block_start[i] = (uint32_t)blocks;
    b.seg_index[i] = si;
    const uint64_t nt = small ? (uint64_t)kEncSmallThreads : (uint64_t)kEncBlockThreads;
    blocks += (nc + nt - 1) / nt;
    b.total_blocks = (uint32_t)blocks;
    chunk += nc;
    out_off += sg.length;
  }
  return si;
}

}  // namespace shn

extern "C" {

uint32_t shn_version(void) { return SHN_VERSION; }

const char* shn_status_string(int status) {
  switch (status) {
    case SHN_OK: return "ok";
    case SHN_ERR_INVALID_ARG: return "invalid argument";
    case SHN_ERR_CAPACITY: return "output buffer too small";
    case SHN_ERR_CORRUPT: return "corrupt stream";
    case SHN_ERR_CUDA: return "CUDA error";
    case SHN_ERR_TIMEOUT: return "device wait timed out";
    case SHN_ERR_UNSUPPORTED: return "unsupported parameters";
    case SHN_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

int shn_check_params(const shn_params* p) { return params_ok(p) ? SHN_OK : SHN_ERR_INVALID_ARG; }

size_t shn_table_bytes(const shn_params* p) { return params_ok(p) ? (size_t)SHN_TABLE_BYTES : 0; }

size_t shn_encode_bound(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs) {
  uint64_t tc = 0;
  if (!params_ok(p) || !segs_ok(h_segs, n_segs, &tc, nullptr, p->chunk_symbols)) return 0;
  // every chunk holds at most C symbols (SHN1 format §6)
  const uint64_t words = tc * chunk_max_words(p->states_per_chunk, p->log2L, p->chunk_symbols);
  return (size_t)round_up(payload_offset(n_segs, p->K, tc) + 4 * words, 16);
}

size_t shn_encode_workspace_bytes(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs) {
  uint64_t tc = 0;
  if (!params_ok(p) || !segs_ok(h_segs, n_segs, &tc, nullptr, p->chunk_symbols)) return 0;
  return enc_work_layout(tc, p).total_slots;
}

size_t shn_encode_workspace_bytes_min(const shn_params* p, const shn_segment* h_segs, uint32_t n_segs) {
  uint64_t tc = 0;
  if (!params_ok(p) || !segs_ok(h_segs, n_segs, &tc, nullptr, p->chunk_symbols)) return 0;
  return enc_work_layout(tc, p).total;
}

size_t shn_decode_workspace_bytes(const shn_params* p) { return params_ok(p) ? 256 : 0; }

int shn_histogram(const uint8_t* d_in, const shn_segment* h_segs, uint32_t n_segs, uint64_t* d_hist,
                  void* stream) {
  if (n_segs == 0) return SHN_OK;
  if (!d_in || !d_hist || !h_segs || (reinterpret_cast<uintptr_t>(d_hist) & 7)) return SHN_ERR_INVALID_ARG;
  if (!segs_ok(h_segs, n_segs, nullptr, nullptr, 0)) return SHN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(d_hist, 0, sizeof(uint64_t) * 256 * (size_t)n_segs, s) != cudaSuccess) return SHN_ERR_CUDA;
  HistBatch b;
  for (uint32_t s0 = 0; s0 < n_segs; s0 += kSegBatch) {
    memset(&b, 0, sizeof(b));
    b.n = (n_segs - s0 < (uint32_t)kSegBatch) ? n_segs - s0 : (uint32_t)kSegBatch;
    uint64_t bytes = 0;
    for (uint32_t i = 0; i < b.n; ++i) bytes += h_segs[s0 + i].length;
    b.bytes_per_block = histogram_bytes_per_block(bytes, sm_count());
    uint64_t blocks = 0;
    for (uint32_t i = 0; i < b.n; ++i) {
      b.offset[i] = h_segs[s0 + i].offset;
      b.length[i] = (uint32_t)h_segs[s0 + i].length;
      b.block_start[i] = (uint32_t)blocks;
      b.hist_index[i] = s0 + i;
      blocks += histogram_blocks_for(h_segs[s0 + i].length, b.bytes_per_block);
    }
    if (blocks >= (1ull << 31)) return SHN_ERR_INVALID_ARG;
    b.total_blocks = (uint32_t)blocks;
    if (launch_histogram(d_in, b, d_hist, 0, s) != cudaSuccess) return SHN_ERR_CUDA;
  }
  return SHN_OK;
}

int shn_build_tables(const uint64_t* d_hist, uint32_t n_tables, const shn_params* p, void* d_tables, void* stream) {
  if (!params_ok(p)) return SHN_ERR_INVALID_ARG;
  if (n_tables == 0) return SHN_OK;
  if (!d_hist || !d_tables || (reinterpret_cast<uintptr_t>(d_tables) & 255) ||
      (reinterpret_cast<uintptr_t>(d_hist) & 7))
    return SHN_ERR_INVALID_ARG;
  if (n_tables >= (1u << 31)) return SHN_ERR_INVALID_ARG;
  if (launch_build_tables(d_hist, n_tables, *p, static_cast<shn_table*>(d_tables), static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SHN_ERR_CUDA;
  return SHN_OK;
}

int shn_encode(const uint8_t* d_in, const shn_segment* h_segs, uint32_t n_segs, const void* d_tables,
               const shn_params* p, void* d_work, size_t work_bytes, uint8_t* d_out, size_t out_capacity,
               uint64_t* d_out_bytes, void* stream) {
  uint64_t tc = 0, ts = 0;
  const int chk = check_encode_args(p, h_segs, n_segs, &tc, &ts);
  if (chk != SHN_OK) return chk;
  if (!d_work || !d_out || !d_out_bytes || (n_segs > 0 && (!d_in || !d_tables))) return SHN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_out) & 15) || (reinterpret_cast<uintptr_t>(d_work) & 255) ||
      (reinterpret_cast<uintptr_t>(d_out_bytes) & 7) || (d_tables && (reinterpret_cast<uintptr_t>(d_tables) & 255)))
    return SHN_ERR_INVALID_ARG;
  const EncWorkLayout wl = enc_work_layout(tc, p);
  if (work_bytes < wl.total) return SHN_ERR_WORKSPACE;
  const bool single_pass = work_bytes >= wl.total_slots;
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

  uint8_t* wb = static_cast<uint8_t*>(d_work);
  EncodeWork w;
  w.status = reinterpret_cast<DeviceStatus*>(wb + wl.status_off);
  w.chunk_words = reinterpret_cast<uint32_t*>(wb + wl.words_off);
  w.word_offset = reinterpret_cast<unsigned long long*>(wb + wl.offsets_off);
  w.block_sums = reinterpret_cast<unsigned long long*>(wb + wl.sums_off);
  w.scan_blocks = wl.scan_blocks;
  w.slots = single_pass ? reinterpret_cast<uint32_t*>(wb + wl.slots_off) : nullptr;
  w.slot_words = single_pass ? wl.slot_words : 0u;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const shn_table* tables = static_cast<const shn_table*>(d_tables);
  if (cudaMemsetAsync(wb, 0, 8, s) != cudaSuccess) return SHN_ERR_CUDA;

  // Segment batches (kernel parameters), built once and reused by every pass (fill_encode_batch:
  // consecutive segments of one kind, so the header pass indexes a contiguous chunk range).
  std::vector<EncBatch> batches;
  {
    uint64_t chunk = 0, out_off = 0;
    for (uint32_t si = 0; si < n_segs;) {
      batches.emplace_back();
      si = fill_encode_batch(*p, h_segs, n_segs, si, chunk, out_off, batches.back());
    }
  }
  // single pass: code every chunk into its slot (recording sizes); two passes: count sizes first
  for (const EncBatch& b : batches) {
    const cudaError_t e = single_pass ? launch_encode_write(d_in, b, tables, lay, w, d_out, true, s)
                                      : launch_encode_sizes(d_in, b, tables, lay, w, 0, s);
    if (e != cudaSuccess) return SHN_ERR_CUDA;
  }
  if (launch_scan(w, tc, s) != cudaSuccess) return SHN_ERR_CUDA;
  bool first = true;
  for (const EncBatch& b : batches) {
    if (launch_encode_header(b, tables, lay, w, d_out, d_out_bytes, first, s) != cudaSuccess) return SHN_ERR_CUDA;
    first = false;
  }
  if (n_segs == 0) {
    if (launch_encode_empty(lay, w, d_out, d_out_bytes, s) != cudaSuccess) return SHN_ERR_CUDA;
  }
  if (single_pass) {
    if (launch_encode_compact(lay, w, d_out, sm_count(), s) != cudaSuccess) return SHN_ERR_CUDA;
  } else {
    for (const EncBatch& b : batches)
      if (launch_encode_write(d_in, b, tables, lay, w, d_out, false, s) != cudaSuccess) return SHN_ERR_CUDA;
  }
  return SHN_OK;
}

int shn_decode(const uint8_t* d_comp, size_t comp_bytes, const shn_params* p, void* d_work, size_t work_bytes,
               uint8_t* d_out, size_t out_capacity, void* stream) {
  if (!params_ok(p)) return SHN_ERR_INVALID_ARG;
  if (!d_comp || !d_work || (!d_out && out_capacity > 0)) return SHN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_comp) & 15) || (reinterpret_cast<uintptr_t>(d_work) & 255))
    return SHN_ERR_INVALID_ARG;
  if (work_bytes < 256) return SHN_ERR_WORKSPACE;
  if (comp_bytes < kHeaderBytes) return SHN_ERR_CORRUPT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceStatus* st = static_cast<DeviceStatus*>(d_work);
  if (cudaMemsetAsync(st, 0, sizeof(DeviceStatus), s) != cudaSuccess) return SHN_ERR_CUDA;
  if (launch_decode(d_comp, comp_bytes, *p, st, d_out, out_capacity, sm_count(), s) != cudaSuccess)
    return SHN_ERR_CUDA;
  return SHN_OK;
}

int shn_decode_bf16(const uint8_t* d_comp, size_t comp_bytes, const shn_params* p, const float* d_scales,
                    size_t n_scales, uint32_t log2_group, void* d_work, size_t work_bytes, uint16_t* d_out,
                    size_t out_elems, void* stream) {
  if (!params_ok(p)) return SHN_ERR_INVALID_ARG;
  if (!d_comp || !d_work || !d_scales || (!d_out && out_elems > 0)) return SHN_ERR_INVALID_ARG;
  if (log2_group < 4 || log2_group > 31) return SHN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_comp) & 15) || (reinterpret_cast<uintptr_t>(d_work) & 255) ||
      (reinterpret_cast<uintptr_t>(d_out) & 15) || (reinterpret_cast<uintptr_t>(d_scales) & 3))
    return SHN_ERR_INVALID_ARG;
  if (work_bytes < 256) return SHN_ERR_WORKSPACE;
  if (comp_bytes < kHeaderBytes) return SHN_ERR_CORRUPT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceStatus* st = static_cast<DeviceStatus*>(d_work);
  if (cudaMemsetAsync(st, 0, sizeof(DeviceStatus), s) != cudaSuccess) return SHN_ERR_CUDA;
  if (launch_decode_bf16(d_comp, comp_bytes, *p, st, d_out, out_elems, d_scales, log2_group, n_scales, sm_count(),
                         s) != cudaSuccess)
    return SHN_ERR_CUDA;
  return SHN_OK;
}

int shn_get_device_status(const void* d_work, uint32_t* h_status, uint32_t* h_detail, void* stream) {
  if (!d_work || !h_status) return SHN_ERR_INVALID_ARG;
  DeviceStatus st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&st, d_work, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess) return SHN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SHN_ERR_CUDA;
  *h_status = st.status;
  if (h_detail) *h_detail = st.detail;
  return SHN_OK;
}

}  // extern "C"
