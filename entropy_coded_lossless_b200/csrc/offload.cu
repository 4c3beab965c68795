// offload.cu — a tensor kept compressed in host memory: pipelined offload and reload.
//
// Shannonic §6.2 motivates the use: compressing before a slow transfer pays off when the codec is
// faster than the link for the bytes it saves, since the link then carries r/8 instead of one byte
// per value. Both directions move whole streams with the copy engine (kernel stores and loads over
// the link are slower than its DMA) and overlap them with the codec work of the neighbouring batch:
//  shn_offload           encodes batch i+1 into one device staging stream while the copy engine
//                        moves batch i's stream (exact size, read back once batch i is encoded) to
//                        host memory;
//  shn_decode_from_host  copies stream i+1 to the device while stream i decodes.
#include <stdint.h>
#include <string.h>

#include "shn_internal.cuh"

namespace {

uint64_t host_ld64(const uint8_t* p) {
  uint64_t v;
  memcpy(&v, p, 8);
  return v;
}
uint32_t host_ld32(const uint8_t* p) {
  uint32_t v;
  memcpy(&v, p, 4);
  return v;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Workspace of shn_offload: per-batch log (status + size), histograms and tables of the largest
// batch, the encoder workspace of the largest batch and two staging streams of the largest bound.
struct OffloadLayout {
  size_t log_off, hist_off, tables_off, enc_off, enc_bytes, stage_off, stage_bytes, total;
};

bool offload_layout(const shn_params* p, const shn_segment* h_segs, const uint32_t* batch_ends,
                           uint32_t n_batches, OffloadLayout* l) {
  uint32_t max_segs = 0, prev = 0;
  size_t max_enc = 0, max_bound = 0;
  for (uint32_t b = 0; b < n_batches; ++b) {
    if (batch_ends[b] < prev) return false;
    const uint32_t ns = batch_ends[b] - prev;
    const shn_segment* sb = h_segs + prev;
    const size_t enc = shn_encode_workspace_bytes(p, sb, ns), bound = shn_encode_bound(p, sb, ns);
    if (enc == 0 || bound == 0) return false;
    max_segs = ns > max_segs ? ns : max_segs;
    max_enc = enc > max_enc ? enc : max_enc;
    max_bound = bound > max_bound ? bound : max_bound;
    prev = batch_ends[b];
  }
  l->log_off = 0;
  l->hist_off = align256(16ull * n_batches);
  l->tables_off = l->hist_off + align256(2048ull * (max_segs ? max_segs : 1));
  l->enc_off = l->tables_off + align256((size_t)SHN_TABLE_BYTES * (max_segs ? max_segs : 1));
  l->enc_bytes = align256(max_enc);
  l->stage_off = l->enc_off + l->enc_bytes;
  l->stage_bytes = align256(max_bound);
  l->total = l->stage_off + 2 * l->stage_bytes;
  return true;
}

}  // namespace

extern "C" {

int shn_decode_from_host(const uint8_t* const* h_streams, const size_t* stream_bytes, uint32_t n_streams,
                         const shn_params* p, uint8_t* d_staging, size_t staging_bytes, void* d_work,
                         size_t work_bytes, uint8_t* d_out, const size_t* out_offsets, size_t out_capacity,
                         void* stream, void* copy_stream) {
  using namespace shn;
  if (n_streams == 0) return SHN_OK;
  if (!p || shn_check_params(p) != SHN_OK) return SHN_ERR_INVALID_ARG;
  if (!h_streams || !stream_bytes || !out_offsets || !d_staging || !d_work || !d_out) return SHN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_staging) & 15) || (reinterpret_cast<uintptr_t>(d_work) & 255))
    return SHN_ERR_INVALID_ARG;
  if (work_bytes < 256) return SHN_ERR_WORKSPACE;
  // the headers are in host memory: check every stream's size and output range before enqueueing
  size_t largest = 0;
  for (uint32_t i = 0; i < n_streams; ++i) {
    const uint8_t* h = h_streams[i];
    if (!h || stream_bytes[i] < kHeaderBytes) return SHN_ERR_CORRUPT;
    if (host_ld32(h) != kMagic) return SHN_ERR_CORRUPT;
    const uint64_t total = host_ld64(h + 24);
    if (out_offsets[i] > out_capacity || total > out_capacity - out_offsets[i]) return SHN_ERR_CAPACITY;
    largest = stream_bytes[i] > largest ? stream_bytes[i] : largest;
  }
  const size_t half = (staging_bytes / 2) & ~static_cast<size_t>(15);
  if (half < largest) return SHN_ERR_WORKSPACE;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t cs = static_cast<cudaStream_t>(copy_stream);
  DeviceStatus* st = static_cast<DeviceStatus*>(d_work);
  if (cudaMemsetAsync(st, 0, sizeof(DeviceStatus), s) != cudaSuccess) return SHN_ERR_CUDA;
  cudaEvent_t copied[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr}, start = nullptr;
  int rc = SHN_OK;
  for (int b = 0; b < 2 && rc == SHN_OK; ++b)
    if (cudaEventCreateWithFlags(&copied[b], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&freed[b], cudaEventDisableTiming) != cudaSuccess)
      rc = SHN_ERR_CUDA;
  // the copy stream starts after the status reset and whatever the caller queued on `stream`
  if (rc == SHN_OK && (cudaEventCreateWithFlags(&start, cudaEventDisableTiming) != cudaSuccess ||
                       cudaEventRecord(start, s) != cudaSuccess || cudaStreamWaitEvent(cs, start, 0) != cudaSuccess))
    rc = SHN_ERR_CUDA;
  const int sms = sm_count_for_launch();
  for (uint32_t i = 0; i < n_streams && rc == SHN_OK; ++i) {
    const int b = (int)(i & 1);
    uint8_t* buf = d_staging + (size_t)b * half;
    if (i >= 2 && cudaStreamWaitEvent(cs, freed[b], 0) != cudaSuccess) rc = SHN_ERR_CUDA;  // stream i-2 decoded
    if (rc == SHN_OK && cudaMemcpyAsync(buf, h_streams[i], stream_bytes[i], cudaMemcpyHostToDevice, cs) != cudaSuccess)
      rc = SHN_ERR_CUDA;
    if (rc == SHN_OK && (cudaEventRecord(copied[b], cs) != cudaSuccess || cudaStreamWaitEvent(s, copied[b], 0) != cudaSuccess))
      rc = SHN_ERR_CUDA;
    if (rc == SHN_OK && launch_decode(buf, stream_bytes[i], *p, st, d_out + out_offsets[i],
                                      out_capacity - out_offsets[i], sms, s) != cudaSuccess)
      rc = SHN_ERR_CUDA;
    if (rc == SHN_OK && cudaEventRecord(freed[b], s) != cudaSuccess) rc = SHN_ERR_CUDA;
  }
  // events are released once the work that records or waits on them has completed
  for (int b = 0; b < 2; ++b) {
    if (copied[b]) cudaEventDestroy(copied[b]);
    if (freed[b]) cudaEventDestroy(freed[b]);
  }
  if (start) cudaEventDestroy(start);
  return rc;
}

size_t shn_offload_workspace_bytes(const shn_params* p, const shn_segment* h_segs, const uint32_t* batch_ends,
                                   uint32_t n_batches) {
  if (!p || shn_check_params(p) != SHN_OK || !batch_ends || n_batches == 0 || !h_segs) return 0;
  OffloadLayout l;
  return offload_layout(p, h_segs, batch_ends, n_batches, &l) ? l.total : 0;
}

int shn_offload(const uint8_t* d_in, const shn_segment* h_segs, const uint32_t* batch_ends, uint32_t n_batches,
                const shn_params* p, void* d_work, size_t work_bytes, uint8_t* h_out, size_t h_capacity,
                size_t* h_stream_offsets, size_t* h_stream_bytes, void* stream, void* copy_stream) {
  using namespace shn;
  if (n_batches == 0) return SHN_OK;
  if (!p || shn_check_params(p) != SHN_OK || !h_segs || !batch_ends || !d_work || !h_out || !h_stream_offsets ||
      !h_stream_bytes || !d_in)
    return SHN_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_work) & 255) return SHN_ERR_INVALID_ARG;
  OffloadLayout l;
  if (!offload_layout(p, h_segs, batch_ends, n_batches, &l)) return SHN_ERR_INVALID_ARG;
  if (work_bytes < l.total) return SHN_ERR_WORKSPACE;
  uint8_t* wb = static_cast<uint8_t*>(d_work);
  uint64_t* log = reinterpret_cast<uint64_t*>(wb + l.log_off);  // [2b] = status word, [2b+1] = stream bytes
  uint64_t* hist = reinterpret_cast<uint64_t*>(wb + l.hist_off);
  void* tables = wb + l.tables_off;
  void* enc = wb + l.enc_off;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t cs = static_cast<cudaStream_t>(copy_stream);
  cudaEvent_t encoded[2] = {nullptr, nullptr}, copied[2] = {nullptr, nullptr};
  int rc = SHN_OK;
  for (int k = 0; k < 2 && rc == SHN_OK; ++k)
    if (cudaEventCreateWithFlags(&encoded[k], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&copied[k], cudaEventDisableTiming) != cudaSuccess)
      rc = SHN_ERR_CUDA;
  size_t h_off = 0;
  // batch j is encoded: learn its size and status, then copy its stream out on the copy engine
  auto flush = [&](uint32_t j) -> int {
    const int k = (int)(j & 1);
    uint64_t rec[2];
    if (cudaEventSynchronize(encoded[k]) != cudaSuccess) return SHN_ERR_CUDA;
    if (cudaMemcpyAsync(rec, log + 2 * j, 16, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
        cudaStreamSynchronize(cs) != cudaSuccess)
      return SHN_ERR_CUDA;
    if ((uint32_t)rec[0] != SHN_OK) return (int)(uint32_t)rec[0];
    const size_t nb = (size_t)rec[1];
    if (h_off > h_capacity || nb > h_capacity - h_off) return SHN_ERR_CAPACITY;
    h_stream_offsets[j] = h_off;
    h_stream_bytes[j] = nb;
    if (cudaMemcpyAsync(h_out + h_off, wb + l.stage_off + (size_t)k * l.stage_bytes, nb, cudaMemcpyDeviceToHost,
                        cs) != cudaSuccess ||
        cudaEventRecord(copied[k], cs) != cudaSuccess)
      return SHN_ERR_CUDA;
    h_off += (nb + 15) & ~static_cast<size_t>(15);
    return SHN_OK;
  };
  uint32_t prev = 0;
  for (uint32_t b = 0; b < n_batches && rc == SHN_OK; ++b) {
    const int k = (int)(b & 1);
    const uint32_t ns = batch_ends[b] - prev;
    const shn_segment* sb = h_segs + prev;
    prev = batch_ends[b];
    uint8_t* stage = wb + l.stage_off + (size_t)k * l.stage_bytes;
    if (b >= 2 && cudaStreamWaitEvent(s, copied[k], 0) != cudaSuccess) rc = SHN_ERR_CUDA;  // batch b-2 copied out
    if (rc == SHN_OK) rc = shn_histogram(d_in, sb, ns, hist, s);
    if (rc == SHN_OK) rc = shn_build_tables(hist, ns, p, tables, s);
    if (rc == SHN_OK)
      rc = shn_encode(d_in, sb, ns, tables, p, enc, l.enc_bytes, stage, l.stage_bytes, log + 2 * b + 1, s);
    if (rc == SHN_OK && (cudaMemcpyAsync(log + 2 * b, enc, 8, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
                         cudaEventRecord(encoded[k], s) != cudaSuccess))
      rc = SHN_ERR_CUDA;
    if (rc == SHN_OK && b >= 1) rc = flush(b - 1);
  }
  if (rc == SHN_OK) rc = flush(n_batches - 1);
  for (int k = 0; k < 2; ++k) {
    if (encoded[k]) cudaEventDestroy(encoded[k]);
    if (copied[k]) cudaEventDestroy(copied[k]);
  }
  return rc;
}

}  // extern "C"
