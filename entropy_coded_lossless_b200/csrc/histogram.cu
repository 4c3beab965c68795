// histogram.cu — 256-bin histogram of INT8 segments, the first preprocessing step of Shannonic
// §4.1 (counts of every value of the tensor); symbol u = byte ^ 0x80, SHN1 format §1.
//
// HBM-bound: every input byte is read once with 128-bit loads. Each block keeps a lane-private
// histogram in shared memory laid out [byte value][lane], so a warp's 32 increments always land in
// 32 different banks and never on the same word (no intra-warp address collisions, whatever the
// data's skew); only lanes of different warps share a counter, through shared-memory atomics.
// At the end the block folds its 32 columns and adds the 256 totals to the u64 output rows.
#include "shn_internal.cuh"

namespace shn {

constexpr int kHistThreadsPerBlock = 512;
// Bytes per block: as many as keep at least kHistMinBlocksPerSm blocks per SM busy, up to 512 KiB,
// so that zeroing and folding the block's 8192 counters is small beside its loads (measured on the
// 2 GiB KV cache: 92 % of the copy bandwidth at 512 KiB, 85 % at 128 KiB); small tensors get
// blocks down to 32 KiB instead of leaving most SMs idle.
constexpr uint32_t kHistMaxBytesPerBlock = 512u << 10;
constexpr uint32_t kHistMinBytesPerBlock = 32u << 10;
constexpr uint64_t kHistMinBlocksPerSm = 4;

__device__ __forceinline__ void count_word(uint32_t* col, uint32_t w) {
  atomicAdd(col + ((w & 0xFFu) << 5), 1u);
  atomicAdd(col + (((w >> 8) & 0xFFu) << 5), 1u);
  atomicAdd(col + (((w >> 16) & 0xFFu) << 5), 1u);
  atomicAdd(col + ((w >> 24) << 5), 1u);
}

__global__ void __launch_bounds__(kHistThreadsPerBlock) histogram_kernel(const uint8_t* __restrict__ in,
                                                                         const __grid_constant__ HistBatch b,
                                                                         unsigned long long* __restrict__ hist) {
  __shared__ uint32_t sh[256 * 32];
  // which segment does this block belong to (largest s with block_start[s] <= blockIdx.x)
  int lo = 0, hi = (int)b.n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (b.block_start[mid] <= blockIdx.x) lo = mid;
    else hi = mid - 1;
  }
  const int seg = lo;
  const uint32_t part = blockIdx.x - b.block_start[seg];
  const uint64_t seg_begin = b.offset[seg];
  const uint64_t seg_end = seg_begin + b.length[seg];
  const uint64_t begin = seg_begin + (uint64_t)part * b.bytes_per_block;
  const uint64_t end = min(seg_end, begin + b.bytes_per_block);

  for (int i = threadIdx.x; i < 256 * 32; i += blockDim.x) sh[i] = 0;
  __syncthreads();

  uint32_t* col = sh + (threadIdx.x & 31);
  const uintptr_t base = reinterpret_cast<uintptr_t>(in);
  // 16-byte aligned interior [a0, a1) of [begin, end)
  uint64_t a0 = (begin + ((16 - ((base + begin) & 15)) & 15));
  if (a0 > end) a0 = end;
  uint64_t a1 = a0 + ((end - a0) & ~(uint64_t)15);
  for (uint64_t i = begin + threadIdx.x; i < a0; i += blockDim.x) atomicAdd(col + ((uint32_t)in[i] << 5), 1u);
  for (uint64_t i = a1 + threadIdx.x; i < end; i += blockDim.x) atomicAdd(col + ((uint32_t)in[i] << 5), 1u);

  const uint4* v = reinterpret_cast<const uint4*>(in + a0);
  const uint32_t nvec = (uint32_t)((a1 - a0) >> 4);
  uint32_t i = threadIdx.x;
  for (; i + kHistThreadsPerBlock < nvec; i += 2 * kHistThreadsPerBlock) {
    const uint4 x = __ldcs(v + i);
    const uint4 y = __ldcs(v + i + kHistThreadsPerBlock);
    count_word(col, x.x);
    count_word(col, x.y);
    count_word(col, x.z);
    count_word(col, x.w);
    count_word(col, y.x);
    count_word(col, y.y);
    count_word(col, y.z);
    count_word(col, y.w);
  }
  for (; i < nvec; i += kHistThreadsPerBlock) {
    const uint4 x = __ldcs(v + i);
    count_word(col, x.x);
    count_word(col, x.y);
    count_word(col, x.z);
    count_word(col, x.w);
  }
  __syncthreads();

  if (threadIdx.x < 256) {
    const uint32_t byte = threadIdx.x;
    uint32_t sum = 0;
#pragma unroll 8
    for (int l = 0; l < 32; ++l) sum += sh[(byte << 5) + ((l + byte) & 31)];  // rotated: conflict-free
    if (sum) atomicAdd(hist + (uint64_t)b.hist_index[seg] * 256 + (byte ^ 0x80u), (unsigned long long)sum);
  }
}

cudaError_t launch_histogram(const uint8_t* d_in, const HistBatch& b, uint64_t* d_hist, int, cudaStream_t s) {
  if (b.total_blocks == 0) return cudaSuccess;
  histogram_kernel<<<b.total_blocks, kHistThreadsPerBlock, 0, s>>>(
      d_in, b, reinterpret_cast<unsigned long long*>(d_hist));
  return cudaGetLastError();
}

uint32_t histogram_bytes_per_block(uint64_t batch_bytes, int sm_count) {
  uint32_t bpb = kHistMaxBytesPerBlock;
  const uint64_t want = kHistMinBlocksPerSm * (uint64_t)(sm_count > 0 ? sm_count : 1);
  while (bpb > kHistMinBytesPerBlock && batch_bytes / bpb < want) bpb >>= 1;
  return bpb;
}

uint32_t histogram_blocks_for(uint64_t length, uint32_t bytes_per_block) {
  return (uint32_t)((length + bytes_per_block - 1) / bytes_per_block);
}

}  // namespace shn
