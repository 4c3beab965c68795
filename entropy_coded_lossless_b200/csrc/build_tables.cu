// build_tables.cu — per-segment range selection and tANS tables, a cluster of blocks per table.
//
// Shannonic §4.1 (preprocessing): partition the 256-value alphabet into K contiguous ranges by the
// DP C[i,k] = min_{j<i} { C[j,k-1] + Cost(j,i-1) } with backtracking from C[256,K]; derive the
// per-range parameters (base, offset bits, encTable start, normalisation bias), rangeId[256], and an
// L-entry tANS table from the range probabilities. The exact integer rules (fixed-point log2, cost,
// tie-breaks, state-count allocation, spread) are SHN1 format §2-§5; this kernel must reproduce them
// bit for bit, so it uses only integer arithmetic.
//
// Work is small (O(K·256²/2) min-plus steps per table) and latency-bound, so a table is built by a
// cluster of G blocks (G = 1, 2, 4 or 8: the launch takes the largest G that still gives every
// block its own SM). The DP's end points i = 1..256 are paired as (256 - g, g + 1), g = 0..127,
// which together have 257 candidate starts whatever g; a group of 4G threads of cluster block r
// owns pair g = group * G + r. A block keeps the per-symbol cost factor (w << 24) - LG(count) of
// the ranges [j, i) ending at its own end points (257 entries per pair) and a copy of the two DP
// rows; after each layer every group writes its two new cells into every block's row copy and its
// argmins into block 0, through distributed shared memory, and the cluster meets at a barrier.
// Block 0 then backtracks and builds the rest of the table alone (state counts, spread, tables).
#include <cooperative_groups.h>

#include "shn_internal.cuh"

namespace cg = cooperative_groups;

namespace shn {

constexpr int kBuildThreads = 512;

// LG(c) for every c < 2^17, filled by lg_table_kernel on the launching stream before a build of
// many tables (more than one wave of blocks); tables whose segment total is below 2^17 then look
// LG up instead of running the 24 squaring steps per range. Values are those of lg_fixed.
constexpr uint32_t kLgTableSize = 1u << 17;
constexpr uint32_t kLgTableMinTables = 256;  // builds of fewer tables compute LG directly
__device__ uint32_t g_lg_table[kLgTableSize];

__global__ void __launch_bounds__(256) lg_table_kernel() {
  for (uint32_t c = blockIdx.x * blockDim.x + threadIdx.x; c < kLgTableSize; c += gridDim.x * blockDim.x)
    g_lg_table[c] = lg_fixed(c);
}

__device__ __forceinline__ uint32_t ceil_log2_width(uint32_t m) { return m <= 1 ? 0u : 32u - __clz(m - 1u); }

// Words per end-point pair of the cost-factor table in a block of a G-block cluster: room for both
// rows (257 words) after row ib's shift of up to 31 words, rounded to 4G modulo 32.
__host__ __device__ constexpr int build_stride(int G) { return 4 * G == 32 ? 288 : 288 + 4 * G; }

struct BuildShared {
  uint32_t pre[257];       // prefix sums of the histogram (total < 2^32)
  long long drow[2][257];  // DP rows D[.][k-1], D[.][k]
  uint32_t lgf[4097];      // LG(f) for f = 0..L
  uint32_t f[256];
  uint32_t cumul[257];
  uint32_t lo[257];
  uint32_t rng[256];       // range of each symbol u
  uint8_t spread[4096];
  uint32_t status;
  long long cost;
};

// Scratch of the threshold allocation, placed over the DP's cost factors (dead by then).
struct NormScratch {
  unsigned long long red64[kBuildThreads / 32];  // block reductions
  uint32_t red32[kBuildThreads / 32];
  uint32_t ties[256];                            // per range: gains equal to the threshold, then those taken
};

// Greedy state allocation on one warp (SHN1 format §4), one state per step, for L <= 128 (K <= 128):
// every range with a count starts with one state; each further state goes to the range with the
// largest N_k * (LG(f_k + 1) - LG(f_k)), ties to the smallest k. kPer ranges per lane (K <= 32 * kPer).
template <int kPer>
__device__ __forceinline__ void normalize_warp(BuildShared& S, int K, uint32_t L, int tid) {
  unsigned long long N[kPer];
  uint32_t f[kPer];
  int nonzero = 0;
  unsigned long long total = 0;
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int k = tid + 32 * r;
    N[r] = (k < K) ? (unsigned long long)(S.pre[S.lo[k + 1]] - S.pre[S.lo[k]]) : 0ull;
    f[r] = N[r] > 0 ? 1u : 0u;
    nonzero += (int)f[r];
    total += N[r];
  }
  for (int o = 16; o > 0; o >>= 1) {
    nonzero += __shfl_xor_sync(0xffffffffu, nonzero, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if (total == 0) {
#pragma unroll
    for (int r = 0; r < kPer; ++r) f[r] = (tid == 0 && r == 0) ? L : 0u;
  } else {
    // K <= L is checked on the host, so nonzero <= L. G[r] caches the gain of the next state of
    // range tid + 32 r (0 for an empty range; every other gain is > 0, as LG is strictly increasing).
    // Only the winning range's gain changes in a step, so one gain is recomputed per step.
    unsigned long long G[kPer];
#pragma unroll
    for (int r = 0; r < kPer; ++r)
      G[r] = N[r] > 0 ? N[r] * (unsigned long long)(S.lgf[f[r] + 1] - S.lgf[f[r]]) : 0ull;
    unsigned long long bg;
    int bk;
    auto rescan = [&]() {  // largest cached gain of this lane, ties to the smallest k (tournament, left wins ties)
      unsigned long long gv[kPer];
      int kv[kPer];
#pragma unroll
      for (int r = 0; r < kPer; ++r) {
        gv[r] = G[r];
        kv[r] = tid + 32 * r;
      }
#pragma unroll
      for (int w = 1; w < kPer; w <<= 1)
#pragma unroll
        for (int r = 0; r + w < kPer; r += 2 * w)
          if (gv[r + w] > gv[r]) {
            gv[r] = gv[r + w];
            kv[r] = kv[r + w];
          }
      bg = gv[0];
      bk = gv[0] > 0 ? kv[0] : 0x7fffffff;
    };
    rescan();
    for (uint32_t step = 0; step < L - (uint32_t)nonzero; ++step) {
      // warp argmax of (gain, then smallest k) with three reductions: the high word of the gain,
      // the low word among lanes at that high word, the smallest k among lanes at the maximum.
      const uint32_t ghi = (uint32_t)(bg >> 32), glo = (uint32_t)bg;
      const uint32_t m1 = __reduce_max_sync(0xffffffffu, ghi);
      const uint32_t m2 = __reduce_max_sync(0xffffffffu, ghi == m1 ? glo : 0u);
      const int win = (int)__reduce_min_sync(0xffffffffu, (ghi == m1 && glo == m2 && bk != 0x7fffffff) ? (uint32_t)bk
                                                                                                        : 0xffffffffu);
      // The winning range's lane gives it one more state and caches its next gain. Every lane runs
      // the same instructions (no divergence); on the others the writes are predicated off and the
      // rescan finds the best it already had.
      const bool mine = (win & 31) == tid;
      const int rw = win >> 5;
      uint32_t fw = f[0];
      unsigned long long nw = N[0];
#pragma unroll
      for (int r = 1; r < kPer; ++r)
        if (r == rw) {
          fw = f[r];
          nw = N[r];
        }
      fw += 1;  // on the winner, fw == L only after the last step (lgf has L + 1 entries)
      const unsigned long long gw = fw < L ? nw * (unsigned long long)(S.lgf[fw + 1] - S.lgf[fw]) : 0ull;
#pragma unroll
      for (int r = 0; r < kPer; ++r)
        if (mine && r == rw) {
          f[r] = fw;
          G[r] = gw;
        }
      rescan();
    }
  }
#pragma unroll
  for (int r = 0; r < kPer; ++r) {
    const int k = tid + 32 * r;
    if (k < K) S.f[k] = f[r];  // S.f[K..255] were zeroed by the caller
  }
}

// State counts (SHN1 format §4): every range with a count starts with one state; each further state
// goes to the range with the largest gain N_k * (LG(f_k + 1) - LG(f_k)), ties to the smallest k.
// Each range's gains form a non-increasing sequence in f_k (LG's fixed-point differences never grow
// for f <= 4096), so the M = L - nonzero states that greedy hands out one by one are the first M
// elements (k, f) in the order (gain down, k up, f up): every element whose gain is above the M-th
// largest gain v, then the elements equal to v in range order. The block finds v by bisection on the
// gain, each thread counting its range's elements above a trial value (thread k holds range k).
// Used from L = 256 up, where it takes fewer block-wide rounds (about 56) than the greedy has steps.
__device__ void normalize_block(BuildShared& S, NormScratch& Z, int K, uint32_t L, int tid) {
  const int lane = tid & 31, wid = tid >> 5;
  const unsigned long long N = tid < K ? (unsigned long long)(S.pre[S.lo[tid + 1]] - S.pre[S.lo[tid]]) : 0ull;
  auto sum_u32 = [&](uint32_t v) -> uint32_t {  // block-wide, every thread gets the sum
    v = __reduce_add_sync(0xffffffffu, v);
    if (lane == 0) Z.red32[wid] = v;
    __syncthreads();
    uint32_t t = 0;
#pragma unroll
    for (int i = 0; i < kBuildThreads / 32; ++i) t += Z.red32[i];
    __syncthreads();
    return t;
  };
  const uint32_t nonzero = sum_u32(N > 0 ? 1u : 0u);
  if (nonzero == 0) {  // an empty segment: all states on range 0
    if (tid < K) S.f[tid] = tid == 0 ? L : 0u;
    return;
  }
  const uint32_t M = L - nonzero;  // K <= L is checked on the host, so nonzero <= L
  // gain of the (f + 1)-th state, f = 1 .. L - 1
  auto gain = [&](uint32_t f) -> unsigned long long { return N * (unsigned long long)(S.lgf[f + 1] - S.lgf[f]); };
  // number of this range's elements with gain > tau: the largest f in [1, L-1] with gain(f) > tau, or
  // 0. Started from f ~ N 2^24 / (tau ln 2) (the gains are close to N 2^24 / (f ln 2)) and corrected
  // in unit steps, which is exact because the gains never increase with f.
  auto count_gt = [&](unsigned long long tau) -> uint32_t {
    if (N == 0) return 0;
    const float est = (float)N * 24204406.32f / fmaxf((float)tau, 1.0f);  // 2^24 / ln 2
    uint32_t f = est >= (float)(L - 1) ? L - 1 : (uint32_t)est;
    while (f + 1 <= L - 1 && gain(f + 1) > tau) ++f;
    while (f >= 1 && gain(f) <= tau) --f;
    return f;
  };
  uint32_t f = N > 0 ? 1u : 0u;
  if (M > 0) {
    unsigned long long hi = N > 0 ? gain(1) : 0ull;  // no element is above the largest first gain
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    if (lane == 0) Z.red64[wid] = hi;
    __syncthreads();
    hi = 0;
#pragma unroll
    for (int i = 0; i < kBuildThreads / 32; ++i) hi = max(hi, Z.red64[i]);
    unsigned long long lo = 0;  // all L - 1 elements of every counted range are above 0, and M <= that
    while (hi - lo > 1) {       // invariant: at least M elements above lo, fewer than M above hi
      const unsigned long long mid = lo + ((hi - lo) >> 1);
      if (sum_u32(count_gt(mid)) >= M) lo = mid;
      else hi = mid;
    }
    const unsigned long long v = hi;  // the M-th largest gain
    const uint32_t above = count_gt(v);
    const uint32_t r = M - sum_u32(above);  // elements equal to v that are taken, in range order
    if (tid < K) Z.ties[tid] = count_gt(v - 1) - above;
    __syncthreads();
    if (tid == 0) {
      uint32_t seen = 0;
      for (int k = 0; k < K; ++k) {
        const uint32_t e = Z.ties[k];
        Z.ties[k] = seen >= r ? 0u : min(e, r - seen);
        seen += e;
      }
    }
    __syncthreads();
    if (N > 0) f = 1 + above + Z.ties[tid];
  }
  if (tid < K) S.f[tid] = f;  // S.f[K..255] were zeroed by the caller
}

// G blocks per table (launched as clusters of G when G > 1).
template <int G>
__global__ void __launch_bounds__(kBuildThreads)
    build_tables_kernel(const unsigned long long* __restrict__ hist_all, shn_params p,
                        shn_table* __restrict__ tables_out, uint32_t use_lg_table) {
  constexpr int T = 4 * G;                 // threads per end-point pair (a power of two that divides 32)
  constexpr int P = 128 / G;               // end-point pairs per block
  constexpr int kStride = build_stride(G);  // words per pair's cost factors
  static_assert(P * T == kBuildThreads, "every thread of a block works on one pair");
  static_assert(sizeof(NormScratch) <= sizeof(uint32_t) * P * kStride, "the allocation scratch fits the cost table");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  BuildShared& S = *reinterpret_cast<BuildShared*>(smem_raw);
  uint32_t* lgc = reinterpret_cast<uint32_t*>(smem_raw + sizeof(BuildShared));  // P x kStride cost factors
  uint8_t* arg = reinterpret_cast<uint8_t*>(lgc + P * kStride);                    // K x 257 (used in block 0)
  // G = 1 is an ordinary launch: block barriers and this block's own shared memory
  cg::cluster_group cluster = cg::this_cluster();
  const uint32_t rank = G > 1 ? cluster.block_rank() : 0u;
  auto cluster_sync = [&]() {
    if constexpr (G > 1) cluster.sync();
    else __syncthreads();
  };
  auto in_block = [&](auto* ptr, int r) {
    if constexpr (G > 1) return cluster.map_shared_rank(ptr, r);
    else return ptr;
  };

  const int tid = threadIdx.x;
  const int K = (int)p.K;
  const int R = (int)p.log2L;
  const uint32_t L = 1u << R;
  const unsigned long long* hist = hist_all + (size_t)(blockIdx.x / G) * 256;
  shn_table* out = tables_out + blockIdx.x / G;

  // ---- prefix sums and the 2^32 bound (every block of the cluster, from the same counts) ------
  if (tid < 32) {  // warp 0: lane l sums counts 8l .. 8l+7, then a shuffle scan over the lanes
    unsigned long long v[8], acc = 0;
#pragma unroll
    for (int r = 0; r < 8; ++r) v[r] = hist[8 * tid + r];  // eight independent loads in flight
#pragma unroll
    for (int r = 0; r < 8; ++r) acc += v[r];
    unsigned long long incl = acc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += y;
    }
    unsigned long long run = incl - acc;  // exclusive prefix of this lane
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      run += v[r];
      S.pre[8 * tid + r + 1] = (uint32_t)run;
    }
    if (tid == 31) {
      S.pre[0] = 0;
      S.status = incl >= (1ull << 32) ? (uint32_t)SHN_ERR_INVALID_ARG : 0u;
      S.cost = 0;
      if (rank == 0) out->n = incl;
    }
  }
  if (rank == 0)
    for (uint32_t f = tid; f <= L; f += kBuildThreads) S.lgf[f] = lg_fixed(f);
  __syncthreads();
  // Every block reaches the same decision from the same counts, so a cluster either runs all of its
  // barriers below or none.
  if (S.status != 0) {
    if (rank == 0 && tid == 0) {
      out->K = K;
      out->log2L = R;
      out->status = S.status;
    }
    return;
  }

  // ---- range selection (SHN1 format §3) ---------------------------------------------------------
  if (K == 256) {
    if (rank != 0) return;
    if (tid < 256) {
      S.lo[tid] = tid;
      const uint32_t n = S.pre[tid + 1] - S.pre[tid];
      // two's-complement sum of -n * LG(n) over the 256 singletons (S.cost starts at 0)
      atomicAdd(reinterpret_cast<unsigned long long*>(&S.cost), 0ull - (unsigned long long)n * lg_fixed(n));
    }
  } else {
    const int grp = tid / T, lane = tid % T;  // a group is T consecutive lanes of one warp
    const int g = grp * G + (int)rank;
    const int ia = 256 - g, ib = g + 1;
    // Row ia, then row ib from word ia + (g mod 32) of the pair's block: with a stride of T mod 32
    // words, both rows of the groups of one warp start T banks apart, so the T lanes of each group
    // read T consecutive banks that no other group of the warp uses.
    uint32_t* lg_a = lgc + grp * kStride;
    uint32_t* lg_b = lg_a + ia + (g & 31);
    // per-symbol cost of range [j, i) in units of 2^-24 bit: w << 24 - LG(count), |.| < 2^30
    const bool lookup = use_lg_table && S.pre[256] < kLgTableSize;  // every count of the segment is < 2^17
    for (int e = lane; e < 257; e += T) {
      const int i = e < ia ? ia : ib, j = e < ia ? e : e - ia;
      const uint32_t c = S.pre[i] - S.pre[j];
      (e < ia ? lg_a : lg_b)[j] = (uint32_t)((int32_t)(ceil_log2_width((uint32_t)(i - j)) << 24) -
                                             (int32_t)(lookup ? __ldg(g_lg_table + c) : lg_fixed(c)));
    }
    for (int i = tid; i <= 256; i += kBuildThreads) S.drow[0][i] = (i == 0) ? 0 : LLONG_MAX;
    cluster_sync();  // every block has started and initialised its rows before any remote write
    uint8_t* arg0 = in_block(arg, 0);
    // Layer k: the group's lanes take every T-th candidate start in ascending j with a strict <, and
    // the group reduction prefers the smaller value, then the smaller j: the smallest j wins ties.
    // Only end points i <= 256 - (K - k) can lie on a split into K non-empty ranges (the K - k ranges
    // still to come need a symbol each), and every cell that does reads only such cells of the layer
    // before; the cells above that band are never read, so they are not computed (at K = 256 the
    // band is the single split into identity ranges).
    const uint32_t pa = S.pre[ia], pb = S.pre[ib];
    for (int k = 1; k <= K; ++k) {
      const long long* prev = S.drow[(k - 1) & 1];
      const int imax = 256 - (K - k);
      const int na = (ia >= k && ia <= imax) ? ((k == 1) ? 1 : ia - k + 1) : 0;  // j = k-1 .. (k == 1 ? 0 : i-1)
      const int nb = (ib >= k && ib <= imax) ? ((k == 1) ? 1 : ib - k + 1) : 0;
      long long best_a = LLONG_MAX, best_b = LLONG_MAX;
      int bj_a = 0x7fffffff, bj_b = 0x7fffffff;
      // Cost(j, i-1) = c * (w << 24) - c * LG(c) = c * lg[j]
      for (int t = lane; t < na; t += T) {
        const int j = (k - 1) + t;
        const long long v = prev[j] + (long long)(pa - S.pre[j]) * (long long)(int32_t)lg_a[j];
        if (v < best_a) {
          best_a = v;
          bj_a = j;
        }
      }
      for (int t = lane; t < nb; t += T) {
        const int j = (k - 1) + t;
        const long long v = prev[j] + (long long)(pb - S.pre[j]) * (long long)(int32_t)lg_b[j];
        if (v < best_b) {
          best_b = v;
          bj_b = j;
        }
      }
#pragma unroll
      for (int o = 1; o < T; o <<= 1) {
        const long long oa = __shfl_xor_sync(0xffffffffu, best_a, o);
        const int oja = __shfl_xor_sync(0xffffffffu, bj_a, o);
        if (oa < best_a || (oa == best_a && oja < bj_a)) {
          best_a = oa;
          bj_a = oja;
        }
        const long long ob = __shfl_xor_sync(0xffffffffu, best_b, o);
        const int ojb = __shfl_xor_sync(0xffffffffu, bj_b, o);
        if (ob < best_b || (ob == best_b && ojb < bj_b)) {
          best_b = ob;
          bj_b = ojb;
        }
      }
      // lanes 0..G-1 write cell ia into blocks 0..G-1, lanes G..2G-1 cell ib; lanes 2G and 2G+1 the
      // argmins (into block 0)
      long long* cur = S.drow[k & 1];
      if (lane < G && na > 0) in_block(cur, lane)[ia] = best_a;
      if (lane >= G && lane < 2 * G && nb > 0) in_block(cur, lane - G)[ib] = best_b;
      if (lane == 2 * G && na > 0) arg0[(size_t)(k - 1) * 257 + ia] = (uint8_t)bj_a;
      if (lane == 2 * G + 1 && nb > 0) arg0[(size_t)(k - 1) * 257 + ib] = (uint8_t)bj_b;
      if (tid < k) cur[tid] = LLONG_MAX;  // cells below the band, in this block's copy (no one else writes them)
      cluster_sync();
    }
    if (rank != 0) return;  // no block reads another's shared memory after the last barrier
    if (tid == 0) {
      S.cost = S.drow[K & 1][256];
      int ii = 256;
      for (int k = K; k >= 1; --k) {
        const int j = arg[(size_t)(k - 1) * 257 + ii];
        S.lo[k - 1] = (uint32_t)j;
        ii = j;
      }
    }
  }
  __syncthreads();
  if (tid == 0) S.lo[K] = 256;
  if (tid < 256) S.f[tid] = 0;
  __syncthreads();

  // ---- state counts (SHN1 format §4): the greedy one state per step on one warp at L <= 128, its
  // result by a threshold on the gains at larger L --------------------------------------------------
  if (L >= 256) {
    normalize_block(S, *reinterpret_cast<NormScratch*>(lgc), K, L, tid);
  } else if (tid < 32) {
    if (K <= 32) normalize_warp<1>(S, K, L, tid);
    else if (K <= 64) normalize_warp<2>(S, K, L, tid);
    else normalize_warp<4>(S, K, L, tid);
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t acc = 0;
    for (int k = 0; k < K; ++k) {
      S.cumul[k] = acc;
      acc += S.f[k];
    }
    S.cumul[K] = acc;
  }
  if (tid < 256) {
    // range of symbol u: largest k with lo[k] <= u
    int a = 0, b2 = K - 1;
    while (a < b2) {
      const int m = (a + b2 + 1) >> 1;
      if (S.lo[m] <= (uint32_t)tid) a = m;
      else b2 = m - 1;
    }
    S.rng[tid] = (uint32_t)a;
  }
  __syncthreads();

  // ---- spread (SHN1 format §5) ------------------------------------------------------------------
  const uint32_t step = (L >> 1) + (L >> 3) + 3;
  for (uint32_t t = tid; t < L; t += kBuildThreads) {
    int a = 0, b2 = K - 1;  // largest k with cumul[k] <= t
    while (a < b2) {
      const int m = (a + b2 + 1) >> 1;
      if (S.cumul[m] <= t) a = m;
      else b2 = m - 1;
    }
    S.spread[(t * step) & (L - 1)] = (uint8_t)a;
  }
  __syncthreads();

  // ---- encode table: enc[cumul_s + j] = L + (j-th slot of s) ---------------------------------
  uint16_t* enc = reinterpret_cast<uint16_t*>(out->opaque + kOpaqueEncOffset);
  for (int k = tid; k < K; k += kBuildThreads) {
    uint32_t j = S.cumul[k];
    if (S.f[k] == 0) continue;
    for (uint32_t i = 0; i < L; ++i)
      if (S.spread[i] == (uint8_t)k) enc[j++] = (uint16_t)(L + i);
  }
  // ---- per raw byte encoder entries -----------------------------------------------------------
  if (tid < 256) {
    const uint32_t bb = (uint32_t)tid;  // raw byte
    const uint32_t u = bb ^ 0x80u;
    const uint32_t s = S.rng[u];
    const uint32_t fs = S.f[s];
    const uint32_t o = u - S.lo[s];
    const uint32_t w = ceil_log2_width(S.lo[s + 1] - S.lo[s]);
    // .x: bias + 2^22 in bits 0-22 (so that (X + .x) >> 16 = nb + 64, with the offset's bits from
    //     bit 8 up), and the offset top-aligned in the w highest bits (a funnel shift of the state
    //     bits into .x appends it below them);
    // .y: w in bits 0-4 (a shift amount as it stands), bit 7 set for a byte whose range has no
    //     states, encTable start + 4096 in bits 16-31.
    const uint32_t off_top = w ? (o << (32u - w)) : 0u;
    uint2 e;
    if (fs == 0) {
      e.x = (1u << 22) + off_top;  // nb = 0; enc index = X - L stays inside the table
      e.y = w | 0x80u | ((4096u - L) << 16);
    } else {
      const uint32_t a = 31u - __clz(fs);
      const uint32_t sh = (uint32_t)R - a;
      e.x = (sh << 16) - (fs << sh) + (1u << 22) + off_top;
      e.y = w | ((uint32_t)((int)S.cumul[s] - (int)fs + 4096) << 16);
    }
    reinterpret_cast<uint2*>(out->opaque + kOpaqueSymOffset)[bb] = e;
    out->f[tid] = (uint16_t)S.f[tid];
    out->lo[tid] = (uint8_t)((tid < K) ? S.lo[tid] : 0u);
  }
  if (tid == 0) {
    uint32_t wmax = 0;
    for (int k = 0; k < K; ++k) wmax = max(wmax, ceil_log2_width(S.lo[k + 1] - S.lo[k]));
    out->K = K;
    out->log2L = R;
    out->status = 0;
    out->w_max = wmax;
    out->dp_cost = S.cost;
  }
}

template <int G>
static cudaError_t launch_build_g(const uint64_t* d_hist, uint32_t n_tables, const shn_params& p, shn_table* d_tables,
                                 uint32_t use_table, cudaStream_t s) {
  const size_t smem = sizeof(BuildShared) + sizeof(uint32_t) * (128 / G) * build_stride(G) + (size_t)p.K * 257;
  cudaError_t e = cudaFuncSetAttribute(build_tables_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tables * G, 1, 1);
  cfg.blockDim = dim3(kBuildThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = G > 1 ? 1 : 0;
  if constexpr (G > 1) {  // a device that cannot place such a cluster builds with one block per table
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, build_tables_kernel<G>, &cfg) != cudaSuccess || clusters < 1) {
      (void)cudaGetLastError();
      return launch_build_g<1>(d_hist, n_tables, p, d_tables, use_table, s);
    }
  }
  return cudaLaunchKernelEx(&cfg, build_tables_kernel<G>, reinterpret_cast<const unsigned long long*>(d_hist), p,
                            d_tables, use_table);
}

cudaError_t launch_build_tables(const uint64_t* d_hist, uint32_t n_tables, const shn_params& p, shn_table* d_tables,
                                cudaStream_t s) {
  if (n_tables == 0) return cudaSuccess;
  const uint32_t use_table = n_tables >= kLgTableMinTables ? 1u : 0u;
  if (use_table) {
    lg_table_kernel<<<128, 256, 0, s>>>();
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // the largest cluster that still gives each block an SM of its own; large batches of tables are
  // throughput-bound and keep one block per table (the fewest instructions per table)
  const uint64_t sms = (uint64_t)sm_count_for_launch();
  if ((uint64_t)n_tables * 8 <= sms) return launch_build_g<8>(d_hist, n_tables, p, d_tables, use_table, s);
  if ((uint64_t)n_tables * 4 <= sms) return launch_build_g<4>(d_hist, n_tables, p, d_tables, use_table, s);
  if ((uint64_t)n_tables * 2 <= sms) return launch_build_g<2>(d_hist, n_tables, p, d_tables, use_table, s);
  return launch_build_g<1>(d_hist, n_tables, p, d_tables, use_table, s);
}

}  // namespace shn
