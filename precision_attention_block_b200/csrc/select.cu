// Block selection (ThriftAttention technical summary, "Heuristische Blokkenselectie"):
// block means of Q and K, the score S^_ij = qbar_i . kbar_j of every valid (query block, key
// block) pair, the k highest pairs per (batch, query head), and their per-row lists.
//
//   means   FP16 sums in float64 are exact (|partial sums| < 2^23 on a 2^-24 grid), divided by
//           the block size (a power of two, exact).
//   scores  float64 products and sums in the order c = 0 .. d-1 with no fused multiply-add, so
//           every score is the correctly rounded result of one fixed evaluation order.
//   top-k   per (batch, query head) a most-significant-digit-first radix select over
//           order-preserving 64-bit keys finds the k-th largest score; keys above it are taken,
//           ties at it are taken in index order (smaller i * nKb + j first) through a block scan.
//           Long rows run on a cluster of CTAs that split the row into contiguous index ranges,
//           stream their keys from L2 for every digit and add up their digit histograms in a
//           per-head histogram in global memory behind a cluster barrier; short rows (at most
//           4096 keys) run on one CTA with the keys in shared memory.
//   lists   one warp per row of mask words; lanes own runs of words, a warp scan places them.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <mutex>

#include "sm100.cuh"
#include "thrift_internal.h"

namespace thrift {

// Fixed device scratch for thrift_block_select_noalloc.  Every GPU that loads the library holds
// these kNoAllocSelectScratchBytes until the process exits; all calls of that entry point share
// it, so calls that overlap on the GPU race on it.
constexpr size_t kNoAllocSelectScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_select_scratch[kNoAllocSelectScratchBytes];

namespace {

// Block sums: one CTA of 256 threads per (batch*head, block).  Sixteen lanes cover a token row
// of d <= 128 halves with 16-byte loads (8 columns each) and the 16 row groups of the CTA stride
// over the block's tokens; the partial sums meet in shared memory.  Every partial and total sum of
// FP16 values here is exact in float64 (the block's |sum| stays below 2^23 on the 2^-24 grid of
// FP16), so the order of the additions does not change the result.
constexpr int kMeanThreads = 256;
__global__ void __launch_bounds__(kMeanThreads) block_mean_kernel(const __half* __restrict__ x, RowMap rows, int N,
                                                                  int d, int bs, double* __restrict__ mean) {
  __shared__ double part[kMeanThreads / 16][128];
  const int64_t bh = blockIdx.y;
  const int blk = blockIdx.x;
  const __half* base = x + rows.off((int)bh, blk * bs);
  const int lane16 = threadIdx.x & 15, grp = threadIdx.x >> 4;
  const int c0 = lane16 * 8;  // first of this thread's 8 columns
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  if (c0 < d) {
    for (int t = grp; t < bs; t += kMeanThreads / 16) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)t * rows.sn + c0));
      const __half2* h = reinterpret_cast<const __half2*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        acc[2 * e] += (double)f.x;
        acc[2 * e + 1] += (double)f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[grp][c0 + e] = acc[e];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += kMeanThreads) {
    double s = 0.0;
#pragma unroll
    for (int g = 0; g < kMeanThreads / 16; ++g) s += part[g][c];
    mean[(bh * (N / bs) + blk) * d + c] = s / (double)bs;
  }
}

// Scores of a 64 x 64 tile of (query block, key block) pairs of one (batch, query head): thread
// (ty, tx) of 16 x 16 owns the 4 x 4 pairs (i0 + ty + 16a, j0 + tx + 16b), so each column step
// reads 8 means from shared memory for 16 products.  Every score is the float64 sum in the order
// c = 0 .. d-1 of the separately rounded products (no fused multiply-add); the columns are staged
// 32 at a time and the sums carried across the chunks in registers, which keeps that order.
// Tiles that lie entirely past the causal diagonal only write -inf.
constexpr int kTileQ = 64, kTileK = 64, kScoreChunk = 32;
__global__ void __launch_bounds__(256) block_score_kernel(const double* __restrict__ qbar,
                                                          const double* __restrict__ kbar, int Hq, int Hkv,
                                                          int nqb, int nkb, int d, int bq, int bk, int causal,
                                                          double* __restrict__ scores) {
  __shared__ double qs[kTileQ][kScoreChunk + 1];
  __shared__ double ks[kTileK][kScoreChunk + 1];
  const int bh = blockIdx.z;
  const int b = bh / Hq, h = bh % Hq, hk = h / (Hq / Hkv);
  const int i0 = blockIdx.y * kTileQ, j0 = blockIdx.x * kTileK;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const double ninf = -__longlong_as_double(0x7ff0000000000000LL);
  double* out = scores + ((int64_t)bh * nqb) * nkb;
  const int i_last = min(nqb, i0 + kTileQ) - 1;
  if (causal && (int64_t)j0 * bk > (int64_t)(i_last + 1) * bq - 1) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        const int i = i0 + ty + 16 * a, j = j0 + tx + 16 * bb;
        if (i < nqb && j < nkb) out[(int64_t)i * nkb + j] = ninf;
      }
    return;
  }
  const double* qb = qbar + ((int64_t)bh * nqb) * d;
  const double* kb = kbar + ((int64_t)(b * Hkv + hk) * nkb) * d;
  double acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) acc[a][bb] = 0.0;
  for (int cc = 0; cc < d; cc += kScoreChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kTileQ * kScoreChunk; e += 256) {
      const int r = e / kScoreChunk, c = e % kScoreChunk;
      qs[r][c] = (i0 + r < nqb) ? __ldg(qb + (int64_t)(i0 + r) * d + cc + c) : 0.0;
      ks[r][c] = (j0 + r < nkb) ? __ldg(kb + (int64_t)(j0 + r) * d + cc + c) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kScoreChunk; ++c) {
      double qv[4], kv[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) qv[a] = qs[ty + 16 * a][c];
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) kv[bb] = ks[tx + 16 * bb][c];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) acc[a][bb] = __dadd_rn(acc[a][bb], __dmul_rn(qv[a], kv[bb]));
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) {
      const int i = i0 + ty + 16 * a, j = j0 + tx + 16 * bb;
      if (i >= nqb || j >= nkb) continue;
      const bool valid = !causal || (int64_t)j * bk <= (int64_t)(i + 1) * bq - 1;
      out[(int64_t)i * nkb + j] = valid ? acc[a][bb] : ninf;
    }
}

// Order-preserving key of a score: larger score -> larger key; invalid (-inf) -> 0.
__device__ __forceinline__ uint64_t score_key(double s) {
  if (s == -__longlong_as_double(0x7ff0000000000000LL)) return 0ull;
  uint64_t u = (uint64_t)__double_as_longlong(s);
  return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

constexpr int kSelThreads = 1024;
constexpr int kSelSmemKeys = 4096;

template <int THREADS>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int& total) {
  int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (THREADS / 32) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive prefix of warp totals
  }
  __syncthreads();
  int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  total = warp_sums[THREADS / 32 - 1];
  __syncthreads();
  return before;
}

// Adds a per-thread count into a shared 64-bit counter: a warp sum first, then one atomic per warp
// (1024 same-address 64-bit shared atomics per block are slow).
__device__ __forceinline__ void warp_add_u64(unsigned long long* ctr, unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0 && v) atomicAdd(ctr, v);
}

struct TopkShared {
  unsigned int hist[256];
  int warp_sums[32];
  unsigned long long prefix;
  long long need;
  unsigned long long nvalid;
};

// Top-k of one row of n order-preserving keys (key_at(t); 0 = invalid pair) by a block of THREADS
// threads: a most-significant-digit-first radix select finds the k-th largest key, every key above
// it is taken and the first `need` ties in index order.  Chosen index t sets bit (t % nkb) of word
// (t / nkb) * mask_words + (t % nkb) / 32 of mk, which the caller has zeroed.
template <int THREADS, typename KeyAt>
__device__ void topk_row(KeyAt key_at, int64_t n, int nkb, int topk_abs, int topk_bp, int mask_words,
                         uint32_t* __restrict__ mk, TopkShared& sh) {
  // count valid pairs
  if (threadIdx.x == 0) sh.nvalid = 0;
  __syncthreads();
  unsigned long long cnt = 0;
  for (int64_t t = threadIdx.x; t < n; t += THREADS) cnt += key_at(t) != 0ull;
  warp_add_u64(&sh.nvalid, cnt);
  __syncthreads();
  long long nvalid = (long long)sh.nvalid;
  long long k = topk_abs >= 0 ? (long long)topk_abs : ((long long)topk_bp * nvalid + 9999) / 10000;
  if (k > nvalid) k = nvalid;
  if (k <= 0) return;

  // radix select: prefix of the k-th largest key, 8 bits at a time from the top
  unsigned long long prefix = 0ull;
  long long need = k;  // rank (1-based) of the wanted key among keys matching the prefix
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += THREADS) sh.hist[b] = 0;
    __syncthreads();
    unsigned long long hi_mask = shift == 56 ? 0ull : (~0ull << (shift + 8));
    // Neighbouring keys of a row are often close (the scores of one query block share most of
    // their leading bytes), so a warp's keys tend to fall in the same bins: one shared-memory
    // atomic per distinct bin of a warp instead of one per key (same-address atomics of a warp
    // serialise).
    for (int64_t base = 0; base < n; base += THREADS) {
      const int64_t t = base + threadIdx.x;
      const uint64_t key = t < n ? key_at(t) : 0ull;
      const bool in = key != 0ull && (key & hi_mask) == prefix;
      const int bin = in ? (int)((key >> shift) & 255) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (in && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], (unsigned)__popc(peers));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // bins from the top: lane l holds bins 255 - 8l .. 248 - 8l; find the bin where the
      // count of keys at or above it first reaches `need`
      const int lane = threadIdx.x;
      long long mine = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) mine += sh.hist[255 - 8 * lane - i];
      long long incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
      const int L = __ffs(hit) - 1;  // need <= total count, so some lane hits
      if (lane == L) {
        long long acc = incl - mine;
        int b = 255 - 8 * lane;
        for (int i = 0; i < 7; ++i, --b) {
          if (acc + (long long)sh.hist[b] >= need) break;
          acc += sh.hist[b];
        }
        sh.prefix = prefix | ((unsigned long long)b << shift);
        sh.need = need - acc;
      }
    }
    __syncthreads();
    prefix = sh.prefix;
    need = sh.need;
    __syncthreads();
  }
  // prefix is now the k-th largest key; take every key above it and the first `need` ties.
  long long taken_ties = 0;
  for (int64_t base = 0; base < n; base += THREADS) {
    int64_t t = base + threadIdx.x;
    uint64_t key = t < n ? key_at(t) : 0ull;
    int tie = (key != 0ull && key == prefix) ? 1 : 0;
    int total;
    int before = block_excl_scan<THREADS>(tie, sh.warp_sums, total);
    bool take = (key > prefix) || (tie && (taken_ties + before) < need);
    if (take) {
      int i = (int)(t / nkb), j = (int)(t % nkb);
      atomicOr(&mk[(int64_t)i * mask_words + (j >> 5)], 1u << (j & 31));
    }
    taken_ties += total;
  }
}

// One CTA per (batch, query head).  THREADS = kSelThreads for long rows; short rows run with fewer
// threads, which makes the block-wide barriers of each pass cheaper.
template <int THREADS>
__global__ void __launch_bounds__(THREADS) topk_kernel(const double* __restrict__ scores, int64_t n,
                                                           int nkb, int topk_abs, int topk_bp, int mask_words,
                                                           uint32_t* __restrict__ mask) {
  __shared__ TopkShared sh;
  __shared__ unsigned long long keys_sm[kSelSmemKeys];
  const double* sc = scores + (int64_t)blockIdx.x * n;
  int nqb = (int)(n / nkb);
  uint32_t* mk = mask + (int64_t)blockIdx.x * nqb * mask_words;
  // rows of up to kSelSmemKeys scores are read from global memory once and kept in shared memory
  const bool in_smem = n <= kSelSmemKeys;
  if (in_smem)
    for (int64_t t = threadIdx.x; t < n; t += THREADS) keys_sm[t] = score_key(sc[t]);
  auto key_at = [&](int64_t t) -> uint64_t { return in_smem ? keys_sm[t] : score_key(sc[t]); };
  topk_row<THREADS>(key_at, n, nkb, topk_abs, topk_bp, mask_words, mk, sh);
}

// Top-k of long rows on a cluster of kTopkCluster CTAs per (batch, query head).  CTA r owns the
// contiguous index range [r * chunk, (r + 1) * chunk) of the row and reads its scores from global
// memory (L2) for every digit, four coalesced loads in flight per thread; with little shared memory
// several clusters share an SM, so all heads run at once.  The radix select takes digits of 12, 12,
// 12, 12, 12 and 4 bits from the top of the key.  For each digit a CTA counts its keys into a
// shared-memory histogram, one atomic per distinct bin of a warp (neighbouring keys, one query
// block's scores, mostly share their leading digits, and same-address atomics serialise), adds the
// non-zero bins into the head's histogram of that digit in global memory (zeroed before the
// launch), and after a cluster barrier every CTA reads the head's totals and takes the same
// decision.  Keys above the k-th key are taken; its ties are taken in index order, CTA r taking the
// first (need - ties held by the CTAs before it) of its own.
constexpr int kTopkCluster = 8;
constexpr int kTopkClusterThreads = 512;
constexpr int kTopkBins = 4096;
constexpr int kTopkDigits = 6;

struct TopkClusterShared {
  unsigned int hist[kTopkBins];
  long long scan_part[32];
  int warp_sums[32];
  unsigned long long nvalid, nties;
  unsigned long long prefix;
  long long need;
  long long bcast;
};

// Inclusive prefix sum of v over the block (thread order), 64-bit.
template <int THREADS>
__device__ __forceinline__ long long block_incl_scan_ll(long long v, long long* part) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) part[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < THREADS / 32 ? part[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    part[lane] = w;
  }
  __syncthreads();
  const long long r = x + (warp > 0 ? part[warp - 1] : 0);
  __syncthreads();
  return r;
}

__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkClusterThreads, 3)
    topk_cluster_kernel(const double* __restrict__ scores, int64_t n, int nkb, int topk_abs, int topk_bp,
                        int mask_words, uint32_t* __restrict__ mask, unsigned int* __restrict__ ghist) {
  namespace cg = cooperative_groups;
  constexpr int THREADS = kTopkClusterThreads;
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int head = blockIdx.x / kTopkCluster;
  __shared__ TopkClusterShared sh;
  const double* sc = scores + (int64_t)head * n;
  const int64_t chunk = (n + kTopkCluster - 1) / kTopkCluster;
  const int64_t t0 = min(n, (int64_t)rank * chunk);
  const int64_t m = min(n, t0 + chunk) - t0;
  const int nqb = (int)(n / nkb);
  uint32_t* mk = mask + (int64_t)head * nqb * mask_words;
  unsigned int* gh = ghist + (int64_t)head * kTopkDigits * kTopkBins;
  const int lane = threadIdx.x & 31;
  auto key_at = [&](int64_t t) -> uint64_t { return score_key(__ldg(sc + t0 + t)); };
  // sum of one 64-bit counter over the CTAs of ranks [0, upto): warp 0 reads one rank per lane
  auto cluster_sum = [&](unsigned long long* local, int upto) -> long long {
    if (threadIdx.x < 32) {
      long long v = threadIdx.x < upto ? (long long)*cl.map_shared_rank(local, (int)threadIdx.x) : 0;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (threadIdx.x == 0) sh.bcast = v;
    }
    __syncthreads();
    const long long r = sh.bcast;
    __syncthreads();
    return r;
  };

  if (threadIdx.x == 0) {
    sh.nvalid = 0;
    sh.nties = 0;
  }
  __syncthreads();
  unsigned long long prefix = 0ull;
  long long need = 0;
#pragma unroll 1
  for (int p = 0; p < kTopkDigits; ++p) {
    const int shift = p < 5 ? 52 - 12 * p : 0, width = p < 5 ? 12 : 4;
    const unsigned int dmask = (1u << width) - 1u;
    unsigned int* hist = sh.hist;
    for (int b = threadIdx.x; b < kTopkBins; b += THREADS) hist[b] = 0;
    __syncthreads();
    const unsigned long long hi_mask = p == 0 ? 0ull : (~0ull << (shift + width));
    unsigned long long valid = 0;
    for (int64_t base = 0; base < m; base += 4 * THREADS) {
      uint64_t kb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t t = base + e * THREADS + threadIdx.x;
        kb[e] = t < m ? key_at(t) : 0ull;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint64_t key = kb[e];
        valid += key != 0ull;
        const bool in = key != 0ull && (key & hi_mask) == prefix;
        const int bin = in ? (int)((key >> shift) & dmask) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (unsigned)__popc(peers));
      }
    }
    if (p == 0) warp_add_u64(&sh.nvalid, valid);
    __syncthreads();
    unsigned int* gp = gh + p * kTopkBins;
    for (int b = threadIdx.x; b < kTopkBins; b += THREADS)
      if (hist[b]) atomicAdd(&gp[b], hist[b]);
    __threadfence();
    cl.sync();
    if (p == 0) {
      const long long nvalid = cluster_sum(&sh.nvalid, kTopkCluster);
      long long k = topk_abs >= 0 ? (long long)topk_abs : ((long long)topk_bp * nvalid + 9999) / 10000;
      if (k > nvalid) k = nvalid;
      if (k <= 0) {
        cl.sync();  // no CTA leaves while another may still read its count
        return;
      }
      need = k;
    }
    // the head's totals into the shared histogram, then thread t holds bins nb-1-8t .. nb-8-8t
    // (descending); the thread whose inclusive count first reaches `need` finds the bin of the
    // k-th key among its eight
    constexpr int BPT = kTopkBins / THREADS;
    const int nb = 1 << width;
    for (int b = threadIdx.x; b < nb; b += THREADS) hist[b] = __ldcg(gp + b);
    __syncthreads();
    unsigned int tot[BPT];
    const int b0 = nb - 1 - BPT * (int)threadIdx.x;
    long long mine = 0;
#pragma unroll
    for (int i = 0; i < BPT; ++i) {
      tot[i] = b0 - i >= 0 ? hist[b0 - i] : 0u;
      mine += tot[i];
    }
    const long long incl = block_incl_scan_ll<THREADS>(mine, sh.scan_part);
    if (incl >= need && incl - mine < need) {
      long long acc = incl - mine;
      int i = 0;
      for (; i < BPT - 1; ++i) {
        if (acc + (long long)tot[i] >= need) break;
        acc += tot[i];
      }
      sh.prefix = prefix | ((unsigned long long)(b0 - i) << shift);
      sh.need = need - acc;
    }
    __syncthreads();
    prefix = sh.prefix;
    need = sh.need;
  }
  // every key of the CTA's range, four coalesced loads in flight per thread
  auto for_keys = [&](auto&& f) {
    for (int64_t base = 0; base < m; base += 4 * THREADS) {
      uint64_t kb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t t = base + e * THREADS + threadIdx.x;
        kb[e] = t < m ? key_at(t) : 0ull;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t t = base + e * THREADS + threadIdx.x;
        if (t < m) f(t, kb[e]);
      }
    }
  };
  // prefix is the k-th largest key; need = how many of its ties to take, in index order
  unsigned long long ties = 0;
  for_keys([&](int64_t, uint64_t key) { ties += key == prefix; });
  warp_add_u64(&sh.nties, ties);
  cl.sync();
  const long long before_me = cluster_sum(&sh.nties, rank);
  const long long my_ties = (long long)sh.nties;
  const long long need_here = need - before_me;
  auto take_at = [&](int64_t t) {
    const int64_t g = t0 + t;
    const int i = (int)(g / nkb), j = (int)(g % nkb);
    if (THRIFT_CHECK(g < n && (j >> 5) < mask_words, nullptr))
      atomicOr(&mk[(int64_t)i * mask_words + (j >> 5)], 1u << (j & 31));
  };
  if (need_here <= 0 || need_here >= my_ties) {
    // none or all of this CTA's ties
    const bool all_ties = need_here > 0;
    for_keys([&](int64_t t, uint64_t key) {
      if (key > prefix || (all_ties && key == prefix)) take_at(t);
    });
  } else {
    long long taken_ties = 0;
    for (int64_t base = 0; base < m; base += THREADS) {
      const int64_t t = base + threadIdx.x;
      const uint64_t key = t < m ? key_at(t) : 0ull;
      const int tie = (key != 0ull && key == prefix) ? 1 : 0;
      int total;
      const int before = block_excl_scan<THREADS>(tie, sh.warp_sums, total);
      if ((key > prefix) || (tie && (taken_ties + before) < need_here)) take_at(t);
      taken_ties += total;
    }
  }
  cl.sync();  // no CTA leaves while another may still read its counts
}

// Whether the cluster top-k can run on the current device: clusters of kTopkCluster CTAs with
// `smem` bytes of dynamic shared memory each must fit (checked once per device and context).
bool topk_cluster_ok(size_t smem) {
  static std::mutex mu;
  static unsigned long long ctx_seen[64] = {0};
  static int ok_at[64] = {0};
  static size_t smem_at[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (ctx != 0 && ctx_seen[dev] == ctx && smem_at[dev] == smem) return ok_at[dev] != 0;
  int ok = 0;
  if (cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kTopkCluster);
    cfg.blockDim = dim3(kTopkClusterThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = kTopkCluster;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, topk_cluster_kernel, &cfg) == cudaSuccess && nclusters > 0) ok = 1;
  }
  (void)cudaGetLastError();  // a refused query leaves no error behind for the next launch check
  ctx_seen[dev] = ctx;
  ok_at[dev] = ok;
  smem_at[dev] = smem;
  return ok != 0;
}

constexpr int kListRowsPerCta = 8;

// Sorted list of the set bits of each mask row: one warp per row, lane l owns a contiguous run of
// the row's mask words; a warp scan of the per-lane counts gives each lane its output offset.
__global__ void __launch_bounds__(32 * kListRowsPerCta) lists_kernel(const uint32_t* __restrict__ mask, int64_t rows,
                                                                      int nkb, int mask_words,
                                                                      int32_t* __restrict__ counts,
                                                                      int16_t* __restrict__ lists) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * kListRowsPerCta + (threadIdx.x >> 5);
  if (r >= rows) return;
  const uint32_t* mw = mask + r * mask_words;
  int16_t* out = lists + r * nkb;
  const int wpl = (mask_words + 31) / 32;
  const int w0 = min(mask_words, lane * wpl), w1 = min(mask_words, w0 + wpl);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(mw[w]);
  int x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  const int total = __shfl_sync(0xffffffffu, x, 31);
  int c = x - cnt;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = mw[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      out[c++] = (int16_t)(w * 32 + b);
    }
  }
  for (int t = total + lane; t < nkb; t += 32) out[t] = -1;
  if (lane == 0) counts[r] = total;
}

// Decode scores S^[b, h, j] = qbar[b, h] . kbar[b, h / G, j]: a CTA forms the means of the Nq
// query rows of the G heads of one KV head (exact FP16 sums in float64, divided by Nq) and stages
// kDecScoreBlocks key-block means in shared memory; thread (hl, jj) scores block jj for query head
// hk*G + hl, the sum in the order c = 0 .. d-1 with no fused multiply-add (the evaluation the
// prefill scores use).  Blocks from nkb_valid on (past the cache's valid length) score -inf, which
// leaves them out of the top-k and its budget.
constexpr int kDecScoreBlocks = 16;
__global__ void decode_score_kernel(const __half* __restrict__ q, int Nq, const double* __restrict__ kbar, int Hq,
                                    int Hkv, int nkb, int nkb_valid, int d, double* __restrict__ scores) {
  __shared__ double ks[kDecScoreBlocks * 129];
  __shared__ double qs[16 * 128];
  const int G = Hq / Hkv, grp = blockIdx.y;
  const int b = grp / Hkv, hk = grp % Hkv;
  const int j0 = blockIdx.x * kDecScoreBlocks;
  const int nb = min(kDecScoreBlocks, nkb - j0);
  const double* kb = kbar + ((int64_t)grp * nkb + j0) * d;
  for (int e = threadIdx.x; e < nb * d; e += blockDim.x) ks[(e / d) * (d + 1) + e % d] = kb[e];
  const __half* qb = q + ((int64_t)b * Hq + (int64_t)hk * G) * Nq * d;
  for (int e = threadIdx.x; e < G * d; e += blockDim.x) {
    const int hl = e / d, c = e % d;
    double sum = 0.0;
    for (int t = 0; t < Nq; ++t) sum = __dadd_rn(sum, (double)__half2float(qb[((int64_t)hl * Nq + t) * d + c]));
    qs[e] = sum / (double)Nq;
  }
  __syncthreads();
  const int jj = threadIdx.x % kDecScoreBlocks, hl = threadIdx.x / kDecScoreBlocks;
  if (jj >= nb || hl >= G) return;
  const double* qr = qs + hl * d;
  const double* kr = ks + jj * (d + 1);
  double acc = 0.0;
#pragma unroll 8
  for (int c = 0; c < d; ++c) acc = __dadd_rn(acc, __dmul_rn(qr[c], kr[c]));
  if (j0 + jj >= nkb_valid) acc = -__builtin_huge_val();
  scores[((int64_t)b * Hq + (int64_t)hk * G + hl) * nkb + j0 + jj] = acc;
}

}  // namespace

SelectLayout select_layout(const thrift_cfg& c) {
  SelectLayout L;
  int64_t nqb = c.N / c.block_q, nkb = c.N / c.block_k;
  L.qbar_off = 0;
  L.kbar_off = align256(L.qbar_off + (size_t)c.B * c.Hq * nqb * c.d * sizeof(double));
  L.scores_off = align256(L.kbar_off + (size_t)c.B * c.Hkv * nkb * c.d * sizeof(double));
  L.topk_hist_off = align256(L.scores_off + (size_t)c.B * c.Hq * nqb * nkb * sizeof(double));
  // per (batch, query head): one histogram per radix digit of the cluster top-k
  L.bytes = align256(L.topk_hist_off + (size_t)c.B * c.Hq * kTopkDigits * kTopkBins * sizeof(unsigned int));
  return L;
}

size_t noalloc_select_scratch_bytes() { return kNoAllocSelectScratchBytes; }

// Device address of g_select_scratch on the current device.  In host code the array's name is
// only a host-side stand-in, so the address comes from cudaGetSymbolAddress, looked up with that
// device current and cached per device and context: after cudaDeviceReset the module is loaded
// into a new context, possibly at another address, and the lookup runs again.
thrift_status noalloc_select_scratch(uint8_t** out) {
  static std::mutex mu;
  static void* cache[64] = {nullptr};
  static unsigned long long cache_ctx[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return THRIFT_ERR_CUDA;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev] || ctx == 0 || cache_ctx[dev] != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_select_scratch) != cudaSuccess || !ptr) return THRIFT_ERR_CUDA;
    cache[dev] = ptr;
    cache_ctx[dev] = current_context_id();  // the lookup made the primary context current if none was
  }
  *out = static_cast<uint8_t*>(cache[dev]);
  return THRIFT_OK;
}

thrift_status select_launch(const void* q, const RowMap& qrows, const void* k, const RowMap& krows,
                            const thrift_cfg& c, uint32_t* mask, int32_t* counts, int16_t* lists, double* scores_out,
                            uint8_t* scratch, cudaStream_t stream) {
  SelectLayout L = select_layout(c);
  int nqb = c.N / c.block_q, nkb = c.N / c.block_k;
  int mask_words = (nkb + 31) / 32;
  double* qbar = reinterpret_cast<double*>(scratch + L.qbar_off);
  double* kbar = reinterpret_cast<double*>(scratch + L.kbar_off);
  double* scores = scores_out ? scores_out : reinterpret_cast<double*>(scratch + L.scores_off);
  block_mean_kernel<<<dim3(nqb, c.B * c.Hq), kMeanThreads, 0, stream>>>(reinterpret_cast<const __half*>(q), qrows,
                                                                         c.N, c.d, c.block_q, qbar);
  block_mean_kernel<<<dim3(nkb, c.B * c.Hkv), kMeanThreads, 0, stream>>>(reinterpret_cast<const __half*>(k), krows,
                                                                          c.N, c.d, c.block_k, kbar);
  dim3 g((nkb + kTileK - 1) / kTileK, (nqb + kTileQ - 1) / kTileQ, c.B * c.Hq);
  block_score_kernel<<<g, 256, 0, stream>>>(qbar, kbar, c.Hq, c.Hkv, nqb, nkb, c.d, c.block_q, c.block_k, c.causal,
                                            scores);
  size_t mask_bytes = (size_t)c.B * c.Hq * nqb * mask_words * sizeof(uint32_t);
  if (cudaMemsetAsync(mask, 0, mask_bytes, stream) != cudaSuccess) return THRIFT_ERR_CUDA;
  const int64_t n = (int64_t)nqb * nkb;
  if (n > kSelSmemKeys && topk_cluster_ok(0)) {
    unsigned int* ghist = reinterpret_cast<unsigned int*>(scratch + L.topk_hist_off);
    if (cudaMemsetAsync(ghist, 0, L.bytes - L.topk_hist_off, stream) != cudaSuccess) return THRIFT_ERR_CUDA;
    topk_cluster_kernel<<<(unsigned)(c.B * c.Hq * kTopkCluster), kTopkClusterThreads, 0, stream>>>(
        scores, n, nkb, c.topk_abs, c.topk_bp, mask_words, mask, ghist);
  } else {
    topk_kernel<kSelThreads><<<c.B * c.Hq, kSelThreads, 0, stream>>>(scores, n, nkb, c.topk_abs, c.topk_bp,
                                                                      mask_words, mask);
  }
  int64_t rows = (int64_t)c.B * c.Hq * nqb;
  lists_kernel<<<(unsigned)((rows + kListRowsPerCta - 1) / kListRowsPerCta), 32 * kListRowsPerCta, 0, stream>>>(
      mask, rows, nkb, mask_words, counts, lists);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status kv_means_launch(const void* k, int64_t outer, int32_t Nk, int32_t d, int32_t block_k, double* kbar,
                              cudaStream_t stream) {
  block_mean_kernel<<<dim3(Nk / block_k, (unsigned)outer), kMeanThreads, 0, stream>>>(
      reinterpret_cast<const __half*>(k), dense_rows(1, Nk, d), Nk, d, block_k, kbar);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

size_t decode_select_scratch_bytes(const thrift_decode_cfg& c) {
  size_t heads = (size_t)c.B * c.Hq, nkb = (size_t)(c.Nk / c.block_k);
  return align256(heads * c.d * sizeof(double)) + align256(heads * nkb * sizeof(double));
}

// The decode selection is the prefill selection with one query block of Nq rows per head.
// Every key block below the valid length holds a key visible to the newest row, so those pairs
// are valid; the blocks past it are not.
thrift_status decode_select_launch(const void* q, const double* kbar, const thrift_decode_cfg& c, uint32_t* mask,
                                   int32_t* counts, int16_t* lists, double* scores_out, uint8_t* scratch,
                                   cudaStream_t stream) {
  const int nkb = c.Nk / c.block_k;
  const int nkb_valid = (decode_valid(c) + c.block_k - 1) / c.block_k;
  const int mask_words = (nkb + 31) / 32;
  const size_t heads = (size_t)c.B * c.Hq;
  double* scores = scores_out ? scores_out
                              : reinterpret_cast<double*>(scratch + align256(heads * c.d * sizeof(double)));
  dim3 g((nkb + kDecScoreBlocks - 1) / kDecScoreBlocks, (unsigned)(c.B * c.Hkv));
  decode_score_kernel<<<g, kDecScoreBlocks * (c.Hq / c.Hkv), 0, stream>>>(
      reinterpret_cast<const __half*>(q), c.Nq, kbar, c.Hq, c.Hkv, nkb, nkb_valid, c.d, scores);
  if (cudaMemsetAsync(mask, 0, heads * mask_words * sizeof(uint32_t), stream) != cudaSuccess) return THRIFT_ERR_CUDA;
  if (nkb <= kSelSmemKeys)
    topk_kernel<256><<<(unsigned)heads, 256, 0, stream>>>(scores, (int64_t)nkb, nkb, c.topk_abs, c.topk_bp,
                                                          mask_words, mask);
  else
    topk_kernel<kSelThreads><<<(unsigned)heads, kSelThreads, 0, stream>>>(scores, (int64_t)nkb, nkb, c.topk_abs,
                                                                          c.topk_bp, mask_words, mask);
  if (counts && lists)
    lists_kernel<<<(unsigned)((heads + kListRowsPerCta - 1) / kListRowsPerCta), 32 * kListRowsPerCta, 0, stream>>>(
        mask, (int64_t)heads, nkb, mask_words, counts, lists);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

}  // namespace thrift
