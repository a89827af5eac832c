// Block selection (ThriftAttention technical summary, "Heuristische Blokkenselectie"):
// block means of Q and K, the score S^_ij = qbar_i . kbar_j of every valid (query block, key
// block) pair, the k highest pairs per (batch, query head), and their per-row lists.
//
//   means   FP16 sums in float64 are exact (|partial sums| < 2^23 on a 2^-24 grid), divided by
//           the block size (a power of two, exact).
//   scores  float64 products and sums in the order c = 0 .. d-1 with no fused multiply-add, so
//           every score is the correctly rounded result of one fixed evaluation order.
//   top-k   one CTA per (batch, query head): a most-significant-digit-first radix select over
//           order-preserving 64-bit keys finds the k-th largest score; keys above it are taken,
//           ties at it are taken in index order (smaller i * nKb + j first) through a block scan.
//   lists   one thread per query block walks its mask words in ascending order.
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

// Block sums: one CTA per (batch*head, block); thread c sums column c over the block's tokens.
__global__ void block_mean_kernel(const __half* __restrict__ x, int N, int d, int bs, double* __restrict__ mean) {
  int64_t bh = blockIdx.y;
  int blk = blockIdx.x;
  const __half* base = x + (bh * N + (int64_t)blk * bs) * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    double s = 0.0;
    for (int t = 0; t < bs; ++t) s = __dadd_rn(s, (double)__half2float(base[(int64_t)t * d + c]));
    mean[(bh * (N / bs) + blk) * d + c] = s / (double)bs;
  }
}

constexpr int kTileQ = 16, kTileK = 16;

// Scores for a 16 x 16 tile of (query block, key block) pairs of one (batch, query head).
__global__ void __launch_bounds__(256) block_score_kernel(const double* __restrict__ qbar,
                                                          const double* __restrict__ kbar, int Hq, int Hkv,
                                                          int nqb, int nkb, int d, int bq, int bk, int causal,
                                                          double* __restrict__ scores) {
  extern __shared__ double sm[];
  double* qs = sm;                          // [kTileQ][d+1]
  double* ks = sm + kTileQ * (d + 1);       // [kTileK][d+1]
  int bh = blockIdx.z;
  int b = bh / Hq, h = bh % Hq, hk = h / (Hq / Hkv);
  int i0 = blockIdx.y * kTileQ, j0 = blockIdx.x * kTileK;
  const double* qb = qbar + ((int64_t)bh * nqb) * d;
  const double* kb = kbar + ((int64_t)(b * Hkv + hk) * nkb) * d;
  for (int e = threadIdx.x; e < kTileQ * d; e += blockDim.x) {
    int r = e / d, c = e % d;
    qs[r * (d + 1) + c] = (i0 + r < nqb) ? qb[(int64_t)(i0 + r) * d + c] : 0.0;
  }
  for (int e = threadIdx.x; e < kTileK * d; e += blockDim.x) {
    int r = e / d, c = e % d;
    ks[r * (d + 1) + c] = (j0 + r < nkb) ? kb[(int64_t)(j0 + r) * d + c] : 0.0;
  }
  __syncthreads();
  int ii = threadIdx.x / kTileK, jj = threadIdx.x % kTileK;
  int i = i0 + ii, j = j0 + jj;
  if (i >= nqb || j >= nkb) return;
  double out;
  if (causal && (int64_t)j * bk > (int64_t)(i + 1) * bq - 1) {
    out = -__longlong_as_double(0x7ff0000000000000LL);
  } else {
    double s = 0.0;
    const double* qr = qs + ii * (d + 1);
    const double* kr = ks + jj * (d + 1);
    for (int c = 0; c < d; ++c) s = __dadd_rn(s, __dmul_rn(qr[c], kr[c]));
    out = s;
  }
  scores[((int64_t)bh * nqb + i) * nkb + j] = out;
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
  atomicAdd(&sh.nvalid, cnt);
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
    if (shift >= 48) {
      // the leading bytes (sign, exponent, top of the mantissa) are shared by most scores of a
      // head, so most keys fall in the same few bins: one shared-memory atomic per distinct bin of
      // a warp instead of one per key
      for (int64_t base = 0; base < n; base += THREADS) {
        const int64_t t = base + threadIdx.x;
        const uint64_t key = t < n ? key_at(t) : 0ull;
        const bool in = key != 0ull && (key & hi_mask) == prefix;
        const int bin = in ? (int)((key >> shift) & 255) : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (in && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], (unsigned)__popc(peers));
      }
    } else {
      for (int64_t t = threadIdx.x; t < n; t += THREADS) {
        const uint64_t key = key_at(t);
        if (key != 0ull && (key & hi_mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & 255], 1u);
      }
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
  L.bytes = align256(L.scores_off + (size_t)c.B * c.Hq * nqb * nkb * sizeof(double));
  return L;
}

size_t noalloc_select_scratch_bytes() { return kNoAllocSelectScratchBytes; }

// Device address of g_select_scratch on the current device.  In host code the array's name is
// only a host-side stand-in, so the address comes from cudaGetSymbolAddress, looked up once per
// device (with that device current) and cached.
thrift_status noalloc_select_scratch(uint8_t** out) {
  static std::mutex mu;
  static void* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return THRIFT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_select_scratch) != cudaSuccess || !ptr) return THRIFT_ERR_CUDA;
    cache[dev] = ptr;
  }
  *out = static_cast<uint8_t*>(cache[dev]);
  return THRIFT_OK;
}

thrift_status select_launch(const void* q, const void* k, const thrift_cfg& c, uint32_t* mask, int32_t* counts,
                            int16_t* lists, double* scores_out, uint8_t* scratch, cudaStream_t stream) {
  SelectLayout L = select_layout(c);
  int nqb = c.N / c.block_q, nkb = c.N / c.block_k;
  int mask_words = (nkb + 31) / 32;
  double* qbar = reinterpret_cast<double*>(scratch + L.qbar_off);
  double* kbar = reinterpret_cast<double*>(scratch + L.kbar_off);
  double* scores = scores_out ? scores_out : reinterpret_cast<double*>(scratch + L.scores_off);
  int tpb = c.d >= 128 ? 128 : c.d;
  block_mean_kernel<<<dim3(nqb, c.B * c.Hq), tpb, 0, stream>>>(reinterpret_cast<const __half*>(q), c.N, c.d,
                                                               c.block_q, qbar);
  block_mean_kernel<<<dim3(nkb, c.B * c.Hkv), tpb, 0, stream>>>(reinterpret_cast<const __half*>(k), c.N, c.d,
                                                                c.block_k, kbar);
  size_t smem = (size_t)(kTileQ + kTileK) * (c.d + 1) * sizeof(double);
  dim3 g((nkb + kTileK - 1) / kTileK, (nqb + kTileQ - 1) / kTileQ, c.B * c.Hq);
  block_score_kernel<<<g, kTileQ * kTileK, smem, stream>>>(qbar, kbar, c.Hq, c.Hkv, nqb, nkb, c.d, c.block_q,
                                                           c.block_k, c.causal, scores);
  size_t mask_bytes = (size_t)c.B * c.Hq * nqb * mask_words * sizeof(uint32_t);
  if (cudaMemsetAsync(mask, 0, mask_bytes, stream) != cudaSuccess) return THRIFT_ERR_CUDA;
  topk_kernel<kSelThreads><<<c.B * c.Hq, kSelThreads, 0, stream>>>(scores, (int64_t)nqb * nkb, nkb, c.topk_abs,
                                                                    c.topk_bp, mask_words, mask);
  int64_t rows = (int64_t)c.B * c.Hq * nqb;
  lists_kernel<<<(unsigned)((rows + kListRowsPerCta - 1) / kListRowsPerCta), 32 * kListRowsPerCta, 0, stream>>>(
      mask, rows, nkb, mask_words, counts, lists);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

thrift_status kv_means_launch(const void* k, int64_t outer, int32_t Nk, int32_t d, int32_t block_k, double* kbar,
                              cudaStream_t stream) {
  int tpb = d >= 128 ? 128 : d;
  block_mean_kernel<<<dim3(Nk / block_k, (unsigned)outer), tpb, 0, stream>>>(reinterpret_cast<const __half*>(k), Nk,
                                                                             d, block_k, kbar);
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
