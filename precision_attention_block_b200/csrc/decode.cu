// Decode form of the selective mixed-precision attention forward (ThriftAttention technical
// summary, "Methodologie" for the method; "Resultaten" for the decode use: a few new query rows
// against a long KV cache held twice, in FP16 and in NVFP4).
//
// A decode step has Nq query rows per query head (the newest cache positions) and reads the
// whole cache once, so it is bound by HBM bandwidth, not by tensor throughput: for each key the
// NVFP4 cache holds d/2 + d/16 bytes of K and the same of V, against 2d + 2d bytes in FP16.
// The rows of the Hq/Hkv query heads that share one KV head (at most 16 rows) form the M side
// of warp-level m16n8k16 tensor-core products, so the cache tile is read once per KV head.
// tcgen05 tiles start at 64 rows; with at most 16 rows they would be mostly idle while the
// cache streams in, which is the bound here.
//
// Kernels of one step:
//   quantise   the query rows as their own NVFP4 tensor (the quantiser of quantize.cu);
//   select     qbar = mean of the Nq rows of each head; S^_j = qbar . kbar_j with kbar the
//              cache's block means (computed once per cache by thrift_kv_block_means); top-k
//              key blocks per (batch, query head) -- select.cu, one query block per head;
//   attend     split over key blocks: CTA (split, batch * KV head) walks its key blocks.  A
//              producer warp streams each block's NVFP4 K and V (and, when one of the group's
//              heads selected the block, its FP16 K and V) into shared memory with bulk and
//              tensor copies; seven consumer warps, each claiming the next unclaimed block,
//              compute S = Q K^T (S fragments in registers), the per-row block maximum M,
//              P^ = exp(S - M), the two-level NVFP4 re-quantisation of P^ (FP16 rounding on
//              selected blocks), P V, and merge with weight exp(M - m) into FP32 partial sums;
//              the warps' partials are combined in shared memory at the end of the split;
//   combine    the splits' partial (O, m, l) of each row into O / l (FP16) and lse.
// The sparse variant (mode 3) runs only the selected blocks, in FP16.
//
// NVFP4 operands enter the tensor cores as FP16: an E2M1 value times its E4M3 scale has at most
// 6 significant bits and lies in [2^-10, 2688], so the FP16 value is exact, the products are
// exact and only the FP32 accumulation rounds -- the sums the method defines.  The contraction
// axis of each product is permuted (lane quad c of a warp owns a contiguous quarter of it), the
// same permutation on both operands, so that every lane reads its operand bytes with one vector
// load.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>

#include "sm100.cuh"
#include "thrift_internal.h"

namespace thrift {

namespace {

constexpr int kRowsMax = 16;           // query rows of one KV-head group (the MMA's M)
constexpr int kConsumers = 224;        // seven consumer warps (with the producer, 256 threads: up to 255 registers)
constexpr int kConsumerWarps = kConsumers / 32;
constexpr int kTab = 2048;             // key blocks of a split whose selection bits are staged
constexpr int kThreads = kConsumers + 32;
constexpr long long kWaitLimit = 1ll << 32;
constexpr int kMinBlocksPerSplit = 4;
constexpr int kMaxSplit = 320;
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct DecodeParams {
  const __half* q;        // [B*Hq*Nq, D]
  const __half* k16;      // [B*Hkv*Nk, D]
  const __half* v16;
  const uint8_t* q4c;     // [B*Hq*Nq, D/2]
  const uint8_t* q4s;     // [B*Hq*Nq, D/16]
  const float* q_ts;
  const uint8_t* k4c;     // [B*Hkv*Nk, D/2]
  const uint8_t* k4s;     // [B*Hkv*Nk, D/16]
  const float* k_ts;
  const uint8_t* v4sm;    // V scales in the MMA layout
  const float* v_ts;
  const uint32_t* mask;   // [B*Hq, mask_words] (mode 0)
  float* part_o;          // [groups, n_split, 16, D]
  float* part_ml;         // [groups, n_split, 16, 2]
  int* status;
  int B, Hq, Hkv, G, Nq, Nk, R, nkb, mask_words, n_split, bps, causal, mode;
  int n_valid;  // keys the cache holds (keys from n_valid on are masked; nkb covers the blocks below)
  float tau;
  long long wait_limit;
};

template <int D, int BK>
struct DLayout {
  static constexpr int K4C = BK * D / 2;
  static constexpr int K4S = BK * D / 16;
  static constexpr int V4C = D * BK / 2;
  static constexpr int V4S = 512 * (BK / 64);
  static constexpr int OFF_K4S = K4C;
  static constexpr int OFF_V4C = K4C + K4S;
  static constexpr int OFF_V4S = OFF_V4C + V4C;
  static constexpr int ST4 = OFF_V4S + V4S;            // one NVFP4 stage: K codes, K scales, V codes, V scales
  static constexpr int ST16 = 2 * BK * D * 2;          // one FP16 slot: K then V
  static constexpr int NST = BK == 64 ? 12 : 6;
  static constexpr int NF = BK == 64 ? 2 : 1;
  static constexpr int OFF_ST16 = NST * ST4;
  static constexpr int OFF_QA = OFF_ST16 + NF * ST16;           // query A fragments: NVFP4, then FP16
  static constexpr int QA_BYTES = 2 * (D / 16) * 32 * 16;
  static constexpr int OFF_PA = OFF_QA + QA_BYTES;              // per-warp P A fragments
  static constexpr int PA_BYTES = kConsumerWarps * (BK / 16) * 32 * 16;
  static constexpr int OFF_TAB = OFF_PA + PA_BYTES;             // FP16-head bits of the split's blocks
  static constexpr int OFF_BAR = OFF_TAB + kTab * 2;
  static constexpr int BAR_BYTES = 8 * (2 * NST + 2 * NF) + 4 * (NST + NF) + 16;  // + abort flag, next block
  static constexpr int SMEM = OFF_BAR + BAR_BYTES;
  // after the main loop the consumer warps' partial results reuse the stage area
  static constexpr int COMB_ML = kConsumerWarps * kRowsMax * D * 4;  // after [warps][16][D] f32 outputs
  static_assert(COMB_ML + kConsumerWarps * kRowsMax * 2 * 4 <= OFF_QA, "combine area");
  static_assert(ST4 % 128 == 0 && ST16 % 128 == 0 && OFF_QA % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
  static_assert(SMEM <= 232448, "shared memory");
};

// ------------------------------------------------------------------ device helpers

// Two E2M1 codes (bits 0-3 and 4-7 of `byte`) to an FP16 pair (low half from bits 0-3); exact.
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t byte) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(out) : "r"(byte));
  return out;
}

// One E4M3 code (bits 0-7) to an FP16 pair holding the value twice; exact.
__device__ __forceinline__ uint32_t e4m3_to_h2x(uint32_t code) {
  uint32_t out;
  const uint16_t two = (uint16_t)((code & 0xFFu) | ((code & 0xFFu) << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(two));
  return out;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t out;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out) : "r"(a), "r"(b));
  return out;
}

// D += A B for one m16n8k16 tile (FP16 operands, FP32 accumulators).
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void named_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

// Named barrier over the consumer warps that also ORs a predicate across them.
__device__ __forceinline__ bool named_sync_or(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "n"(kConsumers)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// FP16-pair bitmask bits of the group's G heads for key block j (bit hl = head hk*G + hl).
__device__ __forceinline__ uint32_t group_bits(const DecodeParams& p, int b, int hk, int j) {
  if (p.mode == 1) return 0u;
  if (p.mode == 2) return (1u << p.G) - 1u;
  uint32_t bits = 0;
  const uint32_t* base = p.mask + ((int64_t)b * p.Hq + (int64_t)hk * p.G) * p.mask_words + (j >> 5);
  for (int hl = 0; hl < p.G; ++hl) bits |= ((__ldg(base + (int64_t)hl * p.mask_words) >> (j & 31)) & 1u) << hl;
  return bits;
}

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2f(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Bounded wait until a shared word holds `want` (see tag4 in decode_attn_kernel).
__device__ __forceinline__ bool wait_tag(volatile int* tag, int want, volatile int* abort_flag, int* status,
                                         long long limit) {
  if (*tag == want) return true;
  const long long t0 = clock64();
  while (*tag != want) {
    if (*abort_flag) return false;
    if (clock64() - t0 > limit) {
      *abort_flag = 1;
      if (status) atomicOr(status, kStatusTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// Key of column n of S n-tile nt.  Lane quad tig of a warp then holds the keys
// [tig*BK/4, (tig+1)*BK/4) of its rows, and the S fragments of n-tiles 2ks and 2ks+1 are the A
// fragment of k-step ks of P V with contraction slot 2*tig+e = key tig*BK/4 + 4*ks + e and slot
// 8+2*tig+e = that key + 2: the order in which the lane reads V's token-grouped codes.
template <int BK>
__device__ __forceinline__ int key_of(int nt, int n) {
  return (n >> 1) * (BK / 4) + 4 * (nt >> 1) + 2 * (nt & 1) + (n & 1);
}

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, 1) decode_attn_kernel(const __grid_constant__ CUtensorMap tm_v4c,
                                                                  const DecodeParams p) {
  using L = DLayout<D, BK>;
  constexpr int NST = L::NST, NF = L::NF;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full4 = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty4 = full4 + NST;
  uint64_t* full16 = empty4 + NST;
  uint64_t* empty16 = full16 + NF;
  // tag4[s] / tag16[s]: the block (FP16-slot use) a stage (slot) is being filled for, written by
  // the producer once the stage's previous use is released.  Consumers take blocks round-robin,
  // so the warp that waits for a use of a stage may come before the warp of the stage's previous
  // use has seen that one complete; a parity wait cannot tell those two phases apart, so a
  // consumer first waits until the tag names its own use.
  volatile int* tag4 = reinterpret_cast<volatile int*>(empty16 + NF);
  volatile int* tag16 = tag4 + NST;
  volatile int* abort_flag = tag16 + NF;
  int* next_block = const_cast<int*>(abort_flag) + 1;  // the next block a consumer warp takes
  uint16_t* tab = reinterpret_cast<uint16_t*>(smem + L::OFF_TAB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = blockIdx.y, split = blockIdx.x;
  const int b = grp / p.Hkv, hk = grp % p.Hkv;
  const int j0 = split * p.bps;
  const int nblk = min(p.bps, p.nkb - j0);
  const uint32_t all_heads = (1u << p.G) - 1u;
  const bool use4 = p.mode <= 1;  // modes 2 and 3 read no NVFP4 operand

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full4[s], 1);
      mbar_init(&empty4[s], 1);
      tag4[s] = -1;
    }
    for (int s = 0; s < NF; ++s) {
      mbar_init(&full16[s], 1);
      mbar_init(&empty16[s], 1);
      tag16[s] = -1;
    }
    *abort_flag = 0;
    *next_block = 0;
    fence_mbar_init();
  }
  {
    // The query rows as m16n8k16 A fragments, [k-step][lane] (rows >= R zero): dequantised NVFP4
    // rows, then FP16 rows.  Contraction slot 2*tig+e of k-step ks holds d = tig*D/4 + 4*ks + e,
    // slot 8+2*tig+e holds d + 2.  Also the selection bits of the split's first kTab blocks.
    const int64_t qrow0 = ((int64_t)b * p.Hq + (int64_t)hk * p.G) * p.Nq;
    uint4* qa = reinterpret_cast<uint4*>(smem + L::OFF_QA);
    for (int f = threadIdx.x; f < 2 * (D / 16) * 32; f += blockDim.x) {
      const bool fp16 = f >= (D / 16) * 32;
      const int ks = (f % ((D / 16) * 32)) / 32, ln = f % 32;
      const int gg = ln >> 2, tg = ln & 3;
      const int d0 = tg * (D / 4) + 4 * ks;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int rs = 0; rs < 2; ++rs) {
        const int r = gg + 8 * rs;
        if (r >= p.R) continue;
        if (fp16) {
          const __half* qr = p.q + (qrow0 + r) * D + d0;
          w[rs] = *reinterpret_cast<const uint32_t*>(qr);
          w[2 + rs] = *reinterpret_cast<const uint32_t*>(qr + 2);
        } else if (use4) {
          const uint8_t* qc = p.q4c + (qrow0 + r) * (D / 2);
          const uint32_t sc = e4m3_to_h2x(__ldg(p.q4s + (qrow0 + r) * (D / 16) + d0 / 16));
          w[rs] = hmul2(e2m1x2_to_h2(__ldg(qc + d0 / 2)), sc);
          w[2 + rs] = hmul2(e2m1x2_to_h2(__ldg(qc + d0 / 2 + 1)), sc);
        }
      }
      qa[f] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int i = threadIdx.x; i < min(nblk, kTab); i += blockDim.x) tab[i] = (uint16_t)group_bits(p, b, hk, j0 + i);
  }
  __syncthreads();
  auto bits_of = [&](int i) -> uint32_t { return i < kTab ? (uint32_t)tab[i] : group_bits(p, b, hk, j0 + i); };

  if (warp == kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tm_v4c);
      const int64_t krow0 = (int64_t)grp * p.Nk;
      const int vrow0 = grp * D;  // first V code row of this KV head
      const int64_t vsf_block = (int64_t)(vrow0 >> 7) * (p.Nk / 64);
      int c16 = 0;
      bool ok = true;
      for (int i = 0; i < nblk && ok; ++i) {
        const int j = j0 + i;
        const uint32_t bits = bits_of(i);
        const int64_t kr = krow0 + (int64_t)j * BK;
        // the key block lies inside the cache
        if (!THRIFT_CHECK((int64_t)(j + 1) * BK <= p.Nk, p.status)) {
          *abort_flag = 1;
          break;
        }
        if (use4) {
          const int s = i % NST;
          ok = mbar_wait(&empty4[s], ((i / NST) & 1) ^ 1, abort_flag, p.status, p.wait_limit);
          if (!ok) break;
          uint8_t* st = smem + s * L::ST4;
          tag4[s] = i;
          mbar_arrive_expect_tx(&full4[s], L::ST4);
          bulk_load(st, p.k4c + kr * (D / 2), L::K4C, &full4[s]);
          bulk_load(st + L::OFF_K4S, p.k4s + kr * (D / 16), L::K4S, &full4[s]);
          tma_load_2d(st + L::OFF_V4C, &tm_v4c, &full4[s], j * (BK / 2), vrow0);
          bulk_load(st + L::OFF_V4S, p.v4sm + (vsf_block + (int64_t)j * (BK / 64)) * 512, L::V4S, &full4[s]);
        }
        if (bits != 0u) {
          const int s = c16 % NF;
          ok = mbar_wait(&empty16[s], ((c16 / NF) & 1) ^ 1, abort_flag, p.status, p.wait_limit);
          if (!ok) break;
          uint8_t* st = smem + L::OFF_ST16 + s * L::ST16;
          tag16[s] = c16;
          mbar_arrive_expect_tx(&full16[s], L::ST16);
          bulk_load(st, p.k16 + kr * D, BK * D * 2, &full16[s]);
          bulk_load(st + BK * D * 2, p.v16 + kr * D, BK * D * 2, &full16[s]);
          ++c16;
        }
      }
      // every copy issued must land before the CTA exits: wait (bounded) for the last fill of
      // each stage and slot; on the normal path the consumers have already waited for them
      if (use4)
        for (int i = max(0, nblk - NST); i < nblk; ++i)
          mbar_wait(&full4[i % NST], (i / NST) & 1, abort_flag, nullptr, p.wait_limit);
      for (int c = max(0, c16 - NF); c < c16; ++c)
        mbar_wait(&full16[c % NF], (c / NF) & 1, abort_flag, nullptr, p.wait_limit);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  // Each consumer warp takes the split's next unclaimed block (in block order) until none is left,
  // and keeps its own output, maximum and denominator for rows g and g + 8, combined with the
  // other warps' at the end.
  const int g = lane >> 2, tig = lane & 3;
  const int R = p.R;
  const float sv4 = use4 ? __ldg(p.v_ts) * (1.0f / 2688.0f) : 0.0f;
  const float sl4 = use4 ? p.tau * __ldg(p.q_ts) * __ldg(p.k_ts) * kLog2e : 0.0f;  // FP4 score -> log2 units
  const float sl16 = p.tau * kLog2e;
  const int64_t qpos0 = (int64_t)p.n_valid - p.Nq;  // position of query row 0 among the keys
  const uint4* qa4 = reinterpret_cast<const uint4*>(smem + L::OFF_QA);             // [D/16][32] A fragments
  const uint4* qa16 = qa4 + (D / 16) * 32;
  uint4* pa_w = reinterpret_cast<uint4*>(smem + L::OFF_PA) + warp * (BK / 16) * 32;  // this warp's P fragments
  const int vrow_in_blk = (grp * D) & 127;  // this head's first row inside its 128-row scale block
  // query row r is the (r % Nq)-th row of head hk*G + r/Nq
  const int hrow[2] = {g / p.Nq, (g + 8) / p.Nq};
  const int64_t qpos[2] = {qpos0 + g % p.Nq, qpos0 + (g + 8) % p.Nq};

  float o[D / 8][4];
#pragma unroll
  for (int t = 0; t < D / 8; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[t][e] = 0.0f;
  float m_ref[2] = {kNegInf, kNegInf}, l_run[2] = {0.0f, 0.0f};  // m in log2 units

  int scan_i = 0, c16_acc = 0;
  bool ok = true;
  for (;;) {
    int i = 0;
    if (lane == 0) i = atomicAdd(next_block, 1);
    i = __shfl_sync(0xffffffffu, i, 0);
    if (i >= nblk) break;
    while (scan_i < i) c16_acc += bits_of(scan_i++) != 0u ? 1 : 0;
    const int j = j0 + i;
    const uint32_t bits = bits_of(i);
    const bool n16 = bits != 0u, n4 = use4 && bits != all_heads;
    if (!n4 && !n16 && !use4) continue;  // sparse variant: no head of the group selected this block
    const int s4 = i % NST, s16 = c16_acc % NF;
    if (use4) {
      ok = wait_tag(&tag4[s4], i, abort_flag, p.status, p.wait_limit);
      ok = ok && mbar_wait(&full4[s4], (i / NST) & 1, abort_flag, p.status, p.wait_limit);
    }
    if (ok && n16) {
      ok = wait_tag(&tag16[s16], c16_acc, abort_flag, p.status, p.wait_limit);
      ok = ok && mbar_wait(&full16[s16], (c16_acc / NF) & 1, abort_flag, p.status, p.wait_limit);
    }
    if (!ok) break;
    const uint8_t* st4 = smem + s4 * L::ST4;
    const uint8_t* st16 = smem + L::OFF_ST16 + s16 * L::ST16;
    const bool f16r[2] = {((bits >> hrow[0]) & 1u) != 0u, ((bits >> hrow[1]) & 1u) != 0u};

    // ---- S = Q K^T (log2 units); n-tile nt holds keys key_of(nt, .).  NVFP4 pass, then FP16 pass
    // for the rows whose head selected the block.
    float sc[BK / 8][4];
    {
      float c[BK / 8][4];
      if (n4) {
#pragma unroll
        for (int nt = 0; nt < BK / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) c[nt][e] = 0.0f;
#pragma unroll
        for (int q = 0; q < D / 64; ++q) {  // the lane's 16-element scale group q
          uint32_t sk[BK / 8];
#pragma unroll
          for (int nt = 0; nt < BK / 8; ++nt)
            sk[nt] = e4m3_to_h2x(st4[L::OFF_K4S + key_of<BK>(nt, g) * (D / 16) + tig * (D / 64) + q]);
#pragma unroll 1
          for (int k4 = 0; k4 < 4; ++k4) {
            const int ks = 4 * q + k4;
            const uint4 a4 = qa4[ks * 32 + lane];
            const uint32_t a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int nt = 0; nt < BK / 8; ++nt) {
              const uint32_t two =
                  *reinterpret_cast<const uint16_t*>(st4 + key_of<BK>(nt, g) * (D / 2) + tig * (D / 8) + 2 * ks);
              mma16816(c[nt], a, hmul2(e2m1x2_to_h2(two & 0xFFu), sk[nt]), hmul2(e2m1x2_to_h2(two >> 8), sk[nt]));
            }
          }
        }
#pragma unroll
        for (int nt = 0; nt < BK / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = c[nt][e] * sl4;
      }
      if (n16) {
#pragma unroll
        for (int nt = 0; nt < BK / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) c[nt][e] = 0.0f;
#pragma unroll 1
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint4 a4 = qa16[ks * 32 + lane];
          const uint32_t a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int nt = 0; nt < BK / 8; ++nt) {
            const uint2 bw = *reinterpret_cast<const uint2*>(reinterpret_cast<const __half*>(st16) +
                                                             key_of<BK>(nt, g) * D + tig * (D / 4) + 4 * ks);
            mma16816(c[nt], a, bw.x, bw.y);
          }
        }
#pragma unroll
        for (int nt = 0; nt < BK / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (f16r[e >> 1] || !n4) sc[nt][e] = c[nt][e] * sl16;
      }
#pragma unroll
      for (int nt = 0; nt < BK / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rs = e >> 1;
          const int kk = tig * (BK / 4) + 4 * (nt >> 1) + 2 * (nt & 1) + (e & 1);
          const int64_t key = (int64_t)j * BK + kk;
          if (g + 8 * rs >= R || (p.causal && key > qpos[rs]) || key >= p.n_valid || (p.mode == 3 && !f16r[rs]))
            sc[nt][e] = kNegInf;
        }
    }

    // ---- per row: block maximum, probabilities (re-quantised for NVFP4 rows), merge weights
    uint32_t pa[BK / 8][2];  // P V A fragments: pa[nt][rs] = keys of S n-tile nt, row g + 8 rs
    float al[2], w4[2], w16[2];
#pragma unroll
    for (int rs = 0; rs < 2; ++rs) {
      float mx = kNegInf;
#pragma unroll
      for (int nt = 0; nt < BK / 8; ++nt) mx = fmaxf(mx, fmaxf(sc[nt][2 * rs], sc[nt][2 * rs + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      const float M = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      float sum = 0.0f;
      if (M == kNegInf) {  // row >= R, or no key of this block visible to it
#pragma unroll
        for (int nt = 0; nt < BK / 8; ++nt) pa[nt][rs] = 0u;
      } else if (!f16r[rs]) {
        // P' = 2688 exp(S - M); s_b = E4M3(max16 P' / 6) per 16 keys (the lane's keys hold whole
        // groups); code = E2M1(P' / s_b) evaluated as exp2(S - M + log2(2688 / s_b))
#pragma unroll
        for (int q = 0; q < BK / 64; ++q) {
          float gm = kNegInf;
#pragma unroll
          for (int nt = 8 * q; nt < 8 * q + 8; ++nt) gm = fmaxf(gm, fmaxf(sc[nt][2 * rs], sc[nt][2 * rs + 1]));
          const float pm = gm != kNegInf ? 448.0f * ex2f(gm - M) : 0.0f;
          const uint32_t sb = cvt_e4m3(pm);
          const float sbv = e4m3_to_f32(sb);
          const float sbe = sbv > 0.0f ? sbv : 448.0f;
          const float bias = (11.392317422778761f - lg2f(sbe)) - M;  // log2(2688 / s_b) - M
          const uint32_t sb2 = e4m3_to_h2x(sb);
          float gs = 0.0f;
#pragma unroll
          for (int nt = 8 * q; nt < 8 * q + 8; ++nt) {
            const float y0 = ex2f(sc[nt][2 * rs] + bias), y1 = ex2f(sc[nt][2 * rs + 1] + bias);
            gs += y0 + y1;
            pa[nt][rs] = hmul2(e2m1x2_to_h2(cvt_e2m1x2(y0, y1)), sb2);  // code * s_b, exact in FP16
          }
          sum = fmaf(gs, sbe * (1.0f / 2688.0f), sum);
        }
      } else {
#pragma unroll
        for (int nt = 0; nt < BK / 8; ++nt) {
          const float p0 = ex2f(sc[nt][2 * rs] - M), p1 = ex2f(sc[nt][2 * rs + 1] - M);
          sum += p0 + p1;
          pa[nt][rs] = pack_h2(p0, p1);
        }
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if (M == kNegInf) {
        al[rs] = 1.0f;
        w4[rs] = w16[rs] = 0.0f;
      } else {
        const float m_new = fmaxf(m_ref[rs], M);
        al[rs] = m_ref[rs] == kNegInf ? 0.0f : ex2f(m_ref[rs] - m_new);
        const float gw = ex2f(M - m_new);
        l_run[rs] = l_run[rs] * al[rs] + gw * sum;
        m_ref[rs] = m_new;
        w4[rs] = f16r[rs] ? 0.0f : gw * sv4;
        w16[rs] = f16r[rs] ? gw : 0.0f;
      }
    }
    // the A fragment of k-step ks is S n-tiles 2ks and 2ks + 1 (rows g, g + 8)
#pragma unroll
    for (int ks = 0; ks < BK / 16; ++ks)
      pa_w[ks * 32 + lane] = make_uint4(pa[2 * ks][0], pa[2 * ks][1], pa[2 * ks + 1][0], pa[2 * ks + 1][1]);
    __syncwarp();
    if (__any_sync(0xffffffffu, al[0] != 1.0f || al[1] != 1.0f)) {
#pragma unroll
      for (int t = 0; t < D / 8; ++t) {
        o[t][0] *= al[0];
        o[t][1] *= al[0];
        o[t][2] *= al[1];
        o[t][3] *= al[1];
      }
    }

    // ---- P V into the running output; n-tile t holds output columns 8t .. 8t + 7.  NVFP4 pass
    // (rows of NVFP4 heads carry weight w4), then FP16 pass (weight w16).
    {
      float c[D / 8][4];
      if (n4) {
#pragma unroll
        for (int t = 0; t < D / 8; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) c[t][e] = 0.0f;
#pragma unroll
        for (int q = 0; q < BK / 64; ++q) {  // the lane's 16-key scale group q
          uint32_t vsc[D / 8];
#pragma unroll
          for (int t = 0; t < D / 8; ++t) {
            const int crow = vrow_in_blk + t * 8 + g;
            const int gg = tig * (BK / 64) + q;  // 16-key group within the block
            vsc[t] = e4m3_to_h2x(st4[L::OFF_V4S + (gg >> 2) * 512 + (crow & 31) * 16 + ((crow >> 5) & 3) * 4 + (gg & 3)]);
          }
#pragma unroll 1
          for (int k4 = 0; k4 < 4; ++k4) {
            const int ks = 4 * q + k4;
            const uint4 a4 = pa_w[ks * 32 + lane];
            const uint32_t a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int t = 0; t < D / 8; ++t) {
              const uint32_t two = *reinterpret_cast<const uint16_t*>(st4 + L::OFF_V4C + (t * 8 + g) * (BK / 2) +
                                                                      tig * (BK / 8) + 2 * ks);
              mma16816(c[t], a, hmul2(e2m1x2_to_h2(two & 0xFFu), vsc[t]), hmul2(e2m1x2_to_h2(two >> 8), vsc[t]));
            }
          }
        }
#pragma unroll
        for (int t = 0; t < D / 8; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[t][e] = fmaf(w4[e >> 1], c[t][e], o[t][e]);
      }
      if (n16) {
#pragma unroll
        for (int t = 0; t < D / 8; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) c[t][e] = 0.0f;
        const __half* vr = reinterpret_cast<const __half*>(st16 + BK * D * 2);
#pragma unroll 1
        for (int ks = 0; ks < BK / 16; ++ks) {
          const uint4 a4 = pa_w[ks * 32 + lane];
          const uint32_t a[4] = {a4.x, a4.y, a4.z, a4.w};
          const int k0 = tig * (BK / 4) + 4 * ks;
#pragma unroll
          for (int t = 0; t < D / 8; ++t) {
            const int n = t * 8 + g;
            const __half2 b0h = __halves2half2(vr[(k0 + 0) * D + n], vr[(k0 + 1) * D + n]);
            const __half2 b1h = __halves2half2(vr[(k0 + 2) * D + n], vr[(k0 + 3) * D + n]);
            mma16816(c[t], a, *reinterpret_cast<const uint32_t*>(&b0h), *reinterpret_cast<const uint32_t*>(&b1h));
          }
        }
#pragma unroll
        for (int t = 0; t < D / 8; ++t)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[t][e] = fmaf(w16[e >> 1], c[t][e], o[t][e]);
      }
    }
    __syncwarp();
    if (lane == 0) {
      if (use4) mbar_arrive(&empty4[s4]);
      if (n16) mbar_arrive(&empty16[s16]);
    }
  }

  // ---- combine the consumer warps' partial results of this split (through the stage area: every
  // copy has landed and been read once all consumer warps are past their loops)
  if (named_sync_or(!ok)) return;
  float* co = reinterpret_cast<float*>(smem);
  float* cml = reinterpret_cast<float*>(smem + L::COMB_ML);
#pragma unroll
  for (int t = 0; t < D / 8; ++t) {
    const int col = t * 8 + 2 * tig;
#pragma unroll
    for (int rs = 0; rs < 2; ++rs) {
      const int r = g + 8 * rs;
      if (r < R)
        *reinterpret_cast<float2*>(co + (warp * kRowsMax + r) * D + col) = make_float2(o[t][2 * rs], o[t][2 * rs + 1]);
    }
  }
  if (tig == 0) {
#pragma unroll
    for (int rs = 0; rs < 2; ++rs) {
      const int r = g + 8 * rs;
      if (r < R) {
        cml[(warp * kRowsMax + r) * 2] = m_ref[rs];
        cml[(warp * kRowsMax + r) * 2 + 1] = l_run[rs];
      }
    }
  }
  named_sync();
  float* po = p.part_o + ((int64_t)grp * p.n_split + split) * kRowsMax * D;
  float* pml = p.part_ml + ((int64_t)grp * p.n_split + split) * kRowsMax * 2;
  for (int idx = threadIdx.x; idx < R * D; idx += kConsumers) {
    const int r = idx / D;
    float m = kNegInf;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) m = fmaxf(m, cml[(w * kRowsMax + r) * 2]);
    float acc = 0.0f, l = 0.0f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float mw = cml[(w * kRowsMax + r) * 2];
      const float f = (mw == kNegInf) ? 0.0f : ex2f(mw - m);
      acc = fmaf(f, co[(w * kRowsMax + r) * D + idx % D], acc);
      l = fmaf(f, cml[(w * kRowsMax + r) * 2 + 1], l);
    }
    po[idx] = acc;
    if (idx % D == 0) {
      pml[2 * r] = m;  // log2 units
      pml[2 * r + 1] = l;
    }
  }
}

// Combine the splits of every row: O = sum_s w_s O_s / sum_s w_s l_s with w_s = 2^(m_s - m)
// (the partial maxima are in log2 units of the tau-scaled scores).  One CTA per (batch * KV head,
// row); thread (part, c) sums output column c over the splits s = part (mod kCombineParts).
constexpr int kCombineParts = 4;
__global__ void __launch_bounds__(512) decode_combine_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_ml, int n_split, int D,
                                                             int Hq, int Hkv, int Nq, __half* __restrict__ out,
                                                             float* __restrict__ lse) {
  extern __shared__ float wsh[];  // [n_split] weights, then [kCombineParts][D] column sums
  __shared__ float red[16];
  const int grp = blockIdx.x, r = blockIdx.y;
  const int b = grp / Hkv, hk = grp % Hkv, G = Hq / Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float* ml = part_ml + (int64_t)grp * n_split * kRowsMax * 2 + 2 * r;
  float m = kNegInf;
  for (int s = threadIdx.x; s < n_split; s += blockDim.x) m = fmaxf(m, ml[(int64_t)s * kRowsMax * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  m = red[0];
  for (int i = 1; i < nw; ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  float l = 0.0f;
  for (int s = threadIdx.x; s < n_split; s += blockDim.x) {
    const float ms = ml[(int64_t)s * kRowsMax * 2];
    const float w = (ms == kNegInf) ? 0.0f : exp2f(ms - m);
    wsh[s] = w;
    l += w * ml[(int64_t)s * kRowsMax * 2 + 1];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  if (lane == 0) red[warp] = l;
  __syncthreads();
  l = 0.0f;
  for (int i = 0; i < nw; ++i) l += red[i];
  const int64_t orow = ((int64_t)b * Hq + (int64_t)hk * G + r / Nq) * Nq + r % Nq;
  const float inv = l > 0.0f ? 1.0f / l : 0.0f;
  const float* po = part_o + ((int64_t)grp * n_split * kRowsMax + r) * D;
  float* colsum = wsh + n_split;
  {
    const int c = threadIdx.x % D, part = threadIdx.x / D;
    float acc = 0.0f;
#pragma unroll 4
    for (int s = part; s < n_split; s += kCombineParts) acc = fmaf(wsh[s], po[(int64_t)s * kRowsMax * D + c], acc);
    colsum[part * D + c] = acc;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.0f;
#pragma unroll
    for (int part = 0; part < kCombineParts; ++part) acc += colsum[part * D + c];
    out[orow * D + c] = __float2half_rn(acc * inv);
  }
  if (threadIdx.x == 0 && lse) lse[orow] = l > 0.0f ? m * kLn2 + logf(l) : kNegInf;
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_u8_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_inner,
                 uint32_t box_rows) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BK>
thrift_status decode_launch_t(const DecodeArgs& a, DecodeParams& prm, cudaStream_t stream) {
  using L = DLayout<D, BK>;
  CUtensorMap tm;
  memset(&tm, 0, sizeof(tm));
  if (prm.mode <= 1) {
    if (!make_u8_map(&tm, a.v4->codes, (uint64_t)prm.Nk / 2, (uint64_t)prm.B * prm.Hkv * D, BK / 2, D))
      return THRIFT_ERR_CUDA;
  } else {
    // no NVFP4 operand is read; the map only has to be valid
    if (!make_u8_map(&tm, a.part_o, 64, 1, 16, 1)) return THRIFT_ERR_CUDA;
  }
  auto kern = decode_attn_kernel<D, BK>;
  // once per device (a host-side attribute; keeping it out of later calls keeps them capturable)
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return THRIFT_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) != cudaSuccess)
      return THRIFT_ERR_CUDA;
    attr_set[dev] = true;
  }
  dim3 grid(prm.n_split, prm.B * prm.Hkv);
  kern<<<grid, kThreads, L::SMEM, stream>>>(tm, prm);
  if (cudaPeekAtLastError() != cudaSuccess) return THRIFT_ERR_CUDA;
  decode_combine_kernel<<<dim3(prm.B * prm.Hkv, prm.R), D * kCombineParts,
                          (prm.n_split + kCombineParts * D) * sizeof(float), stream>>>(
      prm.part_o, prm.part_ml, prm.n_split, D, prm.Hq, prm.Hkv, prm.Nq, reinterpret_cast<__half*>(a.out), a.lse);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

int ctas_per_sm(int D, int BK) {
  int smem = 0;
  if (D == 128 && BK == 64) smem = DLayout<128, 64>::SMEM;
  if (D == 128 && BK == 128) smem = DLayout<128, 128>::SMEM;
  if (D == 64 && BK == 64) smem = DLayout<64, 64>::SMEM;
  if (D == 64 && BK == 128) smem = DLayout<64, 128>::SMEM;
  const int per_sm = 232448;  // shared memory of one SM, 1 KB of it reserved per CTA
  int n = per_sm / (smem + 1024);
  return n < 1 ? 1 : (n > 1 ? 1 : n);  // the kernel is built for one CTA per SM
}

}  // namespace

int decode_split_cap(int nkb) {
  int cap = (nkb + kMinBlocksPerSplit - 1) / kMinBlocksPerSplit;
  return cap < 1 ? 1 : (cap > kMaxSplit ? kMaxSplit : cap);
}

thrift_status decode_attn_launch(const DecodeArgs& a, cudaStream_t stream) {
  const thrift_decode_cfg& c = *a.cfg;
  DecodeParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.q = reinterpret_cast<const __half*>(a.q);
  prm.k16 = reinterpret_cast<const __half*>(a.k);
  prm.v16 = reinterpret_cast<const __half*>(a.v);
  if (a.mode <= 1) {
    prm.q4c = a.q4->codes;
    prm.q4s = a.q4->scales;
    prm.q_ts = a.q4->tensor_scale;
    prm.k4c = a.k4->codes;
    prm.k4s = a.k4->scales;
    prm.k_ts = a.k4->tensor_scale;
    prm.v4sm = a.v4->scales_mma;
    prm.v_ts = a.v4->tensor_scale;
  }
  prm.mask = a.mask;
  prm.part_o = a.part_o;
  prm.part_ml = a.part_ml;
  prm.status = a.status;
  prm.B = c.B;
  prm.Hq = c.Hq;
  prm.Hkv = c.Hkv;
  prm.G = c.Hq / c.Hkv;
  prm.Nq = c.Nq;
  prm.Nk = c.Nk;
  prm.R = prm.G * c.Nq;
  prm.n_valid = decode_valid(c);
  prm.nkb = (prm.n_valid + c.block_k - 1) / c.block_k;  // the blocks below the valid length
  prm.mask_words = (c.Nk / c.block_k + 31) / 32;           // the selection's layout (the capacity)
  prm.causal = c.causal;
  prm.mode = a.mode;
  prm.tau = c.softmax_scale > 0.0f ? c.softmax_scale : 1.0f / sqrtf((float)c.d);
  prm.wait_limit = kWaitLimit;
  // splits: as many CTAs as fit on the GPU at once, at least kMinBlocksPerSplit key blocks each
  const int groups = c.B * c.Hkv;
  const int resident = num_sms() * ctas_per_sm(c.d, c.block_k);
  int n_split = resident / groups;  // one wave: every CTA resident at once
  const int cap = decode_split_cap(prm.nkb);
  if (n_split > cap) n_split = cap;
  if (n_split < 1) n_split = 1;
  prm.bps = (prm.nkb + n_split - 1) / n_split;
  prm.n_split = (prm.nkb + prm.bps - 1) / prm.bps;
  if (c.d == 128 && c.block_k == 64) return decode_launch_t<128, 64>(a, prm, stream);
  if (c.d == 128 && c.block_k == 128) return decode_launch_t<128, 128>(a, prm, stream);
  if (c.d == 64 && c.block_k == 64) return decode_launch_t<64, 64>(a, prm, stream);
  if (c.d == 64 && c.block_k == 128) return decode_launch_t<64, 128>(a, prm, stream);
  return THRIFT_ERR_UNSUPPORTED;
}

}  // namespace thrift
