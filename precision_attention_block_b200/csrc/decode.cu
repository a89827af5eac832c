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
//              key blocks per (batch, query head) -- the kernels of select.cu with one query
//              block;
//   attend     split over key blocks: CTA (split, batch * KV head) walks its key blocks.  A
//              producer warp streams each block's NVFP4 K and V (and, when one of the group's
//              heads selected the block, its FP16 K and V) into shared memory with bulk and
//              tensor copies; eight consumer warps compute S = Q K^T, the per-row block maximum
//              M, P^ = exp(S - M), the two-level NVFP4 re-quantisation of P^ (FP16 rounding on
//              selected blocks), P V, and merge with weight exp(M - m) into FP32 partial sums;
//   combine    the splits' partial (O, m, l) of each row into O / l (FP16) and lse.
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
constexpr int kConsumers = 256;        // eight consumer warps
constexpr int kThreads = kConsumers + 32;
constexpr long long kWaitLimit = 1ll << 32;
constexpr int kMinBlocksPerSplit = 4;
constexpr int kMaxSplit = 320;
constexpr float kNegInf = -__builtin_huge_valf();

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
  static constexpr int ST4 = OFF_V4S + V4S;            // one NVFP4 stage
  static constexpr int ST16 = 2 * BK * D * 2;          // one FP16 slot: K then V
  static constexpr int NST = 4;
  static constexpr int NF = 1;
  static constexpr int OFF_ST16 = NST * ST4;
  static constexpr int OFF_S = OFF_ST16 + NF * ST16;   // S   [16][BK] f32
  static constexpr int OFF_PC = OFF_S + kRowsMax * BK * 4;       // P codes [16][BK/2]
  static constexpr int OFF_PS = OFF_PC + kRowsMax * BK / 2;      // P scales [16][BK/16]
  static constexpr int OFF_P16 = OFF_PS + ((kRowsMax * BK / 16 + 15) & ~15);  // P16 [16][BK]
  static constexpr int OFF_Q16 = OFF_P16 + kRowsMax * BK * 2;    // Q16 [16][D]
  static constexpr int OFF_ROW = OFF_Q16 + kRowsMax * D * 2;     // alpha, gq4, gq16 [16] each
  static constexpr int OFF_BAR = OFF_ROW + 3 * kRowsMax * 4;
  static constexpr int BAR_BYTES = 8 * (2 * NST + 2 * NF) + 16;
  static constexpr int SMEM = OFF_BAR + BAR_BYTES;
  static_assert(ST4 % 128 == 0 && ST16 % 128 == 0 && OFF_S % 16 == 0 && OFF_BAR % 8 == 0, "alignment");
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

template <int D, int BK>
__global__ void __launch_bounds__(kThreads, BK == 64 ? 2 : 1) decode_attn_kernel(const __grid_constant__ CUtensorMap tm_v4c,
                                                               const DecodeParams p) {
  using L = DLayout<D, BK>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full4 = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty4 = full4 + L::NST;
  uint64_t* full16 = empty4 + L::NST;
  uint64_t* empty16 = full16 + L::NF;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty16 + L::NF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = blockIdx.y, split = blockIdx.x;
  const int b = grp / p.Hkv, hk = grp % p.Hkv;
  const int j0 = split * p.bps;
  const int j1 = min(p.nkb, j0 + p.bps);
  const uint32_t all_heads = (1u << p.G) - 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::NST; ++s) {
      mbar_init(&full4[s], 1);
      mbar_init(&empty4[s], kConsumers / 32);
    }
    for (int s = 0; s < L::NF; ++s) {
      mbar_init(&full16[s], 1);
      mbar_init(&empty16[s], kConsumers / 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // zero the P buffers once (rows that never hold probabilities stay finite), the row
  // parameters of rows >= R, and stage the FP16 query rows
  for (int i = threadIdx.x; i < (L::OFF_ROW - L::OFF_PC) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t*>(smem + L::OFF_PC)[i] = 0u;
  __syncthreads();
  {
    const int64_t qrow0 = ((int64_t)b * p.Hq + (int64_t)hk * p.G) * p.Nq;
    __half* q16 = reinterpret_cast<__half*>(smem + L::OFF_Q16);
    for (int i = threadIdx.x; i < p.R * D; i += blockDim.x) q16[i] = p.q[qrow0 * D + i];
    float* rowp = reinterpret_cast<float*>(smem + L::OFF_ROW);
    if (threadIdx.x < kRowsMax) {
      rowp[threadIdx.x] = 1.0f;               // alpha
      rowp[kRowsMax + threadIdx.x] = 0.0f;    // gq4
      rowp[2 * kRowsMax + threadIdx.x] = 0.0f;  // gq16
    }
  }
  __syncthreads();

  if (warp == kConsumers / 32) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tm_v4c);
      const int64_t krow0 = (int64_t)grp * p.Nk;
      const int vrow0 = grp * D;  // first V code row of this KV head
      const int64_t vsf_block = (int64_t)(vrow0 >> 7) * (p.Nk / 64);
      int c4 = 0, c16 = 0;
      bool ok = true;
      for (int j = j0; j < j1 && ok; ++j) {
        const uint32_t bits = group_bits(p, b, hk, j);
        if (bits != all_heads) {
          const int s = c4 % L::NST;
          ok = mbar_wait(&empty4[s], ((c4 / L::NST) & 1) ^ 1, abort_flag, p.status, p.wait_limit);
          if (!ok) break;
          uint8_t* st = smem + s * L::ST4;
          mbar_arrive_expect_tx(&full4[s], L::ST4);
          const int64_t kr = krow0 + (int64_t)j * BK;
          bulk_load(st, p.k4c + kr * (D / 2), L::K4C, &full4[s]);
          bulk_load(st + L::OFF_K4S, p.k4s + kr * (D / 16), L::K4S, &full4[s]);
          tma_load_2d(st + L::OFF_V4C, &tm_v4c, &full4[s], j * (BK / 2), vrow0);
          bulk_load(st + L::OFF_V4S, p.v4sm + (vsf_block + (int64_t)j * (BK / 64)) * 512, L::V4S, &full4[s]);
          ++c4;
        }
        if (bits != 0u) {
          const int s = c16 % L::NF;
          ok = mbar_wait(&empty16[s], ((c16 / L::NF) & 1) ^ 1, abort_flag, p.status, p.wait_limit);
          if (!ok) break;
          uint8_t* st = smem + L::OFF_ST16 + s * L::ST16;
          mbar_arrive_expect_tx(&full16[s], L::ST16);
          const int64_t kr = krow0 + (int64_t)j * BK;
          bulk_load(st, p.k16 + kr * D, BK * D * 2, &full16[s]);
          bulk_load(st + BK * D * 2, p.v16 + kr * D, BK * D * 2, &full16[s]);
          ++c16;
        }
      }
      // every copy issued must land before the CTA exits: wait (bounded) for the last fill of
      // each stage; on the normal path the consumers have already waited for all of them
      for (int i = 0; i < L::NST && i < c4; ++i) {
        const int c = c4 - 1 - i;
        mbar_wait(&full4[c % L::NST], (c / L::NST) & 1, abort_flag, nullptr, p.wait_limit);
      }
      for (int i = 0; i < L::NF && i < c16; ++i) {
        const int c = c16 - 1 - i;
        mbar_wait(&full16[c % L::NF], (c / L::NF) & 1, abort_flag, nullptr, p.wait_limit);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, tig = lane & 3;
  const int R = p.R;
  const float sv4 = (p.mode == 2 ? 0.0f : __ldg(p.v_ts)) * (1.0f / 2688.0f);
  const float mult4 = p.mode == 2 ? 0.0f : p.tau * __ldg(p.q_ts) * __ldg(p.k_ts);
  const int64_t qrow0 = ((int64_t)b * p.Hq + (int64_t)hk * p.G) * p.Nq;

  // dequantised NVFP4 query rows as m16n8k16 A fragments (rows >= R are zero); contraction
  // slot 2*tig+e of k-step ks holds d = tig*D/4 + 4*ks + e, slot 8+2*tig+e holds d + 2
  uint32_t qa[D / 16][4];
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
    for (int i = 0; i < 4; ++i) qa[ks][i] = 0u;
  if (p.mode != 2) {
#pragma unroll
    for (int rs = 0; rs < 2; ++rs) {
      const int r = g + 8 * rs;
      if (r < R) {
        const uint8_t* qc = p.q4c + (qrow0 + r) * (D / 2);
        const uint8_t* qs = p.q4s + (qrow0 + r) * (D / 16);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int d0 = tig * (D / 4) + 4 * ks;
          const uint32_t sc = e4m3_to_h2x(__ldg(qs + d0 / 16));
          qa[ks][rs] = hmul2(e2m1x2_to_h2(__ldg(qc + d0 / 2)), sc);
          qa[ks][2 + rs] = hmul2(e2m1x2_to_h2(__ldg(qc + d0 / 2 + 1)), sc);
        }
      }
    }
  }

  constexpr int NT_QK = BK / 8 / 8;   // key n-tiles per warp
  constexpr int NT_PV = D / 8 / 8;    // output-column n-tiles per warp
  constexpr int KPL = BK / 32;        // keys per lane in the softmax
  float o[NT_PV][4];
#pragma unroll
  for (int t = 0; t < NT_PV; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[t][e] = 0.0f;
  // running maximum and denominator of rows warp and warp + 8 (replicated over the warp)
  float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.0f, 0.0f};

  float* S = reinterpret_cast<float*>(smem + L::OFF_S);
  uint8_t* PC = smem + L::OFF_PC;
  uint8_t* PS = smem + L::OFF_PS;
  __half* P16 = reinterpret_cast<__half*>(smem + L::OFF_P16);
  const __half* Q16 = reinterpret_cast<const __half*>(smem + L::OFF_Q16);
  float* alpha_s = reinterpret_cast<float*>(smem + L::OFF_ROW);
  float* gq4_s = alpha_s + kRowsMax;
  float* gq16_s = gq4_s + kRowsMax;
  const int vrow_in_blk = (grp * D) & 127;  // this head's first row inside its 128-row scale block
  const int64_t qpos0 = (int64_t)p.Nk - p.Nq;  // position of query row 0 among the keys

  int c4 = 0, c16 = 0;
  bool ok = true;
  for (int j = j0; j < j1; ++j) {
    const uint32_t bits = group_bits(p, b, hk, j);
    const bool n4 = bits != all_heads, n16 = bits != 0u;
    const int s4 = c4 % L::NST, s16 = c16 % L::NF;
    if (n4) ok = ok && mbar_wait(&full4[s4], (c4 / L::NST) & 1, abort_flag, p.status, p.wait_limit);
    if (n16) ok = ok && mbar_wait(&full16[s16], (c16 / L::NF) & 1, abort_flag, p.status, p.wait_limit);
    const uint8_t* st4 = smem + s4 * L::ST4;
    const uint8_t* st16 = smem + L::OFF_ST16 + s16 * L::ST16;

    // ---- S = Q K^T for the warp's key n-tiles
    if (ok) {
#pragma unroll
      for (int t = 0; t < NT_QK; ++t) {
        const int nt = warp + 8 * t;
        const int key = nt * 8 + g;
        float c4r[4] = {0.f, 0.f, 0.f, 0.f}, c16r[4] = {0.f, 0.f, 0.f, 0.f};
        if (n4) {
          const uint8_t* kc = st4 + key * (D / 2) + tig * (D / 8);
          uint32_t w[D / 32];
          if constexpr (D == 128) {
            const uint4 v = *reinterpret_cast<const uint4*>(kc);
            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
          } else {
            const uint2 v = *reinterpret_cast<const uint2*>(kc);
            w[0] = v.x; w[1] = v.y;
          }
          const uint8_t* ksc = st4 + L::OFF_K4S + key * (D / 16) + tig * (D / 64);
          uint32_t sc[D / 64];
#pragma unroll
          for (int i = 0; i < D / 64; ++i) sc[i] = e4m3_to_h2x(ksc[i]);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t word = w[ks >> 1];
            const int sh = (ks & 1) * 16;
            const uint32_t s2 = sc[ks >> 2];
            const uint32_t b0 = hmul2(e2m1x2_to_h2((word >> sh) & 0xFFu), s2);
            const uint32_t b1 = hmul2(e2m1x2_to_h2((word >> (sh + 8)) & 0xFFu), s2);
            mma16816(c4r, qa[ks], b0, b1);
          }
        }
        if (n16) {
          const __half* kr = reinterpret_cast<const __half*>(st16) + key * D + tig * (D / 4);
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint2 bw = *reinterpret_cast<const uint2*>(kr + 4 * ks);
            const int d0 = tig * (D / 4) + 4 * ks;
            uint32_t a[4];
            a[0] = *reinterpret_cast<const uint32_t*>(Q16 + g * D + d0);
            a[1] = *reinterpret_cast<const uint32_t*>(Q16 + (g + 8) * D + d0);
            a[2] = *reinterpret_cast<const uint32_t*>(Q16 + g * D + d0 + 2);
            a[3] = *reinterpret_cast<const uint32_t*>(Q16 + (g + 8) * D + d0 + 2);
            if (g >= R) a[0] = a[2] = 0u;
            if (g + 8 >= R) a[1] = a[3] = 0u;
            mma16816(c16r, a, bw.x, bw.y);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = g + 8 * (e >> 1);
          const int kk = nt * 8 + 2 * tig + (e & 1);
          float v = kNegInf;
          if (r < R) {
            const bool f16 = (bits >> (r / p.Nq)) & 1u;
            v = f16 ? c16r[e] * p.tau : c4r[e] * mult4;
            if (p.causal && (int64_t)j * BK + kk > qpos0 + (r % p.Nq)) v = kNegInf;
          }
          S[r * BK + kk] = v;
        }
      }
    }
    // every consumer warp passes each barrier; a failed wait anywhere stops all of them here
    if (named_sync_or(!ok)) {
      ok = false;
      break;
    }

    // ---- softmax, re-quantisation and merge weights for rows warp and warp + 8
#pragma unroll
    for (int rs = 0; rs < 2; ++rs) {
      const int r = warp + 8 * rs;
      if (r >= R) continue;
      float s[KPL];
#pragma unroll
      for (int t = 0; t < KPL; ++t) s[t] = S[r * BK + lane * KPL + t];
      float mx = s[0];
#pragma unroll
      for (int t = 1; t < KPL; ++t) mx = fmaxf(mx, s[t]);
      const float M = warp_max(mx);
      const bool f16 = (bits >> (r / p.Nq)) & 1u;
      if (M == kNegInf) {  // no key of this block is visible to the row
        if (lane == 0) {
          alpha_s[r] = 1.0f;
          gq4_s[r] = 0.0f;
          gq16_s[r] = 0.0f;
        }
        continue;
      }
      float ph[KPL];
      float sum = 0.0f;
#pragma unroll
      for (int t = 0; t < KPL; ++t) {
        ph[t] = s[t] == kNegInf ? 0.0f : expf(s[t] - M);
        sum += ph[t];
      }
      sum = warp_sum(sum);
      if (f16) {
#pragma unroll
        for (int t = 0; t < KPL; ++t) P16[r * BK + lane * KPL + t] = __float2half_rn(ph[t]);
      } else {
        // P' = 2688 P^; s_b = E4M3(amax16(P') / 6); code = E2M1(P' / s_b)
        float pp[KPL];
        float am = 0.0f;
#pragma unroll
        for (int t = 0; t < KPL; ++t) {
          pp[t] = __fmul_rn(2688.0f, ph[t]);
          am = fmaxf(am, pp[t]);
        }
#pragma unroll
        for (int o = 1; o < 16 / KPL; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        const uint32_t sb = cvt_e4m3(__fdiv_rn(am, 6.0f));
        const float sbv = e4m3_to_f32(sb);
        uint32_t byte0 = 0u, byte1 = 0u;
        if (sbv > 0.0f) {
          byte0 = cvt_e2m1x2(__fdiv_rn(pp[0], sbv), __fdiv_rn(pp[1], sbv));
          if constexpr (KPL == 4) byte1 = cvt_e2m1x2(__fdiv_rn(pp[2], sbv), __fdiv_rn(pp[3], sbv));
        }
        if constexpr (KPL == 2) {
          PC[r * (BK / 2) + lane] = (uint8_t)byte0;
        } else {
          *reinterpret_cast<uint16_t*>(PC + r * (BK / 2) + 2 * lane) = (uint16_t)(byte0 | (byte1 << 8));
        }
        if ((lane & (16 / KPL - 1)) == 0) PS[r * (BK / 16) + lane * KPL / 16] = (uint8_t)sb;
      }
      const float m_new = fmaxf(m_run[rs], M);
      const float alpha = m_run[rs] == kNegInf ? 0.0f : expf(m_run[rs] - m_new);
      const float gw = expf(M - m_new);
      l_run[rs] = l_run[rs] * alpha + gw * sum;
      m_run[rs] = m_new;
      if (lane == 0) {
        alpha_s[r] = alpha;
        gq4_s[r] = f16 ? 0.0f : gw * sv4;
        gq16_s[r] = f16 ? gw : 0.0f;
      }
    }
    named_sync();

    // ---- P V for the warp's output-column n-tiles, merged into the partial output
    {
      float al[2], w4[2], w16[2];
#pragma unroll
      for (int rs = 0; rs < 2; ++rs) {
        al[rs] = alpha_s[g + 8 * rs];
        w4[rs] = gq4_s[g + 8 * rs];
        w16[rs] = gq16_s[g + 8 * rs];
      }
      // P operand (rows g and g + 8): slot 2*tig+e of k-step ks holds key tig*BK/4 + 4*ks + e
      uint32_t pw[2][BK / 32];
      uint32_t psc[2][BK / 64];
      if (n4) {
#pragma unroll
        for (int rs = 0; rs < 2; ++rs) {
          const uint8_t* pc = PC + (g + 8 * rs) * (BK / 2) + tig * (BK / 8);
          if constexpr (BK == 64) {
            const uint2 v = *reinterpret_cast<const uint2*>(pc);
            pw[rs][0] = v.x; pw[rs][1] = v.y;
          } else {
            const uint4 v = *reinterpret_cast<const uint4*>(pc);
            pw[rs][0] = v.x; pw[rs][1] = v.y; pw[rs][2] = v.z; pw[rs][3] = v.w;
          }
#pragma unroll
          for (int i = 0; i < BK / 64; ++i) psc[rs][i] = e4m3_to_h2x(PS[(g + 8 * rs) * (BK / 16) + tig * (BK / 64) + i]);
        }
      }
#pragma unroll
      for (int t = 0; t < NT_PV; ++t) {
        const int nt = warp + 8 * t;
        const int n = nt * 8 + g;  // output column (d index) of this lane's B fragment
        float c4r[4] = {0.f, 0.f, 0.f, 0.f}, c16r[4] = {0.f, 0.f, 0.f, 0.f};
        if (n4) {
          const uint8_t* vc = st4 + L::OFF_V4C + n * (BK / 2) + tig * (BK / 8);
          uint32_t vw[BK / 32];
          if constexpr (BK == 64) {
            const uint2 v = *reinterpret_cast<const uint2*>(vc);
            vw[0] = v.x; vw[1] = v.y;
          } else {
            const uint4 v = *reinterpret_cast<const uint4*>(vc);
            vw[0] = v.x; vw[1] = v.y; vw[2] = v.z; vw[3] = v.w;
          }
          const int crow = vrow_in_blk + n;
          uint32_t vsc[BK / 64];
#pragma unroll
          for (int i = 0; i < BK / 64; ++i) {
            const int gg = tig * (BK / 64) + i;  // 16-key group within the block
            vsc[i] = e4m3_to_h2x(st4[L::OFF_V4S + (gg >> 2) * 512 + (crow & 31) * 16 + ((crow >> 5) & 3) * 4 + (gg & 3)]);
          }
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const int sh = (ks & 1) * 16;
            uint32_t a[4];
#pragma unroll
            for (int rs = 0; rs < 2; ++rs) {
              const uint32_t word = pw[rs][ks >> 1];
              a[rs] = hmul2(e2m1x2_to_h2((word >> sh) & 0xFFu), psc[rs][ks >> 2]);
              a[2 + rs] = hmul2(e2m1x2_to_h2((word >> (sh + 8)) & 0xFFu), psc[rs][ks >> 2]);
            }
            const uint32_t word = vw[ks >> 1];
            const uint32_t b0 = hmul2(e2m1x2_to_h2((word >> sh) & 0xFFu), vsc[ks >> 2]);
            const uint32_t b1 = hmul2(e2m1x2_to_h2((word >> (sh + 8)) & 0xFFu), vsc[ks >> 2]);
            mma16816(c4r, a, b0, b1);
          }
        }
        if (n16) {
          const __half* vr = reinterpret_cast<const __half*>(st16 + BK * D * 2);
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const int k0 = tig * (BK / 4) + 4 * ks;
            uint32_t a[4];
#pragma unroll
            for (int rs = 0; rs < 2; ++rs) {
              const uint2 pw16 = *reinterpret_cast<const uint2*>(P16 + (g + 8 * rs) * BK + k0);
              a[rs] = pw16.x;
              a[2 + rs] = pw16.y;
            }
            const __half2 b0h = __halves2half2(vr[(k0 + 0) * D + n], vr[(k0 + 1) * D + n]);
            const __half2 b1h = __halves2half2(vr[(k0 + 2) * D + n], vr[(k0 + 3) * D + n]);
            mma16816(c16r, a, *reinterpret_cast<const uint32_t*>(&b0h), *reinterpret_cast<const uint32_t*>(&b1h));
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int rs = e >> 1;
          o[t][e] = o[t][e] * al[rs] + w4[rs] * c4r[e] + w16[rs] * c16r[e];
        }
      }
    }
    // this warp is done with the stage (and with S, P of this block)
    __syncwarp();
    if (lane == 0) {
      if (n4) mbar_arrive(&empty4[s4]);
      if (n16) mbar_arrive(&empty16[s16]);
    }
    c4 += n4 ? 1 : 0;
    c16 += n16 ? 1 : 0;
  }

  // ---- partial results of this split
  if (ok) {
    float* po = p.part_o + ((int64_t)grp * p.n_split + split) * kRowsMax * D;
#pragma unroll
    for (int t = 0; t < NT_PV; ++t) {
      const int col = (warp + 8 * t) * 8 + 2 * tig;
#pragma unroll
      for (int rs = 0; rs < 2; ++rs) {
        const int r = g + 8 * rs;
        if (r < R) *reinterpret_cast<float2*>(po + r * D + col) = make_float2(o[t][2 * rs], o[t][2 * rs + 1]);
      }
    }
    if (lane == 0) {
      float* pml = p.part_ml + ((int64_t)grp * p.n_split + split) * kRowsMax * 2;
#pragma unroll
      for (int rs = 0; rs < 2; ++rs) {
        const int r = warp + 8 * rs;
        if (r < R) {
          pml[2 * r] = m_run[rs];
          pml[2 * r + 1] = l_run[rs];
        }
      }
    }
  }
}

// Combine the splits of every row: O = sum_s w_s O_s / sum_s w_s l_s with w_s = exp(m_s - m).
// One CTA per (batch, KV head); thread c handles output column c of every row.
__global__ void decode_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml,
                                      int n_split, int D, int R, int Hq, int Hkv, int Nq,
                                      __half* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ float wsh[];  // [n_split] weights of the current row
  __shared__ float s_m, s_l;
  const int grp = blockIdx.x;
  const int b = grp / Hkv, hk = grp % Hkv, G = Hq / Hkv;
  for (int r = 0; r < R; ++r) {
    const float* ml = part_ml + (int64_t)grp * n_split * kRowsMax * 2 + 2 * r;
    if (threadIdx.x == 0) {
      float m = kNegInf;
      for (int s = 0; s < n_split; ++s) m = fmaxf(m, ml[(int64_t)s * kRowsMax * 2]);
      float l = 0.0f;
      for (int s = 0; s < n_split; ++s) {
        const float ms = ml[(int64_t)s * kRowsMax * 2];
        const float w = (ms == kNegInf) ? 0.0f : expf(ms - m);
        wsh[s] = w;
        l += w * ml[(int64_t)s * kRowsMax * 2 + 1];
      }
      s_m = m;
      s_l = l;
    }
    __syncthreads();
    const int64_t orow = ((int64_t)b * Hq + (int64_t)hk * G + r / Nq) * Nq + r % Nq;
    const float inv = s_l > 0.0f ? 1.0f / s_l : 0.0f;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      float acc = 0.0f;
      for (int s = 0; s < n_split; ++s)
        acc += wsh[s] * part_o[(((int64_t)grp * n_split + s) * kRowsMax + r) * D + c];
      out[orow * D + c] = __float2half_rn(acc * inv);
    }
    if (threadIdx.x == 0 && lse) lse[orow] = s_l > 0.0f ? s_m + logf(s_l) : kNegInf;
    __syncthreads();
  }
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
  if (prm.mode != 2) {
    if (!make_u8_map(&tm, a.v4->codes, (uint64_t)prm.Nk / 2, (uint64_t)prm.B * prm.Hkv * D, BK / 2, D))
      return THRIFT_ERR_CUDA;
  } else {
    // no NVFP4 operand is read; the map only has to be valid
    if (!make_u8_map(&tm, a.part_o, 64, 1, 16, 1)) return THRIFT_ERR_CUDA;
  }
  auto kern = decode_attn_kernel<D, BK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  dim3 grid(prm.n_split, prm.B * prm.Hkv);
  kern<<<grid, kThreads, L::SMEM, stream>>>(tm, prm);
  if (cudaPeekAtLastError() != cudaSuccess) return THRIFT_ERR_CUDA;
  decode_combine_kernel<<<prm.B * prm.Hkv, D, prm.n_split * sizeof(float), stream>>>(
      prm.part_o, prm.part_ml, prm.n_split, D, prm.R, prm.Hq, prm.Hkv, prm.Nq, reinterpret_cast<__half*>(a.out),
      a.lse);
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
  return n < 1 ? 1 : (n > 4 ? 4 : n);
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
  if (a.mode != 2) {
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
  prm.nkb = c.Nk / c.block_k;
  prm.mask_words = (prm.nkb + 31) / 32;
  prm.causal = c.causal;
  prm.mode = a.mode;
  prm.tau = c.softmax_scale > 0.0f ? c.softmax_scale : 1.0f / sqrtf((float)c.d);
  prm.wait_limit = kWaitLimit;
  // splits: enough CTAs to fill every SM once, at least kMinBlocksPerSplit key blocks each
  const int groups = c.B * c.Hkv;
  const int resident = num_sms() * ctas_per_sm(c.d, c.block_k);
  int n_split = (resident + groups - 1) / groups;
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
