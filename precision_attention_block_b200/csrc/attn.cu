// Fused selective mixed-precision attention forward for sm_100a (ThriftAttention technical
// summary, "Gemengd-Precisie Berekening & Samenvoeging" and the paragraph on its fused kernel).
//
// One persistent CTA per SM walks (batch, query head, 128-row query tile) units.  For each unit
// the key blocks form a list of entries: first every key block that some row of the tile computes
// in NVFP4, then every key block it computes in FP16 (the order the pages' kernel uses; the FP16
// query tile is fetched only when the first FP16 entry comes up).  Warp roles:
//   warp 0      TMA producer: the unit's NVFP4 query tile, the FP16 query tile on demand, and for
//               every entry its K and V tiles (NVFP4 codes + scales, or FP16) into a slot ring.
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into one of two TMEM score buffers, then the
//               previous entry's PV into the TMEM PV buffer.  NVFP4 products use
//               tcgen05.mma.kind::mxf4nvf4.block_scale.block16 with the E4M3 scale vectors copied
//               into TMEM by tcgen05.cp; FP16 products use tcgen05.mma.kind::f16.
//   warps 2-5   one thread per query row: read S from TMEM, causal mask, the row maximum M of the
//               key block, P^ = exp(S - M); NVFP4 entries re-quantise P' = 2688 P^ with one E4M3
//               scale per 16 keys into shared memory (the PV MMA's A operand), FP16 entries round
//               P^ to FP16; then merge the previous entry's PV into the row's FP32 output with
//               weight exp(M - m) (m = running maximum), and sum the unquantised P^ into l.
// Every wait is bounded; on timeout the CTA records THRIFT_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <cuda_runtime.h>

#include "sm100.cuh"
#include "thrift_internal.h"

namespace thrift {

namespace {

constexpr int kThreads = 608;  // warp 0 producer, 1 QK^T issuer, 2 PV issuer, 3-18 softmax (four per TMEM lane quarter)
constexpr int kSoftmaxThreads = 512;
constexpr int kFirstSoftmaxWarp = 3;
constexpr int kBQ = 128;
constexpr long long kWaitLimit = 1ll << 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kSW128 = 2, kSW64 = 4, kSW32 = 6;

__host__ __device__ constexpr int round1024(int x) { return (x + 1023) & ~1023; }
__host__ __device__ constexpr int swz_for_row_bytes(int b) { return b == 128 ? kSW128 : (b == 64 ? kSW64 : kSW32); }

template <int D, int BK>
struct Layout {
  static constexpr int Q4_BYTES = kBQ * D / 2;
  static constexpr int QSF_BYTES = (D / 64) * 512;
  static constexpr int Q16_BYTES = kBQ * D * 2;
  static constexpr int SLOT_BYTES = BK * D * 2;
  static constexpr int NSLOT = BK == 128 ? 3 : 6;
  static constexpr int P16_BYTES = kBQ * BK * 2;
  static constexpr int P4_BYTES = kBQ * BK / 2;
  static constexpr int PSF_BYTES = (BK / 64) * 512;
  static constexpr int PBUF_BYTES = round1024(P16_BYTES > P4_BYTES + PSF_BYTES ? P16_BYTES : P4_BYTES + PSF_BYTES);
  static constexpr int OFF_Q4 = 0;
  static constexpr int OFF_QSF = Q4_BYTES;
  static constexpr int OFF_Q16 = round1024(OFF_QSF + QSF_BYTES);
  static constexpr int OFF_SLOTS = OFF_Q16 + Q16_BYTES;
  static constexpr int OFF_P = OFF_SLOTS + NSLOT * SLOT_BYTES;
  static constexpr int MAXE = 4096;  // entries per unit (two phases of at most 2048 key blocks)
  static constexpr int OFF_LIST = OFF_P + 2 * PBUF_BYTES;
  static constexpr int OFF_BAR = OFF_LIST + 2 * MAXE * 2;
  static constexpr int BYTES = OFF_BAR + 6144 + 1024;  // barriers + alignment slack
  // TMEM columns
  static constexpr int COL_S = 0;  // two buffers of BK columns
  static constexpr int COL_PV = 2 * BK;
  static constexpr int COL_SFQ = COL_PV + D;
  static constexpr int SFK_COLS = 4 * (D / 64);
  static constexpr int SFKV_COLS = 4 * (BK / 64);
  static constexpr int COL_SFK = COL_SFQ + SFK_COLS;        // two buffers
  static constexpr int COL_SFV = COL_SFK + 2 * SFK_COLS;    // two buffers
  static constexpr int COL_SFP = COL_SFV + 2 * SFKV_COLS;   // two buffers
  static constexpr int TMEM_COLS_USED = COL_SFP + 2 * SFKV_COLS;
  static_assert(TMEM_COLS_USED <= 512, "TMEM budget");
  static_assert(BYTES <= 232448, "shared memory budget");
};

struct Bars {
  uint64_t q_full, q_empty, q16_full, q16_empty;
  uint64_t s_full[2], s_free[2], p_full[2];
  uint64_t pv_full, pv_free;
  uint64_t kv_full[6], kv_empty[6];
  uint64_t list_full[2], list_empty[2];  // per-unit entry lists, double-buffered by unit parity
  int list_count[2];
  uint32_t tmem_base;
  int abort_flag;
  uint64_t pair[4];         // the four softmax warps of each TMEM lane quarter exchange values
  float xch[2][4][128];     // exchange buffers of the four warps of each lane quarter: [parity][warp][row]
};

static_assert(sizeof(Bars) <= 6144, "barrier block");

struct AttnParams {
  const uint32_t* mask;
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* v_sf;
  const float* q_ts;
  const float* k_ts;
  const float* v_ts;
  __half* out;
  float* lse;
  int* status;
  float* dbg;  // optional dump of one entry (S, P bytes, PV) of the first unit of CTA 0
  int dbg_entry;
  int B, Hq, Hkv, N, bq, causal, mode, nqb, nkb, mask_words, n_units;
  float tau;
  long long wait_limit;
};

// The entry list of one unit, regenerated identically by every role.
struct EntryIter {
  const uint32_t* m0;
  const uint32_t* m1;
  int jmax0, jmax1, jmax, two, mode, phase, j;

  __device__ __forceinline__ int sel(const uint32_t* m, int jj) const {
    if (mode == 2) return 1;
    if (mode == 1) return 0;
    return (int)((__ldg(m + (jj >> 5)) >> (jj & 31)) & 1u);
  }
  __device__ __forceinline__ bool next(int& j_out, int& f16_out, int& rm_out) {
    while (phase < 2) {
      while (j < jmax) {
        int jj = j++;
        int want = phase;
        int rm = 0;
        if (jj < jmax0 && sel(m0, jj) == want) rm |= 1;
        if (two && jj < jmax1 && sel(m1, jj) == want) rm |= 2;
        if (rm) {
          j_out = jj;
          f16_out = want;
          rm_out = two ? rm : 3;
          return true;
        }
      }
      ++phase;
      j = 0;
    }
    return false;
  }
};

struct UnitInfo {
  int b, h, hk, t;
};

__device__ __forceinline__ UnitInfo decode_unit(const AttnParams& p, int u) {
  int bh_count = p.B * p.Hq;
  int ntiles = p.N / kBQ;
  UnitInfo ui;
  ui.t = ntiles - 1 - u / bh_count;
  int bh = u % bh_count;
  ui.b = bh / p.Hq;
  ui.h = bh % p.Hq;
  ui.hk = ui.h / (p.Hq / p.Hkv);
  return ui;
}

template <int BK>
__device__ __forceinline__ EntryIter make_iter(const AttnParams& p, const UnitInfo& ui) {
  EntryIter it;
  it.mode = p.mode;
  it.two = p.bq == 64;
  int i0 = it.two ? 2 * ui.t : ui.t;
  int i1 = i0 + 1;
  const uint32_t* base = p.mask ? p.mask + ((int64_t)(ui.b * p.Hq + ui.h) * p.nqb) * p.mask_words : nullptr;
  it.m0 = base ? base + (int64_t)i0 * p.mask_words : nullptr;
  it.m1 = (base && it.two) ? base + (int64_t)i1 * p.mask_words : nullptr;
  if (p.causal) {
    it.jmax0 = ((i0 + 1) * p.bq - 1) / BK + 1;
    it.jmax1 = it.two ? ((i1 + 1) * p.bq - 1) / BK + 1 : 0;
  } else {
    it.jmax0 = p.nkb;
    it.jmax1 = it.two ? p.nkb : 0;
  }
  it.jmax = it.jmax0 > it.jmax1 ? it.jmax0 : it.jmax1;
  it.phase = 0;
  it.j = 0;
  return it;
}

// The unit's entry list, built once by a whole warp: NVFP4 entries, then FP16 entries, each as
// j | fp16 << 13 | row-half mask << 14.  Returns the number of entries (same in every lane).
template <int BK>
__device__ int build_list(const AttnParams& p, const UnitInfo& ui, uint16_t* list, int lane) {
  EntryIter it = make_iter<BK>(p, ui);
  int n = 0;
  for (int phase = 0; phase < 2; ++phase) {
    for (int jb = 0; jb < it.jmax; jb += 32) {
      const int jj = jb + lane;
      int rm = 0;
      if (jj < it.jmax0 && it.sel(it.m0, jj) == phase) rm |= 1;
      if (it.two && jj < it.jmax1 && it.sel(it.m1, jj) == phase) rm |= 2;
      if (!it.two && rm) rm = 3;
      const unsigned b = __ballot_sync(0xffffffffu, rm != 0);
      if (rm) list[n + __popc(b & ((1u << lane) - 1u))] = (uint16_t)(jj | (phase << 13) | (rm << 14));
      n += __popc(b);
    }
  }
  return n;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}


constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kRescale = 8.0f;  // log2 units: rescale O only when the block max grows past 256x

// Rows that do not take part in this block, and keys above the query (causal), become -inf.
template <int n>
__device__ __forceinline__ void mask_s(float (&s)[n], bool part, bool diag, int key0, int row) {
  if (!part) {
#pragma unroll
    for (int i = 0; i < n; ++i) s[i] = kNegInf;
  } else if (diag) {
#pragma unroll
    for (int i = 0; i < n; ++i) s[i] = (key0 + i > row) ? kNegInf : s[i];
  }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int n>
__device__ __forceinline__ void group_max(const float (&s)[n], float* gm) {
#pragma unroll
  for (int q = 0; q < n / 16; ++q) {
    const float* x = s + 16 * q;
    float a = max3(x[0], x[1], x[2]), b = max3(x[3], x[4], x[5]), c = max3(x[6], x[7], x[8]);
    float d = max3(x[9], x[10], x[11]), e = max3(x[12], x[13], x[14]);
    gm[q] = max3(max3(a, b, c), max3(d, e, x[15]), kNegInf);
  }
}

// N consecutive 32-bit TMEM columns of this thread's lane (N = 16 or 32).
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld32(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// FP16 probabilities of N keys: exp2(s * sl2 - Ms) rounded to FP16 pairs; returns their FP32 sum.
template <int N>
__device__ __forceinline__ float probs_fp16(const float (&s)[N], float sl2, float Ms, uint32_t (&hw)[N / 2]) {
  const float2 a2 = make_float2(sl2, sl2), b2 = make_float2(-Ms, -Ms);
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int i = 0; i < N; i += 2) {
    float2 x = __ffma2_rn(make_float2(s[i], s[i + 1]), a2, b2);
    float2 pr = make_float2(ex2(x.x), ex2(x.y));
    acc[(i >> 1) & 1] = __fadd2_rn(acc[(i >> 1) & 1], pr);
    hw[i >> 1] = pack_half2(pr.x, pr.y);
  }
  float2 t = __fadd2_rn(acc[0], acc[1]);
  return t.x + t.y;
}

// Eight FP32 values to eight E2M1 codes packed in one word (element 0 in the low nibble).
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* y) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return out;
}

// NVFP4 re-quantisation of NG 16-key groups of one row:
//   P^ = exp2(s*sl2 - Ms); per group s_b = E4M3(2688 max(P^) / 6); codes = E2M1(2688 P^ / s_b).
// 2688 / s_b is folded into the exponent, so each key costs one FMA and one exp2.  A group whose
// scale underflows to 0 gets all-zero codes (its values are below 2688 * 2^-10 / 6 / 448).
// Returns the FP32 sum of the unquantised P^; writes 2*NG code words and NG scale bytes (sfw).
template <int NG>
__device__ __forceinline__ float probs_nvfp4(const float (&s)[16 * NG], const float* gm, float sl2, float Ms,
                                             uint32_t (&cw)[2 * NG], uint32_t& sfw) {
  float sum = 0.0f;
  sfw = 0u;
  const float2 a2 = make_float2(sl2, sl2);
#pragma unroll
  for (int q = 0; q < NG; ++q) {
    const bool live = gm[q] != kNegInf;
    const float pmax = live ? 2688.0f * ex2(fmaf(gm[q], sl2, -Ms)) : 0.0f;
    const uint32_t sb = cvt_e4m3(pmax * (1.0f / 6.0f));
    const float sbf = e4m3_to_f32(sb);
    const float sbe = sbf > 0.0f ? sbf : 448.0f;
    const float bias = live ? (11.392317422778761f - __log2f(sbe)) - Ms : kNegInf;  // log2(2688 / s_b) - Ms
    const float2 b2 = make_float2(bias, bias);
    float y[16];
    float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < 16; t += 2) {
      float2 x = __ffma2_rn(make_float2(s[16 * q + t], s[16 * q + t + 1]), a2, b2);
      y[t] = ex2(x.x);
      y[t + 1] = ex2(x.y);
      if (t & 2)
        acc1 = __fadd2_rn(acc1, make_float2(y[t], y[t + 1]));
      else
        acc0 = __fadd2_rn(acc0, make_float2(y[t], y[t + 1]));
    }
    cw[2 * q] = cvt_e2m1x8(y);
    cw[2 * q + 1] = cvt_e2m1x8(y + 8);
    const float2 t2 = __fadd2_rn(acc0, acc1);
    sum = fmaf(t2.x + t2.y, sbe * (1.0f / 2688.0f), sum);
    sfw |= sb << (8 * q);
  }
  return sum;
}

template <int D, int BK, bool DBG>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q4, const __grid_constant__ CUtensorMap tm_k4,
                const __grid_constant__ CUtensorMap tm_v4, const __grid_constant__ CUtensorMap tm_q16,
                const __grid_constant__ CUtensorMap tm_k16, const __grid_constant__ CUtensorMap tm_v16,
                const __grid_constant__ AttnParams p) {
  using L = Layout<D, BK>;
  extern __shared__ uint8_t smem_raw[];
  uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023) & ~1023u) - raw_addr);
  uint8_t* sQ4 = smem + L::OFF_Q4;
  uint8_t* sQSF = smem + L::OFF_QSF;
  uint8_t* sQ16 = smem + L::OFF_Q16;
  uint8_t* sSlots = smem + L::OFF_SLOTS;
  uint8_t* sP = smem + L::OFF_P;
  Bars* bars = reinterpret_cast<Bars*>(smem + L::OFF_BAR);
  volatile int* abort_flag = &bars->abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->q16_full, 1);
    mbar_init(&bars->q16_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], kSoftmaxThreads);
      mbar_init(&bars->p_full[i], kSoftmaxThreads);
    }
    mbar_init(&bars->pv_full, 1);
    mbar_init(&bars->pv_free, kSoftmaxThreads);
    for (int i = 0; i < 4; ++i) mbar_init(&bars->pair[i], 128);
    for (int i = 0; i < L::NSLOT; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->list_full[i], 1);
      mbar_init(&bars->list_empty[i], 2 + kSoftmaxThreads);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const long long lim = p.wait_limit;

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    // The whole warp builds each unit's entry list; lane 0 then issues the unit's loads.
    uint16_t* lists = reinterpret_cast<uint16_t*>(smem + L::OFF_LIST);
    if (lane == 0) {
      if (p.mode != 2) {
        prefetch_tmap(&tm_q4);
        prefetch_tmap(&tm_k4);
        prefetch_tmap(&tm_v4);
      }
      if (p.mode != 1) {
        prefetch_tmap(&tm_q16);
        prefetch_tmap(&tm_k16);
        prefetch_tmap(&tm_v16);
      }
    }
    {
      uint32_t slot_ctr = 0, unit_ctr = 0, u16_ctr = 0;
      bool ok = true;
      // lane 0: every load of one unit (returns false after a timeout)
      auto issue_unit = [&](const UnitInfo& ui, const uint16_t* list, int n_entries) -> bool {
          const int qrow0 = (ui.b * p.Hq + ui.h) * p.N + ui.t * kBQ;
          const int kvh = ui.b * p.Hkv + ui.hk;
          if (!mbar_wait(&bars->q_empty, (unit_ctr & 1) ^ 1, abort_flag, p.status, lim)) return false;
          if (p.mode != 2) {
            mbar_arrive_expect_tx(&bars->q_full, L::Q4_BYTES + L::QSF_BYTES);
            tma_load_2d(sQ4, &tm_q4, &bars->q_full, 0, qrow0);
            bulk_load(sQSF, p.q_sf + (size_t)(qrow0 / 128) * L::QSF_BYTES, L::QSF_BYTES, &bars->q_full);
          } else {
            mbar_arrive(&bars->q_full);
          }
          bool q16_loaded = false;
          for (int e = 0; e < n_entries; ++e) {
            const uint32_t x = list[e];
            const int j = x & 0x1fff, f16 = (x >> 13) & 1;
            if (f16 && !q16_loaded) {
              if (!(ok = mbar_wait(&bars->q16_empty, (u16_ctr & 1) ^ 1, abort_flag, p.status, lim))) break;
              mbar_arrive_expect_tx(&bars->q16_full, L::Q16_BYTES);
  #pragma unroll
              for (int cb = 0; cb < D / 64; ++cb) tma_load_2d(sQ16 + cb * kBQ * 128, &tm_q16, &bars->q16_full, cb * 64, qrow0);
              q16_loaded = true;
            }
            const int krow0 = kvh * p.N + j * BK;
            // K tile
            {
              uint32_t s = slot_ctr % L::NSLOT, ph = (slot_ctr / L::NSLOT) & 1;
              ++slot_ctr;
              if (!(ok = mbar_wait(&bars->kv_empty[s], ph ^ 1, abort_flag, p.status, lim))) break;
              uint8_t* dst = sSlots + s * L::SLOT_BYTES;
              if (f16) {
                mbar_arrive_expect_tx(&bars->kv_full[s], BK * D * 2);
  #pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) tma_load_2d(dst + cb * BK * 128, &tm_k16, &bars->kv_full[s], cb * 64, krow0);
              } else {
                mbar_arrive_expect_tx(&bars->kv_full[s], BK * D / 2 + L::QSF_BYTES);
                tma_load_2d(dst, &tm_k4, &bars->kv_full[s], 0, krow0);
                bulk_load(dst + BK * D / 2, p.k_sf + (size_t)(krow0 / 128) * L::QSF_BYTES, L::QSF_BYTES, &bars->kv_full[s]);
              }
            }
            // V tile
            {
              uint32_t s = slot_ctr % L::NSLOT, ph = (slot_ctr / L::NSLOT) & 1;
              ++slot_ctr;
              if (!(ok = mbar_wait(&bars->kv_empty[s], ph ^ 1, abort_flag, p.status, lim))) break;
              uint8_t* dst = sSlots + s * L::SLOT_BYTES;
              if (f16) {
                mbar_arrive_expect_tx(&bars->kv_full[s], BK * D * 2);
  #pragma unroll
                for (int cb = 0; cb < D / 64; ++cb) tma_load_2d(dst + cb * BK * 128, &tm_v16, &bars->kv_full[s], cb * 64, krow0);
              } else {
                const int vrow0 = kvh * D;
                mbar_arrive_expect_tx(&bars->kv_full[s], D * BK / 2 + L::PSF_BYTES);
                tma_load_2d(dst, &tm_v4, &bars->kv_full[s], j * (BK / 2), vrow0);
                size_t sf_off = ((size_t)(vrow0 / 128) * (p.N / 64) + (size_t)j * (BK / 64)) * 512;
                bulk_load(dst + D * BK / 2, p.v_sf + sf_off, L::PSF_BYTES, &bars->kv_full[s]);
              }
            }
          }
          if (q16_loaded) ++u16_ctr;
          return ok;
      };
      for (int u = blockIdx.x; u < p.n_units; u += gridDim.x, ++unit_ctr) {
        UnitInfo ui = decode_unit(p, u);
        const uint32_t lb = unit_ctr & 1;
        uint16_t* list = lists + lb * L::MAXE;
        // the warp is converged here: every exit below is taken by all 32 lanes together
        const bool free_ok = mbar_wait(&bars->list_empty[lb], ((unit_ctr >> 1) & 1) ^ 1, abort_flag, p.status, lim);
        if (!__all_sync(0xffffffffu, free_ok)) break;
        const int n_entries = build_list<BK>(p, ui, list, lane);
        __syncwarp();
        if (lane == 0) {
          bars->list_count[lb] = n_entries;
          mbar_arrive(&bars->list_full[lb]);
          ok = issue_unit(ui, list, n_entries);
        }
        __syncwarp();
        if (!__shfl_sync(0xffffffffu, (int)ok, 0)) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ QK^T issuer
    if (lane == 0) {
      const uint32_t idesc_qk4 = idesc_nvf4(kBQ, BK);
      const uint32_t idesc_qk16 = idesc_f16(kBQ, BK, 0, 0);
      constexpr int SWQ = swz_for_row_bytes(D / 2);
      const uint32_t qb4 = smem_u32(sQ4), qb16 = smem_u32(sQ16);
      uint32_t slot_ctr = 0, unit_ctr = 0, u16_ctr = 0, g = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++unit_ctr) {
        UnitInfo ui = decode_unit(p, u);
        const int kvh = ui.b * p.Hkv + ui.hk;
        if (!(ok = mbar_wait(&bars->q_full, unit_ctr & 1, abort_flag, p.status, lim))) break;
        tc_fence_after();
        if (p.mode != 2) {
#pragma unroll
          for (int kk = 0; kk < D / 64; ++kk)
            tc_copy_sf(tmem + L::COL_SFQ + 4 * kk, make_sdesc(smem_u32(sQSF) + kk * 512, 16, 128, 0));
        }
        bool any16 = false;
        const uint32_t lb = unit_ctr & 1;
        const uint16_t* list = reinterpret_cast<const uint16_t*>(smem + L::OFF_LIST) + lb * L::MAXE;
        if (!(ok = mbar_wait(&bars->list_full[lb], (unit_ctr >> 1) & 1, abort_flag, p.status, lim))) break;
        const int n_entries = bars->list_count[lb];
        for (int e = 0; ok && e < n_entries; ++e) {
          const uint32_t x = list[e];
          const int j = x & 0x1fff, f16 = (x >> 13) & 1;
          const uint32_t kslot = slot_ctr % L::NSLOT, kph = (slot_ctr / L::NSLOT) & 1;
          slot_ctr += 2;  // this entry's V tile takes the next slot (the PV issuer consumes it)
          if (f16 && !any16) {
            if (!(ok = mbar_wait(&bars->q16_full, u16_ctr & 1, abort_flag, p.status, lim))) break;
            any16 = true;
          }
          const uint32_t buf = g & 1;
          if (!(ok = mbar_wait(&bars->kv_full[kslot], kph, abort_flag, p.status, lim))) break;
          if (!(ok = mbar_wait(&bars->s_free[buf], ((g >> 1) & 1) ^ 1, abort_flag, p.status, lim))) break;
          tc_fence_after();
          const uint32_t kbuf = smem_u32(sSlots + kslot * L::SLOT_BYTES);
          const uint32_t dS = tmem + L::COL_S + buf * BK;
          if (f16) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              uint64_t ad = make_sdesc(qb16 + (kk >> 2) * kBQ * 128 + (kk & 3) * 32, 16, 1024, kSW128);
              uint64_t bd = make_sdesc(kbuf + (kk >> 2) * BK * 128 + (kk & 3) * 32, 16, 1024, kSW128);
              mma_f16(dS, ad, bd, idesc_qk16, kk > 0);
            }
          } else {
            const int krow0 = kvh * p.N + j * BK;
            const int sfk_off = (krow0 & 127) >> 5;
            const uint32_t sfk = tmem + L::COL_SFK + buf * L::SFK_COLS;
#pragma unroll
            for (int kk = 0; kk < D / 64; ++kk)
              tc_copy_sf(sfk + 4 * kk, make_sdesc(kbuf + BK * D / 2 + kk * 512, 16, 128, 0));
#pragma unroll
            for (int kk = 0; kk < D / 64; ++kk) {
              uint64_t ad = make_sdesc(qb4 + kk * 32, 16, 8 * (D / 2), SWQ);
              uint64_t bd = make_sdesc(kbuf + kk * 32, 16, 8 * (D / 2), SWQ);
              mma_nvf4(dS, ad, bd, idesc_qk4, tmem + L::COL_SFQ + 4 * kk, sfk + 4 * kk + sfk_off, kk > 0);
            }
          }
          tc_commit(&bars->s_full[buf]);
          tc_commit(&bars->kv_empty[kslot]);
          ++g;
        }
        if (!ok) break;
        mbar_arrive(&bars->list_empty[lb]);
        tc_commit(&bars->q_empty);
        if (any16) {
          tc_commit(&bars->q16_empty);
          ++u16_ctr;
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------------ PV issuer
    if (lane == 0) {
      const uint32_t idesc_pv4 = idesc_nvf4(kBQ, D);
      const uint32_t idesc_pv16 = idesc_f16(kBQ, D, 0, 1);
      constexpr int SWP = swz_for_row_bytes(BK / 2);
      uint32_t slot_ctr = 0, unit_ctr = 0, g = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++unit_ctr) {
        UnitInfo ui = decode_unit(p, u);
        const int sfv_off = (((ui.b * p.Hkv + ui.hk) * D) & 127) >> 5;
        const uint32_t lb = unit_ctr & 1;
        const uint16_t* list = reinterpret_cast<const uint16_t*>(smem + L::OFF_LIST) + lb * L::MAXE;
        if (!(ok = mbar_wait(&bars->list_full[lb], (unit_ctr >> 1) & 1, abort_flag, p.status, lim))) break;
        const int n_entries = bars->list_count[lb];
        for (int e = 0; ok && e < n_entries; ++e) {
          const int f16 = (list[e] >> 13) & 1;
          const uint32_t vslot = (slot_ctr + 1) % L::NSLOT, vph = ((slot_ctr + 1) / L::NSLOT) & 1;
          slot_ctr += 2;
          const uint32_t buf = g & 1;
          if (!(ok = mbar_wait(&bars->p_full[buf], (g >> 1) & 1, abort_flag, p.status, lim))) break;
          if (!(ok = mbar_wait(&bars->pv_free, (g & 1) ^ 1, abort_flag, p.status, lim))) break;
          if (!(ok = mbar_wait(&bars->kv_full[vslot], vph, abort_flag, p.status, lim))) break;
          tc_fence_after();
          const uint32_t pbuf = smem_u32(sP + buf * L::PBUF_BYTES);
          const uint32_t vbuf = smem_u32(sSlots + vslot * L::SLOT_BYTES);
          if (f16) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              uint64_t ad = make_sdesc(pbuf + (kk >> 2) * kBQ * 128 + (kk & 3) * 32, 16, 1024, kSW128);
              uint64_t bd = make_sdesc(vbuf + kk * 16 * 128, BK * 128, 1024, kSW128);
              mma_f16(tmem + L::COL_PV, ad, bd, idesc_pv16, kk > 0);
            }
          } else {
            const uint32_t sfv = tmem + L::COL_SFV + buf * L::SFKV_COLS;
            const uint32_t sfp = tmem + L::COL_SFP + buf * L::SFKV_COLS;
#pragma unroll
            for (int kb = 0; kb < BK / 64; ++kb) {
              tc_copy_sf(sfv + 4 * kb, make_sdesc(vbuf + D * BK / 2 + kb * 512, 16, 128, 0));
              tc_copy_sf(sfp + 4 * kb, make_sdesc(pbuf + L::P4_BYTES + kb * 512, 16, 128, 0));
            }
#pragma unroll
            for (int kb = 0; kb < BK / 64; ++kb) {
              uint64_t ad = make_sdesc(pbuf + kb * 32, 16, 8 * (BK / 2), SWP);
              uint64_t bd = make_sdesc(vbuf + kb * 32, 16, 8 * (BK / 2), SWP);
              mma_nvf4(tmem + L::COL_PV, ad, bd, idesc_pv4, sfp + 4 * kb, sfv + 4 * kb + sfv_off, kb > 0);
            }
          }
          tc_commit(&bars->pv_full);
          tc_commit(&bars->kv_empty[vslot]);
          ++g;
        }
        if (!ok) break;
        mbar_arrive(&bars->list_empty[lb]);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax / merge
    // Four warps share each TMEM lane quarter (the same 32 query rows).  Warp `kq` of the quarter
    // reads keys [kq*BK/4, (kq+1)*BK/4) of the score row, the four swap their maxima to get the
    // row maximum M of the key block, and each produces its keys' probabilities and accumulates
    // output columns [kq*D/4, (kq+1)*D/4).
    const int quarter = warp & 3;
    const int kq = (warp - kFirstSoftmaxWarp) >> 2;
    const int rr = quarter * 32 + lane;  // row of the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    constexpr int DW = D / 4, KW = BK / 4;
    const float q_ts = (p.mode != 2) ? __ldg(p.q_ts) : 1.0f;
    const float k_ts = (p.mode != 2) ? __ldg(p.k_ts) : 1.0f;
    const float v_ts = (p.mode != 2) ? __ldg(p.v_ts) : 1.0f;
    const float sl2_4 = q_ts * k_ts * p.tau * kLog2e;
    const float sl2_16 = p.tau * kLog2e;
    const float pv4_scale = v_ts * (1.0f / 2688.0f);
    uint32_t g = 0, unit_ctr = 0, xk = 0;
    bool ok = true;
    // combine a value over the four warps of this lane quarter (max or sum; bounded wait)
    auto exchange = [&](float v, bool take_max) -> float {
      const uint32_t par = xk & 1;
      bars->xch[par][kq][rr] = v;
      mbar_arrive(&bars->pair[quarter]);
      const bool got = mbar_wait(&bars->pair[quarter], par, abort_flag, p.status, lim);
      ++xk;
      if (!got) {
        ok = false;
        return v;
      }
      const float a = bars->xch[par][0][rr], b = bars->xch[par][1][rr];
      const float c = bars->xch[par][2][rr], d = bars->xch[par][3][rr];
      return take_max ? max3(a, b, fmaxf(c, d)) : (a + b) + (c + d);
    };
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x, ++unit_ctr) {
      UnitInfo ui = decode_unit(p, u);
      const int row = ui.t * kBQ + rr;
      const int half = (p.bq == 64) ? (rr >> 6) : 0;
      float O[DW];
#pragma unroll
      for (int c = 0; c < DW; ++c) O[c] = 0.0f;
      // running state: O and l are relative to exp2(m_ref); m_ref moves only when a block's
      // maximum exceeds it by more than 2^kRescale (the final O / l does not depend on m_ref)
      float m_ref = kNegInf, l_run = 0.0f;
      float pend_M = kNegInf, pend_sum = 0.0f;
      int pend_f16 = 0;
      bool have_pend = false;
      const bool dbg_unit = DBG && p.dbg && blockIdx.x == 0 && u == (int)blockIdx.x;
      int local_e = 0;

      auto merge = [&](uint32_t ge) -> bool {
        if (!mbar_wait(&bars->pv_full, ge & 1, abort_flag, p.status, lim)) return false;
        tc_fence_after();
        const bool need = pend_M != kNegInf && (m_ref == kNegInf || pend_M > m_ref + kRescale);
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? (m_ref == kNegInf ? 0.0f : ex2(m_ref - pend_M)) : 1.0f;
          const float2 a2 = make_float2(alpha, alpha);
          l_run *= alpha;
#pragma unroll
          for (int c = 0; c < DW; c += 2) {
            float2 o = __fmul2_rn(make_float2(O[c], O[c + 1]), a2);
            O[c] = o.x;
            O[c + 1] = o.y;
          }
          if (need) m_ref = pend_M;
        }
        const float gs = (pend_M == kNegInf) ? 0.0f : ex2(pend_M - m_ref);
        l_run = fmaf(gs, pend_sum, l_run);
        const float gpv = pend_f16 ? gs : gs * pv4_scale;
        const float2 g2 = make_float2(gpv, gpv);
        uint32_t r[DW];
        tmem_ld<DW>(tmem + lane_base + L::COL_PV + kq * DW, r);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->pv_free);
#pragma unroll
        for (int i = 0; i < DW; i += 2) {
          float2 o = __ffma2_rn(g2, make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])),
                                make_float2(O[i], O[i + 1]));
          O[i] = o.x;
          O[i + 1] = o.y;
        }
        if constexpr (DBG) {
          if (dbg_unit && (local_e - 1) == p.dbg_entry)
            for (int i = 0; i < DW; ++i) p.dbg[kBQ * BK + kBQ * (BK / 2) + rr * D + kq * DW + i] = __uint_as_float(r[i]);
        }
        return true;
      };

      const uint32_t lb = unit_ctr & 1;
      const uint16_t* list = reinterpret_cast<const uint16_t*>(smem + L::OFF_LIST) + lb * L::MAXE;
      if (!(ok = mbar_wait(&bars->list_full[lb], (unit_ctr >> 1) & 1, abort_flag, p.status, lim))) break;
      const int n_entries = bars->list_count[lb];
      for (int e = 0; e < n_entries; ++e) {
        const uint32_t x = list[e];
        const int j = x & 0x1fff, f16 = (x >> 13) & 1, rm = x >> 14;
        const uint32_t buf = g & 1;
        if (!(ok = mbar_wait(&bars->s_full[buf], (g >> 1) & 1, abort_flag, p.status, lim))) break;
        tc_fence_after();
        const bool part = (rm >> half) & 1;
        const bool diag = p.causal && (j * BK + BK - 1 > ui.t * kBQ);
        const int key0 = j * BK + kq * KW;  // first key of this warp's columns
        const float sl2 = f16 ? sl2_16 : sl2_4;
        const bool dumpP = dbg_unit && local_e == p.dbg_entry;
        const uint32_t pb = smem_u32(sP + buf * L::PBUF_BYTES);

        // this warp's KW scores of the row: one TMEM round trip, then the buffer goes back
        float sv[KW];
        tmem_ld<KW>(tmem + lane_base + L::COL_S + buf * BK + kq * KW, *reinterpret_cast<uint32_t(*)[KW]>(sv));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->s_free[buf]);
        if constexpr (DBG) {
          if (dumpP)
            for (int i = 0; i < KW; ++i) p.dbg[rr * BK + kq * KW + i] = sv[i];
        }
        mask_s(sv, part, diag, key0, row);
        float gmax[KW / 16];
        group_max<KW>(sv, gmax);
        float Mh = gmax[0];
#pragma unroll
        for (int q = 1; q < KW / 16; ++q) Mh = fmaxf(Mh, gmax[q]);
        const float M = exchange(Mh, true);  // the block maximum over the four warps
        if (!ok) break;
        const bool valid = M != kNegInf;     // false when every key of the block is masked for this row
        const float Ms = valid ? M * sl2 : 0.0f;

        // this warp's probabilities, their partial sum, and its part of the PV operand
        float sum;
        if (f16) {
          uint32_t hw[KW / 2];
          sum = probs_fp16<KW>(sv, sl2, Ms, hw);
          if constexpr (DBG) {
            if (dumpP)
              for (int i = 0; i < KW / 2; ++i) reinterpret_cast<uint32_t*>(p.dbg + kBQ * BK + rr * (BK / 2))[kq * (KW / 2) + i] = hw[i];
          }
#pragma unroll
          for (int q = 0; q < KW / 8; ++q) {
            const int chunk = kq * (KW / 8) + q;  // 16-byte chunk of the row (8 keys)
            const int cb = chunk >> 3, c8 = chunk & 7;
            st_shared_v4(pb + cb * kBQ * 128 + rr * 128 + ((c8 ^ (rr & 7)) << 4), hw[4 * q], hw[4 * q + 1],
                         hw[4 * q + 2], hw[4 * q + 3]);
          }
        } else {
          uint32_t cw[KW / 8], sfw = 0u;
          sum = probs_nvfp4<KW / 16>(sv, gmax, sl2, Ms, cw, sfw);
          if constexpr (DBG) {
            if (dumpP) {
              uint8_t* db = reinterpret_cast<uint8_t*>(p.dbg + kBQ * BK + rr * (BK / 2));
              for (int i = 0; i < KW / 8; ++i) reinterpret_cast<uint32_t*>(db + kq * (KW / 2))[i] = cw[i];
              for (int q = 0; q < KW / 16; ++q) db[BK / 2 + kq * (KW / 16) + q] = (uint8_t)(sfw >> (8 * q));
            }
          }
          if constexpr (BK == 64) {
            // 8 code bytes: half of the row's 16-byte chunk kq/2
            const uint32_t addr = pb + rr * 32 + (((kq >> 1) ^ ((rr >> 2) & 1)) << 4) + 8 * (kq & 1);
            asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(cw[0]), "r"(cw[1]) : "memory");
            const uint32_t sfa = pb + L::P4_BYTES + (rr & 31) * 16 + (rr >> 5) * 4 + kq;
            asm volatile("st.shared.b8 [%0], %1;" ::"r"(sfa), "r"(sfw) : "memory");
          } else {
            const uint32_t addr = pb + rr * 64 + ((kq ^ ((rr >> 1) & 3)) << 4);
            st_shared_v4(addr, cw[0], cw[1], cw[2], cw[3]);
            const uint32_t sfa = pb + L::P4_BYTES + (kq >> 1) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + 2 * (kq & 1);
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(sfa), "h"((uint16_t)sfw) : "memory");
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars->p_full[buf]);
        if (have_pend && !(ok = merge(g - 1))) break;
        pend_M = valid ? Ms : kNegInf;
        pend_sum = sum;
        pend_f16 = f16;
        have_pend = true;
        ++g;
        ++local_e;
      }
      if (ok && have_pend) ok = merge(g - 1);
      if (!ok) break;
      mbar_arrive(&bars->list_empty[lb]);
      // combine the four warps' partial denominators
      const float l_tot = exchange(l_run, false);
      if (!ok) break;
      // epilogue: O / l in FP16, lse in natural-log units of the tau-scaled scores
      const float inv_l = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
      const int64_t orow = (int64_t)(ui.b * p.Hq + ui.h) * p.N + row;
      uint4* dst = reinterpret_cast<uint4*>(p.out + orow * D + kq * DW);
#pragma unroll
      for (int c = 0; c < DW / 8; ++c) {
        uint4 v;
        v.x = pack_half2(O[8 * c] * inv_l, O[8 * c + 1] * inv_l);
        v.y = pack_half2(O[8 * c + 2] * inv_l, O[8 * c + 3] * inv_l);
        v.z = pack_half2(O[8 * c + 4] * inv_l, O[8 * c + 5] * inv_l);
        v.w = pack_half2(O[8 * c + 6] * inv_l, O[8 * c + 7] * inv_l);
        dst[c] = v;
      }
      if (p.lse && kq == 0) p.lse[orow] = (m_ref + __log2f(l_tot)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2D map over a row-major [rows, inner] array (inner contiguous).
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t inner, uint64_t rows,
              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * (uint64_t)esize};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle swz_enum(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

template <int D, int BK>
thrift_status launch_t(const void* q, const void* k, const void* v, const thrift_nvfp4* q4, const thrift_nvfp4* k4,
                       const thrift_nvfp4* v4, AttnParams& prm, cudaStream_t stream) {
  using L = Layout<D, BK>;
  CUtensorMap maps[6];
  memset(maps, 0, sizeof(maps));
  const uint64_t qrows = (uint64_t)prm.B * prm.Hq * prm.N, krows = (uint64_t)prm.B * prm.Hkv * prm.N;
  bool ok = true;
  if (prm.mode != 2) {
    ok &= make_map(&maps[0], q4->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D / 2, qrows, D / 2, kBQ, swz_enum(D / 2));
    ok &= make_map(&maps[1], k4->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D / 2, krows, D / 2, BK, swz_enum(D / 2));
    ok &= make_map(&maps[2], v4->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)prm.N / 2,
                   (uint64_t)prm.B * prm.Hkv * D, BK / 2, D, swz_enum(BK / 2));
  }
  if (prm.mode != 1) {
    ok &= make_map(&maps[3], q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, qrows, 64, kBQ, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&maps[4], k, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, krows, 64, BK, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map(&maps[5], v, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, D, krows, 64, BK, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!ok) return THRIFT_ERR_CUDA;
  auto kern = prm.dbg ? attn_kernel<D, BK, true> : attn_kernel<D, BK, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::BYTES) != cudaSuccess)
    return THRIFT_ERR_CUDA;
  int grid = num_sms();
  if (grid > prm.n_units) grid = prm.n_units;
  kern<<<grid, kThreads, L::BYTES, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], prm);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

__global__ void wait_timeout_kernel(int* status, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must give up and record the timeout.
  mbar_wait(&bar, 0, &abort_flag, threadIdx.x == 0 ? status : nullptr, limit);
}

}  // namespace

thrift_status attn_launch_dbg(const void* q, const void* k, const void* v, const thrift_nvfp4* q4,
                              const thrift_nvfp4* k4, const thrift_nvfp4* v4, const uint32_t* mask, int mode,
                              void* out, float* lse, const thrift_cfg& c, int* status, float* dbg, int dbg_entry,
                              cudaStream_t stream) {
  AttnParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.mask = mask;
  if (mode != 2) {
    prm.q_sf = q4->scales_mma;
    prm.k_sf = k4->scales_mma;
    prm.v_sf = v4->scales_mma;
    prm.q_ts = q4->tensor_scale;
    prm.k_ts = k4->tensor_scale;
    prm.v_ts = v4->tensor_scale;
  }
  prm.out = reinterpret_cast<__half*>(out);
  prm.lse = lse;
  prm.status = status;
  prm.dbg = dbg;
  prm.dbg_entry = dbg_entry;
  prm.B = c.B;
  prm.Hq = c.Hq;
  prm.Hkv = c.Hkv;
  prm.N = c.N;
  prm.bq = c.block_q;
  prm.causal = c.causal;
  prm.mode = mode;
  prm.nqb = c.N / c.block_q;
  prm.nkb = c.N / c.block_k;
  prm.mask_words = (prm.nkb + 31) / 32;
  prm.n_units = c.B * c.Hq * (c.N / kBQ);
  prm.tau = c.softmax_scale > 0.0f ? c.softmax_scale : 1.0f / sqrtf((float)c.d);
  if (2 * prm.nkb > 4096) return THRIFT_ERR_UNSUPPORTED;  // the per-unit entry list holds 4096 entries
  prm.wait_limit = kWaitLimit;
  if (c.d == 128 && c.block_k == 64) return launch_t<128, 64>(q, k, v, q4, k4, v4, prm, stream);
  if (c.d == 128 && c.block_k == 128) return launch_t<128, 128>(q, k, v, q4, k4, v4, prm, stream);
  if (c.d == 64 && c.block_k == 64) return launch_t<64, 64>(q, k, v, q4, k4, v4, prm, stream);
  if (c.d == 64 && c.block_k == 128) return launch_t<64, 128>(q, k, v, q4, k4, v4, prm, stream);
  return THRIFT_ERR_UNSUPPORTED;
}

thrift_status attn_launch(const void* q, const void* k, const void* v, const thrift_nvfp4* q4, const thrift_nvfp4* k4,
                          const thrift_nvfp4* v4, const uint32_t* mask, int mode, void* out, float* lse,
                          const thrift_cfg& c, int* status, cudaStream_t stream) {
  return attn_launch_dbg(q, k, v, q4, k4, v4, mask, mode, out, lse, c, status, nullptr, -1, stream);
}

thrift_status wait_timeout_launch(int* status, long long limit, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status, limit);
  return cudaPeekAtLastError() == cudaSuccess ? THRIFT_OK : THRIFT_ERR_CUDA;
}

}  // namespace thrift
